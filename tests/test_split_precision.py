"""The precision argument behind the pooled estimate's and the k-means assignment's use of
bf16 tensor cores for fp32 operands, checked on the CPU.

An fp32 value x is cut into three bf16 parts: hi = bf16(x), mid = bf16(x - hi),
lo = bf16(x - hi - mid), each conversion rounding to nearest even (as __float2bfloat16_rn
does).  The parts sum to x within about 2^-24 |x|.  A dot product of two split vectors
keeps the six cross terms hi.hi + hi.mid + mid.hi + hi.lo + lo.hi + mid.mid; the three it
drops (mid.lo, lo.mid, lo.lo) are below 2^-24 of |q||k| per element.  With fp32
accumulation the logits stay within a few 2^-24 of sum |q_d k_d| of the fp64 dot product,
well inside what the pooled tests need (masses to 1e-5).
"""
import numpy as np
import torch


def _split3(x32: torch.Tensor):
    hi = x32.to(torch.bfloat16).float()
    r1 = x32 - hi                                   # exact: hi holds x's leading 8 bits
    mid = r1.to(torch.bfloat16).float()
    lo = (r1 - mid).to(torch.bfloat16).float()
    return hi, mid, lo


def test_three_bf16_parts_reconstruct_fp32():
    g = torch.Generator().manual_seed(3)
    x = torch.randn(200_000, generator=g, dtype=torch.float32) * \
        torch.exp2(torch.randint(-20, 20, (200_000,), generator=g).float())
    hi, mid, lo = _split3(x)
    back = hi.double() + mid.double() + lo.double()
    rel = ((back - x.double()).abs() / x.double().abs().clamp_min(1e-300)).max().item()
    assert rel <= 2.0 ** -24
    # the first residual is exact in fp32 (hi holds the leading bits of x)
    assert torch.equal((x - hi).double(), x.double() - hi.double())


def test_six_products_give_fp32_accurate_logits():
    g = torch.Generator().manual_seed(4)
    for D in (64, 128):
        q = torch.randn(512, D, generator=g) * 0.3
        k = torch.randn(640, D, generator=g) * 0.3
        qh, qm, ql = _split3(q)
        kh, km, kl = _split3(k)
        # six bf16 products, fp32 accumulation in the order of the K = 6D segments
        six = (qh @ kh.T) + (qh @ km.T) + (qm @ kh.T) + (qh @ kl.T) + (ql @ kh.T) + (qm @ km.T)
        exact = q.double() @ k.double().T
        bound = (q.double().abs() @ k.double().abs().T) * (D + 8) * 2.0 ** -24
        assert torch.all((six.double() - exact).abs() <= bound)
        # one bf16 product alone is far coarser: the split is what buys the precision
        one = qh @ kh.T
        assert ((one.double() - exact).abs() > bound).any()


def test_split_of_the_mean_keeps_the_estimate_within_the_pooled_tolerance():
    """A softmax over kv blocks of logits carrying the six-product error moves masses by
    far less than the pooled tests' 1e-5 absolute bound."""
    rng = np.random.default_rng(5)
    D, n_kb = 128, 1440
    q = torch.from_numpy(rng.standard_normal((64, D)).astype(np.float32)) * 0.5
    k = torch.from_numpy(rng.standard_normal((n_kb, D)).astype(np.float32)) * 0.5
    qh, qm, ql = _split3(q)
    kh, km, kl = _split3(k)
    six = (qh @ kh.T) + (qh @ km.T) + (qm @ kh.T) + (qh @ kl.T) + (ql @ kh.T) + (qm @ km.T)
    scale = 1.0 / np.sqrt(D)
    m_six = torch.softmax(six.double() * scale, dim=-1)
    m_ref = torch.softmax((q.double() @ k.double().T) * scale, dim=-1)
    assert (m_six - m_ref).abs().max().item() < 1e-7
