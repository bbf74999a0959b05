"""The GPU parity comparisons fail on a wrong answer (no GPU needed).

The attention comparisons of the GPU tests go through helpers.assert_attn_close.  Here the
same helper is fed the oracle's outputs for inputs the GPU tests draw on the CPU, with an
all-zero and a perturbed stand-in for the device output: both must be rejected, while the
oracle's output itself (and one rounded to bf16) passes.  For the e4m3 and cluster-order
cases, whose tests also demand a reference output above 10x the absolute bound, the guard
is checked to hold on the very inputs those tests use.  The forward's whole check (outputs,
empty rows, log-sum-exp) is also fed the oracle's answers to wrong computations that a
kernel bug would produce -- a skipped kv block, a missing or doubled log2(e) factor, K or V
of the neighbouring block, unmasked pad keys, rows stored one slot off -- and must reject
every one.
"""
import math

import numpy as np
import pytest
import torch

import helpers as Hp
from block_sparse_attention_25_b200 import synth
from oracle import bsa_oracle as O

WLS = Hp.small_workloads()


def _rejects(got, ref, **kw):
    with pytest.raises(AssertionError):
        Hp.assert_attn_close(got, ref, **kw)


def _bf16(x):
    return torch.from_numpy(x).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("wl", WLS[:2], ids=[w.name for w in WLS[:2]])
@pytest.mark.parametrize("sharp", [1.0, 6.0])
def test_bf16_compare_rejects_zero_and_perturbed_outputs(wl, sharp):
    g = Hp.grid_of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=sharp)
    mass = O.block_mass(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g), g, wl.q_block, 64,
                        Hp.scale_of(wl))
    rp, ci = Hp.csr_from_oracle(mass, 0.9)
    ref, _ = O.masked_attention(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g),
                                Hp.oracle_tiled(v, g), g, wl.q_block, 64, rp, ci, Hp.scale_of(wl))
    Hp.assert_attn_close(_bf16(ref), ref, signal_guard=False)
    _rejects(np.zeros_like(ref), ref, signal_guard=False)
    _rejects(ref * 1.05, ref, signal_guard=False)       # a 5% scale error
    bad = ref.copy()
    bad[0, 0, 5] = -bad[0, 0, 5] + 0.5 * np.abs(ref).max()   # one wrong row
    _rejects(bad, ref, signal_guard=False)


def test_fp8_cases_clear_the_signal_guard_and_reject_zero():
    import test_gpu_parity as TP
    for wl in TP.FP8_WLS:
        g = Hp.grid_of(wl)
        for sharp in (6.0, 8.0):
            q, k, v = TP._fp8_draw(wl, sharp)
            deq = [O.dequant_e4m3_tiles(*O.quant_e4m3_tiles(O.permute_forward(x.float().numpy(), g)))
                   for x in (q, k, v)]
            n_qb, n_kb = wl.Np // wl.q_block, wl.Np // 64
            rp, ci = synth.draw_keep_csr(wl.batch * wl.heads * n_qb, n_kb, 0.5,
                                         seed=wl.seed + 200, empty_rows=(1,))
            ref, _ = O.masked_attention(deq[0], deq[1], deq[2], g, wl.q_block, 64, rp.numpy(),
                                        ci.numpy(), Hp.scale_of(wl))
            assert np.abs(ref).max() >= Hp.SIGNAL_FACTOR * Hp.FP8_MAX_ABS
            Hp.assert_attn_close(ref, ref, fp8=True)
            _rejects(np.zeros_like(ref), ref, fp8=True)
            _rejects(ref * 1.1, ref, fp8=True)


def test_cluster_cases_clear_the_signal_guard():
    import test_gpu_clusters as TC

    class _B:                                  # the case builder only needs the shape type
        @staticmethod
        def ClusterShape(*a):
            return a

    for D in (64, 128):
        for keep, sharp, vs in ((1.0, 1.0, 1.5), (0.3, 3.0, 0.25), (0.05, 3.0, 0.25)):
            _, q, k, v, qs, qn, ks, kn, rp, ci = TC._cluster_case(_B, 2, 2, 1500, D, 9, 23, 40 + D,
                                                                   keep, sharp, vs)
            for b in range(2):
                for h in range(2):          # each (batch, head) is compared on its own
                    r0 = (b * 2 + h) * 9
                    rows = rp[r0:r0 + 10].numpy() - rp[r0].numpy()
                    cols = ci[rp[r0]:rp[r0 + 9]].numpy()
                    ref = O.cluster_attention(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                              v[b, h].double().numpy(), qs[b, h].numpy(),
                                              qn[b, h].numpy(), ks[b, h].numpy(), kn[b, h].numpy(),
                                              rows, cols, 1.0 / math.sqrt(D))
                    assert np.abs(ref).max() >= Hp.SIGNAL_FACTOR * Hp.ATTN_MAX_ABS, (D, keep, b, h)
                    _rejects(np.zeros_like(ref), ref)


# ------------------------------------------------------------------ plausible kernel bugs
def _drop_one_block(rp, ci, which):
    """CSR with the first (which=0) or last (which=-1) kept block of every row removed,
    as a loop bound off by one would leave it."""
    rows, out_rp = [], [0]
    for r in range(len(rp) - 1):
        blocks = list(ci[rp[r]:rp[r + 1]])
        if blocks:
            del blocks[which]
        rows += blocks
        out_rp.append(len(rows))
    return np.array(out_rp, np.int64), np.array(rows, np.int64)


def _attend_with_pad_keys(qt, kt, vt, g, q_block, rp, ci, scale):
    """Attention whose kept blocks also admit their pad slots as keys (zero K and V), as a
    kernel that forgot the key mask would compute it; pad query rows stay empty."""
    B, Hh, Np, D = qt.shape
    valid = O.valid_slots(g)
    n_qb = Np // q_block
    o = np.zeros((B, Hh, Np, D))
    lse = np.full((B, Hh, Np), -math.inf)
    for b in range(B):
        for h in range(Hh):
            for p in np.flatnonzero(valid):
                r = (b * Hh + h) * n_qb + p // q_block
                blocks = ci[rp[r]:rp[r + 1]]
                if blocks.size == 0:
                    continue
                keys = (blocks[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
                lg = scale * (kt[b, h, keys] @ qt[b, h, p])
                mx = lg.max()
                e = np.exp(lg - mx)
                o[b, h, p] = (e / e.sum()) @ vt[b, h, keys]
                lse[b, h, p] = mx + math.log(e.sum())
    return o, lse


@pytest.mark.parametrize("wl", WLS[:2], ids=[w.name for w in WLS[:2]])
@pytest.mark.parametrize("sharp", [1.0, 6.0])
def test_fwd_check_rejects_plausible_kernel_mistakes(wl, sharp):
    """The GPU forward tests' whole check (helpers.assert_fwd_close) is fed the oracle's
    answer to a wrong computation -- what a kernel with that bug would return -- and must
    reject each one, while the right answer rounded to bf16 passes."""
    g = Hp.grid_of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=sharp)
    qt, kt, vt = (Hp.oracle_tiled(x, g) for x in (q, k, v))
    scale = Hp.scale_of(wl)
    mass = O.block_mass(qt, kt, g, wl.q_block, 64, scale)
    rp, ci = Hp.csr_from_oracle(mass, 0.9)
    o_ref, lse_ref = O.masked_attention(qt, kt, vt, g, wl.q_block, 64, rp, ci, scale)
    Hp.assert_fwd_close(_bf16(o_ref), lse_ref, o_ref, lse_ref)

    def attend(qx=qt, kx=kt, vx=vt, r=rp, c=ci, s=scale):
        return O.masked_attention(qx, kx, vx, g, wl.q_block, 64, r, c, s)

    roll = lambda x: np.roll(x, -64, axis=2)          # noqa: E731  block j reads block j+1
    rp_last, ci_last = _drop_one_block(rp, ci, -1)
    rp_first, ci_first = _drop_one_block(rp, ci, 0)
    mistakes = {
        "last kept block skipped": attend(r=rp_last, c=ci_last),
        "first kept block skipped": attend(r=rp_first, c=ci_first),
        "exp2 without the log2(e) factor": attend(s=scale * math.log(2.0)),
        "log2(e) applied twice": attend(s=scale / math.log(2.0)),
        "K of the next kv block": attend(kx=roll(kt)),
        "V of the next kv block": attend(vx=roll(vt)),
        "pad keys not masked": _attend_with_pad_keys(qt, kt, vt, g, wl.q_block, rp, ci, scale),
    }
    for name, (o_bad, lse_bad) in mistakes.items():
        with pytest.raises(AssertionError):
            Hp.assert_fwd_close(o_bad, lse_bad, o_ref, lse_ref)
            raise RuntimeError(name)  # not reached when the check rejects
    # output rows stored one slot off inside each query block
    o_bad, lse_bad = o_ref.copy(), lse_ref.copy()
    o_bad[:, :, 1:] = o_ref[:, :, :-1]
    lse_bad[:, :, 1:] = lse_ref[:, :, :-1]
    with pytest.raises(AssertionError):
        Hp.assert_fwd_close(o_bad, lse_bad, o_ref, lse_ref)


def _mass_with_pad_keys(qt, kt, g, q_block, scale):
    """Block masses whose softmax also admits the pad slots as keys (zero K), as a kernel
    that forgot the key mask would compute them."""
    B, Hh, Np, _ = qt.shape
    valid = O.valid_slots(g)
    n_qb, n_kb = Np // q_block, Np // 64
    out = np.zeros((B, Hh, n_qb, n_kb))
    for b in range(B):
        for h in range(Hh):
            for i in range(n_qb):
                rows = np.arange(i * q_block, (i + 1) * q_block)
                rows = rows[valid[rows]]
                if rows.size == 0:
                    continue
                lg = scale * (qt[b, h, rows] @ kt[b, h].T)
                p = np.exp(lg - lg.max(axis=1, keepdims=True))
                p /= p.sum(axis=1, keepdims=True)
                out[b, h, i] = p.sum(axis=0).reshape(n_kb, 64).sum(axis=1) / rows.size
    return out


@pytest.mark.parametrize("wl", WLS[:2], ids=[w.name for w in WLS[:2]])
@pytest.mark.parametrize("sharp", [1.0, 6.0])
def test_mass_check_rejects_plausible_kernel_mistakes(wl, sharp):
    """The block-mass check of the GPU tests (helpers.assert_mass_close) rejects the masses
    a kernel bug would produce, and accepts the right masses rounded to float32."""
    g = Hp.grid_of(wl)
    q, k, _ = Hp.draw(wl, value_scale=1.0, sharp=sharp)
    qt, kt = Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g)
    scale = Hp.scale_of(wl)
    ref = O.block_mass(qt, kt, g, wl.q_block, 64, scale)
    Hp.assert_mass_close(ref.astype(np.float32).astype(np.float64), ref)
    valid = O.valid_slots(g).reshape(-1, wl.q_block)
    share = (valid.sum(axis=1) / wl.q_block)[None, None, :, None]
    mistakes = {
        "exp2 without the log2(e) factor": O.block_mass(qt, kt, g, wl.q_block, 64,
                                                        scale * math.log(2.0)),
        "mass put in the next kv block": np.roll(ref, 1, axis=-1),
        "mean over every row of the block, pads included": ref * share,
        "pad keys not masked": _mass_with_pad_keys(qt, kt, g, wl.q_block, scale),
        "rows of the neighbouring head": np.roll(ref, 1, axis=1),
        "row of the next query block": np.roll(ref, -1, axis=2),
    }
    for name, bad in mistakes.items():
        with pytest.raises(AssertionError):
            Hp.assert_mass_close(bad, ref)
            raise RuntimeError(name)  # not reached when the check rejects
