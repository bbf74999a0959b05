"""GPU parity at the full workload sizes, in the launch configuration the bench times.

The oracle cannot compute these sizes in full, so it checks sampled outputs one by one:
permuted slots, block-mass rows of sampled (head, query block) pairs and attention rows of
sampled query slots.  The selection is checked on every row through properties that fix
it uniquely at any size (reaches the target; minimal; keeps the largest masses; ties to
the lower index).  Inputs are seeded draws on the GPU; the CSR fed to the oracle is a
seeded synthetic one (no oracle input comes from the CUDA path).
"""
import math

import numpy as np
import pytest
import torch

import helpers as Hp
from block_sparse_attention_25_b200 import synth
from oracle import bsa_oracle as O

pytestmark = pytest.mark.gpu

FULL = ["wan13b_480p", "wan14b_720p", "hunyuan_720p"]


@pytest.fixture(scope="module")
def B(cuda_device):
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    return b


@pytest.fixture(scope="module", params=FULL)
def full(request, B):
    wl = synth.WORKLOADS[request.param]
    s = B.Shape.of(wl)
    q, k, v = synth.draw_qkv(wl, device="cuda")
    qt, kt, vt = (B.tile_permute(x, s) for x in (q, k, v))
    torch.cuda.synchronize()
    yield wl, s, (q, k, v), (qt, kt, vt)
    del q, k, v, qt, kt, vt
    torch.cuda.empty_cache()


def test_permute_full_size(B, full):
    wl, s, (q, k, v), (qt, kt, vt) = full
    g = Hp.grid_of(wl)
    src = O.tile_slot_source(g)
    rng = np.random.default_rng(0)
    slots = rng.integers(0, s.Np, 4096)
    heads = rng.integers(0, s.heads, 4096)
    got = qt[0, torch.as_tensor(heads), torch.as_tensor(slots)].cpu().view(torch.int16)
    pad = src[slots] < 0
    assert torch.all(got[torch.as_tensor(pad)] == 0)
    ok = ~pad
    ref = q[0, torch.as_tensor(src[slots][ok]), torch.as_tensor(heads[ok])].cpu().view(torch.int16)
    assert torch.equal(got[torch.as_tensor(ok)], ref)
    back = B.tile_permute(vt, s, inverse=True)
    assert torch.equal(back.view(torch.int16), v.view(torch.int16))


def _selection_properties(mass_rows_np, rp, ci, tau, n_kb):
    """Vectorised check that each CSR row is the unique (q desc, index asc) minimal set."""
    R = mass_rows_np.shape[0]
    q = np.rint(mass_rows_np.astype(np.float64) * 2.0 ** 40).astype(np.int64)
    total = q.sum(axis=1)
    target = np.ceil(np.float64(np.float32(tau)) * total.astype(np.float64)).astype(np.int64)
    kept = np.zeros((R, n_kb), dtype=bool)
    lens = np.diff(rp)
    rows = np.repeat(np.arange(R), lens)
    kept[rows, ci[:rp[-1]]] = True
    assert np.array_equal(kept.sum(axis=1), lens), "duplicate or unsorted indices"
    ksum = np.where(kept, q, 0).sum(axis=1)
    assert np.all(ksum >= target)
    big = np.iinfo(np.int64).max
    kmin = np.where(kept, q, big).min(axis=1)
    has = lens > 0
    assert np.all(ksum[has] - kmin[has] < target[has])                # minimal
    assert np.all(~has == (target == 0))
    umax = np.where(~kept, q, -1).max(axis=1)
    assert np.all(umax[has] <= kmin[has])                             # largest masses kept
    # ties at the cut value go to the lower indices
    tie = (q == kmin[:, None]) & has[:, None]
    idx = np.arange(n_kb)[None, :]
    last_kept_tie = np.where(tie & kept, idx, -1).max(axis=1)
    first_unkept_tie = np.where(tie & ~kept, idx, n_kb).min(axis=1)
    assert np.all(last_kept_tie < first_unkept_tie)
    # CSR rows ascending
    d = np.diff(ci[:rp[-1]])
    starts = rp[1:-1]
    inner = np.ones(d.size, dtype=bool)
    inner[starts[(starts > 0) & (starts <= d.size)] - 1] = False
    assert np.all(d[inner] > 0)


def test_block_mass_and_selection_full_size(B, full):
    wl, s, _, (qt, kt, vt) = full
    g = Hp.grid_of(wl)
    ws = B.new_workspace(s, B.OP_BLOCK_MASS)
    m = B.block_mass(qt, kt, s, ws=ws)
    assert B.device_status(ws) == 0
    mc = m.cpu()
    # every row with a valid query sums to 1 (fp32)
    valid = torch.from_numpy(O.valid_slots(g))
    has_q = valid.view(-1, wl.q_block).any(dim=1)
    sums = mc.double().sum(dim=-1)
    assert torch.allclose(sums[..., has_q], torch.ones_like(sums[..., has_q]), atol=1e-4)
    assert torch.all(sums[..., ~has_q] == 0)
    # sampled rows against the oracle
    rng = np.random.default_rng(1)
    scale = Hp.scale_of(wl)
    heads = rng.integers(0, s.heads, 6)
    for h in np.unique(heads):
        qh = qt[0:1, h:h + 1].cpu().double().numpy()
        kh = kt[0:1, h:h + 1].cpu().double().numpy()
        for i in rng.integers(0, s.n_qb, 8):
            ref = O.block_mass_row(qh, kh, g, 0, 0, int(i), wl.q_block, 64, scale)
            got = mc[0, h, i].double().numpy()
            assert np.abs(got - ref).max() <= Hp.MASS_ABS
            nz = ref > 0
            assert (np.abs(got - ref)[nz] / ref[nz]).max() < 1e-3
    # selection on the GPU masses, every row, for each threshold of the workload
    mrows = mc.numpy().reshape(-1, s.n_kb)
    for tau in sorted(set(wl.taus) | {0.99}):
        ws_t = B.new_workspace(s, B.OP_TOPP_SELECT)
        rp, ci = B.topp_select(m, s, tau, ws=ws_t)
        assert B.device_status(ws_t) == 0
        _selection_properties(mrows, rp.cpu().numpy().astype(np.int64),
                              ci.cpu().numpy().astype(np.int64), tau, s.n_kb)


def test_fwd_full_size_sampled_rows(B, full):
    wl, s, _, (qt, kt, vt) = full
    g = Hp.grid_of(wl)
    rp, ci = synth.draw_keep_csr(s.rows, s.n_kb, 0.957, seed=wl.seed + 5,
                                 empty_rows=(0, s.rows // 2))
    ws = B.new_workspace(s, B.OP_FWD)
    out, lse = B.bsattn_fwd(qt, kt, vt, rp.cuda(), ci.cuda(), s, want_lse=True, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    rp_np, ci_np = rp.numpy().astype(np.int64), ci.numpy().astype(np.int64)
    rng = np.random.default_rng(2)
    scale = Hp.scale_of(wl)
    heads = np.unique(rng.integers(0, s.heads, 4))
    errs, refmax = [], 0.0
    for h in heads:
        qh, kh, vh = (x[0:1, h:h + 1].cpu().double().numpy() for x in (qt, kt, vt))
        slots = rng.integers(0, s.Np, 128).tolist() + [0, 1, s.Np - 1]
        for p in slots:
            o_ref, l_ref = _oracle_row(qh, kh, vh, g, wl, h, s, int(p), rp_np, ci_np, scale)
            got = out[0, h, p].double().cpu().numpy()
            errs.append(np.abs(got - o_ref).max())
            refmax = max(refmax, np.abs(o_ref).max())
            lg = float(lse[0, h, p])
            if math.isinf(l_ref):
                assert math.isinf(lg) and lg < 0 and np.all(got == 0)
            else:
                assert abs(lg - l_ref) <= 1e-3
    errs = np.array(errs)
    assert errs.max() <= Hp.ATTN_MAX_ABS and errs.mean() <= Hp.ATTN_MEAN_ABS
    # outputs here are ~1e-4; hold the relative error to the bf16 output rounding
    assert errs.max() <= 2e-2 * refmax


def test_dense_fwd_mass_full_size(B, full):
    """The fused calibration at full size: its masses equal bsa_block_mass's within fp32
    rounding, and sampled output rows and log-sum-exps match the oracle's dense rows."""
    wl, s, _, (qt, kt, vt) = full
    g = Hp.grid_of(wl)
    ws = B.new_workspace(s, B.OP_BLOCK_MASS)
    out, mass, lse = B.dense_fwd_mass(qt, kt, vt, s, want_lse=True, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    m2 = B.block_mass(qt, kt, s, ws=ws)
    assert B.device_status(ws) == 0
    assert float((mass - m2).abs().max()) <= 1e-6
    del m2
    rng = np.random.default_rng(3)
    scale = Hp.scale_of(wl)
    all_blocks = np.arange(s.n_kb, dtype=np.int64)
    errs, refmax = [], 0.0
    for h in np.unique(rng.integers(0, s.heads, 3)):
        qh, kh, vh = (x[0:1, h:h + 1].cpu().double().numpy() for x in (qt, kt, vt))
        for p in rng.integers(0, s.Np, 96).tolist() + [0, s.Np - 1]:
            rp1 = np.zeros(s.n_qb + 1, dtype=np.int64)
            rp1[p // wl.q_block + 1:] = s.n_kb  # one dense row: every block kept
            o_ref, l_ref = O.masked_attention_query(qh, kh, vh, g, 0, 0, int(p), wl.q_block, 64,
                                                    rp1, all_blocks, scale)
            got = out[0, h, p].double().cpu().numpy()
            errs.append(np.abs(got - o_ref).max())
            refmax = max(refmax, np.abs(o_ref).max())
            lg = float(lse[0, h, p])
            if math.isinf(l_ref):
                assert math.isinf(lg) and lg < 0 and np.all(got == 0)
            else:
                assert abs(lg - l_ref) <= 1e-3
    errs = np.array(errs)
    assert errs.max() <= Hp.ATTN_MAX_ABS and errs.mean() <= Hp.ATTN_MEAN_ABS
    assert errs.max() <= 2e-2 * refmax
    del out, mass, lse
    torch.cuda.empty_cache()


def test_fwd_raster_full_size_matches_permuted_path(B, full):
    """The fused raster forward at full size, in the bench's launch configuration:
    bit-identical to the tile-major forward permuted back (whose rows the oracle checks)."""
    wl, s, (q, k, v), (qt, kt, vt) = full
    rp, ci = synth.draw_keep_csr(s.rows, s.n_kb, 0.957, seed=wl.seed + 5,
                                 empty_rows=(0, s.rows // 2))
    rp, ci = rp.cuda(), ci.cuda()
    ws = B.new_workspace(s, B.OP_FWD)
    out = B.bsattn_fwd_raster(q, k, v, rp, ci, s, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    back = B.tile_permute(B.bsattn_fwd(qt, kt, vt, rp, ci, s, ws=ws), s, inverse=True)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    assert torch.equal(out.view(torch.int16), back.view(torch.int16))
    del out, back
    torch.cuda.empty_cache()


def _oracle_row(qh, kh, vh, g, wl, h, s, p, rp, ci, scale):
    """Oracle row for head h: the CSR row index includes the head offset."""
    r = h * s.n_qb + p // wl.q_block
    sub_rp = np.array([0, rp[r + 1] - rp[r]])
    sub_ci = ci[rp[r]:rp[r + 1]]
    # a one-row CSR for the single-head arrays: the query's block index must map to row 0
    qb = p // wl.q_block
    rp1 = np.zeros(s.n_qb + 1, dtype=np.int64)
    rp1[qb + 1:] = sub_rp[1]
    return O.masked_attention_query(qh, kh, vh, g, 0, 0, p, wl.q_block, 64, rp1, sub_ci, scale)


def test_fp8_full_size_sampled_rows(B):
    """The FP8 workload's shapes: quantised codes and scales bit-exact on sampled tiles,
    attention rows against the oracle on its own dequantised inputs.  Unit value scale,
    sharp logits and V at 0.7x: the largest sampled output is near 1 (with the literal
    1/sqrt(128) scale outputs are ~1e-4 and the absolute bound would test nothing)."""
    wl = synth.WORKLOADS["wan14b_720p_fp8"].scaled(value_scale=1.0)
    s = B.Shape.of(wl)
    g = Hp.grid_of(wl)
    q, k, v = synth.draw_qkv(wl, device="cuda", sharpness=8.0)
    v = (v.float() * 0.7).to(torch.bfloat16)
    gq = [B.tile_permute_quant_e4m3(x, s) for x in (q, k, v)]
    rp, ci = synth.draw_keep_csr(s.rows, s.n_kb, 0.957, seed=77)
    ws = B.new_workspace(s, B.OP_FWD)
    out = B.bsattn_fwd(gq[0][0], gq[1][0], gq[2][0], rp.cuda(), ci.cuda(), s,
                       scales=(gq[0][1], gq[1][1], gq[2][1]), ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    rng = np.random.default_rng(3)
    scale = Hp.scale_of(wl)
    rp_np, ci_np = rp.numpy().astype(np.int64), ci.numpy().astype(np.int64)
    gots, refs = [], []
    for h in np.unique(rng.integers(0, s.heads, 2)):
        deq = []
        for x, (codes, scales) in zip((q, k, v), gq):
            xh = x[:, :, h:h + 1].float().cpu().numpy()
            rc, rs = O.quant_e4m3_tiles(O.permute_forward(xh, g))
            assert np.array_equal(codes[:, h:h + 1].cpu().numpy(), rc)
            assert np.array_equal(scales[:, h:h + 1].cpu().numpy().view(np.uint32), rs.view(np.uint32))
            deq.append(O.dequant_e4m3_tiles(rc, rs))
        for p in rng.integers(0, s.Np, 64).tolist():
            o_ref, _ = _oracle_row(deq[0], deq[1], deq[2], g, wl, int(h), s, int(p), rp_np, ci_np,
                                   scale)
            gots.append(out[0, h, p].double().cpu().numpy())
            refs.append(o_ref)
    Hp.assert_attn_close(np.stack(gots), np.stack(refs), fp8=True)
