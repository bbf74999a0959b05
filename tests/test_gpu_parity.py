"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element.

Small seeded shapes that the oracle finishes in seconds but that still span several CTAs,
ragged pads in every dimension, a partial last Q tile, an odd kv-block count, whole pad
tiles, both head dims and both query-block sizes.  Integer and index work must be
bit-exact; floating point within the stated tolerances.
"""
import math

import numpy as np
import pytest
import torch

import helpers as Hp
from block_sparse_attention_25_b200 import synth
from oracle import bsa_oracle as O

pytestmark = pytest.mark.gpu

WLS = Hp.small_workloads()
IDS = [w.name for w in WLS]


@pytest.fixture(scope="module")
def B(cuda_device):
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    return b


def _shape(B, wl):
    return B.Shape.of(wl)


# ------------------------------------------------------------------ permutation
@pytest.mark.parametrize("wl", WLS, ids=IDS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_permute_bit_exact(B, wl, dtype):
    g = Hp.grid_of(wl)
    s = _shape(B, wl)
    gen = torch.Generator().manual_seed(wl.seed)
    x = torch.randn(wl.batch, wl.S, wl.heads, wl.head_dim, generator=gen).to(dtype)
    xd = x.cuda()
    y = B.tile_permute(xd, s)
    ref = O.permute_forward(x.view(torch.int16 if dtype == torch.bfloat16 else torch.int32).numpy(), g)
    got = y.cpu().view(torch.int16 if dtype == torch.bfloat16 else torch.int32).numpy()
    assert np.array_equal(got, ref)
    back = B.tile_permute(y, s, inverse=True)
    assert torch.equal(back.cpu().view(torch.uint8), x.view(torch.uint8))
    # inverse of the oracle's tile-major tensor
    ref_inv = O.permute_inverse(ref, g)
    got_inv = B.tile_permute(torch.from_numpy(ref).view(dtype).cuda(), s, inverse=True)
    assert np.array_equal(got_inv.cpu().view(torch.int16 if dtype == torch.bfloat16 else torch.int32).numpy(), ref_inv)


# ------------------------------------------------------------------ FP8 quantisation
@pytest.mark.parametrize("wl", WLS, ids=IDS)
def test_quant_e4m3_bit_exact(B, wl):
    g = Hp.grid_of(wl)
    s = _shape(B, wl)
    q, _, _ = Hp.draw(wl, value_scale=1.0, sharp=3.0)
    q[0, 0, 0] = 0.0                       # a row of exact zeros
    q[0, 1, 0, :3] = -0.0
    codes, scales = B.tile_permute_quant_e4m3(q.cuda(), s)
    xt = O.permute_forward(q.float().numpy(), g)
    ref_codes, ref_scales = O.quant_e4m3_tiles(xt)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_scales.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), ref_codes)


# ------------------------------------------------------------------ block mass
@pytest.mark.parametrize("wl", WLS, ids=IDS)
@pytest.mark.parametrize("sharp", [1.0, 6.0])
def test_block_mass_parity(B, wl, sharp):
    g = Hp.grid_of(wl)
    s = _shape(B, wl)
    q, k, _ = Hp.draw(wl, value_scale=1.0, sharp=sharp)
    qt = B.tile_permute(q.cuda(), s)
    kt = B.tile_permute(k.cuda(), s)
    ws = B.new_workspace(s, B.OP_BLOCK_MASS)
    m = B.block_mass(qt, kt, s, ws=ws)
    assert B.device_status(ws) == 0
    ref = O.block_mass(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g), g, wl.q_block, 64,
                       Hp.scale_of(wl))
    # structural zeros (pad-only kv blocks, query blocks without valid queries) are exact
    Hp.assert_mass_close(m.cpu().double().numpy(), ref)


@pytest.mark.parametrize("wl", [WLS[0], WLS[1], WLS[3]], ids=[IDS[0], IDS[1], IDS[3]])
@pytest.mark.parametrize("ramp", ["ascending", "descending", "odd_blocks"])
def test_block_mass_wide_logit_range(B, wl, ramp):
    """Keys scaled per kv block so that a row's logits span far more than 64 log2 units:
    ascending, each row's first blocks lie far below its later ones, so the kernel raises
    its reference max and rescales the block sums already written; descending, later
    blocks underflow against the first; odd_blocks, the two column halves of a row end
    with reference maxima far apart, so the final merge weights one half by a tiny factor."""
    g = Hp.grid_of(wl)
    s = _shape(B, wl)
    q, k, _ = Hp.draw(wl, value_scale=1.0, sharp=1.0)
    qt64 = Hp.oracle_tiled(q, g)
    kt_bf, kt64, scale, bmax = Hp.wide_range_keys(wl, q, k, ramp)
    # the data does what the docstring says: the spread of a row's block maxima, log2 units
    if ramp == "ascending":
        assert np.median(bmax[..., 0::2].max(-1) - bmax[..., 0]) > 64.0
    if ramp == "odd_blocks":
        assert np.median(bmax[..., 1::2].max(-1) - bmax[..., 0::2].max(-1)) > 64.0
    ws = B.new_workspace(s, B.OP_BLOCK_MASS)
    m = B.block_mass(B.tile_permute(q.cuda(), s), kt_bf.cuda(), s, softmax_scale=scale, ws=ws)
    assert B.device_status(ws) == 0
    ref = O.block_mass(qt64, kt64, g, wl.q_block, 64, scale)
    Hp.assert_mass_close(m.cpu().double().numpy(), ref)


# ------------------------------------------------------------------ top-p selection
def _topp_check(B, s, mass_np32, tau):
    mass = torch.from_numpy(np.ascontiguousarray(mass_np32)).cuda()
    ws = B.new_workspace(s, B.OP_TOPP_SELECT)
    rp, ci = B.topp_select(mass, s, tau, ws=ws)
    assert B.device_status(ws) == 0
    rp_ref, ci_ref = O.topp_select(mass_np32.reshape(-1, s.n_kb), tau)
    rp_got = rp.cpu().numpy().astype(np.int64)
    assert np.array_equal(rp_got, rp_ref)
    nnz = int(rp_got[-1])
    assert np.array_equal(ci[:nnz].cpu().numpy().astype(np.int64), ci_ref)


@pytest.mark.parametrize("kind", ["dirichlet", "peaked", "ties", "uniform"])
@pytest.mark.parametrize("tau", [0.5, 0.9, 0.95, 0.99, 1.0])
def test_topp_bit_exact_synthetic(B, kind, tau):
    wl = synth.WORKLOADS["wan13b_480p"].scaled(heads=2)
    s = _shape(B, wl)
    m = synth.draw_mass_rows(s.rows, s.n_kb, seed=7, kind=kind,
                             zero_frac=0.2 if kind == "dirichlet" else 0.0)
    _topp_check(B, s, m.numpy().reshape(s.batch, s.heads, s.n_qb, s.n_kb), tau)


def test_topp_bit_exact_zero_rows_and_tiny_masses(B):
    wl = WLS[0]
    s = _shape(B, wl)
    m = synth.draw_mass_rows(s.rows, s.n_kb, seed=8, kind="dirichlet").numpy()
    m[0] = 0.0                                  # all-zero row -> empty
    m[1] = m[1] * 1e-7                          # masses below 2^-17 (rounded in fixed point)
    m[2, :] = np.float32(1.0 / s.n_kb)          # all equal
    m[3, ::2] = 0.0
    _topp_check(B, s, m.reshape(s.batch, s.heads, s.n_qb, s.n_kb), 0.99)


@pytest.mark.parametrize("wl", WLS, ids=IDS)
def test_topp_bit_exact_on_oracle_masses(B, wl):
    g = Hp.grid_of(wl)
    s = _shape(B, wl)
    q, k, _ = Hp.draw(wl, value_scale=1.0, sharp=6.0)
    ref = O.block_mass(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g), g, wl.q_block, 64,
                       Hp.scale_of(wl)).astype(np.float32)
    for tau in (0.9, 0.99):
        _topp_check(B, s, ref, tau)


def _structured_rows(n_rows, n, seed):
    """Rows whose shapes stress a pivoting selector: sorted either way, geometric (values
    over many orders of magnitude), two levels, one non-zero, dyadic values whose running
    sums hit the target exactly, and shuffled distinct values."""
    rng = np.random.default_rng(seed)
    rows = []
    for i in range(n_rows):
        kind = i % 8
        if kind == 0:
            r = np.arange(1, n + 1, dtype=np.float64)
        elif kind == 1:
            r = np.arange(n, 0, -1, dtype=np.float64)
        elif kind == 2:
            r = 2.0 ** -np.minimum(np.arange(n), 60)
        elif kind == 3:
            r = np.where(rng.random(n) < 0.5, 1.0, 3.0)
        elif kind == 4:
            r = np.zeros(n)
            r[rng.integers(0, n)] = 1.0
        elif kind == 5:
            r = 2.0 ** -rng.integers(1, 12, n).astype(np.float64)
        elif kind == 6:
            r = rng.permutation(n).astype(np.float64) + 1.0
        else:
            r = 2.0 ** -np.minimum(np.arange(n), 60)[::-1]
        rows.append(r / r.sum())
    return np.asarray(rows, dtype=np.float32)


@pytest.mark.parametrize("tau", [0.5, 0.9, 0.99, 1.0])
def test_topp_bit_exact_structured_rows(B, tau):
    wl = WLS[0]
    s = _shape(B, wl)
    m = _structured_rows(s.rows, s.n_kb, seed=21)
    _topp_check(B, s, m.reshape(s.batch, s.heads, s.n_qb, s.n_kb), tau)


@pytest.mark.parametrize("cols", [1, 2, 3, 31, 33, 257])
def test_topp_rows_bit_exact_short_and_odd_rows(B, cols):
    m = np.concatenate([_structured_rows(16, cols, seed=cols),
                        synth.draw_mass_rows(16, cols, seed=cols, kind="ties").numpy()])
    for tau in (0.5, 0.99, 1.0):
        rp, ci = B.topp_select_rows(torch.from_numpy(m).cuda(), tau)
        rp_ref, ci_ref = O.topp_select(m, tau)
        rp_got = rp.cpu().numpy().astype(np.int64)
        assert np.array_equal(rp_got, rp_ref)
        assert np.array_equal(ci[:int(rp_got[-1])].cpu().numpy().astype(np.int64), ci_ref)


def test_topp_capacity_overflow_is_reported(B):
    wl = WLS[0]
    s = _shape(B, wl)
    m = torch.full((s.batch, s.heads, s.n_qb, s.n_kb), 1.0 / s.n_kb, device="cuda")
    ws = B.new_workspace(s, B.OP_TOPP_SELECT)
    cap = 10
    rp, ci = B.topp_select(m, s, 1.0, col_capacity=cap, ws=ws)
    assert B.device_status(ws) == 3
    assert int(rp[-1]) == s.rows * s.n_kb
    assert ci[:cap].cpu().tolist() == list(range(cap))


# ------------------------------------------------------------------ attention
def _fwd_compare(B, wl, q, k, v, rp, ci, want_lse=True):
    g = Hp.grid_of(wl)
    s = _shape(B, wl)
    qt, kt, vt = (B.tile_permute(x.cuda(), s) for x in (q, k, v))
    rp_d, ci_d = Hp.csr_to_device(rp, ci, "cuda")
    ws = B.new_workspace(s, B.OP_FWD)
    out, lse = B.bsattn_fwd(qt, kt, vt, rp_d, ci_d, s, want_lse=True, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    o_ref, lse_ref = O.masked_attention(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g),
                                        Hp.oracle_tiled(v, g), g, wl.q_block, 64, rp, ci,
                                        Hp.scale_of(wl))
    return Hp.assert_fwd_close(out.cpu().double().numpy(), lse.cpu().double().numpy(),
                               o_ref, lse_ref)


@pytest.mark.parametrize("wl", WLS, ids=IDS)
@pytest.mark.parametrize("sharp", [1.0, 6.0])
@pytest.mark.parametrize("tau", [0.9, 0.99])
def test_fwd_parity_oracle_csr(B, wl, sharp, tau):
    g = Hp.grid_of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=sharp)
    mass = O.block_mass(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g), g, wl.q_block, 64,
                        Hp.scale_of(wl))
    rp, ci = Hp.csr_from_oracle(mass, tau)
    _fwd_compare(B, wl, q, k, v, rp, ci)


@pytest.mark.parametrize("wl", WLS, ids=IDS)
@pytest.mark.parametrize("keep", [1.0, 0.6, 0.15])
def test_fwd_parity_random_csr(B, wl, keep):
    s = synth.Workload  # noqa: F841
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=4.0)
    n_qb, n_kb = wl.Np // wl.q_block, wl.Np // 64
    R = wl.batch * wl.heads * n_qb
    rp, ci = synth.draw_keep_csr(R, n_kb, keep, seed=wl.seed + 100, empty_rows=(0, R - 1))
    _fwd_compare(B, wl, q, k, v, rp.numpy(), ci.numpy())


def test_fwd_all_rows_empty(B):
    wl = WLS[0]
    q, k, v = Hp.draw(wl, value_scale=1.0)
    n_qb, n_kb = wl.Np // wl.q_block, wl.Np // 64
    R = wl.batch * wl.heads * n_qb
    rp = np.zeros(R + 1, np.int64)
    ci = np.zeros(0, np.int64)
    _fwd_compare(B, wl, q, k, v, rp, ci)


def test_fwd_rescale_path(B):
    """Large logits arriving late force the lazy O rescale: the max grows by >> 8 (log2)."""
    wl = WLS[0]
    g = Hp.grid_of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=1.0)
    # scale the keys of later kv blocks up so each new block raises the row max
    kt = O.permute_forward(k.float().numpy(), g)
    n_kb = wl.Np // 64
    for j in range(n_kb):
        kt[:, :, j * 64:(j + 1) * 64] *= (1.0 + 1.5 * j)
    k2 = torch.from_numpy(O.permute_inverse(kt, g)).to(torch.bfloat16)
    q2 = (q.float() * 4.0).to(torch.bfloat16)
    n_qb = wl.Np // wl.q_block
    R = wl.batch * wl.heads * n_qb
    rp = np.arange(R + 1) * n_kb
    ci = np.tile(np.arange(n_kb), R)
    _fwd_compare(B, wl, q2, k2, v, rp, ci)


def test_fwd_reports_bad_csr(B):
    wl = WLS[0]
    s = _shape(B, wl)
    q, k, v = Hp.draw(wl, value_scale=1.0)
    qt, kt, vt = (B.tile_permute(x.cuda(), s) for x in (q, k, v))
    R = s.rows
    rp = torch.arange(R + 1, dtype=torch.int32, device="cuda") * 2
    ci = torch.zeros(2 * R, dtype=torch.int32, device="cuda")   # duplicate indices: not ascending
    ci[1::2] = 0
    ws = B.new_workspace(s, B.OP_FWD)
    B.bsattn_fwd(qt, kt, vt, rp, ci, s, ws=ws)
    assert B.device_status(ws) == 6
    ci2 = torch.full((2 * R,), s.n_kb + 5, dtype=torch.int32, device="cuda")  # out of range
    ws2 = B.new_workspace(s, B.OP_FWD)
    B.bsattn_fwd(qt, kt, vt, rp, ci2, s, ws=ws2)
    assert B.device_status(ws2) == 6


# ------------------------------------------------------------------ whole pipeline
@pytest.mark.parametrize("wl", WLS[:3], ids=IDS[:3])
def test_pipeline_calibrate_then_reuse(B, wl):
    """Calibrate on draw 0 (mass -> select), attend on a correlated re-draw with the frozen
    lists.  The GPU pipeline and the oracle pipeline each run on their own outputs; the
    selections must agree row by row (bar rows whose masses tie at the cut within the
    mass tolerance) and the outputs are compared on the rows where they agree."""
    g = Hp.grid_of(wl)
    s = _shape(B, wl)
    wl1 = wl.scaled(value_scale=1.0, storage="bf16")
    q, k, v = synth.draw_qkv(wl1, sharpness=5.0)
    qt, kt = B.tile_permute(q.cuda(), s), B.tile_permute(k.cuda(), s)
    m = B.block_mass(qt, kt, s)
    rp, ci = B.topp_select(m, s, 0.99)
    mg = m.cpu().numpy().reshape(-1, s.n_kb)
    rpg = rp.cpu().numpy().astype(np.int64)
    cig = ci.cpu().numpy().astype(np.int64)
    # property of the GPU selection on the GPU masses: reaches the target, and is minimal
    for r in range(s.rows):
        kept = cig[rpg[r]:rpg[r + 1]]
        qfp = O.fixed_point_masses(mg[r])
        tgt = O.topp_target(int(qfp.sum()), 0.99)
        assert qfp[kept].sum() >= tgt
        if kept.size:
            assert qfp[kept].sum() - qfp[kept].min() < tgt
    # the oracle pipeline on the same draw
    mo = O.block_mass(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g), g, wl.q_block, 64,
                      Hp.scale_of(wl))
    rpo, cio = Hp.csr_from_oracle(mo, 0.99)
    same = np.array([np.array_equal(cig[rpg[r]:rpg[r + 1]], cio[rpo[r]:rpo[r + 1]])
                     for r in range(s.rows)])
    assert same.mean() >= 0.95, same.mean()
    # re-draw, attend with each side's frozen lists, compare rows whose lists agree
    q2, k2, v2 = synth.redraw_qkv(wl1, 1, sharpness=5.0)
    q2t, k2t, v2t = (B.tile_permute(x.cuda(), s) for x in (q2, k2, v2))
    out = B.bsattn_fwd(q2t, k2t, v2t, rp, ci, s)
    o_ref, _ = O.masked_attention(Hp.oracle_tiled(q2, g), Hp.oracle_tiled(k2, g),
                                  Hp.oracle_tiled(v2, g), g, wl.q_block, 64, rpo, cio,
                                  Hp.scale_of(wl))
    got = out.cpu().double().numpy()
    n_qb = s.n_qb
    rows = np.repeat(same.reshape(s.batch, s.heads, n_qb), wl.q_block, axis=2)
    Hp.assert_attn_close(got[rows], o_ref[rows], signal_guard=False)


# ------------------------------------------------------------------ FP8 attention
FP8_WLS = [w for w in WLS if w.head_dim == 128]
# e4m3 rounds P to 4 significant bits, so the output error is a fraction (<= 2^-4) of the
# output itself.  Sharp logits keep the largest output above 10x the absolute bound (the
# signal guard); V at 0.7x keeps it near 1, where 2^-4 of it stays inside the 6e-2 bound.
FP8_V = 0.7


def _fp8_draw(wl, sharp):
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=sharp)
    return q, k, (v.float() * FP8_V).to(torch.bfloat16)


def _fp8_compare(B, wl, q, k, v, rp, ci):
    """GPU: quantise (bit-exact against the oracle's quantiser) and attend in e4m3.
    Oracle: its own quantisation, dequantised to fp64, masked attention."""
    g = Hp.grid_of(wl)
    s = _shape(B, wl)
    gq = [B.tile_permute_quant_e4m3(x.cuda(), s) for x in (q, k, v)]
    deq = []
    for x, (codes, scales) in zip((q, k, v), gq):
        rc, rs = O.quant_e4m3_tiles(O.permute_forward(x.float().numpy(), g))
        assert np.array_equal(codes.cpu().numpy(), rc)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))
        deq.append(O.dequant_e4m3_tiles(rc, rs))
    rp_d, ci_d = Hp.csr_to_device(rp, ci, "cuda")
    ws = B.new_workspace(s, B.OP_FWD)
    out, lse = B.bsattn_fwd(gq[0][0], gq[1][0], gq[2][0], rp_d, ci_d, s,
                            scales=(gq[0][1], gq[1][1], gq[2][1]), want_lse=True, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    o_ref, lse_ref = O.masked_attention(deq[0], deq[1], deq[2], g, wl.q_block, 64, rp, ci,
                                        Hp.scale_of(wl))
    return Hp.assert_fwd_close(out.cpu().double().numpy(), lse.cpu().double().numpy(),
                               o_ref, lse_ref, fp8=True)


@pytest.mark.parametrize("wl", FP8_WLS, ids=[w.name for w in FP8_WLS])
@pytest.mark.parametrize("sharp", [6.0, 8.0])
def test_fwd_fp8_parity_oracle_csr(B, wl, sharp):
    g = Hp.grid_of(wl)
    q, k, v = _fp8_draw(wl, sharp)
    mass = O.block_mass(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g), g, wl.q_block, 64,
                        Hp.scale_of(wl))
    rp, ci = Hp.csr_from_oracle(mass, 0.99)
    _fp8_compare(B, wl, q, k, v, rp, ci)


@pytest.mark.parametrize("wl", FP8_WLS, ids=[w.name for w in FP8_WLS])
def test_fwd_fp8_parity_random_csr(B, wl):
    q, k, v = _fp8_draw(wl, 8.0)
    n_qb, n_kb = wl.Np // wl.q_block, wl.Np // 64
    R = wl.batch * wl.heads * n_qb
    rp, ci = synth.draw_keep_csr(R, n_kb, 0.5, seed=wl.seed + 200, empty_rows=(1,))
    _fp8_compare(B, wl, q, k, v, rp.numpy(), ci.numpy())


def test_fwd_fp8_rescale_path(B):
    """Growing logits across kv blocks exercise the lazy rescale with e4m3 P."""
    wl = FP8_WLS[0]
    g = Hp.grid_of(wl)
    q, k, v = _fp8_draw(wl, 1.0)
    kt = O.permute_forward(k.float().numpy(), g)
    n_kb = wl.Np // 64
    for j in range(n_kb):
        kt[:, :, j * 64:(j + 1) * 64] *= (1.0 + 1.5 * j)
    k2 = torch.from_numpy(O.permute_inverse(kt, g)).to(torch.bfloat16)
    q2 = (q.float() * 4.0).to(torch.bfloat16)
    n_qb = wl.Np // wl.q_block
    R = wl.batch * wl.heads * n_qb
    rp = np.arange(R + 1) * n_kb
    ci = np.tile(np.arange(n_kb), R)
    _fp8_compare(B, wl, q2, k2, v, rp, ci)


# ------------------------------------------------------------------ frozen lists on disk
def test_forward_on_reloaded_lists_is_bit_identical(B, tmp_path):
    """Calibrate, select, save the lists, load them back: the forward over the loaded lists
    equals the forward over the selection's own lists bit for bit."""
    wl = WLS[0]
    s = _shape(B, wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=6.0)
    qt, kt, vt = (B.tile_permute(x.cuda(), s) for x in (q, k, v))
    rp, ci = B.topp_select(B.block_mass(qt, kt, s), s, 0.95)
    path = tmp_path / "frozen.bin"
    B.save_lists(path, rp, ci, s, 0.95)
    rp2, ci2, tau = B.load_lists(path, s)
    assert np.float32(tau) == np.float32(0.95)
    n = int(rp[-1])
    assert torch.equal(rp2, rp) and torch.equal(ci2[:n], ci[:n])
    out = B.bsattn_fwd(qt, kt, vt, rp, ci, s)
    out2 = B.bsattn_fwd(qt, kt, vt, rp2, ci2, s)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
