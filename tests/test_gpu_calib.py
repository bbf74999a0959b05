"""GPU parity of the fused calibration call: dense attention output and block masses in one
pass, against the oracle's dense attention (every block kept) and its block masses."""
import numpy as np
import pytest

import helpers as Hp
from oracle import bsa_oracle as O

pytestmark = pytest.mark.gpu

WLS = Hp.small_workloads()


@pytest.fixture(scope="module")
def B(cuda_device):
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    return b


@pytest.mark.parametrize("wl", WLS, ids=[w.name for w in WLS])
@pytest.mark.parametrize("sharp", [1.0, 6.0])
def test_dense_fwd_mass_parity(B, wl, sharp):
    g = Hp.grid_of(wl)
    s = B.Shape.of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=sharp)
    qt, kt, vt = (B.tile_permute(x.cuda(), s) for x in (q, k, v))
    ws = B.new_workspace(s, B.OP_BLOCK_MASS)
    out, mass, lse = B.dense_fwd_mass(qt, kt, vt, s, want_lse=True, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    qo, ko, vo = (Hp.oracle_tiled(x, g) for x in (q, k, v))
    m_ref = O.block_mass(qo, ko, g, wl.q_block, 64, Hp.scale_of(wl))
    got_m = mass.cpu().double().numpy()
    assert np.abs(got_m - m_ref).max() <= Hp.MASS_ABS
    assert np.all(got_m[m_ref == 0] == 0)
    n_qb, n_kb = wl.Np // wl.q_block, wl.Np // 64
    R = wl.batch * wl.heads * n_qb
    rp = np.arange(R + 1) * n_kb
    ci = np.tile(np.arange(n_kb), R)
    o_ref, lse_ref = O.masked_attention(qo, ko, vo, g, wl.q_block, 64, rp, ci, Hp.scale_of(wl))
    e = Hp.assert_attn_close(out.cpu().double().numpy(), o_ref, signal_guard=False)
    zero = ~np.isfinite(lse_ref)
    lg = lse.cpu().double().numpy()
    assert np.all(np.isneginf(lg[zero]))
    assert np.abs(lg[~zero] - lse_ref[~zero]).max() <= 1e-3


@pytest.mark.parametrize("wl", [WLS[0], WLS[1], WLS[3]], ids=[WLS[i].name for i in (0, 1, 3)])
@pytest.mark.parametrize("ramp", ["ascending", "descending", "odd_blocks"])
def test_dense_fwd_mass_wide_logit_range(B, wl, ramp):
    """Keys scaled per kv block so that rows raise their reference max mid-walk (ascending:
    the output, the row sum and the block sums already written are rescaled), underflow
    against the first blocks (descending), or alternate between tiny and large blocks."""
    g = Hp.grid_of(wl)
    s = B.Shape.of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=1.0)
    kt_bf, ko, scale, bmax = Hp.wide_range_keys(wl, q, k, ramp)
    if ramp == "ascending":  # most rows raise their reference after the first step
        assert np.median(bmax[..., 2:].max(-1) - bmax[..., :2].max(-1)) > 16.0
    qt, vt = (B.tile_permute(x.cuda(), s) for x in (q, v))
    ws = B.new_workspace(s, B.OP_BLOCK_MASS)
    out, mass, lse = B.dense_fwd_mass(qt, kt_bf.cuda(), vt, s, softmax_scale=scale,
                                      want_lse=True, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    qo, vo = (Hp.oracle_tiled(x, g) for x in (q, v))
    m_ref = O.block_mass(qo, ko, g, wl.q_block, 64, scale)
    got_m = mass.cpu().double().numpy()
    assert np.abs(got_m - m_ref).max() <= Hp.MASS_ABS
    assert np.all(got_m[m_ref == 0] == 0)
    n_qb, n_kb = wl.Np // wl.q_block, wl.Np // 64
    R = wl.batch * wl.heads * n_qb
    rp = np.arange(R + 1) * n_kb
    ci = np.tile(np.arange(n_kb), R)
    o_ref, lse_ref = O.masked_attention(qo, ko, vo, g, wl.q_block, 64, rp, ci, scale)
    e = Hp.assert_attn_close(out.cpu().double().numpy(), o_ref, signal_guard=False)
    zero = ~np.isfinite(lse_ref)
    lg = lse.cpu().double().numpy()
    assert np.all(np.isneginf(lg[zero]))
    assert np.abs(lg[~zero] - lse_ref[~zero]).max() <= 1e-3


def test_dense_fwd_mass_matches_separate_calls(B):
    """The fused masses equal bsa_block_mass's within fp32 rounding, and its output equals
    bsa_fwd over the full list."""
    wl = WLS[0]
    s = B.Shape.of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=4.0)
    qt, kt, vt = (B.tile_permute(x.cuda(), s) for x in (q, k, v))
    out, mass = B.dense_fwd_mass(qt, kt, vt, s)
    m2 = B.block_mass(qt, kt, s)
    assert float((mass - m2).abs().max()) <= 1e-6
    import torch
    R, n_kb = s.rows, s.n_kb
    rp = (torch.arange(R + 1, dtype=torch.int32) * n_kb).cuda()
    ci = torch.arange(n_kb, dtype=torch.int32).repeat(R).cuda()
    o2 = B.bsattn_fwd(qt, kt, vt, rp, ci, s)
    assert float((out.float() - o2.float()).abs().max()) <= 1e-2


# More than twice as many CTAs (head, 256 query slots) as the GPU has SMs, so the
# calibration kernels' workspace slices are claimed, given back and claimed again by later
# CTAs; ragged pads keep partial last CTAs in every head.
MANY = [
    Hp.synth.Workload("many-heads-6x10x11-h64-d128-bq64", 1, 64, 128, 6, 10, 11, 8, 12, 12, 64, 64,
                      seed=21),
    Hp.synth.Workload("many-heads-5x7x9-b2-h80-d64-bq128", 2, 80, 64, 5, 7, 9, 8, 8, 12, 128, 64,
                      seed=22),
]


@pytest.mark.parametrize("wl", MANY, ids=[w.name for w in MANY])
def test_calibration_reuses_workspace_slices(B, wl):
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    items = wl.batch * wl.heads * ((wl.Np + 255) // 256)
    assert items > 2 * sms
    g = Hp.grid_of(wl)
    s = B.Shape.of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=4.0)
    qt, kt, vt = (B.tile_permute(x.cuda(), s) for x in (q, k, v))
    qo, ko, vo = (Hp.oracle_tiled(x, g) for x in (q, k, v))
    m_ref = O.block_mass(qo, ko, g, wl.q_block, 64, Hp.scale_of(wl))
    ws = B.new_workspace(s, B.OP_BLOCK_MASS)
    m = B.block_mass(qt, kt, s, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    got = m.cpu().double().numpy()
    assert np.abs(got - m_ref).max() <= Hp.MASS_ABS
    nz = m_ref > 1e-6
    assert (np.abs(got - m_ref)[nz] / m_ref[nz]).max() < 1e-3
    assert np.all(got[m_ref == 0] == 0)
    out, mass, lse = B.dense_fwd_mass(qt, kt, vt, s, want_lse=True, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    assert float((mass - m).abs().max()) <= 1e-6
    n_qb, n_kb = wl.Np // wl.q_block, wl.Np // 64
    R = wl.batch * wl.heads * n_qb
    o_ref, lse_ref = O.masked_attention(qo, ko, vo, g, wl.q_block, 64, np.arange(R + 1) * n_kb,
                                        np.tile(np.arange(n_kb), R), Hp.scale_of(wl))
    Hp.assert_attn_close(out.cpu().double().numpy(), o_ref, signal_guard=False)
    fin = np.isfinite(lse_ref)
    assert np.abs(lse.cpu().double().numpy()[fin] - lse_ref[fin]).max() <= 1e-3
