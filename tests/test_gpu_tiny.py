"""GPU parity on the tiny workload (4x8x8 tokens = 4 tiles, 2 heads, D = 64, fp32 source),
where the whole oracle runs: every step of the path is compared element by element, and
each selected row is checked by brute force over all 16 subsets of its 4 kv blocks.

The source is fp32.  The permutation runs on the fp32 values (bit-exact); the attention
kernels take bf16, so both sides see the bf16 cast of the drawn values.
"""
import itertools

import numpy as np
import pytest
import torch

import helpers as Hp
from block_sparse_attention_25_b200 import synth
from oracle import bsa_oracle as O

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["tiny"]
TAUS = (0.5, 0.9, 0.99, 1.0)


@pytest.fixture(scope="module")
def B(cuda_device):
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    return b


@pytest.fixture(scope="module")
def tiny(B):
    assert WL.storage == "fp32" and WL.n_kb == 4
    q32, k32, v32 = synth.draw_qkv(WL)
    s = B.Shape.of(WL)
    g = Hp.grid_of(WL)
    qb, kb, vb = (x.to(torch.bfloat16) for x in (q32, k32, v32))
    ref_t = [Hp.oracle_tiled(x, g) for x in (qb, kb, vb)]
    return s, g, (q32, k32, v32), (qb, kb, vb), ref_t


def test_tiny_permute_fp32_bit_exact(B, tiny):
    s, g, src32, _, _ = tiny
    for x in src32:
        y = B.tile_permute(x.cuda(), s)
        ref = O.permute_forward(x.view(torch.int32).numpy(), g)
        assert np.array_equal(y.cpu().view(torch.int32).numpy(), ref)
        back = B.tile_permute(y, s, inverse=True)
        assert torch.equal(back.cpu().view(torch.int32), x.view(torch.int32))


def _gpu_tiled(B, s, xs):
    return [B.tile_permute(x.cuda(), s) for x in xs]


def test_tiny_block_mass_matches_full_oracle(B, tiny):
    s, g, _, bf, (qo, ko, _) = tiny
    qt, kt, _ = _gpu_tiled(B, s, bf)
    ws = B.new_workspace(s, B.OP_BLOCK_MASS)
    m = B.block_mass(qt, kt, s, ws=ws)
    assert B.device_status(ws) == 0
    ref = O.block_mass(qo, ko, g, WL.q_block, 64, Hp.scale_of(WL))
    got = m.cpu().double().numpy()
    assert np.abs(got - ref).max() <= Hp.MASS_ABS
    assert (np.abs(got - ref) / ref).max() < 1e-3          # every block holds valid keys
    np.testing.assert_allclose(got.sum(-1), 1.0, rtol=0, atol=1e-5)


def _brute_force_minimal(qfp: np.ndarray, tau) -> tuple:
    """Smallest kv-block set reaching the fixed-point target; among those the largest sum,
    then the lexicographically smallest index set (the tie rule)."""
    tgt = O.topp_target(int(qfp.sum()), tau)
    n = qfp.size
    for size in range(n + 1):
        best = None
        for sub in itertools.combinations(range(n), size):
            tot = int(qfp[list(sub)].sum())
            if tot >= tgt and (best is None or tot > best[0]):
                best = (tot, sub)            # combinations come in lexicographic order
        if best is not None:
            return best[1]
    raise AssertionError("no subset reaches the target")


@pytest.mark.parametrize("tau", TAUS)
def test_tiny_selection_is_minimal_by_brute_force(B, tiny, tau):
    s, g, _, bf, _ = tiny
    qt, kt, _ = _gpu_tiled(B, s, bf)
    m = B.block_mass(qt, kt, s)
    ws = B.new_workspace(s, B.OP_TOPP_SELECT)
    rp, ci = B.topp_select(m, s, tau, ws=ws)
    assert B.device_status(ws) == 0
    mrows = m.cpu().numpy().reshape(-1, s.n_kb)
    rp_ref, ci_ref = O.topp_select(mrows, tau)          # the oracle on the same masses
    rpg = rp.cpu().numpy().astype(np.int64)
    cig = ci[:int(rpg[-1])].cpu().numpy().astype(np.int64)
    assert np.array_equal(rpg, rp_ref) and np.array_equal(cig, ci_ref)
    for r in range(s.rows):
        kept = tuple(cig[rpg[r]:rpg[r + 1]].tolist())
        assert kept == _brute_force_minimal(O.fixed_point_masses(mrows[r]), tau), (r, kept)


@pytest.mark.parametrize("tau", TAUS)
def test_tiny_attention_on_selected_lists(B, tiny, tau):
    s, g, _, bf, (qo, ko, vo) = tiny
    qt, kt, vt = _gpu_tiled(B, s, bf)
    m = B.block_mass(qt, kt, s)
    rp, ci = B.topp_select(m, s, tau)
    ws = B.new_workspace(s, B.OP_FWD)
    out, lse = B.bsattn_fwd(qt, kt, vt, rp, ci, s, want_lse=True, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    rpn = rp.cpu().numpy().astype(np.int64)
    cin = ci[:int(rpn[-1])].cpu().numpy().astype(np.int64)
    o_ref, lse_ref = O.masked_attention(qo, ko, vo, g, WL.q_block, 64, rpn, cin, Hp.scale_of(WL))
    Hp.assert_attn_close(out.cpu().double().numpy(), o_ref, signal_guard=False)
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= 1e-3


def test_tiny_full_lists_equal_dense_attention(B, tiny):
    """Every block kept: the sparse forward and the fused calibration both give dense
    attention, and the calibration's masses are the oracle's."""
    s, g, _, bf, (qo, ko, vo) = tiny
    qt, kt, vt = _gpu_tiled(B, s, bf)
    rp = torch.arange(s.rows + 1, dtype=torch.int32, device="cuda") * s.n_kb
    ci = torch.arange(s.n_kb, dtype=torch.int32, device="cuda").repeat(s.rows)
    out = B.bsattn_fwd(qt, kt, vt, rp, ci, s)
    dense, mass, lse = B.dense_fwd_mass(qt, kt, vt, s, want_lse=True)
    rpn = np.arange(s.rows + 1) * s.n_kb
    cin = np.tile(np.arange(s.n_kb), s.rows)
    o_ref, lse_ref = O.masked_attention(qo, ko, vo, g, WL.q_block, 64, rpn, cin, Hp.scale_of(WL))
    Hp.assert_attn_close(out.cpu().double().numpy(), o_ref, signal_guard=False)
    Hp.assert_attn_close(dense.cpu().double().numpy(), o_ref, signal_guard=False)
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= 1e-3
    ref_m = O.block_mass(qo, ko, g, WL.q_block, 64, Hp.scale_of(WL))
    assert np.abs(mass.cpu().double().numpy() - ref_m).max() <= Hp.MASS_ABS
