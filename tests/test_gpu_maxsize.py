"""GPU parity at the largest kv-block count the ABI admits (4,096 kv blocks per head).

A 63x62x61-token grid pads to 64x64x64 = 262,144 slots, 4,096 tiles: every row of masses
and every schedule holds the maximum number of kv blocks, with ragged pads in all three
axes.  One head at D = 64 keeps it to ~1 GB on the device.  As at the workload sizes, the
oracle checks sampled block-mass rows and attention rows one by one, and every selection
row through the properties that fix it uniquely; the attention runs on a seeded CSR (no
oracle input comes from the CUDA path).
"""
import math

import numpy as np
import pytest
import torch

import helpers as Hp
from block_sparse_attention_25_b200 import synth
from oracle import bsa_oracle as O
from test_gpu_fullsize import _oracle_row, _selection_properties

pytestmark = pytest.mark.gpu

MAX_WLS = [
    synth.Workload("max-kv-63x62x61-h1-d64-bq64", 1, 1, 64, 63, 62, 61, 64, 64, 64, 64, 64,
                   seed=31, value_scale=1.0),
    synth.Workload("max-kv-63x62x61-h1-d64-bq128", 1, 1, 64, 63, 62, 61, 64, 64, 64, 128, 64,
                   seed=32, value_scale=1.0),
]


@pytest.fixture(scope="module")
def B(cuda_device):
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    return b


@pytest.fixture(scope="module", params=MAX_WLS, ids=[w.name for w in MAX_WLS])
def big(request, B):
    wl = request.param
    s = B.Shape.of(wl)
    assert s.n_kb == 4096  # the ABI's limit
    q, k, v = synth.draw_qkv(wl, device="cuda", sharpness=4.0)
    qt, kt, vt = (B.tile_permute(x, s) for x in (q, k, v))
    del q, k, v
    torch.cuda.synchronize()
    yield wl, s, (qt, kt, vt)
    del qt, kt, vt
    torch.cuda.empty_cache()


def test_block_mass_and_selection_at_max_kv_blocks(B, big):
    wl, s, (qt, kt, _) = big
    g = Hp.grid_of(wl)
    ws = B.new_workspace(s, B.OP_BLOCK_MASS)
    m = B.block_mass(qt, kt, s, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    mc = m.cpu()
    valid = torch.from_numpy(O.valid_slots(g))
    has_q = valid.view(-1, wl.q_block).any(dim=1)
    sums = mc.double().sum(dim=-1)
    assert torch.allclose(sums[..., has_q], torch.ones_like(sums[..., has_q]), atol=1e-4)
    assert torch.all(sums[..., ~has_q] == 0)
    scale = Hp.scale_of(wl)
    qh, kh = (x[0:1, 0:1].cpu().double().numpy() for x in (qt, kt))
    for i in (0, s.n_qb // 3, s.n_qb - 1):  # first, inner and last (ragged) query block
        ref = O.block_mass_row(qh, kh, g, 0, 0, int(i), wl.q_block, 64, scale)
        got = mc[0, 0, i].double().numpy()
        assert np.abs(got - ref).max() <= Hp.MASS_ABS
        nz = ref > 0
        assert (np.abs(got - ref)[nz] / ref[nz]).max() < 1e-3
        assert np.all(got[ref == 0] == 0)
    mrows = mc.numpy().reshape(-1, s.n_kb)
    for tau in (0.9, 0.99):
        ws_t = B.new_workspace(s, B.OP_TOPP_SELECT)
        rp, ci = B.topp_select(m, s, tau, ws=ws_t)
        assert B.device_status(ws_t) == 0
        _selection_properties(mrows, rp.cpu().numpy().astype(np.int64),
                              ci.cpu().numpy().astype(np.int64), tau, s.n_kb)


def test_fwd_at_max_kv_blocks_sampled_rows(B, big):
    wl, s, (qt, kt, vt) = big
    g = Hp.grid_of(wl)
    # half the blocks of every row kept, two rows empty
    rp, ci = synth.draw_keep_csr(s.rows, s.n_kb, 0.5, seed=wl.seed + 1,
                                 empty_rows=(1, s.rows - 1))
    ws = B.new_workspace(s, B.OP_FWD)
    out, lse = B.bsattn_fwd(qt, kt, vt, rp.cuda(), ci.cuda(), s, want_lse=True, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    rp_np, ci_np = rp.numpy().astype(np.int64), ci.numpy().astype(np.int64)
    scale = Hp.scale_of(wl)
    qh, kh, vh = (x[0:1, 0:1].cpu().double().numpy() for x in (qt, kt, vt))
    rng = np.random.default_rng(7)
    slots = rng.integers(0, s.Np, 48).tolist() + [0, wl.q_block + 3, s.Np - 1]
    got_rows, ref_rows = [], []
    for p in slots:
        o_ref, l_ref = _oracle_row(qh, kh, vh, g, wl, 0, s, int(p), rp_np, ci_np, scale)
        got = out[0, 0, p].double().cpu().numpy()
        lg = float(lse[0, 0, p])
        if math.isinf(l_ref):
            assert math.isinf(lg) and lg < 0 and np.all(got == 0)
        else:
            assert abs(lg - l_ref) <= 1e-3
        got_rows.append(got)
        ref_rows.append(o_ref)
    Hp.assert_attn_close(np.stack(got_rows), np.stack(ref_rows), signal_guard=False)
