"""bsa_fwd_raster: block-sparse attention with the 4x4x4 tile permutation fused into the
forward's loads and stores.

The kernel computes on exactly the shared-memory images bsa_fwd sees, so its output must be
bit-identical to bsa_tile_permute(inverse) of bsa_fwd on tile-permuted inputs; it is also
compared with the fp64 oracle directly (oracle attention in tile order, permuted back by the
oracle's own permutation).  Every token row is written (the output starts as NaN), pad slots
never are (the raster tensor has none).
"""
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


def _lse_to_raster(lse_tiles: np.ndarray, g: O.Grid) -> np.ndarray:
    """[B, Hh, Np] slot order -> [B, Hh, S] token order, through the oracle permutation."""
    r = O.permute_inverse(lse_tiles[..., None], g)  # [B, S, Hh, 1]
    return np.ascontiguousarray(r[..., 0].transpose(0, 2, 1))


def _run(B, wl, q, k, v, rp, ci):
    s = B.Shape.of(wl)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    rp_d, ci_d = Hp.csr_to_device(rp, ci, "cuda")
    ws = B.new_workspace(s, B.OP_FWD)
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((s.batch, s.heads, s.S), float("nan"), device="cuda")
    B.bsattn_fwd_raster(qd, kd, vd, rp_d, ci_d, s, want_lse=True, out=out, lse=lse, ws=ws)
    assert B.device_status(ws) == 0, B.device_status_words(ws)
    # the unfused path on the same inputs and lists
    qt, kt, vt = (B.tile_permute(x, s) for x in (qd, kd, vd))
    ws2 = B.new_workspace(s, B.OP_FWD)
    out_t, lse_t = B.bsattn_fwd(qt, kt, vt, rp_d, ci_d, s, want_lse=True, ws=ws2)
    assert B.device_status(ws2) == 0
    back = B.tile_permute(out_t, s, inverse=True)
    torch.cuda.synchronize()
    return s, out, lse, back, lse_t


@pytest.mark.parametrize("wl", WLS, ids=IDS)
@pytest.mark.parametrize("keep", [1.0, 0.5])
def test_raster_bit_identical_to_permuted_fwd(B, wl, keep):
    g = Hp.grid_of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=4.0)
    R = wl.batch * wl.heads * (wl.Np // wl.q_block)
    rp, ci = synth.draw_keep_csr(R, wl.Np // 64, keep, seed=wl.seed + 300,
                                 empty_rows=(0, R - 1))
    s, out, lse, back, lse_t = _run(B, wl, q, k, v, rp.numpy(), ci.numpy())
    assert not torch.isnan(out).any()
    assert torch.equal(out.view(torch.int16), back.view(torch.int16))
    want_lse = _lse_to_raster(lse_t.cpu().double().numpy().reshape(s.batch, s.heads, s.Np), g)
    got_lse = lse.cpu().double().numpy()
    assert not np.isnan(got_lse).any()
    assert np.array_equal(got_lse, want_lse)


@pytest.mark.parametrize("wl", WLS, ids=IDS)
@pytest.mark.parametrize("tau", [0.9, 0.99])
def test_raster_parity_oracle(B, wl, tau):
    g = Hp.grid_of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=6.0)
    qo, ko, vo = (Hp.oracle_tiled(x, g) for x in (q, k, v))
    mass = O.block_mass(qo, ko, g, wl.q_block, 64, Hp.scale_of(wl))
    rp, ci = Hp.csr_from_oracle(mass, tau)
    s, out, lse, _, _ = _run(B, wl, q, k, v, rp, ci)
    o_ref, lse_ref = O.masked_attention(qo, ko, vo, g, wl.q_block, 64, rp, ci, Hp.scale_of(wl))
    o_ref = O.permute_inverse(o_ref, g)
    lse_ref = _lse_to_raster(lse_ref.reshape(s.batch, s.heads, s.Np), g)
    got = out.cpu().double().numpy()
    e = Hp.assert_attn_close(got, o_ref, signal_guard=False)
    lg = lse.cpu().double().numpy()
    fin = np.isfinite(lse_ref)
    assert np.all(np.isneginf(lg[~fin]))
    assert np.abs(lg[fin] - lse_ref[fin]).max() <= 1e-3


def test_raster_empty_lists_write_zeros(B):
    wl = WLS[3]  # batch 2, D = 64
    q, k, v = Hp.draw(wl, value_scale=1.0)
    R = wl.batch * wl.heads * (wl.Np // wl.q_block)
    rp = np.zeros(R + 1, np.int64)
    s, out, lse, back, _ = _run(B, wl, q, k, v, rp, np.zeros(0, np.int64))
    assert torch.all(out == 0)
    assert torch.all(torch.isneginf(lse))


def test_raster_rejects_bad_arguments(B):
    wl = WLS[0]
    s = B.Shape.of(wl)
    q = torch.zeros((s.batch, s.S, s.heads, s.head_dim), dtype=torch.bfloat16, device="cuda")
    rp = torch.zeros(s.rows + 1, dtype=torch.int32, device="cuda")
    ci = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):  # tile-major shape is not the raster one
        B.bsattn_fwd_raster(torch.zeros((s.batch, s.heads, s.Np, s.head_dim),
                                        dtype=torch.bfloat16, device="cuda"), q, q, rp, ci, s)
    ws = B.new_workspace(s, B.OP_FWD)
    small = ws[: ws.numel() // 2]
    with pytest.raises(B.BsaError):
        B.bsattn_fwd_raster(q, q, q, rp, ci, s, ws=small)
