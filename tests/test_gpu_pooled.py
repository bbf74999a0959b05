"""GPU parity of the pooled (block-level) mass estimate, and of the online selection it
drives (estimate -> top-p -> block-sparse forward) against the oracle pipeline."""
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
def test_pooled_mass_parity(B, wl, sharp):
    g = Hp.grid_of(wl)
    s = B.Shape.of(wl)
    q, k, _ = Hp.draw(wl, value_scale=1.0, sharp=sharp)
    qt, kt = B.tile_permute(q.cuda(), s), B.tile_permute(k.cuda(), s)
    ws = B.new_workspace(s, B.OP_POOLED_MASS)
    est = B.pooled_mass(qt, kt, s, ws=ws)
    assert B.device_status(ws) == 0
    ref = O.pooled_block_mass(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g), g, wl.q_block, 64,
                              Hp.scale_of(wl))
    got = est.cpu().double().numpy()
    assert np.abs(got - ref).max() <= 1e-5
    nz = ref > 1e-6
    assert (np.abs(got - ref)[nz] / ref[nz]).max() < 1e-4
    assert np.all(got[ref == 0] == 0)


@pytest.mark.parametrize("wl", WLS[:3], ids=[w.name for w in WLS[:3]])
def test_online_selection_pipeline(B, wl):
    """Estimate -> select -> attend on the GPU and in the oracle; the selections agree row
    by row except where estimates tie at the cut, and outputs agree on agreeing rows."""
    g = Hp.grid_of(wl)
    s = B.Shape.of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=5.0)
    qt, kt, vt = (B.tile_permute(x.cuda(), s) for x in (q, k, v))
    est = B.pooled_mass(qt, kt, s)
    rp, ci = B.topp_select(est, s, 0.9)
    out = B.bsattn_fwd(qt, kt, vt, rp, ci, s)
    qo, ko, vo = (Hp.oracle_tiled(x, g) for x in (q, k, v))
    ref_est = O.pooled_block_mass(qo, ko, g, wl.q_block, 64, Hp.scale_of(wl))
    rpo, cio = Hp.csr_from_oracle(ref_est, 0.9)
    rpg = rp.cpu().numpy().astype(np.int64)
    cig = ci.cpu().numpy().astype(np.int64)
    same = np.array([np.array_equal(cig[rpg[r]:rpg[r + 1]], cio[rpo[r]:rpo[r + 1]])
                     for r in range(s.rows)])
    assert same.mean() >= 0.95, same.mean()
    o_ref, _ = O.masked_attention(qo, ko, vo, g, wl.q_block, 64, rpo, cio, Hp.scale_of(wl))
    rows = np.repeat(same.reshape(s.batch, s.heads, s.n_qb), wl.q_block, axis=2)
    e = Hp.assert_attn_close(out.cpu().double().numpy()[rows], o_ref[rows], signal_guard=False)
