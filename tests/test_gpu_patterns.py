"""GPU parity of the static structured patterns (bit-exact against the oracle) and of the
block-sparse forward driven by them."""
import numpy as np
import pytest

import helpers as Hp
from block_sparse_attention_25_b200 import synth
from oracle import bsa_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda_device):
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    return b


CASES = [
    dict(kinds=O.PAT_DIAGONAL, diag_width=2),
    dict(kinds=O.PAT_MULTI_DIAGONAL, diag_width=1, multi_count=2),
    dict(kinds=O.PAT_MULTI_DIAGONAL | O.PAT_DIAGONAL, diag_width=0, multi_count=1, multi_period=5),
    dict(kinds=O.PAT_VERTICAL_STRIPE, stripe_stride=7, stripe_offset=3),
    dict(kinds=O.PAT_SURROUNDING, radius=(1, 1, 2)),
    dict(kinds=O.PAT_CRISS_CROSS),
    dict(kinds=O.PAT_CRISS_CROSS | O.PAT_SURROUNDING | O.PAT_VERTICAL_STRIPE, radius=(0, 1, 1),
         stripe_stride=9),
]
SHAPES = [
    synth.Workload("p-6x10x11-h2-bq64", 1, 2, 128, 6, 10, 11, 8, 12, 12, 64, 64),
    synth.Workload("p-6x10x11-h1-bq128", 2, 1, 64, 6, 10, 11, 8, 12, 12, 128, 64),
]


@pytest.mark.parametrize("wl", SHAPES, ids=[w.name for w in SHAPES])
@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_pattern_csr_bit_exact(B, wl, case):
    s = B.Shape.of(wl)
    g = Hp.grid_of(wl)
    kw = dict(case)
    kinds = kw.pop("kinds")
    rp, ci = B.pattern_csr(s, kinds, **kw)
    rp_ref, ci_ref = O.pattern_csr(g, wl.q_block, wl.batch, wl.heads, kinds, **kw)
    rp_got = rp.cpu().numpy().astype(np.int64)
    assert np.array_equal(rp_got, rp_ref)
    assert np.array_equal(ci[:rp_got[-1]].cpu().numpy().astype(np.int64), ci_ref)


@pytest.mark.parametrize("case", [CASES[1], CASES[4], CASES[6]], ids=["multi", "surround", "union"])
def test_fwd_over_pattern_csr(B, case):
    wl = Hp.small_workloads()[0]
    g = Hp.grid_of(wl)
    s = B.Shape.of(wl)
    kw = dict(case)
    kinds = kw.pop("kinds")
    rp_ref, ci_ref = O.pattern_csr(g, wl.q_block, wl.batch, wl.heads, kinds, **kw)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=4.0)
    qt, kt, vt = (B.tile_permute(x.cuda(), s) for x in (q, k, v))
    rp, ci = B.pattern_csr(s, kinds, **kw)
    out = B.bsattn_fwd(qt, kt, vt, rp, ci, s)
    o_ref, _ = O.masked_attention(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g),
                                  Hp.oracle_tiled(v, g), g, wl.q_block, 64, rp_ref, ci_ref,
                                  Hp.scale_of(wl))
    e = Hp.assert_attn_close(out.cpu().double().numpy(), o_ref, signal_guard=False)
