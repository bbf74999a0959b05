"""The GPU parity comparisons fail on a wrong answer (no GPU needed).

The attention comparisons of the GPU tests go through helpers.assert_attn_close.  Here the
same helper is fed the oracle's outputs for inputs the GPU tests draw on the CPU, with an
all-zero and a perturbed stand-in for the device output: both must be rejected, while the
oracle's output itself (and one rounded to bf16) passes.  For the e4m3 and cluster-order
cases, whose tests also demand a reference output above 10x the absolute bound, the guard
is checked to hold on the very inputs those tests use.
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
