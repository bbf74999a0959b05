"""The bench's computed-pair count against a plain loop over the forward's CTAs (no GPU).

The forward's CTA owns 256 query slots and walks the union of its query blocks' kv lists;
every query block of the CTA pays for every kv block of that union.  `schedule_work` counts
this with tensor ops; here each CTA's union is formed with Python sets.
"""
import torch

from block_sparse_attention_25_b200 import synth
from block_sparse_attention_25_b200.bsattn import Shape
from block_sparse_attention_25_b200.microbench import schedule_work


def _brute(row_ptr, col_idx, s):
    nq = 256 // s.q_block
    rp, ci = row_ptr.tolist(), col_idx.tolist()
    computed = 0
    for bh in range(s.batch * s.heads):
        for c in range(-(-s.n_qb // nq)):
            union = set()
            for qb in range(c * nq, min((c + 1) * nq, s.n_qb)):
                r = bh * s.n_qb + qb
                union.update(ci[rp[r]:rp[r + 1]])
            computed += len(union) * nq
    return rp[-1], computed


def _case(wl, keep_prob, seed):
    s = Shape.of(wl)
    g = torch.Generator().manual_seed(seed)
    keep = torch.rand(s.rows, s.n_kb, generator=g) < keep_prob
    keep[::7] = False                       # some empty rows
    counts = keep.sum(1)
    row_ptr = torch.zeros(s.rows + 1, dtype=torch.int32)
    row_ptr[1:] = counts.cumsum(0)
    col_idx = keep.nonzero()[:, 1].to(torch.int32)
    return s, row_ptr, col_idx


def test_computed_pairs_match_a_loop_over_ctas():
    W = synth.Workload
    shapes = [
        W("sched-6x10x11-h3-bq64", 1, 3, 128, 6, 10, 11, 8, 12, 12, 64, 64, seed=1),  # 4.5 CTAs
        W("sched-3x7x10-b2-h2-bq128", 2, 2, 64, 3, 7, 10, 4, 8, 12, 128, 64, seed=2),  # 1.5 CTAs
    ]
    for wl in shapes:
        for keep_prob, seed in ((0.0, 3), (0.2, 4), (0.6, 5), (1.0, 6)):
            s, rp, ci = _case(wl, keep_prob, seed)
            w = schedule_work(rp, ci, s)
            kept, computed = _brute(rp, ci, s)
            assert w["kept_pairs"] == kept
            assert w["computed_pairs"] == computed, (wl.name, keep_prob)
            assert computed >= kept


def test_identical_lists_in_a_cta_compute_exactly_the_kept_pairs():
    # every query block of a CTA keeps the same blocks: the union adds nothing
    wl = synth.Workload("sched-same-4x8x8-h2", 1, 2, 64, 4, 8, 8, 4, 8, 8, 64, 64, seed=1)
    s = Shape.of(wl)
    nq = 256 // s.q_block
    assert s.n_qb % nq == 0
    g = torch.Generator().manual_seed(9)
    per_cta = torch.rand(s.batch * s.heads * s.n_qb // nq, s.n_kb, generator=g) < 0.5
    keep = per_cta.repeat_interleave(nq, dim=0)
    row_ptr = torch.zeros(s.rows + 1, dtype=torch.int32)
    row_ptr[1:] = keep.sum(1).cumsum(0)
    col_idx = keep.nonzero()[:, 1].to(torch.int32)
    w = schedule_work(row_ptr, col_idx, s)
    assert w["computed_pairs"] == w["kept_pairs"]
