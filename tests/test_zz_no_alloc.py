"""The allocation-free selection entry point, bsa_topp_select_noalloc.

It exists for callers that cannot hand the library a workspace (a plugin whose host
engine owns all device memory, a latency-critical path that must not hit cudaMalloc's
implicit synchronisation).  Its scratch is a fixed array inside the library, shared by
every call; so the checks below run it several times in a row, on different inputs, and
compare each result bit for bit with the workspace entry point bsa_topp_select (the
selection is integer work, so the tolerance is exact equality).

This file is named to be collected last, so a run that stops at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_25_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda_device):
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    return b


def _noalloc(B, s, mass, tau, cap=None, status=None):
    """Call the C entry point directly through ctypes."""
    R = s.rows
    cap = R * s.n_kb if cap is None else cap
    rp = torch.full((R + 1,), -7, dtype=torch.int32, device="cuda")
    ci = torch.full((max(cap, 1),), -7, dtype=torch.int32, device="cuda")
    st = B.lib().bsa_topp_select_noalloc(
        ctypes.byref(s.c()), ctypes.c_void_p(mass.data_ptr()), ctypes.c_float(tau),
        ctypes.c_void_p(rp.data_ptr()), ctypes.c_void_p(ci.data_ptr()), ctypes.c_int64(cap),
        None if status is None else ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, st
    return rp, ci


def _reference(B, s, mass, tau):
    ws = B.new_workspace(s, B.OP_TOPP_SELECT)
    rp, ci = B.topp_select(mass, s, tau, ws=ws)
    assert B.device_status(ws) == 0
    return rp, ci


def _same(a, b):
    rp_a, ci_a = a
    rp_b, ci_b = b
    assert torch.equal(rp_a, rp_b)
    n = int(rp_a[-1])
    assert torch.equal(ci_a[:n], ci_b[:n])


def _mass(s, seed, kind, zero_frac=0.0):
    m = synth.draw_mass_rows(s.rows, s.n_kb, seed=seed, kind=kind, zero_frac=zero_frac)
    return m.view(s.batch, s.heads, s.n_qb, s.n_kb).cuda()


def test_noalloc_matches_workspace_entry_on_consecutive_calls(B):
    big = B.Shape.of(synth.WORKLOADS["wan14b_720p"])          # 10.6 MB of scratch
    small = B.Shape.of(synth.WORKLOADS["wan13b_480p"].scaled(heads=3))
    calls = [
        (big, _mass(big, 1, "dirichlet", 0.1), 0.99),
        (big, _mass(big, 2, "ties"), 0.9),                     # same shape, new contents
        (small, _mass(small, 3, "peaked"), 0.95),              # smaller shape after a larger one
        (small, _mass(small, 4, "uniform"), 1.0),
    ]
    for s, m, tau in calls:
        got = _noalloc(B, s, m, tau)
        torch.cuda.synchronize()
        _same(got, _reference(B, s, m, tau))


def test_noalloc_status_buffer_and_capacity(B):
    s = B.Shape.of(synth.WORKLOADS["wan13b_480p"].scaled(heads=2))
    m = _mass(s, 5, "dirichlet")
    m[0, 0, 0, 3] = float("nan")                              # flagged as bad input
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    _noalloc(B, s, m, 0.99, status=status)
    torch.cuda.synchronize()
    assert int(status[0]) & 2                                 # DEVICE_INPUT flag
    # a too-small col_idx: row_ptr stays complete, the CAPACITY flag is raised
    m2 = _mass(s, 6, "uniform")
    status.zero_()
    rp, ci = _noalloc(B, s, m2, 1.0, cap=10, status=status)
    torch.cuda.synchronize()
    assert int(status[0]) & 4
    assert int(rp[-1]) == s.rows * s.n_kb
    assert ci[:10].cpu().tolist() == list(range(10))


def test_noalloc_rejects_problems_larger_than_its_array(B):
    s = B.Shape.of(synth.WORKLOADS["wan14b_720p"].scaled(heads=80))  # ~21 MB of scratch
    m = torch.zeros(1, device="cuda")
    st = B.lib().bsa_topp_select_noalloc(
        ctypes.byref(s.c()), ctypes.c_void_p(m.data_ptr()), ctypes.c_float(0.99),
        ctypes.c_void_p(m.data_ptr()), ctypes.c_void_p(m.data_ptr()), ctypes.c_int64(1), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 3                                            # BSA_ERR_CAPACITY, nothing launched
