"""Failure detection on the GPU without a fault: the bounded pipeline wait gives up on a
barrier that nothing completes, reports TIMEOUT through the workspace's status header, and
the CUDA context stays usable for the next calls."""
import math
import time

import numpy as np
import pytest
import torch

import helpers as Hp
from oracle import bsa_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda_device):
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    return b


def test_bounded_wait_gives_up_and_context_stays_usable(B):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    words, res = B.bsattn.selftest_wait(ws, limit_ns=20_000_000)
    elapsed = time.perf_counter() - t0
    assert words[0] & 1                  # TIMEOUT flag
    assert words[1] == 0x1FF             # detail: the self-test's wait
    assert res == [0, 0, 1]              # both waits gave up; the second one saw the abort flag
    assert B.device_status(ws) == 5      # BSA_ERR_TIMEOUT
    assert elapsed < 5.0                 # ended by itself, far inside the 2 s x 8 bound
    B.clear_status(ws)
    assert B.device_status(ws) == 0
    # the context still runs the attention path correctly
    wl = Hp.small_workloads()[0]
    g = Hp.grid_of(wl)
    s = B.Shape.of(wl)
    q, k, v = Hp.draw(wl, value_scale=1.0, sharp=4.0)
    qt, kt, vt = (B.tile_permute(x.cuda(), s) for x in (q, k, v))
    mass = O.block_mass(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g), g, wl.q_block, 64, Hp.scale_of(wl))
    rp, ci = Hp.csr_from_oracle(mass, 0.95)
    rpd, cid = Hp.csr_to_device(rp, ci, "cuda")
    wsf = B.new_workspace(s, B.OP_FWD)
    out = B.bsattn_fwd(qt, kt, vt, rpd, cid, s, ws=wsf)
    assert B.device_status(wsf) == 0
    ref, _ = O.masked_attention(Hp.oracle_tiled(q, g), Hp.oracle_tiled(k, g), Hp.oracle_tiled(v, g),
                                g, wl.q_block, 64, rp, ci, Hp.scale_of(wl))
    e = Hp.assert_attn_close(out.cpu().double().numpy(), ref, signal_guard=False)


def test_repeated_timeouts_leave_the_device_healthy(B):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        B.clear_status(ws)
        words, res = B.bsattn.selftest_wait(ws, limit_ns=5_000_000)
        assert words[0] & 1 and res == [0, 0, 1]
    x = torch.arange(1 << 20, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == float((1 << 20) * ((1 << 20) - 1) / 2)


def test_loaded_kernels_target_sm100(B):
    """The runtime's report for a kernel of the loaded library: built for compute
    capability 10.0 (sm_100a), not JIT-compiled from PTX for another target."""
    import ctypes
    v = ctypes.c_int32(0)
    assert B.lib().bsa_kernel_binary_version(ctypes.byref(v)) == 0
    assert v.value == 100
