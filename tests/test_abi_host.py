"""Host-only checks of the C ABI: the library loads, exports every declared symbol, sizes
workspaces, and rejects bad arguments before launching anything.

Every call here that passes pointers fails host-side validation by construction (bad
shape, null or misaligned pointer, bad threshold, short workspace), so nothing is ever
launched -- these tests are safe with or without a GPU.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsattn.h")


@pytest.fixture(scope="module")
def B():
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    b.lib()
    return b


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"BSA_API\s+[\w\s\*]+?\b(bsa_\w+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_symbols()
    for n in ("bsa_tile_permute", "bsa_block_mass", "bsa_topp_select", "bsa_fwd",
              "bsa_tile_permute_quant_e4m3", "bsa_workspace_bytes", "bsa_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(B):
    out = subprocess.run(["nm", "-D", "--defined-only", B.bsattn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (bsa_\w+)", out))
    missing = [n for n in declared_symbols() if n not in exported]
    assert not missing, missing
    for n in declared_symbols():
        assert hasattr(B.lib(), n)


def test_library_is_built_for_sm100a(B):
    """The build compiles every translation unit for sm_100a only (no PTX fallback); on a
    GPU, test_gpu_failure checks the runtime's own report of the loaded kernels' target."""
    flags = B.build.NVCC_FLAGS
    i = flags.index("-gencode")
    assert flags[i + 1] == "arch=compute_100a,code=sm_100a"
    assert flags.count("-gencode") == 1


WL = dict(batch=1, heads=40, head_dim=128, T=21, H=45, W=80, Tp=24, Hp=48, Wp=80)


def test_workspace_sizes(B):
    s = B.Shape(**WL, q_block=64, kv_block=64)
    R, nkb = s.rows, s.n_kb
    assert B.workspace_bytes(s, B.OP_BLOCK_MASS) >= 256
    assert B.workspace_bytes(s, B.OP_TOPP_SELECT) >= 256 + 4 * R + R * ((nkb + 31) // 32) * 4
    ctas = s.batch * s.heads * ((s.Np + 255) // 256)
    assert B.workspace_bytes(s, B.OP_FWD) >= 256 + 4 * ctas + ctas * nkb * 4
    assert B.workspace_bytes(s, 99) == 0


@pytest.mark.parametrize("bad", [
    dict(head_dim=96), dict(q_block=96), dict(kv_block=128), dict(Tp=22), dict(Tp=20),
    dict(heads=0), dict(W=0),
])
def test_invalid_shapes_have_no_workspace(B, bad):
    kw = dict(WL, q_block=64, kv_block=64)
    kw.update(bad)
    assert B.workspace_bytes(B.Shape(**kw), B.OP_FWD) == 0


def _c(B, **kw):
    d = dict(WL, q_block=64, kv_block=64)
    d.update(kw)
    return ctypes.byref(B.Shape(**d).c())


FAKE = ctypes.c_void_p(0x10000)       # aligned, never dereferenced: every call below fails validation
MISALIGNED = ctypes.c_void_p(0x10008)


def test_rejections_before_launch(B):
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake-pointer validation checks run on hosts without a GPU only")
    L = B.lib()
    n = None
    assert L.bsa_clear_status(n, n) == 1
    assert L.bsa_tile_permute(None, 0, 0, FAKE, FAKE, n) == 1
    assert L.bsa_tile_permute(_c(B), 0, 0, n, FAKE, n) == 1
    assert L.bsa_tile_permute(_c(B), 0, 0, MISALIGNED, FAKE, n) == 1
    assert L.bsa_tile_permute(_c(B), 2, 0, FAKE, FAKE, n) == 2          # e4m3 is not a permute dtype
    assert L.bsa_tile_permute(_c(B), 0, 7, FAKE, FAKE, n) == 1          # inverse must be 0/1
    assert L.bsa_tile_permute(_c(B, head_dim=96), 0, 0, FAKE, FAKE, n) == 2
    assert L.bsa_tile_permute_quant_e4m3(_c(B), FAKE, FAKE, n, n) == 1
    big = 1 << 40
    assert L.bsa_block_mass(_c(B), FAKE, FAKE, 0.088, FAKE, FAKE, 0, n) == 3     # no workspace
    assert L.bsa_block_mass(_c(B), FAKE, FAKE, -1.0, FAKE, FAKE, big, n) == 1    # bad scale
    assert L.bsa_block_mass(_c(B, q_block=96), FAKE, FAKE, 0.088, FAKE, FAKE, big, n) == 2
    # the calibration kernels scale the row max by softmax_scale: it must be finite and > 0
    for sc in (0.0, -1.0, float("nan"), float("inf")):
        assert L.bsa_block_mass(_c(B), FAKE, FAKE, sc, FAKE, FAKE, big, n) == 1
        assert L.bsa_dense_fwd_mass(_c(B), FAKE, FAKE, FAKE, sc, FAKE, n, FAKE, FAKE, big, n) == 1
    dfm = [FAKE, FAKE, FAKE, 0.088, FAKE, n, FAKE, FAKE]  # q, k, v, scale, out, lse, mass, ws
    assert L.bsa_dense_fwd_mass(_c(B), *dfm, 16, n) == 3                          # short workspace
    bad = list(dfm)
    bad[2] = n                                                                    # v missing
    assert L.bsa_dense_fwd_mass(_c(B), *bad, big, n) == 1
    bad = list(dfm)
    bad[5] = ctypes.c_void_p(0x10002)                                             # lse misaligned
    assert L.bsa_dense_fwd_mass(_c(B), *bad, big, n) == 1
    assert L.bsa_dense_fwd_mass(_c(B, head_dim=96), *dfm, big, n) == 2
    assert L.bsa_topp_select(_c(B), FAKE, 1.5, FAKE, FAKE, 10, FAKE, big, n) == 1
    assert L.bsa_topp_select(_c(B), FAKE, 0.0, FAKE, FAKE, 10, FAKE, big, n) == 1
    assert L.bsa_topp_select(_c(B), FAKE, float("nan"), FAKE, FAKE, 10, FAKE, big, n) == 1
    assert L.bsa_topp_select(_c(B), FAKE, 0.99, FAKE, n, 10, FAKE, big, n) == 1  # capacity w/o buffer
    assert L.bsa_topp_select(_c(B), FAKE, 0.99, FAKE, FAKE, 10, FAKE, 16, n) == 3
    args = [FAKE, FAKE, FAKE, n, n, n, FAKE, FAKE, 0.088, FAKE, n, FAKE]
    assert L.bsa_fwd(_c(B), 0, *args, 16, n) == 3                            # short workspace
    assert L.bsa_fwd(_c(B), 2, *args, big, n) == 1                           # e4m3 without scales
    assert L.bsa_fwd(_c(B), 1, *args, big, n) == 2                           # fp32 not an attention dtype
    bad = list(args)
    bad[7] = n                                                               # col_idx missing
    assert L.bsa_fwd(_c(B), 0, *bad, big, n) == 1
    bad = list(args)
    bad[9] = MISALIGNED                                                      # misaligned out
    assert L.bsa_fwd(_c(B), 0, *bad, big, n) == 1
    bad = list(args)
    bad[10] = ctypes.c_void_p(0x10002)                                       # lse not 4-byte aligned
    assert L.bsa_fwd(_c(B), 0, *bad, big, n) == 1
    assert L.bsa_fwd(_c(B, T=30), 0, *args, big, n) == 1                     # T > Tp
    # the raster-layout forward: q, k, v, row_ptr, col_idx, scale, out, lse, ws
    rargs = [FAKE, FAKE, FAKE, FAKE, FAKE, 0.088, FAKE, n, FAKE]
    assert L.bsa_fwd_raster(_c(B), *rargs, 16, n) == 3                      # short workspace
    bad = list(rargs)
    bad[4] = n                                                               # col_idx missing
    assert L.bsa_fwd_raster(_c(B), *bad, big, n) == 1
    bad = list(rargs)
    bad[6] = MISALIGNED                                                      # misaligned out
    assert L.bsa_fwd_raster(_c(B), *bad, big, n) == 1
    bad = list(rargs)
    bad[7] = ctypes.c_void_p(0x10002)                                        # lse not 4-byte aligned
    assert L.bsa_fwd_raster(_c(B), *bad, big, n) == 1
    bad = list(rargs)
    bad[5] = -1.0                                                            # bad scale
    assert L.bsa_fwd_raster(_c(B), *bad, big, n) == 1
    assert L.bsa_fwd_raster(_c(B, T=30), *rargs, big, n) == 1                # T > Tp
    assert L.bsa_fwd_raster(_c(B, head_dim=96), *rargs, big, n) == 2         # unsupported D
    P = B.bsattn._Pattern
    assert L.bsa_pattern_csr(_c(B), None, FAKE, FAKE, 10, FAKE, big, n) == 1
    assert L.bsa_pattern_csr(_c(B), ctypes.byref(P(64)), FAKE, FAKE, 10, FAKE, big, n) == 1
    assert L.bsa_pattern_csr(_c(B), ctypes.byref(P(1, -1)), FAKE, FAKE, 10, FAKE, big, n) == 1
    assert L.bsa_pattern_csr(_c(B), ctypes.byref(P(4, 0, 0, 0, 5, 5)), FAKE, FAKE, 10, FAKE, big,
                             n) == 1                                          # offset >= stride
    assert L.bsa_pattern_csr(_c(B), ctypes.byref(P(1)), FAKE, FAKE, 10, FAKE, 16, n) == 3


def test_misaligned_index_buffers_are_rejected(B):
    """row_ptr and col_idx receive (or supply) int32 words: a pointer that is not 4-byte
    aligned is refused on the host, before it could become a misaligned device access."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake-pointer validation checks run on hosts without a GPU only")
    L = B.lib()
    n = None
    big = 1 << 40
    MIS4 = ctypes.c_void_p(0x10002)
    assert L.bsa_topp_select(_c(B), FAKE, 0.99, MIS4, FAKE, 10, FAKE, big, n) == 1
    assert L.bsa_topp_select(_c(B), FAKE, 0.99, FAKE, MIS4, 10, FAKE, big, n) == 1
    assert L.bsa_topp_select_noalloc(_c(B), FAKE, ctypes.c_float(0.99), MIS4, FAKE,
                                     ctypes.c_int64(10), n, n) == 1
    assert L.bsa_topp_select_noalloc(_c(B), FAKE, ctypes.c_float(0.99), FAKE, MIS4,
                                     ctypes.c_int64(10), n, n) == 1
    args = [FAKE, FAKE, FAKE, n, n, n, MIS4, FAKE, 0.088, FAKE, n, FAKE]
    assert L.bsa_fwd(_c(B), 0, *args, big, n) == 1                           # row_ptr
    args[6], args[7] = FAKE, MIS4
    assert L.bsa_fwd(_c(B), 0, *args, big, n) == 1                           # col_idx
    P = B.bsattn._Pattern
    assert L.bsa_pattern_csr(_c(B), ctypes.byref(P(1)), MIS4, FAKE, 10, FAKE, big, n) == 1
    assert L.bsa_pattern_csr(_c(B), ctypes.byref(P(1)), FAKE, MIS4, 10, FAKE, big, n) == 1


def test_cluster_rejections_before_launch(B):
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake-pointer validation checks run on hosts without a GPU only")
    L = B.lib()
    n = None
    big = 1 << 40

    def cs(**kw):
        d = dict(batch=1, heads=40, head_dim=128, n_tokens=75600, n_q_clusters=256, n_k_clusters=256)
        d.update(kw)
        return ctypes.byref(B.ClusterShape(**d).c())

    # workspace sizes: positive for good shapes, 0 for bad ones
    assert L.bsa_kmeans_workspace_bytes(cs(), 256) > 0
    assert L.bsa_kmeans_workspace_bytes(cs(), 2000) == 0
    assert L.bsa_kmeans_workspace_bytes(cs(head_dim=96), 16) == 0
    assert L.bsa_cluster_fwd_workspace_bytes(cs()) > 0
    assert L.bsa_cluster_fwd_workspace_bytes(cs(n_tokens=0)) == 0
    assert L.bsa_topp_rows_workspace_bytes(100, 5000) == 0
    # k-means
    assert L.bsa_kmeans(cs(), 256, FAKE, 5, FAKE, FAKE, FAKE, FAKE, 16, n) == 3       # short ws
    assert L.bsa_kmeans(cs(), 256, FAKE, 0, FAKE, FAKE, FAKE, FAKE, big, n) == 1      # no round
    assert L.bsa_kmeans(cs(), 1025, FAKE, 5, FAKE, FAKE, FAKE, FAKE, big, n) == 2
    assert L.bsa_kmeans(cs(head_dim=96), 8, FAKE, 5, FAKE, FAKE, FAKE, FAKE, big, n) == 2
    assert L.bsa_kmeans(cs(), 256, MISALIGNED, 5, FAKE, FAKE, FAKE, FAKE, big, n) == 1
    assert L.bsa_kmeans(cs(n_tokens=1 << 25), 8, FAKE, 5, FAKE, FAKE, FAKE, FAKE, big, n) == 2
    # layout, permute, mass
    assert L.bsa_cluster_layout(cs(), 256, FAKE, FAKE, FAKE, n, FAKE, FAKE, big, n) == 1
    assert L.bsa_cluster_layout(cs(), 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, n) == 3
    assert L.bsa_cluster_permute(cs(), 2, FAKE, FAKE, ctypes.c_void_p(0x20000), n) == 1
    assert L.bsa_cluster_permute(cs(), 0, FAKE, FAKE, FAKE, n) == 1                   # in place
    assert L.bsa_cluster_permute(cs(), 0, FAKE, MISALIGNED, ctypes.c_void_p(0x20000), n) == 1
    assert L.bsa_cluster_mass(cs(), FAKE, FAKE, FAKE, FAKE, 0.0, FAKE, n) == 1         # bad scale
    assert L.bsa_cluster_mass(cs(n_k_clusters=0), FAKE, FAKE, FAKE, FAKE, 0.1, FAKE, n) == 1
    # row selection
    assert L.bsa_topp_select_rows(FAKE, 10, 5000, 0.9, FAKE, FAKE, 10, FAKE, big, n) == 2
    assert L.bsa_topp_select_rows(FAKE, 10, 8, 1.5, FAKE, FAKE, 10, FAKE, big, n) == 1
    assert L.bsa_topp_select_rows(FAKE, 10, 8, 0.9, FAKE, n, 10, FAKE, big, n) == 1
    assert L.bsa_topp_select_rows(FAKE, 10, 8, 0.9, FAKE, FAKE, 10, FAKE, 16, n) == 3
    # attention in cluster order
    args = [FAKE] * 9 + [0.088, FAKE, n, FAKE]      # q..col_idx, scale, out, lse, ws
    assert L.bsa_cluster_fwd(cs(), *args, 16, n) == 3
    bad = list(args)
    bad[2] = MISALIGNED
    assert L.bsa_cluster_fwd(cs(), *bad, big, n) == 1
    bad = list(args)
    bad[8] = n                                                                 # col_idx missing
    assert L.bsa_cluster_fwd(cs(), *bad, big, n) == 1
    bad = list(args)
    bad[9] = -1.0
    assert L.bsa_cluster_fwd(cs(), *bad, big, n) == 1
    assert L.bsa_cluster_fwd(cs(head_dim=32), *args, big, n) == 2


def test_selftest_rejections_before_launch(B):
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake-pointer validation checks run on hosts without a GPU only")
    L = B.lib()
    assert L.bsa_selftest_wait(None, 256, 1000000, None) == 1
    assert L.bsa_selftest_wait(FAKE, 100, 1000000, None) == 1           # header does not fit
    assert L.bsa_selftest_wait(MISALIGNED, 256, 1000000, None) == 1
    assert L.bsa_selftest_wait(FAKE, 256, 10, None) == 1                # limit below 1 us
    assert L.bsa_selftest_wait(FAKE, 256, 10**11, None) == 1            # above 10 s


def test_status_strings(B):
    L = B.lib()
    for code in range(8):
        assert L.bsa_status_string(code)
    assert b"sm_100a" in L.bsa_version()


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import block_sparse_attention_25_b200.bsattn as m
    monkeypatch.setattr(m, "_lib_handle", None)
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        m.lib()
