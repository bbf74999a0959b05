"""Thin Python binding of libbsattn.so (ctypes).

Argument marshalling only: every step of the path runs in the library's CUDA kernels.
PyTorch provides device memory and the current CUDA stream.  There is no fallback: if
the library cannot be loaded every call raises.

Names follow the C ABI in include/bsattn.h:
    tile_permute, tile_permute_quant_e4m3, block_mass, dense_fwd_mass, pooled_mass,
    topp_select, topp_select_noalloc, pattern_csr, bsattn_fwd;
    cluster order: kmeans, cluster_layout, cluster_permute, cluster_mass,
    topp_select_rows, cluster_fwd
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libbsattn.so")

BSA_OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "capacity too small",
                4: "CUDA error", 5: "device wait timed out", 6: "device-side input check failed",
                7: "list file missing, unreadable or corrupt"}
BSA_BF16, BSA_FP32, BSA_E4M3 = 0, 1, 2
OP_BLOCK_MASS, OP_TOPP_SELECT, OP_FWD, OP_PATTERN, OP_POOLED_MASS = 0, 1, 2, 3, 4
PAT_DIAGONAL, PAT_MULTI_DIAGONAL, PAT_VERTICAL_STRIPE, PAT_SURROUNDING, PAT_CRISS_CROSS = 1, 2, 4, 8, 16


class _ClusterShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("batch", "heads", "head_dim", "n_tokens",
                                              "n_q_clusters", "n_k_clusters")]


@dataclass(frozen=True)
class ClusterShape:
    """bsa_cluster_shape: S tokens per (batch, head), clustered separately for queries and keys."""
    batch: int
    heads: int
    head_dim: int
    n_tokens: int
    n_q_clusters: int
    n_k_clusters: int

    def c(self) -> _ClusterShape:
        return _ClusterShape(self.batch, self.heads, self.head_dim, self.n_tokens,
                             self.n_q_clusters, self.n_k_clusters)


class BsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} (status {status})")
        self.status = status


class _Pattern(ctypes.Structure):
    _fields_ = [("kinds", ctypes.c_uint32)] + [(n, ctypes.c_int32) for n in (
        "diag_width", "multi_count", "multi_period", "stripe_stride", "stripe_offset",
        "radius_t", "radius_h", "radius_w")]


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("batch", "heads", "head_dim", "T", "H", "W", "Tp", "Hp", "Wp", "q_block", "kv_block")]


@dataclass(frozen=True)
class Shape:
    """Problem shape; mirrors bsa_shape."""
    batch: int
    heads: int
    head_dim: int
    T: int
    H: int
    W: int
    Tp: int
    Hp: int
    Wp: int
    q_block: int = 64
    kv_block: int = 64

    @classmethod
    def of(cls, wl) -> "Shape":
        return cls(*wl.shape_tuple()) if hasattr(wl, "shape_tuple") else cls(*wl)

    @property
    def S(self):
        return self.T * self.H * self.W

    @property
    def Np(self):
        return self.Tp * self.Hp * self.Wp

    @property
    def n_qb(self):
        return self.Np // self.q_block

    @property
    def n_kb(self):
        return self.Np // self.kv_block

    @property
    def rows(self):
        return self.batch * self.heads * self.n_qb

    def c(self) -> _Shape:
        return _Shape(self.batch, self.heads, self.head_dim, self.T, self.H, self.W,
                      self.Tp, self.Hp, self.Wp, self.q_block, self.kv_block)


_lib_handle = None


def lib() -> ctypes.CDLL:
    """Load libbsattn.so (raises if it has not been built)."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                           "`python -m block_sparse_attention_25_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S, F, L64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_int64
    SP = ctypes.POINTER(_Shape)
    CSP = ctypes.POINTER(_ClusterShape)
    sig = {
        "bsa_workspace_bytes": (S, [SP, I]),
        "bsa_clear_status": (I, [P, P]),
        "bsa_device_status": (I, [P, P]),
        "bsa_device_status_words": (I, [P, ctypes.POINTER(ctypes.c_uint32), P]),
        "bsa_status_string": (ctypes.c_char_p, [I]),
        "bsa_tile_permute": (I, [SP, I, I, P, P, P]),
        "bsa_tile_permute_quant_e4m3": (I, [SP, P, P, P, P]),
        "bsa_block_mass": (I, [SP, P, P, F, P, P, S, P]),
        "bsa_dense_fwd_mass": (I, [SP, P, P, P, F, P, P, P, P, S, P]),
        "bsa_pooled_mass": (I, [SP, P, P, F, P, P, S, P]),
        "bsa_topp_select": (I, [SP, P, F, P, P, L64, P, S, P]),
        "bsa_topp_select_noalloc": (I, [SP, P, F, P, P, L64, P, P]),
        "bsa_pattern_csr": (I, [SP, ctypes.POINTER(_Pattern), P, P, L64, P, S, P]),
        "bsa_fwd": (I, [SP, I, P, P, P, P, P, P, P, P, F, P, P, P, S, P]),
        "bsa_version": (ctypes.c_char_p, []),
        "bsa_kmeans_workspace_bytes": (S, [CSP, I]),
        "bsa_cluster_fwd_workspace_bytes": (S, [CSP]),
        "bsa_topp_rows_workspace_bytes": (S, [L64, I]),
        "bsa_kmeans": (I, [CSP, I, P, I, P, P, P, P, S, P]),
        "bsa_cluster_layout": (I, [CSP, I, P, P, P, P, P, P, S, P]),
        "bsa_cluster_permute": (I, [CSP, I, P, P, P, P]),
        "bsa_cluster_mass": (I, [CSP, P, P, P, P, F, P, P]),
        "bsa_topp_select_rows": (I, [P, L64, I, F, P, P, L64, P, S, P]),
        "bsa_cluster_fwd": (I, [CSP, P, P, P, P, P, P, P, P, P, F, P, P, P, S, P]),
        "bsa_selftest_wait": (I, [P, S, L64, P]),
        "bsa_fwd_raster": (I, [SP, P, P, P, P, P, F, P, P, P, S, P]),
        "bsa_kernel_binary_version": (I, [ctypes.POINTER(ctypes.c_int32)]),
        "bsa_lists_save": (I, [ctypes.c_char_p, SP, F, P, P]),
        "bsa_lists_read_header": (I, [ctypes.c_char_p, SP, ctypes.POINTER(F),
                                      ctypes.POINTER(L64)]),
        "bsa_lists_load": (I, [ctypes.c_char_p, SP, ctypes.POINTER(F), P, P, L64]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib_handle = L
    return L


EXPORTED_SYMBOLS = ("bsa_workspace_bytes", "bsa_clear_status", "bsa_device_status",
                    "bsa_device_status_words", "bsa_status_string", "bsa_tile_permute",
                    "bsa_tile_permute_quant_e4m3", "bsa_block_mass", "bsa_topp_select", "bsa_fwd",
                    "bsa_topp_select_noalloc", "bsa_pattern_csr", "bsa_dense_fwd_mass",
                    "bsa_pooled_mass", "bsa_version", "bsa_kmeans_workspace_bytes",
                    "bsa_cluster_fwd_workspace_bytes", "bsa_topp_rows_workspace_bytes",
                    "bsa_kmeans", "bsa_cluster_layout", "bsa_cluster_permute", "bsa_cluster_mass",
                    "bsa_topp_select_rows", "bsa_cluster_fwd", "bsa_selftest_wait",
                    "bsa_fwd_raster", "bsa_kernel_binary_version", "bsa_lists_save",
                    "bsa_lists_read_header", "bsa_lists_load")


def _check(status: int, what: str):
    if status != BSA_OK:
        raise BsaError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _is_device(t) -> bool:
    return t.is_cuda


def _need(t, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not _is_device(t) or not t.is_contiguous():
        raise ValueError(f"{name}: must be a contiguous CUDA tensor")


def _dev(t, dtype, name, shape=None, min_numel=None):
    """A buffer the library reads or writes through a raw pointer (an output, a workspace, a
    list): of `dtype`, contiguous and on the GPU, and of `shape` or at least `min_numel`
    elements when given -- so a host tensor or a short buffer is refused here instead of
    reaching a kernel.  None passes (an optional output the caller did not ask for)."""
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name}: needs at least {min_numel} elements, has {t.numel()}")
    if not _is_device(t) or not t.is_contiguous():
        raise ValueError(f"{name}: must be a contiguous CUDA tensor")


def workspace_bytes(shape: Shape, op: int) -> int:
    return int(lib().bsa_workspace_bytes(ctypes.byref(shape.c()), op))


def new_workspace(shape: Shape, op: int, device="cuda") -> torch.Tensor:
    """Allocate a workspace for `op` and clear its status header."""
    n = workspace_bytes(shape, op)
    if n == 0:
        raise BsaError(1, "workspace size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _dev(ws, torch.uint8, "ws")
    _check(lib().bsa_clear_status(_ptr(ws), _stream()), "bsa_clear_status")
    return ws


def clear_status(ws: torch.Tensor, stream=None):
    _dev(ws, torch.uint8, "ws")
    _check(lib().bsa_clear_status(_ptr(ws), _stream(stream)), "bsa_clear_status")


def device_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise and return the workspace's device status code (0 = ok)."""
    return int(lib().bsa_device_status(_ptr(ws), _stream(stream)))


def device_status_words(ws: torch.Tensor, stream=None):
    w = (ctypes.c_uint32 * 4)()
    _check(lib().bsa_device_status_words(_ptr(ws), w, _stream(stream)), "bsa_device_status_words")
    return list(w)


def tile_permute(x: torch.Tensor, shape: Shape, inverse: bool = False, out=None, stream=None):
    """Raster [B,S,Hh,D] -> tile-major [B,Hh,Np,D] (inverse=False) or back."""
    dt = {torch.bfloat16: BSA_BF16, torch.float32: BSA_FP32}.get(x.dtype)
    if dt is None:
        raise TypeError("tile_permute: bf16 or fp32")
    raster = (shape.batch, shape.S, shape.heads, shape.head_dim)
    tiled = (shape.batch, shape.heads, shape.Np, shape.head_dim)
    src_shape, dst_shape = (tiled, raster) if inverse else (raster, tiled)
    _need(x, x.dtype, src_shape, "src")
    if out is None:
        out = torch.empty(dst_shape, dtype=x.dtype, device=x.device)
    _need(out, x.dtype, dst_shape, "dst")
    _check(lib().bsa_tile_permute(ctypes.byref(shape.c()), dt, int(bool(inverse)), _ptr(x),
                                  _ptr(out), _stream(stream)), "bsa_tile_permute")
    return out


def tile_permute_quant_e4m3(x: torch.Tensor, shape: Shape, out=None, scales=None, stream=None):
    """Raster bf16 -> (tile-major e4m3 codes uint8 [B,Hh,Np,D], fp32 scales [B,Hh,Np/64])."""
    _need(x, torch.bfloat16, (shape.batch, shape.S, shape.heads, shape.head_dim), "src")
    if out is None:
        out = torch.empty((shape.batch, shape.heads, shape.Np, shape.head_dim), dtype=torch.uint8,
                          device=x.device)
    if scales is None:
        scales = torch.empty((shape.batch, shape.heads, shape.Np // 64), dtype=torch.float32,
                             device=x.device)
    _dev(out, torch.uint8, "dst", (shape.batch, shape.heads, shape.Np, shape.head_dim))
    _dev(scales, torch.float32, "scales", (shape.batch, shape.heads, shape.Np // 64))
    _check(lib().bsa_tile_permute_quant_e4m3(ctypes.byref(shape.c()), _ptr(x), _ptr(out),
                                             _ptr(scales), _stream(stream)),
           "bsa_tile_permute_quant_e4m3")
    return out, scales


def default_scale(shape: Shape) -> float:
    return 1.0 / math.sqrt(shape.head_dim)


def block_mass(q, k, shape: Shape, softmax_scale=None, out=None, ws=None, stream=None):
    """Exact block masses fp32 [B,Hh,Np/q_block,Np/64] of tile-major bf16 q, k."""
    tiled = (shape.batch, shape.heads, shape.Np, shape.head_dim)
    _need(q, torch.bfloat16, tiled, "q")
    _need(k, torch.bfloat16, tiled, "k")
    if out is None:
        out = torch.empty((shape.batch, shape.heads, shape.n_qb, shape.n_kb), dtype=torch.float32,
                          device=q.device)
    if ws is None:
        ws = new_workspace(shape, OP_BLOCK_MASS, q.device)
    _dev(out, torch.float32, "mass", (shape.batch, shape.heads, shape.n_qb, shape.n_kb))
    _dev(ws, torch.uint8, "ws")
    scale = default_scale(shape) if softmax_scale is None else float(softmax_scale)
    _check(lib().bsa_block_mass(ctypes.byref(shape.c()), _ptr(q), _ptr(k), scale, _ptr(out),
                                _ptr(ws), ws.numel(), _stream(stream)), "bsa_block_mass")
    return out


def dense_fwd_mass(q, k, v, shape: Shape, softmax_scale=None, want_lse=False, out=None, lse=None,
                   mass=None, ws=None, stream=None):
    """bsa_dense_fwd_mass: dense attention output and exact block masses in one call.
    Returns (out, mass) or (out, mass, lse)."""
    tiled = (shape.batch, shape.heads, shape.Np, shape.head_dim)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, tiled, n)
    if out is None:
        out = torch.empty(tiled, dtype=torch.bfloat16, device=q.device)
    if mass is None:
        mass = torch.empty((shape.batch, shape.heads, shape.n_qb, shape.n_kb), dtype=torch.float32,
                           device=q.device)
    if want_lse and lse is None:
        lse = torch.empty((shape.batch, shape.heads, shape.Np), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = new_workspace(shape, OP_BLOCK_MASS, q.device)
    _dev(out, torch.bfloat16, "out", tiled)
    _dev(mass, torch.float32, "mass", (shape.batch, shape.heads, shape.n_qb, shape.n_kb))
    _dev(lse, torch.float32, "lse", (shape.batch, shape.heads, shape.Np))
    _dev(ws, torch.uint8, "ws")
    scale = default_scale(shape) if softmax_scale is None else float(softmax_scale)
    _check(lib().bsa_dense_fwd_mass(ctypes.byref(shape.c()), _ptr(q), _ptr(k), _ptr(v), scale,
                                    _ptr(out), _ptr(lse), _ptr(mass), _ptr(ws), ws.numel(),
                                    _stream(stream)), "bsa_dense_fwd_mass")
    return (out, mass, lse) if want_lse else (out, mass)


def pooled_mass(q, k, shape: Shape, softmax_scale=None, out=None, ws=None, stream=None):
    """bsa_pooled_mass: block-level estimate of the block masses (feed to topp_select)."""
    tiled = (shape.batch, shape.heads, shape.Np, shape.head_dim)
    _need(q, torch.bfloat16, tiled, "q")
    _need(k, torch.bfloat16, tiled, "k")
    if out is None:
        out = torch.empty((shape.batch, shape.heads, shape.n_qb, shape.n_kb), dtype=torch.float32,
                          device=q.device)
    if ws is None:
        ws = new_workspace(shape, OP_POOLED_MASS, q.device)
    _dev(out, torch.float32, "mass_est", (shape.batch, shape.heads, shape.n_qb, shape.n_kb))
    _dev(ws, torch.uint8, "ws")
    scale = default_scale(shape) if softmax_scale is None else float(softmax_scale)
    _check(lib().bsa_pooled_mass(ctypes.byref(shape.c()), _ptr(q), _ptr(k), scale, _ptr(out),
                                 _ptr(ws), ws.numel(), _stream(stream)), "bsa_pooled_mass")
    return out


def topp_select(mass, shape: Shape, threshold: float = 0.99, col_capacity=None, ws=None,
                row_ptr=None, col_idx=None, stream=None):
    """CSR (row_ptr int32 [R+1], col_idx int32 [capacity]) of the kept kv blocks.

    col_idx is returned at full capacity (R * n_kb entries by default); the valid prefix
    is row_ptr[-1] entries long.
    """
    R = shape.rows
    _need(mass, torch.float32, (shape.batch, shape.heads, shape.n_qb, shape.n_kb), "mass")
    cap = R * shape.n_kb if col_capacity is None else int(col_capacity)
    if row_ptr is None:
        row_ptr = torch.empty(R + 1, dtype=torch.int32, device=mass.device)
    if col_idx is None:
        col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=mass.device)
    if ws is None:
        ws = new_workspace(shape, OP_TOPP_SELECT, mass.device)
    _dev(row_ptr, torch.int32, "row_ptr", (R + 1,))
    _dev(col_idx, torch.int32, "col_idx", min_numel=cap)
    _dev(ws, torch.uint8, "ws")
    _check(lib().bsa_topp_select(ctypes.byref(shape.c()), _ptr(mass), float(threshold),
                                 _ptr(row_ptr), _ptr(col_idx), cap, _ptr(ws), ws.numel(),
                                 _stream(stream)), "bsa_topp_select")
    return row_ptr, col_idx


def save_lists(path, row_ptr, col_idx, shape: Shape, threshold: float):
    """bsa_lists_save: write frozen lists (device or host int32 tensors) to `path`."""
    rp = row_ptr.detach().to("cpu", torch.int32).contiguous()
    if rp.numel() != shape.rows + 1:
        raise ValueError(f"row_ptr: expected {shape.rows + 1} entries, got {rp.numel()}")
    nnz = int(rp[-1])
    ci = col_idx.detach()[:nnz].to("cpu", torch.int32).contiguous()
    _check(lib().bsa_lists_save(os.fsencode(path), ctypes.byref(shape.c()), float(threshold),
                                _ptr(rp), _ptr(ci) if nnz else None), "bsa_lists_save")


def load_lists(path, shape: Shape, device="cuda"):
    """bsa_lists_load: (row_ptr, col_idx, threshold) from a list file written for `shape`;
    row_ptr and col_idx land on `device` (col_idx holds exactly nnz entries, at least one)."""
    L = lib()
    stored = _Shape()
    tau = ctypes.c_float(0.0)
    nnz = ctypes.c_int64(0)
    _check(L.bsa_lists_read_header(os.fsencode(path), ctypes.byref(stored), ctypes.byref(tau),
                                   ctypes.byref(nnz)), "bsa_lists_read_header")
    # refuse a file for another shape before sizing any buffer from its header
    if bytes(stored) != bytes(shape.c()):
        raise BsaError(1, "bsa_lists_load: the file holds lists of another shape")
    if not 0 <= nnz.value <= shape.rows * shape.n_kb:
        raise BsaError(7, "bsa_lists_load: entry count out of range")
    rp = torch.empty(shape.rows + 1, dtype=torch.int32)
    ci = torch.zeros(max(nnz.value, 1), dtype=torch.int32)
    _check(L.bsa_lists_load(os.fsencode(path), ctypes.byref(shape.c()), ctypes.byref(tau),
                            _ptr(rp), _ptr(ci), nnz.value), "bsa_lists_load")
    return rp.to(device), ci.to(device), float(tau.value)


def topp_select_noalloc(mass, shape: Shape, threshold: float = 0.99, row_ptr=None, col_idx=None,
                        col_capacity=None, status=None, stream=None):
    """bsa_topp_select_noalloc: the same selection with the library's own fixed scratch (for
    callers that cannot provide a workspace).  status: optional int32/uint32 CUDA tensor of
    4 words receiving the device-side flags."""
    R = shape.rows
    _need(mass, torch.float32, (shape.batch, shape.heads, shape.n_qb, shape.n_kb), "mass")
    cap = R * shape.n_kb if col_capacity is None else int(col_capacity)
    if row_ptr is None:
        row_ptr = torch.empty(R + 1, dtype=torch.int32, device=mass.device)
    if col_idx is None:
        col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=mass.device)
    _dev(row_ptr, torch.int32, "row_ptr", (R + 1,))
    _dev(col_idx, torch.int32, "col_idx", min_numel=cap)
    if status is not None:
        _dev(status, status.dtype, "status", min_numel=4)
        if status.dtype not in (torch.int32, torch.uint32):
            raise TypeError("status: int32 or uint32")
    _check(lib().bsa_topp_select_noalloc(ctypes.byref(shape.c()), _ptr(mass), float(threshold),
                                         _ptr(row_ptr), _ptr(col_idx), cap, _ptr(status),
                                         _stream(stream)), "bsa_topp_select_noalloc")
    return row_ptr, col_idx


def pattern_csr(shape: Shape, kinds: int, diag_width=0, multi_count=0, multi_period=0,
                stripe_stride=0, stripe_offset=0, radius=(0, 0, 0), col_capacity=None, ws=None,
                row_ptr=None, col_idx=None, device="cuda", stream=None):
    """bsa_pattern_csr: static structured kv-block lists (union of the enabled kinds)."""
    R = shape.rows
    cap = R * shape.n_kb if col_capacity is None else int(col_capacity)
    if row_ptr is None:
        row_ptr = torch.empty(R + 1, dtype=torch.int32, device=device)
    if col_idx is None:
        col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=device)
    if ws is None:
        ws = new_workspace(shape, OP_PATTERN, device)
    _dev(row_ptr, torch.int32, "row_ptr", (R + 1,))
    _dev(col_idx, torch.int32, "col_idx", min_numel=cap)
    _dev(ws, torch.uint8, "ws")
    pat = _Pattern(int(kinds), diag_width, multi_count, multi_period, stripe_stride, stripe_offset,
                   *radius)
    _check(lib().bsa_pattern_csr(ctypes.byref(shape.c()), ctypes.byref(pat), _ptr(row_ptr),
                                 _ptr(col_idx), cap, _ptr(ws), ws.numel(), _stream(stream)),
           "bsa_pattern_csr")
    return row_ptr, col_idx


def bsattn_fwd_raster(q, k, v, row_ptr, col_idx, shape: Shape, softmax_scale=None,
                      want_lse=False, out=None, lse=None, ws=None, stream=None):
    """bsa_fwd_raster: block-sparse attention on raster bf16 [B, S, Hh, D] (the tile
    permutation fused into the kernel).  Returns out (raster) or (out, lse [B, Hh, S])."""
    raster = (shape.batch, shape.S, shape.heads, shape.head_dim)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, raster, n)
    _need(row_ptr, torch.int32, (shape.rows + 1,), "row_ptr")
    _dev(col_idx, torch.int32, "col_idx")
    if out is None:
        out = torch.empty(raster, dtype=torch.bfloat16, device=q.device)
    if want_lse and lse is None:
        lse = torch.empty((shape.batch, shape.heads, shape.S), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = new_workspace(shape, OP_FWD, q.device)
    _dev(out, torch.bfloat16, "out", raster)
    _dev(lse, torch.float32, "lse", (shape.batch, shape.heads, shape.S))
    _dev(ws, torch.uint8, "ws")
    scale = default_scale(shape) if softmax_scale is None else float(softmax_scale)
    _check(lib().bsa_fwd_raster(ctypes.byref(shape.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr),
                                _ptr(col_idx), scale, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                _stream(stream)), "bsa_fwd_raster")
    return (out, lse) if want_lse else out


def bsattn_fwd(q, k, v, row_ptr, col_idx, shape: Shape, softmax_scale=None, scales=None,
               want_lse=False, out=None, lse=None, ws=None, stream=None):
    """Block-sparse attention over CSR lists.  bf16 q/k/v, or e4m3 codes (uint8) with
    scales=(q_scales, k_scales, v_scales).  Returns out (bf16 tile-major) or (out, lse)."""
    tiled = (shape.batch, shape.heads, shape.Np, shape.head_dim)
    fp8 = q.dtype == torch.uint8
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.uint8 if fp8 else torch.bfloat16, tiled, n)
    _need(row_ptr, torch.int32, (shape.rows + 1,), "row_ptr")
    _dev(col_idx, torch.int32, "col_idx")
    sq = sk = sv = None
    if fp8:
        if scales is None:
            raise ValueError("e4m3 inputs need per-tile scales")
        sq, sk, sv = scales
        for t, n in ((sq, "q_scales"), (sk, "k_scales"), (sv, "v_scales")):
            _need(t, torch.float32, (shape.batch, shape.heads, shape.Np // 64), n)
    if out is None:
        out = torch.empty(tiled, dtype=torch.bfloat16, device=q.device)
    if want_lse and lse is None:
        lse = torch.empty((shape.batch, shape.heads, shape.Np), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = new_workspace(shape, OP_FWD, q.device)
    _dev(out, torch.bfloat16, "out", tiled)
    _dev(lse, torch.float32, "lse", (shape.batch, shape.heads, shape.Np))
    _dev(ws, torch.uint8, "ws")
    scale = default_scale(shape) if softmax_scale is None else float(softmax_scale)
    _check(lib().bsa_fwd(ctypes.byref(shape.c()), BSA_E4M3 if fp8 else BSA_BF16, _ptr(q), _ptr(k),
                         _ptr(v), _ptr(sq), _ptr(sk), _ptr(sv), _ptr(row_ptr), _ptr(col_idx), scale,
                         _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)), "bsa_fwd")
    return (out, lse) if want_lse else out


# ------------------------------------------------------------------ cluster order
def _i32(t, shape, name):
    _need(t, torch.int32, shape, name)


def kmeans(x, cs: ClusterShape, n_clusters: int, init, rounds: int, labels=None, counts=None,
           ws=None, stream=None):
    """bsa_kmeans on raster bf16 x [B, S, Hh, D].  init (fp32 [B, Hh, C, D]) is updated in
    place to the final centroids.  Returns (centroids, labels int32 [B,Hh,S], counts)."""
    B, Hh, S, D = cs.batch, cs.heads, cs.n_tokens, cs.head_dim
    _need(x, torch.bfloat16, (B, S, Hh, D), "x")
    _need(init, torch.float32, (B, Hh, n_clusters, D), "centroids")
    if labels is None:
        labels = torch.empty((B, Hh, S), dtype=torch.int32, device=x.device)
    if counts is None:
        counts = torch.empty((B, Hh, n_clusters), dtype=torch.int32, device=x.device)
    if ws is None:
        ws = new_cluster_workspace(cs, n_clusters, x.device)
    _dev(labels, torch.int32, "labels", (B, Hh, S))
    _dev(counts, torch.int32, "counts", (B, Hh, n_clusters))
    _dev(ws, torch.uint8, "ws")
    _check(lib().bsa_kmeans(ctypes.byref(cs.c()), int(n_clusters), _ptr(x), int(rounds), _ptr(init),
                            _ptr(labels), _ptr(counts), _ptr(ws), ws.numel(), _stream(stream)),
           "bsa_kmeans")
    return init, labels, counts


def new_cluster_workspace(cs: ClusterShape, n_clusters: int, device="cuda") -> torch.Tensor:
    n = int(lib().bsa_kmeans_workspace_bytes(ctypes.byref(cs.c()), int(n_clusters)))
    if n == 0:
        raise BsaError(1, "cluster workspace size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _dev(ws, torch.uint8, "ws")
    _check(lib().bsa_clear_status(_ptr(ws), _stream()), "bsa_clear_status")
    return ws


def cluster_layout(labels, cs: ClusterShape, n_clusters: int, ws=None, stream=None):
    """bsa_cluster_layout: (counts, starts, token_of_slot, slot_of_token), int32."""
    B, Hh, S = cs.batch, cs.heads, cs.n_tokens
    _i32(labels, (B, Hh, S), "labels")
    dev = labels.device
    counts = torch.empty((B, Hh, n_clusters), dtype=torch.int32, device=dev)
    starts = torch.empty_like(counts)
    tos = torch.empty((B, Hh, S), dtype=torch.int32, device=dev)
    sot = torch.empty_like(tos)
    if ws is None:
        ws = new_cluster_workspace(cs, n_clusters, dev)
    _dev(ws, torch.uint8, "ws")
    _check(lib().bsa_cluster_layout(ctypes.byref(cs.c()), int(n_clusters), _ptr(labels), _ptr(counts),
                                    _ptr(starts), _ptr(tos), _ptr(sot), _ptr(ws), ws.numel(),
                                    _stream(stream)), "bsa_cluster_layout")
    return counts, starts, tos, sot


def cluster_permute(x, cs: ClusterShape, token_of_slot, inverse: bool = False, out=None, stream=None):
    """bsa_cluster_permute: raster [B,S,Hh,D] -> cluster order [B,Hh,S,D], or back."""
    B, Hh, S, D = cs.batch, cs.heads, cs.n_tokens, cs.head_dim
    raster, perm = (B, S, Hh, D), (B, Hh, S, D)
    _need(x, torch.bfloat16, perm if inverse else raster, "src")
    _i32(token_of_slot, (B, Hh, S), "token_of_slot")
    if out is None:
        out = torch.zeros(raster if inverse else perm, dtype=torch.bfloat16, device=x.device)
    _dev(out, torch.bfloat16, "dst", raster if inverse else perm)
    _check(lib().bsa_cluster_permute(ctypes.byref(cs.c()), int(bool(inverse)), _ptr(token_of_slot),
                                     _ptr(x), _ptr(out), _stream(stream)), "bsa_cluster_permute")
    return out


def cluster_mass(cs: ClusterShape, q_centroids, q_counts, k_centroids, k_counts, softmax_scale=None,
                 out=None, stream=None):
    """bsa_cluster_mass: fp32 [B, Hh, Cq, Ck]."""
    B, Hh, D, Cq, Ck = cs.batch, cs.heads, cs.head_dim, cs.n_q_clusters, cs.n_k_clusters
    _need(q_centroids, torch.float32, (B, Hh, Cq, D), "q_centroids")
    _need(k_centroids, torch.float32, (B, Hh, Ck, D), "k_centroids")
    _i32(q_counts, (B, Hh, Cq), "q_counts")
    _i32(k_counts, (B, Hh, Ck), "k_counts")
    if out is None:
        out = torch.empty((B, Hh, Cq, Ck), dtype=torch.float32, device=q_centroids.device)
    _dev(out, torch.float32, "mass", (B, Hh, Cq, Ck))
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    _check(lib().bsa_cluster_mass(ctypes.byref(cs.c()), _ptr(q_centroids), _ptr(q_counts),
                                  _ptr(k_centroids), _ptr(k_counts), scale, _ptr(out),
                                  _stream(stream)), "bsa_cluster_mass")
    return out


def topp_select_rows(mass, threshold: float = 0.99, col_capacity=None, ws=None, row_ptr=None,
                     col_idx=None, stream=None):
    """bsa_topp_select_rows on a [..., cols] fp32 tensor viewed as rows x cols."""
    if mass.dtype != torch.float32 or not _is_device(mass) or not mass.is_contiguous():
        raise TypeError("mass: contiguous float32 CUDA tensor")
    cols = int(mass.shape[-1])
    rows = mass.numel() // cols
    cap = rows * cols if col_capacity is None else int(col_capacity)
    if row_ptr is None:
        row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=mass.device)
    if col_idx is None:
        col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=mass.device)
    if ws is None:
        n = int(lib().bsa_topp_rows_workspace_bytes(rows, cols))
        if n == 0:
            raise BsaError(2, "topp rows workspace size")
        ws = torch.empty(n, dtype=torch.uint8, device=mass.device)
        _dev(ws, torch.uint8, "ws")
        _check(lib().bsa_clear_status(_ptr(ws), _stream()), "bsa_clear_status")
    _dev(row_ptr, torch.int32, "row_ptr", (rows + 1,))
    _dev(col_idx, torch.int32, "col_idx", min_numel=cap)
    _dev(ws, torch.uint8, "ws")
    _check(lib().bsa_topp_select_rows(_ptr(mass), rows, cols, float(threshold), _ptr(row_ptr),
                                      _ptr(col_idx), cap, _ptr(ws), ws.numel(), _stream(stream)),
           "bsa_topp_select_rows")
    return row_ptr, col_idx


def new_cluster_fwd_workspace(cs: ClusterShape, device="cuda") -> torch.Tensor:
    n = int(lib().bsa_cluster_fwd_workspace_bytes(ctypes.byref(cs.c())))
    if n == 0:
        raise BsaError(1, "cluster fwd workspace size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _dev(ws, torch.uint8, "ws")
    _check(lib().bsa_clear_status(_ptr(ws), _stream()), "bsa_clear_status")
    return ws


def cluster_fwd(q, k, v, cs: ClusterShape, q_starts, q_counts, k_starts, k_counts, row_ptr,
                col_idx, softmax_scale=None, want_lse=False, out=None, lse=None, ws=None,
                stream=None):
    """bsa_cluster_fwd: attention in cluster order; returns out (or (out, lse))."""
    B, Hh, S, D, Cq, Ck = cs.batch, cs.heads, cs.n_tokens, cs.head_dim, cs.n_q_clusters, cs.n_k_clusters
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, (B, Hh, S, D), n)
    _i32(q_starts, (B, Hh, Cq), "q_starts")
    _i32(q_counts, (B, Hh, Cq), "q_counts")
    _i32(k_starts, (B, Hh, Ck), "k_starts")
    _i32(k_counts, (B, Hh, Ck), "k_counts")
    _i32(row_ptr, (B * Hh * Cq + 1,), "row_ptr")
    _dev(col_idx, torch.int32, "col_idx")
    if out is None:
        out = torch.empty((B, Hh, S, D), dtype=torch.bfloat16, device=q.device)
    if want_lse and lse is None:
        lse = torch.empty((B, Hh, S), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = new_cluster_fwd_workspace(cs, q.device)
    _dev(out, torch.bfloat16, "out", (B, Hh, S, D))
    _dev(lse, torch.float32, "lse", (B, Hh, S))
    _dev(ws, torch.uint8, "ws")
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    _check(lib().bsa_cluster_fwd(ctypes.byref(cs.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(q_starts),
                                 _ptr(q_counts), _ptr(k_starts), _ptr(k_counts), _ptr(row_ptr),
                                 _ptr(col_idx), scale, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                 _stream(stream)), "bsa_cluster_fwd")
    return (out, lse) if want_lse else out


def selftest_wait(ws, limit_ns: int = 20_000_000, stream=None):
    """bsa_selftest_wait: a bounded wait that must give up (see include/bsattn.h).
    Returns the status header words after the kernel: (flags, detail, ...) and the three
    result words (first wait completed, second wait completed, abort flag seen)."""
    _dev(ws, torch.uint8, "ws")
    _check(lib().bsa_selftest_wait(_ptr(ws), ws.numel(), int(limit_ns), _stream(stream)),
           "bsa_selftest_wait")
    torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
    words = ws[:64].view(torch.int32).cpu().tolist()
    return words[:4], words[8:11]
