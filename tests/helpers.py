"""Shared helpers for the GPU parity tests: seeded inputs, oracle calls, comparisons."""
from __future__ import annotations

import math

import numpy as np
import torch

from block_sparse_attention_25_b200 import synth
from oracle import bsa_oracle as O

# Tolerances (bf16 attention output against fp64; masses; FP8 output).
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
MASS_ABS = 1e-4
FP8_MAX_ABS = 6e-2
# Error relative to the largest reference output.  bf16: P and O are rounded to 8
# significant bits (half-ulp 2^-9) -- 2e-2 leaves room for the sums of many such
# roundings.  e4m3: P is rounded to 4 significant bits before PV, a relative step of at
# most 2^-4 per probability; its contribution to an output element is bounded by 2^-4 of
# the probability-weighted |v| of the row, and the test inputs keep the largest output of
# a case within a small factor of that, so the bound is 2^-4 of the largest output.
ATTN_REL_TO_MAX = 2e-2
FP8_REL_TO_MAX = 2.0 ** -4
# A comparison is only meaningful where the reference output is well above the absolute
# tolerance: an all-zero output must fail it.
SIGNAL_FACTOR = 10.0


def grid_of(wl) -> O.Grid:
    return O.Grid(wl.T, wl.H, wl.W, wl.Tp, wl.Hp, wl.Wp)


def small_workloads():
    """Shapes the oracle finishes in seconds that span several CTAs and ragged tails."""
    W = synth.Workload
    return [
        # ragged pads in t, h, w; Np = 1152 -> 4.5 CTAs of 256 rows; 18 kv blocks
        W("ragged-6x10x11-h3-d128-bq64", 1, 3, 128, 6, 10, 11, 8, 12, 12, 64, 64, seed=11),
        # odd kv-block count (9), partial last Q tile, q_block 128 needs Np % 128 == 0
        W("odd-3x9x10-h2-d128-bq64", 1, 2, 128, 3, 9, 10, 4, 12, 12, 64, 64, seed=12),
        W("ragged-6x10x11-h2-d128-bq128", 1, 2, 128, 6, 10, 11, 8, 12, 12, 128, 64, seed=13),
        W("ragged-5x7x9-h2-d64-bq64", 2, 2, 64, 5, 7, 9, 8, 8, 12, 64, 64, seed=14),
        W("whole-pad-tiles-3x4x9-h2-d64-bq128", 1, 2, 64, 3, 4, 9, 8, 4, 12, 128, 64, seed=15),
    ]


def draw(wl, device="cpu", sharp=1.0, value_scale=None):
    """bf16 raster q, k, v (CPU) for a workload; value_scale overrides the recipe's."""
    if value_scale is not None:
        wl = wl.scaled(value_scale=value_scale)
    wl = wl.scaled(storage="bf16")
    return synth.draw_qkv(wl, device=device, sharpness=sharp)


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_tiled(x_raster_bf16: torch.Tensor, g: O.Grid) -> np.ndarray:
    """Oracle permutation of a bf16 raster tensor, as float64."""
    return O.permute_forward(to_np64(x_raster_bf16), g)


def attn_errors(got: np.ndarray, ref: np.ndarray):
    err = np.abs(got - ref)
    scale = max(np.abs(ref).max(), 1e-30)
    return dict(max_abs=float(err.max()), mean_abs=float(err.mean()),
                max_rel_to_max=float(err.max() / scale),
                rms_rel=float(np.sqrt((err ** 2).mean()) / max(np.sqrt((ref ** 2).mean()), 1e-30)))


def assert_attn_close(got: np.ndarray, ref: np.ndarray, fp8: bool = False,
                      signal_guard: bool = True) -> dict:
    """Element-wise check of an attention output against the oracle's.

    bf16: max abs <= ATTN_MAX_ABS, mean abs <= ATTN_MEAN_ABS, max |err| / max |ref| <=
    ATTN_REL_TO_MAX.  e4m3: max abs <= FP8_MAX_ABS and max |err| / max |ref| <=
    FP8_REL_TO_MAX.  With signal_guard the reference's largest output must be at least
    SIGNAL_FACTOR x the absolute bound, so that the absolute bound alone already rejects an
    all-zero output.  The relative bound rejects it in any case (its ratio is 1)."""
    e = attn_errors(got, ref)
    refmax = float(np.abs(ref).max()) if ref.size else 0.0
    e["ref_max"] = refmax
    abs_tol = FP8_MAX_ABS if fp8 else ATTN_MAX_ABS
    if signal_guard:
        assert refmax >= SIGNAL_FACTOR * abs_tol, ("reference output too small to test", e)
    assert refmax > 0.0, ("all-zero reference", e)
    assert e["max_abs"] <= abs_tol, e
    if fp8:
        assert e["max_rel_to_max"] <= FP8_REL_TO_MAX, e
    else:
        assert e["mean_abs"] <= ATTN_MEAN_ABS, e
        assert e["max_rel_to_max"] <= ATTN_REL_TO_MAX, e
    return e


def assert_mass_close(got: np.ndarray, ref: np.ndarray):
    """Block masses against the oracle's: abs error <= MASS_ABS everywhere, relative error
    < 1e-3 wherever the reference exceeds 1e-6, and the structural zeros (pad-only kv
    blocks, query blocks without valid queries) exactly zero."""
    err = np.abs(got - ref)
    assert err.max() <= MASS_ABS, err.max()
    nz = ref > 1e-6
    assert (err[nz] / ref[nz]).max() < 1e-3
    assert np.all(got[ref == 0] == 0)


LSE_ABS = 1e-3  # natural-log units; a dropped share p of a row's mass moves it by -log(1-p)


def assert_fwd_close(got: np.ndarray, lse_got: np.ndarray, o_ref: np.ndarray,
                     lse_ref: np.ndarray, fp8: bool = False):
    """The forward's whole check against the oracle: outputs element-wise
    (assert_attn_close; e4m3 with its signal guard), rows the oracle leaves empty exactly
    zero with log-sum-exp -inf, and every other row's log-sum-exp within LSE_ABS."""
    zero = ~np.isfinite(lse_ref)
    if fp8:
        e = assert_attn_close(got, o_ref, fp8=True)
    else:
        # every row empty: nothing to compare but the exact zeros below
        e = None if zero.all() else assert_attn_close(got, o_ref, signal_guard=False)
    assert np.all(got[zero] == 0)
    assert np.all(np.isneginf(lse_got[zero]))
    if (~zero).any():
        assert np.abs(lse_got[~zero] - lse_ref[~zero]).max() <= LSE_ABS
    return e


def csr_from_oracle(mass64: np.ndarray, tau: float):
    rp, ci = O.topp_select(mass64.astype(np.float32).reshape(-1, mass64.shape[-1]), tau)
    return rp, ci


def csr_to_device(rp, ci, device):
    rp_t = torch.as_tensor(np.asarray(rp, dtype=np.int32), device=device)
    ci_np = np.asarray(ci, dtype=np.int32)
    if ci_np.size == 0:
        ci_np = np.zeros(1, dtype=np.int32)
    return rp_t, torch.as_tensor(ci_np, device=device)


def scale_of(wl) -> float:
    return 1.0 / math.sqrt(wl.head_dim)


def wide_range_keys(wl, q, k, ramp, target_log2=85.0):
    """Keys scaled per kv block so that a row's logits span far more than 64 log2 units.

    ramp "ascending": each column half's first block (kv blocks 0 and 1) at 2% of the rest;
    "descending": a linear ramp from 1 down to 0.02; "odd_blocks": even blocks at 2% of the
    odd ones.  The softmax scale puts the median valid row's max logit at target_log2.
    Returns (tile-major bf16 keys on the CPU, the same as float64, the scale, each valid
    row's block maxima [B, Hh, valid rows, n_kb] in log2 units)."""
    g = grid_of(wl)
    qt64 = oracle_tiled(q, g)
    kt64 = oracle_tiled(k, g)
    n_kb = g.Np // 64
    j = np.arange(n_kb)
    if ramp == "ascending":
        r = np.where(j < 2, 0.02, 1.0)
    elif ramp == "descending":
        r = 1.0 - 0.98 * j / (n_kb - 1)
    elif ramp == "odd_blocks":
        r = np.where(j % 2 == 1, 1.0, 0.02)
    else:
        raise ValueError(ramp)
    kt_bf = torch.from_numpy(kt64 * np.repeat(r, 64)[None, None, :, None]).to(torch.bfloat16)
    kt64 = kt_bf.double().numpy()
    valid = O.valid_slots(g)
    z = np.einsum("bhqd,bhkd->bhqk", qt64, kt64)
    z[..., ~valid] = -np.inf
    scale = target_log2 * math.log(2.0) / float(np.median(z[:, :, valid].max(-1)))
    bmax = (z * (scale / math.log(2.0))).reshape(*z.shape[:3], n_kb, 64).max(-1)[:, :, valid]
    return kt_bf, kt64, scale, bmax

