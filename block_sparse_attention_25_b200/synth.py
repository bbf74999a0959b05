"""Seeded synthetic inputs shaped like video-DiT self-attention workloads.

This module only draws numbers. It holds none of the attention method's arithmetic
(no tile permutation, no softmax, no block selection), so both the CUDA path and the
CPU oracle can be fed from it without sharing any computation.

Recipe (a reading of the workload descriptions; the pages fix no data):

* 3D random Fourier features. One map per tensor pair: Omega ~ N(0,1) of shape [3, D],
  phase b ~ U(0, 2*pi)^D and a per-head frequency f_h ~ U(0.5, 4).  For token
  position p = (t, h, w) (integers) the feature is cos(f_h * (p @ Omega) + b),
  normalised to unit L2 norm over D.  Q and K share one map, so q.k carries a
  spatial-locality kernel; V uses its own map.
* X = 0.7 * RFF + 0.3 * N(0, 1), then multiplied by the workload's value scale
  (1/sqrt(128) for the long-sequence workloads), then cast to the storage dtype.
* A re-draw r of a workload (the later denoising steps of the calibrate-then-reuse
  cycle) is X_r = rho * X + sqrt(1 - rho^2) * X'_r with rho = 0.95, where X'_r is an
  independent draw of the same recipe from the stream seed 1000 * seed + r.
* The "local" generator (an auxiliary workload, not one of the five): Q and K are
  LOCAL_GAIN * (RFF + LOCAL_NOISE * N(0, 1)) with the per-head frequency drawn from
  U(LOCAL_FREQ) -- smooth features with little noise, so attention concentrates on a
  spatial neighbourhood spanning several tiles and the retained-mass lists are really
  sparse (about 60% of the kv blocks kept at 0.99, between ~45% and ~85% per head); V
  follows the standard recipe.  With the standard recipe the N(0, 1) term dominates q.k
  and every block's mass is close to uniform, whatever the scale.

The draws use torch's seeded generator on the requested device (MT19937 on the CPU,
Philox on CUDA), so the same seed gives different numbers on different devices;
every comparison feeds one drawn array to both sides.

Layout of every drawn Q/K/V: raster token order, [B, S, Hh, D] with S = T * H * W and
token s = (t * H + h) * W + w.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

__all__ = [
    "Workload", "WORKLOADS", "draw_qkv", "redraw_qkv", "draw_mass_rows",
    "draw_keep_csr", "workload_by_name",
]


@dataclass(frozen=True)
class Workload:
    """Shapes of one attention call over a (T, H, W) video token grid.

    (T, H, W) is the valid grid; (Tp, Hp, Wp) the padded grid (multiples of 4).
    q_block / kv_block are token counts (64 = one 4x4x4 tile, 128 = two tiles).
    """
    name: str
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
    seed: int = 0
    value_scale: float = 1.0
    storage: str = "bf16"            # "fp32" or "bf16"
    taus: tuple = (0.99,)
    redraws: int = 0
    fp8: bool = False
    generator: str = "rff"           # "rff" (the recipe above) or "local"
    # kept fraction that the calibration gives at 0.99 on this workload (measured on the
    # GPU); sizes the seeded lists of the host-side timing sample only
    nominal_kept: float = 0.957
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def S(self) -> int:
        return self.T * self.H * self.W

    @property
    def Np(self) -> int:
        return self.Tp * self.Hp * self.Wp

    @property
    def n_qb(self) -> int:
        return self.Np // self.q_block

    @property
    def n_kb(self) -> int:
        return self.Np // self.kv_block

    @property
    def rows(self) -> int:
        return self.batch * self.heads * self.n_qb

    def shape_tuple(self):
        return (self.batch, self.heads, self.head_dim, self.T, self.H, self.W,
                self.Tp, self.Hp, self.Wp, self.q_block, self.kv_block)

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


_INV_SQRT128 = 1.0 / math.sqrt(128.0)

# The "local" generator of Q and K (see the module docstring).
LOCAL_FREQ = (0.05, 0.3)
LOCAL_NOISE = 0.1
LOCAL_GAIN = 10.0

# The five workloads: a tiny case the oracle finishes in seconds, then three
# video-DiT-shaped long sequences and the FP8 variant of the 720p one.
WORKLOADS = {
    "tiny": Workload("tiny-4x8x8-h2-d64", 1, 2, 64, 4, 8, 8, 4, 8, 8,
                     64, 64, seed=0, value_scale=1.0, storage="fp32"),
    "wan13b_480p": Workload("wan1.3b-480p-21x30x52-h12-d128", 1, 12, 128, 21, 30, 52, 24, 32, 52,
                            64, 64, seed=1, value_scale=_INV_SQRT128),
    "wan14b_720p": Workload("wan14b-720p-21x45x80-h40-d128", 1, 40, 128, 21, 45, 80, 24, 48, 80,
                            64, 64, seed=2, value_scale=_INV_SQRT128, redraws=10),
    "hunyuan_720p": Workload("hunyuan-720p-33x45x80-h24-d128-bq128", 1, 24, 128, 33, 45, 80, 36, 48, 80,
                             128, 64, seed=3, value_scale=_INV_SQRT128, taus=(0.90, 0.95, 0.99)),
    "wan14b_720p_fp8": Workload("wan14b-720p-fp8-e4m3", 1, 40, 128, 21, 45, 80, 24, 48, 80,
                                64, 64, seed=2, value_scale=_INV_SQRT128, redraws=10, fp8=True),
    # auxiliary: the 720p shape with spatially local attention (about 60% kept at 0.99)
    "wan14b_720p_local": Workload("wan14b-720p-local-21x45x80-h40-d128", 1, 40, 128, 21, 45, 80,
                                  24, 48, 80, 64, 64, seed=2, value_scale=1.0, redraws=10,
                                  generator="local", nominal_kept=0.663),
}


def workload_by_name(name: str) -> Workload:
    return WORKLOADS[name]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _positions(wl: Workload, device) -> torch.Tensor:
    t = torch.arange(wl.T, device=device, dtype=torch.float32)
    h = torch.arange(wl.H, device=device, dtype=torch.float32)
    w = torch.arange(wl.W, device=device, dtype=torch.float32)
    tt, hh, ww = torch.meshgrid(t, h, w, indexing="ij")
    return torch.stack([tt.reshape(-1), hh.reshape(-1), ww.reshape(-1)], dim=1)  # [S, 3]


def _rff(pos, omega, phase, freq):
    proj = pos @ omega                                    # [S, D]
    arg = freq.view(1, -1, 1) * proj.unsqueeze(1) + phase.view(1, 1, -1)
    f = torch.cos(arg)                                    # [S, Hh, D]
    return f / f.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def _draw_fp32(wl: Workload, seed: int, device, sharpness: float = 1.0):
    """Q, K, V in fp32, raster layout [B, S, Hh, D], before the storage cast."""
    g = _gen(seed, device)
    D, Hh = wl.head_dim, wl.heads
    pos = _positions(wl, device)
    out = []
    maps = []
    local = wl.generator == "local"
    for m in range(2):  # map 0 shared by Q and K, map 1 for V
        omega = torch.randn(3, D, generator=g, device=device)
        phase = torch.rand(D, generator=g, device=device) * (2.0 * math.pi)
        lo, hi = LOCAL_FREQ if (local and m == 0) else (0.5, 4.0)
        freq = lo + (hi - lo) * torch.rand(Hh, generator=g, device=device)
        maps.append((omega, phase, freq))
    for which in ("q", "k", "v"):
        omega, phase, freq = maps[1 if which == "v" else 0]
        xs = []
        for _b in range(wl.batch):
            rff = _rff(pos, omega, phase, freq)
            noise = torch.randn(rff.shape, generator=g, device=device)
            if local and which != "v":
                xs.append(LOCAL_GAIN * (rff + LOCAL_NOISE * noise))
            else:
                xs.append((0.7 * rff + 0.3 * noise) * wl.value_scale)
        x = torch.stack(xs, 0)
        if which != "v" and sharpness != 1.0:
            x = x * sharpness
        out.append(x)
    return out


def _store(x: torch.Tensor, wl: Workload) -> torch.Tensor:
    return x.to(torch.bfloat16) if wl.storage == "bf16" else x.contiguous()


def draw_qkv(wl: Workload, device="cpu", sharpness: float = 1.0, seed: int | None = None):
    """Draw (q, k, v) for a workload, raster layout [B, S, Hh, D].

    sharpness multiplies Q and K only (it scales every logit by sharpness^2); 1.0 is the
    recipe above.  Returns tensors in the workload's storage dtype.
    """
    s = wl.seed if seed is None else seed
    q, k, v = _draw_fp32(wl, s, device, sharpness)
    return _store(q, wl), _store(k, wl), _store(v, wl)


def redraw_qkv(wl: Workload, r: int, device="cpu", rho: float = 0.95, sharpness: float = 1.0):
    """The r-th correlated re-draw (r >= 1): rho * X + sqrt(1 - rho^2) * X'_r."""
    base = _draw_fp32(wl, wl.seed, device, sharpness)
    fresh = _draw_fp32(wl, 1000 * wl.seed + r, device, sharpness)
    c = math.sqrt(1.0 - rho * rho)
    return tuple(_store(rho * a + c * b, wl) for a, b in zip(base, fresh))


def draw_mass_rows(n_rows: int, n_kb: int, seed: int, kind: str = "dirichlet",
                   zero_frac: float = 0.0) -> torch.Tensor:
    """Synthetic fp32 block-mass rows (each row non-negative, summing to ~1).

    kind: "dirichlet" (spread), "peaked" (few large entries), "ties" (values drawn
    from a handful of levels so many entries tie exactly), "uniform".
    zero_frac: fraction of entries forced to exactly zero.
    """
    g = _gen(seed, "cpu")
    if kind == "dirichlet":
        x = -torch.log(torch.rand(n_rows, n_kb, generator=g, dtype=torch.float64).clamp_min(1e-300))
    elif kind == "peaked":
        x = torch.rand(n_rows, n_kb, generator=g, dtype=torch.float64) ** 12
    elif kind == "ties":
        lv = torch.tensor([1.0, 2.0, 3.0, 5.0], dtype=torch.float64)
        x = lv[torch.randint(0, 4, (n_rows, n_kb), generator=g)]
    elif kind == "uniform":
        x = torch.ones(n_rows, n_kb, dtype=torch.float64)
    else:
        raise ValueError(kind)
    if zero_frac > 0:
        z = torch.rand(n_rows, n_kb, generator=g, dtype=torch.float64) < zero_frac
        x = torch.where(z, torch.zeros_like(x), x)
    s = x.sum(dim=1, keepdim=True)
    x = torch.where(s > 0, x / torch.where(s > 0, s, torch.ones_like(s)), x)
    return x.to(torch.float32)


def draw_keep_csr(n_rows: int, n_kb: int, keep_prob: float, seed: int, empty_rows=()):
    """A seeded random CSR of kept kv-block indices (ascending within each row).

    Each (row, block) is kept independently with probability keep_prob; rows listed in
    empty_rows keep nothing.  Returns (row_ptr int32 [R+1], col_idx int32 [nnz]).
    """
    g = _gen(seed, "cpu")
    keep = torch.rand(n_rows, n_kb, generator=g) < keep_prob
    for r in empty_rows:
        keep[r] = False
    counts = keep.sum(dim=1).to(torch.int64)
    row_ptr = torch.zeros(n_rows + 1, dtype=torch.int64)
    row_ptr[1:] = torch.cumsum(counts, 0)
    col_idx = keep.nonzero()[:, 1]
    return row_ptr.to(torch.int32), col_idx.to(torch.int32)


def draw_cluster_labels(batch: int, heads: int, n_tokens: int, n_clusters: int, seed: int,
                        empty=(), device="cpu") -> torch.Tensor:
    """Seeded cluster labels int32 [B, Hh, S] with uneven cluster sizes (sizes drawn from a
    power-law mixture, so some clusters span several 256-row tiles and others hold a few
    tokens); the clusters in `empty` receive no token."""
    g = _gen(seed, "cpu")
    weights = torch.rand((batch, heads, n_clusters), generator=g, dtype=torch.float64) ** 3 + 1e-3
    for c in empty:
        weights[..., c] = 0.0
    probs = weights / weights.sum(dim=-1, keepdim=True)
    labels = torch.multinomial(probs.view(-1, n_clusters), n_tokens, replacement=True, generator=g)
    return labels.view(batch, heads, n_tokens).to(torch.int32).to(device)


def draw_blobs(batch: int, heads: int, n_tokens: int, n_clusters: int, head_dim: int, seed: int,
               spread: float = 0.02):
    """Tokens in well-separated Gaussian blobs, raster bf16 [B, S, Hh, D], with the blob of
    every token ([B, Hh, S] int64) and initial centroids (one member token of each blob,
    fp32 [B, Hh, C, D]).  Every blob holds at least one token."""
    g = _gen(seed, "cpu")
    centers = 4.0 * torch.randn((batch, heads, n_clusters, head_dim), generator=g)
    ids = torch.randint(0, n_clusters, (batch, heads, n_tokens), generator=g)
    ids[..., :n_clusters] = torch.arange(n_clusters)  # every blob non-empty
    pts = torch.gather(centers, 2, ids[..., None].expand(-1, -1, -1, head_dim))
    pts = pts + spread * torch.randn(pts.shape, generator=g)
    x = pts.permute(0, 2, 1, 3).contiguous().to(torch.bfloat16)   # [B, S, Hh, D]
    xf = x.float().permute(0, 2, 1, 3)                             # the stored values
    init = xf[:, :, :n_clusters, :].contiguous()                   # token c is in blob c
    return x, ids, init
