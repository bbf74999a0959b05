"""Pins for the CPU oracle: closed forms, invariants, brute force and library routines.

Every check here compares the oracle with something other than itself, chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand, a missing
pad mask) fails at least one test.  No GPU is used.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import bsa_oracle as O

GRIDS = [
    O.Grid(4, 8, 8, 4, 8, 8),          # exact tiles
    O.Grid(3, 5, 6, 4, 8, 8),          # ragged pads in every dimension
    O.Grid(5, 4, 9, 8, 4, 12),         # one whole pad tile layer in t
    O.Grid(4, 4, 4, 4, 4, 4),          # a single tile
]


# ------------------------------------------------------------------ permutation
@pytest.mark.parametrize("g", GRIDS)
def test_permute_round_trip_identity(g):
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, g.S, 3, 5)).astype(np.float32)
    y = O.permute_forward(x, g)
    assert y.shape == (2, 3, g.Np, 5)
    assert np.array_equal(O.permute_inverse(y, g), x)


@pytest.mark.parametrize("g", GRIDS)
def test_permute_is_bijection_onto_valid_slots(g):
    src = O.tile_slot_source(g)
    valid = src[src >= 0]
    assert valid.size == g.S
    assert np.array_equal(np.sort(valid), np.arange(g.S))
    # pad slots of the forward permutation are exactly zero
    x = np.ones((1, g.S, 1, 1), np.float32)
    y = O.permute_forward(x, g)
    assert np.array_equal(y[0, 0, :, 0] == 1.0, src >= 0)


@pytest.mark.parametrize("g", GRIDS)
def test_every_block_is_one_aligned_4x4x4_cube(g):
    """The 3D tile is the unit: the 64 slots of each block cover one aligned 4x4x4 cube."""
    src = O.tile_slot_source(g)
    for blk in range(g.Np // 64):
        toks = src[blk * 64:(blk + 1) * 64]
        toks = toks[toks >= 0]
        if toks.size == 0:
            continue
        t = toks // (g.H * g.W)
        h = (toks // g.W) % g.H
        w = toks % g.W
        assert len(set((t // 4).tolist())) == 1
        assert len(set((h // 4).tolist())) == 1
        assert len(set((w // 4).tolist())) == 1
        # the cube holds every valid token of its 4x4x4 region
        t0, h0, w0 = 4 * (t[0] // 4), 4 * (h[0] // 4), 4 * (w[0] // 4)
        n_expect = (min(4, g.T - t0) * min(4, g.H - h0) * min(4, g.W - w0))
        assert toks.size == n_expect


def test_tile_grid_is_walked_w_fastest():
    g = O.Grid(4, 8, 8, 4, 8, 8)
    src = O.tile_slot_source(g)
    # block 1 is the next tile along w, block 2 the next along h
    assert src[64] == 4 and src[128] == 4 * 8
    # inside a tile, row-major over (dt, dh, dw): slot 1 is the next token along w, slot 4
    # the next along h, slot 16 the next along t (token index (t * H + h) * W + w)
    assert src[0] == 0 and src[1] == 1 and src[4] == 8 and src[16] == 64
    assert src[63] == (3 * 8 + 3) * 8 + 3


def _block_tile_coords(g):
    """(tile t, tile h, tile w) of every block, read off the raster positions of the
    tokens the permutation puts there (independent of any tile-index arithmetic)."""
    src = O.tile_slot_source(g)
    out = []
    for blk in range(g.Np // 64):
        toks = src[blk * 64:(blk + 1) * 64]
        tok = int(toks[toks >= 0][0])
        out.append((tok // (g.H * g.W) // 4, (tok // g.W) % g.H // 4, tok % g.W // 4))
    return out


# ------------------------------------------------------------------ block mass
def _qk(g, heads=2, D=16, seed=0, scale_qk=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, heads, g.Np, D)) * scale_qk
    k = rng.standard_normal((1, heads, g.Np, D)) * scale_qk
    valid = O.valid_slots(g)
    q[:, :, ~valid] = 0
    k[:, :, ~valid] = 0
    return q, k


@pytest.mark.parametrize("g", GRIDS)
@pytest.mark.parametrize("bq", [64, 128])
def test_mass_rows_sum_to_one_and_pad_blocks_are_zero(g, bq):
    if g.Np % bq:
        pytest.skip("q block does not divide the slots")
    q, k = _qk(g, scale_qk=2.0)
    m = O.block_mass(q, k, g, bq, 64, 0.25)
    valid = O.valid_slots(g)
    for i in range(g.Np // bq):
        has_q = valid[i * bq:(i + 1) * bq].any()
        s = m[0, :, i].sum(axis=-1)
        if has_q:
            assert np.allclose(s, 1.0, atol=1e-12, rtol=0)
        else:
            assert np.all(m[0, :, i] == 0)
    for j in range(g.Np // 64):
        if not valid[j * 64:(j + 1) * 64].any():
            assert np.all(m[..., j] == 0)


@pytest.mark.parametrize("g", GRIDS)
def test_mass_uniform_attention_closed_form(g):
    """Identical keys give uniform attention: mass(i, j) = valid keys in j / all valid keys."""
    rng = np.random.default_rng(1)
    q = rng.standard_normal((1, 1, g.Np, 8))
    k = np.tile(rng.standard_normal(8), (1, 1, g.Np, 1))
    m = O.block_mass(q, k, g, 64, 64, 0.7)
    valid = O.valid_slots(g)
    nvk = np.array([valid[j * 64:(j + 1) * 64].sum() for j in range(g.Np // 64)], float)
    for i in range(g.Np // 64):
        if valid[i * 64:(i + 1) * 64].any():
            assert np.allclose(m[0, 0, i], nvk / nvk.sum(), atol=1e-13, rtol=0)


def test_mass_one_hot_attention_closed_form():
    """Queries aimed at one key colour: mass counts where that colour's keys sit.

    Key t has colour c(t) (one-hot direction); query p is c * e_{a(p)} with a large c,
    so each query splits its attention evenly over the valid keys of colour a(p).
    """
    g = O.Grid(3, 7, 8, 4, 8, 8)
    D = 64
    rng = np.random.default_rng(2)
    valid = O.valid_slots(g)
    colour = rng.integers(0, D, g.Np)
    aim = rng.integers(0, D, g.Np)
    k = np.zeros((1, 1, g.Np, D))
    k[0, 0, np.arange(g.Np), colour] = 1.0
    q = np.zeros((1, 1, g.Np, D))
    q[0, 0, np.arange(g.Np), aim] = 400.0
    q[:, :, ~valid] = 0
    k[:, :, ~valid] = 0
    # make every aimed colour present among valid keys
    present = set(colour[valid].tolist())
    aim = np.array([a if a in present else next(iter(present)) for a in aim])
    q[:] = 0
    q[0, 0, np.arange(g.Np), aim] = 400.0
    q[:, :, ~valid] = 0
    m = O.block_mass(q, k, g, 64, 64, 1.0)
    n_kb = g.Np // 64
    expect = np.zeros((g.Np // 64, n_kb))
    for i in range(g.Np // 64):
        qs = [p for p in range(i * 64, (i + 1) * 64) if valid[p]]
        for p in qs:
            keys = [t for t in range(g.Np) if valid[t] and colour[t] == aim[p]]
            for t in keys:
                expect[i, t // 64] += 1.0 / len(keys)
        if qs:
            expect[i] /= len(qs)
    assert np.allclose(m[0, 0], expect, atol=1e-12, rtol=0)


def test_mass_single_block_is_one():
    g = O.Grid(4, 4, 4, 4, 4, 4)
    q, k = _qk(g, heads=3, D=8, scale_qk=3.0)
    m = O.block_mass(q, k, g, 64, 64, 1.0)
    assert m.shape == (1, 3, 1, 1)
    assert np.allclose(m, 1.0, atol=1e-14, rtol=0)


def test_mass_matches_torch_softmax_block_sums():
    """Library routine: torch.softmax over the masked logit matrix, then block sums."""
    g = O.Grid(3, 5, 6, 4, 8, 8)
    q, k = _qk(g, heads=1, D=16, scale_qk=1.5, seed=4)
    valid = torch.from_numpy(O.valid_slots(g))
    m = O.block_mass(q, k, g, 128, 64, 0.3)
    logits = 0.3 * torch.from_numpy(q[0, 0]) @ torch.from_numpy(k[0, 0]).T
    logits[:, ~valid] = -math.inf
    p = torch.softmax(logits, dim=1)
    p[~valid] = 0
    per_block = p.reshape(g.Np, g.Np // 64, 64).sum(-1)           # [queries, kv blocks]
    per_qb = per_block.reshape(g.Np // 128, 128, -1).sum(1)
    nvq = valid.reshape(-1, 128).sum(1, keepdim=True).to(torch.float64)
    ref = torch.where(nvq > 0, per_qb / nvq.clamp_min(1), torch.zeros_like(per_qb))
    assert np.allclose(m[0, 0], ref.numpy(), atol=1e-13, rtol=0)


# ------------------------------------------------------------------ top-p selection
def _brute_force_check(m_row, tau, kept):
    q = O.fixed_point_masses(m_row)
    total = int(q.sum())
    target = O.topp_target(total, tau)
    kept = [int(j) for j in kept]
    assert kept == sorted(kept) and len(set(kept)) == len(kept)
    assert sum(int(q[j]) for j in kept) >= target
    n = len(q)
    best = None
    for r in range(0, n + 1):
        sets = [c for c in itertools.combinations(range(n), r)
                if sum(int(q[j]) for j in c) >= target]
        if sets:
            best = sets
            break
    # minimal cardinality
    assert len(kept) == len(best[0])
    # maximum mass among the minimal sets
    best_mass = max(sum(int(q[j]) for j in c) for c in best)
    assert sum(int(q[j]) for j in kept) == best_mass
    # ties resolved toward lower indices: lexicographically smallest among max-mass sets
    cands = sorted(c for c in best if sum(int(q[j]) for j in c) == best_mass)
    assert tuple(kept) == cands[0]


@pytest.mark.parametrize("seed", range(12))
def test_topp_minimal_by_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(4, 15))
    kind = seed % 3
    if kind == 0:
        m = rng.dirichlet(np.ones(n))
    elif kind == 1:
        m = rng.dirichlet(np.full(n, 0.3))
    else:
        m = rng.choice([0.0, 0.1, 0.2, 0.3], size=n)     # exact ties and zeros
        m = m / max(m.sum(), 1e-30)
    m = m.astype(np.float32)
    for tau in (0.5, 0.9, 0.99, 1.0):
        _brute_force_check(m, tau, O.topp_select_row(m, tau))


def test_topp_uniform_closed_form():
    for n in (4, 7, 16, 1440):
        m = np.full(n, 1.0 / n, np.float32)
        q = int(O.fixed_point_masses(m)[0])
        for tau in (0.5, 0.9, 0.99, 1.0):
            target = math.ceil(float(np.float32(tau)) * (q * n))
            k = -(-target // q)
            kept = O.topp_select_row(m, tau)
            assert kept.tolist() == list(range(k))


def test_topp_zero_row_and_tau_one():
    assert O.topp_select_row(np.zeros(9, np.float32), 0.99).size == 0
    m = np.array([0.0, 0.25, 0.0, 0.5, 0.25], np.float32)
    assert O.topp_select_row(m, 1.0).tolist() == [1, 3, 4]


def test_topp_hand_examples():
    # dyadic masses are exact in float32 and sum to exactly 1
    m = np.array([0.0625, 0.5, 0.125, 0.3125], np.float32)
    assert O.topp_select_row(m, 0.5).tolist() == [1]
    assert O.topp_select_row(m, 0.8).tolist() == [1, 3]
    assert O.topp_select_row(m, 0.82).tolist() == [1, 2, 3]
    assert O.topp_select_row(m, 0.99).tolist() == [0, 1, 2, 3]
    # equal masses: the lower index wins
    m = np.array([0.125, 0.375, 0.125, 0.375], np.float32)
    assert O.topp_select_row(m, 0.8).tolist() == [0, 1, 3]
    # float32 rounding counts: 0.05 + 0.5 + 0.15 + 0.3 stored in float32 sums above 1,
    # so 0.5 is just short of half the total
    m = np.array([0.05, 0.5, 0.15, 0.3], np.float32)
    assert O.topp_select_row(m, 0.5).tolist() == [1, 3]
    # the kept mass must reach tau of the total, not just its integer part: masses 3, 2, 2
    # units of 2^-40 and a threshold just above 3/7 need 3.00000x units, so block 0 alone
    # (3 units) is not enough
    m = np.array([3, 2, 2], np.float32) * np.float32(2.0 ** -40)
    tau = np.nextafter(np.float32(3 / 7), np.float32(1))
    assert float(tau) * 7 > 3
    assert O.topp_select_row(m, tau).tolist() == [0, 1]
    # the threshold is the float32 value: 0.9 as float32 is 0.899999976..., which the top
    # block here holds exactly, so it is kept alone (a float64 0.9 would need both blocks)
    t32 = np.float32(0.9)
    m = np.array([t32, np.float32(1.0) - t32], np.float32)
    assert float(m[0]) + float(m[1]) == 1.0 and float(t32) < 0.9
    assert O.topp_select_row(m, 0.9).tolist() == [0]
    assert O.topp_select_row(m, np.float32(0.9)).tolist() == [0]


def test_fixed_point_masses_round_half_to_even():
    """q = m * 2^40 rounded to the nearest integer, halves to even; values hand-computed
    from float32 masses whose scaled value has a fractional part."""
    u = 2.0 ** -40
    m = np.array([0.25 * u, 0.5 * u, 0.75 * u, 1.5 * u, 2.5 * u, 3.0 * u, 1.0], np.float32)
    assert O.fixed_point_masses(m).tolist() == [0, 0, 1, 2, 2, 3, 2 ** 40]


def test_topp_target_is_the_exact_ceiling_where_the_product_is_exact():
    """For totals below 2^29 the float32 threshold times the total is exact in float64, so
    the target is the exact rational ceiling of tau * total."""
    from fractions import Fraction
    rng = np.random.default_rng(11)
    for _ in range(2000):
        total = int(rng.integers(0, 2 ** 29))
        tau = np.float32(rng.uniform(0.0, 1.0))
        exact = Fraction(float(tau)) * total
        want = exact.numerator // exact.denominator + (exact.denominator != 1 and exact > 0)
        assert O.topp_target(total, tau) == want
    for total, tau, want in ((7, 0.5, 4), (8, 0.5, 4), (10, 1.0, 10), (0, 0.99, 0)):
        assert O.topp_target(total, tau) == want


def test_topp_rejects_bad_masses():
    with pytest.raises(ValueError):
        O.topp_select_row(np.array([0.5, -0.1], np.float32), 0.9)
    with pytest.raises(ValueError):
        O.topp_select_row(np.array([0.5, np.nan], np.float32), 0.9)


# ------------------------------------------------------------------ masked attention
def _qkv(g, heads=2, D=16, seed=0, s=1.0):
    rng = np.random.default_rng(seed)
    out = [rng.standard_normal((1, heads, g.Np, D)) * s for _ in range(3)]
    valid = O.valid_slots(g)
    for x in out:
        x[:, :, ~valid] = 0
    return out


def _full_csr(R, n_kb):
    row_ptr = np.arange(R + 1) * n_kb
    col_idx = np.tile(np.arange(n_kb), R)
    return row_ptr, col_idx


@pytest.mark.parametrize("g", GRIDS[:3])
@pytest.mark.parametrize("bq", [64, 128])
def test_attention_full_csr_equals_sdpa(g, bq):
    if g.Np % bq:
        pytest.skip("q block does not divide the slots")
    q, k, v = _qkv(g, heads=2, D=16, s=1.3)
    n_qb, n_kb = g.Np // bq, g.Np // 64
    rp, ci = _full_csr(2 * n_qb, n_kb)
    o, lse = O.masked_attention(q, k, v, g, bq, 64, rp, ci, 0.4)
    valid = torch.from_numpy(O.valid_slots(g))
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=valid.view(1, 1, 1, -1), scale=0.4)
    ref[:, :, ~valid] = 0
    assert np.allclose(o, ref.numpy(), atol=1e-12, rtol=0)
    logits = 0.4 * tq @ tk.transpose(-1, -2)
    logits[..., ~valid] = -math.inf
    ref_lse = torch.logsumexp(logits, dim=-1)
    ref_lse[:, :, ~valid] = -math.inf
    assert np.allclose(lse, ref_lse.numpy(), atol=1e-12, rtol=0)


def test_attention_constant_values_closed_form():
    g = O.Grid(3, 5, 6, 4, 8, 8)
    q, k, _ = _qkv(g, heads=1, D=8, s=2.0)
    v = np.tile(np.arange(8.0), (1, 1, g.Np, 1))
    rp, ci = O.topp_select(np.full((g.Np // 64, g.Np // 64), 1.0 / (g.Np // 64), np.float32), 0.6)
    o, _ = O.masked_attention(q, k, v, g, 64, 64, rp, ci, 1.0)
    valid = O.valid_slots(g)
    assert np.allclose(o[0, 0, valid], np.arange(8.0), atol=1e-12)
    assert np.all(o[0, 0, ~valid] == 0)


def test_attention_single_block_identical_keys_is_block_mean():
    g = O.Grid(3, 5, 6, 4, 8, 8)
    q, _, v = _qkv(g, heads=1, D=8)
    k = np.zeros_like(q)
    valid = O.valid_slots(g)
    n_qb = g.Np // 64
    j = 2
    rp = np.arange(n_qb + 1)
    ci = np.full(n_qb, j)
    o, _ = O.masked_attention(q, k, v, g, 64, 64, rp, ci, 1.0)
    blk = np.arange(j * 64, (j + 1) * 64)
    mean_v = v[0, 0, blk[valid[blk]]].mean(axis=0)
    assert np.allclose(o[0, 0, valid], mean_v, atol=1e-12)


def test_attention_kept_set_renormalises():
    """With two kept blocks, output equals softmax attention restricted to their keys."""
    g = O.Grid(4, 8, 8, 4, 8, 8)
    q, k, v = _qkv(g, heads=1, D=8, s=1.5, seed=7)
    rp = np.array([0, 2, 3, 3, 4])
    ci = np.array([1, 3, 0, 2])
    o, lse = O.masked_attention(q, k, v, g, 64, 64, rp, ci, 0.5)
    tq, tk, tv = (torch.from_numpy(x[0, 0]) for x in (q, k, v))
    for qb, blocks in ((0, [1, 3]), (1, [0]), (3, [2])):
        keys = torch.cat([torch.arange(b * 64, (b + 1) * 64) for b in blocks])
        ref = torch.softmax(0.5 * tq[qb * 64:(qb + 1) * 64] @ tk[keys].T, -1) @ tv[keys]
        assert np.allclose(o[0, 0, qb * 64:(qb + 1) * 64], ref.numpy(), atol=1e-12)
    # query block 2 has an empty list: zeros and -inf
    assert np.all(o[0, 0, 128:192] == 0) and np.all(np.isneginf(lse[0, 0, 128:192]))


# ------------------------------------------------------------------ FP8 e4m3
def test_e4m3_decode_matches_torch():
    tab = O.e4m3_decode_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(tab), nan)
    assert np.array_equal(tab[~nan], ref[~nan])
    assert tab[0x7E] == 448.0 and tab[0x01] == 2.0 ** -9 and tab[0x08] == 2.0 ** -6


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(5)
    tab = O.e4m3_decode_table()
    fin = tab[np.isfinite(tab)]
    mids = ((np.sort(fin)[1:] + np.sort(fin)[:-1]) / 2).astype(np.float32)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 50,
        rng.standard_normal(5000).astype(np.float32) * 0.01,
        mids, -mids, fin.astype(np.float32),
    ])
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(x)
    # torch keeps the sign of zero as well; compare codes exactly
    assert np.array_equal(got, ref)


def test_e4m3_saturates():
    x = np.array([448.0, 449.0, 463.9, 464.0, 1e6, -500.0], np.float32)
    assert O.e4m3_encode(x).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_quant_tiles_scale_and_error_bound():
    rng = np.random.default_rng(6)
    g = O.Grid(3, 5, 6, 4, 8, 8)
    x = rng.standard_normal((1, 2, g.Np, 16)).astype(np.float32) * 0.1
    x[:, :, ~O.valid_slots(g)] = 0
    x[0, 1, 0:64] = 0                                     # an all-zero tile
    codes, scales = O.quant_e4m3_tiles(x)
    tab = O.e4m3_decode_table()
    assert scales[0, 1, 0] == 1.0 and np.all(codes[0, 1, 0:64] == 0)
    vals = tab[codes.astype(np.int64)]
    for h in range(2):
        for t in range(g.Np // 64):
            tile = x[0, h, t * 64:(t + 1) * 64]
            if np.abs(tile).max() == 0:
                continue
            # the largest element maps onto +-448
            assert np.abs(vals[0, h, t * 64:(t + 1) * 64]).max() == 448.0
            assert scales[0, h, t] == np.float32(np.abs(tile).max()) / np.float32(448.0)
    deq = O.dequant_e4m3_tiles(codes, scales)
    s = np.repeat(scales.astype(np.float64), 64, axis=2)[..., None]
    err = np.abs(deq - x.astype(np.float64))
    rel_bound = 2.0 ** -4 * np.abs(x) * (1 + 1e-6) + s * 2.0 ** -10 + 1e-12
    assert np.all(err <= rel_bound)


# ------------------------------------------------------------------ structured patterns
def _rows(rp, ci):
    return [ci[rp[r]:rp[r + 1]].tolist() for r in range(len(rp) - 1)]


def test_pattern_diagonal_band_closed_form():
    g = O.Grid(8, 8, 12, 8, 8, 12)          # 2 x 2 x 3 tiles = 12 blocks
    n = g.Np // 64
    for w in (0, 1, 3):
        rows = _rows(*O.pattern_csr(g, 64, 1, 1, O.PAT_DIAGONAL, diag_width=w))
        for i, r in enumerate(rows):
            assert r == list(range(max(0, i - w), min(n - 1, i + w) + 1))


def test_pattern_diagonal_128_token_query_blocks_cover_both_tiles():
    g = O.Grid(8, 8, 12, 8, 8, 12)
    rows = _rows(*O.pattern_csr(g, 128, 1, 1, O.PAT_DIAGONAL, diag_width=0))
    assert rows == [[2 * i, 2 * i + 1] for i in range(6)]


def test_pattern_multi_diagonal_hits_same_place_in_other_frames():
    g = O.Grid(12, 8, 8, 12, 8, 8)          # 3 temporal layers of 2 x 2 tiles
    rows = _rows(*O.pattern_csr(g, 64, 1, 1, O.PAT_MULTI_DIAGONAL, multi_count=2))
    # layer stride 4: block u also sees u - 8, u - 4, u + 4, u + 8 (within range), not itself
    for u, r in enumerate(rows):
        assert r == sorted(v for v in (u - 8, u - 4, u + 4, u + 8) if 0 <= v < 12)


def test_pattern_vertical_stripes_are_the_same_for_every_row():
    g = O.Grid(8, 8, 12, 8, 8, 12)
    rows = _rows(*O.pattern_csr(g, 64, 2, 3, O.PAT_VERTICAL_STRIPE, stripe_stride=5,
                                stripe_offset=2))
    assert len(rows) == 2 * 3 * 12 and all(r == [2, 7] for r in rows)


def test_pattern_surrounding_counts_closed_form():
    g = O.Grid(12, 12, 12, 12, 12, 12)      # 3 x 3 x 3 tiles
    rows = _rows(*O.pattern_csr(g, 64, 1, 1, O.PAT_SURROUNDING, radius=(1, 1, 1)))
    for u, r in enumerate(rows):
        t, h, w = u // 9, (u // 3) % 3, u % 3
        expect = 1
        for c in (t, h, w):
            expect *= 3 - (c == 0) - (c == 2)   # neighbours along one axis, edges have 2
        assert len(r) == expect
    assert len(rows[13]) == 27                 # the centre tile sees the whole 3x3x3 cube
    rows0 = _rows(*O.pattern_csr(g, 64, 1, 1, O.PAT_SURROUNDING, radius=(0, 0, 0)))
    assert rows0 == [[u] for u in range(27)]


def test_pattern_surrounding_asymmetric_radii_on_a_non_cubic_grid():
    """Radii (0, 1, 2) on 2 x 3 x 4 tiles: the kept set is the box of tiles around the
    query tile, with coordinates taken from the tokens' raster positions."""
    g = O.Grid(7, 11, 14, 8, 12, 16)        # ragged in every axis
    xyz = _block_tile_coords(g)
    rows = _rows(*O.pattern_csr(g, 64, 1, 1, O.PAT_SURROUNDING, radius=(0, 1, 2)))
    for u, r in enumerate(rows):
        tu, hu, wu = xyz[u]
        assert r == [v for v, (tv, hv, wv) in enumerate(xyz)
                     if tv == tu and abs(hv - hu) <= 1 and abs(wv - wu) <= 2]
    assert len(rows[xyz.index((0, 1, 1))]) == 3 * 4


def test_pattern_criss_cross_sets_on_a_non_cubic_grid():
    g = O.Grid(12, 12, 16, 12, 12, 16)      # 3 x 3 x 4 tiles
    xyz = _block_tile_coords(g)
    rows = _rows(*O.pattern_csr(g, 64, 1, 1, O.PAT_CRISS_CROSS))
    for u, r in enumerate(rows):
        assert r == [v for v, c in enumerate(xyz)
                     if sum(int(a == b) for a, b in zip(c, xyz[u])) >= 2]


def test_pattern_criss_cross_is_three_axis_lines():
    g = O.Grid(12, 12, 16, 12, 12, 16)      # 3 x 3 x 4 tiles
    rows = _rows(*O.pattern_csr(g, 64, 1, 1, O.PAT_CRISS_CROSS))
    for r in rows:
        assert len(r) == 1 + 2 + 2 + 3     # itself + other t + other h + other w


def test_pattern_union_of_kinds():
    g = O.Grid(8, 8, 12, 8, 8, 12)
    a = _rows(*O.pattern_csr(g, 64, 1, 1, O.PAT_DIAGONAL, diag_width=1))
    b = _rows(*O.pattern_csr(g, 64, 1, 1, O.PAT_VERTICAL_STRIPE, stripe_stride=4))
    u = _rows(*O.pattern_csr(g, 64, 1, 1, O.PAT_DIAGONAL | O.PAT_VERTICAL_STRIPE,
                             diag_width=1, stripe_stride=4))
    assert u == [sorted(set(x) | set(y)) for x, y in zip(a, b)]


# ------------------------------------------------------------------ pooled estimate
def test_pooled_estimate_is_exact_when_blocks_are_constant():
    """With every key of a block equal (and every query of a block equal), block-level
    attention is exact: the estimate equals the exact block mass."""
    g = O.Grid(3, 5, 6, 4, 8, 8)
    rng = np.random.default_rng(9)
    n_kb = g.Np // 64
    kb = rng.standard_normal((n_kb, 8))
    qb = rng.standard_normal((n_kb, 8)) * 2
    k = np.repeat(kb, 64, axis=0)[None, None]
    q = np.repeat(qb, 64, axis=0)[None, None]
    valid = O.valid_slots(g)
    k = np.where(valid[None, None, :, None], k, 0.0)
    q = np.where(valid[None, None, :, None], q, 0.0)
    est = O.pooled_block_mass(q, k, g, 64, 64, 0.7)
    exact = O.block_mass(q, k, g, 64, 64, 0.7)
    assert np.allclose(est, exact, atol=1e-13, rtol=0)


def test_pooled_estimate_rows_and_zero_scale():
    g = O.Grid(5, 4, 9, 8, 4, 12)
    q, k = _qk(g, heads=2, D=16, scale_qk=1.5, seed=11)
    est = O.pooled_block_mass(q, k, g, 128, 64, 0.4)
    valid = O.valid_slots(g)
    for i in range(g.Np // 128):
        s = est[0, :, i].sum(axis=-1)
        if valid[i * 128:(i + 1) * 128].any():
            assert np.allclose(s, 1.0, atol=1e-12, rtol=0)
        else:
            assert np.all(est[0, :, i] == 0)
    # scale -> 0: every valid key weighs the same, so the estimate is the key-count share
    z = O.pooled_block_mass(q, k, g, 64, 64, 0.0)
    nvk = np.array([valid[j * 64:(j + 1) * 64].sum() for j in range(g.Np // 64)], float)
    for i in range(g.Np // 64):
        if valid[i * 64:(i + 1) * 64].any():
            assert np.allclose(z[0, 0, i], nvk / nvk.sum(), atol=1e-14, rtol=0)
    # a whole temporal layer of pad tiles: its query blocks get all-zero rows and its kv
    # blocks zero mass in every row
    g2 = O.Grid(4, 4, 9, 8, 4, 12)
    q2, k2 = _qk(g2, heads=1, D=8, seed=12)
    e2 = O.pooled_block_mass(q2, k2, g2, 64, 64, 0.4)
    v2 = O.valid_slots(g2)
    empty = [i for i in range(g2.Np // 64) if not v2[i * 64:(i + 1) * 64].any()]
    assert empty == [3, 4, 5]
    for i in empty:
        assert np.all(e2[0, 0, i] == 0) and np.all(e2[0, 0, :, i] == 0)
    for i in range(3):
        assert np.allclose(e2[0, 0, i].sum(), 1.0, atol=1e-12, rtol=0)


# ------------------------------------------------------------------ semantic clusters
def _blobs(seed, n_per, centers, spread):
    """Well-separated Gaussian blobs; returns points, ground-truth ids, one seed point per blob."""
    rng = np.random.default_rng(seed)
    pts, ids = [], []
    for j, c in enumerate(centers):
        pts.append(c + spread * rng.standard_normal((n_per[j], len(c))))
        ids += [j] * n_per[j]
    x = np.concatenate(pts)
    ids = np.array(ids)
    perm = rng.permutation(x.shape[0])
    x, ids = x[perm], ids[perm]
    init = np.stack([x[np.flatnonzero(ids == j)[0]] for j in range(len(centers))])
    return x, ids, init


def test_kmeans_recovers_separated_blobs():
    rng = np.random.default_rng(1)
    centers = 10.0 * rng.standard_normal((5, 16))
    x, ids, init = _blobs(2, [30, 1, 12, 40, 7], centers, 0.05)
    labels, c, counts = O.kmeans_lloyd(x, init, rounds=4)
    assert np.array_equal(labels, ids)
    assert counts.tolist() == [30, 1, 12, 40, 7]
    for j in range(5):   # the centroids are the blob means of the generating partition
        np.testing.assert_allclose(c[j], x[ids == j].mean(axis=0), rtol=0, atol=1e-12)


def test_kmeans_matches_sklearn_lloyd():
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(3)
    x = rng.standard_normal((400, 8))
    init = x[rng.choice(400, 6, replace=False)]
    def fit(rounds):
        return KMeans(n_clusters=6, init=init, n_init=1, max_iter=rounds, tol=0.0,
                      algorithm="lloyd").fit(x)
    for rounds in (2, 4, 10):
        labels, c, _ = O.kmeans_lloyd(x, init, rounds)
        np.testing.assert_allclose(c, fit(rounds).cluster_centers_, rtol=0, atol=1e-9)
        # sklearn's labels_ come from one more assignment against its final centres, so the
        # oracle's last assignment (against the centres of round - 1) is sklearn's labels_
        # after rounds - 1 rounds
        assert np.array_equal(labels, fit(rounds - 1).labels_)
    # one round: the assignment against the initial centres, by brute-force distances
    labels, _, _ = O.kmeans_lloyd(x, init, 1)
    d = np.array([[((xi - cj) ** 2).sum() for cj in init] for xi in x])
    assert np.array_equal(labels, d.argmin(axis=1))


def test_kmeans_inertia_never_increases_and_empty_cluster_keeps_centroid():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((200, 4))
    far = np.full(4, 1e3)                      # a centroid no point is nearest to
    init = np.concatenate([x[:3], far[None]])
    prev = np.inf
    for rounds in range(1, 6):
        labels, c, counts = O.kmeans_lloyd(x, init, rounds)
        inertia = ((x - c[labels]) ** 2).sum()
        assert inertia <= prev + 1e-9
        prev = inertia
        assert counts[3] == 0 and np.array_equal(c[3], far)


def test_kmeans_ties_go_to_lowest_index():
    x = np.array([[0.0, 0.0], [2.0, 0.0]])
    c = np.array([[1.0, 1.0], [1.0, -1.0], [1.0, 1.0]])   # every point equidistant
    assert O.kmeans_assign(x, c).tolist() == [0, 0]


def test_kmeans_distance_is_the_definition_far_from_the_origin():
    # 1e4 from the origin, centroids 1.5 and 1.0 away: the expanded |c|^2 - 2 x.c form in
    # float32 rounds both to the same value (ulp 8 at 1e8); the squared difference does not
    x = np.array([[1.0e4, 0.0]])
    c = np.array([[1.0e4 - 1.5, 0.0], [1.0e4 + 1.0, 0.0]])
    np.testing.assert_allclose(O.kmeans_distances(x, c), [[2.25, 1.0]], rtol=0, atol=1e-9)
    assert O.kmeans_assign(x, c).tolist() == [1]
    # brute force on random data, one distance at a time
    rng = np.random.default_rng(9)
    xs, cs = rng.standard_normal((20, 5)), rng.standard_normal((4, 5))
    brute = [[sum((xs[i, d] - cs[j, d]) ** 2 for d in range(5)) for j in range(4)] for i in range(20)]
    np.testing.assert_allclose(O.kmeans_distances(xs, cs), brute, rtol=1e-14, atol=0)


def test_cluster_layout_is_stable_counting_sort():
    rng = np.random.default_rng(5)
    labels = rng.integers(0, 7, size=300)
    labels[labels == 4] = 5                                 # an empty cluster
    starts, tos, sot = O.cluster_layout(labels, 7)
    # brute force: walk the clusters in order, tokens in raster order
    expect = [t for j in range(7) for t in range(300) if labels[t] == j]
    assert tos.tolist() == expect
    assert np.array_equal(sot[tos], np.arange(300))
    counts = np.bincount(labels, minlength=7)
    for j in range(7):
        assert np.all(labels[tos[starts[j]:starts[j] + counts[j]]] == j)
    assert starts[4] == starts[5]


def test_cluster_mass_is_exact_for_constant_clusters():
    # every token equals its cluster's centroid: the estimate is the exact softmax mass
    rng = np.random.default_rng(6)
    D, Cq, Ck = 8, 3, 4
    qc, kc = rng.standard_normal((Cq, D)), rng.standard_normal((Ck, D))
    nq, nk = np.array([2, 5, 1]), np.array([3, 1, 4, 2])
    q = np.repeat(qc, nq, axis=0)
    k = np.repeat(kc, nk, axis=0)
    scale = 0.7
    est = O.cluster_mass(qc, nq, kc, nk, scale)
    kid = np.repeat(np.arange(Ck), nk)
    qid = np.repeat(np.arange(Cq), nq)
    p = torch.softmax(torch.tensor(scale * q @ k.T), dim=-1).numpy()
    for i in range(Cq):
        exact = [p[qid == i][:, kid == j].sum(axis=1).mean() for j in range(Ck)]
        np.testing.assert_allclose(est[i], exact, rtol=1e-12, atol=1e-15)


def test_cluster_mass_empty_clusters():
    est = O.cluster_mass(np.ones((2, 3)), np.array([0, 4]), np.ones((3, 3)), np.array([2, 0, 2]), 1.0)
    assert np.all(est[0] == 0) and est[1, 1] == 0
    np.testing.assert_allclose(est[1].sum(), 1.0)


def test_cluster_attention_matches_masked_sdpa():
    rng = np.random.default_rng(7)
    S, D = 60, 8
    labels_q = rng.integers(0, 4, size=S)
    labels_k = rng.integers(0, 5, size=S)
    q, k, v = (rng.standard_normal((S, D)) for _ in range(3))
    qs, qtos, _ = O.cluster_layout(labels_q, 4)
    ks, ktos, _ = O.cluster_layout(labels_k, 5)
    qn, kn = np.bincount(labels_q, minlength=4), np.bincount(labels_k, minlength=5)
    sel = [[0, 2], [1], [0, 1, 2, 3, 4], []]               # cluster 3 keeps nothing
    row_ptr = np.concatenate([[0], np.cumsum([len(r) for r in sel])])
    col_idx = np.array([j for r in sel for j in r])
    scale = 0.4
    out = O.cluster_attention(q[qtos], k[ktos], v[ktos], qs, qn, ks, kn, row_ptr, col_idx, scale)
    # reference: SDPA in raster order with the boolean mask of selected cluster pairs
    allowed = np.zeros((S, S), dtype=bool)
    for t in range(S):
        allowed[t] = np.isin(labels_k, sel[labels_q[t]])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None],
        attn_mask=torch.tensor(allowed)[None], scale=scale)[0].numpy()
    ref[~allowed.any(axis=1)] = 0.0
    np.testing.assert_allclose(out, ref[qtos], rtol=1e-10, atol=1e-12)
