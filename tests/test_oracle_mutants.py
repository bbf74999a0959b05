"""The oracle's pins catch plausible mistakes: each case plants one slip in a copy of the
oracle's source (a dropped term, a wrong sign, index or axis, a transposed operand, a
missing pad mask, an off-by-one bound, a wrong rounding rule) and runs the pins of
tests/test_oracle_pins.py against that copy; at least one of the named pins must fail.

The mistake is planted in the oracle, on the CPU, in a module built from the source text
for this test only; the oracle file itself is never changed.  Every planted snippet must
occur exactly once in the source, so a case that no longer matches the oracle fails
loudly instead of testing nothing.
"""
import itertools
import os
import sys
import types

import pytest

import test_oracle_pins as pins

ORACLE_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "oracle", "bsa_oracle.py")
with open(ORACLE_PATH) as _f:
    SOURCE = _f.read()

# (case id, snippet in the oracle, planted replacement, pins expected to catch it)
MUTANTS = [
    # permutation, reading R1
    ("tiles-walk-h-fastest",
     "tile = ((t // TILE) * nth + h // TILE) * ntw + w // TILE",
     "tile = ((t // TILE) * ntw + w // TILE) * nth + h // TILE",
     ["test_tile_grid_is_walked_w_fastest"]),
    ("inside-tile-h-and-w-swapped",
     "inner = ((t % TILE) * TILE + h % TILE) * TILE + w % TILE",
     "inner = ((t % TILE) * TILE + w % TILE) * TILE + h % TILE",
     ["test_tile_grid_is_walked_w_fastest"]),
    ("inside-tile-t-fastest",
     "inner = ((t % TILE) * TILE + h % TILE) * TILE + w % TILE",
     "inner = ((w % TILE) * TILE + h % TILE) * TILE + t % TILE",
     ["test_tile_grid_is_walked_w_fastest"]),
    ("pad-slots-not-zeroed",
     "out = np.zeros((B, Hh, g.Np, D), dtype=x.dtype)",
     "out = np.ones((B, Hh, g.Np, D), dtype=x.dtype)",
     ["test_permute_is_bijection_onto_valid_slots"]),
    ("pad-tokens-kept-in-ragged-tiles",
     "if t < g.T and h < g.H and w < g.W:",
     "if t < g.Tp and h < g.Hp and w < g.Wp:",
     ["test_permute_is_bijection_onto_valid_slots", "test_every_block_is_one_aligned_4x4x4_cube"]),
    # block mass, reading R2
    ("mass-scale-dropped",
     "p = _softmax_rows(scale * (q @ k.T))",
     "p = _softmax_rows(q @ k.T)",
     ["test_mass_matches_torch_softmax_block_sums", "test_mass_one_hot_attention_closed_form"]),
    ("mass-q-and-k-transposed",
     "q = qt[b, h, rows, :].astype(np.float64)\n    k = kt[b, h, keys, :].astype(np.float64)\n"
     "    p = _softmax_rows",
     "q = kt[b, h, rows, :].astype(np.float64)\n    k = qt[b, h, keys, :].astype(np.float64)\n"
     "    p = _softmax_rows",
     ["test_mass_matches_torch_softmax_block_sums", "test_mass_one_hot_attention_closed_form"]),
    ("mass-pad-keys-in-softmax",
     "keys = np.nonzero(valid)[0]",
     "keys = np.arange(valid.size)",
     ["test_mass_rows_sum_to_one_and_pad_blocks_are_zero", "test_mass_uniform_attention_closed_form"]),
    ("mass-mean-over-all-rows-of-the-block",
     "return mass / rows.size",
     "return mass / q_block",
     ["test_mass_rows_sum_to_one_and_pad_blocks_are_zero"]),
    ("mass-softmax-over-the-wrong-axis",
     "return e / e.sum(axis=1, keepdims=True)",
     "return e / e.sum(axis=0, keepdims=True)",
     ["test_mass_rows_sum_to_one_and_pad_blocks_are_zero",
      "test_mass_matches_torch_softmax_block_sums"]),
    ("mass-block-of-key-off-by-one-tile",
     "np.add.at(mass, keys // kv_block, per_key)",
     "np.add.at(mass, (keys + 1) // kv_block % n_kb, per_key)",
     ["test_mass_one_hot_attention_closed_form", "test_mass_uniform_attention_closed_form"]),
    # selection, reading R3
    ("topp-floor-target",
     "return int(math.ceil(float(np.float64(np.float32(tau)))",
     "return int(math.floor(float(np.float64(np.float32(tau)))",
     ["test_topp_hand_examples", "test_topp_target_is_the_exact_ceiling_where_the_product_is_exact"]),
    ("topp-ascending-order",
     "key=lambda j: (-int(q[j]), j)",
     "key=lambda j: (int(q[j]), j)",
     ["test_topp_minimal_by_brute_force", "test_topp_hand_examples"]),
    ("topp-ties-to-the-higher-index",
     "key=lambda j: (-int(q[j]), j)",
     "key=lambda j: (-int(q[j]), -j)",
     ["test_topp_minimal_by_brute_force", "test_topp_hand_examples",
      "test_topp_uniform_closed_form"]),
    ("topp-one-block-too-many",
     "while acc < target:",
     "while acc <= target:",
     ["test_topp_minimal_by_brute_force", "test_topp_hand_examples"]),
    ("topp-target-from-the-float-sum",
     "target = topp_target(int(q.sum()), tau)",
     "target = int(math.ceil(float(tau) * float(q.sum())))",
     ["test_topp_hand_examples"]),
    ("topp-negative-masses-accepted",
     "np.any(m < 0) or ",
     "",
     ["test_topp_rejects_bad_masses"]),
    ("topp-fixed-point-truncated",
     "return np.rint(m * FP_SCALE).astype(np.int64)",
     "return np.floor(m * FP_SCALE).astype(np.int64)",
     ["test_fixed_point_masses_round_half_to_even"]),
    ("topp-fixed-point-scale-2-32",
     "FP_SCALE = 2.0 ** 40",
     "FP_SCALE = 2.0 ** 32",
     ["test_topp_hand_examples", "test_fixed_point_masses_round_half_to_even"]),
    # attention, reading R4
    ("attn-scale-dropped",
     "logits = scale * (k @ q)",
     "logits = k @ q",
     ["test_attention_full_csr_equals_sdpa", "test_attention_kept_set_renormalises"]),
    ("attn-lse-without-the-max",
     "return (e / z) @ v, float(mx + math.log(z))",
     "return (e / z) @ v, float(math.log(z))",
     ["test_attention_full_csr_equals_sdpa"]),
    ("attn-pad-keys-of-kept-blocks-attended",
     "keys = keys[valid[keys]]\n    if keys.size == 0:\n        return np.zeros(D), -math.inf",
     "if keys.size == 0:\n        return np.zeros(D), -math.inf",
     ["test_attention_full_csr_equals_sdpa", "test_attention_single_block_identical_keys_is_block_mean"]),
    ("attn-values-from-keys",
     "v = vt[b, h, keys, :].astype(np.float64)",
     "v = kt[b, h, keys, :].astype(np.float64)",
     ["test_attention_full_csr_equals_sdpa", "test_attention_constant_values_closed_form"]),
    ("attn-row-of-the-next-query-block",
     "r = (b * Hh + h) * n_qb + p // q_block",
     "r = ((b * Hh + h) * n_qb + p // q_block + 1) % (row_ptr.size - 1)",
     ["test_attention_kept_set_renormalises"]),
    ("attn-pad-query-rows-attend",
     "if not valid[p]:\n        return np.zeros(D), -math.inf",
     "if False:\n        return np.zeros(D), -math.inf",
     ["test_attention_full_csr_equals_sdpa", "test_attention_constant_values_closed_form"]),
    # e4m3, reading R5
    ("e4m3-subnormal-exponent",
     "out[c] = sign * (m / 8.0) * 2.0 ** -6",
     "out[c] = sign * (m / 8.0) * 2.0 ** -7",
     ["test_e4m3_decode_matches_torch"]),
    ("e4m3-exponent-bias-8",
     "out[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)",
     "out[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 8)",
     ["test_e4m3_decode_matches_torch"]),
    ("e4m3-ties-away-from-zero",
     "pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))",
     "pick_hi = (d_hi <= d_lo)",
     ["test_e4m3_encode_matches_torch_cast_in_range"]),
    ("e4m3-truncation",
     "pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))",
     "pick_hi = np.zeros_like(d_hi, dtype=bool)",
     ["test_e4m3_encode_matches_torch_cast_in_range", "test_quant_tiles_scale_and_error_bound"]),
    ("e4m3-sign-of-zero-dropped",
     "return np.where(neg, code | 0x80, code).astype(np.uint8)",
     "return np.where(neg & (code > 0), code | 0x80, code).astype(np.uint8)",
     ["test_e4m3_encode_matches_torch_cast_in_range"]),
    ("fp8-scale-for-another-format",
     "absmax / np.float32(448.0)",
     "absmax / np.float32(240.0)",
     ["test_quant_tiles_scale_and_error_bound"]),
    ("fp8-zero-tile-scale-zero",
     "np.where(absmax == 0, np.float32(1.0),",
     "np.where(absmax == 0, np.float32(0.0),",
     ["test_quant_tiles_scale_and_error_bound"]),
    ("fp8-dequant-scales-tiled-not-repeated",
     "s = np.repeat(np.asarray(scales, dtype=np.float64), TILE_TOKENS, axis=2)",
     "s = np.tile(np.asarray(scales, dtype=np.float64), (1, 1, TILE_TOKENS))",
     ["test_quant_tiles_scale_and_error_bound"]),
    # structured patterns
    ("pattern-band-exclusive",
     "if kinds & PAT_DIAGONAL and abs(j - u) <= diag_width:",
     "if kinds & PAT_DIAGONAL and abs(j - u) < diag_width:",
     ["test_pattern_diagonal_band_closed_form"]),
    ("pattern-query-block-covers-one-tile",
     "for u in range(i * per, (i + 1) * per):",
     "for u in range(i * per, i * per + 1):",
     ["test_pattern_diagonal_128_token_query_blocks_cover_both_tiles"]),
    ("pattern-period-from-the-wrong-axes",
     "L = multi_period if multi_period > 0 else (g.Hp // TILE) * (g.Wp // TILE)",
     "L = multi_period if multi_period > 0 else (g.Tp // TILE) * (g.Wp // TILE)",
     ["test_pattern_multi_diagonal_hits_same_place_in_other_frames"]),
    ("pattern-own-frame-in-multi-diagonal",
     "if k != 0 and abs(j - (u + k * L)) <= diag_width:",
     "if abs(j - (u + k * L)) <= diag_width:",
     ["test_pattern_multi_diagonal_hits_same_place_in_other_frames"]),
    ("pattern-stripe-offset-ignored",
     "j % stripe_stride == stripe_offset:",
     "j % stripe_stride == 0:",
     ["test_pattern_vertical_stripes_are_the_same_for_every_row"]),
    ("pattern-surrounding-radii-swapped",
     "abs(jh - uh) <= radius[1] \\\n                and abs(jw - uw) <= radius[2]",
     "abs(jh - uh) <= radius[2] \\\n                and abs(jw - uw) <= radius[1]",
     ["test_pattern_surrounding_asymmetric_radii_on_a_non_cubic_grid"]),
    ("pattern-criss-cross-one-shared-axis",
     "(int(jt == ut) + int(jh == uh) + int(jw == uw)) >= 2",
     "(int(jt == ut) + int(jh == uh) + int(jw == uw)) >= 1",
     ["test_pattern_criss_cross_is_three_axis_lines"]),
    ("pattern-tile-coords-h-and-w-swapped",
     "return j // (nth * ntw), (j // ntw) % nth, j % ntw",
     "return j // (nth * ntw), j % nth, (j // nth) % ntw",
     ["test_pattern_surrounding_asymmetric_radii_on_a_non_cubic_grid",
      "test_pattern_criss_cross_sets_on_a_non_cubic_grid"]),
    # pooled estimate, reading R8
    ("pooled-key-count-weight-dropped",
     "w = n_keys[keep] * np.exp(z)",
     "w = np.exp(z)",
     ["test_pooled_estimate_is_exact_when_blocks_are_constant",
      "test_pooled_estimate_rows_and_zero_scale"]),
    ("pooled-kbar-sum-not-mean",
     "kbar[j] = k[rows].mean(axis=0)",
     "kbar[j] = k[rows].sum(axis=0)",
     ["test_pooled_estimate_is_exact_when_blocks_are_constant"]),
    ("pooled-qbar-over-pad-rows-too",
     "qbar = q[rows].mean(axis=0)",
     "qbar = q[i * q_block:(i + 1) * q_block].mean(axis=0)",
     ["test_pooled_estimate_is_exact_when_blocks_are_constant"]),
    ("pooled-scale-dropped",
     "logits = scale * (kbar @ qbar)",
     "logits = kbar @ qbar",
     ["test_pooled_estimate_is_exact_when_blocks_are_constant",
      "test_pooled_estimate_rows_and_zero_scale"]),
    ("pooled-empty-query-blocks-not-skipped",
     "                if rows.size == 0:\n                    continue\n                qbar",
     "                qbar",
     ["test_pooled_estimate_rows_and_zero_scale",
      "test_pooled_estimate_is_exact_when_blocks_are_constant"]),
    # k-means and cluster attention, reading R10
    ("kmeans-farthest-centroid",
     "return np.argmin(kmeans_distances(x, centroids), axis=1)",
     "return np.argmax(kmeans_distances(x, centroids), axis=1)",
     ["test_kmeans_recovers_separated_blobs", "test_kmeans_matches_sklearn_lloyd"]),
    ("kmeans-l1-distance",
     "d[:, j] = (diff * diff).sum(axis=1)",
     "d[:, j] = np.abs(diff).sum(axis=1)",
     ["test_kmeans_matches_sklearn_lloyd", "test_kmeans_distance_is_the_definition_far_from_the_origin"]),
    ("kmeans-empty-cluster-reset",
     "if member.any():\n                c[j] = x[member].mean(axis=0)",
     "c[j] = x[member].mean(axis=0) if member.any() else 0.0",
     ["test_kmeans_inertia_never_increases_and_empty_cluster_keeps_centroid"]),
    ("kmeans-ties-to-the-last-index",
     "return np.argmin(kmeans_distances(x, centroids), axis=1)",
     "return (centroids.shape[0] - 1 - np.argmin(kmeans_distances(x, centroids)[:, ::-1], axis=1))",
     ["test_kmeans_ties_go_to_lowest_index"]),
    ("layout-inclusive-starts",
     "starts = np.concatenate([[0], np.cumsum(counts)[:-1]]).astype(np.int64)",
     "starts = np.cumsum(counts).astype(np.int64)",
     ["test_cluster_layout_is_stable_counting_sort"]),
    ("layout-tokens-in-reverse-order",
     "token_of_slot = np.argsort(labels, kind=\"stable\").astype(np.int64)",
     "token_of_slot = (labels.size - 1 - np.argsort(labels[::-1], kind=\"stable\")).astype(np.int64)",
     ["test_cluster_layout_is_stable_counting_sort"]),
    ("cluster-count-weight-dropped",
     "w = nk[keep] * np.exp(logits - logits.max())",
     "w = np.exp(logits - logits.max())",
     ["test_cluster_mass_is_exact_for_constant_clusters"]),
    ("cluster-mass-empty-query-cluster-filled",
     "        if q_counts[i] == 0:\n            continue\n        logits = scale * (kc[keep] @ qc[i])",
     "        logits = scale * (kc[keep] @ qc[i])",
     ["test_cluster_mass_empty_clusters"]),
    ("kmeans-one-round-too-many",
     "    for _ in range(rounds):\n        labels = kmeans_assign(x, c)",
     "    for _ in range(rounds + 1):\n        labels = kmeans_assign(x, c)",
     ["test_kmeans_matches_sklearn_lloyd"]),
    ("cluster-attention-last-key-of-a-cluster-dropped",
     "np.arange(k_starts[j], k_starts[j] + k_counts[j])",
     "np.arange(k_starts[j], k_starts[j] + k_counts[j] - 1)",
     ["test_cluster_attention_matches_masked_sdpa"]),
    ("cluster-attention-scale-dropped",
     "logits = scale * (k[keys] @ q[p])",
     "logits = k[keys] @ q[p]",
     ["test_cluster_attention_matches_masked_sdpa"]),
]


def _mutant_module(old, new):
    assert SOURCE.count(old) == 1, f"snippet not found exactly once in the oracle: {old!r}"
    name = "bsa_oracle_mutant"
    mod = types.ModuleType(name)
    mod.__file__ = ORACLE_PATH
    sys.modules[name] = mod  # dataclasses look the defining module up while the class is built
    try:
        exec(compile(SOURCE.replace(old, new), ORACLE_PATH + " (mutant)", "exec"), mod.__dict__)
    finally:
        del sys.modules[name]
    return mod


def _cases(fn):
    """Every parameter combination of a pin's parametrize marks (none: one empty case)."""
    axes = []
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names, values = mark.args[0], mark.args[1]
        names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
        axes.append([dict(zip(names, v if len(names) > 1 else (v,))) for v in values])
    for combo in itertools.product(*axes):
        kw = {}
        for part in combo:
            kw.update(part)
        yield kw


def _failures(module, pin_names):
    """(pin, case) pairs that fail when the pins run against `module`."""
    failed = []
    saved = pins.O
    pins.O = module
    try:
        for name in pin_names:
            fn = getattr(pins, name)
            for kw in _cases(fn):
                try:
                    fn(**kw)
                except pytest.skip.Exception:
                    continue
                except (Exception, pytest.fail.Exception) as e:  # noqa: BLE001
                    failed.append((name, kw, type(e).__name__))
    finally:
        pins.O = saved
    return failed


def test_every_named_pin_exists():
    for case, _, _, names in MUTANTS:
        for n in names:
            assert callable(getattr(pins, n, None)), (case, n)


def test_unplanted_copy_passes_the_same_pins():
    """The runner itself: a copy of the oracle with nothing planted fails no pin."""
    names = sorted({n for *_, ns in MUTANTS for n in ns})
    clean = _mutant_module("TILE = 4          # tile edge", "TILE = 4          # tile edge")
    assert _failures(clean, names) == []


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # a planted mistake may divide by zero
@pytest.mark.parametrize("case,old,new,names", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(case, old, new, names):
    mutant = _mutant_module(old, new)
    assert _failures(mutant, names), f"no pin caught the planted mistake {case!r}"
