"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each case rewrites one line of one oracle function into a plausible
mistake: a dropped term, a wrong sign, a non-strict comparison, a
transposed operand, an off-by-one exponent, a reversed tie order.  Then it
runs the pins that guard that function, and at least one of them must
fail.  A case that every pin lets through would mark a gap in the pins.

The rewrite works on the function's source text, so the mutant is the
oracle's own code with the one change.  It replaces every reference to the
original function in the oracle package and in the pin modules for the
duration of the case.
"""
import inspect
import sys
import textwrap

import pytest

import oracle
import oracle.attention
import oracle.backward
import oracle.lite
import oracle.masks
import oracle.permute
import oracle.pyramid
import test_golden as pins_golden
from _golden import matrix
import test_oracle_attention as pins_attn
import test_oracle_backward as pins_bwd
import test_oracle_masks as pins_masks
import test_oracle_permute as pins_perm
import test_oracle_pyramid_lite as pins_pl


def _mutant(module, name, old, new):
    fn = getattr(module, name)
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) == 1, f"{name}: the text to mutate must occur exactly once: {old!r}"
    ns = dict(module.__dict__)
    exec(compile(src.replace(old, new), f"<mutant of {module.__name__}.{name}>", "exec"), ns)
    return fn, ns[name]


def _install(monkeypatch, original, mutant):
    """Replace every module-level reference to `original` in the oracle and pin modules."""
    mods = [m for k, m in list(sys.modules.items())
            if m is not None and (k == "oracle" or k.startswith("oracle.") or k.startswith("test_"))]
    for m in mods:
        for attr, val in list(vars(m).items()):
            if val is original:
                monkeypatch.setattr(m, attr, mutant)


def _golden(test, name):
    """One parametrized golden pin over all records of its fixture."""
    from _golden import records
    fixture = {"test_axis_orders": "axis_orders.txt", "test_tau_rows": "tau_rows.txt",
               "test_global_heads": "global_heads.txt", "test_radial_rows": "radial_rows.txt",
               "test_level_rows": "level_rows.txt", "test_pyramid_rows": "pyramid_rows.txt", "test_tau_rows_through_the_mask_wrapper": "tau_rows.txt",
               "test_level_rows_through_the_map_wrapper": "level_rows.txt",
               "test_global_heads_through_the_mask_wrapper": "global_heads.txt",
               "test_lite_skip": "lite_skip.txt"}[name]

    def run():
        for rec in records(fixture):
            test(rec)
    return run


def _square(test):
    """The global wrapper pin takes the square fixtures only (the library's masks are Nb x Nb)."""
    def run(rec):
        if len(matrix(rec["p"])) == len(matrix(rec["p"])[0]):
            test(rec)
    return run


def _margin(kind):
    """The margin-flag pins of one decision kind (tests/golden/margin_flags.txt)."""
    from _golden import records

    def run():
        for rec in records("margin_flags.txt"):
            if rec["kind"] == kind:
                pins_golden.check_margin_flags(rec)
    return run


PIN_SETS = {
    "attention": [pins_attn.test_all_ones_mask_equals_dense_sdpa_tiny_config,
                  lambda: pins_attn.test_brute_force_token_level_matches_block_path(21, 8),
                  pins_attn.test_rows_sum_to_one_with_unit_values,
                  pins_attn.test_single_kept_block_is_attention_over_that_block,
                  pins_attn.test_lse_matches_scipy_logsumexp_on_kept_columns,
                  pins_attn.test_causal_all_ones_equals_sdpa_is_causal,
                  pins_attn.test_causal_block_mask_equals_token_level_brute_force],
    "dense": [pins_attn.test_all_ones_mask_equals_dense_sdpa_tiny_config],
    "tau": [pins_masks.test_tau_uniform_scores_keep_first_ceil_tau_n,
            pins_masks.test_tau_block_exactly_at_the_threshold_is_dropped,
            pins_masks.test_tau_to_zero_keeps_only_argmax,
            pins_masks.test_tau_brute_force_minimum_cardinality_prefix,
            pins_masks.test_tau_monotone,
            _golden(pins_golden.test_tau_rows, "test_tau_rows"),
            _margin("tau")],
    "levels": [pins_masks.test_level_quotas_and_order, pins_masks.test_level_ties_break_by_index, _margin("level"),
               _golden(pins_golden.test_level_rows, "test_level_rows")],
    "scores": [pins_masks.test_block_means_closed_form_with_partial_tail, pins_masks.test_block_scores_closed_form],
    "radial": [lambda: pins_masks.test_radial_matches_bruteforce(17, 4, 9, 8),
               lambda: pins_masks.test_radial_matches_bruteforce(9, 8, 16, 16),
               pins_masks.test_radial_structure,
               _golden(pins_golden.test_radial_rows, "test_radial_rows")],
    "global": [pins_masks.test_global_single_row_equals_tau_row,
               pins_masks.test_global_hand_built_peaked_and_uniform_rows,
               pins_masks.test_global_pair_exactly_at_the_threshold_is_dropped,
               pins_masks.test_global_brute_force_shortest_prefix,
               _golden(pins_golden.test_global_heads, "test_global_heads"),
               _margin("global")],
    "skipflags": [_margin("skip")],
    "lite": [pins_pl.test_infinite_eps_never_skips_and_equals_block_attention,
             pins_pl.test_hand_built_gap_of_twelve,
             pins_pl.test_skipped_blocks_are_exponentially_suppressed,
             pins_pl.test_first_visited_block_never_skipped_and_chain_monotone,
             _golden(pins_golden.test_lite_skip, "test_lite_skip")],
    "visit": [pins_pl.test_radial_visit_order_hand_listed],
    "permute": [lambda: pins_perm.test_axis_orders_equal_grid_transposes("hwt"),
                pins_perm.test_hand_listed_hwt,
                pins_perm.test_cell_partitions_equal_blocked_transposes,
                pins_perm.test_bijection_inverse_and_per_head_orders,
                _golden(pins_golden.test_axis_orders, "test_axis_orders")],
    "pyramid": [pins_pl.test_pool_partial_group_and_progressive_equals_direct,
                pins_pl.test_all_level_zero_equals_block_attention,
                pins_pl.test_constant_groups_make_any_level_mix_exact,
                pins_pl.test_causal_constant_groups_equal_causal_attention,
                _golden(pins_golden.test_pyramid_rows, "test_pyramid_rows")],
    "backward": [pins_bwd.test_empty_rows_and_columns_and_key_shift_invariance,
                 pins_bwd.test_dense_case_equals_torch_autograd,
                 pins_bwd.test_causal_finite_differences],
    "wrappers": [_golden(pins_golden.test_tau_rows_through_the_mask_wrapper, "test_tau_rows_through_the_mask_wrapper"),
                 _golden(pins_golden.test_level_rows_through_the_map_wrapper,
                         "test_level_rows_through_the_map_wrapper"),
                 _golden(_square(pins_golden.test_global_heads_through_the_mask_wrapper),
                         "test_global_heads_through_the_mask_wrapper")],
    "backward_rows": [lambda: pins_bwd.test_sampled_rows_equal_full_gradients(False),
                      lambda: pins_bwd.test_sampled_rows_equal_full_gradients(True)],
    "chain": [pins_pl.test_first_visited_block_never_skipped_and_chain_monotone],
}

A, M, L, P, Y, W = (oracle.attention, oracle.masks, oracle.lite, oracle.permute, oracle.pyramid,
                    oracle.backward)
MUTATIONS = [
    # (id, module, function, original text, mistaken text, pin set)
    ("attn-no-scale", A, "attention_qblock", "s = (qh[r0:r1] @ kh[c].T) * scale", "s = (qh[r0:r1] @ kh[c].T)",
     "attention"),
    ("attn-lse-without-max", A, "attention_qblock", "lse = (m + np.log(z))", "lse = (np.log(z))", "attention"),
    ("attn-mask-ignored", A, "attention_qblock", "for j in np.nonzero(keep_row)[0]]", "for j in range(len(keep_row))]",
     "attention"),
    ("attn-causal-drops-diagonal", A, "attention_qblock", "c[None, :] <= np.arange(r0, r1)[:, None]",
     "c[None, :] < np.arange(r0, r1)[:, None]", "attention"),
    ("dense-unnormalised", A, "dense_attention", "e / z, v)", "e, v)", "dense"),
    ("dense-lse-without-max", A, "dense_attention", "(m + np.log(z))", "(np.log(z))", "dense"),
    ("token-mask-transposed", A, "block_mask_to_token_mask", "return m[idx][:, idx]", "return m.T[idx][:, idx]",
     "backward"),
    ("tau-mask-first-row-only", M, "tau_mask", "tau_row(S[b, h, i], tau)", "tau_row(S[b, h, 0], tau)", "wrappers"),
    ("tau-mask-first-head-only", M, "tau_mask", "tau_row(S[b, h, i], tau)", "tau_row(S[b, 0, i], tau)", "wrappers"),
    ("level-map-first-row-only", M, "level_map", "level_row(S[b, h, i], counts)", "level_row(S[b, h, 0], counts)",
     "wrappers"),
    ("global-mask-first-head-only", M, "global_mask", "global_head(S[b, h], tau)", "global_head(S[b, 0], tau)",
     "wrappers"),
    ("scores-transposed", M, "block_scores", '"bhid,bhjd->bhij"', '"bhid,bhjd->bhji"', "wrappers"),
    ("tau-non-strict", M, "tau_row", "keep = mass_before < tau", "keep = mass_before <= tau", "tau"),
    ("tau-mass-includes-self", M, "tau_row", "mass_before[j] = acc\n        acc += p[j]",
     "acc += p[j]\n        mass_before[j] = acc", "tau"),
    ("rank-ascending", M, "_order", "np.lexsort((np.arange(row.shape[0]), -row))",
     "np.lexsort((np.arange(row.shape[0]), row))", "tau"),
    ("rank-ties-reversed", M, "_order", "np.lexsort((np.arange(row.shape[0]), -row))",
     "np.lexsort((-np.arange(row.shape[0]), -row))", "tau"),
    ("level-quota-floor", M, "level_counts", "math.ceil(f * nkb - 1e-9)", "math.floor(f * nkb + 1e-9)", "levels"),
    ("level-ties-reversed", M, "_order", "np.lexsort((np.arange(row.shape[0]), -row))",
     "np.lexsort((-np.arange(row.shape[0]), -row))", "levels"),
    ("means-divide-by-block", M, "block_means", "/ (r1 - r0)", "/ block", "scores"),
    ("scores-no-scale", M, "block_scores", 'qm, km) * scale', 'qm, km)', "scores"),
    # (Δt = 1 needs no band of its own: the window rule keeps every offset there.)
    ("radial-band-too-wide", M, "radial_mask", "if t <= 1:", "if t <= 2:", "radial"),
    ("radial-log2-off-by-one", M, "radial_mask", "kexp = t.bit_length() - 1", "kexp = t.bit_length()", "radial"),
    ("radial-non-strict-window", M, "radial_mask", "(1 << kexp) < S", "(1 << kexp) <= S", "radial"),
    ("radial-last-token-position", M, "radial_mask", "first = np.arange(nb, dtype=np.int64) * block",
     "first = np.minimum(np.arange(nb, dtype=np.int64) * block + block - 1, N - 1)", "radial"),
    ("global-non-strict", M, "global_head", "keep = mass_before < target", "keep = mass_before <= target", "global"),
    ("global-target-per-row", M, "global_head", "target = tau * nqb", "target = tau", "global"),
    ("global-ties-reversed", M, "global_head", "np.lexsort((np.arange(flat.size), -flat))",
     "np.lexsort((-np.arange(flat.size), -flat))", "global"),
    # margin flags: each decision's "within 1e-3 of the cut" rule
    ("tau-flag-margin-wide", M, "tau_row", "flag = np.abs(mass_before - tau) < MARGIN",
     "flag = np.abs(mass_before - tau) < 10 * MARGIN", "tau"),
    ("tau-flag-margin-narrow", M, "tau_row", "flag = np.abs(mass_before - tau) < MARGIN",
     "flag = np.abs(mass_before - tau) < 0.1 * MARGIN", "tau"),
    ("tau-flag-mass-after", M, "tau_row", "np.abs(mass_before - tau)", "np.abs(mass_before + p - tau)", "tau"),
    ("tau-flag-no-swap-kept", M, "tau_row", "flag |= keep & (np.abs(p - p_out) <= MARGIN * p_out)", "pass", "tau"),
    ("tau-flag-no-swap-dropped", M, "tau_row", "flag |= (~keep) & (np.abs(p - p_in) <= MARGIN * p_in)", "pass",
     "tau"),
    ("tau-flag-swap-absolute", M, "tau_row", "<= MARGIN * p_out", "<= MARGIN", "tau"),
    ("level-code-is-level", M, "level_row", "code[rank < counts[lvl]] = lvl + 1", "code[rank < counts[lvl]] = lvl",
     "levels"),
    ("level-coarse-overwrites-fine", M, "level_row", "for lvl in (2, 1, 0):", "for lvl in (0, 1, 2):", "levels"),
    ("level-flag-margin-wide", M, "level_row", "(s - s_out < MARGIN)", "(s - s_out < 10 * MARGIN)", "levels"),
    ("level-flag-sign", M, "level_row", "(s - s_out < MARGIN)", "(s_out - s < MARGIN)", "levels"),
    ("level-flag-no-lower-side", M, "level_row", "flag |= (rank >= c) & (s_in - s < MARGIN)", "pass", "levels"),
    ("level-flag-relative", M, "level_row", "(s_in - s < MARGIN)", "(s_in - s < MARGIN * abs(s_in))", "levels"),
    ("global-flag-margin-absolute", M, "global_head", "< MARGIN * nqb", "< MARGIN", "global"),
    ("global-flag-margin-wide", M, "global_head", "< MARGIN * nqb", "< 10 * MARGIN * nqb", "global"),
    ("global-flag-no-swap-kept", M, "global_head", "flag |= keep & (np.abs(flat - p_out) <= MARGIN * p_out)",
     "pass", "global"),
    ("global-flag-swap-absolute", M, "global_head", "<= MARGIN * p_in)", "<= MARGIN)", "global"),
    ("skip-flag-wide", L, "skip_flags", "np.abs(m) < MARGIN", "np.abs(m) < 10 * MARGIN", "skipflags"),
    ("skip-flag-signed", L, "skip_flags", "np.abs(m) < MARGIN", "m < MARGIN", "skipflags"),
    ("skip-any-row", L, "lite_qblock", "mg = np.max(local - running + eps)", "mg = np.min(local - running + eps)",
     "lite"),
    ("skip-eps-sign", L, "lite_qblock", "mg = np.max(local - running + eps)", "mg = np.max(local - running - eps)",
     "lite"),
    ("skip-last-block-max", L, "lite_qblock", "running = np.maximum(running, local)", "running = local", "lite"),
    ("skip-first-block-tested", L, "lite_qblock", "if n_vis > 0:", "if n_vis >= 0:", "lite"),
    ("skip-never-tested", L, "lite_qblock", "if n_vis > 0:", "if n_vis < 0:", "lite"),
    ("radial-order-ties-descending", L, "visit_order", "key=lambda t: (dist(t), t)", "key=lambda t: (dist(t), -t)",
     "visit"),
    ("perm-slowest-axis-last", P, "permutation", "np.lexsort(keys[::-1])", "np.lexsort(keys)", "permute"),
    ("perm-cell-and-inner-swapped", P, "permutation",
     "keys = [coord[a] // cell[a] for a in order] + [coord[a] % cell[a] for a in order]",
     "keys = [coord[a] % cell[a] for a in order] + [coord[a] // cell[a] for a in order]", "permute"),
    ("pool-divide-by-c", Y, "pyramid_pool", "/ (r1 - r0)", "/ c", "pyramid"),
    ("pyramid-bias-sign", Y, "_level_keys", "np.log(counts)", "-np.log(counts)", "pyramid"),
    ("pyramid-bias-missing", Y, "_level_keys", "np.log(counts)", "0.0 * counts", "pyramid"),
    ("pyramid-values-subsampled", Y, "_level_keys", "pooled_v[level][g0:g1], np.log(counts)",
     "vh[r0:r1:c], np.log(counts)", "pyramid"),
    ("pyramid-causal-diagonal-pooled", Y, "pyramid_attention", "if causal and j == i and code:\n                code = 1",
     "if causal and j == i and code:\n                code = code", "pyramid"),
    ("bwd-no-delta", W, "attention_bwd_head", "dr = np.sum(p * dp, axis=1, keepdims=True)", "dr = 0.0", "backward"),
    ("bwd-dk-no-scale", W, "attention_bwd_head", "scale * (ds.T @ qh)", "(ds.T @ qh)", "backward"),
    ("bwd-dv-transposed", W, "attention_bwd_head", "dv = p.T @ doh", "dv = p @ doh", "backward"),
    ("bwd-rows-no-delta", W, "masked_attention_bwd_rows", "dr = np.sum(doh[r0:r1] * o, axis=1, keepdims=True)",
     "dr = 0.0", "backward_rows"),
    ("bwd-rows-causal-drops-diagonal", W, "masked_attention_bwd_rows",
     "np.arange(N)[None, :] <= rows[:, None]", "np.arange(N)[None, :] < rows[:, None]", "backward_rows"),
    ("bwd-rows-dk-no-scale", W, "masked_attention_bwd_rows", "dk += scale * (dsc.T @ qh[r0:r1])",
     "dk += dsc.T @ qh[r0:r1]", "backward_rows"),
    ("perm-inverse-applies-forward", P, "permute_tokens", "out[:, h, perm] = x[:, h]", "out[:, h] = x[:, h, perm]",
     "permute"),
    ("chain-skip-not-carried", L, "lite_chain", "skip = S if feed is None else feed(s, S)",
     "skip = skip0 if feed is None else feed(s, S)", "chain"),
]


@pytest.mark.parametrize("case", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(case, monkeypatch):
    _, module, name, old, new, pin_set = case
    original, mutant = _mutant(module, name, old, new)
    _install(monkeypatch, original, mutant)
    caught = []
    for pin in PIN_SETS[pin_set]:
        try:
            pin()
        except Exception as e:          # an AssertionError, or the mutant breaking a shape or index
            caught.append(type(e).__name__)
    assert caught, f"no pin of '{pin_set}' fails with the planted mistake {case[0]}"


def test_unmutated_pins_pass():
    """Control: every pin set passes on the oracle as it is."""
    for pins in PIN_SETS.values():
        for pin in pins:
            pin()
