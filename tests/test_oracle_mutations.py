"""Planted mistakes in the oracle: each one must make some pin fail.

Each case rewrites one expression of one oracle function -- a plausible slip
in the step that function restates (a strict comparison for an inclusive
one, a dropped scale or maximum, an off-by-one window, the misprinted
threshold, a wrong rounding or exponent bias) -- compiles the rewritten
function in a copy of its module's namespace, installs it with monkeypatch
on the CPU, and runs the pin tests named for it.  At least one of them must
fail; a mutation no pin catches would mean the pins do not constrain that
step.  The original functions are restored after each case, and the
unmutated pins pass in their own test files.
"""

import inspect
import textwrap

import pytest

import test_oracle_anchor as t_anchor
import test_oracle_attention as t_att
import test_oracle_decode as t_dec
import test_oracle_fp8 as t_fp8
import test_oracle_sale as t_sale
from oracle import attention as oatt
from oracle import decode as odec
from oracle import fp8 as ofp8
from oracle import selection as osel


def _mutant(module, name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(module, name)))
    assert src.count(old) == 1, (module.__name__, name, old)
    ns = dict(vars(module))
    exec(compile(src.replace(old, new), f"<planted {module.__name__}.{name}>", "exec"), ns)
    return ns[name]


def _param_sets(fn):
    """Keyword sets of a pin from its parametrize marks (cartesian product)."""
    sets = [{}]
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names = mark.args[0]
        names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
        grown = []
        for base in sets:
            for val in mark.args[1]:
                val = val.values if hasattr(val, "values") else val
                vals = tuple(val) if len(names) > 1 else (val,)
                grown.append({**base, **dict(zip(names, vals))})
        sets = grown
    needed = set(inspect.signature(fn).parameters)
    for kw in sets:
        assert set(kw) == needed, (fn.__name__, needed)
    return sets


def _some_pin_fails(pins):
    for fn in pins:
        for kw in _param_sets(fn):
            try:
                fn(**kw)
            except Exception:
                return True
    return False


CASES = [
    # AnchorAttention Eq. (2): ties keep (<=)
    ("anchor_strict_compare", osel, "anchor_block", "keep = diff <= theta", "keep = diff < theta",
     [t_anchor.test_handmade_exact_ties_keep, t_anchor.test_handmade_anchor_cases]),
    # Eq. (2): avgpool of the anchor is a mean over the block's rows
    ("anchor_max_over_rows", osel, "anchor_block", "xbar_a = float(x_a.mean())",
     "xbar_a = float(x_a.max())", [t_anchor.test_handmade_anchor_cases,
                                   t_anchor.test_avgpool_linearity]),
    # Eq. (2): pooled score carries the 1/sqrt(d) scale
    ("anchor_dropped_scale", osel, "anchor_block", "sbar = (kh[cand] @ qbar) * sc",
     "sbar = (kh[cand] @ qbar)", [t_anchor.test_handmade_anchor_cases]),
    # Eq. (1): the anchor sees the diagonal key (causal j <= i)
    ("anchor_causal_cut", osel, "anchor_block", "causal = slk[None, :] <= rows[:, None]",
     "causal = slk[None, :] < rows[:, None]", [t_anchor.test_handmade_anchor_cases,
                                               t_anchor.test_anchor_head_equals_per_block]),
    # block-aligned local window [(b+1) bq - local, (b+1) bq)
    ("local_window_shift", osel, "block_geometry", "ls = max(0, (qb + 1) * bq - local)",
     "ls = max(0, qb * bq - local)", [t_anchor.test_theta_minus_inf_is_sink_plus_local_window,
                                      t_anchor.test_handmade_anchor_cases]),
    # step grouping stays inside the block's own candidate range
    ("step_union_unclipped", osel, "step_union",
     "return keys[(keys >= cand_lo) & (keys < cand_hi)]", "return keys",
     [t_anchor.test_step_grouping_pins]),
    # SALE Eq. (4) as corrected: ln(tau el) + em, not ln(tau el + em)
    ("sale_printed_threshold", osel, "sale_threshold", "return em + np.log(tau * el)",
     "return np.log(tau * el + em)", [t_sale.test_threshold_rewrite_matches_relative_score,
                                      t_sale.test_handmade_sale_cases]),
    # int4 step: absmax / 7
    ("sale_quant_step", osel, "_quantize_rows_fp32", "seven = np.float32(7.0)",
     "seven = np.float32(8.0)", [t_sale.test_integer_inputs_quantise_exactly,
                                 t_sale.test_quantisation_properties_on_generated_data]),
    # SALE smoothing mean: summed in fp64 (not fp32) ...
    ("sale_mean_fp32_sum", osel, "sale_smooth_mean", "kh32.astype(np.float64).sum(axis=0)",
     "kh32.astype(np.float32).sum(axis=0, dtype=np.float32)",
     [t_sale.test_smoothing_mean_is_the_exact_mean_rounded_once]),
    # ... and rounded to fp32 once, after the division
    ("sale_mean_rounded_before_division", osel, "sale_smooth_mean",
     "(kh32.astype(np.float64).sum(axis=0) / float(L)).astype(np.float32)",
     "kh32.astype(np.float64).sum(axis=0).astype(np.float32) / np.float32(L)",
     [t_sale.test_smoothing_mean_is_the_exact_mean_rounded_once]),
    # FP8 smoothing: the same mean reading
    ("fp8_mean_fp32_sum", ofp8, "smooth_k", "kh32.astype(np.float64).sum(axis=0)",
     "kh32.astype(np.float32).sum(axis=0, dtype=np.float32)",
     [t_fp8.test_smoothing_mean_is_the_exact_mean_rounded_once]),
    # a block is kept when its largest relative score reaches tau
    ("sale_block_min", osel, "sale_block", "margin = excess.reshape(-1, bk).max(axis=1)",
     "margin = excess.reshape(-1, bk).min(axis=1)", [t_sale.test_handmade_sale_cases,
                                                      t_sale.test_tiny_tau_keeps_every_candidate_block]),
    # LSE = m + ln(sum exp(s - m))
    ("attn_lse_without_max", oatt, "attend_row", "float(m + np.log(den))", "float(np.log(den))",
     [t_att.test_attend_row_brute_force]),
    # the sink stays in every row's kept set
    ("attn_dropped_sink", oatt, "kept_keys_for_row", "sink_part = np.arange(0, min(sink, i + 1))",
     "sink_part = np.arange(0, 0)", [t_att.test_kept_pairs_closed_form,
                                     t_anchor.test_theta_minus_inf_is_sink_plus_local_window]),
    # decode: the window starts at the last block's local start
    ("decode_window_off_by_one", odec, "decode_keys", "np.arange(geo.ls, p + 1)",
     "np.arange(geo.ls + 1, p + 1)", [t_dec.test_decode_at_last_prefill_row_is_that_row,
                                      t_dec.test_nothing_selected_decode_is_sink_plus_window]),
    # decode: the sink prefix is part of the key set
    ("decode_dropped_sink", odec, "decode_keys", "np.arange(0, min(sink, p + 1))",
     "np.arange(0, 0)", [t_dec.test_nothing_selected_decode_is_sink_plus_window]),
    # KVpop transposed attention: exp(s - LSE)
    ("key_mass_without_lse", odec, "key_mass", "* sc - lse[n])", "* sc)",
     [t_dec.test_key_mass_equals_masked_softmax_column_sums]),
    # E4M3: round half to even
    ("e4m3_ties_away", ofp8, "e4m3_round", "q = np.rint(a[nrm] / step) * step",
     "q = np.floor(a[nrm] / step + 0.5) * step", [t_fp8.test_ties_to_even_and_saturation]),
    # E4M3: saturating at 448
    ("e4m3_no_saturation", ofp8, "e4m3_round", "out = np.minimum(out, E4M3_MAX)", "out = out",
     [t_fp8.test_ties_to_even_and_saturation]),
    # E4M3: exponent bias 7
    ("e4m3_bias", ofp8, "e4m3_decode", "2.0 ** (e - 7)", "2.0 ** (e - 8)",
     [t_fp8.test_codes_are_fixed_points_and_the_whole_range]),
    # FP8 K is smoothed by its mean before scaling
    ("fp8_k_unsmoothed", ofp8, "quantize_k", "ks = smooth_k(kh32)", "ks = kh32",
     [t_fp8.test_quantised_k_is_invariant_to_a_common_key_shift]),
    # FP8 V scale per channel (absmax over the sequence of that channel)
    ("fp8_v_scale_by_row", ofp8, "quantize_v", "scale_of(np.max(np.abs(vh32[:, c])))",
     "scale_of(np.max(np.abs(vh32[c, :])))", [t_fp8.test_dequantised_operands_within_half_a_step]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_planted_mistake_is_caught(case, monkeypatch):
    _, module, name, old, new, pins = case
    monkeypatch.setattr(module, name, _mutant(module, name, old, new))
    assert _some_pin_fails(pins), f"no pin caught the planted mistake {case[0]}"


def test_named_pins_pass_on_the_unmutated_oracle():
    # the control: the catching above is the mutation's doing, not the harness's
    pins = {fn for case in CASES for fn in case[5]}
    for fn in sorted(pins, key=lambda f: f.__name__):
        assert not _some_pin_fails([fn]), fn.__name__
