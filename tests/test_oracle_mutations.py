"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a temporary copy of oracle/uno_oracle.c (a dropped term,
a wrong sign, a flipped comparison, a transposed index, an off-by-one count), rebuilds it
on the CPU, routes the oracle wrappers to the mutated build and requires at least one of
the pin tests to fail. The committed oracle is never modified.
"""
import tempfile
from pathlib import Path

import pytest

import oracle
from tests import test_oracle_gated_lora as pins_lora
from tests import test_oracle_noise as pins_noise
from tests import test_oracle_tv as pins_tv
from tests import test_oracle_verify as pins_verify

SRC = Path(oracle.__file__).resolve().parent / "uno_oracle.c"

PINS = [
    pins_lora.test_hand_example, pins_lora.test_ungated_rows_are_the_base_layer,
    pins_lora.test_linear_in_gate_and_scale, pins_lora.test_adapter_term_is_rank_r_in_row_space,
    pins_verify.test_warp_golden, pins_verify.test_warp_unfiltered_is_softmax,
    pins_verify.test_topk_equals_sort_selection, pins_verify.test_topp_keeps_shortest_prefix,
    pins_verify.test_inv_cdf_golden, pins_verify.test_exact_disjoint_support_always_rejects,
    pins_verify.test_greedy_top1_is_argmax_verify, pins_verify.test_position0_is_the_ar_token,
    pins_verify.test_supplied_drafts_zero_probabilities, pins_verify.test_block_of_one,
    pins_verify.test_identical_rows_accept_everything,
    pins_tv.test_identical_is_zero, pins_tv.test_range_symmetry_and_overlap_identity,
    pins_tv.test_two_token_closed_form, pins_tv.test_mean_over_mask_and_masked_gradient,
    pins_tv.test_gradient_rows_sum_to_zero, pins_tv.test_gradient_finite_differences,
    pins_noise.test_hand_example, pins_noise.test_extremes_of_the_uniform, pins_noise.test_block_of_one_keeps_the_block,
    pins_noise.test_noised_tokens_are_uniform,
]
PINS_EXACT = [lambda c=c: pins_verify.test_exact_losslessness(c) for c in range(6)]

MUTATIONS = {
    "acceptance_ratio_inverted": ("acc[i] = (ui[1] * qd < pd) ? 1 : 0;", "acc[i] = (ui[1] * pd < qd) ? 1 : 0;"),
    "acceptance_not_strict": ("acc[i] = (ui[1] * qd < pd) ? 1 : 0;", "acc[i] = (ui[1] * qd <= pd && pd > 0.0 && ui[1] > 0.3) ? 1 : 0;"),
    "residual_sign_flipped": ("double dlt = wp[v] / Zp - wq[v] / Zq;", "double dlt = wq[v] / Zq - wp[v] / Zp;"),
    "residual_not_clamped": ("res[v] = dlt > 0.0 ? dlt : 0.0;", "res[v] = fabs(dlt);"),
    "inv_cdf_non_strict": ("if (cum > target) {", "if (cum >= target) {"),
    "topk_ties_to_higher_id": ("return (a->id < b->id) ? -1 : (a->id > b->id);", "return (a->id > b->id) ? -1 : (a->id < b->id);"),
    "topp_drops_crossing_token": ("cut = j + 1;", "cut = j > 0 ? j : 1;"),
    "topp_before_normalising": ("r[nk].key = w[v] / S;", "r[nk].key = w[v];"),
    "temperature_multiplies": ("logit[v] / T", "logit[v] * T"),
    "softmax_missing_max_shift": ("w[v] = exp(logit[v] / T - zmax);", "w[v] = exp(logit[v] / T - zmax) + 1e-3;"),
    "count_includes_correction": ("int64_t n = first_reject < 0 ? K : first_reject;",
                                  "int64_t n = first_reject < 0 ? K : first_reject + 1;"),
    "position0_from_drafter": ("else x0 = oracle_inv_cdf(wp, V, Zp, ui[0], &mg[0]);",
                               "else { double Zq0 = oracle_warp_row(qrow, V, T, top_k, top_p, wq, NULL, NULL); x0 = oracle_inv_cdf(wq, V, Zq0, ui[0], &mg[0]); }"),
    "tv_missing_half": ("tv[t] = 0.5 * d;", "tv[t] = d;"),
    "grad_sign_flipped": ("grad[t * V + v] = f * q[v] * (sv - c);", "grad[t * V + v] = f * q[v] * (c - sv);"),
    "grad_missing_softmax_coupling": ("grad[t * V + v] = f * q[v] * (sv - c);", "grad[t * V + v] = f * q[v] * sv;"),
    "grad_mean_over_all_tokens": ("double f = on ? grad_scale / (double)n_mask : 0.0;",
                                  "double f = on ? grad_scale / (double)N : 0.0;"),
    "lora_gate_ignored": ("y[m * d_out + o] = base + scale * gm * lora;", "y[m * d_out + o] = base + scale * lora;"),
    "lora_scale_dropped": ("y[m * d_out + o] = base + scale * gm * lora;", "y[m * d_out + o] = base + gm * lora;"),
    "w0_transposed": ("base += xm[k] * w0[o * d_in + k];", "base += xm[k] * w0[(k * d_out + o) % (d_in * d_out)];"),
    "lora_b_index_swapped": ("lora += t[j] * b[o * rank + j];", "lora += t[j] * b[(j * d_out + o) % (d_out * rank)];"),
    "noise_position0_noised": ("            if (i == 0) {\n                out[o] = clean[o];",
                               "            if (i < 0) {\n                out[o] = clean[o];"),
    "noise_rounds_up": ("double t = floor((double)u[o] * (double)V);", "double t = ceil((double)u[o] * (double)V);"),
    "noise_not_clamped": ("if (t > (double)(V - 1)) t = (double)(V - 1);", "if (t > (double)V) t = (double)V;"),
    "noise_skips_last_token": ("double t = floor((double)u[o] * (double)V);",
                               "double t = floor((double)u[o] * (double)(V - 1));"),
}


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    old, new = MUTATIONS[name]
    src = SRC.read_text()
    assert src.count(old) >= 1, f"mutation anchor not found: {old}"
    with tempfile.TemporaryDirectory() as d:
        mut_src = Path(d) / "mutant.c"
        mut_src.write_text(src.replace(old, new))
        lib = oracle.compile_source(mut_src, Path(d) / "libmutant.so")
        with oracle.use_library(lib):
            caught = [f.__name__ if hasattr(f, "__name__") else "exact" for f in PINS + PINS_EXACT if _fails(f)]
    assert caught, f"no pin catches the planted mistake {name}"
