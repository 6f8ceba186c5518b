"""Plants plausible mistakes in copies of the oracle and checks that the pins
in ``test_oracle.py`` catch every one of them (CPU only).

Each mutant is a one-line textual edit of ``oracle/oracle.cpp`` compiled into
a temporary library; the pins run against it with the default oracle swapped
out, and at least one pin must fail.
"""
import os
import tempfile

import pytest

import oracle
import tests.test_oracle as pins

MUTANTS = {
    "dropped_scale": ("acc * inv_sqrt_d", "acc"),
    "key_head_modulo": ("return i * hk / hq;", "return i % hk;"),
    "value_head_modulo": ("return i * hv / hq;", "return i % hv;"),
    "transposed_cache_index": ("K + ((bb * l_cap + j) * hk + kh) * d", "K + ((bb * hk + kh) * l_cap + j) * d"),
    "threshold_off_by_one": ("v.begin() + (N - 1), v.end()", "v.begin() + N, v.end()"),
    "strict_compare": ("sr[j] >= t_eff", "sr[j] > t_eff"),
    "softmax_sign": ("std::exp(static_cast<double>(sr[j]) - m)", "std::exp(m - static_cast<double>(sr[j]))"),
    "no_empty_set_rule": ("std::min(tau[r], m_all)", "tau[r]"),
    "refresh_phase": ("if (t % n == 0) oracle_nth_largest", "if (t % n == 1) oracle_nth_largest"),
    "value_row_of_wrong_batch": ("V + ((bb * l_cap + j) * hv + vh) * d", "V + ((j) * hv + vh) * d"),
    "missing_normalisation": ("acc[c] / denom", "acc[c]"),
}


def _pin_calls():
    return [
        lambda: pins.test_logits_match_float64_matmul(64, 8, 2, None),
        lambda: pins.test_logits_match_float64_matmul(128, 12, 1, 230),
        lambda: pins.test_threshold_matches_full_sort(257, 64),
        lambda: pins.test_threshold_matches_full_sort(31, 5),
        lambda: pins.test_threshold_counts_duplicates(),
        lambda: pins.test_select_definition_and_empty_set_reading(),
        lambda: pins.test_N_at_least_l_is_full_attention(8, 2, 4, 64),
        lambda: pins.test_hk_equal_hv_is_grouped_query_attention(),
        lambda: pins.test_refresh_every_step_is_exact_topN(),
        lambda: pins.test_kept_weights_sum_to_one(),
        lambda: pins.test_N1_unique_max_returns_that_value_row(),
        lambda: pins.test_zero_query_keeps_everything_and_averages(),
        lambda: pins.test_reuse_steps_keep_the_refresh_threshold(),
        lambda: pins.test_worked_example_closed_form(),
    ]


@pytest.fixture(scope="module")
def source():
    return open(oracle.SOURCE).read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, source, monkeypatch):
    old, new = MUTANTS[name]
    assert source.count(old) >= 1, f"mutation site for {name} not found"
    with tempfile.TemporaryDirectory() as tmp:
        src = os.path.join(tmp, "mutant.cpp")
        with open(src, "w") as f:
            f.write(source.replace(old, new))
        lib = oracle.compile_library(src, os.path.join(tmp, "libmutant.so"))
        monkeypatch.setattr(oracle, "_default", oracle.Oracle(lib))
        failures = 0
        for call in _pin_calls():
            try:
                call()
            except AssertionError:
                failures += 1
        assert failures > 0, f"no pin caught the planted mistake '{name}'"


def test_unmutated_oracle_passes_the_same_calls():
    for call in _pin_calls():
        call()
