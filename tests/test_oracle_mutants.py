"""The oracle's pins catch plausible mistakes.  Each mutant below is a decode
written here with one slip planted (on the CPU, never in the oracle itself):
a wrong query-head -> K/V-head map, a dropped scale, no max-subtraction, rows
past the length attended, K weighted instead of V, and a step that attends
before it appends.  The pins of test_oracle.py are run against each mutant and
at least one must fail.  The same decode with no slip passes every pin, so a
failure comes from the slip and not from the harness."""
import numpy as np
import pytest

import test_oracle as T
from conftest import read_golden
from oracle import oracle_decode, oracle_kv_append

SLIPS = ["group", "no_scale", "no_max", "unmasked", "v_is_k"]


def mutant_decode(slip):
    """Scaled masked softmax attention per (sequence, head), with `slip`
    planted (None: no slip)."""
    def decode(q, k_cache, v_cache, lens, g, scale, return_weights=False, window=0):
        if window:
            raise NotImplementedError("the pins run here use no window")
        q = np.asarray(q, np.float64)
        K = np.asarray(k_cache, np.float64)
        V = np.asarray(v_cache, np.float64)
        b, h, _ = q.shape
        m, hq = K.shape[1], h // g
        o = np.zeros((b, h, V.shape[3]))
        lse = np.full((b, h), -np.inf)
        weights = []
        with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
            for bi in range(b):
                L = int(lens[bi])
                wb = np.zeros((h, max(L, 0)))
                if L > 0:
                    n = m if slip == "unmasked" else L
                    for i in range(h):
                        j = i % g if slip == "group" else i // hq
                        Kj, Vj = K[bi, :n, j], V[bi, :n, j]
                        s = (Kj @ q[bi, i]) * (1.0 if slip == "no_scale" else scale)
                        mu = 0.0 if slip == "no_max" else s.max()
                        e = np.exp(s - mu)
                        w = e / e.sum()
                        o[bi, i] = w @ (Kj if slip == "v_is_k" else Vj)
                        lse[bi, i] = mu + np.log(e.sum())
                        wb[i] = w[:L]
                weights.append(wb)
        return (o, lse, weights) if return_weights else (o, lse)
    return decode


def step_attend_then_append(q, k_cache, v_cache, k_new, v_new, lens_before, g, scale, window=0):
    """The step in the wrong order: attend over the old rows, then append."""
    o, lse = oracle_decode(q, k_cache, v_cache, lens_before, g, scale, window=window)
    k2, v2 = oracle_kv_append(k_cache, v_cache, k_new, v_new, lens_before)
    return o, lse, k2, v2


PINS = [
    ("worked example, scale 1", lambda: T.test_worked_example_two_keys_scale_one(read_golden)),
    ("worked example, scale 1/sqrt 2", lambda: T.test_worked_example_two_keys_scaled(read_golden)),
    ("shape example", lambda: T.test_shape_example(read_golden)),
] + [
    (f"per-head brute force h={h} g={g}", lambda h=h, g=g: T.test_oracle_matches_per_head_brute_force(h, g))
    for h, g in [(4, 1), (4, 2), (4, 4), (6, 3)]
] + [
    ("MQA == MHA with replicated K/V", T.test_mqa_equals_mha_with_replicated_kv),
    ("GQA == MQA per group", T.test_gqa_is_mqa_per_group),
    ("GQA-h == MHA, GQA-1 == MQA", T.test_gqa_h_is_mha_and_gqa_1_is_mqa),
    ("weights sum to one, match lse", T.test_weights_sum_to_one_and_match_lse),
    ("convex combination of V rows", T.test_output_is_a_convex_combination_of_the_valid_v_rows),
    ("length one returns V", T.test_length_one_cache_returns_v),
    ("identical keys give the mean", T.test_identical_keys_return_mean_of_v),
    ("masked rows never read", T.test_masked_rows_are_never_read),
    ("large logits pick the argmax", T.test_large_logits_are_stable_and_pick_the_argmax),
    ("scale folds into q", T.test_scale_folds_into_q),
    ("row permutation, V linearity", T.test_row_permutation_and_v_linearity),
    ("zero length", T.test_zero_length_gives_zero_row),
    ("append before attend", T.test_step_appends_before_attending),
]


def failing_pins():
    failed = []
    for name, pin in PINS:
        try:
            pin()
        except Exception:   # an assertion, or the slip's own breakage (NaN, shape)
            failed.append(name)
    return failed


def test_the_mutant_harness_without_a_slip_passes_every_pin(monkeypatch):
    monkeypatch.setattr(T, "oracle_decode", mutant_decode(None))
    assert failing_pins() == []


@pytest.mark.parametrize("slip", SLIPS)
def test_a_pin_catches_the_planted_slip(monkeypatch, slip):
    monkeypatch.setattr(T, "oracle_decode", mutant_decode(slip))
    assert failing_pins(), f"no pin fails with the slip '{slip}'"


def test_a_pin_catches_attending_before_appending(monkeypatch):
    monkeypatch.setattr(T, "oracle_decode_step", step_attend_then_append)
    assert failing_pins() == ["append before attend"]
