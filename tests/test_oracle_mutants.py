"""The oracle's pins catch plausible mistakes.  Each mutant below is a decode,
prefill or beam step written here with one slip planted (on the CPU, never in
the oracle itself): a wrong query-head -> K/V-head map, a dropped scale, no
max-subtraction, rows past the length attended, K weighted instead of V, a local
window one row too wide, a step that attends before it appends, an append
one row off, in place or without its range check, a causal mask one row off, keys taken across
sequence boundaries, another beam's suffix, a dropped prefix.  The pins of
test_oracle.py are run against each mutant and at least one must fail.  The
same code with no slip passes every pin, so a failure comes from the slip and
not from the harness."""
import numpy as np
import pytest

import test_oracle as T
from conftest import read_golden
from oracle import oracle_decode, oracle_kv_append

SLIPS = ["group", "no_scale", "no_max", "unmasked", "v_is_k", "window_off_by_one"]


def mutant_decode(slip):
    """Scaled masked softmax attention per (sequence, head), with `slip`
    planted (None: no slip)."""
    def decode(q, k_cache, v_cache, lens, g, scale, return_weights=False, window=0):
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
                    lo = max(0, L - window) if window > 0 else 0
                    if slip == "window_off_by_one" and window > 0:
                        lo = max(0, lo - 1)
                    hi = m if slip == "unmasked" else L
                    for i in range(h):
                        j = i % g if slip == "group" else i // hq
                        Kj, Vj = K[bi, lo:hi, j], V[bi, lo:hi, j]
                        s = (Kj @ q[bi, i]) * (1.0 if slip == "no_scale" else scale)
                        mu = 0.0 if slip == "no_max" else s.max()
                        e = np.exp(s - mu)
                        w = e / e.sum()
                        o[bi, i] = w @ (Kj if slip == "v_is_k" else Vj)
                        lse[bi, i] = mu + np.log(e.sum())
                        wb[i, lo:L] = w[:L - lo]
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
    ("window 1 returns the newest V row", lambda: T.test_window_one_returns_the_newest_row_of_v(read_golden)),
    ("window covering the cache", lambda: T.test_window_covering_the_cache_is_full_attention(read_golden)),
] + [
    (f"window {w} brute force", lambda w=w: T.test_window_is_brute_force_on_the_newest_rows(w)) for w in (1, 3, 5, 32)
] + [
    ("window 32 = current + 31", T.test_notes_window_is_current_plus_31_previous),
]


def failing_pins(pins=None):
    failed = []
    for name, pin in PINS if pins is None else pins:
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


# ------------------------------------------------------------ prefill

def mutant_prefill(slip):
    """Per position t of each packed sequence: softmax attention over keys
    0..t of that sequence (all n keys without the mask), with `slip` planted."""
    def prefill(q, k, v, cu_seqlens, g, scale, causal=True):
        q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
        cu = [int(x) for x in cu_seqlens]
        T_, h, _ = q.shape
        hq = h // g
        o = np.zeros((T_, h, v.shape[2]))
        lse = np.full((T_, h), -np.inf)
        for si in range(len(cu) - 1):
            a, n = cu[si], cu[si + 1] - cu[si]
            for t in range(n):
                last = t if causal else n - 1
                if slip == "mask_off_by_one":
                    last = min(last + 1, n - 1)
                first = 0 if slip == "across_sequences" else a
                for i in range(h):
                    j = i % g if slip == "group" else i // hq
                    s = (k[first:a + last + 1, j] @ q[a + t, i]) * scale
                    mu = s.max()
                    e = np.exp(s - mu)
                    o[a + t, i] = (e / e.sum()) @ v[first:a + last + 1, j]
                    lse[a + t, i] = mu + np.log(e.sum())
        return o, lse
    return prefill


PREFILL_PINS = [
    (f"prefill brute force h={h} g={g}", lambda h=h, g=g: T.test_prefill_is_brute_force_over_the_causal_prefix(h, g))
    for h, g in [(4, 1), (4, 2), (4, 4)]
] + [
    ("prefill first position", T.test_prefill_first_position_returns_its_own_v),
    ("prefill without mask", T.test_prefill_without_mask_sees_the_whole_sequence),
    ("prefill causality", T.test_prefill_prefix_is_unchanged_by_later_tokens),
    ("prefill last position == decode", T.test_prefill_last_position_is_the_decode_step),
    ("prefill MQA == MHA", T.test_prefill_mqa_equals_mha_with_replicated_kv),
]


def test_prefill_mutant_without_a_slip_passes_every_pin(monkeypatch):
    monkeypatch.setattr(T, "oracle_prefill", mutant_prefill(None))
    assert failing_pins(PREFILL_PINS) == []


@pytest.mark.parametrize("slip", ["mask_off_by_one", "across_sequences", "group"])
def test_a_prefill_pin_catches_the_planted_slip(monkeypatch, slip):
    monkeypatch.setattr(T, "oracle_prefill", mutant_prefill(slip))
    assert failing_pins(PREFILL_PINS), f"no prefill pin fails with the slip '{slip}'"


# ------------------------------------------------------------ beams sharing a prefix

def mutant_beam(slip):
    """Beam (s, w) attends over sequence s's prefix rows, then the beam's own
    suffix rows, with `slip` planted."""
    def beam(q, prefix_k, prefix_v, prefix_lens, suffix_k, suffix_v, suffix_lens, g, scale):
        q = np.asarray(q, np.float64)
        b, W, h, _ = q.shape
        o = np.zeros((b, W, h, np.asarray(prefix_v).shape[3]))
        lse = np.full((b, W, h), -np.inf)
        for si in range(b):
            for w in range(W):
                r = si * W + ((w + 1) % W if slip == "other_beam" else w)
                lp = 0 if slip == "no_prefix" else int(prefix_lens[si])
                K = np.concatenate([prefix_k[si, :lp], suffix_k[r, :int(suffix_lens[r])]])[None]
                V = np.concatenate([prefix_v[si, :lp], suffix_v[r, :int(suffix_lens[r])]])[None]
                if K.shape[1]:
                    ob, lb = oracle_decode(q[si, w][None], K, V, [K.shape[1]], g, scale)
                    o[si, w], lse[si, w] = ob[0], lb[0]
        return o, lse
    return beam


BEAM_PINS = [
    ("beam brute force", T.test_beam_is_brute_force_over_prefix_then_suffix),
    ("beams with the same suffix agree", T.test_beams_with_the_same_suffix_agree),
    ("beam with empty suffix or prefix", T.test_beam_with_empty_suffix_or_prefix_is_plain_decode),
]


def test_beam_mutant_without_a_slip_passes_every_pin(monkeypatch):
    monkeypatch.setattr(T, "oracle_decode_beam", mutant_beam(None))
    assert failing_pins(BEAM_PINS) == []


@pytest.mark.parametrize("slip", ["other_beam", "no_prefix"])
def test_a_beam_pin_catches_the_planted_slip(monkeypatch, slip):
    monkeypatch.setattr(T, "oracle_decode_beam", mutant_beam(slip))
    assert failing_pins(BEAM_PINS), f"no beam pin fails with the slip '{slip}'"


# ------------------------------------------------------------ append

def mutant_append(slip):
    """Write k_new[b] / v_new[b] at row pos[b] of copies of the caches (rows
    outside [0, m) write nothing), with `slip` planted."""
    def append(k_cache, v_cache, k_new, v_new, pos):
        k_out = k_cache if slip == "in_place" else np.array(k_cache, copy=True)
        v_out = v_cache if slip == "in_place" else np.array(v_cache, copy=True)
        for bi, p in enumerate(int(x) for x in pos):
            p = p + 1 if slip == "row_off_by_one" else p
            if slip == "no_range_check" or 0 <= p < k_out.shape[1]:
                k_out[bi, p] = k_new[bi]
                v_out[bi, p] = v_new[bi]
        return k_out, v_out
    return append


APPEND_PINS = [
    ("append is the concat", T.test_append_is_the_concat_of_the_review),
    ("append out of range writes nothing", T.test_append_out_of_range_row_writes_nothing),
]


def test_append_mutant_without_a_slip_passes_every_pin(monkeypatch):
    monkeypatch.setattr(T, "oracle_kv_append", mutant_append(None))
    assert failing_pins(APPEND_PINS) == []


@pytest.mark.parametrize("slip", ["row_off_by_one", "in_place", "no_range_check"])
def test_an_append_pin_catches_the_planted_slip(monkeypatch, slip):
    monkeypatch.setattr(T, "oracle_kv_append", mutant_append(slip))
    assert failing_pins(APPEND_PINS), f"no append pin fails with the slip '{slip}'"
