"""Seeded workload generators (CPU): determinism, shapes, rounding, NaN tails."""
import numpy as np
import torch

from grouped_query_attention_mqa_b200.workloads import (WORKLOADS, append_algorithmic_bytes, bf16_bits_to_f32,
                                                         decode_algorithmic_bytes, decode_flops, f32_to_bf16_bits,
                                                         host_inputs, kv_cache_bytes)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10.0 ** rng.integers(-8, 8, 10000),
                        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, np.inf, -np.inf], np.float32)])
    ours = f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(bf16_bits_to_f32(ours), torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16).float().numpy())
    assert f32_to_bf16_bits(np.array([np.nan], np.float32))[0] == 0x7FC0


def test_inputs_are_deterministic_and_shaped():
    wl = WORKLOADS["tiny_mqa_f32"].with_(b=3, len_lo=5, len_hi=60)
    a = host_inputs(wl, seed=1)
    b = host_inputs(wl, seed=1)
    c = host_inputs(wl, seed=2)
    for key in ("lens", "k", "v", "q", "k_new", "v_new"):
        assert np.array_equal(a[key], b[key], equal_nan=True)
    assert not np.array_equal(a["q"], c["q"])
    assert a["k"].shape == (3, 64, 1, 32) and a["q"].shape == (3, 4, 32) and a["k_new"].shape == (3, 1, 32)
    assert ((a["lens"] >= 5) & (a["lens"] <= 60)).all()
    for bi, L in enumerate(a["lens"]):
        assert np.isfinite(a["k"][bi, :L]).all() and np.isnan(a["k"][bi, L:]).all()
        assert np.isnan(a["v"][bi, L:]).all()


def test_bf16_inputs_carry_nan_tails_as_bits():
    wl = WORKLOADS["long_mqa_b64_m8k"].with_(b=2, m_max=32, len_lo=3, len_hi=30)
    a = host_inputs(wl, seed=3)
    assert a["k"].dtype == np.uint16
    L = a["lens"][0]
    assert (a["k"][0, L:] == 0x7FC0).all()
    assert np.array_equal(bf16_bits_to_f32(a["k"][0, :L]), a["k_f32"][0, :L])
    # q of the long-context workload is drawn with std 1/sqrt(128)
    assert 0.05 < a["q_f32"].std() < 0.15


def test_byte_and_flop_counts():
    wl = WORKLOADS["long_mqa_b64_m8k"]
    lens = np.full(wl.b, 4608)
    kv = 64 * 4608 * 1 * 256 * 2
    assert decode_algorithmic_bytes(wl, lens) == kv + 64 * 32 * 256 * 2
    assert append_algorithmic_bytes(wl) == 2 * 64 * 256 * 2
    assert decode_flops(wl, lens) == 64 * 4608 * 32 * 2 * 256
    # MQA at h = 32: 32 FLOP per byte of K/V (the tensor-core case)
    assert decode_flops(wl, lens) / kv == 32


def test_counts_follow_the_incremental_complexity_analysis():
    """Study notes §5 (complexity: §5.1 incremental MHA, §5.2 incremental MQA),
    with k = v = d/h: the MHA K+V cache is 2·b·n·h·d_h = 2·b·n·d and the MQA one
    2·b·n·d_h = 2·b·n·d/h; every query head still computes its own scores and
    weighted sum (h·n·d_h = n·d per sequence), so the FLOPs do not change; the
    memory-to-arithmetic term that grows with n goes from n/d to n/(d·h)."""
    b, n, h, dh, e = 4, 1000, 8, 16, 2
    d = h * dh
    assert kv_cache_bytes(b, n, h, dh, dh, e) == 2 * b * n * d * e
    assert kv_cache_bytes(b, n, 1, dh, dh, e) * h == 2 * b * n * d * e
    mha = WORKLOADS["mha_b16_m16k"].with_(b=b, h=h, g=h, d_k=dh, d_v=dh, m_max=n)
    mqa = mha.with_(g=1)
    lens = np.full(b, n)
    assert decode_flops(mha, lens) == decode_flops(mqa, lens) == b * n * h * 2 * (dh + dh)
    kv = lambda wl: decode_algorithmic_bytes(wl, lens) - b * h * 2 * dh * e   # drop q and o
    assert kv(mha) == h * kv(mqa)
    assert (kv(mha) / decode_flops(mha, lens)) / (kv(mqa) / decode_flops(mqa, lens)) == h


def test_prefill_flops_count_the_attended_pairs():
    """4·h·d FLOPs per attended (query, key) pair; the pairs are those the
    causal mask keeps (key u <= query t), or all n² without it."""
    from grouped_query_attention_mqa_b200.workloads import PrefillWorkload, prefill_flops
    for causal in (True, False):
        wl = PrefillWorkload("t", b=3, n=7, h=4, g=2, d=16, causal=causal, scale=1.0)
        keep = np.tril(np.ones((7, 7))) if causal else np.ones((7, 7))
        assert prefill_flops(wl) == 4 * 4 * 16 * int(keep.sum()) * 3


def test_beam_bytes_read_the_shared_prefix_once():
    """The beams' step moves W-1 fewer copies of each prefix than the same step
    over caches holding the prefix once per beam (the b·W-sequence layout)."""
    from grouped_query_attention_mqa_b200.workloads import BEAM_WORKLOADS, Workload, beam_algorithmic_bytes
    bw = BEAM_WORKLOADS["beam4_mqa_b64_p8k"]
    rng = np.random.default_rng(0)
    lp = rng.integers(bw.lp_lo, bw.lp_hi + 1, size=bw.b)
    ls = rng.integers(bw.ls_lo, bw.ls_hi + 1, size=bw.b * bw.W)
    copied = Workload("copied", b=bw.b * bw.W, h=bw.h, g=bw.g, d_k=bw.d, d_v=bw.d, m_max=bw.m_p + bw.m_s,
                      len_lo=1, len_hi=bw.m_p + bw.m_s, dtype="bf16", scale=bw.scale)
    lens_copied = np.repeat(lp, bw.W) + ls
    saved = (bw.W - 1) * int(lp.sum()) * bw.g * 2 * bw.d * 2
    assert decode_algorithmic_bytes(copied, lens_copied) - beam_algorithmic_bytes(bw, lp, ls) == saved
