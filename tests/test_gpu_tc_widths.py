"""The tensor-core decode at head sizes 64 and 128, keys and values of equal or
unequal widths ("Fast Transformer Decoding", velog paper review §2.1 and §3:
the per-head sizes k and v are free parameters of the method).

Compared element by element with the float64 oracle on seeded inputs whose
masked rows hold NaN: group widths h/g from 1 to 64, lengths at the 128-row
tile edges, CTA counts forced low (sequences split between CTAs, exercising
the log-sum-exp merge) and left to the library; the fused append + decode
step with the caches checked bit for bit; the local window; and the automatic
choice, which must take the tensor-core path for these head sizes in bf16."""
import math

import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from grouped_query_attention_mqa_b200.workloads import Workload, host_inputs
from oracle import oracle_decode, oracle_decode_step, oracle_kv_append

from gpu_util import assert_close, bits, dev, host64

pytestmark = pytest.mark.gpu

EDGE_LENS = [1, 2, 127, 128, 129, 255, 256, 257, 400, 513]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


def wl_of(b, h, g, d_k, d_v, m_max, lo=1, hi=None):
    return Workload(f"tc_{b}_{h}_{g}_{d_k}_{d_v}_{m_max}", b=b, h=h, g=g, d_k=d_k, d_v=d_v, m_max=m_max,
                    len_lo=lo, len_hi=hi or m_max, dtype="bf16", scale=1 / math.sqrt(d_k))


def run(wl, inp, lens, **kw):
    o = binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                       torch.from_numpy(lens).cuda(), wl.scale, **kw)
    torch.cuda.synchronize()
    return host64(o)


@pytest.mark.parametrize("widths", [(64, 64), (64, 128), (128, 64)], ids=lambda w: f"dk{w[0]}_dv{w[1]}")
@pytest.mark.parametrize("hq", [1, 8, 32, 64])
def test_tensor_cores_match_oracle_at_tile_edges(hq, widths):
    d_k, d_v = widths
    g = 2 if hq <= 32 else 1
    wl = wl_of(len(EDGE_LENS), hq * g, g, d_k, d_v, 513)
    lens = np.array(EDGE_LENS, np.int32)
    inp = host_inputs(wl, seed=hq + d_k + d_v, nan_tail=True, lens=lens)
    ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, g, wl.scale)
    for ctas in (0, 1, 3, 7):
        out = run(wl, inp, lens, path="tcgen05", num_ctas=ctas)
        assert_close(out, ref, "bf16", f"h/g={hq} d_k={d_k} d_v={d_v} ctas={ctas}")


@pytest.mark.parametrize("widths", [(64, 64), (64, 128), (128, 64)], ids=lambda w: f"dk{w[0]}_dv{w[1]}")
def test_automatic_choice_takes_tensor_cores(widths):
    """bf16 with head sizes 64/128: the automatic path is the tensor-core
    kernel (same bits as forcing it), and it matches the oracle."""
    d_k, d_v = widths
    wl = wl_of(6, 32, 1, d_k, d_v, 700)
    inp = host_inputs(wl, seed=5, nan_tail=True)
    lens = inp["lens"]
    auto = run(wl, inp, lens)
    tc = run(wl, inp, lens, path="tcgen05")
    assert np.array_equal(auto, tc)
    ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, wl.g, wl.scale)
    assert_close(auto, ref, "bf16", "auto")


@pytest.mark.parametrize("widths", [(64, 64), (128, 64)], ids=lambda w: f"dk{w[0]}_dv{w[1]}")
def test_fused_step_at_head_size_64(widths):
    """The new row goes into both caches bit for bit, and the step's output is
    the oracle step's, with sequences whole and split between CTAs."""
    d_k, d_v = widths
    wl = wl_of(5, 16, 2, d_k, d_v, 600)
    lens = np.array([1, 128, 129, 384, 600], np.int32)
    for ctas in (0, 1, 5):
        inp = host_inputs(wl, seed=int(lens.sum()) + ctas, nan_tail=True, lens=lens - 1)
        K, V = dev(inp["k"], "bf16"), dev(inp["v"], "bf16")
        o = binding.decode_append(dev(inp["q"], "bf16"), K, V, dev(inp["k_new"], "bf16"), dev(inp["v_new"], "bf16"),
                                  torch.from_numpy(lens).cuda(), wl.scale, path="tcgen05", num_ctas=ctas)
        torch.cuda.synchronize()
        ref, _, _, _ = oracle_decode_step(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["k_new_f32"],
                                          inp["v_new_f32"], lens - 1, wl.g, wl.scale)
        assert_close(host64(o), ref, "bf16", f"ctas={ctas}")
        Kb, Vb = oracle_kv_append(inp["k"], inp["v"], inp["k_new"], inp["v_new"], lens - 1)
        assert np.array_equal(bits(K), Kb) and np.array_equal(bits(V), Vb)


def test_window_at_head_size_64():
    wl = wl_of(4, 32, 1, 64, 64, 900)
    lens = np.array([1, 100, 513, 900], np.int32)
    inp = host_inputs(wl, seed=9, nan_tail=True, lens=lens)
    for window in (1, 32, 129, 600):
        out = run(wl, inp, lens, path="tcgen05", window=window, num_ctas=5)
        ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, wl.g, wl.scale, window=window)
        assert_close(out, ref, "bf16", f"window={window}")


def test_single_tile_sequences_at_head_size_64():
    """Caches of one tile: no merge follows; an empty sequence gets zeros."""
    wl = wl_of(6, 8, 1, 64, 64, 128)
    lens = np.array([1, 128, 0, 64, 127, 2], np.int32)
    inp = host_inputs(wl, seed=4, nan_tail=True, lens=lens)
    out = run(wl, inp, lens, path="tcgen05")
    ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, wl.g, wl.scale)
    assert np.all(out[2] == 0.0)
    assert_close(out, ref, "bf16", "single tile")


PAIR_EDGE_LENS = [1, 127, 128, 129, 255, 256, 257, 383, 384, 385, 511, 512, 513, 767, 768, 769]


@pytest.mark.parametrize("hq", [1, 16, 32])
def test_head_size_64_tiles_of_256_rows(hq):
    """At head size 64 with up to 32 heads per group a tile is 256 rows (two
    128-row halves in one pair of products): lengths at and around both
    half and whole tile edges, segments whole and split between CTAs."""
    g = 2
    wl = wl_of(len(PAIR_EDGE_LENS), hq * g, g, 64, 64, 769)
    lens = np.array(PAIR_EDGE_LENS, np.int32)
    inp = host_inputs(wl, seed=100 + hq, nan_tail=True, lens=lens)
    ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, g, wl.scale)
    for ctas in (0, 1, 2, 5, 11):
        out = run(wl, inp, lens, path="tcgen05", num_ctas=ctas)
        assert_close(out, ref, "bf16", f"h/g={hq} ctas={ctas}")


@pytest.mark.parametrize("hq", [8, 32])
def test_head_size_64_rescales_for_growing_logits(hq):
    """Logits growing along the sequence move the running maximum within a
    segment, in either row half of a 256-row tile, so O is rescaled in
    tensor memory (both halves' blocks of it)."""
    from grouped_query_attention_mqa_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
    wl = wl_of(3, hq, 1, 64, 64, 1100, lo=1100)
    lens = np.array([1100, 700, 300], np.int32)
    inp = host_inputs(wl, seed=31, nan_tail=True, lens=lens)
    ramp = np.linspace(0.0, 6.0, wl.m_max, dtype=np.float32)[None, :, None, None]
    k = f32_to_bf16_bits(bf16_bits_to_f32(inp["k"]) * 0 + inp["q_f32"][:, :1, None, :] * ramp * 3)
    kf = bf16_bits_to_f32(k)
    ref, _ = oracle_decode(inp["q_f32"], kf, inp["v_f32"], lens, 1, wl.scale)
    for ctas in (0, 1, 4):
        o = binding.decode(dev(inp["q"], "bf16"), dev(k, "bf16"), dev(inp["v"], "bf16"), torch.from_numpy(lens).cuda(),
                           wl.scale, path="tcgen05", num_ctas=ctas)
        torch.cuda.synchronize()
        assert_close(host64(o), ref, "bf16", f"ramp h/g={hq} ctas={ctas}")
