"""The one-segment-per-CTA decode: when every attended span fits one 128-row
tile and there are no more (sequence, K/V head) segments than CTAs, CTA c
takes segment c whole and no schedule is computed.

This is the incremental decoder of the study notes' §6.2 (Table 2: a
decoder stepping one position at a time over caches of at most 128 rows,
with MQA's single K/V head of the review's §3).  Compared element by element
with the float64 oracle on inputs whose masked rows hold NaN; the outputs must
also equal, bit for bit, those of the general kernel run on few CTAs (each
segment is still processed whole there, in the same arithmetic order)."""
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


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


def wl_of(b, h, g, d_k, d_v, m_max):
    return Workload(f"one_{b}_{h}_{g}_{d_k}_{d_v}_{m_max}", b=b, h=h, g=g, d_k=d_k, d_v=d_v, m_max=m_max,
                    len_lo=1, len_hi=m_max, dtype="bf16", scale=1 / math.sqrt(d_k))


def decode(wl, inp, lens, **kw):
    o = binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                       torch.from_numpy(lens).cuda(), wl.scale, path="tcgen05", **kw)
    torch.cuda.synchronize()
    return host64(o)


def sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("widths", [(128, 128), (64, 64), (128, 64)], ids=lambda w: f"dk{w[0]}_dv{w[1]}")
@pytest.mark.parametrize("b,h,g", [(36, 32, 4), (128, 8, 1), (2, 64, 1), (20, 64, 2)])
def test_one_segment_per_cta_matches_oracle(b, h, g, widths):
    d_k, d_v = widths
    assert b * g <= sms()
    wl = wl_of(b, h, g, d_k, d_v, 128)
    rng = np.random.default_rng(b * h + g + d_k + d_v)
    lens = rng.integers(0, 129, size=b).astype(np.int32)
    lens[::5] = 0
    lens[1::7] = 128
    lens[2::11] = 1
    inp = host_inputs(wl, seed=b + h, nan_tail=True, lens=np.maximum(lens, 1))
    ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, g, wl.scale)
    one = decode(wl, inp, lens)
    assert_close(one, ref, "bf16", f"b={b} h={h} g={g}")
    assert (one[lens == 0] == 0).all()
    general = decode(wl, inp, lens, num_ctas=7)
    assert np.array_equal(one, general)


def test_segment_count_at_and_past_the_cta_count():
    """b*g equal to the SM count takes the one-segment kernel, one more takes
    the general schedule; both match the oracle."""
    n = sms()
    for b in (n, n + 1):
        wl = wl_of(b, 8, 1, 128, 128, 128)
        lens = np.random.default_rng(b).integers(1, 129, size=b).astype(np.int32)
        lens[-1] = 128
        inp = host_inputs(wl, seed=b, nan_tail=True, lens=lens)
        ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, 1, wl.scale)
        assert_close(decode(wl, inp, lens), ref, "bf16", f"b={b}")


def test_one_segment_window():
    """Caches longer than a tile with a window of at most one tile: the span is
    the newest rows, still one tile per segment."""
    wl = wl_of(24, 32, 2, 128, 128, 700)
    lens = np.random.default_rng(3).integers(1, 701, size=24).astype(np.int32)
    lens[0], lens[1], lens[2] = 1, 128, 700
    inp = host_inputs(wl, seed=7, nan_tail=True, lens=lens)
    for window in (1, 32, 128):
        ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, wl.g, wl.scale, window=window)
        assert_close(decode(wl, inp, lens, window=window), ref, "bf16", f"window={window}")


@pytest.mark.parametrize("widths", [(128, 128), (64, 64)], ids=lambda w: f"dk{w[0]}_dv{w[1]}")
def test_one_segment_fused_step(widths):
    """The fused append + decode on the one-segment kernel: the new row lands
    in both caches bit for bit and the output is the oracle step's."""
    d_k, d_v = widths
    wl = wl_of(40, 16, 2, d_k, d_v, 128)
    lens = np.random.default_rng(11).integers(1, 129, size=40).astype(np.int32)
    lens[0], lens[1] = 1, 128
    inp = host_inputs(wl, seed=12, nan_tail=True, lens=lens - 1)
    K, V = dev(inp["k"], "bf16"), dev(inp["v"], "bf16")
    o = binding.decode_append(dev(inp["q"], "bf16"), K, V, dev(inp["k_new"], "bf16"), dev(inp["v_new"], "bf16"),
                              torch.from_numpy(lens).cuda(), wl.scale, path="tcgen05")
    torch.cuda.synchronize()
    ref, _, _, _ = oracle_decode_step(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["k_new_f32"],
                                      inp["v_new_f32"], lens - 1, wl.g, wl.scale)
    assert_close(host64(o), ref, "bf16", "fused")
    Kb, Vb = oracle_kv_append(inp["k"], inp["v"], inp["k_new"], inp["v_new"], lens - 1)
    assert np.array_equal(bits(K), Kb) and np.array_equal(bits(V), Vb)
