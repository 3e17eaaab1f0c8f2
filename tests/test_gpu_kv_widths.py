"""Keys and values of different widths (d_k != d_v).

The paper's per-head sizes are k for queries and keys and v for values and
outputs, and nothing in the method ties them together ("Fast Transformer
Decoding", velog paper review §2.4 and §3: logits over the k axis, outputs
over the v axis).  Every pairing of d_k, d_v in {32, 64, 128} is built on the
CUDA-core path; the tensor-core path takes bf16 pairings of 64 and 128, and
the automatic choice takes it there.  Each bf16 case runs on the automatic
choice and on the CUDA-core path.  Compared element
by element with the float64 oracle on seeded inputs whose masked rows hold
NaN, with sequences split between CTAs (merge) and kept whole, through the
fused append + decode step (cache bits checked exactly), the local window and
the no-allocation entry point."""
import ctypes
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


def wl_of(dtype, b, h, g, d_k, d_v, m_max, lo, hi):
    return Workload(f"kv_{dtype}_{b}_{h}_{g}_{d_k}_{d_v}_{m_max}", b=b, h=h, g=g, d_k=d_k, d_v=d_v, m_max=m_max,
                    len_lo=lo, len_hi=hi, dtype=dtype, scale=1 / math.sqrt(d_k))


SHAPES = [
    # dtype, b, h, g, d_k, d_v, m_max, len_lo, len_hi
    ("bf16", 4, 8, 2, 64, 128, 300, 1, 300),      # GQA h/g = 4, wider values
    ("bf16", 3, 4, 1, 128, 32, 200, 60, 200),     # MQA, narrower values
    ("bf16", 2, 32, 1, 32, 128, 513, 129, 513),   # MQA h = 32: h/g * d_v = 4096, the path's limit
    ("bf16", 3, 16, 16, 128, 64, 257, 1, 257),    # MHA
    ("f32", 3, 8, 8, 32, 64, 257, 100, 257),      # MHA
    ("f32", 2, 16, 1, 128, 64, 700, 300, 700),    # MQA h = 16
    ("f32", 5, 4, 2, 64, 32, 150, 1, 150),        # GQA h/g = 2
]


@pytest.mark.parametrize("path", ["auto", "simt"])
@pytest.mark.parametrize("num_ctas", [0, 1, 5])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "_".join(map(str, s[:7])))
def test_unequal_widths_match_oracle(shape, num_ctas, path):
    wl = wl_of(*shape)
    if path == "simt" and wl.dtype == "f32":
        pytest.skip("fp32 always takes the CUDA-core path")
    inp = host_inputs(wl, seed=7 + num_ctas, nan_tail=True)
    o = binding.decode(dev(inp["q"], wl.dtype), dev(inp["k"], wl.dtype), dev(inp["v"], wl.dtype),
                       torch.from_numpy(inp["lens"]).cuda(), wl.scale, num_ctas=num_ctas, path=path)
    torch.cuda.synchronize()
    assert tuple(o.shape) == (wl.b, wl.h, wl.d_v)
    ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["lens"], wl.g, wl.scale)
    assert_close(host64(o), ref, wl.dtype, f"ctas={num_ctas}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_single_tile_sequences_unequal_widths(dtype):
    """m_max within one tile: no merge follows, the decode writes every row,
    and an empty sequence gets zeros over d_v columns."""
    wl = wl_of(dtype, 5, 8, 2, 128, 64, 64, 1, 64)
    lens = np.array([1, 64, 0, 33, 63], np.int32)
    inp = host_inputs(wl, seed=3, nan_tail=True, lens=lens)
    o = binding.decode(dev(inp["q"], dtype), dev(inp["k"], dtype), dev(inp["v"], dtype),
                       torch.from_numpy(lens).cuda(), wl.scale)
    torch.cuda.synchronize()
    ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, wl.g, wl.scale)
    out = host64(o)
    assert np.all(out[2] == 0.0)
    assert_close(out, ref, dtype, "single tile")


@pytest.mark.parametrize("case", [("bf16", 4, 8, 1, 64, 128, 300, [1, 64, 65, 300]),
                                  ("f32", 3, 4, 2, 128, 32, 200, [2, 129, 200])],
                         ids=lambda c: "_".join(map(str, c[:7])))
def test_fused_step_unequal_widths(case):
    """The new row of each sequence is written into both caches (bit for bit)
    by the CTA that stages it, and the step's output matches the oracle step."""
    dtype, b, h, g, d_k, d_v, m_max, lens = case
    wl = wl_of(dtype, b, h, g, d_k, d_v, m_max, 1, m_max)
    lens = np.array(lens, np.int32)
    for ctas in (0, 1, 3):
        inp = host_inputs(wl, seed=int(lens.sum()) + ctas, nan_tail=True, lens=lens - 1)
        K, V = dev(inp["k"], dtype), dev(inp["v"], dtype)
        o = binding.decode_append(dev(inp["q"], dtype), K, V, dev(inp["k_new"], dtype), dev(inp["v_new"], dtype),
                                  torch.from_numpy(lens).cuda(), wl.scale, num_ctas=ctas)
        torch.cuda.synchronize()
        ref, _, _, _ = oracle_decode_step(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["k_new_f32"],
                                          inp["v_new_f32"], lens - 1, g, wl.scale)
        assert_close(host64(o), ref, dtype, f"ctas={ctas}")
        Kb, Vb = oracle_kv_append(inp["k"], inp["v"], inp["k_new"], inp["v_new"], lens - 1)
        view = np.uint16 if dtype == "bf16" else np.uint32
        assert np.array_equal(bits(K), Kb.view(view)) and np.array_equal(bits(V), Vb.view(view))


def test_window_unequal_widths():
    wl = wl_of("bf16", 4, 8, 2, 32, 128, 400, 1, 400)
    lens = np.array([1, 100, 257, 400], np.int32)
    inp = host_inputs(wl, seed=11, nan_tail=True, lens=lens)
    for window in (1, 64, 100):
        o = binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                           torch.from_numpy(lens).cuda(), wl.scale, window=window, num_ctas=7)
        torch.cuda.synchronize()
        ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, wl.g, wl.scale, window=window)
        assert_close(host64(o), ref, "bf16", f"window={window}")


def test_tensor_core_path_takes_head_sizes_64_and_128_only():
    """Keys and values of 64 or 128 columns, in any pairing, are served by the
    tensor-core path; a 32-column head is not (it stays on the CUDA cores)."""
    wl = wl_of("bf16", 1, 8, 1, 32, 128, 16, 1, 16)
    inp = host_inputs(wl, seed=1)
    with pytest.raises(binding.MqaError) as e:
        binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                       torch.from_numpy(inp["lens"]).cuda(), wl.scale, path="tcgen05")
    assert e.value.status == binding.MQA_ERR_UNSUPPORTED


def test_noalloc_unequal_widths():
    lib = binding.lib()
    wl = wl_of("bf16", 3, 16, 2, 64, 128, 500, 1, 500)
    inp = host_inputs(wl, seed=5, nan_tail=True)
    q, K, V = dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16")
    lens = torch.from_numpy(inp["lens"]).cuda()
    out = torch.full((wl.b, wl.h, wl.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.mqa_decode_noalloc(p(out), p(q), p(K), p(V), p(lens), wl.b, wl.h, wl.g, wl.m_max, wl.d_k, wl.d_v,
                                wl.scale, binding.MQA_BF16, None, stream)
    assert st == binding.MQA_OK
    torch.cuda.synchronize()
    ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["lens"], wl.g, wl.scale)
    assert_close(host64(out), ref, "bf16", "noalloc")
