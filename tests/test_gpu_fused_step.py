"""mqa_decode_append, the fused incremental step (append the new K/V row at
lens-1, then attend over lens rows), against the oracle's step: the output
within tolerance and the caches bit for bit.  The cache rows from lens-1 on
hold NaN before the call, so attending to a stale row instead of the new one
shows up."""
import math

import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from grouped_query_attention_mqa_b200.workloads import WORKLOADS, Workload, bf16_bits_to_f32, device_inputs, host_inputs
from oracle import oracle_decode, oracle_decode_step, oracle_kv_append

from gpu_util import assert_close, bits, check_full_size_step, dev, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


def step_inputs(wl, seed, lens):
    inp = host_inputs(wl, seed, nan_tail=True, lens=np.asarray(lens, np.int32) - 1)   # NaN from row lens-1 on
    return inp


CASES = [
    ("tcgen05", "bf16", 4, 32, 1, 128, 700, [1, 128, 129, 700]),
    ("tcgen05", "bf16", 3, 64, 8, 128, 400, [200, 257, 400]),
    ("tcgen05", "bf16", 5, 16, 2, 128, 300, [2, 65, 127, 256, 300]),
    ("simt", "bf16", 4, 8, 8, 128, 300, [1, 64, 65, 300]),
    ("simt", "bf16", 3, 4, 1, 64, 200, [63, 64, 200]),
    ("simt", "f32", 3, 4, 2, 32, 150, [1, 100, 150]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "_".join(map(str, c[:7])))
def test_fused_step_matches_oracle_step(case):
    path, dtype, b, h, g, d, m_max, lens = case
    wl = Workload("fused", b=b, h=h, g=g, d_k=d, d_v=d, m_max=m_max, len_lo=1, len_hi=m_max, dtype=dtype,
                  scale=1 / math.sqrt(d))
    lens = np.array(lens, np.int32)
    for ctas in (0, 1, 3, 7):
        inp = step_inputs(wl, seed=int(lens.sum()) + ctas, lens=lens)
        K, V = dev(inp["k"], dtype), dev(inp["v"], dtype)
        o = binding.decode_append(dev(inp["q"], dtype), K, V, dev(inp["k_new"], dtype), dev(inp["v_new"], dtype),
                                  torch.from_numpy(lens).cuda(), wl.scale, path=path, num_ctas=ctas)
        torch.cuda.synchronize()
        ref, _, K2, V2 = oracle_decode_step(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["k_new_f32"],
                                            inp["v_new_f32"], lens - 1, g, wl.scale)
        assert_close(host64(o), ref, dtype, f"{path} ctas={ctas}")
        Kb, Vb = oracle_kv_append(inp["k"], inp["v"], inp["k_new"], inp["v_new"], lens - 1)
        view = np.uint16 if dtype == "bf16" else np.uint32
        assert np.array_equal(bits(K), Kb.view(view)) and np.array_equal(bits(V), Vb.view(view))


def test_fused_equals_append_then_decode():
    """One launch and the two separate calls give the same output and caches."""
    wl = Workload("f2", b=6, h=32, g=1, d_k=128, d_v=128, m_max=1000, len_lo=1, len_hi=1000, dtype="bf16",
                  scale=1 / math.sqrt(128))
    lens = np.array([1, 999, 1000, 384, 385, 17], np.int32)
    inp = step_inputs(wl, 5, lens)
    K1, V1 = dev(inp["k"], "bf16"), dev(inp["v"], "bf16")
    K2, V2 = dev(inp["k"], "bf16"), dev(inp["v"], "bf16")
    kn, vn, q = dev(inp["k_new"], "bf16"), dev(inp["v_new"], "bf16"), dev(inp["q"], "bf16")
    lt = torch.from_numpy(lens).cuda()
    o1 = binding.decode_append(q, K1, V1, kn, vn, lt, wl.scale)
    binding.kv_append(K2, V2, kn, vn, torch.from_numpy(lens - 1).cuda())
    o2 = binding.decode(q, K2, V2, lt, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(K1.view(torch.int16), K2.view(torch.int16)) and torch.equal(V1.view(torch.int16),
                                                                                  V2.view(torch.int16))
    assert_close(host64(o1), host64(o2).astype(np.float64), "bf16", "fused vs separate")


@pytest.mark.parametrize("path", ["auto", "simt"])
def test_paper_decoder_128_fused_steps(path):
    """The paper-shaped decoder (b=128, h=8, g=1, d=128) for 128 fused steps,
    the cache growing from 1 to 128 rows, each step against the oracle."""
    wl = WORKLOADS["paper_mqa_b128_m128"]
    from grouped_query_attention_mqa_b200.workloads import f32_to_bf16_bits
    rng = np.random.Generator(np.random.PCG64(12))
    b, h, g, d, m = wl.b, wl.h, wl.g, wl.d_k, wl.m_max
    K_host = np.full((b, m, g, d), 0x7FC0, np.uint16)
    V_host = K_host.copy()
    Kd, Vd = dev(K_host, "bf16"), dev(V_host, "bf16")
    for t in range(1, wl.steps + 1):
        q = f32_to_bf16_bits(rng.standard_normal((b, h, d), dtype=np.float32))
        kn = f32_to_bf16_bits(rng.standard_normal((b, g, d), dtype=np.float32))
        vn = f32_to_bf16_bits(rng.standard_normal((b, g, d), dtype=np.float32))
        lens = np.full(b, t, np.int32)
        o = binding.decode_append(dev(q, "bf16"), Kd, Vd, dev(kn, "bf16"), dev(vn, "bf16"),
                                  torch.from_numpy(lens).cuda(), wl.scale, path=path)
        K_host, V_host = oracle_kv_append(K_host, V_host, kn, vn, lens - 1)
        ref, _ = oracle_decode(bf16_bits_to_f32(q), bf16_bits_to_f32(K_host), bf16_bits_to_f32(V_host), lens, g,
                               wl.scale)
        assert_close(host64(o), ref, "bf16", f"step {t}")
    assert np.array_equal(bits(Kd), K_host) and np.array_equal(bits(Vd), V_host)


@pytest.mark.parametrize("name", ["long_mqa_b64_m8k", "gqa8_b32_m32k", "mqa_b16_m16k", "mha_b16_m16k",
                                  "long_mqa_d64_b64_m8k"])
def test_full_size_fused_step_every_sequence(name):
    """The bench's step (mqa_decode_append, default path and CTA count) on the
    full-size workloads; every sequence against the oracle, and the caches:
    old rows untouched, row lens-1 the step's new row."""
    wl = WORKLOADS[name]
    inp = device_inputs(wl, seed=4, device="cuda")
    lens = inp["lens"]
    K, V = inp["k"][0], inp["v"][0]
    o = binding.decode_append(inp["q"], K, V, inp["k_new"], inp["v_new"], torch.from_numpy(lens).cuda(), wl.scale)
    torch.cuda.synchronize()
    check_full_size_step(o, wl, 4, lens, name, K, V, inp["k_new"], inp["v_new"])
    del inp, K, V, o
    torch.cuda.empty_cache()
