"""The paper-shaped decoder workload: b=128 sequences, h=8 query heads sharing
one K/V head, d=128, 128 successive steps of append + decode with the cache
growing from 1 to 128 rows; every step is compared with the oracle's step."""
import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from grouped_query_attention_mqa_b200.workloads import WORKLOADS, bf16_bits_to_f32, f32_to_bf16_bits
from oracle import oracle_decode, oracle_kv_append

from gpu_util import assert_close, bits, dev, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


@pytest.mark.parametrize("path", ["auto", "simt"])
def test_paper_decoder_128_steps(path):
    wl = WORKLOADS["paper_mqa_b128_m128"]
    rng = np.random.Generator(np.random.PCG64(2))
    b, h, g, d, m = wl.b, wl.h, wl.g, wl.d_k, wl.m_max
    K_host = np.full((b, m, g, d), 0x7FC0, np.uint16)          # NaN until written
    V_host = K_host.copy()
    Kd, Vd = dev(K_host, "bf16"), dev(V_host, "bf16")
    for t in range(1, wl.steps + 1):
        q = f32_to_bf16_bits(rng.standard_normal((b, h, d), dtype=np.float32))
        kn = f32_to_bf16_bits(rng.standard_normal((b, g, d), dtype=np.float32))
        vn = f32_to_bf16_bits(rng.standard_normal((b, g, d), dtype=np.float32))
        pos = np.full(b, t - 1, np.int32)
        binding.kv_append(Kd, Vd, dev(kn, "bf16"), dev(vn, "bf16"), torch.from_numpy(pos).cuda())
        o = binding.decode(dev(q, "bf16"), Kd, Vd, torch.from_numpy(pos + 1).cuda(), wl.scale, path=path)
        ref, K_host, V_host = _step(q, K_host, V_host, kn, vn, pos, g, wl.scale)
        assert_close(host64(o), ref, "bf16", f"step {t}")
    assert np.array_equal(bits(Kd), K_host) and np.array_equal(bits(Vd), V_host)


def _step(q, K_bits, V_bits, kn, vn, pos, g, scale):
    """Oracle step on bit patterns: the append is done on the bits (bitwise),
    the attention on their float values."""
    K2, V2 = oracle_kv_append(K_bits, V_bits, kn, vn, pos)
    o, _ = oracle_decode(bf16_bits_to_f32(q), bf16_bits_to_f32(K2), bf16_bits_to_f32(V2), pos + 1, g, scale)
    return o, K2, V2
