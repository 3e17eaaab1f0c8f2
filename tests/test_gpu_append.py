"""mqa_kv_append on the GPU: bit-exact against the oracle's scatter, nothing
else touched, out-of-range rows skipped and flagged."""
import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from oracle import oracle_kv_append

from gpu_util import bits, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


@pytest.mark.parametrize("dtype,b,m,g,d", [("bf16", 5, 40, 1, 128), ("bf16", 3, 17, 8, 64), ("f32", 4, 9, 2, 32),
                                           ("bf16", 1, 1, 1, 32), ("f32", 7, 130, 4, 128)])
def test_append_bit_exact(dtype, b, m, g, d):
    rng = np.random.default_rng(b * 100 + m)
    if dtype == "bf16":
        K = rng.integers(0, 2**16, size=(b, m, g, d), dtype=np.uint16)
        V = rng.integers(0, 2**16, size=(b, m, g, d), dtype=np.uint16)
        kn = rng.integers(0, 2**16, size=(b, g, d), dtype=np.uint16)
        vn = rng.integers(0, 2**16, size=(b, g, d), dtype=np.uint16)
    else:   # arbitrary bit patterns, NaNs included: the copy must be bitwise
        K = rng.integers(0, 2**32, size=(b, m, g, d), dtype=np.uint32).view(np.float32)
        V = rng.integers(0, 2**32, size=(b, m, g, d), dtype=np.uint32).view(np.float32)
        kn = rng.integers(0, 2**32, size=(b, g, d), dtype=np.uint32).view(np.float32)
        vn = rng.integers(0, 2**32, size=(b, g, d), dtype=np.uint32).view(np.float32)
    pos = rng.integers(0, m, size=b).astype(np.int32)
    Kd, Vd = dev(K, dtype), dev(V, dtype)
    binding.kv_append(Kd, Vd, dev(kn, dtype), dev(vn, dtype), torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    K2, V2 = oracle_kv_append(K, V, kn, vn, pos)
    view = np.uint16 if dtype == "bf16" else np.uint32
    assert np.array_equal(bits(Kd), K2.view(view))
    assert np.array_equal(bits(Vd), V2.view(view))


def test_append_out_of_range_rows_are_skipped_and_flagged():
    b, m, g, d = 4, 8, 1, 64
    K = torch.zeros((b, m, g, d), dtype=torch.bfloat16, device="cuda")
    V = torch.zeros_like(K)
    kn = torch.ones((b, g, d), dtype=torch.bfloat16, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = torch.tensor([0, -1, 8, 7], dtype=torch.int32, device="cuda")
    binding.kv_append(K, V, kn, kn, pos, status_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & binding.MQA_FLAG_POS_SKIPPED
    assert (K[0, 0] == 1).all() and (K[3, 7] == 1).all()
    assert (K[1] == 0).all() and (K[2] == 0).all()
    assert int(K.float().sum().item()) == 2 * d
    flags.zero_()
    binding.kv_append(K, V, kn, kn, torch.tensor([1, 1, 1, 1], dtype=torch.int32, device="cuda"), status_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
