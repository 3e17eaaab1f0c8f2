"""Full-size workloads in the launch configuration the bench times (default
path and CTA count): one step = append at row lens-1 (mqa_kv_append), then
decode over lens rows (mqa_decode).  Every sequence's output is checked
against the oracle, which recomputes it from a fresh draw of the same seeded
inputs."""
import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from grouped_query_attention_mqa_b200.workloads import WORKLOADS, device_inputs

from gpu_util import check_full_size_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


@pytest.mark.parametrize("name", ["long_mqa_b64_m8k", "gqa8_b32_m32k", "mqa_b16_m16k", "mha_b16_m16k",
                                  "long_mqa_d64_b64_m8k"])
def test_full_size_step_every_sequence(name):
    wl = WORKLOADS[name]
    inp = device_inputs(wl, seed=3, device="cuda")
    lens = inp["lens"]
    K, V = inp["k"][0], inp["v"][0]
    pos = torch.from_numpy(lens - 1).cuda()
    binding.kv_append(K, V, inp["k_new"], inp["v_new"], pos)
    o = binding.decode(inp["q"], K, V, torch.from_numpy(lens).cuda(), wl.scale)
    torch.cuda.synchronize()
    check_full_size_step(o, wl, 3, lens, name, K, V, inp["k_new"], inp["v_new"])
    del inp, K, V, o
    torch.cuda.empty_cache()


def test_mha_vs_mqa_cache_bytes_on_device():
    """The MHA point holds exactly h = 32 times the MQA point's cache bytes."""
    mha, mqa = WORKLOADS["mha_b16_m16k"], WORKLOADS["mqa_b16_m16k"]
    a = device_inputs(mha.with_(m_max=64), seed=1, device="cuda")
    c = device_inputs(mqa.with_(m_max=64), seed=1, device="cuda")
    nbytes = lambda d: sum(t.numel() * t.element_size() for t in d["k"] + d["v"])
    assert nbytes(a) == 32 * nbytes(c)
