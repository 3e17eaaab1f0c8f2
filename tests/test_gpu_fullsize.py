"""Full-size workloads in the launch configuration the bench times (default
path and CTA count): one step = append at row lens-1, then decode over lens.
The oracle recomputes sampled sequences one by one from copies of their rows
taken before the step; every output must be finite."""
import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from grouped_query_attention_mqa_b200.workloads import WORKLOADS, device_inputs
from oracle import oracle_decode_step

from gpu_util import assert_close, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


def _sample(lens, k=3):
    order = np.argsort(lens)
    picks = {0, len(lens) - 1, int(order[-1]), int(order[0]), len(lens) // 2}
    return sorted(picks)[: max(k, 5)]


@pytest.mark.parametrize("name", ["long_mqa_b64_m8k", "gqa8_b32_m32k", "mqa_b16_m16k", "mha_b16_m16k"])
def test_full_size_step_sampled(name):
    wl = WORKLOADS[name]
    inp = device_inputs(wl, seed=3, device="cuda")
    lens = inp["lens"]
    K, V = inp["k"][0], inp["v"][0]
    picks = _sample(lens)
    before = {bi: (K[bi, : lens[bi]].float().cpu().numpy(), V[bi, : lens[bi]].float().cpu().numpy()) for bi in picks}
    pos = torch.from_numpy(lens - 1).cuda()
    binding.kv_append(K, V, inp["k_new"], inp["v_new"], pos)
    o = binding.decode(inp["q"], K, V, torch.from_numpy(lens).cuda(), wl.scale)
    out = host64(o)
    assert np.isfinite(out).all()
    qf = inp["q"].float().cpu().numpy()
    knf = inp["k_new"].float().cpu().numpy()
    vnf = inp["v_new"].float().cpu().numpy()
    for bi in picks:
        Kb, Vb = before[bi]
        L = int(lens[bi])
        ref, _, _, _ = oracle_decode_step(qf[bi:bi + 1], Kb[None], Vb[None], knf[bi:bi + 1], vnf[bi:bi + 1],
                                          np.array([L - 1]), wl.g, wl.scale)
        assert_close(out[bi:bi + 1], ref, wl.dtype, f"{name} seq {bi} len {L}")
    del inp, K, V, o
    torch.cuda.empty_cache()


def test_mha_vs_mqa_cache_bytes_on_device():
    """The MHA point holds exactly h = 32 times the MQA point's cache bytes."""
    mha, mqa = WORKLOADS["mha_b16_m16k"], WORKLOADS["mqa_b16_m16k"]
    a = device_inputs(mha.with_(m_max=64), seed=1, device="cuda")
    c = device_inputs(mqa.with_(m_max=64), seed=1, device="cuda")
    nbytes = lambda d: sum(t.numel() * t.element_size() for t in d["k"] + d["v"])
    assert nbytes(a) == 32 * nbytes(c)
