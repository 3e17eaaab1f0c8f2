"""Local-window decode on the GPU against the float64 oracle: each sequence
attends to its newest `window` rows only ("Fast Transformer Decoding" study
notes §6.1, §6.4).  Rows before the window and after the sequence hold NaN,
so a kernel that read one of them would fail.  Both paths, windows shorter
and longer than the sequences and at the 128-row tile edges, split and whole
sequences, and the fused append step."""
import math

import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from grouped_query_attention_mqa_b200.workloads import WORKLOADS, Workload, host_inputs
from oracle import oracle_decode, oracle_decode_step

from gpu_util import assert_close, dev, host64

pytestmark = pytest.mark.gpu

WINDOWS = [1, 7, 32, 127, 128, 129, 300, 100000]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


def _wl(b, h, g, m_max, dtype="bf16", d=128):
    return Workload(f"win_{b}_{h}_{g}_{m_max}", b=b, h=h, g=g, d_k=d, d_v=d, m_max=m_max, len_lo=1, len_hi=m_max,
                    dtype=dtype, scale=1 / math.sqrt(d))


def _poison_before_window(inp, window):
    """NaN in the cache rows before each sequence's window (the rows after the
    sequence are NaN already)."""
    for key in ("k", "v"):
        arr = inp[key]
        nan = np.uint16(0x7FC0) if arr.dtype == np.uint16 else np.float32("nan")
        for bi, L in enumerate(inp["lens"]):
            lo = max(0, int(L) - window)
            arr[bi, :lo] = nan


@pytest.mark.parametrize("path,h,g", [("tcgen05", 32, 1), ("tcgen05", 16, 2), ("simt", 8, 1), ("simt", 8, 4)])
@pytest.mark.parametrize("window", WINDOWS)
def test_window_matches_oracle(path, h, g, window):
    wl = _wl(6, h, g, 700)
    lens = np.array([700, 1, 129, 300, 64, 513], np.int32)
    inp = host_inputs(wl, seed=window + h + g, nan_tail=True, lens=lens)
    _poison_before_window(inp, window)
    for ctas in (0, 1, 5, 40):
        o = binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                           torch.from_numpy(lens).cuda(), wl.scale, path=path, num_ctas=ctas, window=window)
        ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, g, wl.scale, window=window)
        assert_close(host64(o), ref, "bf16", f"{path} window={window} ctas={ctas}")


@pytest.mark.parametrize("path", ["tcgen05", "simt"])
def test_window_one_returns_the_newest_v_row(path):
    """With window 1 every head returns its group's V row at lens-1, rounded to
    bf16 once: bit-exact against the cache row."""
    wl = _wl(5, 16, 2, 400)
    lens = np.array([400, 1, 128, 129, 250], np.int32)
    inp = host_inputs(wl, seed=11, nan_tail=True, lens=lens)
    _poison_before_window(inp, 1)
    o = binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                       torch.from_numpy(lens).cuda(), wl.scale, path=path, window=1)
    o = o.view(torch.int16).cpu().numpy().view(np.uint16)
    for bi, L in enumerate(lens):
        for i in range(wl.h):
            np.testing.assert_array_equal(o[bi, i], inp["v"][bi, L - 1, i // (wl.h // wl.g)])


@pytest.mark.parametrize("path", ["tcgen05", "simt"])
@pytest.mark.parametrize("window", [1, 32, 200])
def test_fused_step_with_window(path, window):
    """mqa_decode_append with a window: the appended row is the newest, so it is
    always attended; the cache holds it afterwards."""
    wl = _wl(4, 16, 1, 600)
    before = np.array([599, 0, 127, 300], np.int32)
    inp = host_inputs(wl, seed=window, nan_tail=True, lens=before + 1)
    K, V = dev(inp["k"], "bf16"), dev(inp["v"], "bf16")
    o = binding.decode_append(dev(inp["q"], "bf16"), K, V, dev(inp["k_new"], "bf16"), dev(inp["v_new"], "bf16"),
                              torch.from_numpy(before + 1).cuda(), wl.scale, path=path, window=window)
    ref, _, k2, v2 = oracle_decode_step(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["k_new_f32"],
                                        inp["v_new_f32"], before, wl.g, wl.scale, window=window)
    assert_close(host64(o), ref, "bf16", f"{path} window={window}")
    kb = K.view(torch.int16).cpu().numpy().view(np.uint16)
    for bi, p in enumerate(before):
        np.testing.assert_array_equal(kb[bi, p], inp["k_new"][bi])


def test_window_at_full_size_sampled():
    """The long-context MQA batch (b=64, h=32, m_max=8192) with a 1024-row
    window, in the launch configuration the bench uses; eight sequences are
    checked against the oracle."""
    wl = WORKLOADS["long_mqa_b64_m8k"]
    inp = host_inputs(wl, seed=5, nan_tail=False)
    window = 1024
    o = host64(binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                              torch.from_numpy(inp["lens"]).cuda(), wl.scale, window=window))
    pick = np.random.default_rng(5).choice(wl.b, size=8, replace=False)
    for bi in pick:
        L = int(inp["lens"][bi])
        lo = max(0, L - window)
        ref, _ = oracle_decode(inp["q_f32"][bi:bi + 1], inp["k_f32"][bi:bi + 1, lo:L], inp["v_f32"][bi:bi + 1, lo:L],
                               [L - lo], wl.g, wl.scale)
        assert_close(o[bi:bi + 1], ref, "bf16", f"seq {bi}")
