"""mqa_prefill on the GPU against the float64 oracle: packed sequences whose
lengths sit at the 128-key tile edges, MQA / GQA / MHA and group widths from
1 to 128 query heads per K/V head, with and without the causal mask."""
import math

import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from grouped_query_attention_mqa_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
from oracle import oracle_decode, oracle_prefill

from gpu_util import assert_close, dev, host64

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


def packed_inputs(lens, h, g, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    T = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    out = {"cu": cu, "T": T}
    for name, shape in (("q", (T, h, D)), ("k", (T, g, D)), ("v", (T, g, D))):
        bits = f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))
        out[name] = bits
        out[name + "_f32"] = bf16_bits_to_f32(bits)
    return out


def run(inp, h, g, causal, scale):
    cu = torch.from_numpy(inp["cu"]).cuda()
    lens = np.diff(inp["cu"])
    o = binding.prefill(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"), cu, int(lens.max()),
                        scale, causal=causal)
    torch.cuda.synchronize()
    return host64(o)


@pytest.mark.parametrize("h,g", [(8, 1), (32, 1), (16, 2), (64, 8), (8, 8), (4, 1), (128, 1)])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_matches_oracle(h, g, causal):
    lens = [1, 127, 128, 129, 300, 2]
    inp = packed_inputs(lens, h, g, seed=h + g + causal)
    scale = 1 / math.sqrt(D)
    o = run(inp, h, g, causal, scale)
    ref, _ = oracle_prefill(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["cu"], g, scale, causal=causal)
    assert_close(o, ref, "bf16", f"h={h} g={g} causal={causal}")


@pytest.mark.parametrize("h,g", [(32, 1), (8, 8)])
def test_prefill_first_position_returns_its_v_row(h, g):
    """Causal position 0 sees one key: o = v[0] rounded once, bit for bit."""
    lens = [5, 200, 1]
    inp = packed_inputs(lens, h, g, seed=7)
    cu = torch.from_numpy(inp["cu"]).cuda()
    o = binding.prefill(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"), cu, 200, 0.1)
    o = o.view(torch.int16).cpu().numpy().view(np.uint16)
    for a in inp["cu"][:-1]:
        for i in range(h):
            np.testing.assert_array_equal(o[a, i], inp["v"][a, i // (h // g)])


def test_prefill_long_sequences_sampled():
    """Four 2000-token MQA sequences (h=32): sampled positions checked one by
    one against the decode oracle over their causal prefix."""
    h, g = 32, 1
    lens = [2000, 1500, 2047, 700]
    inp = packed_inputs(lens, h, g, seed=11)
    scale = 1 / math.sqrt(D)
    o = run(inp, h, g, True, scale)
    rng = np.random.default_rng(3)
    for si, n in enumerate(lens):
        a = int(inp["cu"][si])
        for t in sorted(set(rng.integers(0, n, size=6).tolist()) | {0, n - 1}):
            ref, _ = oracle_decode(inp["q_f32"][a + t][None], inp["k_f32"][a:a + t + 1][None],
                                   inp["v_f32"][a:a + t + 1][None], [t + 1], g, scale)
            assert_close(o[a + t][None], ref, "bf16", f"seq {si} pos {t}")


def test_prefill_lengths_past_the_limits_are_cut_and_flagged():
    """A sequence longer than max_seqlen is cut there (flag set); rows past the
    cut keep what the output held."""
    h, g = 8, 1
    lens = [100, 60]
    inp = packed_inputs(lens, h, g, seed=13)
    cu = torch.from_numpy(inp["cu"]).cuda()
    out = torch.full((inp["T"], h, D), 7.0, dtype=torch.bfloat16, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.prefill(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"), cu, 80, 0.1, out=out,
                    status_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & binding.MQA_FLAG_LEN_CLAMPED
    o = host64(out)
    assert (o[80:100] == 7.0).all()                  # positions 80..99 of sequence 0 untouched
    ref, _ = oracle_prefill(inp["q_f32"][:80], inp["k_f32"][:80], inp["v_f32"][:80], [0, 80], g, 0.1)
    assert_close(o[:80], ref, "bf16", "cut sequence")
    ref, _ = oracle_prefill(inp["q_f32"][100:], inp["k_f32"][100:], inp["v_f32"][100:], [0, 60], g, 0.1)
    assert_close(o[100:], ref, "bf16", "second sequence")


def test_prefill_empty_batch_is_a_no_op():
    q = torch.zeros((0, 8, D), dtype=torch.bfloat16, device="cuda")
    o = binding.prefill(q, q[:, :1], q[:, :1], torch.zeros(1, dtype=torch.int32, device="cuda"), 0, 1.0)
    assert o.shape == (0, 8, D)


@pytest.mark.parametrize("name", ["prefill_mqa_b8_n4096", "prefill_gqa8_b4_n8192"])
def test_prefill_bench_sizes_sampled(name):
    """The bench's prefill workloads at full size, in the launch the bench
    times: per sequence, positions in the first and in the last query tile
    (the end of the sequence included), at 128-key tile edges and at random,
    each against the decode oracle over its causal prefix."""
    from grouped_query_attention_mqa_b200.workloads import PREFILL_WORKLOADS, prefill_device_inputs
    wl = PREFILL_WORKLOADS[name]
    inp = prefill_device_inputs(wl, seed=5, device="cuda")
    o = binding.prefill(inp["q"], inp["k"], inp["v"], inp["cu"], wl.n, wl.scale, causal=wl.causal)
    torch.cuda.synchronize()
    kf = inp["k"].float().cpu().numpy()
    vf = inp["v"].float().cpu().numpy()
    rng = np.random.default_rng(17)
    n = wl.n
    rows_per_tile = 128 // (wl.h // wl.g)       # positions per 128-row query tile of one K/V group
    for si in range(wl.b):
        a = si * n
        picks = {0, 1, rows_per_tile - 1, 127, 128, n - rows_per_tile, n - 2, n - 1}
        picks |= set(rng.integers(0, n, size=6).tolist())
        for t in sorted(p for p in picks if 0 <= p < n):
            qt = inp["q"][a + t].float().cpu().numpy()[None]
            ref, _ = oracle_decode(qt, kf[a:a + t + 1][None], vf[a:a + t + 1][None], [t + 1], wl.g, wl.scale)
            assert_close(host64(o[a + t])[None], ref, "bf16", f"{name} seq {si} pos {t}")
    del inp, o
    torch.cuda.empty_cache()
