"""mqa_decode_beam on the GPU against the float64 oracle: W beams per sequence
share the sequence's prefix and read their own suffixes.  Cache rows past each
length hold NaN, prefix and suffix lengths sit at tile edges and at zero, and
long prefixes are split between CTAs."""
import math

import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from grouped_query_attention_mqa_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
from oracle import oracle_decode_beam

from gpu_util import assert_close, dev, host64

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


def beam_inputs(b, W, h, g, m_p, m_s, lp, ls, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    shapes = {"q": (b, W, h, D), "pk": (b, m_p, g, D), "pv": (b, m_p, g, D), "sk": (b * W, m_s, g, D),
              "sv": (b * W, m_s, g, D)}
    for name, shape in shapes.items():
        x = rng.standard_normal(shape, dtype=np.float32)
        if name in ("pk", "pv"):
            x[np.arange(m_p)[None, :] >= np.asarray(lp)[:, None]] = np.nan
        if name in ("sk", "sv"):
            x[np.arange(m_s)[None, :] >= np.asarray(ls)[:, None]] = np.nan
        bits = f32_to_bf16_bits(x)
        out[name] = bits
        out[name + "_f32"] = bf16_bits_to_f32(bits)
    return out


@pytest.mark.parametrize("b,W,h,g", [(2, 4, 8, 1), (2, 4, 16, 2), (2, 2, 32, 1), (3, 4, 8, 8), (2, 1, 8, 1)])
def test_beam_matches_oracle(b, W, h, g):
    m_p, m_s = 3000, 300
    rng = np.random.default_rng(b * 100 + W * 10 + h + g)
    lp = rng.integers(1, m_p + 1, size=b).astype(np.int32)
    lp[0] = m_p
    ls = rng.integers(0, m_s + 1, size=b * W).astype(np.int32)
    ls[0] = 0
    ls[-1] = 129
    inp = beam_inputs(b, W, h, g, m_p, m_s, lp, ls, seed=h + W)
    scale = 1 / math.sqrt(D)
    o = binding.decode_beam(dev(inp["q"], "bf16"), dev(inp["pk"], "bf16"), dev(inp["pv"], "bf16"),
                            torch.from_numpy(lp).cuda(), dev(inp["sk"], "bf16"), dev(inp["sv"], "bf16"),
                            torch.from_numpy(ls).cuda(), scale)
    ref, _ = oracle_decode_beam(inp["q_f32"], inp["pk_f32"], inp["pv_f32"], lp, inp["sk_f32"], inp["sv_f32"], ls,
                                g, scale)
    assert_close(host64(o), ref, "bf16", f"b={b} W={W} h={h} g={g}")


def test_beam_edges_of_prefix_and_suffix():
    """Prefix lengths 0, 1, 127, 128, 129 with suffixes of 0..129 rows; a beam
    with neither gets a zero row."""
    b, W, h, g = 5, 4, 8, 1
    m_p, m_s = 200, 200
    lp = np.array([0, 1, 127, 128, 129], np.int32)
    ls = np.array([0, 1, 128, 129] * 5, np.int32)
    inp = beam_inputs(b, W, h, g, m_p, m_s, lp, ls, seed=5)
    o = host64(binding.decode_beam(dev(inp["q"], "bf16"), dev(inp["pk"], "bf16"), dev(inp["pv"], "bf16"),
                                   torch.from_numpy(lp).cuda(), dev(inp["sk"], "bf16"), dev(inp["sv"], "bf16"),
                                   torch.from_numpy(ls).cuda(), 0.1))
    ref, _ = oracle_decode_beam(inp["q_f32"], inp["pk_f32"], inp["pv_f32"], lp, inp["sk_f32"], inp["sv_f32"], ls,
                                g, 0.1)
    assert_close(o, ref, "bf16", "edges")
    assert (o[0, 0] == 0).all()   # no prefix, no suffix


def test_beam_shapes_not_built_are_rejected():
    q = torch.zeros((1, 4, 32, D), dtype=torch.bfloat16, device="cuda")     # W * h/g = 128 > 64
    pk = torch.zeros((1, 8, 1, D), dtype=torch.bfloat16, device="cuda")
    sk = torch.zeros((4, 8, 1, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.MqaError):
        binding.decode_beam(q, pk, pk, torch.ones(1, dtype=torch.int32, device="cuda"), sk, sk,
                            torch.ones(4, dtype=torch.int32, device="cuda"), 1.0)


def test_beam_empty_sequences_and_beams():
    """A sequence with no prefix and no suffix rows in any beam gets zero rows
    (nothing reads its caches); a sequence with no prefix but suffix rows
    attends over those only; prefixes long enough to be split between CTAs sit
    beside them."""
    b, W, h, g = 4, 4, 8, 1
    m_p, m_s = 2000, 160
    lp = np.array([0, 0, 1999, 640], np.int32)
    ls = np.array([0, 0, 0, 0, 5, 0, 160, 129, 0, 0, 0, 0, 1, 2, 3, 4], np.int32)
    inp = beam_inputs(b, W, h, g, m_p, m_s, lp, ls, seed=21)
    o = host64(binding.decode_beam(dev(inp["q"], "bf16"), dev(inp["pk"], "bf16"), dev(inp["pv"], "bf16"),
                                   torch.from_numpy(lp).cuda(), dev(inp["sk"], "bf16"), dev(inp["sv"], "bf16"),
                                   torch.from_numpy(ls).cuda(), 1 / math.sqrt(D)))
    ref, _ = oracle_decode_beam(inp["q_f32"], inp["pk_f32"], inp["pv_f32"], lp, inp["sk_f32"], inp["sv_f32"], ls,
                                g, 1 / math.sqrt(D))
    assert_close(o, ref, "bf16", "empty sequences and beams")
    assert (o[0] == 0).all()           # no rows at all
    assert (o[1, 1] == 0).all()        # no prefix, empty suffix
    assert np.isfinite(o).all()


def test_beam_suffix_lengths_are_clamped_and_flagged():
    """Suffix lengths past the suffix cache are clamped to it and reported
    through the status word; the result is the clamped step's."""
    b, W, h, g = 2, 2, 16, 2
    m_p, m_s = 300, 100
    lp = np.array([300, 17], np.int32)
    ls_given = np.array([100, 250, -3, 40], np.int32)
    ls_used = np.clip(ls_given, 0, m_s).astype(np.int32)
    inp = beam_inputs(b, W, h, g, m_p, m_s, lp, ls_used, seed=22)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = host64(binding.decode_beam(dev(inp["q"], "bf16"), dev(inp["pk"], "bf16"), dev(inp["pv"], "bf16"),
                                   torch.from_numpy(lp).cuda(), dev(inp["sk"], "bf16"), dev(inp["sv"], "bf16"),
                                   torch.from_numpy(ls_given).cuda(), 0.2, status_flags=flags))
    ref, _ = oracle_decode_beam(inp["q_f32"], inp["pk_f32"], inp["pv_f32"], lp, inp["sk_f32"], inp["sv_f32"],
                                ls_used, g, 0.2)
    assert_close(o, ref, "bf16", "clamped suffixes")
    assert int(flags.item()) & binding.MQA_FLAG_LEN_CLAMPED


def test_beam_many_sequences_weighted_schedule():
    """More sequences than the decode CTA has threads (353 > 352): the schedule
    takes its general path, where the tile walkers count suffix tiles from
    global memory; results still match the oracle."""
    b, W, h, g = 353, 2, 8, 1
    m_p, m_s = 300, 40
    rng = np.random.default_rng(353)
    lp = rng.integers(0, m_p + 1, size=b).astype(np.int32)
    ls = rng.integers(0, m_s + 1, size=b * W).astype(np.int32)
    inp = beam_inputs(b, W, h, g, m_p, m_s, lp, ls, seed=353)
    scale = 1 / math.sqrt(D)
    o = host64(binding.decode_beam(dev(inp["q"], "bf16"), dev(inp["pk"], "bf16"), dev(inp["pv"], "bf16"),
                                   torch.from_numpy(lp).cuda(), dev(inp["sk"], "bf16"), dev(inp["sv"], "bf16"),
                                   torch.from_numpy(ls).cuda(), scale))
    ref, _ = oracle_decode_beam(inp["q_f32"], inp["pk_f32"], inp["pv_f32"], lp, inp["sk_f32"], inp["sv_f32"], ls,
                                g, scale)
    assert_close(o, ref, "bf16", "353 sequences")
