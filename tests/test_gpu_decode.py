"""mqa_decode on the GPU against the float64 oracle, element by element, on
seeded inputs whose masked rows hold NaN.  Sizes span several tiles and ragged
tails; the CTA count is forced low and high so sequences are split between
CTAs (exercising the log-sum-exp merge) and kept whole."""
import math

import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from grouped_query_attention_mqa_b200.workloads import WORKLOADS, Workload, host_inputs
from oracle import oracle_decode, oracle_decode_step

from gpu_util import TOL, assert_close, dev, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    binding.load_library()


def tc_available(wl):
    return (wl.dtype == "bf16" and wl.d_k in (64, 128) and wl.d_v in (64, 128) and 1 <= wl.heads_per_group <= 64
            and _tc_built())


def _tc_built():
    # the tensor-core path answers MQA_ERR_UNSUPPORTED when it is not built
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 1, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.ones(1, dtype=torch.int32, device="cuda")
    try:
        binding.decode(q, k, k, lens, 1.0, path="tcgen05")
        return True
    except binding.MqaError as e:
        if e.status == binding.MQA_ERR_UNSUPPORTED:
            return False
        raise


def run_case(wl, seed, lens=None, path="auto", num_ctas=0):
    inp = host_inputs(wl, seed, nan_tail=True, lens=lens)
    o = binding.decode(dev(inp["q"], wl.dtype), dev(inp["k"], wl.dtype), dev(inp["v"], wl.dtype),
                       torch.from_numpy(inp["lens"]).cuda(), wl.scale, path=path, num_ctas=num_ctas)
    torch.cuda.synchronize()
    ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["lens"], wl.g, wl.scale)
    return host64(o), ref


def small(dtype, b, h, g, d, m_max, lo, hi, scale=None):
    return Workload(f"t_{dtype}_{b}_{h}_{g}_{d}_{m_max}", b=b, h=h, g=g, d_k=d, d_v=d, m_max=m_max, len_lo=lo,
                    len_hi=hi, dtype=dtype, scale=scale if scale is not None else 1 / math.sqrt(d))


def test_tiny_mqa_f32_step():
    """The tiny fp32 MQA workload: b=1 h=4 g=1 d=32, append the 64th row, decode."""
    wl = WORKLOADS["tiny_mqa_f32"]
    inp = host_inputs(wl, seed=1, nan_tail=True, lens=np.array([63], np.int32))
    K, V = dev(inp["k"], "f32"), dev(inp["v"], "f32")
    binding.kv_append(K, V, dev(inp["k_new"], "f32"), dev(inp["v_new"], "f32"),
                      torch.tensor([63], dtype=torch.int32, device="cuda"))
    o = binding.decode(dev(inp["q"], "f32"), K, V, torch.tensor([64], dtype=torch.int32, device="cuda"), wl.scale)
    torch.cuda.synchronize()
    ref, _, _, _ = oracle_decode_step(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["k_new_f32"], inp["v_new_f32"],
                                      inp["lens"], wl.g, wl.scale)
    assert_close(host64(o), ref, "f32", "tiny")


SHAPES = [
    # dtype, b, h, g, d, m_max, len_lo, len_hi
    ("bf16", 3, 1, 1, 128, 300, 1, 300),      # MHA-like single head
    ("bf16", 4, 8, 8, 128, 257, 100, 257),    # MHA g = h
    ("bf16", 2, 4, 2, 64, 200, 60, 200),      # GQA h/g = 2
    ("bf16", 5, 8, 2, 128, 400, 1, 400),      # GQA h/g = 4
    ("bf16", 3, 8, 1, 128, 513, 200, 513),    # MQA h = 8
    ("bf16", 2, 16, 1, 128, 700, 129, 700),   # MQA h = 16
    ("bf16", 3, 32, 1, 128, 600, 64, 600),    # MQA h = 32 (long-context shape)
    ("bf16", 2, 64, 8, 128, 640, 300, 640),   # GQA-8 shape
    ("bf16", 2, 32, 1, 32, 90, 1, 90),        # small head size
    ("f32", 2, 4, 1, 32, 150, 1, 150),
    ("f32", 3, 8, 2, 64, 129, 1, 129),
    ("f32", 2, 16, 4, 128, 200, 65, 200),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "_".join(map(str, s)))
@pytest.mark.parametrize("num_ctas", [0, 1, 3, 7])
def test_decode_matches_oracle(shape, num_ctas):
    wl = small(*shape)
    out, ref = run_case(wl, seed=sum(shape[1:]) + num_ctas, path="simt" if shape[0] == "f32" else "auto",
                        num_ctas=num_ctas)
    assert_close(out, ref, wl.dtype, wl.name)


@pytest.mark.parametrize("hq", [1, 2, 4])
def test_automatic_path_takes_tensor_cores_for_small_groups(hq):
    """bf16, d = 128: the automatic choice is the tensor-core kernel at every
    group width it serves, MHA (h/g = 1) included, where it streams the cache
    at more than twice the CUDA-core kernel's rate.  Same path and CTA count
    give the same bits."""
    wl = small("bf16", 4, 8, 8 // hq, 128, 400, 1, 400)
    if not tc_available(wl):
        pytest.skip("tensor-core path not built")
    auto, ref = run_case(wl, seed=hq, path="auto")
    tc, _ = run_case(wl, seed=hq, path="tcgen05")
    assert np.array_equal(auto, tc)
    assert_close(auto, ref, "bf16", f"auto hq={hq}")


@pytest.mark.parametrize("path", ["simt", "tcgen05"])
@pytest.mark.parametrize("hq", [1, 4, 8, 12, 16, 32, 48, 64])
def test_both_paths_on_group_widths(path, hq):
    wl = small("bf16", 3, hq, 1, 128, 530, 1, 530)
    if path == "tcgen05" and not tc_available(wl):
        pytest.skip("tensor-core path not built")
    if path == "simt" and hq * 128 > 4096:
        pytest.skip("SIMT path takes h/g*d <= 4096")
    for num_ctas in (0, 2, 5):
        out, ref = run_case(wl, seed=hq + num_ctas, path=path, num_ctas=num_ctas)
        assert_close(out, ref, "bf16", f"{path} hq={hq} ctas={num_ctas}")


@pytest.mark.parametrize("g", [1, 2, 8])
def test_tensor_core_path_gqa_and_tile_edges(g):
    """The tensor-core path with several K/V heads and lengths at its 128-row
    tile edges, whole sequences and sequences split between CTAs."""
    wl = small("bf16", 4, 8 * g, g, 128, 400, 1, 1)
    if not tc_available(wl):
        pytest.skip("tensor-core path not built")
    for lens in ([127, 128, 129, 400], [1, 2, 255, 256], [257, 383, 384, 385]):
        for num_ctas in (0, 1, 3, 9):
            out, ref = run_case(wl, seed=sum(lens) + num_ctas, lens=np.array(lens, np.int32), path="tcgen05",
                                num_ctas=num_ctas)
            assert_close(out, ref, "bf16", f"tc g={g} lens={lens} ctas={num_ctas}")


def test_tensor_core_path_rescales_for_growing_logits():
    """Logits that grow along the sequence force the running maximum to move
    (and O in tensor memory to be rescaled) several times within a segment."""
    wl = small("bf16", 2, 32, 1, 128, 1024, 1024, 1024)
    if not tc_available(wl):
        pytest.skip("tensor-core path not built")
    inp = host_inputs(wl, seed=21, nan_tail=True)
    from grouped_query_attention_mqa_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
    ramp = np.linspace(0.0, 6.0, wl.m_max, dtype=np.float32)[None, :, None, None]
    k = f32_to_bf16_bits(bf16_bits_to_f32(inp["k"]) * 0 + inp["q_f32"][:, :1, None, :] * ramp * 3)
    kf = bf16_bits_to_f32(k)
    for path, ctas in (("tcgen05", 0), ("tcgen05", 1), ("simt", 0)):
        o = binding.decode(dev(inp["q"], "bf16"), dev(k, "bf16"), dev(inp["v"], "bf16"),
                           torch.from_numpy(inp["lens"]).cuda(), wl.scale, path=path, num_ctas=ctas)
        ref, _ = oracle_decode(inp["q_f32"], kf, inp["v_f32"], inp["lens"], 1, wl.scale)
        assert_close(host64(o), ref, "bf16", f"ramp {path} ctas={ctas}")


@pytest.mark.parametrize("tile_edge", [1, 63, 64, 65, 127, 128, 129, 255, 256, 257])
def test_lengths_at_tile_edges(tile_edge):
    """Lengths one below, at and above the tile sizes of both paths (64, 128)."""
    for wl in (small("bf16", 4, 32, 1, 128, 260, 1, 1), small("bf16", 4, 2, 1, 128, 260, 1, 1)):
        lens = np.array([tile_edge, 1, 260, max(1, tile_edge - 1)], np.int32)
        for num_ctas in (0, 3):
            out, ref = run_case(wl, seed=tile_edge, lens=lens, num_ctas=num_ctas)
            assert_close(out, ref, "bf16", f"len={tile_edge} hq={wl.heads_per_group}")


def test_degenerate_inputs():
    """Length-1 cache returns v; identical keys return the mean of V; a query
    with huge logits picks the row of the largest one (no overflow)."""
    b, h, m, d = 3, 32, 200, 128
    rng = np.random.default_rng(5)
    q = rng.standard_normal((b, h, d)).astype(np.float32)
    K = rng.standard_normal((b, m, 1, d)).astype(np.float32)
    V = rng.standard_normal((b, m, 1, d)).astype(np.float32)
    K[1] = K[1, 0]                    # sequence 1: every key the same
    q[2] *= 300.0                     # sequence 2: near one-hot weights
    from grouped_query_attention_mqa_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
    qb, Kb, Vb = (f32_to_bf16_bits(x) for x in (q, K, V))
    lens = np.array([1, 150, 200], np.int32)
    for path in ("simt", "auto"):
        if path == "simt" and h * d > 4096:
            continue
        o = host64(binding.decode(dev(qb, "bf16"), dev(Kb, "bf16"), dev(Vb, "bf16"),
                                  torch.from_numpy(lens).cuda(), 1 / math.sqrt(d), path=path))
        Vf = bf16_bits_to_f32(Vb).astype(np.float64)
        np.testing.assert_allclose(o[0], np.broadcast_to(Vf[0, 0, 0], (h, d)), atol=TOL["bf16"], rtol=0)
        np.testing.assert_allclose(o[1], np.broadcast_to(Vf[1, :150, 0].mean(axis=0), (h, d)), atol=TOL["bf16"],
                                   rtol=0)
        ref, _ = oracle_decode(bf16_bits_to_f32(qb), bf16_bits_to_f32(Kb), Vf, lens, 1, 1 / math.sqrt(d))
        assert_close(o, ref, "bf16", "degenerate")


def test_lengths_out_of_range_are_clamped_and_flagged():
    wl = small("bf16", 4, 8, 1, 128, 100, 1, 100)
    inp = host_inputs(wl, seed=9, nan_tail=False, lens=np.array([50, 100, 1, 1], np.int32))
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    bad = torch.tensor([50, 1000, 0, -5], dtype=torch.int32, device="cuda")
    o = host64(binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"), bad, wl.scale,
                              status_flags=flags))
    assert int(flags.item()) & binding.MQA_FLAG_LEN_CLAMPED
    ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], np.array([50, 100, 0, 0]), 1, wl.scale)
    assert_close(o, ref, "bf16", "clamped")
    assert (o[2:] == 0).all()
    flags.zero_()
    binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                   torch.tensor([50, 100, 1, 1], dtype=torch.int32, device="cuda"), wl.scale, status_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0


def test_empty_batch_is_a_no_op():
    q = torch.zeros((0, 8, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((0, 4, 1, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.zeros(0, dtype=torch.int32, device="cuda")
    out = binding.decode(q, k, k, lens, 1.0)
    assert out.shape == (0, 8, 128)


def test_workspace_too_small_is_rejected():
    q = torch.zeros((2, 8, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((2, 4, 1, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.ones(2, dtype=torch.int32, device="cuda")
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.MqaError) as e:
        binding.decode(q, k, k, lens, 1.0, workspace=ws)
    assert e.value.status == binding.MQA_ERR_INVALID_ARG


def test_workspace_reused_across_shapes():
    """One workspace serves decodes of different shapes in turn; whatever an
    earlier call left in it, every result matches the oracle."""
    shapes = [(5, 32, 1, 700, 1, 700), (3, 64, 8, 500, 100, 500), (9, 16, 2, 300, 1, 300), (5, 32, 1, 700, 1, 700)]
    need = max(binding.decode_workspace_size(b, h, g, 128) for b, h, g, *_ in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for n, (b, h, g, m, lo, hi) in enumerate(shapes):
        wl = small("bf16", b, h, g, 128, m, lo, hi)
        assert binding.decode_workspace_size(b, h, g, 128) <= ws.numel()
        inp = host_inputs(wl, seed=40 + n, nan_tail=True)
        for ctas in (0, 7):
            o = binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                               torch.from_numpy(inp["lens"]).cuda(), wl.scale, workspace=ws, num_ctas=ctas)
            ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["lens"], g, wl.scale)
            assert_close(host64(o), ref, "bf16", f"shape {n} ctas {ctas}")


@pytest.mark.parametrize("path", ["tcgen05", "simt"])
def test_mixed_and_empty_lengths_many_ctas(path):
    """Zero-length sequences (zero rows out), single-row sequences, long ones,
    and more CTAs than tiles: the work partition must give every tile to
    exactly one CTA and the merge must find every partial."""
    wl = small("bf16", 12, 32 if path == "tcgen05" else 8, 1, 128, 900, 1, 1)
    lens = np.array([0, 1, 900, 0, 129, 128, 2, 0, 700, 1, 255, 0], np.int32)
    inp = host_inputs(wl, seed=77, nan_tail=False, lens=np.maximum(lens, 1))
    for ctas in (0, 1, 5, 40, 300):
        o = host64(binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                                  torch.from_numpy(lens).cuda(), wl.scale, path=path, num_ctas=ctas))
        ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, 1, wl.scale)
        assert_close(o, ref, "bf16", f"{path} ctas={ctas}")
        assert (o[lens == 0] == 0).all()


@pytest.mark.parametrize("b", [352, 353, 700])
def test_tensor_core_path_large_batches(b):
    """Batches on both sides of the one-sequence-per-thread schedule (one
    tensor-core CTA has 352 threads): every tile is owned by exactly one CTA
    and zero-length sequences give zero rows."""
    wl = small("bf16", b, 8, 1, 128, 300, 1, 1)
    if not tc_available(wl):
        pytest.skip("tensor-core path not built")
    rng = np.random.default_rng(b)
    lens = rng.integers(0, 301, size=b).astype(np.int32)
    lens[rng.integers(0, b, size=b // 10)] = 0
    inp = host_inputs(wl, seed=b, nan_tail=True, lens=np.maximum(lens, 1))
    for ctas in (0, 37):
        o = host64(binding.decode(dev(inp["q"], "bf16"), dev(inp["k"], "bf16"), dev(inp["v"], "bf16"),
                                  torch.from_numpy(lens).cuda(), wl.scale, path="tcgen05", num_ctas=ctas))
        ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, 1, wl.scale)
        assert_close(o, ref, "bf16", f"b={b} ctas={ctas}")
        assert (o[lens == 0] == 0).all()


@pytest.mark.parametrize("path,h,m_max,window,dtype", [
    ("tcgen05", 32, 128, 0, "bf16"),     # every sequence fits one 128-row tile
    ("tcgen05", 8, 600, 100, "bf16"),    # long sequences, but a window of one tile
    ("simt", 4, 64, 0, "bf16"),          # one 64-row SIMT tile
    ("simt", 4, 300, 64, "f32"),
])
def test_single_tile_sequences_need_no_merge(path, h, m_max, window, dtype):
    """When no sequence spans two tiles no segment can be split, the merge
    kernel is left out and the decode writes every output row itself,
    including the zero rows of empty sequences.  The output starts as NaN, so
    a row left unwritten fails."""
    b = 40
    wl = small(dtype, b, h, 1, 128 if dtype == "bf16" else 64, m_max, 1, 1)
    rng = np.random.default_rng(h + m_max)
    lens = rng.integers(0, m_max + 1, size=b).astype(np.int32)
    lens[::7] = 0
    inp = host_inputs(wl, seed=m_max, nan_tail=True, lens=np.maximum(lens, 1))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    for ctas in (0, 1, 7, 300):
        out = torch.full((b, h, wl.d_v), float("nan"), dtype=tdt, device="cuda")
        binding.decode(dev(inp["q"], dtype), dev(inp["k"], dtype), dev(inp["v"], dtype), torch.from_numpy(lens).cuda(),
                       wl.scale, out=out, path=path, num_ctas=ctas, window=window)
        ref, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], lens, 1, wl.scale, window=window)
        o = host64(out)
        assert_close(o, ref, dtype, f"{path} ctas={ctas}")
        assert (o[lens == 0] == 0).all()
