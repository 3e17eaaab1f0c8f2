"""mqa_decode_noalloc, the decode for callers that cannot allocate device
memory (a plugin inside an application that owns every allocation, a runtime
with a fixed pool, a call site where allocating could synchronise the device).
It keeps its split partials in a library-owned device array instead of a
caller workspace.  Called here through the C ABI and compared with
mqa_decode on the same inputs, twice in a row on different inputs, so that
contents left in the shared array by one call cannot leak into the next.

This file is collected last on purpose: a run that stops at the first failure
has run every other test before it."""
import ctypes
import math

import numpy as np
import pytest
import torch

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build
from grouped_query_attention_mqa_b200.workloads import Workload, host_inputs

from oracle import oracle_decode

from gpu_util import TOL, assert_close, dev, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _both(lib, wl, seed, with_oracle=False):
    """Run mqa_decode (caller workspace) and mqa_decode_noalloc on one input;
    with_oracle also returns the oracle's output on the same input."""
    inp = host_inputs(wl, seed, nan_tail=True)
    q, K, V = dev(inp["q"], wl.dtype), dev(inp["k"], wl.dtype), dev(inp["v"], wl.dtype)
    lens = torch.from_numpy(inp["lens"]).cuda()
    dt = binding.MQA_BF16 if wl.dtype == "bf16" else binding.MQA_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ref = torch.empty((wl.b, wl.h, wl.d_v), dtype=q.dtype, device="cuda")
    ws = binding.new_workspace(wl.b, wl.h, wl.g, wl.d_v)
    st = lib.mqa_decode(_p(ref), _p(q), _p(K), _p(V), _p(lens), wl.b, wl.h, wl.g, wl.m_max, wl.d_k, wl.d_v,
                        wl.scale, dt, _p(ws), ws.numel(), None, stream)
    assert st == binding.MQA_OK
    out = torch.full_like(ref, float("nan"))
    st = lib.mqa_decode_noalloc(_p(out), _p(q), _p(K), _p(V), _p(lens), wl.b, wl.h, wl.g, wl.m_max, wl.d_k,
                                wl.d_v, wl.scale, dt, None, stream)
    assert st == binding.MQA_OK
    torch.cuda.synchronize()
    if with_oracle:
        want, _ = oracle_decode(inp["q_f32"], inp["k_f32"], inp["v_f32"], inp["lens"], wl.g, wl.scale)
        return host64(out), host64(ref), want
    return host64(out), host64(ref)


CASES = [
    Workload("noalloc_mqa", b=6, h=32, g=1, d_k=128, d_v=128, m_max=700, len_lo=1, len_hi=700, dtype="bf16",
             scale=1 / math.sqrt(128)),
    Workload("noalloc_gqa", b=3, h=16, g=4, d_k=64, d_v=64, m_max=300, len_lo=40, len_hi=300, dtype="f32",
             scale=1 / math.sqrt(64)),
    # bf16 at head size 64: the tensor-core kernel's 256-row tiles
    Workload("noalloc_d64", b=5, h=32, g=2, d_k=64, d_v=64, m_max=900, len_lo=1, len_hi=900, dtype="bf16",
             scale=1 / math.sqrt(64)),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_noalloc_matches_decode_on_two_calls_in_a_row(lib, wl):
    for seed in (11, 12):   # second call: new inputs over the array the first call left behind
        out, ref, want = _both(lib, wl, seed, with_oracle=True)
        assert np.isfinite(out).all()
        err = float(np.abs(out - ref).max())
        assert err <= TOL[wl.dtype], f"{wl.name} seed {seed}: max-abs {err:.3e}"
        assert_close(out, want, wl.dtype, f"{wl.name} seed {seed} against the oracle")


def test_noalloc_lowers_its_cta_count_to_fit_the_array(lib):
    """960 sequences with 32 heads: each split partial takes 32 x 129 floats,
    so only about 1000 slots fit the 16 MiB array next to the 960 segments and
    the call runs on far fewer CTAs than the GPU has SMs.  Every sequence is
    checked against the oracle and against mqa_decode, on two calls in a
    row."""
    wl = Workload("noalloc_lowered", b=960, h=32, g=1, d_k=128, d_v=128, m_max=300, len_lo=1, len_hi=300,
                  dtype="bf16", scale=1 / math.sqrt(128))
    per_slot = 32 * 4 + 32 * 128 * 4
    assert (binding.MQA_NOALLOC_SCRATCH_BYTES - wl.b * 8) // per_slot - wl.b < torch.cuda.get_device_properties(
        0).multi_processor_count
    for seed in (21, 22):
        out, ref, want = _both(lib, wl, seed, with_oracle=True)
        assert_close(out, want, "bf16", f"lowered grid seed {seed} against the oracle")
        err = float(np.abs(out - ref).max())
        assert err <= TOL["bf16"], f"lowered grid seed {seed}: max-abs {err:.3e} against mqa_decode"


def test_noalloc_single_tile_caches_skip_the_merge(lib):
    """Caches of at most one tile: no sequence is split, the decode writes
    every row itself (zero rows for empty sequences included)."""
    wl = Workload("noalloc_short", b=40, h=16, g=2, d_k=128, d_v=128, m_max=128, len_lo=0, len_hi=128,
                  dtype="bf16", scale=1 / math.sqrt(128))
    for seed in (31, 32):
        out, ref, want = _both(lib, wl, seed, with_oracle=True)
        assert_close(out, want, "bf16", f"single-tile seed {seed} against the oracle")
        assert np.array_equal(out, ref)


def test_noalloc_rejects_shapes_beyond_its_array(lib):
    """b*g segments whose partials exceed the 16 MiB array are refused before
    any launch (the pointers below are never dereferenced)."""
    fake = ctypes.c_void_p(0x10000)
    b, h, g, d = 4096, 64, 64, 128        # 262144 segments x 129 floats > 16 MiB
    st = lib.mqa_decode_noalloc(fake, fake, fake, fake, fake, b, h, g, 8, d, d, 1.0, binding.MQA_BF16, None, None)
    assert st == binding.MQA_ERR_INVALID_ARG
