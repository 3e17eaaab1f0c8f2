"""The C ABI without a GPU: the library builds and loads, exports every symbol
include/mqa.h declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest

from grouped_query_attention_mqa_b200 import binding
from grouped_query_attention_mqa_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def header_symbols():
    text = open(os.path.join(ROOT, "include", "mqa.h")).read()
    return sorted(set(re.findall(r"MQA_API\s+[\w\s\*]+?\b(mqa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert header_symbols() == sorted(["mqa_kv_append", "mqa_decode_workspace_size", "mqa_decode",
                                       "mqa_decode_ex", "mqa_decode_append", "mqa_decode_noalloc",
                                       "mqa_prefill", "mqa_decode_beam", "mqa_decode_beam_workspace_size",
                                       "mqa_status_string"])


def test_library_exports_every_declared_symbol(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name
    assert set(header_symbols()) == set(binding.SIGNATURES)


def test_status_strings(lib):
    assert binding.status_string(0) == "MQA_OK"
    assert binding.status_string(1) == "MQA_ERR_INVALID_ARG"
    assert binding.status_string(2) == "MQA_ERR_UNSUPPORTED"
    assert binding.status_string(3) == "MQA_ERR_CUDA"
    assert binding.status_string(99) == "MQA_STATUS_UNKNOWN"


def test_workspace_size(lib):
    ws = binding.decode_workspace_size
    assert ws(64, 32, 1, 128) > 0
    # grows with the batch and the group width
    assert ws(128, 32, 1, 128) > ws(64, 32, 1, 128)
    assert ws(64, 64, 1, 128) > ws(64, 32, 1, 128)
    # partial slots: one per persistent CTA plus one per (sequence, K/V head)
    slots = binding.MQA_MAX_CTAS + 64
    assert ws(64, 32, 1, 128) >= slots * 32 * 129 * 4
    for bad in ((64, 32, 3, 128), (-1, 8, 1, 128), (4, 0, 1, 128), (4, 8, 0, 128), (4, 8, 1, 0)):
        assert ws(*bad) == 0
    assert ws(0, 8, 1, 128) > 0   # empty batch: only the per-CTA slots


FAKE = ctypes.c_void_p(0x10000)   # aligned, never dereferenced: every call below fails its checks first


def _decode(lib, **kw):
    a = dict(o=FAKE, q=FAKE, k=FAKE, v=FAKE, lens=FAKE, b=2, h=8, g=1, m_max=16, d_k=128, d_v=128, scale=1.0,
             dtype=binding.MQA_BF16, ws=FAKE, ws_bytes=1 << 40, flags=None, opts=None, stream=None)
    a.update(kw)
    return lib.mqa_decode_ex(a["o"], a["q"], a["k"], a["v"], a["lens"], a["b"], a["h"], a["g"], a["m_max"],
                             a["d_k"], a["d_v"], a["scale"], a["dtype"], a["ws"], a["ws_bytes"], a["flags"],
                             a["opts"], a["stream"])


def test_decode_rejects_bad_arguments_without_launching(lib):
    INV, UNS = binding.MQA_ERR_INVALID_ARG, binding.MQA_ERR_UNSUPPORTED
    assert _decode(lib, g=3) == INV                      # h % g != 0
    assert _decode(lib, g=0) == INV
    assert _decode(lib, q=None) == INV
    assert _decode(lib, ws=None) == INV
    assert _decode(lib, o=ctypes.c_void_p(0x10008)) == INV        # misaligned
    assert _decode(lib, ws=ctypes.c_void_p(0x10010)) == INV       # workspace not 256-aligned
    assert _decode(lib, ws_bytes=100) == INV             # workspace too small
    assert _decode(lib, scale=float("nan")) == INV
    assert _decode(lib, scale=float("inf")) == INV
    assert _decode(lib, dtype=7) == INV
    assert _decode(lib, m_max=0) == INV
    assert _decode(lib, d_k=96, d_v=96) == UNS           # head size not built
    assert _decode(lib, d_k=128, d_v=96) == UNS          # value width not built
    opts = binding.DecodeOptions(2, 0)                   # tensor cores: head sizes 64 and 128 only
    assert _decode(lib, d_k=128, d_v=32, opts=ctypes.byref(opts)) == UNS
    assert _decode(lib, d_k=32, d_v=64, opts=ctypes.byref(opts)) == UNS
    opts = binding.DecodeOptions(1, 0)                   # SIMT: h/g * d_v <= 4096 as well
    assert _decode(lib, h=64, d_k=32, d_v=128, opts=ctypes.byref(opts)) == UNS
    opts = binding.DecodeOptions(9, 0)
    assert _decode(lib, opts=ctypes.byref(opts)) == INV  # unknown path
    opts = binding.DecodeOptions(0, binding.MQA_MAX_CTAS + 1)
    assert _decode(lib, opts=ctypes.byref(opts)) == INV
    opts = binding.DecodeOptions(0, 0, -1)               # negative local window
    assert _decode(lib, opts=ctypes.byref(opts)) == INV
    opts = binding.DecodeOptions(1, 0)                   # SIMT cannot take h/g*d > 4096
    assert _decode(lib, h=64, opts=ctypes.byref(opts)) == UNS
    opts = binding.DecodeOptions(2, 0)                   # tensor cores need bf16
    assert _decode(lib, dtype=binding.MQA_F32, opts=ctypes.byref(opts)) == UNS
    assert _decode(lib, b=0) == binding.MQA_OK           # empty batch: nothing to do


def _noalloc(lib, **kw):
    a = dict(o=FAKE, q=FAKE, k=FAKE, v=FAKE, lens=FAKE, b=2, h=8, g=1, m_max=16, d_k=128, d_v=128, scale=1.0,
             dtype=binding.MQA_BF16, flags=None, stream=None)
    a.update(kw)
    return lib.mqa_decode_noalloc(a["o"], a["q"], a["k"], a["v"], a["lens"], a["b"], a["h"], a["g"], a["m_max"],
                                  a["d_k"], a["d_v"], a["scale"], a["dtype"], a["flags"], a["stream"])


def test_noalloc_rejects_bad_arguments_without_launching(lib):
    """mqa_decode_noalloc checks its arguments as mqa_decode does, before it
    touches the device; every call below fails a check."""
    INV, UNS = binding.MQA_ERR_INVALID_ARG, binding.MQA_ERR_UNSUPPORTED
    assert _noalloc(lib, g=3) == INV                     # h % g != 0
    assert _noalloc(lib, lens=None) == INV
    assert _noalloc(lib, q=ctypes.c_void_p(0x10008)) == INV        # misaligned
    assert _noalloc(lib, scale=float("nan")) == INV
    assert _noalloc(lib, dtype=7) == INV
    assert _noalloc(lib, m_max=0) == INV
    assert _noalloc(lib, d_k=96, d_v=96) == UNS          # head size not built
    assert _noalloc(lib, d_k=128, d_v=48) == UNS         # value width not built
    assert _noalloc(lib, h=64, d_k=32, d_v=128) == UNS   # SIMT (unequal widths): h/g * d_v > 4096
    assert _noalloc(lib, b=4096, h=64, g=64) == INV      # partials beyond the 16 MiB array
    assert _noalloc(lib, b=0) == binding.MQA_OK          # empty batch: nothing to do


def _fused(lib, **kw):
    a = dict(o=FAKE, q=FAKE, k=FAKE, v=FAKE, kn=FAKE, vn=FAKE, lens=FAKE, b=2, h=8, g=1, m_max=16, d_k=128, d_v=128,
             scale=1.0, dtype=binding.MQA_BF16, ws=FAKE, ws_bytes=1 << 40, flags=None, opts=None, stream=None)
    a.update(kw)
    return lib.mqa_decode_append(a["o"], a["q"], a["k"], a["v"], a["kn"], a["vn"], a["lens"], a["b"], a["h"], a["g"],
                                 a["m_max"], a["d_k"], a["d_v"], a["scale"], a["dtype"], a["ws"], a["ws_bytes"],
                                 a["flags"], a["opts"], a["stream"])


def test_fused_step_rejects_bad_arguments_without_launching(lib):
    INV, UNS = binding.MQA_ERR_INVALID_ARG, binding.MQA_ERR_UNSUPPORTED
    assert _fused(lib, kn=None) == INV                   # the new rows are required
    assert _fused(lib, vn=None) == INV
    assert _fused(lib, kn=ctypes.c_void_p(0x10004)) == INV         # misaligned new row
    assert _fused(lib, g=3) == INV
    assert _fused(lib, ws_bytes=100) == INV
    assert _fused(lib, d_k=96, d_v=96) == UNS
    opts = binding.DecodeOptions(2, 0)                   # tensor cores: head sizes 64 and 128 only
    assert _fused(lib, d_v=32, opts=ctypes.byref(opts)) == UNS
    assert _fused(lib, b=0, kn=None, vn=None) == binding.MQA_OK


def _beam(lib, **kw):
    a = dict(o=FAKE, q=FAKE, pk=FAKE, pv=FAKE, pl=FAKE, sk=FAKE, sv=FAKE, sl=FAKE, b=2, W=4, h=8, g=1, m_p=64, m_s=8,
             d_k=128, d_v=128, scale=1.0, dtype=binding.MQA_BF16, ws=FAKE, ws_bytes=1 << 40, flags=None, stream=None)
    a.update(kw)
    return lib.mqa_decode_beam(a["o"], a["q"], a["pk"], a["pv"], a["pl"], a["sk"], a["sv"], a["sl"], a["b"], a["W"],
                               a["h"], a["g"], a["m_p"], a["m_s"], a["d_k"], a["d_v"], a["scale"], a["dtype"], a["ws"],
                               a["ws_bytes"], a["flags"], a["stream"])


def test_beam_rejects_bad_arguments_without_launching(lib):
    INV, UNS = binding.MQA_ERR_INVALID_ARG, binding.MQA_ERR_UNSUPPORTED
    ws = lib.mqa_decode_beam_workspace_size
    assert ws(2, 4, 8, 1, 128) == lib.mqa_decode_workspace_size(2, 32, 1, 128)   # W beams' heads share a segment
    assert ws(2, 0, 8, 1, 128) == 0 and ws(2, 4, 8, 3, 128) == 0
    assert _beam(lib, W=0) == INV
    assert _beam(lib, m_s=0) == INV
    assert _beam(lib, sl=None) == INV
    assert _beam(lib, sk=ctypes.c_void_p(0x10008)) == INV          # misaligned suffix cache
    assert _beam(lib, ws=ctypes.c_void_p(0x10010)) == INV          # workspace not 256-aligned
    assert _beam(lib, ws_bytes=ws(2, 4, 8, 1, 128) - 1) == INV     # one byte short
    assert _beam(lib, scale=float("inf")) == INV
    assert _beam(lib, dtype=binding.MQA_F32) == UNS      # tensor cores only: bf16
    assert _beam(lib, d_k=64, d_v=64) == UNS             # d = 128 only
    assert _beam(lib, W=16, h=8) == UNS                  # W * h/g = 128 > 64 query columns
    assert _beam(lib, b=0) == binding.MQA_OK


def test_append_rejects_bad_arguments_without_launching(lib):
    INV = binding.MQA_ERR_INVALID_ARG
    f = lib.mqa_kv_append
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 0, 1, 128, 128, 1, None, None) == INV       # m_max
    assert f(None, FAKE, FAKE, FAKE, FAKE, 2, 8, 1, 128, 128, 1, None, None) == INV
    assert f(FAKE, FAKE, FAKE, FAKE, None, 2, 8, 1, 128, 128, 1, None, None) == INV
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 1, 4, 4, 1, None, None) == INV           # 8-byte rows
    assert f(FAKE, FAKE, ctypes.c_void_p(0x10004), FAKE, FAKE, 2, 8, 1, 128, 128, 1, None, None) == INV
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 1, 128, 128, 5, None, None) == INV       # dtype
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 8, 1, 128, 128, 1, None, None) == INV
    assert f(None, None, None, None, None, 0, 8, 1, 128, 128, 1, None, None) == binding.MQA_OK


def test_binding_fails_loudly_without_the_library(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        binding.load_library(str(tmp_path / "libmqa.so"))


def _prefill(lib, **kw):
    a = dict(o=FAKE, q=FAKE, k=FAKE, v=FAKE, cu=FAKE, b=2, total=64, max_seqlen=40, h=8, g=1, d_k=128, d_v=128,
             scale=1.0, causal=1, dtype=binding.MQA_BF16, flags=None, stream=None)
    a.update(kw)
    return lib.mqa_prefill(a["o"], a["q"], a["k"], a["v"], a["cu"], a["b"], a["total"], a["max_seqlen"], a["h"],
                           a["g"], a["d_k"], a["d_v"], a["scale"], a["causal"], a["dtype"], a["flags"], a["stream"])


def test_prefill_rejects_bad_arguments_without_launching(lib):
    INV, UNS = binding.MQA_ERR_INVALID_ARG, binding.MQA_ERR_UNSUPPORTED
    assert _prefill(lib, g=3) == INV                     # h % g != 0
    assert _prefill(lib, q=None) == INV
    assert _prefill(lib, cu=None) == INV
    assert _prefill(lib, o=ctypes.c_void_p(0x10008)) == INV
    assert _prefill(lib, total=-1) == INV
    assert _prefill(lib, max_seqlen=-1) == INV
    assert _prefill(lib, causal=2) == INV
    assert _prefill(lib, scale=float("nan")) == INV
    assert _prefill(lib, dtype=binding.MQA_F32) == UNS   # only bf16 is built
    assert _prefill(lib, d_k=64, d_v=64) == UNS          # only d = 128
    assert _prefill(lib, h=12, g=1) == UNS               # h/g must divide 128
    assert _prefill(lib, b=0) == binding.MQA_OK          # nothing to do
    assert _prefill(lib, total=0) == binding.MQA_OK
