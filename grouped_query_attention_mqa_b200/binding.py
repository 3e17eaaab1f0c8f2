"""ctypes binding of libmqa (include/mqa.h).

Argument marshalling only: shapes and dtypes of torch tensors are read, their
device pointers and the current CUDA stream are handed to the C ABI, and a
non-OK status becomes an ``MqaError``.  Every step of the computation runs in
the library's CUDA kernels; there is no other implementation behind these
functions and no fallback — if ``libmqa.so`` is missing they raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmqa.so")

MQA_OK, MQA_ERR_INVALID_ARG, MQA_ERR_UNSUPPORTED, MQA_ERR_CUDA = 0, 1, 2, 3
MQA_F32, MQA_BF16 = 0, 1
MQA_FLAG_LEN_CLAMPED, MQA_FLAG_POS_SKIPPED, MQA_FLAG_PIPE_TIMEOUT = 1, 2, 4
PATHS = {"auto": 0, "simt": 1, "tcgen05": 2}
MQA_MAX_CTAS = 2048
MQA_NOALLOC_SCRATCH_BYTES = 16 << 20

# Every symbol include/mqa.h declares, with its ctypes signature.
_c_int, _c_size, _c_ptr, _c_float = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float


class DecodeOptions(ctypes.Structure):
    _fields_ = [("path", _c_int), ("num_ctas", _c_int), ("window", _c_int)]


SIGNATURES = {
    "mqa_kv_append": (_c_int, [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_int, _c_int, _c_int, _c_int, _c_int,
                               _c_int, _c_ptr, _c_ptr]),
    "mqa_decode_workspace_size": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "mqa_decode": (_c_int, [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                            _c_float, _c_int, _c_ptr, _c_size, _c_ptr, _c_ptr]),
    "mqa_decode_ex": (_c_int, [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_int, _c_int, _c_int, _c_int, _c_int,
                               _c_int, _c_float, _c_int, _c_ptr, _c_size, _c_ptr, ctypes.POINTER(DecodeOptions),
                               _c_ptr]),
    "mqa_decode_append": (_c_int, [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_int, _c_int, _c_int,
                                   _c_int, _c_int, _c_int, _c_float, _c_int, _c_ptr, _c_size, _c_ptr,
                                   ctypes.POINTER(DecodeOptions), _c_ptr]),
    "mqa_decode_noalloc": (_c_int, [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_int, _c_int, _c_int, _c_int, _c_int,
                                    _c_int, _c_float, _c_int, _c_ptr, _c_ptr]),
    "mqa_decode_beam_workspace_size": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "mqa_decode_beam": (_c_int, [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_int, _c_int,
                                 _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_ptr, _c_size,
                                 _c_ptr, _c_ptr]),
    "mqa_prefill": (_c_int, [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                             _c_int, _c_float, _c_int, _c_int, _c_ptr, _c_ptr]),
    "mqa_status_string": (ctypes.c_char_p, [_c_int]),
}


class MqaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


_LIB = None


def load_library(path: str = LIB_PATH):
    """Load libmqa.so and declare its signatures.  Raises if it is missing."""
    global _LIB
    if _LIB is not None and path == LIB_PATH:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"libmqa.so not built at {path}; run grouped_query_attention_mqa_b200.build.build()")
    lib_ = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib_, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _LIB = lib_
    return lib_


def lib():
    return load_library()


def status_string(status: int) -> str:
    return lib().mqa_status_string(int(status)).decode()


def decode_workspace_size(b: int, h: int, g: int, d_v: int) -> int:
    return int(lib().mqa_decode_workspace_size(b, h, g, d_v))


def new_workspace(b: int, h: int, g: int, d_v: int, device="cuda"):
    """A decode workspace (torch uint8 tensor) for these sizes; its contents
    on entry to a decode do not matter."""
    import torch
    return torch.empty(max(256, decode_workspace_size(b, h, g, d_v)), dtype=torch.uint8, device=device)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return MQA_F32
    if t.dtype == torch.bfloat16:
        return MQA_BF16
    raise TypeError(f"libmqa takes float32 or bfloat16 tensors, got {t.dtype}")


def _stream_handle(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _check_cuda(*tensors):
    for t in tensors:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libmqa needs contiguous CUDA tensors")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def kv_append(k_cache, v_cache, k_new, v_new, pos, status_flags=None, stream=None):
    """Write k_new [b,g,d_k] / v_new [b,g,d_v] at row pos[b] of the caches
    [b,m_max,g,d] (mqa_kv_append)."""
    import torch
    _check_cuda(k_cache, v_cache, k_new, v_new, pos, status_flags)
    b, m_max, g, d_k = k_cache.shape
    d_v = v_cache.shape[3]
    if pos.dtype != torch.int32:
        raise TypeError("pos must be int32")
    if tuple(v_cache.shape[:3]) != (b, m_max, g) or tuple(k_new.shape) != (b, g, d_k) or \
            tuple(v_new.shape) != (b, g, d_v) or tuple(pos.shape) != (b,):
        raise ValueError("kv_append: inconsistent shapes")
    dt = _dtype_code(k_cache)
    if any(_dtype_code(t) != dt for t in (v_cache, k_new, v_new)):
        raise TypeError("kv_append: caches and new rows must share one dtype")
    st = lib().mqa_kv_append(_ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new), _ptr(pos), b, m_max, g, d_k,
                             d_v, dt, _ptr(status_flags), _stream_handle(stream))
    if st != MQA_OK:
        raise MqaError(st, "mqa_kv_append")


@dataclass
class _WsCache:
    tensor: object = None


_ws = _WsCache()


def decode(q, k_cache, v_cache, lens, scale, out=None, workspace=None, status_flags=None, path="auto",
           num_ctas=0, stream=None, window=0):
    """o [b,h,d_v] = softmax over rows t < lens[b] of scale·q·K, times V
    (mqa_decode_ex); with ``window`` > 0 over the newest ``window`` rows only.
    ``workspace`` defaults to a torch-allocated buffer of
    mqa_decode_workspace_size bytes, kept for reuse."""
    import torch
    _check_cuda(q, k_cache, v_cache, lens, out, workspace, status_flags)
    b, h, d_k = q.shape
    _, m_max, g, _ = k_cache.shape
    d_v = v_cache.shape[3]
    if lens.dtype != torch.int32 or tuple(lens.shape) != (b,):
        raise ValueError("lens must be int32 [b]")
    if tuple(k_cache.shape) != (b, m_max, g, d_k) or tuple(v_cache.shape[:3]) != (b, m_max, g):
        raise ValueError("decode: inconsistent cache shapes")
    dt = _dtype_code(q)
    if any(_dtype_code(t) != dt for t in (k_cache, v_cache)):
        raise TypeError("decode: q and caches must share one dtype")
    if out is None:
        out = torch.empty((b, h, d_v), dtype=q.dtype, device=q.device)
    elif tuple(out.shape) != (b, h, d_v) or out.dtype != q.dtype:
        raise ValueError("decode: out must be [b,h,d_v] in q's dtype")
    need = decode_workspace_size(b, h, g, d_v)
    if workspace is None:
        ws = _ws.tensor
        if ws is None or ws.numel() < need or ws.device != q.device:
            ws = new_workspace(b, h, g, d_v, device=q.device)
            _ws.tensor = ws
        workspace = ws
    opts = DecodeOptions(PATHS[path], int(num_ctas), int(window))
    st = lib().mqa_decode_ex(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(lens), b, h, g, m_max, d_k, d_v,
                             float(scale), dt, _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _ptr(status_flags), ctypes.byref(opts), _stream_handle(stream))
    if st != MQA_OK:
        raise MqaError(st, "mqa_decode")
    return out


def decode_beam(q, prefix_k, prefix_v, prefix_lens, suffix_k, suffix_v, suffix_lens, scale, out=None,
                workspace=None, status_flags=None, stream=None):
    """One decode step of W beams sharing each sequence's prefix
    (mqa_decode_beam): q [b,W,h,d]; prefix caches [b,m_p,g,d] with lens [b];
    suffix caches [b*W,m_s,g,d] with lens [b*W].  Returns o [b,W,h,d]."""
    import torch
    _check_cuda(q, prefix_k, prefix_v, prefix_lens, suffix_k, suffix_v, suffix_lens, out, workspace, status_flags)
    b, W, h, d_k = q.shape
    _, m_p, g, _ = prefix_k.shape
    m_s = suffix_k.shape[1]
    d_v = prefix_v.shape[3]
    if tuple(prefix_k.shape) != (b, m_p, g, d_k) or tuple(suffix_k.shape) != (b * W, m_s, g, d_k):
        raise ValueError("decode_beam: inconsistent cache shapes")
    if prefix_lens.dtype != torch.int32 or suffix_lens.dtype != torch.int32 or prefix_lens.numel() != b \
            or suffix_lens.numel() != b * W:
        raise ValueError("decode_beam: lens must be int32 [b] and [b*W]")
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((b, W, h, d_v), dtype=q.dtype, device=q.device)
    need = lib().mqa_decode_beam_workspace_size(b, W, h, g, d_v)
    if workspace is None:
        workspace = torch.empty(max(256, need), dtype=torch.uint8, device=q.device)
    st = lib().mqa_decode_beam(_ptr(out), _ptr(q), _ptr(prefix_k), _ptr(prefix_v), _ptr(prefix_lens), _ptr(suffix_k),
                               _ptr(suffix_v), _ptr(suffix_lens), b, W, h, g, m_p, m_s, d_k, d_v, float(scale), dt,
                               _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status_flags),
                               _stream_handle(stream))
    if st != MQA_OK:
        raise MqaError(st, "mqa_decode_beam")
    return out


def prefill(q, k, v, cu_seqlens, max_seqlen, scale, causal=True, out=None, status_flags=None, stream=None):
    """Batched (prefill) attention over packed sequences (mqa_prefill): q [T,h,d],
    k/v [T,g,d], cu_seqlens int32 [b+1] on the device, max_seqlen the longest
    sequence.  Returns o [T,h,d]."""
    import torch
    _check_cuda(q, k, v, cu_seqlens, out, status_flags)
    T, h, d_k = q.shape
    if tuple(k.shape[:1]) != (T,) or k.shape[0] != v.shape[0] or k.shape[1] != v.shape[1]:
        raise ValueError("prefill: k/v must be [T,g,d] with q's T")
    g = k.shape[1]
    d_v = v.shape[2]
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be int32 [b+1]")
    dt = _dtype_code(q)
    if any(_dtype_code(t) != dt for t in (k, v)):
        raise TypeError("prefill: q, k and v must share one dtype")
    if out is None:
        out = torch.empty((T, h, d_v), dtype=q.dtype, device=q.device)
    elif tuple(out.shape) != (T, h, d_v) or out.dtype != q.dtype:
        raise ValueError("prefill: out must be [T,h,d_v] in q's dtype")
    st = lib().mqa_prefill(_ptr(out), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), cu_seqlens.numel() - 1, T,
                           int(max_seqlen), h, g, d_k, d_v, float(scale), 1 if causal else 0, dt, _ptr(status_flags),
                           _stream_handle(stream))
    if st != MQA_OK:
        raise MqaError(st, "mqa_prefill")
    return out


def decode_append(q, k_cache, v_cache, k_new, v_new, lens, scale, out=None, workspace=None, status_flags=None,
                  path="auto", num_ctas=0, stream=None, window=0):
    """One incremental step (mqa_decode_append): write k_new/v_new [b,g,d] at
    row lens[b]-1 of the caches, then attend over lens[b] rows (the newest
    ``window`` of them when window > 0).  Returns o."""
    plan = DecodePlan(q, k_cache, v_cache, lens, scale, out=out, workspace=workspace, status_flags=status_flags,
                      path=path, num_ctas=num_ctas, stream=stream, k_new=k_new, v_new=v_new, window=window)
    return plan.run()


class AppendPlan:
    """mqa_kv_append with its arguments marshalled once, for loops that repeat
    the same call (a decode step on fixed buffers): ``run()`` is one C call."""

    def __init__(self, k_cache, v_cache, k_new, v_new, pos, status_flags=None, stream=None):
        import torch
        _check_cuda(k_cache, v_cache, k_new, v_new, pos, status_flags)
        b, m_max, g, d_k = k_cache.shape
        d_v = v_cache.shape[3]
        if pos.dtype != torch.int32 or tuple(k_new.shape) != (b, g, d_k) or tuple(v_new.shape) != (b, g, d_v):
            raise ValueError("AppendPlan: inconsistent arguments")
        self._keep = (k_cache, v_cache, k_new, v_new, pos, status_flags)
        self._fn = lib().mqa_kv_append
        self._args = (_ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new), _ptr(pos), b, m_max, g, d_k, d_v,
                      _dtype_code(k_cache), _ptr(status_flags), _stream_handle(stream))

    def run(self):
        st = self._fn(*self._args)
        if st != MQA_OK:
            raise MqaError(st, "mqa_kv_append")


class DecodePlan:
    """mqa_decode_ex with its arguments marshalled once; ``run()`` is one C call
    that writes ``self.out``."""

    def __init__(self, q, k_cache, v_cache, lens, scale, out=None, workspace=None, status_flags=None, path="auto",
                 num_ctas=0, stream=None, k_new=None, v_new=None, window=0):
        import torch
        _check_cuda(q, k_cache, v_cache, lens, out, workspace, status_flags, k_new, v_new)
        b, h, d_k = q.shape
        _, m_max, g, _ = k_cache.shape
        d_v = v_cache.shape[3]
        if lens.dtype != torch.int32 or tuple(lens.shape) != (b,):
            raise ValueError("lens must be int32 [b]")
        if tuple(k_cache.shape) != (b, m_max, g, d_k) or tuple(v_cache.shape[:3]) != (b, m_max, g):
            raise ValueError("DecodePlan: inconsistent cache shapes")
        if (k_new is None) != (v_new is None):
            raise ValueError("DecodePlan: give both k_new and v_new, or neither")
        if k_new is not None and (tuple(k_new.shape) != (b, g, d_k) or tuple(v_new.shape) != (b, g, d_v)):
            raise ValueError("DecodePlan: k_new/v_new must be [b,g,d]")
        if out is None:
            out = torch.empty((b, h, d_v), dtype=q.dtype, device=q.device)
        if workspace is None:
            workspace = new_workspace(b, h, g, d_v, device=q.device)
        self.out = out
        self._opts = DecodeOptions(PATHS[path], int(num_ctas), int(window))
        self._keep = (q, k_cache, v_cache, lens, out, workspace, status_flags, k_new, v_new)
        common = (ctypes.c_float(scale), _dtype_code(q), _ptr(workspace), workspace.numel() * workspace.element_size(),
                  _ptr(status_flags), ctypes.byref(self._opts), _stream_handle(stream))
        if k_new is None:
            self._fn = lib().mqa_decode_ex
            self._args = (_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(lens), b, h, g, m_max, d_k,
                          d_v) + common
        else:
            self._fn = lib().mqa_decode_append
            self._args = (_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new), _ptr(lens), b,
                          h, g, m_max, d_k, d_v) + common

    def run(self):
        st = self._fn(*self._args)
        if st != MQA_OK:
            raise MqaError(st, "mqa_decode")
        return self.out
