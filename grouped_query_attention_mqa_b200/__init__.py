"""libmqa: single-token incremental-decode attention (MQA / GQA / MHA) over a
KV cache on NVIDIA B200 (sm_100a).

The work is done by hand-written CUDA kernels behind a C ABI (``include/mqa.h``,
built into ``libmqa.so`` next to this file).  This package holds the ctypes
binding (``binding``), the build step (``build``) and the seeded workload
generators (``workloads``).  The binding is imported lazily so that the
workloads can be used on machines without the library.
"""
from . import workloads  # noqa: F401

_BINDING_NAMES = {
    "kv_append", "decode", "decode_workspace_size", "status_string", "lib", "MqaError",
    "load_library", "DecodeOptions", "AppendPlan", "DecodePlan", "new_workspace", "decode_append",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
