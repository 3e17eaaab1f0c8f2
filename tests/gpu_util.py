"""Helpers of the GPU parity tests: host arrays to device tensors and back,
and the tolerance check.  Tolerances (max-abs, outputs of order one): 2e-3 on
the fp32 path, 1.5e-2 with bf16 inputs and outputs (fp32 accumulation)."""
import numpy as np
import torch

TOL = {"f32": 2e-3, "bf16": 1.5e-2}


def dev(arr, dtype):
    """Host array -> CUDA tensor: uint16 bit patterns become bfloat16."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).cuda()


def host64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits(t):
    """CUDA tensor -> raw bits (uint16 for bf16, uint32 for float32)."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy().view(np.uint32)


def assert_close(out, ref, dtype, what=""):
    out = np.asarray(out, dtype=np.float64)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref).max() if out.size else 0.0
    assert err <= TOL[dtype], f"{what}: max-abs error {err:.3e} > {TOL[dtype]}"
    return err
