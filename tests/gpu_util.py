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


def check_full_size_step(out, wl, seed, lens, what, K_after=None, V_after=None, k_new=None, v_new=None):
    """Check every sequence of a full-size fused step against the oracle.

    The oracle's inputs are a second, fresh draw of the workload's seeded
    device inputs (the same values the step started from, in buffers no
    kernel of the library touched); each sequence's rows go to the host one
    at a time.  With K_after/V_after given, the step's caches are checked too:
    rows before lens-1 unchanged, row lens-1 equal to the step's new row bit
    for bit."""
    from grouped_query_attention_mqa_b200.workloads import device_inputs
    from oracle import oracle_decode_step

    fresh = device_inputs(wl, seed=seed, device="cuda")
    assert np.array_equal(fresh["lens"], lens)
    Kf, Vf = fresh["k"][0], fresh["v"][0]
    qf, knf, vnf = (fresh[x].float().cpu().numpy() for x in ("q", "k_new", "v_new"))
    o = host64(out)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    worst = 0.0
    for bi in range(wl.b):
        L = int(lens[bi])
        Kb = Kf[bi, :L].float().cpu().numpy()[None]
        Vb = Vf[bi, :L].float().cpu().numpy()[None]
        ref, _, _, _ = oracle_decode_step(qf[bi:bi + 1], Kb, Vb, knf[bi:bi + 1], vnf[bi:bi + 1], np.array([L - 1]),
                                          wl.g, wl.scale)
        worst = max(worst, assert_close(o[bi:bi + 1], ref, wl.dtype, f"{what} seq {bi} len {L}"))
        if K_after is not None:
            assert torch.equal(K_after[bi, :L - 1], Kf[bi, :L - 1]) and torch.equal(V_after[bi, :L - 1], Vf[bi, :L - 1])
            assert torch.equal(K_after[bi, L - 1].view(torch.int16), k_new[bi].view(torch.int16))
            assert torch.equal(V_after[bi, L - 1].view(torch.int16), v_new[bi].view(torch.int16))
    del fresh, Kf, Vf
    torch.cuda.empty_cache()
    return worst
