"""Decode-attention benchmark: query-tokens/s and achieved HBM bandwidth of one
decode step (append the step's K/V, then attend over every valid row) on the
long-context MQA serving batch (b=64 sequences, h=32 query heads sharing one
K/V head, d=128, m_max=8192, lengths uniform in [1024, 8192]).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  Under torchrun each rank runs the same
per-GPU workload on its own GPU (weak scaling: sequences are independent, so
no collective sits on the data path); the timed region is bracketed by a
barrier and a device synchronize, and the step time is the maximum over ranks.
``--impl reference`` times the CPU float64 oracle on a bounded sample of the
same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from grouped_query_attention_mqa_b200.workloads import (BEAM_WORKLOADS, PREFILL_WORKLOADS, WORKLOADS,  # noqa: E402
                                                         append_algorithmic_bytes, decode_algorithmic_bytes,
                                                         draw_lens, f32_to_bf16_bits, bf16_bits_to_f32,
                                                         prefill_flops)

METRIC = "decode-attention achieved HBM GB/s vs peak; query-tokens/s at MQA b=64 m=8K"
UNIT = "query-tokens/s"
DEFAULT_WORKLOAD = "long_mqa_b64_m8k"
SEED = 3
L2_BYTES = 126 * 2**20


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20000)
    p.add_argument("--warmup", type=int, default=200)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD,
                   choices=sorted(WORKLOADS) + sorted(PREFILL_WORKLOADS) + sorted(BEAM_WORKLOADS))
    p.add_argument("--path", default="auto", choices=["auto", "simt", "tcgen05"])
    p.add_argument("--num-ctas", type=int, default=0)
    p.add_argument("--window", type=int, default=0, help="local attention: attend to the newest W rows (0 = all)")
    p.add_argument("--e2e-steps", type=int, default=3000)
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true", help="time the named workload only (no other workloads)")
    return p.parse_args()


# ------------------------------------------------------------------ CPU side

def cpu_sample(wl, seed, n_seq):
    """A bounded sample of the workload for the oracle: the first n_seq
    sequences with the workload's lengths, each holding only its valid rows
    (bf16-rounded N(0,1) values, like the device inputs)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = draw_lens(wl, rng)[:n_seq]
    seqs = []
    for L in lens:
        def draw(shape, std=1.0):
            x = rng.standard_normal(shape, dtype=np.float32) * np.float32(std)
            return bf16_bits_to_f32(f32_to_bf16_bits(x)) if wl.dtype == "bf16" else x
        seqs.append(dict(L=int(L), k=draw((1, int(L) - 1, wl.g, wl.d_k)), v=draw((1, int(L) - 1, wl.g, wl.d_v)),
                         q=draw((1, wl.h, wl.d_k), wl.q_std), k_new=draw((1, wl.g, wl.d_k)),
                         v_new=draw((1, wl.g, wl.d_v))))
    return seqs


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [x.get("num_threads", 0) for x in threadpool_info() if x.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(wl, seconds, n_seq=16, window=0):
    """Oracle steps (append, then attend) over sampled sequences until about
    `seconds` of CPU time has passed.  Returns (tokens/s, sequences, seconds)."""
    from oracle import oracle_decode_step   # test infrastructure: only this leg of the bench runs it

    seqs = cpu_sample(wl, SEED, n_seq)
    done, t0 = 0, time.perf_counter()
    while True:
        for s in seqs:
            # the cache holds L-1 rows; the step appends row L-1 and attends over L rows
            cache_k = np.concatenate([s["k"], np.zeros((1, 1, wl.g, wl.d_k), np.float32)], axis=1)
            cache_v = np.concatenate([s["v"], np.zeros((1, 1, wl.g, wl.d_v), np.float32)], axis=1)
            oracle_decode_step(s["q"], cache_k, cache_v, s["k_new"], s["v_new"], np.array([s["L"] - 1]), wl.g,
                               wl.scale, window=window)
            done += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            return done / el, done, el


def cpu_baseline_obj(wl, seconds, window=0):
    v, n, el = time_oracle(wl, seconds, window=window)
    return {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} sequence-steps of {wl.name} (first 16 sequences of seed {SEED}, valid rows only), "
                      f"NumPy float64 append+attend, {el:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    per_step = max(1.0, min(args.cpu_seconds, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        time_oracle(wl, 0.0, n_seq=2, window=args.window)
    rates, total_n, total_t = [], 0, 0.0
    for _ in range(args.steps):
        v, n, el = time_oracle(wl, per_step, window=args.window)
        rates.append(v)
        total_n += n
        total_t += el
    value = total_n / total_t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "b": wl.b, "h": wl.h, "g": wl.g, "d": wl.d_k, "m_max": wl.m_max,
                       "lens": f"U[{wl.len_lo},{wl.len_hi}]", "step": "kv_append + decode"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{total_n} sequence-steps of {wl.name}, {per_step:.1f} s per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ranks

def rank_seed(rank: int) -> int:
    """Each rank decodes its own independent batch (weak scaling)."""
    return SEED + rank


def reduce_over_ranks(values, device):
    """Max over ranks of each timing: the slowest rank sets the job's time.
    Runs on whatever process group is initialised (NCCL on GPUs, gloo in the
    CPU tests); returns the values unchanged on a single process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_value(world: int, b: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job query-tokens/s: every rank decodes b new tokens per step."""
    return world * b * steps / (elapsed_ms / 1e3)


# ------------------------------------------------------------------ GPU side

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            ident = str(device_index)
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", ident, "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 4:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                bits = int(parts[3], 16)
            except ValueError:
                continue
            for bit, name in self.REASONS.items():
                if bits & bit:
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def source_digest(path_name):
    """Digest of the sources that build the decode kernel behind a recorded
    ncu traffic figure (the merge kernel is not part of that figure): the code
    only (comments and blank lines dropped), so a comment edit keeps it."""
    files = ["common.cuh", "sm100.cuh", "decode_tc.cu" if path_name == "tcgen05" else "decode_simt.cu"]
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "grouped_query_attention_mqa_b200", "csrc", f)) as fh:
            for line in fh:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload, digest):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel source as it stands (profiles/dram_traffic.txt)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        parts = line.split()
        if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload:
            kv = dict(p.split("=", 1) for p in parts[2:] if "=" in p)
            if kv.get("src_sha256") == digest:
                return int(kv["bytes_per_launch"])
    return None


def resolve_path(binding, torch, requested):
    if requested != "auto":
        return requested
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 1, 128), dtype=torch.bfloat16, device="cuda")
    try:
        binding.decode(q, k, k, torch.ones(1, dtype=torch.int32, device="cuda"), 1.0, path="tcgen05")
        return "tcgen05"
    except binding.MqaError:
        return "simt"


def capture_steps(torch, stream, fn, i0, n):
    """A CUDA graph of the n steps fn(i0) .. fn(i0 + n - 1)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(i0, i0 + n):
            fn(i)
    return g


class GraphSteps:
    """Exactly K steps fn(0) .. fn(K-1), captured in CUDA graphs: one graph of
    G = min(K, g_max) steps replayed K // G times, then one graph of the
    K % G remaining steps.  With g_max a multiple of the rotation period of
    fn, every step of the run uses the input that fn(i) names."""

    def __init__(self, torch, stream, fn, K, g_max):
        self.torch, self.stream, self.K = torch, stream, K
        self.G = min(K, g_max)
        self.R, r = divmod(K, self.G)
        self.full = capture_steps(torch, stream, fn, 0, self.G)
        self.rest = capture_steps(torch, stream, fn, self.R * self.G, r) if r else None
        self.replays(1)                      # untimed: first replays upload the graphs
        torch.cuda.synchronize()

    def launch(self):
        if self.R == 1 and self.rest is None:
            return f"one CUDA graph of the {self.K} steps, replayed once"
        tail = f" + one graph of {self.K - self.R * self.G} steps" if self.rest is not None else ""
        return f"CUDA graph of {self.G} steps replayed {self.R} times{tail} (exactly {self.K} steps)"

    def replays(self, n_runs):
        with self.torch.cuda.stream(self.stream):
            for _ in range(n_runs):
                for _ in range(self.R):
                    self.full.replay()
                if self.rest is not None:
                    self.rest.replay()

    def time(self, world, burn_in_s=0.25, device_index=0):
        """Burn-in replays (untimed, so the clock record has samples under
        load), then the timed run of exactly K steps between CUDA events on
        the steps' stream.  Returns (elapsed ms, clock record)."""
        torch = self.torch
        import torch.distributed as dist
        clocks = ClockSampler(device_index)
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < burn_in_s or n < 1:
            self.replays(1)
            torch.cuda.synchronize()
            n += 1
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(self.stream):
            start.record(self.stream)
            self.replays(1)
            end.record(self.stream)
        torch.cuda.synchronize()
        clk = clocks.stop()
        if clk is not None:
            clk["window"] = f"{burn_in_s:.2f} s of the same steps replayed back to back just before the timed run, and the run"
        if world > 1:
            dist.barrier()
        return start.elapsed_time(end), clk


def launches_per_step(wl, path, window):
    """Kernels one fused step launches: the decode, and the merge unless no
    sequence can span two tiles (128 rows on tcgen05, 64 on the CUDA cores)."""
    span = min(wl.m_max, window) if window > 0 else wl.m_max
    return 1 + (span > (128 if path == "tcgen05" else 64))


def decode_workload_entry(torch, binding, wl, K, path, world, rank, local, seed_base=SEED, g_max=1200):
    """One fused-step workload timed like the headline (device-resident
    inputs, rotating cache copies, exactly K steps from CUDA graphs)."""
    from grouped_query_attention_mqa_b200.workloads import device_inputs
    cache_bytes = wl.b * wl.m_max * wl.g * (wl.d_k + wl.d_v) * wl.elem_bytes
    copies = max(3, min(8, -(-3 * L2_BYTES // cache_bytes) + 1))
    inp = device_inputs(wl, seed=seed_base + rank, device="cuda", copies=copies)
    lens_np = inp["lens"]
    lens = torch.from_numpy(lens_np).cuda()
    out = torch.empty((wl.b, wl.h, wl.d_v), dtype=inp["q"].dtype, device="cuda")
    ws = binding.new_workspace(wl.b, wl.h, wl.g, wl.d_v)
    stream = torch.cuda.Stream()
    plans = [binding.DecodePlan(inp["q"], inp["k"][c], inp["v"][c], lens, wl.scale, out=out, workspace=ws, path=path,
                                stream=stream, k_new=inp["k_new"], v_new=inp["v_new"]) for c in range(copies)]
    with torch.cuda.stream(stream):
        for i in range(3):
            plans[i % copies].run()
    torch.cuda.synchronize()
    gs = GraphSteps(torch, stream, lambda i: plans[i % copies].run(), K, g_max - g_max % copies)
    ms, clk = gs.time(world, device_index=local)
    ms = reduce_over_ranks([ms], "cuda")[0] / K
    alg = decode_algorithmic_bytes(wl, lens_np) + append_algorithmic_bytes(wl)
    peak, _ = peaks()
    entry = {"us_per_step": 1e3 * ms, "query_tokens_per_s": world * wl.b / (ms / 1e3),
             "achieved_gbs": alg / (ms / 1e3) / 1e9, "frac": alg / (ms / 1e3) / 1e9 / peak,
             "algorithmic_bytes_per_step": alg, "kv_cache_bytes": cache_bytes,
             "shape": f"b={wl.b} h={wl.h} g={wl.g} d={wl.d_k} m_max={wl.m_max} lens U[{wl.len_lo},{wl.len_hi}] "
                      f"mean {float(lens_np.mean()):.0f}", "path": path, "steps": K, "launch": gs.launch(),
             "l2": f"{copies} rotating cache copies", "clocks": clk}
    del gs, plans, inp, out, ws
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry


def paper_decoder_entry(torch, binding, world, rank, local, K):
    """The paper-shaped decoder: 128 sequences, h=8, g=1, d=128, 128 fused
    steps with the cache growing from 1 to 128 rows (all sequences equal), as
    one CUDA graph of the 128 steps; the average step time over the growth.
    The whole cache is 8 MiB, so it stays in L2 as it would in the pages'
    setting."""
    wl = WORKLOADS["paper_mqa_b128_m128"]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1000 + rank)
    rnd = lambda *s: torch.randn(s, generator=gen, device="cuda", dtype=torch.float32).to(torch.bfloat16)
    K_c, V_c = rnd(wl.b, wl.m_max, wl.g, wl.d_k), rnd(wl.b, wl.m_max, wl.g, wl.d_v)
    q, kn, vn = rnd(wl.b, wl.h, wl.d_k), rnd(wl.b, wl.g, wl.d_k), rnd(wl.b, wl.g, wl.d_v)
    T = wl.steps
    lens = [torch.full((wl.b,), t, dtype=torch.int32, device="cuda") for t in range(1, T + 1)]
    out = torch.empty((wl.b, wl.h, wl.d_v), dtype=torch.bfloat16, device="cuda")
    ws = binding.new_workspace(wl.b, wl.h, wl.g, wl.d_v)
    stream = torch.cuda.Stream()
    plans = [binding.DecodePlan(q, K_c, V_c, lens[t], wl.scale, out=out, workspace=ws, stream=stream, k_new=kn,
                                v_new=vn) for t in range(T)]
    with torch.cuda.stream(stream):
        for p in plans:
            p.run()
    torch.cuda.synchronize()
    n = T * max(1, -(-K // T))               # whole growth sequences, at least K steps
    gs = GraphSteps(torch, stream, lambda i: plans[i % T].run(), n, T * max(1, 1200 // T))
    ms, clk = gs.time(world, device_index=local)
    ms = reduce_over_ranks([ms], "cuda")[0] / n
    alg = sum(decode_algorithmic_bytes(wl, np.full(wl.b, t)) for t in range(1, T + 1)) / T + append_algorithmic_bytes(wl)
    entry = {"us_per_step": 1e3 * ms, "query_tokens_per_s": world * wl.b / (ms / 1e3),
             "achieved_gbs": alg / (ms / 1e3) / 1e9, "bound": "latency (8 MiB cache, L2-resident)",
             "shape": "b=128 h=8 g=1 d=128, cache grows 1..128 over 128 steps", "steps": n, "launch": gs.launch(),
             "clocks": clk}
    del gs, plans, K_c, V_c, out, ws
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry


def beam_entry(torch, binding, wl, K, local, seed=SEED):
    """mqa_decode_beam timed like the headline (exactly K steps from CUDA
    graphs, two rotating copies of the prefix caches), beside the same step
    with the prefix copied into every beam's cache (b*W sequences through
    mqa_decode), which must agree with it."""
    from grouped_query_attention_mqa_b200.workloads import beam_algorithmic_bytes, beam_device_inputs
    inp = beam_device_inputs(wl, seed, "cuda")
    lp, ls = torch.from_numpy(inp["lp"]).cuda(), torch.from_numpy(inp["ls"]).cuda()
    copies = [(inp["pk"], inp["pv"]), (inp["pk"].clone(), inp["pv"].clone())]
    out = torch.empty((wl.b, wl.W, wl.h, wl.d), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(256, binding.lib().mqa_decode_beam_workspace_size(wl.b, wl.W, wl.h, wl.g, wl.d)),
                     dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()

    def step(i):
        pk, pv = copies[i % 2]
        binding.decode_beam(inp["q"], pk, pv, lp, inp["sk"], inp["sv"], ls, wl.scale, out=out, workspace=ws,
                            stream=stream)

    with torch.cuda.stream(stream):
        for i in range(3):
            step(i)
    torch.cuda.synchronize()
    gs = GraphSteps(torch, stream, step, K, 400)
    ms, clk = gs.time(1, device_index=local)
    ms /= K
    launch = gs.launch()
    del gs
    # the same step with the prefix copied into every beam's cache (b*W independent sequences)
    rows = wl.m_p + wl.m_s
    rk = torch.zeros((wl.b * wl.W, rows, wl.g, wl.d), dtype=torch.bfloat16, device="cuda")
    rv = torch.zeros_like(rk)
    for s_ in range(wl.b):
        for w in range(wl.W):
            r, a, c = s_ * wl.W + w, int(inp["lp"][s_]), int(inp["ls"][s_ * wl.W + w])
            rk[r, :a] = inp["pk"][s_, :a]
            rv[r, :a] = inp["pv"][s_, :a]
            rk[r, a:a + c] = inp["sk"][r, :c]
            rv[r, a:a + c] = inp["sv"][r, :c]
    rlens = (lp.repeat_interleave(wl.W) + ls).to(torch.int32)
    rout = torch.empty((wl.b * wl.W, wl.h, wl.d), dtype=torch.bfloat16, device="cuda")
    rplan = binding.DecodePlan(inp["q"].view(wl.b * wl.W, wl.h, wl.d), rk, rv, rlens, wl.scale, out=rout,
                               stream=stream)
    with torch.cuda.stream(stream):
        rplan.run()
    torch.cuda.synchronize()
    Kr = max(3, K // 4)
    gr = GraphSteps(torch, stream, lambda i: rplan.run(), Kr, 400)
    ms_rep, _ = gr.time(1, burn_in_s=0.05, device_index=local)
    ms_rep /= Kr
    del gr
    step(0)
    torch.cuda.synchronize()
    if not torch.allclose(rout.float(), out.view(wl.b * wl.W, wl.h, wl.d).float(), atol=1.5e-2, rtol=0):
        raise RuntimeError("the shared-prefix and the replicated step disagree")
    alg = beam_algorithmic_bytes(wl, inp["lp"], inp["ls"])
    peak, _ = peaks()
    tok = wl.b * wl.W
    entry = {"us_per_step": 1e3 * ms, "query_tokens_per_s": tok / (ms / 1e3), "achieved_gbs": alg / (ms / 1e3) / 1e9,
             "frac": alg / (ms / 1e3) / 1e9 / peak, "algorithmic_bytes_per_step": alg,
             "shape": f"b={wl.b} beams={wl.W} h={wl.h} g={wl.g} d={wl.d} prefixes U[{wl.lp_lo},{wl.lp_hi}] "
                      f"suffixes U[{wl.ls_lo},{wl.ls_hi}]",
             "replicated_prefix_us_per_step": 1e3 * ms_rep, "shared_over_replicated_speedup": ms_rep / ms,
             "steps": K, "launch": launch, "l2": "2 rotating prefix-cache copies", "clocks": clk}
    del inp, copies, out, ws, rk, rv, rout, rplan
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry


def prefill_entry(torch, binding, wl, K, rank, local):
    """mqa_prefill on packed equal-length sequences, exactly K launches from
    CUDA graphs: TFLOP/s (4 h d FLOPs per attended pair) against the measured
    bf16 tensor peak (burst and sustained)."""
    from grouped_query_attention_mqa_b200.workloads import prefill_device_inputs
    inp = prefill_device_inputs(wl, seed=rank_seed(rank), device="cuda")
    out = torch.empty_like(inp["q"])
    stream = torch.cuda.Stream()

    def step(i):
        binding.prefill(inp["q"], inp["k"], inp["v"], inp["cu"], wl.n, wl.scale, causal=wl.causal, out=out,
                        stream=stream)

    with torch.cuda.stream(stream):
        for i in range(3):
            step(i)
    torch.cuda.synchronize()
    gs = GraphSteps(torch, stream, step, K, 100)
    ms, clk = gs.time(1, device_index=local)
    ms /= K
    flops = prefill_flops(wl)
    tf = flops / (ms / 1e3) / 1e12
    burst, sustained = tensor_peaks()
    entry = {"ms_per_step": ms, "tflops": tf, "frac_of_burst_peak": tf / burst if burst else None,
             "frac_of_sustained_peak": tf / sustained if sustained else None, "algorithmic_flops_per_step": flops,
             "shape": f"b={wl.b} n={wl.n} h={wl.h} g={wl.g} d={wl.d} causal={wl.causal}", "steps": K,
             "launch": gs.launch(), "clocks": clk}
    del gs, inp, out
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry


def tensor_peaks():
    """Measured dense bf16 peaks (burst, sustained) in TFLOP/s, or the
    fallback figures when no measurement is present."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained") or p["bf16_tflops"])
    except (OSError, KeyError, ValueError):
        return 1590.0, 1400.0


def extra_entries(torch, binding, world, rank, local, K):
    """The other workloads of the metric's family, each timed in this run:
    GQA-8, the MHA/MQA pair on identical shapes, and the paper-shaped decoder;
    then the beam step and the prefill (their own units)."""
    ex = {}
    for name in ("gqa8_b32_m32k", "mha_b16_m16k", "mqa_b16_m16k", "long_mqa_d64_b64_m8k"):
        wl = WORKLOADS[name]
        ex[name] = decode_workload_entry(torch, binding, wl, K, resolve_path(binding, torch, "auto"), world, rank,
                                         local)
    mha, mqa = ex["mha_b16_m16k"], ex["mqa_b16_m16k"]
    ex["mha_over_mqa"] = {"time_ratio": mha["us_per_step"] / mqa["us_per_step"],
                          "kv_cache_bytes_ratio": mha["kv_cache_bytes"] / mqa["kv_cache_bytes"],
                          "note": "same b, h, d and lengths; g = h = 32 against g = 1"}
    ex["paper_mqa_b128_m128"] = paper_decoder_entry(torch, binding, world, rank, local, K)
    ex["beam4_mqa_b64_p8k"] = beam_entry(torch, binding, BEAM_WORKLOADS["beam4_mqa_b64_p8k"], K, local)
    ex["prefill_mqa_b8_n4096"] = prefill_entry(torch, binding, PREFILL_WORKLOADS["prefill_mqa_b8_n4096"], K, rank,
                                               local)
    return ex


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from grouped_query_attention_mqa_b200 import binding
    from grouped_query_attention_mqa_b200.build import LIB, build
    from grouped_query_attention_mqa_b200.workloads import device_inputs

    if not os.path.exists(LIB):
        build()
    binding.load_library()
    wl = WORKLOADS[args.workload]
    b, h, g, d = wl.b, wl.h, wl.g, wl.d_k
    path = resolve_path(binding, torch, args.path)
    cache_bytes = wl.b * wl.m_max * wl.g * (wl.d_k + wl.d_v) * wl.elem_bytes
    # enough copies that >= 2 other steps (and >= 3x L2 of cache) pass between two uses of one copy
    copies = max(3, min(8, -(-3 * L2_BYTES // cache_bytes) + 1))
    inp = device_inputs(wl, seed=rank_seed(rank), device="cuda", copies=copies)
    lens_np = inp["lens"]
    lens = torch.from_numpy(lens_np).cuda()
    out = torch.empty((b, h, wl.d_v), dtype=inp["q"].dtype, device="cuda")
    ws = binding.new_workspace(b, h, g, wl.d_v)
    stream = torch.cuda.Stream()   # the steps' stream; their launches are captured in CUDA graphs
    # one pre-marshalled fused step (append at row lens-1, then decode) per cache copy
    steps = [binding.DecodePlan(inp["q"], inp["k"][c], inp["v"][c], lens, wl.scale, out=out, workspace=ws,
                                window=args.window, path=path, num_ctas=args.num_ctas, stream=stream,
                                k_new=inp["k_new"], v_new=inp["v_new"])
             for c in range(copies)]

    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            steps[i % copies].run()
    torch.cuda.synchronize()

    # Timed region: exactly K steps back to back, replayed from CUDA graphs as
    # a serving loop would, CUDA events on the steps' stream around the whole
    # run (events between steps would break the programmatic dependent launch
    # between one step's kernels and the next step's).
    K = args.steps
    gs = GraphSteps(torch, stream, lambda i: steps[i % copies].run(), K, 40 * copies)
    elapsed_ms, clk = gs.time(world, device_index=local)
    elapsed_ms = reduce_over_ranks([elapsed_ms], "cuda")[0]
    dec_avg_ms = elapsed_ms / K          # average duration of one step's launches
    ms_per_step = elapsed_ms / K
    value = job_value(world, b, K, elapsed_ms)
    launch_desc = gs.launch()
    del gs

    # End to end through the public API, pipelined the way a serving loop
    # overlaps transfers with compute: while step i runs its kernels, step
    # i+1's inputs come in on one copy stream and step i-1's output goes out on
    # another.  Two device slots of inputs and outputs; events order each
    # slot's reuse.  Every step still copies its own inputs from pinned host
    # memory and its own output back.  The steps are captured in a CUDA graph
    # of G steps (a multiple of the slot and cache-copy counts), replayed
    # back to back, so the host issues one launch per G steps.
    # one staging buffer per step: q, k_new, v_new and lens at 256-byte aligned offsets, one copy in
    parts = [(inp["q"], "q"), (inp["k_new"], "kn"), (inp["v_new"], "vn"), (lens, "lens")]
    offs, total = [], 0
    for t, _ in parts:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    in_h = torch.empty(total, dtype=torch.uint8).pin_memory()

    def views(buf):
        return {name: buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                for (t, name), o in zip(parts, offs)}

    for (t, name), v in zip(parts, views(in_h).values()):
        v.copy_(t.cpu())
    h2d = total
    d2h = out.numel() * out.element_size()
    n_slots = 2
    G = 100 * n_slots * copies
    R = max(1, args.e2e_steps // G)
    E = R * G
    cap = torch.cuda.Stream()
    slots = []
    for _ in range(n_slots):
        in_d = torch.empty(total, dtype=torch.uint8, device=out.device)
        sl = dict(views(in_d), in_d=in_d, out=torch.empty_like(out),
                  o_h=torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                  in_ready=torch.cuda.Event(), computed=torch.cuda.Event(), out_done=torch.cuda.Event())
        sl["plans"] = [binding.DecodePlan(sl["q"], inp["k"][c], inp["v"][c], sl["lens"], wl.scale, out=sl["out"],
                                          window=args.window,
                                          workspace=ws, path=path, num_ctas=args.num_ctas, stream=cap,
                                          k_new=sl["kn"], v_new=sl["vn"]) for c in range(copies)]
        slots.append(sl)
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_step(i):
        sl = slots[i % n_slots]
        with torch.cuda.stream(h2d_stream):
            if i >= n_slots:   # the decode of step i-2 has read this slot's inputs
                h2d_stream.wait_event(sl["computed"])
            sl["in_d"].copy_(in_h, non_blocking=True)
            sl["in_ready"].record(h2d_stream)
        cap.wait_event(sl["in_ready"])
        if i >= n_slots:       # step i-2's output has left this slot
            cap.wait_event(sl["out_done"])
        sl["plans"][i % copies].run()
        sl["computed"].record(cap)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(sl["computed"])
            sl["o_h"].copy_(sl["out"], non_blocking=True)
            sl["out_done"].record(d2h_stream)

    def e2e_steps(n):          # n steps issued from `cap`, the copy streams forked from and joined to it
        fork = torch.cuda.Event()
        fork.record(cap)
        h2d_stream.wait_event(fork)
        d2h_stream.wait_event(fork)
        for i in range(n):
            e2e_step(i)
        for sl in slots:
            cap.wait_event(sl["out_done"])

    with torch.cuda.stream(cap):
        e2e_steps(G)           # eager warm-up of the same work
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        e2e_steps(G)
    graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):   # the replays and the events that bracket them share one stream
        s2.record(stream)
        for _ in range(R):
            graph.replay()
        e2.record(stream)
    torch.cuda.synchronize()
    # same inputs and a deterministic partition: the last pipelined output equals the device-resident
    # step's on the same cache copy
    steps[(G - 1) % copies].run()
    torch.cuda.synchronize()
    if not torch.equal(slots[(G - 1) % n_slots]["o_h"], out.cpu()):
        raise RuntimeError("pipelined end-to-end output differs from the device-resident step")
    e2e_ms = reduce_over_ranks([s2.elapsed_time(e2)], "cuda")[0]
    e2e_value = job_value(world, b, E, e2e_ms)
    del graph, slots, steps
    del inp
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    alg_bytes = decode_algorithmic_bytes(wl, lens_np, args.window) + append_algorithmic_bytes(wl)
    peak, peak_kind = peaks()
    achieved = alg_bytes / (dec_avg_ms / 1e3) / 1e9
    kernel = "decode_tc_kernel" if path == "tcgen05" else "decode_simt_kernel"
    traffic = recorded_traffic(kernel, wl.name, source_digest(path))
    per_step = launches_per_step(wl, path, args.window)

    extras = None
    if args.workload == DEFAULT_WORKLOAD and not args.window and not args.no_extra:
        extras = extra_entries(torch, binding, world, rank, local, K)

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline_obj(wl, args.cpu_seconds, args.window)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "b": b, "h": h, "g": g, "d": d, "m_max": wl.m_max,
                       "lens": f"U[{wl.len_lo},{wl.len_hi}] (seed {SEED}+rank), mean {float(lens_np.mean()):.0f}",
                       "step": "mqa_decode_append: new K/V row written at lens-1, then attention over lens rows"
                               + (f" (the newest {args.window}: local window)" if args.window else ""),
                       "path": path,
                       "l2": f"{copies} rotating K/V cache copies ({copies * cache_bytes / 2**20:.0f} MiB) so each "
                             f"step's rows were evicted by >= 2 other steps' reads",
                       "parallelism": f"replicated per GPU x{world} (independent sequences, no collective)",
                       "launch": launch_desc,
                       **({"window": args.window} if args.window else {})},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic, "peak_kind": peak_kind,
                         "kernel": f"one step = mqa_decode_append call ({kernel}"
                                   + (" + merge_kernel" if per_step > 1 else "") + f"), average over the {K} "
                                   "timed steps",
                         "algorithmic_bytes_per_launch": alg_bytes, "launch_ms": dec_avg_ms},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": E, "pipeline": f"2 slots; one staging copy in, kernels, output out, on three streams; CUDA graph of "
                                            f"{G} steps replayed {R} times"},
            "gpu_launches": per_step * K,
            "clocks": clk,
        }
        if extras is not None:
            line["workloads"] = extras
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ prefill

PREFILL_METRIC = "batched (prefill) attention TFLOP/s"


def time_oracle_prefill(wl, seconds, n=512):
    """The prefill oracle on one sequence of n tokens of the workload's shape,
    repeated until about `seconds` of CPU time; returns (FLOP/s, runs, s)."""
    from oracle import oracle_prefill   # test infrastructure: only the CPU legs of the bench run it
    rng = np.random.default_rng(SEED)
    q = bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((n, wl.h, wl.d), dtype=np.float32)))
    k = bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((n, wl.g, wl.d), dtype=np.float32)))
    v = bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((n, wl.g, wl.d), dtype=np.float32)))
    pairs = n * (n + 1) // 2 if wl.causal else n * n
    done, t0 = 0, time.perf_counter()
    while True:
        oracle_prefill(q, k, v, [0, n], wl.g, wl.scale, causal=wl.causal)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            return done * 4 * wl.h * wl.d * pairs / el, done, el


def run_prefill(args):
    """mqa_prefill on packed equal-length sequences: TFLOP/s of the attention
    (4 h d FLOPs per attended pair) against the measured bf16 tensor peak."""
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = PREFILL_WORKLOADS[args.workload]
    if args.impl == "reference":
        if rank != 0:
            return
        per = max(1.0, min(args.cpu_seconds, 60.0 / max(1, args.steps + args.warmup)))
        for _ in range(args.warmup):
            time_oracle_prefill(wl, 0.0, n=128)
        rates, runs, total = [], 0, 0.0
        for _ in range(args.steps):
            r, n_runs, el = time_oracle_prefill(wl, per)
            rates.append(r)
            runs += n_runs
            total += el
        value = float(np.median(rates)) / 1e12
        print(json.dumps({"impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s",
                          "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
                          "config": {"workload": wl.name}, "data": "synthetic",
                          "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(),
                                           "kind": "oracle",
                                           "sample": f"{runs} runs of one 512-token sequence of {wl.name}'s shape, "
                                                     f"NumPy float64, {total:.1f} s"},
                          "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}), flush=True)
        return
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from grouped_query_attention_mqa_b200 import binding
    from grouped_query_attention_mqa_b200.build import LIB, build
    from grouped_query_attention_mqa_b200.workloads import prefill_device_inputs
    if not os.path.exists(LIB):
        build()
    binding.load_library()
    K = args.steps
    ent = prefill_entry(torch, binding, wl, K, rank, local)
    ms = reduce_over_ranks([ent["ms_per_step"]], "cuda")[0]
    flops = prefill_flops(wl)
    tflops = flops / (ms / 1e3) / 1e12
    value = tflops * world

    # end to end: q, k, v copied in from pinned host memory and o copied out, every step
    inp = prefill_device_inputs(wl, seed=rank_seed(rank), device="cuda")
    out = torch.empty_like(inp["q"])
    host = {name: inp[name].cpu().pin_memory() for name in ("q", "k", "v")}
    o_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dev_in = {name: torch.empty_like(inp[name]) for name in ("q", "k", "v")}
    E = max(3, min(args.e2e_steps, 50))
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record()
    for _ in range(E):
        for name in ("q", "k", "v"):
            dev_in[name].copy_(host[name], non_blocking=True)
        binding.prefill(dev_in["q"], dev_in["k"], dev_in["v"], inp["cu"], wl.n, wl.scale, causal=wl.causal, out=out)
        o_h.copy_(out, non_blocking=True)
    e2.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_over_ranks([s2.elapsed_time(e2)], "cuda")[0] / E
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size()
    burst, sustained = tensor_peaks()
    peak_kind = "measured" if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else "fallback"
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            r, runs, el = time_oracle_prefill(wl, args.cpu_seconds)
            cpu = {"value": r / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                   "sample": f"{runs} runs of one 512-token sequence of {wl.name}'s shape, NumPy float64, {el:.1f} s"}
        print(json.dumps({
            "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "b": wl.b, "n": wl.n, "h": wl.h, "g": wl.g, "d": wl.d,
                       "causal": wl.causal, "tokens_per_s": wl.total * world / (ms / 1e3),
                       "l2": "q and o (2 x %d MiB) exceed the L2; K/V tiles are meant to be reused from it"
                             % (inp["q"].numel() * 2 // 2**20), "launch": ent["launch"],
                       "parallelism": f"replicated per GPU x{world} (independent sequences, no collective)"},
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": burst, "unit": "TFLOP/s",
                         "frac": tflops / burst, "frac_of_sustained": tflops / sustained, "traffic": None,
                         "peak_kind": peak_kind,
                         "kernel": "prefill_tc_kernel, average over the timed steps",
                         "algorithmic_flops_per_launch": flops, "launch_ms": ms},
            "cpu_baseline": cpu,
            "e2e": {"value": flops / (e2e_ms / 1e3) / 1e12 * world, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": E},
            "gpu_launches": K,
            "clocks": ent["clocks"],
        }), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ beams sharing a prefix

BEAM_METRIC = "beam decode (shared prefix) achieved HBM GB/s vs peak; query-tokens/s"


def run_beam(args):
    """mqa_decode_beam: query-tokens/s (b*W per step) and GB/s of algorithmic
    bytes (each prefix row once).  Beside it, the same step with every beam
    holding its own copy of the prefix (b*W sequences through mqa_decode)."""
    import torch
    from grouped_query_attention_mqa_b200 import binding
    from grouped_query_attention_mqa_b200.build import LIB, build
    from grouped_query_attention_mqa_b200.workloads import beam_algorithmic_bytes, beam_device_inputs

    wl = BEAM_WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        from oracle import oracle_decode_beam   # test infrastructure: only the CPU legs of the bench run it
        rng = np.random.default_rng(SEED)
        b = 2                                    # a bounded sample: two sequences of the workload's shape
        lp = rng.integers(wl.lp_lo, wl.lp_hi + 1, size=b)
        ls = rng.integers(wl.ls_lo, wl.ls_hi + 1, size=b * wl.W)
        arr = {n: rng.standard_normal(sh, dtype=np.float32) for n, sh in (
            ("q", (b, wl.W, wl.h, wl.d)), ("pk", (b, wl.m_p, wl.g, wl.d)), ("pv", (b, wl.m_p, wl.g, wl.d)),
            ("sk", (b * wl.W, wl.m_s, wl.g, wl.d)), ("sv", (b * wl.W, wl.m_s, wl.g, wl.d)))}
        rates = []
        for _ in range(max(1, args.steps)):
            t0 = time.perf_counter()
            oracle_decode_beam(arr["q"], arr["pk"], arr["pv"], lp, arr["sk"], arr["sv"], ls, wl.g, wl.scale)
            rates.append(b * wl.W / (time.perf_counter() - t0))
        value = float(np.median(rates))
        print(json.dumps({"impl": "reference", "metric": BEAM_METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
                          "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
                          "config": {"workload": wl.name}, "data": "synthetic",
                          "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                           "sample": f"2 sequences x {wl.W} beams of {wl.name}, NumPy float64"},
                          "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if not os.path.exists(LIB):
        build()
    binding.load_library()
    K = args.steps
    ent = beam_entry(torch, binding, wl, K, local)
    ms = ent["us_per_step"] / 1e3
    # end to end: q in from pinned host memory and o out, every step
    inp = beam_device_inputs(wl, SEED, "cuda")
    lp, ls = torch.from_numpy(inp["lp"]).cuda(), torch.from_numpy(inp["ls"]).cuda()
    out = torch.empty((wl.b, wl.W, wl.h, wl.d), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(256, binding.lib().mqa_decode_beam_workspace_size(wl.b, wl.W, wl.h, wl.g, wl.d)),
                     dtype=torch.uint8, device="cuda")
    q_h = inp["q"].cpu().pin_memory()
    o_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    q_d = torch.empty_like(inp["q"])

    def e2e_step():
        q_d.copy_(q_h, non_blocking=True)
        binding.decode_beam(q_d, inp["pk"], inp["pv"], lp, inp["sk"], inp["sv"], ls, wl.scale, out=out, workspace=ws)
        o_h.copy_(out, non_blocking=True)

    E = max(10, K // 4)
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(E):
        e2e_step()
    s1.record()
    torch.cuda.synchronize()
    e2e_ms = s0.elapsed_time(s1) / E
    peak, peak_kind = peaks()
    tok = wl.b * wl.W
    print(json.dumps({
        "metric": BEAM_METRIC, "value": tok / (ms / 1e3), "unit": UNIT, "n_gpus": 1, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "b": wl.b, "beams": wl.W, "h": wl.h, "g": wl.g, "d": wl.d,
                   "prefix_lens": f"U[{wl.lp_lo},{wl.lp_hi}]", "suffix_lens": f"U[{wl.ls_lo},{wl.ls_hi}]",
                   "replicated_prefix_ms_per_step": ent["replicated_prefix_us_per_step"] / 1e3,
                   "replicated_prefix_query_tokens_per_s": tok / (ent["replicated_prefix_us_per_step"] / 1e6),
                   "launch": ent["launch"], "l2": ent["l2"]},
        "roofline": {"bound": "hbm", "achieved": ent["achieved_gbs"], "peak": peak, "unit": "GB/s",
                     "frac": ent["frac"], "traffic": None, "peak_kind": peak_kind,
                     "kernel": "one step = decode_tc_beam_kernel (prefix once for the W beams, then each beam's "
                               "suffix) + merge_kernel", "algorithmic_bytes_per_launch": ent["algorithmic_bytes_per_step"],
                     "launch_ms": ms},
        "cpu_baseline": None,
        "e2e": {"value": tok / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": q_h.numel() * 2,
                "d2h_bytes_per_step": o_h.numel() * 2, "steps": E},
        "gpu_launches": 2 * K,
        "clocks": ent["clocks"],
    }), flush=True)


def main():
    args = parse()
    if args.workload in BEAM_WORKLOADS:
        run_beam(args)
    elif args.workload in PREFILL_WORKLOADS:
        run_prefill(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
