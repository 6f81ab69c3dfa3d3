"""Device-timed benchmark of causal self-attention forward + backward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one forward (gpt2_attn_fwd) plus one backward (the two steps of
gpt2_attn_bwd: dQ with Delta, then dK/dV) over one batch of the GPT-2 124M training shape B=16, T=1024,
H=12, D=64, bf16 (seeded synthetic q, k, v, dO ~ N(0, 1)). The metric is
causal attention fwd+bwd TFLOPS with the FLOPs counted as 2*B*H*T^2*D for the
forward and 2.5x that for the backward, reported against the B200 dense bf16
tensor-core peak.

Timing: W untimed warm-up steps, then exactly K steps between CUDA events on
the launching stream, with a barrier and torch.cuda.synchronize() on both
sides; the max over ranks is taken. Each step uses the next of four input/
output buffer sets (~0.8 GB in all), so no step finds its inputs in the
126 MB L2. Events recorded between the three launches of every step give each
kernel's average duration, which feeds the roofline object. With --gpus N > 1
(torchrun, one process per GPU) every rank runs its own replica: attention
has no exchange step, so the scaling is weak and there is no data-path
collective.

--impl reference times the CPU oracle (fp64 NumPy) on a bounded sample of the
same workload on this host's cores.

--context times torch's scaled_dot_product_attention (forward + backward
through autograd) on the same workload and prints one line: a context
figure, not this library's result.

--fp8 times the FP8 forward (gpt2_attn_fwd_fp8) and its quantisation pass,
with the bf16 forward on the same inputs for reference. --linear times the
dense layers around attention (c_attn, c_proj) at the workload's B, T, C.

--v16 times the inference path with v in fp16 from c_attn: the forward that
reads it (gpt2_attn_fwd_v16) next to the bf16 forward on the same values, and
c_attn writing the fp16 v slot (gpt2_attn_qkv_proj_v16).

--decode times decode attention instead (gpt2_attn_decode: the newest row
t = T-1 of every (b, h) over the keys and values of rows 0..T-1), one GPU,
and prints its own line: bytes of k and v read per second against the
measured HBM copy bandwidth.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "gpt2-124m-b16-t1024"
METRIC = "causal attn fwd+bwd TFLOPS at GPT-2 124M shape (bf16), % of B200 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
N_SETS = 4


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# The sources each kernel's code comes from: its own header plus the shared
# helpers and the host file that configures its launch.
KERNEL_SOURCES = {
    "fwd": ("fwd.cuh",),
    "bwd_dq": ("bwd.cuh",),
    "bwd_dkdv": ("bwd.cuh",),
    "bwd_prepare": ("bwd.cuh",),
    "bwd_fused": ("bwd_fused.cuh", "bwd.cuh"),
}
COMMON_SOURCES = ("common.cuh", "ptx.cuh", "gpt2attn.cu")


def kernel_digest(kernel: str, csrc: str | None = None) -> str:
    """Digest of the sources a kernel is built from (changes when its code can)."""
    csrc = csrc or os.path.join(ROOT, "causal_self_attention_flashattention_b200", "csrc")
    h = hashlib.sha256()
    for name in COMMON_SOURCES + KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def load_traffic():
    """DRAM bytes per launch from the last committed ncu capture, for the
    kernels whose sources are unchanged since that capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return {}
    return {k: v for k, v in d.get("kernels", {}).items()
            if k in KERNEL_SOURCES and v.get("src_digest") == kernel_digest(k)}


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "power_w_max": max(power), "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# CPU oracle timing (the reported baseline and the --impl reference arm)
# ---------------------------------------------------------------------------
def _oracle_head(args):
    Q, K, V, dO, scale = args
    from oracle import oracle as orc

    orc.head_forward(Q, K, V, scale)
    orc.head_backward(Q, K, V, dO, scale)
    return 0


def _pool_init():
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"


class OracleTimer:
    """Times the fp64 oracle's forward + backward on whole heads of the
    workload, one head per worker process at a time."""

    def __init__(self, wl, seed=0):
        import multiprocessing as mp

        from causal_self_attention_flashattention_b200.workload import make_inputs

        self.wl = wl
        self.cores = len(os.sched_getaffinity(0))
        qkv, dout = make_inputs(1, wl.T, min(wl.H, 4), wl.D, seed=seed, qk_std=wl.qk_std)
        q64 = qkv.double().numpy()
        d64 = dout.double().numpy()
        self.heads = [(q64[0, :, 0, h].copy(), q64[0, :, 1, h].copy(), q64[0, :, 2, h].copy(),
                       d64[0, :, h].copy(), wl.scale) for h in range(q64.shape[3])]
        self.pool = mp.get_context("spawn").Pool(self.cores, initializer=_pool_init)
        self.pool.map(_oracle_head, [self.heads[0]] * self.cores)  # warm the workers

    def head_flops(self):
        wl = self.wl
        return 7.0 * wl.T * wl.T * wl.D  # 2*T^2*D forward + 2.5x backward, one head

    def run(self, n_heads):
        tasks = [self.heads[i % len(self.heads)] for i in range(n_heads)]
        t0 = time.perf_counter()
        self.pool.map(_oracle_head, tasks, chunksize=1)
        return time.perf_counter() - t0

    def close(self):
        self.pool.terminate()
        self.pool.join()


def cpu_baseline(wl, budget_s=15.0):
    timer = OracleTimer(wl)
    try:
        n = timer.cores
        elapsed = timer.run(n)
        total_heads, total_t = n, elapsed
        while total_t < budget_s:
            n_more = max(timer.cores, int(timer.cores * (budget_s - total_t) / max(elapsed, 1e-3)))
            n_more = min(n_more, 8 * timer.cores)
            elapsed = timer.run(n_more)
            total_heads += n_more
            total_t += elapsed
        tflops = total_heads * timer.head_flops() / total_t / 1e12
        return {"value": tflops, "unit": "TFLOPS", "cores": timer.cores, "kind": "oracle",
                "sample": f"{total_heads} whole heads (T={wl.T}, D={wl.D}) of {wl.name}, fp64 "
                          f"NumPy fwd+bwd, one process per core, {total_t:.1f} s"}
    finally:
        timer.close()


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    timer = OracleTimer(wl)
    try:
        n = timer.cores
        for _ in range(args.warmup):
            timer.run(n)
        t = 0.0
        for _ in range(args.steps):
            t += timer.run(n)
        flops = args.steps * n * timer.head_flops()
        value = flops / t / 1e12
        line = {
            "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "H": wl.H, "D": wl.D,
                       "step": f"{n} whole heads of the workload (one per core)"},
            "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": timer.cores,
                             "kind": "oracle",
                             "sample": f"{n} heads (T={wl.T}, D={wl.D}) per step, fp64 NumPy "
                                       "fwd+bwd, one process per core"},
            "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
    finally:
        timer.close()
    return 0


# ---------------------------------------------------------------------------
# The CUDA path
# ---------------------------------------------------------------------------
def max_over_ranks(x: float, device) -> float:
    """The maximum of x over all ranks of the process group (x itself when
    there is none): a multi-rank time is the slowest rank's."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, steps: int, step_flops: float, ms: float) -> float:
    """Whole-job throughput: every rank ran `steps` steps of `step_flops` in at
    most `ms` milliseconds (weak scaling)."""
    return world * steps * step_flops / (ms * 1e-3) / 1e12


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)

    # The oracle's worker pool (spawned) is started before any kernel runs.
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, budget_s=args.cpu_seconds)

    from causal_self_attention_flashattention_b200 import build
    build.build()
    from causal_self_attention_flashattention_b200 import ops
    from causal_self_attention_flashattention_b200.workload import (algorithmic_bytes,
                                                                    attention_flops, make_inputs)

    B, T, H, D, scale = wl.B, wl.T, wl.H, wl.D, wl.scale
    qkv_cpu, dout_cpu = make_inputs(B, T, H, D, seed=rank, qk_std=wl.qk_std)
    n_sets = args.sets
    sets = []
    for _ in range(n_sets):
        sets.append(dict(
            qkv=qkv_cpu.to(dev), dout=dout_cpu.to(dev),
            out=torch.empty(B, T, H, D, dtype=torch.bfloat16, device=dev),
            lse=torch.empty(B, H, T, dtype=torch.float32, device=dev),
            delta=torch.empty(B, H, T, dtype=torch.float32, device=dev),
            dqkv=torch.empty(B, T, 3, H, D, dtype=torch.bfloat16, device=dev)))
    stream = torch.cuda.current_stream()

    def step(s, ev=None):
        if ev is not None:
            ev[0].record(stream)
        ops.attn_fwd(s["qkv"], scale, out=s["out"], lse=s["lse"], stream=stream)
        ops.attn_bwd_split_steps(s["qkv"], s["out"], s["dout"], s["lse"], s["delta"], s["dqkv"],
                                 scale, stream=stream, events=None if ev is None else ev[1:])

    for i in range(args.warmup):
        step(sets[i % n_sets])
    torch.cuda.synchronize()
    st, word = ops.last_device_status()
    if st != ops.GA_OK:
        raise RuntimeError(f"device status after warm-up: {ops.status_string(st)} ({word:#x})")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = None
    if rank == 0:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
        sampler.start()

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    t_start.record(stream)
    for i in range(K):
        step(sets[i % n_sets], evs[i])
    evs[-1][3].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    st, word = ops.last_device_status()
    if st != ops.GA_OK:
        raise RuntimeError(f"device status after timing: {ops.status_string(st)} ({word:#x})")

    total_ms = t_start.elapsed_time(t_end)
    # Host cost of issuing a step (the Python binding, the C-ABI argument
    # checks, tensor-map lookups and three launches), without the per-kernel
    # events: wall-clock time of K_h back-to-back steps before the device
    # catches up, per step. At small shapes this, not the kernels, sets the
    # step time.
    k_host = min(K, 200)
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    for i in range(k_host):
        step(sets[i % n_sets])
    host_us = (time.perf_counter() - h0) / k_host * 1e6
    torch.cuda.synchronize()
    names = ["fwd", "bwd_dq", "bwd_dkdv"]
    per = {n: 0.0 for n in names}
    for ev in evs:
        for k, n in enumerate(names):
            per[n] += ev[k].elapsed_time(ev[k + 1])
    per = {n: v / K for n, v in per.items()}

    total_ms = max_over_ranks(total_ms, dev)

    fwd_flops, bwd_flops = attention_flops(B, T, H, D)
    step_flops = fwd_flops + bwd_flops
    value = job_tflops(world, K, step_flops, total_ms)
    peaks, peak_src = load_peaks()
    peak_tflops = float(peaks["bf16_tflops"])

    # Per-kernel figures. Tensor-core kernels: the causal-triangle matmul FLOPs
    # each one performs (units of B*H*T^2*D: fwd 2, dK/dV 4, dQ 3).
    unit = float(B) * H * T * T * D
    kflops = {"fwd": 2 * unit, "bwd_dkdv": 4 * unit, "bwd_dq": 3 * unit}
    fwd_bytes, _ = algorithmic_bytes(B, T, H, D)
    o_bytes = B * T * H * D * 2
    lse_bytes = B * H * T * 4
    qkv_bytes = 3 * o_bytes
    kbytes = {
        "fwd": fwd_bytes,
        # q, k, v, dO read; dk, dv written; lse and Delta read.
        "bwd_dkdv": qkv_bytes + o_bytes + 2 * lse_bytes + 2 * o_bytes,
        # q, k, v, dO, O and lse read; dq and Delta written.
        "bwd_dq": qkv_bytes + 2 * o_bytes + 2 * lse_bytes + o_bytes,
    }
    kernels = {}
    for n in names:
        ms = per[n]
        d = {"ms": ms, "gbs": kbytes[n] / (ms * 1e-3) / 1e9}
        if n in kflops:
            d["tflops"] = kflops[n] / (ms * 1e-3) / 1e12
            d["frac_of_peak"] = d["tflops"] / peak_tflops
        else:
            d["frac_of_hbm"] = d["gbs"] / float(peaks["hbm_gbs"])
        kernels[n] = d
    dominant = max(names, key=lambda n: per[n])
    traffic = load_traffic()
    dom = kernels[dominant]
    if dominant in kflops:
        roof = {"kernel": dominant, "bound": "tensor", "achieved": dom["tflops"],
                "peak": peak_tflops, "unit": "TFLOP/s", "frac": dom["tflops"] / peak_tflops,
                "peak_source": f"bf16_tflops (burst) of {peak_src}"}
    else:
        roof = {"kernel": dominant, "bound": "hbm", "achieved": dom["gbs"],
                "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                "frac": dom["gbs"] / float(peaks["hbm_gbs"]), "peak_source": f"hbm_gbs of {peak_src}"}
    roof["traffic"] = traffic.get(dominant, {}).get("dram_bytes_per_launch")

    # End to end through the public API: pinned host buffers, copies in the timed region.
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, wl, ops, dev, qkv_cpu, dout_cpu, step_flops, world)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "pct_of_peak": 100.0 * value / (world * peak_tflops),
            "config": {"workload": wl.name, "B": B, "T": T, "H": H, "D": D, "scale": scale,
                       "flops_per_step": step_flops, "parallelism": f"replicas x{world}",
                       "l2": f"{n_sets} rotating input/output sets "
                             f"({n_sets * (2 * qkv_bytes + 3 * o_bytes) / 1e9:.2f} GB; "
                             f"{2 * qkv_bytes + 3 * o_bytes + 2 * lse_bytes} B touched per step) "
                             "> 126 MB L2",
                       "step": "gpt2_attn_fwd + gpt2_attn_bwd (dQ with Delta, dK/dV)"},
            "clocks": clocks, "e2e": e2e, "gpu_launches": 3 * K,
            "host": {"issue_us_per_step": host_us, "steps": k_host,
                     "what": "wall-clock per step of issuing fwd + bwd from Python (binding, "
                             "checks, tensor maps, 3 launches); not in the timed region"},
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu,
            "wall_s_timed_region": wall,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(args, wl, ops, dev, qkv_cpu, dout_cpu, step_flops, world):
    """The metric through the public API with host buffers: every step copies
    its inputs from pinned host memory, runs gpt2_attn_fwd + gpt2_attn_bwd and
    copies out, lse and dqkv back. Steps are pipelined over two device buffer
    sets and three streams (copy-in, compute, copy-out), so one step's copies
    overlap the neighbouring steps' compute and copies in the other direction,
    as a training loop that prefetches its next batch does."""
    import torch
    import torch.distributed as dist

    B, T, H, D, scale = wl.B, wl.T, wl.H, wl.D, wl.scale
    h_qkv = qkv_cpu.pin_memory()
    h_dout = dout_cpu.pin_memory()
    n_sets = 2
    host_out = [dict(out=torch.empty(B, T, H, D, dtype=torch.bfloat16).pin_memory(),
                     lse=torch.empty(B, H, T, dtype=torch.float32).pin_memory(),
                     dqkv=torch.empty(B, T, 3, H, D, dtype=torch.bfloat16).pin_memory())
                for _ in range(n_sets)]
    dev_sets = [dict(qkv=torch.empty_like(qkv_cpu, device=dev),
                     dout=torch.empty_like(dout_cpu, device=dev),
                     out=torch.empty(B, T, H, D, dtype=torch.bfloat16, device=dev),
                     lse=torch.empty(B, H, T, dtype=torch.float32, device=dev),
                     dqkv=torch.empty(B, T, 3, H, D, dtype=torch.bfloat16, device=dev),
                     ws=torch.empty(ops.bwd_workspace_size(B, T, H, D), dtype=torch.uint8,
                                    device=dev))
                for _ in range(n_sets)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(n_sets)]
    ev_comp = [torch.cuda.Event() for _ in range(n_sets)]
    ev_out = [torch.cuda.Event() for _ in range(n_sets)]
    used = [False] * n_sets

    def step(i):
        k = i % n_sets
        d, h = dev_sets[k], host_out[k]
        if used[k]:
            # Set k is free once the step that used it two steps ago has copied
            # its results out (its compute finished before that copy began).
            s_in.wait_event(ev_out[k])
        used[k] = True
        with torch.cuda.stream(s_in):
            d["qkv"].copy_(h_qkv, non_blocking=True)
            d["dout"].copy_(h_dout, non_blocking=True)
            ev_in[k].record(s_in)
        s_comp.wait_event(ev_in[k])
        ops.attn_fwd(d["qkv"], scale, out=d["out"], lse=d["lse"], stream=s_comp)
        ops.attn_bwd(d["qkv"], d["out"], d["dout"], d["lse"], scale, dqkv=d["dqkv"],
                     workspace=d["ws"], stream=s_comp)
        ev_comp[k].record(s_comp)
        s_out.wait_event(ev_comp[k])
        with torch.cuda.stream(s_out):
            h["out"].copy_(d["out"], non_blocking=True)
            h["lse"].copy_(d["lse"], non_blocking=True)
            h["dqkv"].copy_(d["dqkv"], non_blocking=True)
            ev_out[k].record(s_out)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    K = max(3, min(args.steps, args.e2e_steps))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    a.record(s_in)
    for i in range(K):
        step(3 + i)
    b.record(s_out)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    st, word = ops.last_device_status()
    if st != ops.GA_OK:
        raise RuntimeError(f"device status after the end-to-end run: {ops.status_string(st)} ({word:#x})")
    ms = max_over_ranks(ms, dev)
    h2d = h_qkv.numel() * 2 + h_dout.numel() * 2
    d2h = sum(host_out[0][n].numel() * host_out[0][n].element_size() for n in ("out", "lse", "dqkv"))
    return {"value": job_tflops(world, K, step_flops, ms), "unit": "TFLOPS",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K,
            "ms_per_step": ms / K,
            "pipeline": "2 device buffer sets; copy-in, compute and copy-out streams"}


def run_decode(args, wl):
    import torch

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from causal_self_attention_flashattention_b200 import build
    build.build()
    from causal_self_attention_flashattention_b200 import ops
    from causal_self_attention_flashattention_b200.workload import make_inputs

    B, T, H, D, scale = wl.B, wl.T, wl.H, wl.D, wl.scale
    t = T - 1
    qkv_cpu, _ = make_inputs(B, T, H, D, seed=0, qk_std=wl.qk_std)
    # Rotating qkv buffers: 4 x 75 MB > L2, so each step reads k and v from HBM.
    sets = [qkv_cpu.to(dev) for _ in range(args.sets)]
    out = torch.empty(B, H, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, dtype=torch.float32, device=dev)
    ws = torch.empty(ops.decode_workspace_size(B, T, H, D), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        ops.attn_decode(sets[i % len(sets)], t, scale, out=out, lse=lse, workspace=ws, stream=stream)
    torch.cuda.synchronize()
    st, word = ops.last_device_status()
    if st != ops.GA_OK:
        raise RuntimeError(f"device status after warm-up: {ops.status_string(st)} ({word:#x})")
    K = args.steps
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for i in range(K):
        ops.attn_decode(sets[i % len(sets)], t, scale, out=out, lse=lse, workspace=ws, stream=stream)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / K
    kv_bytes = 2 * B * H * (t + 1) * D * 2          # k and v rows 0..t, bf16
    step_bytes = kv_bytes + B * H * D * 2 * 2 + B * H * 4  # + q read, out write, lse write
    peaks, peak_src = load_peaks()
    gbs = step_bytes / (ms * 1e-3) / 1e9
    line = {
        "metric": "decode attention: bytes of q, k, v read and out, lse written per second",
        "value": gbs, "unit": "GB/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "B": B, "T": T, "H": H, "D": D, "t": t,
                   "l2": f"{len(sets)} rotating qkv buffers of {qkv_cpu.numel() * 2} B > 126 MB L2",
                   "step": "gpt2_attn_decode (partial per 128-key chunk, TMA-staged, then combine)"},
        "roofline": {"kernel": "decode", "bound": "hbm", "achieved": gbs,
                     "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                     "frac": gbs / float(peaks["hbm_gbs"]), "peak_source": f"hbm_gbs of {peak_src}",
                     "algorithmic_bytes": step_bytes},
        "gpu_launches": 2 * K,
    }
    print(json.dumps(line), flush=True)
    return 0


def _time_device(fn, steps, warmup, stream):
    """Average device time (ms) of fn() over `steps` calls on `stream`."""
    import torch

    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def run_fp8(args, wl):
    """The FP8 forward (gpt2_attn_fwd_fp8) and its quantisation pass
    (gpt2_attn_fp8_quantize), timed separately, next to the bf16 forward on the
    same inputs: forward TFLOPS (2*B*H*T^2*D) against the dense e4m3 peak,
    taken as the measured bf16 peak times 2, the nominal fp8/bf16 ratio."""
    import torch

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from causal_self_attention_flashattention_b200 import build
    build.build()
    from causal_self_attention_flashattention_b200 import ops
    from causal_self_attention_flashattention_b200.workload import attention_flops, make_inputs

    B, T, H, D, scale = wl.B, wl.T, wl.H, wl.D, wl.scale
    qkv_cpu, _ = make_inputs(B, T, H, D, seed=0, qk_std=wl.qk_std)
    sets = []
    for _ in range(args.sets):
        qkv = qkv_cpu.to(dev)
        qkv8, scales = ops.fp8_quantize(qkv)
        sets.append(dict(qkv=qkv, qkv8=qkv8, scales=scales,
                         out=torch.empty(B, T, H, D, dtype=torch.bfloat16, device=dev),
                         lse=torch.empty(B, H, T, dtype=torch.float32, device=dev)))
    stream = torch.cuda.current_stream()
    n = len(sets)
    ms_fp8 = _time_device(lambda i: ops.attn_fwd_fp8(sets[i % n]["qkv8"], sets[i % n]["scales"], scale,
                                                     out=sets[i % n]["out"], lse=sets[i % n]["lse"],
                                                     stream=stream), args.steps, args.warmup, stream)
    ms_q = _time_device(lambda i: ops.fp8_quantize(sets[i % n]["qkv"], qkv8=sets[i % n]["qkv8"],
                                                   scales=sets[i % n]["scales"], stream=stream),
                        args.steps, args.warmup, stream)
    ms_bf16 = _time_device(lambda i: ops.attn_fwd(sets[i % n]["qkv"], scale, out=sets[i % n]["out"],
                                                  lse=sets[i % n]["lse"], stream=stream),
                           args.steps, args.warmup, stream)
    st, word = ops.last_device_status()
    if st != ops.GA_OK:
        raise RuntimeError(f"device status: {ops.status_string(st)} ({word:#x})")
    fwd_flops, _ = attention_flops(B, T, H, D)
    peaks, peak_src = load_peaks()
    fp8_peak = 2.0 * float(peaks["bf16_tflops"])
    tf = fwd_flops / (ms_fp8 * 1e-3) / 1e12
    line = {
        "metric": "causal attention FP8 forward TFLOPS (e4m3 q, k, v; per-tensor scales)",
        "value": tf, "unit": "TFLOPS", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_fp8, "higher_is_better": True, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": wl.name, "B": B, "T": T, "H": H, "D": D,
                   "l2": f"{n} rotating input sets"},
        "roofline": {"kernel": "fwd_fp8", "bound": "tensor", "achieved": tf, "peak": fp8_peak,
                     "unit": "TFLOP/s", "frac": tf / fp8_peak,
                     "peak_source": f"bf16_tflops of {peak_src} x 2 (nominal e4m3/bf16 ratio)"},
        "quantize_ms": ms_q, "bf16_fwd_ms": ms_bf16,
        "gpu_launches": args.steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_v16(args, wl):
    """The fp16-v forward (gpt2_attn_fwd_v16) on the workload's q, k, v with
    the v slot stored as fp16, next to the bf16 forward (gpt2_attn_fwd) on the
    same values, and c_attn writing that qkv (gpt2_attn_qkv_proj_v16): forward
    TFLOPS (2*B*H*T^2*D) against the measured bf16 peak (the products run in
    bf16 and fp16, which share the peak)."""
    import torch

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from causal_self_attention_flashattention_b200 import build
    build.build()
    from causal_self_attention_flashattention_b200 import ops
    from causal_self_attention_flashattention_b200.workload import (attention_flops, make_inputs,
                                                                   make_linear_inputs)

    B, T, H, D, scale = wl.B, wl.T, wl.H, wl.D, wl.scale
    C = H * D
    qkv_cpu, _ = make_inputs(B, T, H, D, seed=0, qk_std=wl.qk_std)
    q16_cpu = qkv_cpu.clone()
    q16_cpu[:, :, 2] = qkv_cpu[:, :, 2].to(torch.float16).view(torch.bfloat16)
    sets = [dict(qkv=qkv_cpu.to(dev), q16=q16_cpu.to(dev),
                 out=torch.empty(B, T, H, D, dtype=torch.bfloat16, device=dev),
                 lse=torch.empty(B, H, T, dtype=torch.float32, device=dev))
            for _ in range(args.sets)]
    stream = torch.cuda.current_stream()
    n = len(sets)
    ms_v16 = _time_device(lambda i: ops.attn_fwd_v16(sets[i % n]["q16"], scale, out=sets[i % n]["out"],
                                                     lse=sets[i % n]["lse"], stream=stream),
                          args.steps, args.warmup, stream)
    ms_bf16 = _time_device(lambda i: ops.attn_fwd(sets[i % n]["qkv"], scale, out=sets[i % n]["out"],
                                                  lse=sets[i % n]["lse"], stream=stream),
                           args.steps, args.warmup, stream)
    x, w, b = make_linear_inputs(B, T, C, 3 * C, seed=0)
    lin_sets = [dict(x=x.to(dev), w=w.to(dev), b=b.to(dev),
                     qkv=torch.empty(B, T, 3, H, D, dtype=torch.bfloat16, device=dev))
                for _ in range(args.sets)]
    ms_proj = _time_device(lambda i: ops.qkv_proj(lin_sets[i % n]["x"], lin_sets[i % n]["w"],
                                                  lin_sets[i % n]["b"], H, qkv=lin_sets[i % n]["qkv"],
                                                  stream=stream, v_fp16=True),
                           args.steps, args.warmup, stream)
    st, word = ops.last_device_status()
    if st != ops.GA_OK:
        raise RuntimeError(f"device status: {ops.status_string(st)} ({word:#x})")
    fwd_flops, _ = attention_flops(B, T, H, D)
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    tf = fwd_flops / (ms_v16 * 1e-3) / 1e12
    line = {
        "metric": "causal attention forward TFLOPS, v in fp16 from c_attn (gpt2_attn_fwd_v16)",
        "value": tf, "unit": "TFLOPS", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_v16, "higher_is_better": True, "dtype": "bf16 q,k / fp16 v",
        "data": "synthetic",
        "config": {"workload": wl.name, "B": B, "T": T, "H": H, "D": D,
                   "l2": f"{n} rotating input sets"},
        "roofline": {"kernel": "fwd_v16", "bound": "tensor", "achieved": tf, "peak": peak,
                     "unit": "TFLOP/s", "frac": tf / peak,
                     "peak_source": f"bf16_tflops of {peak_src}"},
        "bf16_fwd_ms": ms_bf16, "qkv_proj_v16_ms": ms_proj,
        "gpu_launches": args.steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_linear(args, wl):
    """The dense layers around attention (gpt2_attn_qkv_proj, gpt2_attn_out_proj)
    at the workload's B, T and width C = 64 H: TFLOPS against the measured bf16
    peak, one line each."""
    import torch

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from causal_self_attention_flashattention_b200 import build
    build.build()
    from causal_self_attention_flashattention_b200 import ops
    from causal_self_attention_flashattention_b200.workload import make_linear_inputs

    B, T, H = wl.B, wl.T, wl.H
    C = 64 * H
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    for name, n_out in (("c_attn (gpt2_attn_qkv_proj)", 3 * C), ("c_proj (gpt2_attn_out_proj)", C)):
        x, w, b = make_linear_inputs(B, T, C, n_out, seed=0)
        sets = [dict(x=x.to(dev), w=w.to(dev), b=b.to(dev),
                     y=torch.empty(B, T, n_out, dtype=torch.bfloat16, device=dev))
                for _ in range(args.sets)]
        n = len(sets)
        if n_out == 3 * C:
            fn = lambda i: ops.qkv_proj(sets[i % n]["x"], sets[i % n]["w"], sets[i % n]["b"], H,
                                        qkv=sets[i % n]["y"].view(B, T, 3, H, 64), stream=stream)
        else:
            fn = lambda i: ops.out_proj(sets[i % n]["x"].view(B, T, H, 64), sets[i % n]["w"],
                                        sets[i % n]["b"], y=sets[i % n]["y"], stream=stream)
        ms = _time_device(fn, args.steps, args.warmup, stream)
        flops = 2.0 * B * T * C * n_out
        tf = flops / (ms * 1e-3) / 1e12
        print(json.dumps({
            "metric": f"{name} TFLOPS", "value": tf, "unit": "TFLOPS", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "M": B * T, "N": n_out, "K": C,
                       "l2": f"{n} rotating input/output sets"},
            "roofline": {"kernel": "linear", "bound": "tensor", "achieved": tf, "peak": peak,
                         "unit": "TFLOP/s", "frac": tf / peak,
                         "peak_source": f"bf16_tflops (burst) of {peak_src}"},
            "gpu_launches": args.steps}), flush=True)
    st, word = ops.last_device_status()
    if st != ops.GA_OK:
        raise RuntimeError(f"device status: {ops.status_string(st)} ({word:#x})")
    return 0


def run_context(args, wl):
    """torch's scaled_dot_product_attention (fwd + bwd through autograd) on the
    same inputs, as a context figure: one JSON line."""
    import torch

    from causal_self_attention_flashattention_b200.workload import attention_flops, make_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, T, H, D, scale = wl.B, wl.T, wl.H, wl.D, wl.scale
    qkv_cpu, dout_cpu = make_inputs(B, T, H, D, seed=0, qk_std=wl.qk_std)
    sets = [(qkv_cpu.to(dev).requires_grad_(True), dout_cpu.to(dev)) for _ in range(args.sets)]
    fwd_flops, bwd_flops = attention_flops(B, T, H, D)

    def sdpa(qkv):
        q, k, v = (qkv[:, :, i].transpose(1, 2) for i in range(3))
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
        return o.transpose(1, 2)

    line = {"impl": "context", "library": "torch SDPA", "metric": METRIC, "unit": "TFLOPS",
            "config": {"workload": wl.name, "B": B, "T": T, "H": H, "D": D}}
    try:
        def step(i):
            qkv, dout = sets[i % len(sets)]
            torch.autograd.grad(sdpa(qkv), qkv, dout)
        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(args.steps):
            step(i)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / args.steps
        line.update(value=(fwd_flops + bwd_flops) / (ms * 1e-3) / 1e12, ms_per_step=ms,
                    steps=args.steps)
    except Exception as e:  # no kernel for this GPU in the installed torch
        line["unavailable"] = f"{type(e).__name__}: {str(e).splitlines()[0][:160]}"
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--e2e-steps", type=int, default=30)
    p.add_argument("--sets", type=int, default=N_SETS,
                   help="input/output buffer sets rotated through (default 4)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=15.0)
    p.add_argument("--decode", action="store_true",
                   help="time decode attention (gpt2_attn_decode) instead")
    p.add_argument("--fp8", action="store_true",
                   help="time the FP8 forward (and its quantisation pass) instead")
    p.add_argument("--linear", action="store_true",
                   help="time the dense layers around attention (c_attn, c_proj) instead")
    p.add_argument("--v16", action="store_true",
                   help="time the forward that reads v in fp16 from c_attn instead")
    p.add_argument("--context", action="store_true",
                   help="time torch SDPA on the same workload, for context")
    args = p.parse_args(argv)
    if args.warmup < 3:
        p.error("--warmup must be at least 3")
    from causal_self_attention_flashattention_b200.workload import WORKLOADS

    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.decode:
        return run_decode(args, wl)
    if args.context:
        return run_context(args, wl)
    if args.fp8:
        return run_fp8(args, wl)
    if args.linear:
        return run_linear(args, wl)
    if args.v16:
        return run_v16(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
