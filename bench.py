#!/usr/bin/env python3
"""Benchmark of the CKDA forward on B200.

One step = one ckda_chunk_fwd over the 1.3B-model-shaped layer workload
(B=8, T=4096, H=16, d_k=d_v=128, bf16 q/k/v, fp32 alpha/beta/state, S0 = 0, output
o and S_T), inputs resident in HBM. Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs under torchrun, one process per GPU; every rank processes its own full
layer batch (the path shards over independent (batch, head) sequences with no
exchange), timing is the max over ranks and `value` counts all ranks' tokens.
`--impl reference` times the fp64 CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
from delta_rule_attention_ckda_b200.replicas import aggregate_throughput  # noqa: E402

METRIC = "CKDA fwd tokens/s at H=16,d=128,T=4096; % of tensor-core/HBM roofline"
WORKLOAD = dict(B=8, T=4096, H=16, dk=128, dv=128)
BYTES_PER_TOKEN_HEAD = 2 * 128 * 2 + 128 * 2 + 128 * 4 + 4 + 128 * 4   # q,k,v bf16; alpha, beta, o fp32
FLOPS_PER_TOKEN_HEAD = 64 * (3 * 128 + 2 * 128) + 6 * 128 * 128         # minimal count, chunk 64
FLOPS_DENSE_TILE_PER_TOKEN_HEAD = 2 * 64 * (3 * 128 + 2 * 128) + 6 * 128 * 128   # 64 x 64 tiles in full
# Multiply-adds the chunk kernel issues per 64-token chunk (tcgen05, M = 128, K = 16 each):
#   [P;A]  8 x N=128 + 8 x N=64;  C1  24 x N=128;  U  12 x N=128 + 8 x N=64;
#   O / state  12 x N=192 + 4 x N=128
ISSUED_MMA_MACS_PER_CHUNK = 128 * 16 * (8 * 128 + 8 * 64 + 24 * 128 + 12 * 128 + 8 * 64 + 12 * 192 + 4 * 128)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-extras", action="store_true")
    p.add_argument("--cp", action="store_true",
                   help="with N > 1: also time the long workload split over the ranks by tokens "
                        "(context parallelism, one all-gather per step)")
    p.add_argument("--batch", type=int, default=WORKLOAD["B"],
                   help="batch size of the layer workload (smaller values for profiling captures)")
    p.add_argument("--only", default="all", choices=["all", "chunk", "decode", "bwd"],
                   help="run only the forward legs, the decode leg or the backward leg (profiling captures)")
    return p.parse_args()


# ----------------------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 TFLOP/s: the burst figure of MEASURED_PEAKS.json (the layer step is a short
    kernel timed on its own), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


# device sources that make up each profiled kernel (its code and the primitives it uses)
KERNEL_SOURCES = {
    "chunk_fwd_chunk_tc_layer": ["kernels/common.cuh", "kernels/chunk_tc.cuh", "kernels/tc_primitives.cuh",
                                 "kernels/tc_host.cuh"],
    "decode128": ["kernels/common.cuh", "kernels/decode.cuh"],
}


def _code_only(text):
    """Source text without comments and blank space, so that a comment edit keeps the hash."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(" ".join(line.split()) for line in text.splitlines() if line.strip())


def kernel_source_hash(kernel_key):
    """Hash of the code (comments stripped) of one kernel's sources; its committed
    DRAM-traffic figure is only reported while it matches."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "delta_rule_attention_ckda_b200", "csrc")
    for rel in KERNEL_SOURCES[kernel_key]:
        p = os.path.join(csrc, rel)
        if os.path.exists(p):
            with open(p, encoding="utf-8") as f:
                h.update(rel.encode())
                h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def committed_profile(kernel_key):
    """The committed ncu figures of a kernel (profiles/dram_traffic.json), or None once the
    kernel's code no longer hashes to the value recorded with them."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        ent = d.get(kernel_key)
        if ent and ent.get("source_hash") == kernel_source_hash(kernel_key):
            return ent
    except Exception:
        pass
    return None


def committed_traffic(kernel_key):
    ent = committed_profile(kernel_key)
    return None if ent is None else float(ent["bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        import torch
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.gpu = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.gpu = str(device_index)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", self.gpu], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample(inp, n_seq, threads=None):
    """Run the fp64 oracle on the first n_seq (b, h) sequences of the workload."""
    import oracle
    B, T, H, dk, dv = inp.shape
    pairs = [(i // H, i % H) for i in range(n_seq)]
    q = torch_stack(inp.q, pairs)
    k = torch_stack(inp.k, pairs)
    v = torch_stack(inp.v, pairs)
    a = torch_stack(inp.alpha, pairs)
    import torch
    b = torch.stack([inp.beta[bb, :, h] for bb, h in pairs])[:, :, None]
    if threads:
        oracle.set_threads(threads)
    t0 = time.perf_counter()
    oracle.oracle_fwd(q, k, v, a, b, None)
    return time.perf_counter() - t0


def torch_stack(x, pairs):
    import torch
    return torch.stack([x[b, :, h] for b, h in pairs])[:, :, None]


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(inp, target_s=12.0):
    import oracle
    oracle.build()
    cores = cpu_cores()
    oracle.set_threads(cores)
    B, T, H, dk, dv = inp.shape
    t1 = oracle_sample(inp, min(cores, B * H))       # calibration: one sequence per core
    per_round = max(t1, 1e-3)
    rounds = max(1, min(int(target_s / per_round), (B * H) // min(cores, B * H)))
    n_seq = min(B * H, rounds * min(cores, B * H))
    dt = oracle_sample(inp, n_seq)
    tokens = n_seq * T / H            # token-heads / H = tokens with all heads
    # one thread, two sequences, scaled by count to the whole layer workload
    oracle.set_threads(1)
    n1 = 2
    d1 = oracle_sample(inp, n1)
    oracle.set_threads(cores)
    return {"value": tokens / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{n_seq} of {B * H} (batch, head) sequences x T={T} of the layer workload, "
                      f"fp64 sequential loop, OpenMP over sequences, {dt:.2f} s wall",
            "seconds": dt,
            "one_thread": {"sequences": n1, "seconds": d1, "layer_seconds_est": d1 / n1 * B * H,
                           "value": n1 * T / H / d1, "unit": "tokens/s",
                           "how": f"{n1} sequences x T={T} on one thread, scaled by count to the "
                                  f"{B * H} sequences of the layer workload"}}


# ----------------------------------------------------------------------------- arms

def reference_arm(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    from ckda_inputs import make_workload
    import oracle
    oracle.build()
    inp = make_workload("layer")
    B, T, H, dk, dv = inp.shape
    cores = cpu_cores()
    oracle.set_threads(cores)
    n_seq = min(B * H, cores)
    for _ in range(args.warmup):
        oracle_sample(inp, n_seq)
    times = [oracle_sample(inp, n_seq) for _ in range(args.steps)]
    tot = sum(times)
    tokens = n_seq * T / H * args.steps
    value = tokens / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "layer B=8 T=4096 H=16 dk=dv=128", **WORKLOAD,
                       "sample_per_step": f"{n_seq} (batch, head) sequences x T={T}"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: {n_seq} of {B * H} sequences x T={T}, fp64 oracle"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def fwd_launches(ck, B, T, H, dk, dv, dtype=None):
    """Kernel launches of one chunk_fwd call: the tensor-core direct launch is two (the
    instance without the exact path, then the general one over the sequences it left), the
    segmented one three (segment maps, the fold, the segments from their entering states),
    the recurrent path one."""
    import torch
    dtype = dtype or torch.bfloat16
    if ck.chunk_path(B, T, H, dk, dv, dtype) != ck.PATH_CHUNK_TC:
        return 1
    return 2 if ck.chunk_segments(B, T, H, dk, dv, dtype) == 1 else 3


def time_launches(fn, steps, stream):
    import torch
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        fn()
    ev1.record(stream)
    ev1.synchronize()
    return ev0.elapsed_time(ev1) / 1e3


def ours_arm(args):
    import torch
    world, rank, local = dist_setup(args.gpus)
    import delta_rule_attention_ckda_b200 as ck
    from ckda_inputs import make_workload
    ck.load()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()

    if args.only == "decode":
        line = {"decode": decode_measure(ck, dev, stream, world)}
        if rank == 0:
            print(json.dumps(line), flush=True)
        return 0
    inp = make_workload("layer", B=args.batch)
    B, T, H, dk, dv = inp.shape
    if args.only == "bwd":
        q, k, v, a, b = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.alpha, inp.beta))
        line = {"bwd": bwd_measure(ck, q, k, v, a, b, stream, world, reps=max(1, args.steps))}
        if rank == 0:
            print(json.dumps(line), flush=True)
        return 0
    q, k, v, a, b = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.alpha, inp.beta))
    o = torch.empty(B, T, H, dv, device=dev)
    ST = torch.empty(B, H, dk, dv, device=dev)
    wsb = ck.workspace_bytes(B, T, H, dk, dv)
    ws = torch.empty(max(wsb, 16), device=dev, dtype=torch.uint8)
    path = "chunk_tc" if ck.chunk_path(B, T, H, dk, dv) == ck.PATH_CHUNK_TC else "recurrent"

    def step():
        ck.chunk_fwd(q, k, v, a, b, None, o=o, S_T=ST, workspace=ws if wsb else None)

    for _ in range(args.warmup):
        step()
    assert ck.get_device_error() == 0
    sampler = ClockSampler(dev.index)
    barrier(world)
    sampler.start()
    time.sleep(0.15)
    barrier(world)
    secs = time_launches(step, args.steps, stream)
    barrier(world)
    clocks = sampler.stop()
    if ck.get_device_error() != 0:
        raise RuntimeError("device error word set during the timed region")
    # replicas: every rank ran its own batch; whole-job tokens over the slowest rank's time
    value, secs = aggregate_throughput(B * T * args.steps, secs, world, device="cuda")
    per_launch = secs / args.steps
    alg_bytes = B * T * H * BYTES_PER_TOKEN_HEAD + B * H * dk * dv * 4
    hbm, src = peaks()
    achieved = alg_bytes / per_launch / 1e9
    kernel_key = f"chunk_fwd_{path}_layer"
    prof = committed_profile(kernel_key)
    tpeak, tsrc = tensor_peak()
    nchunks = B * H * ((T + 63) // 64)
    issued = 2.0 * ISSUED_MMA_MACS_PER_CHUNK * nchunks / per_launch / 1e12
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": None if prof is None else float(prof["bytes_per_launch"]),
            "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else "fallback 6.65 TB/s",
            "kernel": kernel_key, "alg_bytes_per_launch": alg_bytes,
            "tflops_minimal": B * T * H * FLOPS_PER_TOKEN_HEAD / per_launch / 1e12,
            "tflops_dense_tile": B * T * H * FLOPS_DENSE_TILE_PER_TOKEN_HEAD / per_launch / 1e12,
            "tflops_issued_mma": issued,
            "issued_mma_frac_of_bf16_peak": issued / tpeak,
            "bf16_peak_tflops": tpeak, "bf16_peak_source": f"{tsrc} (MEASURED_PEAKS.json bf16_tflops, burst)",
            "tensor_pipe_pct": None if prof is None else prof.get("tensor_pipe_pct"),
            "tensor_pipe_pct_source": "committed ncu capture (max over SMs / mean over 148 SMs), "
                                      "null once the kernel's code changed since"}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * per_launch,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"layer B={B} T={T} H={H} dk=dv={dk} chunk=64", **WORKLOAD, "B": B,
                       "global_batch": B * world, "seq_len": T, "parallelism": f"replicas x{world}",
                       "path": path, "l2": "inputs larger than L2 (~950 MB per step vs 126 MB), no flush",
                       "state": "S0 = 0 (not read), S_T written"},
            "roofline": roof, "gpu_launches": args.steps * fwd_launches(ck, B, T, H, dk, dv), "clocks": clocks}

    if not args.no_extras:
        line["kda"] = kda_measure(ck, q, k, v, a, b, o, ST, stream, world, args.steps, value)
        line["configs"] = configs_measure(ck, dev, stream, world)
        line["bwd"] = bwd_measure(ck, q, k, v, a, b, stream, world)
        line["normalize_qk"] = norm_measure(ck, q, k, v, a, b, o, ST, stream, world, args.steps, value)
    if not args.no_e2e:
        line["e2e"] = e2e_measure(ck, inp, dev, stream, world, args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp)
    if not args.no_extras and args.only == "all":
        line["decode"] = decode_measure(ck, dev, stream, world)
    if args.cp and world > 1:
        line["cp"] = cp_measure(ck, dev, stream, world, rank)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def configs_measure(ck, dev, stream, world):
    """The workloads' other configurations: small (L2-resident and launch-bound: latency
    only) and long (one head batch of 65536 tokens with an initial state: 16 sequences,
    so 16 SMs work; tokens/s and the fraction of the HBM roofline)."""
    import torch
    from ckda_inputs import make_workload
    out = {}
    for name, reps in (("small", 20), ("long", 3)):
        inp = make_workload(name)
        B, T, H, dk, dv = inp.shape
        q, k, v, a, b = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.alpha, inp.beta))
        S0 = inp.S0.to(dev)
        o = torch.empty(B, T, H, dv, device=dev)
        ST = torch.empty(B, H, dk, dv, device=dev)

        def step():
            ck.chunk_fwd(q, k, v, a, b, S0, o=o, S_T=ST)

        step()
        torch.cuda.synchronize()
        assert ck.get_device_error() == 0
        secs = time_launches(step, reps, stream)
        value, secs = aggregate_throughput(B * T * reps, secs, world, device="cuda")
        per = secs / reps
        path = "chunk_tc" if ck.chunk_path(B, T, H, dk, dv, inp.q.dtype) == ck.PATH_CHUNK_TC else "recurrent"
        ent = {"shape": f"B={B} T={T} H={H} dk={dk} dv={dv} {str(inp.q.dtype).replace('torch.', '')}",
               "path": path, "us_per_launch": per * 1e6}
        if name == "long":
            bytes_tok = 2 * dk * 2 + dv * 2 + dk * 4 + 4 + dv * 4
            alg = B * T * H * bytes_tok + 2 * B * H * dk * dv * 4
            hbm, src = peaks()
            ent.update({"tokens_per_s": value, "roofline": {"bound": "hbm", "achieved": alg / per / 1e9,
                        "peak": hbm, "unit": "GB/s", "frac": alg / per / 1e9 / hbm,
                        "alg_bytes_per_launch": alg}})
        out[name] = ent
    return out


def cp_measure(ck, dev, stream, world, rank, reps=3):
    """Context parallelism (N > 1 only): the long workload (one batch of 16 heads x 65536
    tokens with an initial state) split over the ranks in token order, each rank its
    slice; one all-gather of the slices' affine maps per step (NCCL). Strong scaling: the
    whole job is the one sequence batch; tokens/s over the slowest rank's time."""
    import torch
    from ckda_inputs import make_workload
    from delta_rule_attention_ckda_b200 import context_parallel as cp
    inp = make_workload("long")
    B, T, H, dk, dv = inp.shape
    lo, hi = (T * rank) // world, (T * (rank + 1)) // world
    q, k, v, a, b = (x[:, lo:hi].contiguous().to(dev) for x in (inp.q, inp.k, inp.v, inp.alpha, inp.beta))
    S0 = inp.S0.to(dev) if rank == 0 else None

    def step():
        return cp.cp_chunk_fwd(q, k, v, a, b, S0)

    step()
    barrier(world)
    assert ck.get_device_error() == 0
    barrier(world)
    secs = time_launches(step, reps, stream)
    barrier(world)
    value, secs = aggregate_throughput((hi - lo) * B * reps, secs, world, device="cuda")
    return {"workload": f"long B={B} T={T} H={H} dk={dk} dv={dv} bf16, tokens split over {world} ranks",
            "scaling": "strong", "tokens_per_s": value, "ms_per_step": 1e3 * secs / reps,
            "exchange_bytes_per_rank": 4 * B * H * dk * (dk + dv), "collective": "all_gather (NCCL)"}


def bwd_measure(ck, q, k, v, a, b, stream, world, reps=3):
    """The backward pass (ckda_bwd) of the same layer step: gradients of <dO, o> for q,
    k, v, alpha, beta and S0, from a fixed synthetic cotangent dO. Tokens/s and the
    algorithmic HBM bytes (inputs and cotangent read once, gradients written once). Then
    forward + backward for the signed gate and for KDA's form of it (g = ln|alpha| through
    the log-gate mode), the pair the pages compare."""
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    g = torch.Generator(device="cpu").manual_seed(11)
    dO = torch.randn(B, T, H, dv, generator=g).to(q.device)
    grads = {n: torch.empty(s, device=q.device) for n, s in (
        ("dq", (B, T, H, dk)), ("dk", (B, T, H, dk)), ("dv", (B, T, H, dv)), ("dalpha", (B, T, H, dk)),
        ("dbeta", (B, T, H)), ("dS0", (B, H, dk, dv)))}
    ws = torch.empty(ck.bwd_workspace_bytes(B, T, H, dk, dv), device=q.device, dtype=torch.uint8)
    tc = ck.bwd_path(B, T, H, dk, dv, q.dtype) == ck.BWD_CHUNK_TC

    def step():
        ck.bwd(q, k, v, a, b, dO, None, None, grads=grads, workspace=ws)

    step()
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    barrier(world)
    secs = time_launches(step, reps, stream)
    assert ck.get_device_error() == 0
    value, secs = aggregate_throughput(B * T * reps, secs, world, device="cuda")
    per = secs / reps
    in_bytes = 2 * dk * 2 + dv * 2 + dk * 4 + 4 + dv * 4          # q, k, v (bf16), alpha, beta, dO
    out_bytes = 3 * dk * 4 + dv * 4 + 4                             # dq, dk, dalpha, dv, dbeta
    alg = B * T * H * (in_bytes + out_bytes) + B * H * dk * dv * 4   # + dS0
    hbm, _ = peaks()
    kernels = ("chunk_tc_kernel (forward with chunk checkpoints, then its redo pass) + chunk_bwd_chain_kernel + "
               "chunk_bwd_grad_kernel + chunk_bwd_grad_exact_kernel (tcgen05)" if tc
               else "bwd_ckpt_kernel + bwd_grad_kernel + bwd_sum_kernel (fp32 CUDA cores)")
    out = {"workload": f"layer B={B} T={T} H={H} dk={dk} dv={dv}, backward of <dO, o> (S0 = 0)",
           "path": "chunk_tc" if tc else "recurrent",
           "value": value, "unit": "tokens/s", "ms_per_step": 1e3 * per, "gpu_launches": (5 if tc else 3) * reps,
           "roofline": {"bound": "hbm", "achieved": alg / per / 1e9, "peak": hbm, "unit": "GB/s",
                        "frac": alg / per / 1e9 / hbm, "alg_bytes_per_launch": alg, "kernels": kernels}}

    # forward + backward, signed gate against KDA's non-negative log gate
    o = torch.empty(B, T, H, dv, device=q.device)
    ST = torch.empty(B, H, dk, dv, device=q.device)
    glog = torch.log(a.abs())
    steps = {}
    for name, gate, gin in (("ckda", "signed", a), ("kda", "log", glog)):
        def fwd_bwd(gate=gate, gin=gin):
            ck.chunk_fwd(q, k, v, gin, b, None, o=o, S_T=ST, gate=gate)
            ck.bwd(q, k, v, gin, b, dO, None, None, grads=grads, workspace=ws, gate=gate)

        fwd_bwd()
        torch.cuda.synchronize()
        assert ck.get_device_error() == 0
        steps[name] = fwd_bwd
    # trials alternating the two gates; each arm's median (one trial is a few ms, so a single one
    # is at the mercy of a transient)
    trials = 5
    fb = {name: [] for name in steps}
    barrier(world)
    for _ in range(trials):
        for name, fn in steps.items():
            s = time_launches(fn, reps, stream)
            assert ck.get_device_error() == 0
            _, s = aggregate_throughput(B * T * reps, s, world, device="cuda")
            fb[name].append(1e3 * s / reps)
    med = {name: sorted(t)[len(t) // 2] for name, t in fb.items()}
    out["fwd_bwd"] = {"workload": "layer: forward (o, S_T) then backward, per step",
                      "ckda_ms": med["ckda"], "kda_ms": med["kda"],
                      "timing": f"median of {trials} trials of {reps} steps per gate, the gates alternating",
                      "kda_gate": "g = ln|alpha| (non-negative gate) through the log-gate mode",
                      "ckda_over_kda_throughput": med["kda"] / med["ckda"],
                      "gpu_launches": (fwd_launches(ck, B, T, H, dk, dv) + (5 if tc else 3)) * reps * trials}
    del ws
    return out


def norm_measure(ck, q, k, v, a, b, o, ST, stream, world, steps, plain_value):
    """The layer step with q and k L2-normalised inside the kernel (CKDA_OPT_NORMALIZE_QK),
    next to the same step fed by a separate normalisation pass (torch, bf16 in and out)."""
    import torch
    B, T, H, dk = q.shape

    def fused():
        ck.chunk_fwd(q, k, v, a, b, None, o=o, S_T=ST, normalize_qk=True)

    def separate():
        qn = torch.nn.functional.normalize(q.float(), dim=-1).to(q.dtype)
        kn = torch.nn.functional.normalize(k.float(), dim=-1).to(k.dtype)
        ck.chunk_fwd(qn, kn, v, a, b, None, o=o, S_T=ST)

    out = {"workload": "layer, q and k L2-normalised per token and head"}
    for name, fn in (("fused", fused), ("separate_torch_pass", separate)):
        for _ in range(3):
            fn()
        assert ck.get_device_error() == 0
        barrier(world)
        secs = time_launches(fn, steps, stream)
        value, secs = aggregate_throughput(B * T * steps, secs, world, device="cuda")
        out[name] = {"value": value, "unit": "tokens/s", "ms_per_step": 1e3 * secs / steps}
    out["fused_over_plain"] = out["fused"]["value"] / plain_value
    out["gpu_launches"] = steps * fwd_launches(ck, B, T, H, dk, v.shape[-1])
    return out


def kda_measure(ck, q, k, v, a, b, o, ST, stream, world, steps, ckda_value):
    """The same layer step with the gate in KDA's form: g = ln |alpha| (the same
    magnitudes, never negative), through the log-gate mode of the same kernels. Reports
    CKDA's throughput over KDA's, the comparison the pages make for the signed gate."""
    import torch
    B, T, H, dk = q.shape
    g = torch.log(a.abs())

    def step():
        ck.chunk_fwd(q, k, v, g, b, None, o=o, S_T=ST, gate="log")

    for _ in range(3):
        step()
    assert ck.get_device_error() == 0
    barrier(world)
    secs = time_launches(step, steps, stream)
    assert ck.get_device_error() == 0
    value, secs = aggregate_throughput(B * T * steps, secs, world, device="cuda")
    return {"workload": "layer, gate given as g = ln|alpha| (non-negative gate, KDA form)",
            "value": value, "unit": "tokens/s", "ms_per_step": 1e3 * secs / steps,
            "ckda_over_kda": ckda_value / value, "gpu_launches": steps * fwd_launches(ck, B, T, H, dk, dk)}


def e2e_measure(ck, inp, dev, stream, world, args):
    """Same metric through the public Python API with pinned host buffers; every step
    copies its inputs host->device and reads o and S_T back. Steps are pipelined over
    three streams (inputs in, compute, results out) and two device buffer sets, so the
    copies of neighbouring steps overlap the compute and each other, as a serving loop
    would run them."""
    import torch
    B, T, H, dk, dv = inp.shape
    hq, hk, hv, ha, hb = (x.pin_memory() for x in (inp.q, inp.k, inp.v, inp.alpha, inp.beta))
    ho = torch.empty(B, T, H, dv, pin_memory=True)
    hS = torch.empty(B, H, dk, dv, pin_memory=True)
    sets = []
    for _ in range(2):
        sets.append({"in": [torch.empty_like(x, device=dev) for x in (hq, hk, hv, ha, hb)],
                     "o": torch.empty(B, T, H, dv, device=dev), "S": torch.empty(B, H, dk, dv, device=dev)})
    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of set i copied
    ev_cmp = [torch.cuda.Event() for _ in range(2)]     # set i computed
    ev_out = [torch.cuda.Event() for _ in range(2)]     # results of set i read back
    for e in ev_out:
        e.record(stream)

    def step(i):
        st = sets[i % 2]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[i % 2])              # the set's previous compute is done
            for d, h in zip(st["in"], (hq, hk, hv, ha, hb)):
                d.copy_(h, non_blocking=True)
            ev_in[i % 2].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[i % 2])
            s_cmp.wait_event(ev_out[i % 2])             # its previous results have left
            q, k, v, a, b = st["in"]
            ck.chunk_fwd(q, k, v, a, b, None, o=st["o"], S_T=st["S"], stream=s_cmp)
            ev_cmp[i % 2].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[i % 2])
            ho.copy_(st["o"], non_blocking=True)
            hS.copy_(st["S"], non_blocking=True)
            ev_out[i % 2].record(s_out)

    for e in ev_cmp:
        e.record(stream)
    step(0)
    step(1)
    torch.cuda.synchronize()
    n = max(4, min(args.steps, 8))
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for x in (s_in, s_cmp, s_out):
        x.wait_event(t0)
    for i in range(n):
        step(i)
    for x in (s_in, s_cmp, s_out):
        stream.wait_stream(x)
    t1.record(stream)
    t1.synchronize()
    assert ck.get_device_error() == 0
    secs = t0.elapsed_time(t1) / 1e3
    value, secs = aggregate_throughput(B * T * n, secs, world, device="cuda")
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, ha, hb))
    d2h = ho.numel() * 4 + hS.numel() * 4
    return {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n,
            "pipeline": "3 streams (in, compute, out), 2 device buffer sets; pinned host buffers"}


def decode_measure(ck, dev, stream, world):
    """The decode workload: 256 sequences x 16 heads, d = 128, fp32 state updated in
    place, 1024 calls (call t reads input set t % 64)."""
    import torch
    from ckda_inputs import DECODE, make_decode_pool
    pool = make_decode_pool()
    P, N, H, D = DECODE["pool"], DECODE["N"], DECODE["H"], DECODE["dk"]
    dq, dk_, dv_, da, db = (x.to(dev) for x in (pool.q, pool.k, pool.v, pool.alpha, pool.beta))
    S = pool.S0.to(dev)
    o = torch.empty(N, H, D, device=dev)
    calls = DECODE["steps"]
    for t in range(8):
        ck.decode_step(dq[t % P], dk_[t % P], dv_[t % P], da[t % P], db[t % P], S, o=o)
    barrier(world)
    it = iter(range(calls))

    def one():
        t = next(it)
        ck.decode_step(dq[t % P], dk_[t % P], dv_[t % P], da[t % P], db[t % P], S, o=o)

    secs = time_launches(one, calls, stream)
    assert ck.get_device_error() == 0
    tok_s, secs = aggregate_throughput(N * calls, secs, world, device="cuda")
    per = secs / calls
    bytes_call = N * H * (2 * D * D * 4 + 3 * D * 2 + D * 4 + 4 + D * 4)
    hbm, src = peaks()
    gbs = bytes_call / per / 1e9
    traffic = committed_traffic("decode128")
    roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
            "alg_bytes_per_launch": bytes_call, "kernel": "decode128", "traffic": traffic}
    if traffic is not None:
        # part of the 268 MB state stays in the 126 MB L2 between back-to-back calls, so the
        # DRAM bytes of a call are below its algorithmic bytes: the fraction on DRAM bytes
        roof["dram_gbs"] = traffic / per / 1e9
        roof["dram_frac"] = traffic / per / 1e9 / hbm
    return {"workload": "decode N=256 H=16 d=128 fp32 state, 1024 calls", "us_per_call": per * 1e6,
            "tokens_per_s": tok_s, "roofline": roof, "gpu_launches": calls}


def main():
    args = parse()
    if args.impl == "reference":
        return reference_arm(args)
    return ours_arm(args)


if __name__ == "__main__":
    sys.exit(main())
