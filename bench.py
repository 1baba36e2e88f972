#!/usr/bin/env python
"""Throughput of the fused low-rank MoE router (MoRE) on B200.

One step = one routing call over the workload's N tokens: z = x.R1, the M logits
z.R2, top-k with softmax gates, per-expert counts ("MoRE: Scaling mixture of
experts with hardware-aware low-rank routing", App. F, Algorithm 1).  Default
workload: prefill, N = 262,144 tokens (256 sequences x 1024), h = 2048, M = 4096,
r = 32, k = 8, X rows at unit RMS, R1 ~ N(0, 1/h), R2 ~ N(0, 1/r), seed 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--variant auto|fused_tc|small_n|cluster|unfused|unfused_tc|train|dispatch|
                             dispatch_shared|backward]
                  [--workload NAME]

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank routes its own
N-token shard of a larger synthetic token set (weak scaling, no collective on the
data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # name: (N, h, r, M, k, x_unit_rms)
    "prefill_r32": (262144, 2048, 32, 4096, 8, True),
    "prefill_r16": (262144, 2048, 16, 4096, 8, True),
    "prefill_r64": (262144, 2048, 64, 4096, 8, True),
    "prefill_r128": (262144, 2048, 128, 4096, 8, True),
    "many_experts": (32768, 4096, 64, 65536, 8, False),
    "sweep_M1024": (65536, 512, 32, 1024, 8, False),
    "sweep_M2048": (65536, 512, 32, 2048, 8, False),
    "sweep_M4096": (65536, 512, 32, 4096, 8, False),
    "sweep_M8192": (65536, 512, 32, 8192, 8, False),
    "sweep_M16384": (65536, 512, 32, 16384, 8, False),
    "tiny": (4096, 128, 32, 192, 4, False),
    "decode_N1": (1, 2048, 32, 4096, 8, False),
    "decode_N8": (8, 2048, 32, 4096, 8, False),
    "decode_N64": (64, 2048, 32, 4096, 8, False),
    "decode_N256": (256, 2048, 32, 4096, 8, False),
    # fused vs unfused against the batch (App. H.6, Fig. 24): N = B x 1024, h = 2048, M = 4096, r = 16, k = 4
    "fig24_B2": (2048, 2048, 16, 4096, 4, True),
    "fig24_B16": (16384, 2048, 16, 4096, 4, True),
    "fig24_B64": (65536, 2048, 16, 4096, 4, True),
    "fig24_B256": (262144, 2048, 16, 4096, 4, True),
    # the standard full-rank router (App. H.3, Figs. 20-21 prefill: N = 262,144, M = 4096, k = 4);
    # r is that of the MoRE layer the figures compare with and only the low-rank variants use it
    "fullrank_h1024": (262144, 1024, 64, 4096, 4, True),
    "fullrank_h2048": (262144, 2048, 64, 4096, 4, True),
}
METRIC = "routed tokens/s (fused low-rank router + top-k)"
FULLRANK_METRIC = "routed tokens/s (fused full-rank router + top-k, App. H.3)"
BACKWARD_METRIC = "router backward tokens/s (App. F Algorithm 3: gradients of X, R1, R2)"
# DRAM bytes (read + write) per token of the fused kernel, from one ncu capture at N = 65,536
# (summarised under profiles/, scaled by tokens), keyed to the SHA-256 of the kernel source that
# was captured: once route_tc.cu differs from that source the figure is stale and traffic is
# reported null.  Workloads without a capture report traffic null.
NCU_TRAFFIC = {    # workload -> (bytes per token, sha256 of route_tc.cu at capture time)
    "prefill_r32": ((269128960 + 4530432) / 65536,
                    "6c8948233b0fcb6b5ca0c1295b3c677ff694bfefe8d374bfafbc5ae569f85503"),
}
L2_BYTES = 126 * 1024 * 1024


def kernel_source_digest():
    """SHA-256 of the fused kernel's source, or None where the source is not shipped."""
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "mixture_experts_rank_b200", "csrc",
                        "route_tc.cu")
    try:
        with open(path, "rb") as f:
            return hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None


def describe(name):
    N, h, r, M, k, unit = WORKLOADS[name]
    return (f"{name}: N={N} h={h} M={M} r={r} k={k}, X bf16 N(0,1)"
            f"{' rows at unit RMS' if unit else ''}, R1 N(0,1/h), R2 N(0,1/r), seed 0")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0)) or None, \
            "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, flag in zip(names, parts[5:9]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args, world, rank):
    """The fp64 oracle on the host cores, on a bounded sample of the workload per step."""
    if rank != 0:
        return 0
    import oracle
    import synthetic as syn
    N, h, r, M, k, unit = WORKLOADS[args.workload]
    cores = os.cpu_count() or 1
    R1 = syn.normal_bf16(0, syn.TENSOR_R1, h, r, 1.0 / np.sqrt(h))
    R2 = syn.normal_bf16(0, syn.TENSOR_R2, r, M, 1.0 / np.sqrt(r))
    backward = args.variant == "backward"
    fullrank = args.variant == "fullrank"
    W = syn.normal_bf16(0, syn.TENSOR_R2, h, M, 1.0 / np.sqrt(h)) if fullrank else None
    rng = np.random.default_rng(1)

    def one_step(X, S):
        if backward:  # the oracle's Algorithm 3 on the sample, seeded selections and gradients
            oracle.router_backward(X, R1, R2, S, h, r, M, rng.integers(0, M, (S, k)),
                                   rng.standard_normal((S, k)), rng.standard_normal(M))
        elif fullrank:
            oracle.route_fullrank(X, W, S, h, M, k, threads=cores)
        else:
            oracle.route(X, R1, R2, S, h, r, M, k, threads=cores)

    # size the per-step sample from a short probe: about args.ref_step_seconds of CPU work
    probe = max(cores, 16)
    Xp = syn.normal_bf16(0, syn.TENSOR_X, N, h, 1.0, unit, 0, probe)
    t = time.perf_counter()
    one_step(Xp, probe)
    per_tok = (time.perf_counter() - t) / probe
    S = int(max(cores, min(N, args.ref_step_seconds / max(per_tok, 1e-9), 32768 if backward else N)))
    X = syn.normal_bf16(0, syn.TENSOR_X, N, h, 1.0, unit, 0, S)
    for _ in range(args.warmup):
        one_step(X, S)
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        one_step(X, S)
        times.append(time.perf_counter() - t)
    if backward:
        cores = blas_threads()
    step = sum(times) / len(times)
    value = S / step
    sample = f"first {S} tokens of the workload per step ({S / N:.4%} of N), all M experts"
    metric = BACKWARD_METRIC if backward else (FULLRANK_METRIC if fullrank else METRIC)
    line = {"impl": "reference", "metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": describe(args.workload), "N": N, "h": h, "r": r,
                                            "M": M, "k": k, "tokens_per_step": S},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(workload, seconds, fullrank=False):
    import oracle
    import synthetic as syn
    N, h, r, M, k, unit = WORKLOADS[workload]
    cores = os.cpu_count() or 1
    if fullrank:
        W = syn.normal_bf16(0, syn.TENSOR_R2, h, M, 1.0 / np.sqrt(h))
        route = lambda X, S: oracle.route_fullrank(X, W, S, h, M, k, threads=cores)
    else:
        R1 = syn.normal_bf16(0, syn.TENSOR_R1, h, r, 1.0 / np.sqrt(h))
        R2 = syn.normal_bf16(0, syn.TENSOR_R2, r, M, 1.0 / np.sqrt(r))
        route = lambda X, S: oracle.route(X, R1, R2, S, h, r, M, k, threads=cores)
    probe = max(cores, 16)
    Xp = syn.normal_bf16(0, syn.TENSOR_X, N, h, 1.0, unit, 0, probe)
    t = time.perf_counter()
    route(Xp, probe)
    per_tok = (time.perf_counter() - t) / probe
    S = int(max(probe, min(N, seconds / max(per_tok, 1e-9))))
    X = syn.normal_bf16(0, syn.TENSOR_X, N, h, 1.0, unit, 0, S)
    t = time.perf_counter()
    route(X, S)
    el = time.perf_counter() - t
    return {"value": S / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {S} of the {N} tokens, all M experts, {el:.1f} s on {cores} threads"}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        counts = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(counts) if counts else 1
    except Exception:  # pragma: no cover
        return 1


def backward_cpu_baseline(workload, seconds):
    """The oracle's backward (numpy fp64) on a bounded sample of tokens: a sample's X, R1 and
    R2 gradients; the selections and gradients are seeded draws."""
    import oracle
    import synthetic as syn
    N, h, r, M, k, unit = WORKLOADS[workload]
    R1 = syn.normal_bf16(0, syn.TENSOR_R1, h, r, 1.0 / np.sqrt(h))
    R2 = syn.normal_bf16(0, syn.TENSOR_R2, r, M, 1.0 / np.sqrt(r))
    rng = np.random.default_rng(1)

    def run(S):
        X = syn.normal_bf16(0, syn.TENSOR_X, N, h, 1.0, unit, 0, S)
        idx = rng.integers(0, M, (S, k))
        t = time.perf_counter()
        oracle.router_backward(X, R1, R2, S, h, r, M, idx, rng.standard_normal((S, k)), rng.standard_normal(M))
        return time.perf_counter() - t

    probe = 256
    per_tok = run(probe) / probe
    S = int(max(probe, min(N, seconds / max(per_tok, 1e-9), 32768)))
    el = run(S)
    threads = blas_threads()
    return {"value": S / el, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"first {S} of the {N} tokens, all M experts, {el:.1f} s (numpy, {threads} BLAS threads)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--variant", default="auto",
                    choices=["auto", "fused_tc", "small_n", "cluster", "unfused", "unfused_tc", "fullrank", "train", "dispatch", "dispatch_shared",
                             "backward"],
                    help="train: more_route_train (routing plus the full-softmax statistics m, Z, psum); "
                         "dispatch: routing followed by more_dispatch of its indices (dispatch_shared: with the "
                         "shared-memory dispatch kernels); "
                         "backward: more_route_backward (Algorithm 3) given the forward's selections, m and Z")
    ap.add_argument("--workload", default="prefill_r32", choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle sample size, in CPU seconds")
    ap.add_argument("--ref-step-seconds", type=float, default=3.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--tokens", type=int, default=0, help="override N (profiling a smaller case)")
    ap.add_argument("--launch", default="auto", choices=["auto", "eager", "graph"],
                    help="graph: each timed step replays a CUDA graph of one routing call (auto: N <= 65536)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup()
    if args.impl == "reference":
        return run_reference(args, world, rank)

    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import mixture_experts_rank_b200 as more
    from mixture_experts_rank_b200 import shard
    import synthetic as syn

    N, h, r, M, k, unit = WORKLOADS[args.workload]
    if args.tokens:
        N = args.tokens
    # weak scaling: rank i routes rows [i N, (i+1) N) of one synthetic set of N x world tokens (seed 0)
    begin, count = shard.shard_range(N * world, world, rank)
    Xh = syn.normal_bf16(0, syn.TENSOR_X, N * world, h, 1.0, unit, begin, count)
    R1h = syn.normal_bf16(0, syn.TENSOR_R1, h, r, 1.0 / np.sqrt(h))
    R2h = syn.normal_bf16(0, syn.TENSOR_R2, r, M, 1.0 / np.sqrt(r))

    def dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()

    X, R1, R2 = dev(Xh), dev(R1h), dev(R2h)
    idx = torch.empty((N, k), dtype=torch.int32, device="cuda")
    gate = torch.empty((N, k), dtype=torch.float32, device="cuda")
    cnt = torch.empty((M,), dtype=torch.int32, device="cuda")
    logits = torch.empty((N, k), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    scratch = None
    if args.variant == "train":
        m_buf = torch.empty((N,), dtype=torch.float32, device="cuda")
        z_buf = torch.empty((N,), dtype=torch.float32, device="cuda")
        psum_buf = torch.empty((M,), dtype=torch.float32, device="cuda")
    if args.variant in ("dispatch", "dispatch_shared"):
        d_scratch = torch.empty(max(more.dispatch_scratch_bytes(N, k, M), 16), dtype=torch.uint8, device="cuda")
        d_off = torch.empty((M + 1,), dtype=torch.int32, device="cuda")
        d_sorted = torch.empty((N * k,), dtype=torch.int32, device="cuda")
    if args.variant == "fullrank":
        W = dev(syn.normal_bf16(0, syn.TENSOR_R2, h, M, 1.0 / np.sqrt(h)))   # W ~ N(0, 1/h), h x M
    if args.variant in ("unfused", "unfused_tc"):
        scratch = torch.empty(more.unfused_scratch_bytes(N, r, M), dtype=torch.uint8, device="cuda")
    if args.variant == "backward":
        # the forward's selections and statistics (untimed), seeded incoming gradients
        b_m = torch.empty((N,), dtype=torch.float32, device="cuda")
        b_Z = torch.empty((N,), dtype=torch.float32, device="cuda")
        more.route_train(X, R1, R2, k, out_idx=idx, out_gate=gate, out_expert_count=cnt, out_logits=logits,
                         out_m=b_m, out_Z=b_Z, out_psum=torch.empty((M,), dtype=torch.float32, device="cuda"))
        grng = np.random.default_rng(2)
        b_tvb = torch.from_numpy(grng.standard_normal((N, k)).astype(np.float32)).cuda()
        b_pbar = torch.from_numpy(grng.standard_normal(M).astype(np.float32)).cuda()
        b_scratch = torch.empty(max(more.route_backward_scratch_bytes(N, h, r, M), 16), dtype=torch.uint8,
                                device="cuda")
        b_out = (torch.empty((N, h), dtype=torch.float32, device="cuda"),
                 torch.empty((h, r), dtype=torch.float32, device="cuda"),
                 torch.empty((r, M), dtype=torch.float32, device="cuda"),
                 torch.empty((N,), dtype=torch.float32, device="cuda"))

    def step(st=None):
        st = stream if st is None else st
        if args.variant == "train":
            more.route_train(X, R1, R2, k, out_idx=idx, out_gate=gate, out_expert_count=cnt, out_logits=logits,
                             out_m=m_buf, out_Z=z_buf, out_psum=psum_buf, stream=st)
        elif args.variant in ("dispatch", "dispatch_shared"):
            more.route(X, R1, R2, k, out_idx=idx, out_gate=gate, out_expert_count=cnt, out_logits=logits, stream=st)
            more.dispatch(idx, M, scratch=d_scratch, out_offsets=d_off, out_sorted=d_sorted,
                          variant="shared" if args.variant == "dispatch_shared" else "auto", stream=st)
        elif args.variant == "backward":
            more.route_backward(X, R1, R2, k, top_idx=idx, top_vals_bar=b_tvb, pbar=b_pbar, m=b_m, Z=b_Z,
                                scratch=b_scratch, out_Xbar=b_out[0], out_R1bar=b_out[1], out_R2bar=b_out[2],
                                out_g=b_out[3], stream=st)
        elif args.variant == "unfused":
            more.route_unfused(X, R1, R2, k, scratch=scratch, out_idx=idx, out_gate=gate, out_expert_count=cnt,
                               out_logits=logits, stream=st)
        elif args.variant == "fullrank":
            more.route_fullrank(X, W, k, out_idx=idx, out_gate=gate, out_expert_count=cnt, out_logits=logits,
                                stream=st)
        elif args.variant == "unfused_tc":
            more.route_unfused_tc(X, R1, R2, k, scratch=scratch, out_idx=idx, out_gate=gate,
                                  out_expert_count=cnt, out_logits=logits, stream=st)
        else:
            more.route(X, R1, R2, k, out_idx=idx, out_gate=gate, out_expert_count=cnt, out_logits=logits,
                       variant=args.variant, stream=st)

    variant_used = args.variant
    if args.variant == "auto":
        variant_used = more.auto_variant(N, h, r, M, k)
    launches_per_step = {"unfused": 3, "unfused_tc": 2, "train": 2, "dispatch": 5, "dispatch_shared": 5,
                         "backward": 5}.get(args.variant, 1)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if more.device_status() != 0:
        raise RuntimeError("a kernel recorded a device error during warm-up")

    # small batches are launch-bound: each step is then the replay of a CUDA graph holding
    # one routing call (the C-ABI call is asynchronous and allocates nothing, so it captures)
    use_graph = args.launch == "graph" or (args.launch == "auto" and N <= 65536)
    graph = None
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(torch.cuda.current_stream())
        graph.replay()
        torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    ev[0].record(stream)
    for i in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    total_ms = ev[0].elapsed_time(ev[-1])
    per_launch = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    if dist is not None:
        total_ms = shard.max_over_ranks(total_ms, torch.device("cuda", local))
    if more.device_status() != 0:
        raise RuntimeError("a kernel recorded a device error during the timed steps")
    ms = total_ms / args.steps
    value = N * world / (ms / 1e3)

    # end to end: pinned host X in, route through the public API, results out
    e2e = None  # through the public routing API; the other variants' steps are not routing calls
    if not args.no_e2e and args.variant in more.VARIANTS:
        router = more.Router(R1, R2, k, N, variant=args.variant)
        Xpin = torch.from_numpy(Xh.view(np.int16)).view(torch.bfloat16).pin_memory()
        for _ in range(2):
            router.route_host(Xpin)
        barrier()
        torch.cuda.synchronize()
        e_steps = max(3, min(args.steps, 10))
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(e_steps):
            router.route_host(Xpin, synchronize=False)
        t1.record(stream)
        torch.cuda.synchronize()
        e_ms = t0.elapsed_time(t1) / e_steps
        if dist is not None:
            e_ms = shard.max_over_ranks(e_ms, torch.device("cuda", local))
        bi, bo = router.bytes_per_call(N)
        e2e = {"value": N * world / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": bi,
               "d2h_bytes_per_step": bo, "ms_per_step": e_ms}

    if rank == 0:
        hbm, tc, tc_sus, src = peaks()
        x_bytes = 2.0 * N * h                        # algorithmic bytes of one launch: X read once
        flops = 2.0 * N * r * (h + M)                # z = x.R1 and l = z.R2
        launch_ms = statistics.mean(per_launch) if launches_per_step == 1 else None
        kernel_ms = launch_ms if launch_ms is not None else ms
        achieved = x_bytes / (kernel_ms / 1e3) / 1e9
        traffic = None
        if variant_used == "fused_tc" and args.workload in NCU_TRAFFIC:
            per_token, digest = NCU_TRAFFIC[args.workload]
            if kernel_source_digest() == digest:
                traffic = per_token * N  # bytes per launch
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": traffic, "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured"
                else "fallback 6.65 TB/s",
                "tensor": {"achieved_tflops": flops / (kernel_ms / 1e3) / 1e12, "peak_tflops": tc,
                           "frac": flops / (kernel_ms / 1e3) / 1e12 / tc}}
        if args.variant == "fullrank":
            # tensor-bound: 2 N h M FLOP of x . W per launch (X read once: 2 N h bytes)
            fflops = 2.0 * N * h * M / (kernel_ms / 1e3) / 1e12
            roof = {"bound": "tensor", "achieved": fflops, "peak": tc, "unit": "TFLOP/s", "frac": fflops / tc,
                    "traffic": None, "peak_source": f"{src} (MEASURED_PEAKS.json bf16_tflops)" if src == "measured"
                    else "fallback 1.59 PFLOP/s",
                    "hbm": {"achieved_gbs": achieved, "peak_gbs": hbm, "frac": achieved / hbm}}
        if args.variant == "backward":
            # fp32 FMA work without recompute: z, logits, zbar, Xbar, R1bar, R2bar (6 r (h + M) per
            # token) plus g (2 M); timed over the whole step (five launches)
            bflops = N * (6.0 * r * (h + M) + 2.0 * M)
            fp32_peak = 148 * 128 * 2 * 1.965e9 / 1e12
            achieved_t = bflops / (ms / 1e3) / 1e12
            roof = {"bound": "alu", "achieved": achieved_t, "peak": fp32_peak, "unit": "TFLOP/s",
                    "frac": achieved_t / fp32_peak, "traffic": None, "timed": "whole backward step",
                    "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz clocks.max.sm"}
        metric = {"backward": BACKWARD_METRIC, "fullrank": FULLRANK_METRIC}.get(args.variant, METRIC)
        line = {"metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32" if args.variant == "backward" else "bf16", "data": "synthetic",
                "config": {"workload": describe(args.workload) + (f" (N overridden to {N})" if args.tokens else ""),
                           "N_per_gpu": N, "h": h, "r": r, "M": M, "k": k,
                           "variant": variant_used, "parallelism": f"token shards x{world}",
                           "launch": "CUDA graph replay of one call per step" if graph is not None else "eager",
                           "l2": f"inputs larger than L2 (X = {x_bytes / 1e9:.2f} GB per GPU)"
                           if x_bytes > L2_BYTES else "inputs fit in L2; no flush (L2-warm)"},
                "roofline": roof, "gpu_launches": launches_per_step * args.steps, "clocks": clocks}
        if e2e is not None:
            line["e2e"] = e2e
        if not args.no_cpu_baseline and world == 1:
            if args.variant == "backward":
                line["cpu_baseline"] = backward_cpu_baseline(args.workload, args.cpu_seconds)
            else:
                line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds, args.variant == "fullrank")
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
