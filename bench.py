#!/usr/bin/env python3
"""Benchmark of the MXFP4 routed-expert MoE layer on B200.

One step = one k3moe_layer call over one batch of the workload's tokens (the
whole hot path: router, softmax, top-k, dispatch, routed gate/up + SwiGLU,
down projections with the weighted combine, shared expert).  Default workload: the K3-shape
decode layer (d=7168, ff=1536, 896 experts, top-16, bf16 shared expert
ff=1536, T=1 token), all 896 experts resident in HBM (15.7 GB).

Timing: W warm-up steps, then K timed steps; before every step a 256 MiB
buffer is written and another 256 MiB read, so L2 (126 MB) holds none of the
weights and no dirty lines whose write-back the step would pay; each step is
bracketed by CUDA events on the launching stream (the flush stays outside),
and the per-kernel durations come from K further steps in which the library
records events between its kernels (k3moe_layer_timed; those events
serialise the kernels, so those steps stay out of the headline).  Multi-GPU: replicas only (each rank runs
its own layer instance on its own GPU, no collective in the data path);
value = tokens of all ranks / max-over-ranks time.

--impl reference times the fp64 CPU oracle on the same workload.
"""
from __future__ import annotations

import argparse
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

import k3gen  # noqa: E402

METRIC = "MoE-layer tokens/s"
UNIT = "tokens/s"


def workload_desc(cfg):
    return (f"{cfg.name}: d={cfg.d}, ff={cfg.ff}, E={cfg.E}, top-{cfg.k}, shared ff={cfg.ff_shared},"
            f" T={cfg.T}, bias={cfg.bias or 'none'}")


def alg_bytes(cfg, U):
    """Algorithmic HBM bytes of one layer call: router weights, shared expert,
    each distinct selected expert once, activations in and out."""
    router = cfg.E * cfg.d * 4
    shared = 3 * cfg.d * cfg.ff_shared * 2
    experts = U * cfg.blob_bytes
    act = cfg.T * cfg.d * 2 * 2
    return router + shared + experts + act


def launches_per_step(cfg, T):
    """The library's kernel launches for one layer call: 3 per 8-token pass
    (decode); for more tokens per grouped-prefill pass (up to 8192 tokens):
    router GEMM (+ its split-K sum), top-k, 4 dispatch kernels, the
    quantising pass, gate/up, down, combine."""
    if T <= 8:
        return 3
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n = 0
    for t0 in range(0, T, 8192):
        tq = min(8192, T - t0)
        gx, gy = -(-cfg.E // 128), -(-tq // 128)
        ns = max(1, min(8, cfg.d // 256, -(-(2 * sms) // (gx * gy))))
        n += 10 + (1 if ns > 1 else 0)
    return n


def layer_flops(cfg, T):
    """Algorithmic FLOPs of one layer call (2 per multiply-add): router, the
    k routed experts of every token (gate, up, down), the shared expert."""
    return 2 * T * (cfg.E * cfg.d + cfg.k * 3 * cfg.d * cfg.ff + 3 * cfg.d * cfg.ff_shared)


def gu_bytes(cfg, U, pairs):
    """Algorithmic bytes of one gate/up launch: W_g and W_u of each distinct
    routed expert (nibbles + scales) and of the bf16 shared expert, x in, the
    SwiGLU activations out (counted as fp32, one per selected pair and token)."""
    return (U * 2 * cfg.d * cfg.ff * 17 // 32 + 2 * cfg.d * cfg.ff_shared * 2 + cfg.T * cfg.d * 2
            + (pairs * cfg.ff + cfg.T * cfg.ff_shared) * 4)


def down_bytes(cfg, U, pairs):
    """Algorithmic bytes of one down launch: W_d of each distinct routed expert
    and of the shared expert, the activations in (fp32 equivalent), y out."""
    return (U * cfg.d * cfg.ff * 17 // 32 + cfg.d * cfg.ff_shared * 2
            + (pairs * cfg.ff + cfg.T * cfg.ff_shared) * 4 + cfg.T * cfg.d * (4 if cfg.out_fp32 else 2))


def route_bytes(cfg):
    """Algorithmic bytes of one route launch: fp32 router weights, x in."""
    return cfg.E * cfg.d * 4 + cfg.T * cfg.d * 2


# The committed ncu summary that holds the DRAM traffic of each timed kernel
# (K3 decode shape, T=1, 16 distinct experts): kernel name -> profile file.
TRAFFIC_PROFILES = {"expert_gu": "expert_gu_k3_decode_e64.md"}


def captured_traffic(cfg, kernel):
    """DRAM bytes (read + write) of one launch of `kernel` from its committed
    ncu summary, while the kernel sources still hash to the captured ones and
    the launch moves the same bytes (d, ff, k, shared ff, T and 16 distinct
    experts); otherwise None."""
    import hashlib
    here = os.path.dirname(os.path.abspath(__file__))
    prof = TRAFFIC_PROFILES.get(kernel)
    if prof is None:
        return None
    try:
        text = open(os.path.join(here, "profiles", prof)).read()
    except OSError:
        return None
    fields = dict(line.split(": ", 1) for line in text.splitlines()
                  if line.startswith(("traffic_bytes_per_launch: ", "source_sha256: ", "source_files: ")))
    files = fields.get("source_files", "umma_kernels.cuh umma.cuh common.cuh layout.cuh").split()
    src = os.path.join(here, "mxfp4_routed_expert_softmax_b200", "csrc")
    h = hashlib.sha256()
    try:
        for f in files:
            h.update(open(os.path.join(src, f), "rb").read())
    except OSError:
        return None
    if fields.get("source_sha256", "").strip() != h.hexdigest():
        return None
    if (cfg.d, cfg.ff, cfg.k, cfg.ff_shared, cfg.T) != (7168, 1536, 16, 1536, 1):
        return None
    return int(fields["traffic_bytes_per_launch"])


def load_bf16_peak():
    """Measured dense bf16 TFLOP/s (burst) and its kind, else the fallback 1590."""
    here = os.path.dirname(os.path.abspath(__file__))
    try:
        with open(os.path.join(here, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        v = d.get("bf16_tflops")
        if isinstance(v, dict):
            v = v.get("value")
        return float(v), "measured"
    except (OSError, ValueError, TypeError):
        return 1590.0, "fallback"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
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
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def omp_threads(n=None):
    """The OpenMP thread count the oracle's parallel regions use (the process's
    libgomp, which the oracle links); with n, set it first."""
    import ctypes
    gomp = ctypes.CDLL("libgomp.so.1")
    if n is not None:
        gomp.omp_set_num_threads(int(n))
    return int(gomp.omp_get_max_threads())


def cpu_oracle_time(cfg, seconds=10.0, threads=None):
    """Time the fp64 oracle (as it stands) on whole tokens of the workload
    until ~`seconds` of work (at least one token), on `threads` OpenMP threads
    (None: as configured); -> (tokens/s, threads used, n_tokens, seconds)."""
    import oracle
    orc = oracle.oracle()
    before = omp_threads()
    if threads is not None:
        omp_threads(threads)
    try:
        return _cpu_oracle_time(orc, cfg, seconds)
    finally:
        omp_threads(before)


def _cpu_oracle_time(orc, cfg, seconds):
    # tokens beyond the workload's own T are further draws of the same
    # distribution (stream 0), so a small-T workload still gives a sample of
    # ~`seconds` of oracle work
    x = k3gen.hidden(cfg, T=max(cfg.T, 256))
    w = k3gen.router(cfg)
    b = k3gen.bias(cfg)
    sh = k3gen.shared(cfg) if cfg.ff_shared else None
    cache = {}
    threads = omp_threads()
    done = 0
    t_total = 0.0
    while t_total < seconds and done < x.shape[0]:
        xs = x[done:done + 1]
        # blob generation is input preparation, kept outside the timed region
        _, _, idx, _ = orc.route(xs, w, b, cfg.k)
        for e in idx[0]:
            if int(e) not in cache:
                cache[int(e)] = k3gen.expert_blob(cfg, int(e))
        t0 = time.perf_counter()
        _, _, idx, wt = orc.route(xs, w, b, cfg.k)
        orc.combine(xs, wt, [cache[int(e)] for e in idx[0]], sh, cfg.d, cfg.ff)
        t_total += time.perf_counter() - t0
        done += 1
    return done / t_total, threads, done, t_total


def arm_config(cfg, world):
    """The workload description both arms report."""
    return {"workload": workload_desc(cfg), "global_batch": world * cfg.T, "seq_len": 1,
            "parallelism": f"replicas x{world}"}


def max_over_ranks(value, world, device):
    """The largest of every rank's value (each rank calls it; the ranks are
    independent replicas and exchange nothing else)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, T, steps, max_ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * T * steps / (max_ms / 1000.0)


def run_reference(args, cfg, rank, world):
    """The reference arm: the fp64 CPU oracle as it stands, on the host cores,
    rank 0 only.  A step is one token of the workload (route + combine); W
    untimed steps, then K timed ones."""
    if rank != 0:
        return
    import oracle
    orc = oracle.oracle()
    n = args.warmup + args.steps
    x = k3gen.hidden(cfg, T=max(cfg.T, n))
    w = k3gen.router(cfg)
    b = k3gen.bias(cfg)
    sh = k3gen.shared(cfg) if cfg.ff_shared else None
    threads = omp_threads()
    cache = {}
    t_total = 0.0
    for i in range(n):
        xs = x[i:i + 1]
        _, _, idx, _ = orc.route(xs, w, b, cfg.k)
        for e in idx[0]:  # input preparation (blob generation) outside the timed region
            if int(e) not in cache:
                cache[int(e)] = k3gen.expert_blob(cfg, int(e))
        t0 = time.perf_counter()
        _, _, idx, wt = orc.route(xs, w, b, cfg.k)
        orc.combine(xs, wt, [cache[int(e)] for e in idx[0]], sh, cfg.d, cfg.ff)
        if i >= args.warmup:
            t_total += time.perf_counter() - t0
    tok_s = args.steps / t_total
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": arm_config(cfg, world),
        "cpu_baseline": {"value": tok_s, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"one token of the workload per step, {args.steps} timed steps after "
                                   f"{args.warmup} warm-up, fp64 scalar C oracle (OpenMP over output rows)"},
        "e2e": {"value": tok_s, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="k3_decode", choices=list(k3gen.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true", help="profiling mode: no e2e/cpu legs")
    ap.add_argument("--layers", type=int, default=92,
                    help="also time one token through this many K3 MoE layers in a row (0: skip)")
    ap.add_argument("--cache-slots", type=int, nargs="*", default=[64, 128, 256],
                    help="expert-cache slot counts to simulate (the middle one also timed); none: skip")
    ap.add_argument("--one-launch", action="store_true",
                    help="decode passes as one cooperative launch (K3MOE_ONE_LAUNCH) instead of three")
    ap.add_argument("--no-configs", action="store_true",
                    help="measure the headline workload only (not the T=8 / prefill workloads)")
    ap.add_argument("--route-only", action="store_true",
                    help="profiling: time the routing alone (k3moe_route: router, softmax, top-k) on "
                         "the workload's router; only the router and x are on the device")
    ap.add_argument("--experts", type=int, default=None,
                    help="profiling: keep only this many experts resident (same d, ff, top-k); the "
                         "routed and shared bytes per token stay those of the workload, the router shrinks")
    args = ap.parse_args()
    if args.warmup < 3 and not args.quick:
        args.warmup = 3
    cfg = k3gen.CONFIGS[args.config]
    if args.experts is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}_e{args.experts}", E=args.experts)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, cfg, rank, world)
        return

    import torch
    import torch.distributed as dist
    import mxfp4_routed_expert_softmax_b200 as k3
    from k3gen import device as kdev

    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    if args.route_only:
        measure_route_only(cfg, k3, args)
        return

    W = kdev.weights(cfg)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    rflush = torch.ones(64 << 20, dtype=torch.float32, device="cuda")  # 256 MiB, read after the write

    def flush_l2(i):
        # write a buffer twice the L2, then read another: the written lines
        # leave L2 here (their write-back is not charged to the next step)
        flush.fill_(i & 255)
        rflush.sum()

    stream = torch.cuda.current_stream()
    peak, _ = load_peaks()

    # the headline workload, then (default run) the other K3 workloads on the
    # same resident weights, each measured the same way
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    head = measure(cfg, W, k3, args, flush_l2, stream, world, e2e=not args.quick, one_launch=args.one_launch)
    others = {}
    alt = None
    if args.config == "k3_decode" and args.experts is None and not args.quick and not args.no_configs:
        # the other decode implementation on the same workload (K3MOE_ONE_LAUNCH toggled)
        alt = measure(cfg, W, k3, args, flush_l2, stream, world, e2e=False, one_launch=not args.one_launch)
    if args.config == "k3_decode" and args.experts is None and not args.quick and not args.no_configs:
        for name in ("k3_decode_t8", "k3_prefill_512", "k3_prefill_4096"):
            others[name] = measure(k3gen.CONFIGS[name], W, k3, args, flush_l2, stream, world, e2e=False)
    model = None
    if args.config == "k3_decode" and args.experts is None and not args.quick and args.layers > 0:
        model = measure_model(cfg, W, k3, args, flush_l2, stream, world, args.layers)
    cache = None
    if args.config == "k3_decode" and args.experts is None and not args.quick and args.cache_slots:
        cache = measure_cache(W, k3, args, stream)
    clk = clocks.stop()

    T = head["T"]
    ms_per_step = head["ms_per_step"]
    value = head["value"]
    roofline = head["roofline"]
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.quick:
        tok_s, threads, n, t = cpu_oracle_time(cfg, seconds=10.0)
        cpu = {"value": tok_s, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{n} token(s) of the workload ({t:.1f} s), fp64 scalar C oracle, "
                         f"OpenMP over output rows ({threads} threads: the process's OpenMP setting)",
               "cpu_model": cpu_model()}
        tok_1, _, n1, t1 = cpu_oracle_time(cfg, seconds=5.0, threads=1)
        cpu["single_thread"] = {"value": tok_1, "unit": UNIT, "cores": 1,
                                "sample": f"{n1} token(s) of the workload ({t1:.1f} s) on one OpenMP thread"}
        for name, r in others.items():
            tok_s, threads, n, t = cpu_oracle_time(k3gen.CONFIGS[name], seconds=4.0)
            r["cpu_baseline"] = {"value": tok_s, "unit": UNIT, "cores": threads, "kind": "oracle",
                                 "sample": f"{n} token(s) of the workload ({t:.1f} s)"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "mxf4 (E2M1 x E2M1, E8M0 block scales) tcgen05 MMA, f32 accumulate",
        "data": "synthetic",
        "config": dict(arm_config(cfg, world),
                       l2="256 MiB buffer written, then another 256 MiB read, before every step, outside the timed events",
                       distinct_experts=head["U"]),
        "layer_hbm_gbs": head["layer_gbs"],
        "layer_hbm_frac": round(head["layer_gbs"] / peak, 4),
        "per_kernel_ms": head["per_kernel_ms"],
        "per_kernel_gbs": head["per_kernel_gbs"],
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": head["e2e"],
        "gpu_launches": head["launches"] * args.steps,
        "clocks": clk,
    }
    line["config"]["decode"] = "one launch (K3MOE_ONE_LAUNCH)" if args.one_launch else "three launches (default)"
    if alt is not None:
        line["other_decode"] = dict(summary(alt, peak),
                                    decode="three launches (default)" if args.one_launch else "one launch (K3MOE_ONE_LAUNCH)")
    if others:
        line["configs"] = {name: summary(r, peak) for name, r in others.items()}
    if model is not None:
        line["model_decode"] = model
    if cache is not None:
        line["expert_cache"] = cache
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_model(cfg, W, k3, args, flush_l2, stream, world, n_layers):
    """One decode token through n_layers K3 MoE layers in a row (the steps of
    a pre-norm block: RMSNorm, the layer, the residual add; k3moe_layer_residual
    with the residual stream updated in place, one launch per layer), every
    layer with its own router,
    shared expert and norm weights and its own permutation of the resident
    experts, captured in a CUDA graph.  L2 is flushed before each token, not
    between layers: consecutive layers stream different weights.  The layers
    share one workspace, so its tensor maps (cached per expert id) change with
    every layer: the one-launch decode kernel (K3MOE_ONE_LAUNCH) rewrites them
    in its set-up, off the routing path, where the three-launch path rewrites
    the selected experts' maps at dispatch, on it."""
    import torch
    E, d = cfg.E, cfg.d
    dims = k3.make_dims(cfg.d, cfg.ff, cfg.E, cfg.k, cfg.ff_shared, k3.K3MOE_ONE_LAUNCH)
    ws = k3.new_workspace(dims, 1)
    layers = []
    for l in range(n_layers):
        seed = 1000 + l
        wr = torch.from_numpy(k3gen.router(cfg, seed)).cuda()
        sg, su, sd = (torch.from_numpy(a.view(np.int16)).cuda() for a in k3gen.shared(cfg, seed))
        g = torch.from_numpy(k3gen.norm_weights(cfg, seed).view(np.int16)).cuda()
        perm = np.random.default_rng(seed).permutation(E)
        ptrs = W.blob_ptrs[torch.from_numpy(perm).cuda()].contiguous()
        layers.append((wr, sg, su, sd, g, ptrs))
    h0 = torch.from_numpy(k3gen.hidden(cfg, T=1).view(np.int16)).cuda()
    h = h0.clone()

    def token():
        for (wr, sg, su, sd, g, ptrs) in layers:
            k3.check(k3.k3moe_layer_residual(h, 1, g, 1e-6, wr, None, ptrs, sg, su, sd, dims, h, ws),
                     "k3moe_layer_residual")

    for _ in range(2):
        h.copy_(h0)
        token()
    torch.cuda.synchronize()
    k3.check(k3.k3moe_device_status(ws), "device status")
    graph = None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            token()
        graph.replay()
        torch.cuda.synchronize()
        k3.check(k3.k3moe_device_status(ws), "device status")
    except Exception as ex:  # capture refused: time the launches themselves
        graph = None
        capture_error = str(ex).splitlines()[0][:200]
    steps = max(3, min(args.steps, 10))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        h.copy_(h0)
        flush_l2(i)
        ev[i][0].record(stream)
        if graph is not None:
            graph.replay()
        else:
            token()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    k3.check(k3.k3moe_device_status(ws), "device status")
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, "cuda")
    ms = total_ms / steps
    peak, _ = load_peaks()
    gbs = n_layers * alg_bytes(cfg, cfg.k) / (ms / 1000.0) / 1e9  # 16 distinct experts per layer at T=1
    out = {"layers": n_layers, "tokens_per_step": 1, "steps": steps, "ms_per_token": round(ms, 4),
           "value": round(world * 1000.0 / ms, 2), "unit": "tokens/s (all layers)",
           "us_per_layer": round(1000.0 * ms / n_layers, 2), "hbm_gbs": round(gbs, 1),
           "hbm_frac": round(gbs / peak, 4), "cuda_graph": graph is not None,
           "gpu_launches_per_token": n_layers, "decode": "one launch (K3MOE_ONE_LAUNCH)"}
    if graph is None:
        out["cuda_graph_error"] = capture_error
    del graph, layers
    torch.cuda.empty_cache()
    return out


def measure_cache(W, k3, args, stream):
    """The expert cache under the Zipf-skewed routing of the 512-token K3
    workload, decoded one token at a time: the hit rate of the cache's own
    policy (k3moe_cache_plan over the tokens' routing) for each slot count,
    and, for the middle one, real k3moe_layer_cached calls with the experts in
    page-locked host memory (only the experts these tokens ever select are
    materialised on the host; the others are never fetched)."""
    import torch
    cfg = k3gen.CONFIGS["k3_prefill_512"]
    inp = kdev_inputs(cfg)
    T = inp.T
    dims = k3.make_dims(cfg.d, cfg.ff, cfg.E, cfg.k, cfg.ff_shared, 0)
    ws = k3.new_workspace(dims, 8)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    k3.check(k3.k3moe_route(inp.x, T, W.w_router, inp.bias, dims, idx, wts, ws), "route")
    idx = idx.cpu().numpy()
    used = sorted(set(idx.reshape(-1).tolist()))
    sb = k3.k3moe_cache_slot_bytes(dims)
    out = {"workload": workload_desc(cfg) + ", decoded one token per call", "tokens": T,
           "distinct_experts": len(used), "policy": "least recently used over slots", "slots": {}}
    for S in args.cache_slots:
        fake = type("F", (), {"data_ptr": lambda self: 1 << 40, "numel": lambda self: S * sb,
                              "element_size": lambda self: 1})()
        c = k3.ExpertCache(dims, S, fake, [0x1000] * cfg.E)
        for t in range(T):
            k3.check(c.plan(idx[t])[0], "cache plan")
        st = c.stats()
        c.close()
        out["slots"][str(S)] = {"hit_rate": round(st["hits"] / st["requests"], 4), "fills": st["fills"],
                                "device_bytes": S * sb}
    S = args.cache_slots[len(args.cache_slots) // 2]
    host = torch.empty((len(used), cfg.blob_bytes), dtype=torch.uint8).pin_memory()
    ptrs = [0] * cfg.E
    for i, e in enumerate(used):
        host[i].copy_(W.blobs[e].cpu())
        ptrs[e] = host.data_ptr() + i * cfg.blob_bytes
    dummy = torch.zeros(16, dtype=torch.uint8).pin_memory()  # never fetched: no token selects these
    ptrs = [p if p else dummy.data_ptr() for p in ptrs]
    slots = torch.empty(S * sb, dtype=torch.uint8, device="cuda")
    table = torch.zeros(cfg.E, dtype=torch.int64, device="cuda")
    cache = k3.ExpertCache(dims, S, slots, ptrs)
    idx_host = torch.empty(cfg.k, dtype=torch.int32).pin_memory()
    y = torch.empty((1, cfg.d), dtype=torch.int16, device="cuda")
    sg, su, sd = W.shared
    n = min(T, 256)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for t in range(n):
        k3.check(k3.k3moe_layer_cached(cache, inp.x[t:t + 1], 1, W.w_router, inp.bias, table, sg, su, sd, dims,
                                       y, idx_host, ws), "k3moe_layer_cached")
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    k3.check(k3.k3moe_device_status(ws), "device status")
    st = cache.stats()
    out["timed"] = {"slots": S, "tokens": n, "tokens_per_s": round(n / wall, 1),
                    "ms_per_token": round(1000.0 * wall / n, 3), "hit_rate": round(st["hits"] / st["requests"], 4),
                    "fills": st["fills"], "host_to_device_gb": round(st["fills"] * cfg.blob_bytes / 1e9, 3),
                    "clock": "host wall clock (each call synchronises on its routing)"}
    cache.close()
    del host, slots
    torch.cuda.empty_cache()
    return out


def kdev_inputs(cfg):
    from k3gen import device as kdev
    return kdev.DeviceInputs(cfg)


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def summary(r, peak):
    """The per-workload record of the bench line's `configs` key."""
    out = {"workload": workload_desc(r["cfg"]), "tokens": r["T"], "steps": r["steps"],
           "ms_per_step": r["ms_per_step"], "value": r["value"], "unit": UNIT,
           "distinct_experts": r["U"], "layer_hbm_gbs": r["layer_gbs"],
           "layer_hbm_frac": round(r["layer_gbs"] / peak, 4), "roofline": r["roofline"],
           "gpu_launches_per_step": r["launches"]}
    if r["per_kernel_ms"]:
        out["per_kernel_ms"] = r["per_kernel_ms"]
        out["per_kernel_gbs"] = r["per_kernel_gbs"]
    if "cpu_baseline" in r:
        out["cpu_baseline"] = r["cpu_baseline"]
    return out


def kernel_names(n):
    """Names of the library's kernels in launch order for an 8-token pass."""
    return {3: ["route", "expert_gu", "expert_down"], 1: ["layer"]}.get(n, [f"k{i}" for i in range(n)])


def kernel_bytes(cfg, U, pairs, name):
    return {"route": route_bytes(cfg), "expert_gu": gu_bytes(cfg, U, pairs),
            "expert_down": down_bytes(cfg, U, pairs), "layer": alg_bytes(cfg, U)}.get(name)


def measure_route_only(cfg, k3, args):
    """Profiling mode: W warm-up and K timed k3moe_route calls (the router
    GEMV, softmax and top-k of the workload's first T tokens), L2 flushed
    before each, CUDA events on the launching stream; prints one JSON line
    (not a bench line: the routing alone)."""
    import torch
    wr = torch.from_numpy(k3gen.router(cfg)).cuda()
    b = k3gen.bias(cfg)
    bias = torch.from_numpy(b).cuda() if b is not None else None
    T = min(cfg.T, 8)
    x = torch.from_numpy(k3gen.hidden(cfg, T=T).view(np.int16)).cuda()
    dims = k3.make_dims(cfg.d, cfg.ff, cfg.E, cfg.k, cfg.ff_shared, 0)
    ws = k3.new_workspace(dims, T)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    ms = []
    for i in range(args.warmup + args.steps):
        flush.fill_(i & 255)
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        k3.check(k3.k3moe_route(x, T, wr, bias, dims, idx, wts, ws), "k3moe_route")
        e.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            ms.append(a.elapsed_time(e))
    k3.check(k3.k3moe_device_status(ws), "device status")
    us = 1000.0 * sum(ms) / len(ms)
    nbytes = cfg.E * cfg.d * 4 + T * cfg.d * 2
    print(json.dumps({"mode": "route-only", "workload": workload_desc(cfg), "tokens": T, "steps": args.steps,
                      "us_per_call": round(us, 2), "us_min": round(1000.0 * min(ms), 2),
                      "router_gbs": round(nbytes / (us * 1e-6) / 1e9, 1)}), flush=True)


def measure(cfg, W, k3, args, flush_l2, stream, world, e2e=False, one_launch=False):
    """W warm-up and K timed layer calls on one workload (L2 flushed before
    each, CUDA events on the launching stream, max over ranks); for passes of
    up to 8 tokens also K calls with events between the library's kernels,
    and (e2e) K calls through k3moe_layer_from_host with the copies timed."""
    import torch
    from k3gen import device as kdev
    inp = kdev.DeviceInputs(cfg)
    T = inp.T
    dims = k3.make_dims(cfg.d, cfg.ff, cfg.E, cfg.k, cfg.ff_shared,
                        (k3.K3MOE_OUT_FP32 if cfg.out_fp32 else 0) | (k3.K3MOE_ONE_LAUNCH if one_launch else 0))
    ws = k3.new_workspace(dims, T, host_staging=e2e)
    ybytes = 4 if cfg.out_fp32 else 2
    y = torch.empty((T, cfg.d), dtype=torch.float32 if cfg.out_fp32 else torch.int16, device="cuda")
    sg, su, sd = W.shared

    def step_plain():
        k3.check(k3.k3moe_layer(inp.x, T, W.w_router, inp.bias, W.blob_ptrs, sg, su, sd, dims, y,
                                None, None, ws), "k3moe_layer")

    for _ in range(args.warmup):
        flush_l2(1)
        step_plain()
    torch.cuda.synchronize()
    k3.check(k3.k3moe_device_status(ws), "device status")
    # distinct experts of the batch (for the algorithmic byte count)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    k3.check(k3.k3moe_route(inp.x, T, W.w_router, inp.bias, dims, idx, wts, ws), "route")
    U = len(np.unique(idx.cpu().numpy()))
    pairs = T * cfg.k

    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2(i)
        step_ev[i][0].record(stream)
        step_plain()
        step_ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    k3.check(k3.k3moe_device_status(ws), "device status")
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in step_ev), world, "cuda")
    ms_per_step = total_ms / args.steps
    value = job_throughput(world, T, args.steps, total_ms)

    # per-kernel durations: K more calls with events between the library's
    # kernels (k3moe_layer_timed; the events serialise the kernels, so these
    # calls are not part of the headline number)
    per_kernel = {}
    n_kernels = None
    if T <= 8:
        nev = 6
        kern_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
        for i in range(args.steps):
            flush_l2(i)
            st, n_kernels = k3.k3moe_layer_timed(inp.x, T, W.w_router, inp.bias, W.blob_ptrs, sg, su,
                                                 sd, dims, y, ws, kern_ev[i])
            k3.check(st, "k3moe_layer_timed")
        torch.cuda.synchronize()
        k3.check(k3.k3moe_device_status(ws), "device status")
        for j, name in enumerate(kernel_names(n_kernels)):
            per_kernel[name] = statistics.mean(kern_ev[i][j].elapsed_time(kern_ev[i][j + 1])
                                               for i in range(args.steps))

    peak, peak_kind = load_peaks()
    layer_gbs = alg_bytes(cfg, U) / (ms_per_step / 1000.0) / 1e9
    roofline = None
    if per_kernel:
        # the dominant kernel against the HBM copy peak
        name = max(per_kernel, key=per_kernel.get)
        gb = kernel_bytes(cfg, U, pairs, name)
        ach = gb / (per_kernel[name] / 1000.0) / 1e9
        roofline = {"bound": "hbm", "kernel": name, "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                    "frac": round(ach / peak, 4),
                    "peak_kind": f"{peak_kind} (burst copy, MEASURED_PEAKS.json hbm_gbs)"
                    if peak_kind == "measured" else "fallback 6.65 TB/s",
                    "traffic": captured_traffic(cfg, name) if U == 16 else None,
                    "alg_bytes_per_launch": gb}
    else:
        # many tokens (grouped prefill): the whole layer against its bound.  The
        # block-scaled fp4 tensor peak is the measured bf16 peak x 4 (the
        # nominal dense fp4/bf16 ratio, 9 / 2.25 PFLOP/s); the layer is
        # HBM-bound when its bytes take longer at the copy peak than its FLOPs
        # at that tensor peak.  Both fractions are reported.
        fl = layer_flops(cfg, T)
        bf16_peak, bf16_kind = load_bf16_peak()
        tensor_peak = bf16_peak * 4.0
        t_hbm = alg_bytes(cfg, U) / (peak * 1e9)
        t_tc = fl / (tensor_peak * 1e12)
        tf = fl / (ms_per_step / 1000.0) / 1e12
        hb = {"bound": "hbm", "kernel": "layer (all kernels of the grouped prefill)",
              "achieved": round(layer_gbs, 1), "peak": peak, "unit": "GB/s",
              "frac": round(layer_gbs / peak, 4), "traffic": None, "alg_bytes_per_launch": alg_bytes(cfg, U)}
        tc = {"bound": "tensor", "kernel": "layer (all kernels of the grouped prefill)",
              "achieved": round(tf, 2), "peak": round(tensor_peak, 1), "unit": "TFLOP/s",
              "frac": round(tf / tensor_peak, 4), "traffic": None, "alg_flops_per_launch": fl,
              "peak_kind": f"{bf16_kind} dense bf16 x 4 (nominal dense fp4 / bf16 ratio)"}
        roofline = dict(hb if t_hbm >= t_tc else tc)
        roofline["other_bound"] = tc if t_hbm >= t_tc else hb

    e2e_rec = None
    if e2e:
        xh = torch.from_numpy(inp.x_host.view(np.int16)).pin_memory()
        yh = torch.empty((T, cfg.d), dtype=torch.float32 if cfg.out_fp32 else torch.int16).pin_memory()
        e_ms = 0.0
        for i in range(args.warmup + args.steps):
            flush_l2(i)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            k3.check(k3.k3moe_layer_from_host(xh, T, W.w_router, inp.bias, W.blob_ptrs, sg, su, sd,
                                              dims, yh, ws), "from_host")
            b.record(stream)
            b.synchronize()  # the result is on the host here
            if i >= args.warmup:
                e_ms += a.elapsed_time(b)
        e_ms = max_over_ranks(e_ms, world, "cuda")
        e2e_rec = {"value": job_throughput(world, T, args.steps, e_ms), "unit": UNIT,
                   "h2d_bytes_per_step": T * cfg.d * 2, "d2h_bytes_per_step": T * cfg.d * ybytes}
    launches = n_kernels if (T <= 8 and n_kernels) else launches_per_step(cfg, T)
    del ws
    return {"cfg": cfg, "T": T, "U": U, "steps": args.steps, "ms_per_step": ms_per_step, "value": value,
            "layer_gbs": round(layer_gbs, 1), "per_kernel_ms": {k: round(v, 5) for k, v in per_kernel.items()},
            "per_kernel_gbs": {k: round(kernel_bytes(cfg, U, pairs, k) / (v / 1000.0) / 1e9, 1)
                               for k, v in per_kernel.items() if kernel_bytes(cfg, U, pairs, k)},
            "roofline": roofline, "e2e": e2e_rec, "launches": launches}


if __name__ == "__main__":
    main()
