#!/usr/bin/env python
"""Benchmark of the fused MoE layer forward on B200.

One step = one whole layer forward (router logits, top-k gating, histogram and
scan, permutation and row gather, gate/up grouped GEMM with SwiGLU, down
grouped GEMM, combine) over one batch of seeded synthetic tokens, through
moe_layer_forward.  Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode64]
                    [--T ..] [--alpha ..] [--fp8] [--impl ours|reference]

``--fp8`` times moe_layer_forward_fp8 (e4m3 expert weights with 128 x 128
block scales, quantised once before the timed region).

Multi-GPU (torchrun) runs independent replicas: the layer has no exchange
step, so every rank times its own copy and the value is the tokens of all
ranks over the slowest rank's time.

``--impl reference`` times the CPU oracle (the plain fp64 definition of the
layer) on the host cores on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from grouped_gemm_02_b200 import stats  # noqa: E402
from grouped_gemm_02_b200 import workload as wl  # noqa: E402

METRIC = "fused MoE layer µs & tokens/s on 1 B200; % of HBM / tensor-core roofline"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "roofline_traffic.json")
KERNEL_SOURCES = ["grouped_gemm_02_b200/csrc/grouped_gemm.cuh", "grouped_gemm_02_b200/csrc/ptx.cuh",
                  "grouped_gemm_02_b200/csrc/common.cuh"]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------ harness helpers (CPU-testable)

def dist_env():
    """(rank, local_rank, world) from the torchrun environment, (0, 0, 1) otherwise."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks of a float (identity when world == 1)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            p = json.load(open(path))
            return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
        except Exception:
            pass
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()[:16]


def committed_traffic(workload_name: str):
    """DRAM bytes per launch of the gate/up GEMM from the committed ncu summary,
    or None when absent, for another workload, or taken on older kernel source."""
    try:
        rec = json.load(open(PROFILE_TRAFFIC))
    except Exception:
        return None
    if rec.get("workload") != workload_name or rec.get("source_sha") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_ids):
        self.proc = None
        self.path = os.path.join("/tmp", f"moe_bench_clocks_{os.getpid()}.csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", ",".join(str(i) for i in gpu_ids)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def wait_first_sample(self, timeout=3.0):
        t0 = time.time()
        while self.proc and time.time() - t0 < timeout:
            if os.path.exists(self.path) and os.path.getsize(self.path) > 0:
                return
            time.sleep(0.02)

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), hw=parts[5], hwt=parts[6],
                                 swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r["sm"] for r in rows])), "sm_max_mhz": max(r["smax"] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ workload

def parse_workload(args) -> wl.LayerShape:
    kw = {}
    if args.T is not None:
        kw["T"] = args.T
    if args.alpha is not None:
        kw["alpha"] = args.alpha
    s = wl.shape(args.workload, **kw)
    return s


def workload_label(s: wl.LayerShape) -> str:
    lab = f"{s.name} T={s.T} d={s.d} f={s.f} E={s.E} k={s.k} alpha={s.alpha:g}"
    if s.f_shared:
        lab += f" shared_f={s.f_shared}"
    return lab


def gemm_fused(P: int, f: int) -> bool:
    """Whether the library runs both expert GEMMs as one launch for P pairs and width f."""
    forced = os.environ.get("MOE_GEMM_SPLIT", "")
    if forced in ("0", "1"):
        return forced == "0"
    return P <= 256 and f <= 4096


def algorithmic(s: wl.LayerShape, counts: np.ndarray, fp8: bool = False):
    """Algorithmic bytes and flops of the layer and of the gate/up GEMM launch.

    bf16: 2 bytes per weight and activation.  FP8: 1 byte per weight and
    activation plus one fp32 scale per 128 x 128 weight block and per 1 x 128
    activation block."""
    active = int((counts > 0).sum())
    P = int(counts.sum())
    fs = s.f_shared
    wb = 1 if fp8 else 2
    wsc = (4.0 / (128 * 128)) if fp8 else 0.0    # weight-scale bytes per weight
    asc = (4.0 / 128) if fp8 else 0.0            # activation-scale bytes per activation

    def mat(rows, cols):
        return rows * cols * (wb + wsc)

    def act(rows, cols):
        return rows * cols * (wb + asc)

    w_act = active * 3 * mat(s.d, s.f) + (3 * mat(s.d, fs) if fs else 0)
    flops = 6.0 * P * s.d * s.f + (6.0 * s.T * s.d * fs if fs else 0)
    g1_bytes = active * 2 * mat(s.f, s.d) + act(P, s.d) + act(P, s.f)
    g1_flops = 4.0 * P * s.d * s.f
    g2_bytes = active * mat(s.d, s.f) + act(P, s.f) + P * s.d * 2     # y_p is bf16
    g2_flops = 2.0 * P * s.d * s.f
    if fs:
        g1_bytes += 2 * mat(fs, s.d) + act(s.T, s.d) + act(s.T, fs)
        g1_flops += 4.0 * s.T * s.d * fs
        g2_bytes += mat(s.d, fs) + act(s.T, fs) + s.T * s.d * 2
        g2_flops += 2.0 * s.T * s.d * fs
    return dict(active=active, pairs=P, w_act=w_act, flops=flops, g1_bytes=g1_bytes, g1_flops=g1_flops,
                g2_bytes=g2_bytes, g2_flops=g2_flops)


# ------------------------------------------------------------------ CPU oracle timing

class OracleRun:
    """The CPU oracle on a token sample of a workload (host arrays prepared once)."""

    def __init__(self, s: wl.LayerShape, inp_host: dict):
        import oracle
        self.oracle = oracle
        self.s = s
        self.threads = oracle.default_threads()
        self.x = wl.bf16_bits(inp_host["x"])
        self.Wg = wl.bf16_bits(inp_host["Wg"])
        self.bias = inp_host["bias"].numpy()
        self.W1 = [wl.bf16_bits(inp_host["W1"][e]) for e in range(s.E)]
        self.W3 = [wl.bf16_bits(inp_host["W3"][e]) for e in range(s.E)]
        self.W2 = [wl.bf16_bits(inp_host["W2"][e]) for e in range(s.E)]
        self.shared = None
        if s.f_shared:
            self.shared = {n: wl.bf16_bits(inp_host[n]) for n in ("Ws1", "Ws3", "Ws2")}
        self.next = 0

    def batch(self, n: int) -> int:
        """Routing and expert FFNs of the next n tokens (wrapping around T)."""
        o = self.oracle
        toks = np.arange(self.next, self.next + n) % self.s.T
        self.next += n
        xs = np.ascontiguousarray(self.x[toks])
        L = o.router_logits(xs, self.Wg, self.bias).astype(np.float32)
        idx, w = o.topk(L, self.s.k)
        o.permutation(idx, self.s.E)
        o.moe_ffn(xs, self.W1, self.W3, self.W2, idx, w, shared=self.shared, nthreads=self.threads)
        return n

    def timed(self, budget_s: float, n: int):
        """Batches of n tokens until budget_s has passed: (tokens, seconds, threads used)."""
        done = 0
        t0 = time.perf_counter()
        while True:
            done += self.batch(n)
            el = time.perf_counter() - t0
            if el >= budget_s:
                return done, el, min(self.threads, n)


# ------------------------------------------------------------------ GPU arm

def run_ours(args, s: wl.LayerShape):
    from grouped_gemm_02_b200 import moe
    rank, local_rank, world = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    # inputs: R rotating weight sets so that consecutive steps never find their
    # weights in L2 (each set is larger than L2 already for the default layer)
    one = wl.make_weights(s, seed=args.seed, device=dev)
    wbytes = sum(t.numel() * t.element_size() for t in one.values())
    free, _ = torch.cuda.mem_get_info(dev)
    want = max(2, math.ceil(3 * L2_BYTES / max(wbytes, 1)))
    R = int(max(1, min(want, args.sets or want, (free * 0.6) // max(wbytes, 1))))
    sets = [one] + [wl.make_weights(s, seed=args.seed + 1000 * (i + 1), device=dev) for i in range(R - 1)]
    base = wl.make_inputs(s, seed=args.seed, device=dev, weights=False)
    x, Wg, bias = base["x"], base["Wg"], base["bias"]
    out = torch.empty(s.T, s.d, dtype=torch.bfloat16, device=dev)
    if args.fp8:
        # e4m3 weights with 128 x 128 block scales (quantised once, outside the timed region)
        qsets = [moe.quantize_layer_fp8(w) for w in sets]
        ws = moe.new_workspace_fp8(s.T, s.d, s.f, s.E, s.k, s.f_shared, device=dev)
        wbytes = sum(t.numel() * t.element_size() for t in qsets[0].values())
        sets = one = None                   # the bf16 weights are not used any more
        torch.cuda.empty_cache()
    else:
        ws = moe.new_workspace(s.T, s.d, s.f, s.E, s.k, s.f_shared, device=dev)

    def step(i, prof_events=None):
        if prof_events is not None:
            moe.moe_record_phase_events(prof_events)
        if args.fp8:
            moe.moe_layer_forward_fp8(x, Wg, bias, qsets[i % R], s.k, ws, out=out)
            return
        w = sets[i % R]
        moe.moe_layer_forward(x, Wg, bias, w["W1"], w["W3"], w["W2"], s.k, ws, Ws1=w.get("Ws1"),
                              Ws3=w.get("Ws3"), Ws2=w.get("Ws2"), out=out)

    sampler = ClockSampler([torch.cuda.current_device()]) if rank == 0 else None
    # warm-up (at least 3 steps; also lets the clock sampler start)
    for i in range(max(3, args.warmup)):
        step(i)
    if sampler:
        sampler.wait_first_sample()
    torch.cuda.synchronize()
    if moe.moe_get_device_error(ws) != 0:
        raise RuntimeError("device error after warm-up")

    # timed region: K steps of the layer, nothing else on the stream
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    n0 = moe.moe_launch_counter()
    start.record(stream)
    for i in range(K):
        step(i)
    end.record(stream)
    torch.cuda.synchronize()
    launches = moe.moe_launch_counter() - n0
    clocks = sampler.stop() if sampler else None
    ms = start.elapsed_time(end)
    ms_max = reduce_max(ms, world, dev)
    ms_per_step = ms_max / K
    if moe.moe_get_device_error(ws) != 0:
        raise RuntimeError("device error in the timed region")

    # per-phase pass: the same steps with CUDA events between the phases (an event
    # between two kernels keeps the second from starting early, so these phase
    # times are upper bounds); gives the gate/up GEMM's own duration
    Kp = min(K, 500)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(Kp)]
    for row in ev:          # torch creates the CUDA event on its first record
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    for i in range(Kp):
        step(i, ev[i])
    torch.cuda.synchronize()
    phase = np.array([[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(5)] for i in range(Kp)])
    phase_ms = phase.mean(axis=0)

    # end to end through the C ABI: pinned host x -> device, layer, device out -> pinned host
    e2e = None
    if not args.no_e2e:
        x_host = x.cpu().pin_memory()
        out_host = torch.empty(s.T, s.d, dtype=torch.bfloat16).pin_memory()
        for i in range(3):
            x.copy_(x_host, non_blocking=True)
            step(i)
            out_host.copy_(out, non_blocking=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for i in range(K):
            x.copy_(x_host, non_blocking=True)
            step(i)
            out_host.copy_(out, non_blocking=True)
        s1.record(stream)
        torch.cuda.synchronize()
        e_ms = reduce_max(s0.elapsed_time(s1), world, dev)
        e2e = {"value": s.T * K * world / (e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": s.T * s.d * 2, "d2h_bytes_per_step": s.T * s.d * 2,
               "ms_per_step": e_ms / K}

    # realised histogram and roofline
    if args.fp8:
        views = moe.workspace_views_fp8(ws, s.T, s.d, s.f, s.E, s.k, s.f_shared)
    else:
        views = moe.workspace_views(ws, s.T, s.d, s.f, s.E, s.k, s.f_shared)
    counts = views["counts"].cpu().numpy()
    alg = algorithmic(s, counts, fp8=args.fp8)
    pk, pk_kind = peaks()
    bw = pk["hbm_gbs"] * 1e9
    # FP8 tensor peak: the measured bf16 figure times the nominal fp8 / bf16 ratio (4.5 / 2.25)
    tc = pk["bf16_tflops_sustained"] * 1e12 * (2.0 if args.fp8 else 1.0)
    # the dominant kernel is the expert GEMM: one launch (gate/up + SwiGLU, then down) for
    # P <= 256 and f <= 4096, else the two launches together (the library's rule; the
    # MOE_GEMM_SPLIT variable overrides it there and here)
    t_g = (phase_ms[2] + phase_ms[3]) / 1e3
    g_bytes = alg["g1_bytes"] + alg["g2_bytes"]
    g_flops = alg["g1_flops"] + alg["g2_flops"]
    if g_bytes / bw >= g_flops / tc:
        roof = {"bound": "hbm", "achieved": g_bytes / t_g / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": g_flops / t_g / 1e12, "peak": tc / 1e12,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    # the record names the workload as the JSON line does (" fp8" for the FP8 kernels)
    roof["traffic"] = committed_traffic(workload_label(s) + (" fp8" if args.fp8 else ""))
    roof["kernel"] = ("grouped_gemm_fp8_kernel<gate/up>+<down>" if args.fp8 else
                      ("grouped_gemm_kernel<fused gate/up + down>" if gemm_fused(s.P, s.f)
                       else "grouped_gemm_kernel<gate/up>+<down>"))
    roof["algorithmic_bytes_per_launch"] = g_bytes
    roof["launch_us"] = t_g * 1e6
    roof["peak_source"] = f"{pk_kind} ({('2 x sustained bf16 (fp8)' if args.fp8 else 'sustained bf16') if roof['bound'] == 'tensor' else 'HBM copy'})"
    t_roof = max(alg["w_act"] / bw, alg["flops"] / tc)
    layer_roof = {"bound": "hbm" if alg["w_act"] / bw >= alg["flops"] / tc else "tensor",
                  "t_roof_us": t_roof * 1e6, "t_meas_us": ms_per_step * 1e3, "frac": t_roof / (ms_per_step / 1e3),
                  "w_act_bytes": alg["w_act"], "flops": alg["flops"], "peak_source": pk_kind}

    line = {"metric": METRIC, "value": s.T * K * world / (ms_max / 1e3), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp8-e4m3 (fp32 accumulate)" if args.fp8 else "bf16",
            "data": "synthetic",
            "config": {"workload": workload_label(s) + (" fp8" if args.fp8 else ""), "T": s.T, "d": s.d, "f": s.f,
                       "E": s.E, "k": s.k,
                       "alpha": s.alpha, "f_shared": s.f_shared, "seed": args.seed,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": f"inputs larger than L2: {R} rotating weight sets of {wbytes / 2**20:.0f} MiB",
                       "histogram": stats.histogram_stats(counts),
                       "us_per_layer": ms_per_step * 1e3,
                       "phase_note": "per-phase means from a second pass with CUDA events between phases",
                       "phase_us": {n: float(v * 1e3) for n, v in
                                    zip(("route", "permute", "gemm_gate_up", "gemm_down", "combine"), phase_ms)}},
            "roofline": roof, "layer_roofline": layer_roof, "e2e": e2e, "gpu_launches": int(launches),
            "clocks": clocks}
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.fp8:
        host = {n: v.cpu() for n, v in base.items()}
        host.update({n: v.cpu() for n, v in one.items()})
        orc = OracleRun(s, host)
        toks, secs, cores = orc.timed(args.cpu_budget, orc.threads)
        line["cpu_baseline"] = {"value": toks / secs, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"{toks} tokens of {workload_label(s)} (full routing + expert FFNs per "
                                          f"token, fp64), {secs:.1f} s on {cores} host threads"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return line if rank == 0 else None


# ------------------------------------------------------------------ reference arm (the CPU oracle)

def run_reference(args, s: wl.LayerShape):
    rank, _, world = dist_env()
    if rank != 0:
        return None
    orc = OracleRun(s, wl.make_inputs(s, seed=args.seed))
    # calibrate one batch, then size each step so the whole run stays within a few minutes
    t0 = time.perf_counter()
    orc.batch(orc.threads)
    per_batch = time.perf_counter() - t0
    budget = 150.0
    steps_total = max(1, args.steps + args.warmup)
    tokens_per_step = int(max(1, min(orc.threads, orc.threads * budget / steps_total / max(per_batch, 1e-9))))
    for _ in range(args.warmup):
        orc.batch(tokens_per_step)
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        done += orc.batch(tokens_per_step)
    el = time.perf_counter() - t0
    value = done / el
    cores = min(orc.threads, tokens_per_step)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_label(s), "T": s.T, "d": s.d, "f": s.f, "E": s.E, "k": s.k,
                       "alpha": s.alpha, "f_shared": s.f_shared, "seed": args.seed},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{tokens_per_step} tokens per step of {workload_label(s)} "
                                       f"(full routing + expert FFNs, fp64)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="decode64", choices=sorted(wl.FAMILIES))
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--alpha", type=float, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--sets", type=int, default=0, help="rotating weight sets (0: enough to exceed 3x L2)")
    ap.add_argument("--fp8", action="store_true", help="FP8 block-scaled expert GEMMs (moe_layer_forward_fp8)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    s = parse_workload(args)
    line = run_reference(args, s) if args.impl == "reference" else run_ours(args, s)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
