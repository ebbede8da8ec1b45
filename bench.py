#!/usr/bin/env python
"""Benchmark of the fused MoE layer forward on B200.

One step = one whole layer forward (router logits, top-k gating, histogram and
scan, permutation and row gather, gate/up grouped GEMM with SwiGLU, down
grouped GEMM, combine) over one batch of seeded synthetic tokens, through
moe_layer_forward.  Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--T ..] [--alpha ..] [--E ..] [--fp8 | --fp4] [--impl ours|reference]

With no --workload the line times the largest layer of the workload table
that fits one GPU: the DeepSeek-V3-shaped layer at T=16384 (d=7168, f=2048,
E=256 routed experts, top-8, Dirichlet alpha=0.5, plus the always-on shared
expert of f=2048), in bf16.  The same line carries a sub-record for the
decode-shaped layer (decode64: T=32, d=2048, f=1024, E=64, top-8, alpha=1),
the small-T, weight-streaming end of the table.

``--fp8`` times moe_layer_forward_fp8 (e4m3 expert weights with 128 x 128
block scales, quantised once before the timed region); ``--fp4`` times
moe_layer_forward_fp4 (e2m1 expert weights with 1 x 32 power-of-two scales,
e4m3 activations).

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
# The round figures the layer's targets are stated against: about 8 TB/s of HBM3e and
# 2.25 PFLOP/s of dense bf16 (4.5 fp8).  Fractions of these are reported beside the
# fractions of the measured peaks.
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
DTYPES = {"bf16": "bf16", "fp8": "fp8-e4m3 (fp32 accumulate)",
          "fp4": "fp4-e2m1 weights x fp8-e4m3 activations (fp32 accumulate)"}
HEADLINE = dict(workload="deepseek_v3", T=16384, alpha=0.5)
DECODE_SUB = dict(workload="decode64", T=32, alpha=1.0)
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "roofline_traffic.json")
KERNEL_SOURCES = ["grouped_gemm_02_b200/csrc/grouped_gemm.cuh", "grouped_gemm_02_b200/csrc/ptx.cuh",
                  "grouped_gemm_02_b200/csrc/common.cuh"]
FP8_KERNEL_SOURCES = ["grouped_gemm_02_b200/csrc/fp8.cuh", "grouped_gemm_02_b200/csrc/ptx.cuh",
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


def kernel_source_hash(fp8: bool = False) -> str:
    """Hash of the dominant kernel's sources (the FP8 kernel serves FP4 weights too)."""
    h = hashlib.sha256()
    for rel in (FP8_KERNEL_SOURCES if fp8 else KERNEL_SOURCES):
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()[:16]


def traffic_records():
    try:
        rec = json.load(open(PROFILE_TRAFFIC))
    except Exception:
        return []
    return rec if isinstance(rec, list) else [rec]


def committed_traffic(workload_name: str, kernel: str = None):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary,
    or None when absent, for another workload or kernel, or taken on older kernel
    source.  A record taken on a reduced case carries the full launch's bytes
    scaled from it (its "scaled_from" says how)."""
    fp8 = workload_name.endswith((" fp8", " fp4"))
    for rec in traffic_records():
        if rec.get("workload") != workload_name:
            continue
        if kernel is not None and rec.get("kernel_role", kernel) != kernel:
            continue
        if rec.get("source_sha") != kernel_source_hash(fp8):
            return None
        return rec.get("dram_bytes_per_launch")
    return None


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
    name = getattr(args, "workload", None)
    if name is None:
        name = HEADLINE["workload"]
        kw.update(T=HEADLINE["T"], alpha=HEADLINE["alpha"])
    if getattr(args, "T", None) is not None:
        kw["T"] = args.T
    if getattr(args, "alpha", None) is not None:
        kw["alpha"] = args.alpha
    if getattr(args, "E", None) is not None:
        kw["E"] = args.E
    return wl.shape(name, **kw)


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


def algorithmic(s: wl.LayerShape, counts: np.ndarray, fp8: bool = False, fmt: str = None):
    """Algorithmic bytes and flops of the layer and of the gate/up GEMM launch.

    bf16: 2 bytes per weight and activation.  FP8: 1 byte per weight and
    activation plus one fp32 scale per 128 x 128 weight block and per 1 x 128
    activation block.  FP4 (fmt="fp4"): half a byte per weight plus one scale
    byte per 32 weights; activations as FP8."""
    fmt = fmt or ("fp8" if fp8 else "bf16")
    active = int((counts > 0).sum())
    P = int(counts.sum())
    fs = s.f_shared
    wb = {"bf16": 2, "fp8": 1, "fp4": 0.5}[fmt]
    wsc = {"bf16": 0.0, "fp8": 4.0 / (128 * 128), "fp4": 1.0 / 32}[fmt]    # weight-scale bytes per weight
    asc = 0.0 if fmt == "bf16" else 4.0 / 128                                # activation-scale bytes per activation

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


def weight_sets(wbytes: int) -> int:
    """Rotating weight sets so that no step finds its weights in L2: enough sets to
    exceed 3x L2, and at least two unless one set alone is ten times L2."""
    want = max(1, math.ceil(3 * L2_BYTES / max(wbytes, 1)))
    if wbytes < 10 * L2_BYTES:
        want = max(want, 2)
    return want


def fmt_suffix(fmt):
    return "" if fmt in (None, "bf16") else " " + fmt


def weight_format(args):
    return "fp4" if getattr(args, "fp4", False) else "fp8" if args.fp8 else "bf16"


def kernel_roofline(s, alg, phase_ms, fp8, pk, pk_kind, fmt=None):
    """The dominant kernel's roofline: the single expert-GEMM launch when the
    library fuses both GEMMs, else the gate/up launch (2/3 of the flops and the
    largest launch of the layer)."""
    bw = pk["hbm_gbs"] * 1e9
    tc = pk["bf16_tflops_sustained"] * 1e12 * (2.0 if fp8 else 1.0)
    tc_nom = NOMINAL_PEAKS["bf16_tflops"] * 1e12 * (2.0 if fp8 else 1.0)
    bw_nom = NOMINAL_PEAKS["hbm_gbs"] * 1e9
    fused = gemm_fused(s.P, s.f)
    if fused:
        t = (phase_ms[2] + phase_ms[3]) / 1e3
        nbytes = alg["g1_bytes"] + alg["g2_bytes"]
        nflops = alg["g1_flops"] + alg["g2_flops"]
        role = "fused"
    else:
        t = phase_ms[2] / 1e3
        nbytes = alg["g1_bytes"]
        nflops = alg["g1_flops"]
        role = "gate_up"
    if nbytes / bw >= nflops / tc:
        roof = {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s"}
        roof["frac_nominal"] = nbytes / t / bw_nom
    else:
        roof = {"bound": "tensor", "achieved": nflops / t / 1e12, "peak": tc / 1e12, "unit": "TFLOP/s"}
        roof["frac_nominal"] = nflops / t / tc_nom
    roof["frac"] = roof["achieved"] / roof["peak"]
    name = ("grouped_gemm_fp8_kernel" if fp8 else "grouped_gemm_kernel") + ("<e2m1 weights>" if fmt == "fp4" else "")
    roof["kernel"] = f"{name}<{'fused gate/up + down' if fused else 'gate/up + SwiGLU'}>"
    roof["kernel_role"] = role
    roof["scope"] = "one expert-GEMM launch (the layer's fraction is layer_roofline.frac)"
    roof["algorithmic_bytes_per_launch"] = nbytes
    roof["algorithmic_flops_per_launch"] = nflops
    roof["launch_us"] = t * 1e6
    if roof["bound"] == "tensor":
        roof["peak_source"] = f"{pk_kind} ({'2 x sustained bf16 (the f8f6f4 MMA rate)' if fp8 else 'sustained bf16'})"
    else:
        roof["peak_source"] = f"{pk_kind} (HBM copy)"
    roof["nominal_peak"] = (tc_nom / 1e12 if roof["bound"] == "tensor" else bw_nom / 1e9)
    roof["traffic"] = committed_traffic(workload_label(s) + fmt_suffix(fmt), role)
    return roof


def layer_roofline(alg, ms_per_step, fp8, pk, pk_kind):
    """t_roof = max(active weight bytes / HBM, layer flops / tensor peak) over the layer time."""
    bw = pk["hbm_gbs"] * 1e9
    tc = pk["bf16_tflops_sustained"] * 1e12 * (2.0 if fp8 else 1.0)
    bw_nom = NOMINAL_PEAKS["hbm_gbs"] * 1e9
    tc_nom = NOMINAL_PEAKS["bf16_tflops"] * 1e12 * (2.0 if fp8 else 1.0)
    t_meas = ms_per_step / 1e3
    t_roof = max(alg["w_act"] / bw, alg["flops"] / tc)
    t_nom = max(alg["w_act"] / bw_nom, alg["flops"] / tc_nom)
    return {"bound": "hbm" if alg["w_act"] / bw >= alg["flops"] / tc else "tensor",
            "t_roof_us": t_roof * 1e6, "t_meas_us": t_meas * 1e6, "frac": t_roof / t_meas,
            "t_roof_nominal_us": t_nom * 1e6, "frac_nominal": t_nom / t_meas,
            "w_act_bytes": alg["w_act"], "flops": alg["flops"],
            "peak_source": f"{pk_kind}; nominal = {NOMINAL_PEAKS['hbm_gbs']:.0f} GB/s and "
                           f"{NOMINAL_PEAKS['bf16_tflops'] * (2 if fp8 else 1):.0f} TFLOP/s"}


# ------------------------------------------------------------------ CPU oracle timing

class OracleRun:
    """The CPU oracle on a token sample of a layer: per batch, fp64 router logits,
    top-k, the permutation and the per-token expert FFNs (+ shared expert).

    Host memory stays bounded: the sample is drawn from a pool of tokens whose k
    experts all lie in a small set of experts, and only those experts' weights
    are brought to the host (``expert_fn(e)`` returns W1[e], W3[e], W2[e] as
    host bf16 tensors, on first use).  Every token costs the same k expert FFNs
    of the same shape, so the oracle's time per token does not depend on which
    experts the pool holds."""

    def __init__(self, s: wl.LayerShape, x: torch.Tensor, Wg: torch.Tensor, bias: torch.Tensor,
                 expert_fn, shared=None, pool=None):
        import oracle
        self.oracle = oracle
        self.s = s
        self.threads = oracle.default_threads()
        self.pool = np.arange(x.shape[0]) if pool is None else np.asarray(pool, dtype=np.int64)
        self.x = wl.bf16_bits(x)
        self.Wg = wl.bf16_bits(Wg)
        self.bias = bias.numpy()
        self.expert_fn = expert_fn
        self.W1 = [None] * s.E
        self.W3 = [None] * s.E
        self.W2 = [None] * s.E
        self.shared = None
        if shared:
            self.shared = {n: wl.bf16_bits(shared[n]) for n in ("Ws1", "Ws3", "Ws2")}
        self.next = 0

    def load(self, experts):
        for e in sorted(set(int(v) for v in experts)):
            if self.W1[e] is None:
                w = self.expert_fn(e)
                self.W1[e], self.W3[e], self.W2[e] = (wl.bf16_bits(w[n]) for n in ("W1", "W3", "W2"))

    def batch(self, n: int) -> int:
        """Routing and expert FFNs of the next n pool tokens (wrapping around)."""
        o = self.oracle
        toks = self.pool[np.arange(self.next, self.next + n) % self.pool.size]
        self.next += n
        xs = np.ascontiguousarray(self.x[toks])
        L = o.router_logits(xs, self.Wg, self.bias).astype(np.float32)
        idx, w = o.topk(L, self.s.k)
        o.permutation(idx, self.s.E)
        self.load(idx.ravel())
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


def token_pool(idx: np.ndarray, E: int, want: int = 256, max_experts: int = 48):
    """Tokens whose k experts all lie among the most-used experts: grows the expert
    set (by count, descending) until `want` tokens qualify or it holds
    `max_experts`.  Returns (pool tokens, expert set); the pool may be small."""
    counts = np.bincount(idx.ravel(), minlength=E)
    order = np.argsort(-counts, kind="stable")
    m = min(E, max(idx.shape[1], 8))
    while True:
        allowed = np.zeros(E, dtype=bool)
        allowed[order[:m]] = True
        ok = np.nonzero(allowed[idx].all(axis=1))[0]
        if ok.size >= want or m >= min(E, max_experts):
            break
        m = min(E, m + 8)
    if ok.size == 0:                     # no token fits: take the first token's experts
        ok = np.array([0])
    return ok, order[:m]


def pool_note(pool, experts, s):
    return (f"tokens drawn from a pool of {pool.size} tokens whose {s.k} experts lie among the "
            f"{len(experts)} most-used experts (host copies of those experts only; every token costs the "
            f"same {s.k} expert FFNs{' + the shared expert' if s.f_shared else ''})")


# ------------------------------------------------------------------ GPU arm

def _make_step(moe, s, fp8, x, Wg, bias, sets, qsets, ws, out, R):
    def step(i, prof_events=None):
        if prof_events is not None:
            moe.moe_record_phase_events(prof_events)
        if fp8 == "fp4":
            moe.moe_layer_forward_fp4(x, Wg, bias, qsets[i % R], s.k, ws, out=out)
            return
        if fp8:
            moe.moe_layer_forward_fp8(x, Wg, bias, qsets[i % R], s.k, ws, out=out)
            return
        w = sets[i % R]
        moe.moe_layer_forward(x, Wg, bias, w["W1"], w["W3"], w["W2"], s.k, ws, Ws1=w.get("Ws1"),
                              Ws3=w.get("Ws3"), Ws2=w.get("Ws2"), out=out)
    return step


def measure_layer(s: wl.LayerShape, args, steps: int, warmup: int, world: int, dev, sampler=None,
                  phases_in_timed: bool = True, with_e2e: bool = True, sets_override: int = 0):
    """Times `steps` layer forwards after `warmup`; returns the measured record
    (and the host-side handles the CPU baseline needs)."""
    from grouped_gemm_02_b200 import moe
    stream = torch.cuda.current_stream()
    one = wl.make_weights(s, seed=args.seed, device=dev)
    wbytes = sum(t.numel() * t.element_size() for t in one.values())
    free, _ = torch.cuda.mem_get_info(dev)
    R = int(max(1, min(weight_sets(wbytes), sets_override or weight_sets(wbytes),
                       (free * 0.6) // max(wbytes, 1))))
    sets = [one] + [wl.make_weights(s, seed=args.seed + 1000 * (i + 1), device=dev) for i in range(R - 1)]
    base = wl.make_inputs(s, seed=args.seed, device=dev, weights=False)
    x, Wg, bias = base["x"], base["Wg"], base["bias"]
    out = torch.empty(s.T, s.d, dtype=torch.bfloat16, device=dev)
    qsets = None
    fmt = weight_format(args)
    if fmt != "bf16":
        # e4m3 weights with 128 x 128 block scales, or e2m1 with 1 x 32 scales
        # (quantised once, outside the timed region)
        quant = moe.quantize_layer_fp4 if fmt == "fp4" else moe.quantize_layer_fp8
        qsets = [quant(w) for w in sets]
        sets = None
        wbytes = sum(t.numel() * t.element_size() for t in qsets[0].values())
        # the quantised sets are smaller: add sets until they again exceed 3x L2
        free, _ = torch.cuda.mem_get_info(dev)
        want = int(max(1, min(weight_sets(wbytes), sets_override or weight_sets(wbytes),
                              (free * 0.5) // max(wbytes, 1))))
        for i in range(len(qsets), want):
            w = wl.make_weights(s, seed=args.seed + 1000 * (i + 1), device=dev)
            qsets.append(quant(w))
            del w
        R = len(qsets)
        ws = moe.new_workspace_fp8(s.T, s.d, s.f, s.E, s.k, s.f_shared, device=dev)
        torch.cuda.empty_cache()
    else:
        ws = moe.new_workspace(s.T, s.d, s.f, s.E, s.k, s.f_shared, device=dev)
    step = _make_step(moe, s, "fp4" if fmt == "fp4" else fmt == "fp8", x, Wg, bias, sets, qsets, ws, out, R)

    for i in range(warmup):
        step(i)
    if sampler:
        sampler.wait_first_sample()
    torch.cuda.synchronize()
    if moe.moe_get_device_error(ws) != 0:
        raise RuntimeError("device error after warm-up")
    if phases_in_timed:
        # events between the phases keep the next kernel from starting early (no
        # programmatic overlap), a cost that only long layers can absorb: layers
        # under 1 ms get their phase split from a second pass instead
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(3):
            step(i)
        b.record(stream)
        torch.cuda.synchronize()
        phases_in_timed = a.elapsed_time(b) / 3 >= 1.0

    # CUDA events for the per-phase split: inside the timed region itself (each
    # step records six events on the layer's stream), or in a second pass
    n_ev = steps if phases_in_timed else min(steps, 500)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(n_ev)]
    for row in ev:          # torch creates the CUDA event on its first record
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    n0 = moe.moe_launch_counter()
    start.record(stream)
    for i in range(steps):
        step(i, ev[i] if phases_in_timed else None)
    end.record(stream)
    torch.cuda.synchronize()
    launches = moe.moe_launch_counter() - n0
    if world > 1:
        dist.barrier()
    ms = start.elapsed_time(end)
    ms_max = reduce_max(ms, world, dev)
    if moe.moe_get_device_error(ws) != 0:
        raise RuntimeError("device error in the timed region")
    if not phases_in_timed:
        # events between phases keep the next kernel from starting early, so
        # these phase times are upper bounds
        for i in range(n_ev):
            step(i, ev[i])
        torch.cuda.synchronize()
    phase = np.array([[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(5)] for i in range(n_ev)])
    phase_ms = phase.mean(axis=0)

    e2e = None
    if with_e2e:
        # end to end through the C ABI: pinned host x -> device, layer, device out -> pinned host
        x_host = x.cpu().pin_memory()
        out_host = torch.empty(s.T, s.d, dtype=torch.bfloat16).pin_memory()
        for i in range(min(3, warmup)):
            x.copy_(x_host, non_blocking=True)
            step(i)
            out_host.copy_(out, non_blocking=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for i in range(steps):
            x.copy_(x_host, non_blocking=True)
            step(i)
            out_host.copy_(out, non_blocking=True)
        s1.record(stream)
        torch.cuda.synchronize()
        e_ms = reduce_max(s0.elapsed_time(s1), world, dev)
        e2e = {"value": s.T * steps * world / (e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": s.T * s.d * 2, "d2h_bytes_per_step": s.T * s.d * 2,
               "ms_per_step": e_ms / steps}

    if fmt != "bf16":
        views = moe.workspace_views_fp8(ws, s.T, s.d, s.f, s.E, s.k, s.f_shared)
    else:
        views = moe.workspace_views(ws, s.T, s.d, s.f, s.E, s.k, s.f_shared)
    counts = views["counts"].cpu().numpy()
    idx = views["topk_idx"].cpu().numpy()
    alg = algorithmic(s, counts, fmt=fmt)
    lowp = fmt != "bf16"
    pk, pk_kind = peaks()
    ms_per_step = ms_max / steps
    rec = {"ms_per_step": ms_per_step, "ms_total": ms_max, "launches": int(launches), "phase_ms": phase_ms,
           "phases_in_timed": phases_in_timed, "counts": counts, "alg": alg, "e2e": e2e, "R": R,
           "wbytes": wbytes,
           "roofline": kernel_roofline(s, alg, phase_ms, lowp, pk, pk_kind, fmt),
           "layer_roofline": layer_roofline(alg, ms_per_step, lowp, pk, pk_kind)}
    host = None
    if not lowp:
        host = {"x": x, "Wg": Wg, "bias": bias, "weights": one, "idx": idx}
    return rec, host


def sub_record(s, rec, fmt):
    """The compact form of a second workload measured in the same run."""
    return {"workload": workload_label(s) + fmt_suffix(fmt), "value": s.T / (rec["ms_per_step"] / 1e3),
            "unit": UNIT, "us_per_layer": rec["ms_per_step"] * 1e3, "steps": rec["steps"],
            "layer_roofline": rec["layer_roofline"], "roofline": rec["roofline"],
            "histogram": stats.histogram_stats(rec["counts"]),
            "phase_us": {n: float(v * 1e3) for n, v in
                         zip(("route", "permute", "gemm_gate_up", "gemm_down", "combine"), rec["phase_ms"])},
            "phase_note": ("per-phase means from CUDA events recorded between the phases inside the timed region"
                           if rec.get("phases_in_timed") else
                           "per-phase means from a second pass with CUDA events between phases")}


def cpu_baseline(s, host, budget_s):
    """The oracle, as it stands, on the host cores for about budget_s seconds."""
    pool, experts = token_pool(host["idx"], s.E)
    W = host["weights"]
    shared = {n: W[n].cpu() for n in ("Ws1", "Ws3", "Ws2")} if s.f_shared else None
    orc = OracleRun(s, host["x"].cpu(), host["Wg"].cpu(), host["bias"].cpu(),
                    lambda e: {n: W[n][e].cpu() for n in ("W1", "W3", "W2")}, shared=shared, pool=pool)
    orc.load(experts)
    toks, secs, cores = orc.timed(budget_s, orc.threads)
    return {"value": toks / secs, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{toks} tokens of {workload_label(s)} (fp64 router logits, top-k, permutation and expert "
                      f"FFNs per token), {secs:.1f} s on {cores} host threads; {pool_note(pool, experts, s)}"}


def run_ours(args, s: wl.LayerShape):
    rank, local_rank, world = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    torch.cuda.set_device(dev)

    sampler = ClockSampler([torch.cuda.current_device()]) if rank == 0 else None
    rec, host = measure_layer(s, args, args.steps, args.warmup, world, dev, sampler=sampler,
                              phases_in_timed=True, with_e2e=not args.no_e2e, sets_override=args.sets)
    clocks = sampler.stop() if sampler else None
    K = args.steps
    ms_per_step = rec["ms_per_step"]
    line = {"metric": METRIC, "value": s.T * K * world / (rec["ms_total"] / 1e3), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPES[weight_format(args)],
            "data": "synthetic (seeded; Dirichlet routing skew; random-init weights of the layer's shape)",
            "config": {"workload": workload_label(s) + fmt_suffix(weight_format(args)), "T": s.T, "d": s.d, "f": s.f,
                       "E": s.E, "k": s.k,
                       "alpha": s.alpha, "f_shared": s.f_shared, "seed": args.seed,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": f"inputs larger than L2: {rec['R']} rotating weight set(s) of "
                             f"{rec['wbytes'] / 2**20:.0f} MiB",
                       "histogram": stats.histogram_stats(rec["counts"]),
                       "us_per_layer": ms_per_step * 1e3,
                       "phase_note": ("per-phase means from CUDA events recorded between the phases inside the "
                                      "timed region" if rec["phases_in_timed"] else
                                      "per-phase means from a second pass with CUDA events between phases"),
                       "phase_us": {n: float(v * 1e3) for n, v in
                                    zip(("route", "permute", "gemm_gate_up", "gemm_down", "combine"),
                                        rec["phase_ms"])}},
            "roofline": rec["roofline"], "layer_roofline": rec["layer_roofline"], "e2e": rec["e2e"],
            "gpu_launches": rec["launches"], "clocks": clocks}
    if not args.no_sub and weight_format(args) == "bf16" and args.lowp_steps > 0:
        # the same layer with FP8 and with FP4 expert weights (quantised outside the timed region)
        import copy
        for fmt in ("fp8", "fp4"):
            a2 = copy.copy(args)
            a2.fp8, a2.fp4 = fmt == "fp8", fmt == "fp4"
            lrec, _ = measure_layer(s, a2, args.lowp_steps, max(3, args.warmup), world, dev, phases_in_timed=True,
                                    with_e2e=False)
            lrec["steps"] = args.lowp_steps
            line[fmt] = sub_record(s, lrec, fmt)
            torch.cuda.empty_cache()
    if not args.no_sub and s.name != DECODE_SUB["workload"]:
        ds = wl.shape(DECODE_SUB["workload"], T=DECODE_SUB["T"], alpha=DECODE_SUB["alpha"])
        drec, _ = measure_layer(ds, args, args.sub_steps, 20, world, dev, phases_in_timed=False, with_e2e=False)
        drec["steps"] = args.sub_steps
        line["decode64"] = sub_record(ds, drec, weight_format(args))
    if rank == 0 and world == 1 and not args.no_cpu_baseline and host is not None:
        line["cpu_baseline"] = cpu_baseline(s, host, args.cpu_budget)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return line if rank == 0 else None


# ------------------------------------------------------------------ reference arm (the CPU oracle)

def reference_setup(s: wl.LayerShape, seed: int):
    """Host inputs for the oracle's timed sample: x, Wg and bias as the workload
    draws them, a token pool picked from a float32 routing of every token, and
    the routed experts drawn one by one on first use."""
    inp = wl.make_inputs(s, seed=seed, weights=False)
    # the pool selection only picks which tokens to sample; the timed oracle routes them itself
    L = inp["x"].float() @ inp["Wg"].float().T + inp["bias"]
    idx = torch.topk(L, s.k, dim=1).indices.numpy()
    pool, experts = token_pool(idx, s.E)
    shared = wl.make_shared_weights(s, seed) if s.f_shared else None
    orc = OracleRun(s, inp["x"], inp["Wg"], inp["bias"], lambda e: wl.make_expert_weights(s, seed, e),
                    shared=shared, pool=pool)
    orc.load(experts)
    return orc, pool, experts


def run_reference(args, s: wl.LayerShape):
    rank, _, world = dist_env()
    if rank != 0:
        return None
    orc, pool, experts = reference_setup(s, args.seed)
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
                             "sample": f"{tokens_per_step} tokens per step of {workload_label(s)} (fp64 router "
                                       f"logits, top-k, permutation and expert FFNs); {pool_note(pool, experts, s)}"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def build_parser():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=None, choices=sorted(wl.FAMILIES),
                    help="layer family (default: deepseek_v3 at T=16384, alpha=0.5)")
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--alpha", type=float, default=None)
    ap.add_argument("--E", type=int, default=None, help="override the number of routed experts (profiling cases)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--sets", type=int, default=0, help="rotating weight sets (0: enough to exceed 3x L2)")
    fmt = ap.add_mutually_exclusive_group()
    fmt.add_argument("--fp8", action="store_true", help="FP8 block-scaled expert GEMMs (moe_layer_forward_fp8)")
    fmt.add_argument("--fp4", action="store_true", help="FP4 expert weights, FP8 activations (moe_layer_forward_fp4)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="skip the decode64 sub-record")
    ap.add_argument("--sub-steps", type=int, default=2000, help="timed steps of the decode64 sub-record")
    ap.add_argument("--lowp-steps", type=int, default=20,
                    help="timed steps of the FP8 and FP4 sub-records of a bf16 run (0: none)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    return ap


def main(argv=None):
    args = build_parser().parse_args(argv)
    args.warmup = max(3, args.warmup)
    s = parse_workload(args)
    line = run_reference(args, s) if args.impl == "reference" else run_ours(args, s)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
