#!/usr/bin/env python
"""Offline tuning of the tile tables (csrc/tile_table.h) on a B200.

The histogram-matched tile policy (Decoding the Skew, abstract: a kernel
configuration chosen on the GPU by matching the live routing histogram to
distributions tuned offline, the skew produced by Dirichlet reverse modelling)
keeps one tile cap per histogram class; the static token-bucket policy it is
measured against keeps one tile width per bucket of T.  This script measures
both on the seeded Dirichlet workloads of the layer table and writes the
tables:

    python -m grouped_gemm_02_b200.tune_tiles measure  --out tile_sweep.json   (GPU)
    python -m grouped_gemm_02_b200.tune_tiles write    --sweep tile_sweep.json (host)
    python -m grouped_gemm_02_b200.tune_tiles ablation --out ablation.json     (GPU, after a rebuild)

`measure` times every workload under each forced cap (widths following the
live counts) and each forced token-bucket width, and records each workload's
histogram class as the plan step computes it.  `write` picks, per class, the
cap with the lowest geometric-mean layer time over that class's workloads and,
per T bucket, the width with the lowest geometric-mean time over that bucket's
workloads (every alpha), and writes csrc/tile_table.h.  `ablation` times the
built library's two policies against each other.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
TABLE_H = os.path.join(HERE, "csrc", "tile_table.h")
CAPS = (64, 128, 256)
WIDTHS = (16, 32, 64, 128, 256)
N_CLASSES, N_BUCKETS = 15, 6
L2_BYTES = 126 * 1024 * 1024


def sweep_shapes():
    from . import workload as wl
    out = []
    for name, points in wl.SWEEP.items():
        if name == "tiny":
            continue
        for kw in points:
            out.append(wl.shape(name, **kw))
    return out


def token_bucket(T: int) -> int:
    return 0 if T <= 16 else 1 if T <= 64 else 2 if T <= 256 else 3 if T <= 1024 else 4 if T <= 4096 else 5


def _time_layer(moe, torch, s, sets, base, ws, out, steps, warmup):
    stream = torch.cuda.current_stream()
    R = len(sets)

    def step(i):
        w = sets[i % R]
        moe.moe_layer_forward(base["x"], base["Wg"], base["bias"], w["W1"], w["W3"], w["W2"], s.k, ws,
                              Ws1=w.get("Ws1"), Ws3=w.get("Ws3"), Ws2=w.get("Ws2"), out=out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    if moe.moe_get_device_error(ws) != 0:
        raise RuntimeError(f"device error while timing {s}")
    return a.elapsed_time(b) * 1e3 / steps


def _plan_header(moe, ws, s):
    v = moe.workspace_views(ws, s.T, s.d, s.f, s.E, s.k, s.f_shared)
    p = v["plan"].cpu().numpy()
    return {"cls": int(p[6]), "cap": int(p[7]), "pair": int(p[5])}


def _setup(moe, wl, torch, s, seed=0):
    dev = torch.device("cuda")
    one = wl.make_weights(s, seed=seed, device=dev)
    wbytes = sum(t.numel() * t.element_size() for t in one.values())
    R = max(1, math.ceil(3 * L2_BYTES / wbytes)) if wbytes < 10 * L2_BYTES else 1
    sets = [one] + [wl.make_weights(s, seed=seed + 1000 * (i + 1), device=dev) for i in range(R - 1)]
    base = wl.make_inputs(s, seed=seed, device=dev, weights=False)
    ws = moe.new_workspace(s.T, s.d, s.f, s.E, s.k, s.f_shared, device=dev)
    out = torch.empty(s.T, s.d, dtype=torch.bfloat16, device=dev)
    return sets, base, ws, out


def _steps_for(us: float):
    return max(10, min(2000, int(40000 / max(us, 1.0))))


def measure(args):
    import torch
    from . import moe, workload as wl
    torch.cuda.set_device(0)
    rec = []
    for s in sweep_shapes():
        sets, base, ws, out = _setup(moe, wl, torch, s)
        moe.moe_set_policy(moe.POLICY_TILES, 0)
        moe.moe_set_policy(moe.POLICY_TILE_CAP, -1)
        t0 = _time_layer(moe, torch, s, sets, base, ws, out, 5, 3)
        hdr = _plan_header(moe, ws, s)
        steps = _steps_for(t0)
        row = {"workload": f"{s.name} T={s.T} alpha={s.alpha:g}", "T": s.T, "bucket": token_bucket(s.T),
               "cls": hdr["cls"], "cap_us": {}, "width_us": {}}
        for cap in CAPS:
            moe.moe_set_policy(moe.POLICY_TILES, 0)
            moe.moe_set_policy(moe.POLICY_TILE_CAP, cap)
            row["cap_us"][cap] = _time_layer(moe, torch, s, sets, base, ws, out, steps, 3)
        for w in WIDTHS:
            moe.moe_set_policy(moe.POLICY_TILES, 1)
            moe.moe_set_policy(moe.POLICY_TILE_CAP, w)
            row["width_us"][w] = _time_layer(moe, torch, s, sets, base, ws, out, steps, 3)
        moe.moe_set_policy(moe.POLICY_TILES, -1)
        moe.moe_set_policy(moe.POLICY_TILE_CAP, -1)
        print(json.dumps(row), flush=True)
        rec.append(row)
        del sets, base, ws, out
        torch.cuda.empty_cache()
    json.dump({"device": torch.cuda.get_device_name(0), "rows": rec}, open(args.out, "w"), indent=1)


def _best(rows, key, options):
    if not rows:
        return None
    score = {o: sum(math.log(r[key][str(o)] if str(o) in r[key] else r[key][o]) for r in rows) for o in options}
    return min(options, key=lambda o: (score[o], -o))


def write(args):
    data = json.load(open(args.sweep))
    rows = data["rows"]
    caps = [256] * N_CLASSES
    for c in range(N_CLASSES):
        b = _best([r for r in rows if r["cls"] == c], "cap_us", CAPS)
        if b is not None:
            caps[c] = b
    default_w = [16, 32, 64, 128, 256, 256]
    widths = list(default_w)
    for t in range(N_BUCKETS):
        b = _best([r for r in rows if r["bucket"] == t], "width_us", WIDTHS)
        if b is not None:
            widths[t] = b
    tuned_c = sorted({r["cls"] for r in rows})
    tuned_b = sorted({r["bucket"] for r in rows})
    src = f"""// tile_table.h -- written by grouped_gemm_02_b200/tune_tiles.py; do not edit by hand.
//
// Tuned on {data.get('device', 'a B200')} over {len(rows)} seeded Dirichlet workloads of the layer table
// (measurement record: {os.path.basename(args.sweep)}).  Classes measured: {tuned_c}; the
// others keep the widest tiles.  Token buckets measured: {tuned_b}.
#pragma once

// Largest tile width (tokens) per histogram class (tile_class in schedule.h).
#define MOE_TILE_CAP_TABLE {{{', '.join(str(v) for v in caps)}}}

// Fixed tile width per token bucket (token_bucket in schedule.h) of the static policy.
#define MOE_TOKEN_BUCKET_WIDTH {{{', '.join(str(v) for v in widths)}}}
"""
    open(args.table, "w").write(src)
    print(src)


def ablation(args):
    import torch
    from . import moe, workload as wl
    torch.cuda.set_device(0)
    rows = []
    for s in sweep_shapes():
        sets, base, ws, out = _setup(moe, wl, torch, s)
        moe.moe_set_policy(moe.POLICY_TILE_CAP, -1)
        res = {}
        for name, v in (("matched", 0), ("bucket", 1), ("matched2", 0), ("bucket2", 1)):
            moe.moe_set_policy(moe.POLICY_TILES, v)
            t0 = _time_layer(moe, torch, s, sets, base, ws, out, 5, 3)
            res[name] = _time_layer(moe, torch, s, sets, base, ws, out, _steps_for(t0), 3)
            if name == "matched":
                res["plan"] = _plan_header(moe, ws, s)
        moe.moe_set_policy(moe.POLICY_TILES, -1)
        m = min(res["matched"], res["matched2"])
        b = min(res["bucket"], res["bucket2"])
        row = {"workload": f"{s.name} T={s.T} alpha={s.alpha:g}", "matched_us": m, "bucket_us": b,
               "speedup": b / m, "cls": res["plan"]["cls"], "cap": res["plan"]["cap"]}
        print(json.dumps(row), flush=True)
        rows.append(row)
        del sets, base, ws, out
        torch.cuda.empty_cache()
    geo = math.exp(sum(math.log(r["speedup"]) for r in rows) / len(rows))
    fam = {}
    for r in rows:
        fam.setdefault(r["workload"].split()[0], []).append(r["speedup"])
    summary = {"geomean_speedup": geo,
               "per_family": {k: math.exp(sum(math.log(v) for v in vs) / len(vs)) for k, vs in fam.items()}}
    print(json.dumps(summary))
    json.dump({"device": torch.cuda.get_device_name(0), "rows": rows, "summary": summary}, open(args.out, "w"),
              indent=1)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("what", choices=("measure", "write", "ablation"))
    ap.add_argument("--out", default="tile_sweep.json")
    ap.add_argument("--sweep", default="tile_sweep.json")
    ap.add_argument("--table", default=TABLE_H)
    args = ap.parse_args(argv)
    {"measure": measure, "write": write, "ablation": ablation}[args.what](args)


if __name__ == "__main__":
    sys.path.insert(0, os.path.dirname(HERE))
    main()
