"""Host-side logic of bench.py: rank environment, max-over-ranks timing across
two gloo processes, algorithmic byte counts, the traffic record's source check,
and clock-sample parsing."""

import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
from grouped_gemm_02_b200 import workload as wl


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    r, lr, w = bench.dist_env()
    got = bench.reduce_max(10.0 + 5.0 * rank, w)
    dist.barrier()
    dist.destroy_process_group()
    q.put((r, lr, w, got))


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 0, 2, 15.0), (1, 1, 2, 15.0)]


def test_dist_env_defaults(monkeypatch):
    for v in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(v, raising=False)
    assert bench.dist_env() == (0, 0, 1)
    assert bench.reduce_max(3.5, 1) == 3.5


def test_algorithmic_counts():
    s = wl.DECODE64
    counts = np.zeros(s.E, dtype=np.int64)
    counts[:4] = [100, 100, 50, 6]
    a = bench.algorithmic(s, counts)
    assert a["active"] == 4 and a["pairs"] == 256
    assert a["w_act"] == 4 * 3 * s.d * s.f * 2
    assert a["flops"] == 6.0 * 256 * s.d * s.f
    assert a["g1_bytes"] == 4 * 2 * s.f * s.d * 2 + 256 * s.d * 2 + 256 * s.f * 2
    assert a["g2_bytes"] == 4 * s.d * s.f * 2 + 256 * s.f * 2 + 256 * s.d * 2
    assert a["g1_flops"] + a["g2_flops"] == a["flops"]
    sh = wl.DEEPSEEK_V3.with_(T=8)
    c2 = np.zeros(sh.E, dtype=np.int64)
    c2[0] = 64
    b = bench.algorithmic(sh, c2)
    assert b["w_act"] == (1 * 3 + 3) * sh.d * sh.f * 2          # f_shared == f here


def test_traffic_record_tied_to_kernel_source(tmp_path, monkeypatch):
    rec = {"workload": "w", "source_sha": bench.kernel_source_hash(), "dram_bytes_per_launch": 123}
    p = tmp_path / "t.json"
    p.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(p))
    assert bench.committed_traffic("w") == 123
    assert bench.committed_traffic("other") is None
    assert bench.committed_traffic("w fp8") is None          # another kernel's record
    rec["source_sha"] = "0" * 16
    p.write_text(json.dumps(rec))
    assert bench.committed_traffic("w") is None


def test_clock_sampler_parse(tmp_path):
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.path = str(tmp_path / "c.csv")
    lines = ["0, 1965, 1965, 700.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
             "0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "0, 1700, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active"]
    open(cs.path, "w").write("\n".join(lines) + "\n")

    class P:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    cs.proc = P()
    r = cs.stop()
    assert r["sm_mhz"] == 1800.0 and r["sm_max_mhz"] == 1965.0 and r["reasons"] == ["sw_power_cap"]


def test_workload_label_and_parse():
    class A:
        workload, T, alpha = "deepseek_v3", 64, 0.05
    s = bench.parse_workload(A)
    assert s.T == 64 and s.alpha == 0.05 and s.f_shared == 2048
    assert "shared_f=2048" in bench.workload_label(s)


def test_gemm_launch_rule(monkeypatch):
    monkeypatch.delenv("MOE_GEMM_SPLIT", raising=False)
    assert bench.gemm_fused(256, 1024) and bench.gemm_fused(64, 2048)
    assert not bench.gemm_fused(512, 2048) and not bench.gemm_fused(32, 14336)
    monkeypatch.setenv("MOE_GEMM_SPLIT", "1")
    assert not bench.gemm_fused(256, 1024)
    monkeypatch.setenv("MOE_GEMM_SPLIT", "0")
    assert bench.gemm_fused(32768, 14336)


def test_default_workload_is_the_largest_single_gpu_layer():
    args = bench.build_parser().parse_args([])
    s = bench.parse_workload(args)
    assert (s.name, s.T, s.d, s.f, s.E, s.k, s.alpha, s.f_shared) == ("deepseek_v3", 16384, 7168, 2048, 256, 8, 0.5,
                                                                       2048)
    args = bench.build_parser().parse_args(["--workload", "deepseek_v3", "--T", "1024", "--E", "16"])
    s = bench.parse_workload(args)
    assert (s.T, s.E, s.alpha) == (1024, 16, 0.5)


def test_weight_sets_exceed_l2():
    L2 = bench.L2_BYTES
    assert bench.weight_sets(22 * 2**30) == 1                  # one set is far larger than L2
    assert bench.weight_sets(805 * 2**20) == 2                 # decode64: at least two sets
    assert bench.weight_sets(6 * 2**20) * 6 * 2**20 >= 3 * L2   # the tiny layer: enough sets for 3x L2


def test_token_pool_keeps_experts_bounded():
    idx = wl.random_routing(4096, 256, 8, 0.5, seed=3).numpy()
    pool, experts = bench.token_pool(idx, 256, want=64, max_experts=48)
    assert len(experts) <= 48 and pool.size >= 1
    allowed = np.zeros(256, dtype=bool)
    allowed[experts] = True
    assert allowed[idx[pool]].all()
    # a pool that cannot be filled still returns at least one token
    pool, experts = bench.token_pool(idx, 256, want=10**6, max_experts=16)
    assert pool.size >= 1 and len(experts) <= 16


def test_layer_roofline_fractions():
    pk = {"hbm_gbs": 6531.0, "bf16_tflops": 1668.8, "bf16_tflops_sustained": 1403.8}
    alg = {"w_act": 6.531e9, "flops": 1e9}
    r = bench.layer_roofline(alg, 2.0, False, pk, "measured")           # 1 ms roofline over 2 ms
    assert r["bound"] == "hbm" and abs(r["frac"] - 0.5) < 1e-12
    assert abs(r["frac_nominal"] - 6.531e9 / 8e12 / 2e-3) < 1e-12
    alg = {"w_act": 1e6, "flops": 1.4038e12}
    r = bench.layer_roofline(alg, 4.0, False, pk, "measured")
    assert r["bound"] == "tensor" and abs(r["frac"] - 0.25) < 1e-12
    assert abs(r["frac_nominal"] - 1.4038e12 / 2.25e15 / 4e-3) < 1e-12


def test_reference_sample_on_a_small_layer():
    s = wl.TINY.with_(T=32)
    orc, pool, experts = bench.reference_setup(s, seed=0)
    assert pool.size >= 1
    assert orc.batch(4) == 4
    assert all(orc.W1[e] is not None for e in experts)


def test_tile_table_writer(tmp_path):
    """tune_tiles.py write: the best cap per measured class and width per token bucket."""
    from grouped_gemm_02_b200 import tune_tiles
    rows = [
        {"workload": "a", "T": 8, "bucket": 0, "cls": 2, "cap_us": {"64": 5.0, "128": 4.0, "256": 4.5},
         "width_us": {"16": 9.0, "32": 8.0, "64": 8.5, "128": 9.5, "256": 9.9}},
        {"workload": "b", "T": 10, "bucket": 0, "cls": 2, "cap_us": {"64": 5.0, "128": 4.2, "256": 4.1},
         "width_us": {"16": 9.0, "32": 8.0, "64": 8.5, "128": 9.5, "256": 9.9}},
        {"workload": "c", "T": 5000, "bucket": 5, "cls": 13, "cap_us": {"64": 9.0, "128": 8.0, "256": 7.0},
         "width_us": {"16": 20.0, "32": 15.0, "64": 12.0, "128": 11.0, "256": 10.0}},
    ]
    sweep = tmp_path / "s.json"
    sweep.write_text(json.dumps({"device": "test", "rows": rows}))
    table = tmp_path / "t.h"
    tune_tiles.main(["write", "--sweep", str(sweep), "--table", str(table)])
    import re
    src = table.read_text()
    caps = [int(v) for v in re.search(r"MOE_TILE_CAP_TABLE \{([^}]*)\}", src).group(1).split(",")]
    widths = [int(v) for v in re.search(r"MOE_TOKEN_BUCKET_WIDTH \{([^}]*)\}", src).group(1).split(",")]
    assert caps[2] == 128 and caps[13] == 256 and caps[0] == 256 and len(caps) == 15
    assert widths[0] == 32 and widths[5] == 256 and widths[3] == 128 and len(widths) == 6


def test_algorithmic_bytes_per_weight_format():
    """Weight bytes per element: bf16 2, FP8 1 + a 4-byte scale per 128 x 128 block, FP4 half a byte + a scale
    byte per 32; the flops do not depend on the format."""
    s = wl.LayerShape("a", T=4, d=128, f=128, E=3, k=2, alpha=1.0)
    counts = np.array([5, 3, 0])
    per = {"bf16": 2.0, "fp8": 1.0 + 4.0 / (128 * 128), "fp4": 0.5 + 1.0 / 32}
    flops = None
    for fmt, b in per.items():
        a = bench.algorithmic(s, counts, fmt=fmt)
        assert a["active"] == 2 and a["pairs"] == 8
        assert a["w_act"] == pytest.approx(2 * 3 * 128 * 128 * b)
        flops = flops or a["flops"]
        assert a["flops"] == flops == 6.0 * 8 * 128 * 128
    assert bench.algorithmic(s, counts, fp8=True) == bench.algorithmic(s, counts, fmt="fp8")


def test_weight_format_and_traffic_key(tmp_path, monkeypatch):
    """--fp4 selects the FP4 weights; an FP4 workload's traffic record is keyed to the FP8 kernel's source."""
    args = bench.build_parser().parse_args(["--fp4"])
    assert bench.weight_format(args) == "fp4" and bench.fmt_suffix("fp4") == " fp4"
    assert bench.weight_format(bench.build_parser().parse_args([])) == "bf16"
    with pytest.raises(SystemExit):
        bench.build_parser().parse_args(["--fp4", "--fp8"])
    rec = [{"workload": "w fp4", "kernel_role": "gate_up", "source_sha": bench.kernel_source_hash(True),
            "dram_bytes_per_launch": 7}]
    p = tmp_path / "t.json"
    p.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(p))
    assert bench.committed_traffic("w fp4", "gate_up") == 7
    assert bench.committed_traffic("w fp4", "down") is None
