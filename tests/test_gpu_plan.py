"""The skew-aware scheduler's tile plan, read back from the workspace after the
layer forward (marked gpu).

For skewed routings (Dirichlet alpha from 0.02 to 10), E from 1 to 512, with
and without the shared expert, on both the one-CTA permutation (T*k <= 1024)
and the multi-CTA one, the plan built on the device from the live histogram
satisfies its invariants (tests/gpu_helpers.check_plan: one block per active
expert, heaviest first, every routed row covered exactly once by the tiles,
prefixes and widest tile consistent), routing is bit-exact on identical fp32
logits, and the layer output matches the oracle on a sample of tokens."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_02_b200 import moe
from grouped_gemm_02_b200 import workload as wl
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("T,E,k,alpha,fs", [
    (50, 1, 1, 1.0, 0),
    (1000, 8, 2, 0.1, 64),       # multi-CTA permutation, shared expert
    (100, 64, 8, 0.02, 0),       # extreme skew: most experts empty
    (300, 256, 8, 0.5, 128),
    (2000, 384, 8, 0.02, 0),     # many tokens on a handful of experts: several units per block
    (700, 512, 4, 10.0, 64),     # near-uniform over 512 experts
    (33, 512, 8, 1.0, 0),
    (17, 300, 8, 0.05, 192),     # one launch for both GEMMs, shared expert wider than one M-tile
])
def test_plan_from_live_histogram(T, E, k, alpha, fs):
    s = wl.LayerShape("plan", T=T, d=128, f=128, E=E, k=k, alpha=alpha, f_shared=fs)
    inp = wl.make_inputs(s, seed=T + E)
    d = {n: v.to(DEV) for n, v in inp.items()}
    ws = moe.new_workspace(s.T, s.d, s.f, s.E, s.k, s.f_shared)
    out = moe.moe_layer_forward(d["x"], d["Wg"], d["bias"], d["W1"], d["W3"], d["W2"], s.k, ws,
                                Ws1=d.get("Ws1"), Ws3=d.get("Ws3"), Ws2=d.get("Ws2"))
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    views = moe.workspace_views(ws, s.T, s.d, s.f, s.E, s.k, s.f_shared)
    what = f"plan T={T} E={E} k={k} alpha={alpha} fs={fs}"
    g_L, o_idx, o_w, counts, offsets = H.check_routing(views, s, what)
    H.check_layer_plan(views, s, counts, offsets, what)
    tokens = H.sample_tokens(o_idx, s.E, 24, seed=T)
    sh = {n: H.bits(inp[n]) for n in ("Ws1", "Ws3", "Ws2")} if fs else None
    ref = oracle.moe_ffn(H.bits(inp["x"][tokens]), H.bits(inp["W1"]), H.bits(inp["W3"]), H.bits(inp["W2"]),
                         o_idx[tokens], o_w[tokens], shared=sh)
    H.assert_close(out.float().cpu().numpy()[tokens], ref, what)


@pytest.mark.parametrize("pairs", [0, 1])
@pytest.mark.parametrize("T,E,k,alpha,fs", [(1000, 8, 2, 0.1, 64), (300, 256, 8, 0.5, 128), (17, 300, 8, 0.05, 192)])
def test_plan_for_single_ctas_and_pairs(T, E, k, alpha, fs, pairs):
    with H.policy(pairs=pairs):
        test_plan_from_live_histogram(T, E, k, alpha, fs)
