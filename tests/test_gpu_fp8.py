"""FP8 block-scaled path against the CPU oracle, through the C ABI (marked gpu).

Quantised codes and scales are integer / power-of-two results of the same
definition on both sides: bit-exact.  Layer outputs: the FP8 tolerance,
|y - y_ref| <= 1e-2 + 3e-2 |y_ref| per element and relative Frobenius error
<= 3e-2 (h is requantised from fp32 on the GPU and from fp64 in the oracle, so
a few h codes may differ by one step; the tolerance absorbs that).
"""

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
FP8_RTOL = 3e-2


def _values(R, C, seed):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(R, C, generator=gen) * torch.logspace(-4, 4, R)[:, None]
    x[0, :] = 0.0                                    # an all-zero block: scale 1
    x[1, 5] = 3.0e38                                 # a huge value in one block
    x[2, :128] = torch.arange(128) * 448.0 / 127    # amax exactly 448
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("R,C", [(7, 128), (33, 384), (300, 2048)])
def test_quantize_rows_bit_exact(R, C):
    x = _values(R, C, seed=R)
    q, sc = moe.moe_quantize_fp8_rows(x.to(DEV))
    rq, rs = oracle.quantize_rows_fp8(H.bits(x))
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(sc.cpu().numpy().astype(np.float64), rs)


@pytest.mark.parametrize("R,C", [(128, 128), (256, 384), (1024, 2048)])
def test_quantize_blocks_bit_exact(R, C):
    W = _values(R, C, seed=C)
    q, sc = moe.moe_quantize_fp8_blocks(W.to(DEV))
    rq, rs = oracle.quantize_blocks_fp8(H.bits(W))
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(sc.cpu().numpy().astype(np.float64), rs)


def _oracle_weights(W: torch.Tensor, experts):
    """Oracle quantisation of the listed experts' matrices (per expert: codes, scales)."""
    codes, scales = [None] * W.shape[0], [None] * W.shape[0]
    for e in sorted(set(int(v) for v in experts)):
        codes[e], scales[e] = oracle.quantize_blocks_fp8(H.bits(W[e]))
    return codes, scales


def _fp8_layer_check(s: wl.LayerShape, seed: int, n_sample=None, device_inputs=False):
    inp = wl.make_inputs(s, seed=seed, device=DEV if device_inputs else "cpu")
    d_inp = {n: v.to(DEV) for n, v in inp.items()}
    Q = moe.quantize_layer_fp8(d_inp)
    ws = moe.new_workspace_fp8(s.T, s.d, s.f, s.E, s.k, s.f_shared)
    out = moe.moe_layer_forward_fp8(d_inp["x"], d_inp["Wg"], d_inp["bias"], Q, s.k, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    views = moe.workspace_views_fp8(ws, s.T, s.d, s.f, s.E, s.k, s.f_shared)
    g_idx = views["topk_idx"].cpu().numpy()
    g_L = views["logits"].cpu().numpy()
    x_h = inp["x"].cpu()
    tokens = np.arange(s.T) if n_sample is None else H.sample_tokens(g_idx, s.E, n_sample, seed)
    # activations: GPU codes and scales equal the oracle's
    xq, sx = oracle.quantize_rows_fp8(H.bits(x_h[tokens]))
    assert np.array_equal(views["x8"].cpu().numpy()[tokens], xq)
    assert np.array_equal(views["sx"].cpu().numpy()[tokens].astype(np.float64), sx)
    # routing (bf16 router, as in the bf16 layer)
    L64 = oracle.router_logits(H.bits(x_h[tokens]), H.bits(inp["Wg"].cpu()), inp["bias"].cpu().numpy())
    L32 = L64.astype(np.float32)
    o_idx, o_w = oracle.topk(L32, s.k)
    dL = np.abs(g_L[tokens].astype(np.float64) - L64)
    delta = 4 * dL.max(axis=1) + 1e-6 * (1 + np.abs(L64).max(axis=1))
    clear = H.clear_margin_tokens(L32.astype(np.float64), s.k, delta)
    assert np.array_equal(g_idx[tokens][clear], o_idx[clear])
    keep = clear
    used = np.unique(o_idx[keep])
    W1q, s1 = _oracle_weights(inp["W1"], used)
    W3q, s3 = _oracle_weights(inp["W3"], used)
    W2q, s2 = _oracle_weights(inp["W2"], used)
    # weights: GPU codes and scales equal the oracle's for one used expert
    e0 = int(used[0])
    rows1 = s.f // 128
    assert np.array_equal(Q["W1q"][e0].cpu().numpy(), W1q[e0])
    assert np.array_equal(Q["W1s"][e0 * rows1:(e0 + 1) * rows1].cpu().numpy().astype(np.float64), s1[e0])
    sh = None
    if s.f_shared:
        sh = {}
        for n, key in (("Ws1", "1"), ("Ws3", "3"), ("Ws2", "2")):
            q_, s_ = oracle.quantize_blocks_fp8(H.bits(inp[n].cpu()))
            sh["W%sq" % key], sh["s%s" % key] = q_, s_
    ref = oracle.moe_ffn_fp8(xq[keep], sx[keep], W1q, s1, W3q, s3, W2q, s2, o_idx[keep], o_w[keep], shared=sh)
    H.assert_close(out.float().cpu().numpy()[tokens[keep]], ref, f"fp8 layer {s}", atol=1e-2, rtol=FP8_RTOL,
                   frob=FP8_RTOL)


@pytest.mark.parametrize("name,kw", [
    ("tiny", dict()),
    ("decode64", dict(alpha=0.1)),
    ("decode64", dict(alpha=1.0)),
    ("kimi_k2", dict(T=8)),
    ("deepseek_v3", dict(T=16, alpha=0.05)),    # one launch for both GEMMs, with the shared expert
    ("deepseek_v3", dict(T=64, alpha=0.5)),
])
def test_fp8_layer_small(name, kw):
    s = wl.shape(name, **kw)
    sample = None if s.T * s.k * s.f * s.d <= 32 * 8 * 2048 * 2048 else 16
    _fp8_layer_check(s, seed=0, n_sample=sample)


@pytest.mark.parametrize("name,kw", [
    ("deepseek_v3", dict(T=1024, alpha=0.5)),
    ("deepseek_v3", dict(T=16384, alpha=5.0)),
])
def test_fp8_layer_full_size_sampled(name, kw):
    s = wl.shape(name, **kw)
    _fp8_layer_check(s, seed=0, n_sample=12, device_inputs=True)
    torch.cuda.empty_cache()


def test_fp8_deterministic():
    s = wl.DECODE64.with_(alpha=0.1)
    d = {n: v.to(DEV) for n, v in wl.make_inputs(s, seed=5).items()}
    Q = moe.quantize_layer_fp8(d)
    ws = moe.new_workspace_fp8(s.T, s.d, s.f, s.E, s.k)
    a = moe.moe_layer_forward_fp8(d["x"], d["Wg"], d["bias"], Q, s.k, ws)
    b = moe.moe_layer_forward_fp8(d["x"], d["Wg"], d["bias"], Q, s.k, ws)
    assert torch.equal(a, b)


def test_fp8_hand_worked_layer_exact():
    """The hand-worked FP8 layer of tests/golden/hand_worked_fp8_layer.json through the C ABI:
    every intermediate is exact in fp32, so the GPU reproduces y = 1.5 / -3.0 exactly."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked_fp8_layer.json")))
    d, f, split = g["d"], g["f"], g["W2_split_row"]
    bf = lambda a: torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).to(DEV)
    x = bf(np.full((1, d), g["x_fill"]))
    W2 = np.full((1, d, f), g["W2_rows_lo"])
    W2[:, split:] = g["W2_rows_hi"]
    w = {"W1": bf(np.full((1, f, d), g["W1_fill"])), "W3": bf(np.full((1, f, d), g["W3_fill"])), "W2": bf(W2)}
    Wg = bf(np.zeros((1, d)))
    bias = torch.zeros(1, dtype=torch.float32, device=DEV)
    Q = moe.quantize_layer_fp8(w)
    ws = moe.new_workspace_fp8(1, d, f, 1, 1)
    out = moe.moe_layer_forward_fp8(x, Wg, bias, Q, 1, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    y = out.float().cpu().numpy()[0]
    assert np.all(y[:split] == g["expected_y_lo"]) and np.all(y[split:] == g["expected_y_hi"])
