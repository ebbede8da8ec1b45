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


def _e4m3_grid():
    """Every finite e4m3 value, ascending, and each code's index on that grid."""
    vals = np.array([oracle.e4m3_decode(c) for c in range(256)])
    fin = np.isfinite(vals)
    grid = np.unique(vals[fin])
    pos = np.full(256, -10**6, dtype=np.int64)
    pos[fin] = np.searchsorted(grid, vals[fin])
    return vals, pos


def check_h8(views, s, g_idx, tokens, xq, sx, W1q, s1, W3q, s3, sh_w, what):
    """The GPU's requantised h (codes h8, K-block-major scales sh) for every pair of the
    sampled tokens against the oracle's: h is formed in fp32 on the GPU and in fp64 in
    the oracle, so a block's scale may differ only where its amax sits at a power-of-two
    boundary, and a code by at most one e4m3 step."""
    vals, pos = _e4m3_grid()
    inv = views["inv_perm"].cpu().numpy()
    h8 = views["h8"].cpu().numpy()
    shg = views["sh"].cpu().numpy()
    nb = s.f // 128
    n_blocks = n_scale_diff = 0
    for i, t in enumerate(tokens):
        for j in range(s.k):
            e = int(g_idx[t, j])
            r = int(inv[t * s.k + j])
            hq, shq = oracle.expert_h_fp8(xq[i], sx[i], W1q[e], s1[e], W3q[e], s3[e])
            for b in range(nb):
                n_blocks += 1
                gs = float(shg[b, r])
                if gs != shq[b]:
                    n_scale_diff += 1
                    assert gs in (2 * shq[b], shq[b] / 2), f"{what}: h scale {gs} vs {shq[b]}"
                    continue
                d = np.abs(pos[h8[r, 128 * b:128 * (b + 1)]] - pos[hq[128 * b:128 * (b + 1)]])
                assert d.max() <= 1, f"{what}: h code off by {d.max()} steps (token {t}, expert {e})"
    assert n_scale_diff <= max(1, n_blocks // 100), f"{what}: {n_scale_diff}/{n_blocks} h scales differ"
    if s.f_shared:
        hs8 = views["hs8"].cpu().numpy()
        shs = views["shs"].cpu().numpy()
        for i, t in enumerate(tokens[:4]):
            hq, shq = oracle.expert_h_fp8(xq[i], sx[i], *sh_w)
            for b in range(s.f_shared // 128):
                if float(shs[b, t]) == shq[b]:
                    d = np.abs(pos[hs8[t, 128 * b:128 * (b + 1)]] - pos[hq[128 * b:128 * (b + 1)]])
                    assert d.max() <= 1, f"{what}: shared h code off by {d.max()} steps"


def _fp8_layer_check(s: wl.LayerShape, seed: int, n_sample=None, device_inputs=False):
    inp = wl.make_inputs(s, seed=seed, device=DEV if device_inputs else "cpu")
    d_inp = {n: v.to(DEV) for n, v in inp.items()}
    Q = moe.quantize_layer_fp8(d_inp)
    ws = moe.new_workspace_fp8(s.T, s.d, s.f, s.E, s.k, s.f_shared)
    out = moe.moe_layer_forward_fp8(d_inp["x"], d_inp["Wg"], d_inp["bias"], Q, s.k, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    views = moe.workspace_views_fp8(ws, s.T, s.d, s.f, s.E, s.k, s.f_shared)
    what = f"fp8 layer {s}"
    # routing (the bf16 router, as in the bf16 layer): bit-exact on identical fp32 logits
    g_L, o_idx, o_w, counts, offsets = H.check_routing(views, s, what)
    H.check_layer_plan(views, s, counts, offsets, what, fp8=True)
    x_h = inp["x"].cpu()
    tokens = np.arange(s.T) if n_sample is None else H.sample_tokens(o_idx, s.E, n_sample, seed)
    L64 = oracle.router_logits(H.bits(x_h[tokens]), H.bits(inp["Wg"].cpu()), inp["bias"].cpu().numpy())
    dL = np.abs(g_L[tokens].astype(np.float64) - L64)
    assert np.all(dL <= 1e-3 + 1e-3 * np.abs(L64)), f"router logits off by {dL.max()}"
    # activations: GPU codes and scales equal the oracle's
    xq, sx = oracle.quantize_rows_fp8(H.bits(x_h[tokens]))
    assert np.array_equal(views["x8"].cpu().numpy()[tokens], xq)
    assert np.array_equal(views["sx"].cpu().numpy()[tokens].astype(np.float64), sx)
    used = np.unique(o_idx[tokens])
    W1q, s1 = _oracle_weights(inp["W1"], used)
    W3q, s3 = _oracle_weights(inp["W3"], used)
    W2q, s2 = _oracle_weights(inp["W2"], used)
    # weights: GPU codes and scales equal the oracle's for one used expert
    e0 = int(used[0])
    rows1 = s.f // 128
    assert np.array_equal(Q["W1q"][e0].cpu().numpy(), W1q[e0])
    assert np.array_equal(Q["W1s"][e0 * rows1:(e0 + 1) * rows1].cpu().numpy().astype(np.float64), s1[e0])
    sh = None
    sh_w = None
    if s.f_shared:
        sh = {}
        for n, key in (("Ws1", "1"), ("Ws3", "3"), ("Ws2", "2")):
            q_, s_ = oracle.quantize_blocks_fp8(H.bits(inp[n].cpu()))
            sh["W%sq" % key], sh["s%s" % key] = q_, s_
        sh_w = (sh["W1q"], sh["s1"], sh["W3q"], sh["s3"])
    # the requantised h the down projection reads
    check_h8(views, s, o_idx, tokens, xq, sx, W1q, s1, W3q, s3, sh_w, what)
    ref = oracle.moe_ffn_fp8(xq, sx, W1q, s1, W3q, s3, W2q, s2, o_idx[tokens], o_w[tokens], shared=sh)
    H.assert_close(out.float().cpu().numpy()[tokens], ref, what, atol=1e-2, rtol=FP8_RTOL, frob=FP8_RTOL)


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


# Small layers for the two tile shapes of the two-launch form:
#   odd:    d = 384 is not a multiple of 256, so the second CTA of the last down
#           pair tile lies past d (its rows are dropped, its weight scales held to
#           the last tile); with a shared expert;
#   skew:   Dirichlet alpha = 0.02 over 16 experts, so a few experts take most of
#           the 2048 pairs and get the widest tiles (224 tokens on pairs);
#   shared: f = 384 (three gate/up pair tiles) with a shared expert of 256;
#   tall:   more token rows per expert than weight rows (tiles taken unit-major).
TILE_SHAPES = {
    "odd": wl.LayerShape("odd", T=300, d=384, f=256, E=8, k=2, alpha=1.0, f_shared=128),
    "skew": wl.LayerShape("skew", T=512, d=1024, f=512, E=16, k=4, alpha=0.02, f_shared=0),
    "shared": wl.LayerShape("shared", T=200, d=512, f=384, E=8, k=2, alpha=1.0, f_shared=256),
    # more token rows per expert than weight rows: tiles taken unit-major
    "tall": wl.LayerShape("tall", T=2048, d=256, f=128, E=4, k=2, alpha=1.0, f_shared=128),
}


@pytest.mark.parametrize("pairs", [0, 1])
@pytest.mark.parametrize("name", sorted(TILE_SHAPES))
def test_fp8_layer_tile_shapes(name, pairs):
    """Both tile shapes of the two-launch form (CTA pairs of up to 224 tokens, single
    CTAs of up to 112) against the oracle on every token."""
    with H.policy(pairs=pairs):
        _fp8_layer_check(TILE_SHAPES[name], seed=1)


@pytest.mark.parametrize("tiles,cap", [(1, -1), (1, 64), (-1, 96)])
def test_fp8_pair_tile_policies(tiles, cap):
    """The pair tiles under the token-bucket policy and a forced cap (widths rounded to 32)."""
    with H.policy(tiles=tiles, cap=cap):
        _fp8_layer_check(TILE_SHAPES["skew"], seed=2)


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
