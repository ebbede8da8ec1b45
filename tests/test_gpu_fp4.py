"""FP4 expert weights (e2m1, 1 x 32 power-of-two scales) against the CPU oracle,
through the C ABI (marked gpu).

Codes and scales are integer / power-of-two results of the same definition on
both sides: bit-exact.  Layer outputs: the FP8 tolerance, |y - y_ref| <=
1e-2 + 3e-2 |y_ref| per element and relative Frobenius error <= 3e-2 -- both
sides compute on the same dequantised weights; only h's e4m3 requantisation
(fp32 on the GPU, fp64 in the oracle) and summation order differ.
"""

from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_02_b200 import moe
from grouped_gemm_02_b200 import workload as wl
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda"
RTOL = 3e-2


def unpack_fp4(q: torch.Tensor, atoms: torch.Tensor):
    """GPU packed codes [R, C/2] and scale atoms [R/128, C/128, 512] -> (codes [R, C], scales [R, C/32])."""
    qb = q.reshape(-1, q.shape[-1]).cpu().numpy()
    R = qb.shape[0]
    codes = np.empty((R, qb.shape[1] * 2), dtype=np.uint8)
    codes[:, 0::2] = qb & 15
    codes[:, 1::2] = qb >> 4
    a = atoms.cpu().numpy()
    nkb = a.shape[1]
    r = np.arange(R)
    sc = np.empty((R, nkb * 4), dtype=np.float64)
    for kb in range(nkb):
        for j in range(4):
            byte = 16 * (r % 32) + 4 * ((r % 128) // 32) + j
            e = a[r // 128, kb, byte].astype(np.int64) - 127
            sc[:, 4 * kb + j] = np.ldexp(1.0, e)
    return codes, sc


def _values(R, C, seed):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(R, C, generator=gen) * torch.logspace(-4, 4, R)[:, None]
    x[0, :] = 0.0                                     # all-zero blocks: scale 1
    x[1, 5] = 3.0e38                                  # a huge value in one block
    x[2, :32] = torch.arange(32) * 6.0 / 31           # amax exactly 6
    x[3, 32:64] = -1e-38                              # a block near the bottom of the scale range
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("R,C", [(128, 128), (256, 384), (1024, 2048)])
def test_quantize_fp4_bit_exact(R, C):
    W = _values(R, C, seed=R + C)
    q, atoms = moe.moe_quantize_fp4_rows(W.to(DEV))
    codes, sc = unpack_fp4(q, atoms)
    rq, rs = oracle.quantize_rows_fp4(H.bits(W))
    assert np.array_equal(codes, rq)
    assert np.array_equal(sc, rs)


def test_fp4_hand_worked_layer_exact():
    """The hand-worked layer of tests/golden/hand_worked_fp8_layer.json with FP4 weights: its fills are
    e2m1 values times powers of two (W1 2^-7 = 4 * 2^-9, W3 = 4 * 2^-8, W2 rows 4 * 2^-9 and -4 * 2^-8),
    so every intermediate is exact in fp32 and the GPU reproduces y = 1.5 / -3.0 exactly."""
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked_fp8_layer.json")))
    d, f, split = g["d"], g["f"], g["W2_split_row"]
    bf = lambda a: torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).to(DEV)
    x = bf(np.full((1, d), g["x_fill"]))
    W2 = np.full((1, d, f), g["W2_rows_lo"])
    W2[:, split:] = g["W2_rows_hi"]
    w = {"W1": bf(np.full((1, f, d), g["W1_fill"])), "W3": bf(np.full((1, f, d), g["W3_fill"])), "W2": bf(W2)}
    Q = moe.quantize_layer_fp4(w)
    ws = moe.new_workspace_fp8(1, d, f, 1, 1)
    out = moe.moe_layer_forward_fp4(x, bf(np.zeros((1, d))), torch.zeros(1, dtype=torch.float32, device=DEV), Q, 1, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    y = out.float().cpu().numpy()[0]
    assert np.all(y[:split] == g["expected_y_lo"]) and np.all(y[split:] == g["expected_y_hi"])


def _oracle_fp4(W: torch.Tensor, experts):
    codes, scales = [None] * W.shape[0], [None] * W.shape[0]
    for e in sorted(set(int(v) for v in experts)):
        codes[e], scales[e] = oracle.quantize_rows_fp4(H.bits(W[e]))
    return codes, scales


def _fp4_layer_check(s: wl.LayerShape, seed: int, n_sample=None, device_inputs=False):
    inp = wl.make_inputs(s, seed=seed, device=DEV if device_inputs else "cpu")
    d_inp = {n: v.to(DEV) for n, v in inp.items()}
    Q = moe.quantize_layer_fp4(d_inp)
    ws = moe.new_workspace_fp8(s.T, s.d, s.f, s.E, s.k, s.f_shared)
    out = moe.moe_layer_forward_fp4(d_inp["x"], d_inp["Wg"], d_inp["bias"], Q, s.k, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    views = moe.workspace_views_fp8(ws, s.T, s.d, s.f, s.E, s.k, s.f_shared)
    what = f"fp4 layer {s}"
    g_L, o_idx, o_w, counts, offsets = H.check_routing(views, s, what)
    H.check_layer_plan(views, s, counts, offsets, what, fp8=True)
    x_h = inp["x"].cpu()
    tokens = np.arange(s.T) if n_sample is None else H.sample_tokens(o_idx, s.E, n_sample, seed)
    xq, sx = oracle.quantize_rows_fp8(H.bits(x_h[tokens]))
    assert np.array_equal(views["x8"].cpu().numpy()[tokens], xq)
    used = np.unique(o_idx[tokens])
    W1q, s1 = _oracle_fp4(inp["W1"], used)
    W3q, s3 = _oracle_fp4(inp["W3"], used)
    W2q, s2 = _oracle_fp4(inp["W2"], used)
    # one used expert's GPU codes and scales equal the oracle's
    e0 = int(used[0])
    rows = s.f // 128
    codes, sc = unpack_fp4(Q["W1q"][e0], Q["W1sf"][e0 * rows:(e0 + 1) * rows])
    assert np.array_equal(codes, W1q[e0]) and np.array_equal(sc, s1[e0])
    sh = None
    if s.f_shared:
        sh = {}
        for n, key in (("Ws1", "1"), ("Ws3", "3"), ("Ws2", "2")):
            sh["W%sq" % key], sh["s%s" % key] = oracle.quantize_rows_fp4(H.bits(inp[n].cpu()))
    ref = oracle.moe_ffn_fp4(xq, sx, W1q, s1, W3q, s3, W2q, s2, o_idx[tokens], o_w[tokens], shared=sh)
    H.assert_close(out.float().cpu().numpy()[tokens], ref, what, atol=1e-2, rtol=RTOL, frob=RTOL)


@pytest.mark.parametrize("name,kw", [
    ("tiny", dict()),
    ("decode64", dict(alpha=0.1)),
    ("decode64", dict(alpha=1.0)),
    ("kimi_k2", dict(T=8)),
    ("deepseek_v3", dict(T=16, alpha=0.05)),    # one launch for both GEMMs, with the shared expert
    ("deepseek_v3", dict(T=64, alpha=0.5)),     # two launches, with the shared expert
])
def test_fp4_layer_small(name, kw):
    s = wl.shape(name, **kw)
    sample = None if s.T * s.k * s.f * s.d <= 32 * 8 * 2048 * 2048 else 16
    _fp4_layer_check(s, seed=0, n_sample=sample, device_inputs=s.d * s.f * s.E > 2**31)


@pytest.mark.parametrize("pairs", [0, 1])
@pytest.mark.parametrize("name", ["odd", "skew"])
def test_fp4_layer_tile_shapes(name, pairs):
    """FP4 weights on both tile shapes of the two-launch form (the small layers of the
    FP8 tests: "odd" has d = 384, so the last down pair tile's second CTA lies past d
    and its atom is held to the last tile)."""
    from tests.test_gpu_fp8 import TILE_SHAPES
    with H.policy(pairs=pairs):
        _fp4_layer_check(TILE_SHAPES[name], seed=1)


@pytest.mark.parametrize("name,kw", [("deepseek_v3", dict(T=1024, alpha=0.5)), ("mixtral", dict(T=256))])
def test_fp4_layer_full_size_sampled(name, kw):
    s = wl.shape(name, **kw)
    _fp4_layer_check(s, seed=0, n_sample=12, device_inputs=True)
    torch.cuda.empty_cache()
