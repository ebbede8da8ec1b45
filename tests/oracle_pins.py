"""Checks that pin the CPU oracle to things other than itself.

Each ``pin_*`` function raises AssertionError when the oracle in use disagrees
with an independent fact: an exhaustive brute force, a closed form, an
invariant, or a special case that reduces to a library routine.  The pages
print no worked example, so these are the oracle's only anchors; the planted-
mistake test runs every pin against deliberately broken oracle builds to show
that each plausible mistake is caught by at least one of them.
"""

from __future__ import annotations

import itertools
import math

import numpy as np
import torch

import oracle
from grouped_gemm_02_b200 import workload as wl


def _bits(a: torch.Tensor) -> np.ndarray:
    return wl.bf16_bits(a)


def _f64(a: torch.Tensor) -> torch.Tensor:
    return a.to(torch.float64)


def _dense_swiglu(x64: torch.Tensor, W1: torch.Tensor, W3: torch.Tensor, W2: torch.Tensor) -> torch.Tensor:
    """Dense SwiGLU FFN with library calls: silu(x W1^T) * (x W3^T), then W2."""
    g = x64 @ _f64(W1).T
    u = x64 @ _f64(W3).T
    return (torch.nn.functional.silu(g) * u) @ _f64(W2).T


# --------------------------------------------------------------------------- widening

def pin_bf16_widening_exhaustive():
    """All 65536 bf16 patterns through the logits step with Wg = 1, d = 1, no bias."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = pats.reshape(-1, 1)
    one = np.array([[0x3F80]], dtype=np.uint16)          # bf16 1.0
    L = oracle.router_logits(x, one, None)[:, 0]
    ref = torch.from_numpy(pats.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(L), nan)
    assert np.array_equal(L[~nan], ref[~nan])


# --------------------------------------------------------------------------- logits

def pin_router_logits_matmul():
    s = wl.TINY.with_(T=9, d=40, E=6)
    inp = wl.make_inputs(s, seed=3, weights=False)
    L = oracle.router_logits(_bits(inp["x"]), _bits(inp["Wg"]), inp["bias"].numpy())
    ref = (_f64(inp["x"]) @ _f64(inp["Wg"]).T + inp["bias"].to(torch.float64)).numpy()
    assert np.allclose(L, ref, rtol=1e-12, atol=1e-12)
    L0 = oracle.router_logits(_bits(inp["x"]), _bits(inp["Wg"]), None)
    assert np.allclose(L0, (_f64(inp["x"]) @ _f64(inp["Wg"]).T).numpy(), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- top-k

def _rank_key(v: float, i: int):
    return (1 if math.isnan(v) else 0, 0.0 if math.isnan(v) else -v, i)


def pin_topk_bruteforce():
    """For E <= 7 and every k: the chosen set is the only k-subset whose members all
    rank ahead of every non-member; found by enumerating every subset."""
    rng = np.random.default_rng(11)
    for E in range(1, 8):
        for trial in range(6):
            L = rng.integers(-2, 3, size=(3, E)).astype(np.float32) * 0.5   # many ties
            if trial == 5 and E > 2:
                L[0, 1] = np.nan
            for k in range(1, E + 1):
                idx, w = oracle.topk(L, k)
                for t in range(L.shape[0]):
                    row = L[t]
                    winners = []
                    for S in itertools.combinations(range(E), k):
                        rest = [j for j in range(E) if j not in S]
                        if all(_rank_key(row[i], i) < _rank_key(row[j], j) for i in S for j in rest):
                            winners.append(set(S))
                    assert len(winners) == 1
                    assert set(idx[t].tolist()) == winners[0]
                    keys = [_rank_key(row[i], i) for i in idx[t]]
                    assert all(keys[a] < keys[a + 1] for a in range(k - 1))


def pin_topk_full_softmax():
    """k = E: the gates are the full softmax (library routine), taken in chosen order."""
    L = wl.random_logits(5, 9, seed=4).numpy()
    idx, w = oracle.topk(L, 9)
    ref = torch.softmax(torch.from_numpy(L).to(torch.float64), dim=1).numpy()
    assert np.allclose(w, np.take_along_axis(ref, idx.astype(np.int64), axis=1), rtol=1e-13, atol=1e-15)


def pin_gate_invariants():
    L = wl.random_logits(40, 64, seed=5).numpy() * 3
    for k in (1, 2, 8):
        idx, w = oracle.topk(L, k)
        assert np.allclose(w.sum(axis=1), 1.0, atol=1e-12)
        assert np.all(np.diff(w, axis=1) <= 1e-15)
        assert np.all(w > 0)
        # the largest gate belongs to the largest logit of the token
        assert np.array_equal(idx[:, 0], np.argmax(L, axis=1))


# --------------------------------------------------------------------------- permutation

def pin_permutation():
    for seed, (T, E, k, alpha) in enumerate([(1, 1, 1, 1.0), (50, 8, 2, 1.0), (300, 64, 8, 0.1),
                                             (7, 384, 8, 0.02), (0, 4, 2, 1.0)]):
        idx = wl.random_routing(T, E, k, alpha, seed).numpy()
        counts, offsets, perm, inv = oracle.permutation(idx, E)
        flat = idx.ravel()
        P = flat.size
        assert np.array_equal(counts, np.bincount(flat, minlength=E))
        assert counts.sum() == P and offsets[0] == 0 and offsets[-1] == P
        assert np.all(np.diff(offsets) == counts)
        assert np.all(counts <= T)
        assert np.array_equal(np.sort(perm), np.arange(P))
        assert np.array_equal(inv[perm], np.arange(P))
        # library stable sort of the expert ids is the same permutation
        assert np.array_equal(perm, np.argsort(flat, kind="stable"))
        for e in range(E):
            seg = perm[offsets[e]:offsets[e + 1]]
            assert np.all(flat[seg] == e)
            assert np.all(np.diff(seg) > 0)


# --------------------------------------------------------------------------- expert FFN

def _small_layer(E=5, k=2, T=11, d=24, f=16, seed=7, fs=0):
    s = wl.LayerShape("pin", T=T, d=d, f=f, E=E, k=k, alpha=1.0, f_shared=fs)
    return s, wl.make_inputs(s, seed=seed)


def pin_ffn_expert_major_bruteforce():
    """Expert-major evaluation of every expert on every token, masked by the routing
    (y = sum_e mask[t,e] w[t,e] FFN_e(x_t)), with library matmuls."""
    s, inp = _small_layer(fs=12)
    idx = wl.random_routing(s.T, s.E, s.k, 1.0, 1).numpy()
    w = wl.random_gates(s.T, s.k, 1).numpy().astype(np.float64)
    shared = {n: _bits(inp[n]) for n in ("Ws1", "Ws3", "Ws2")}
    y = oracle.moe_ffn(_bits(inp["x"]), _bits(inp["W1"]), _bits(inp["W3"]), _bits(inp["W2"]),
                       idx, w, shared=shared)
    x64 = _f64(inp["x"])
    ref = torch.zeros(s.T, s.d, dtype=torch.float64)
    for e in range(s.E):
        gate = torch.zeros(s.T, dtype=torch.float64)
        for t in range(s.T):
            for j in range(s.k):
                if idx[t, j] == e:
                    gate[t] += w[t, j]
        ref += gate[:, None] * _dense_swiglu(x64, inp["W1"][e], inp["W3"][e], inp["W2"][e])
    ref += _dense_swiglu(x64, inp["Ws1"], inp["Ws3"], inp["Ws2"])
    assert np.allclose(y, ref.numpy(), rtol=1e-11, atol=1e-12)


def pin_ffn_identical_experts():
    """Identical experts and gates summing to 1 give the dense SwiGLU FFN."""
    s, inp = _small_layer(E=6, k=3, seed=8)
    W1 = inp["W1"][2:3].expand(s.E, -1, -1).contiguous()
    W3 = inp["W3"][4:5].expand(s.E, -1, -1).contiguous()
    W2 = inp["W2"][0:1].expand(s.E, -1, -1).contiguous()
    L = oracle.router_logits(_bits(inp["x"]), _bits(inp["Wg"]), inp["bias"].numpy()).astype(np.float32)
    idx, w = oracle.topk(L, s.k)
    y = oracle.moe_ffn(_bits(inp["x"]), _bits(W1), _bits(W3), _bits(W2), idx, w)
    ref = _dense_swiglu(_f64(inp["x"]), W1[0], W3[0], W2[0]).numpy()
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-12)


def pin_ffn_single_expert_dense():
    """E = 1, k = 1: the layer is one dense SwiGLU FFN with gate 1."""
    s, inp = _small_layer(E=1, k=1, seed=9)
    idx = np.zeros((s.T, 1), dtype=np.int32)
    w = np.ones((s.T, 1))
    y = oracle.moe_ffn(_bits(inp["x"]), _bits(inp["W1"]), _bits(inp["W3"]), _bits(inp["W2"]), idx, w)
    ref = _dense_swiglu(_f64(inp["x"]), inp["W1"][0], inp["W3"][0], inp["W2"][0]).numpy()
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-12)


def pin_ffn_unrouted_expert_is_inert():
    """Changing the weights of an expert no token is routed to changes nothing; a
    missing (None) expert that no token uses is accepted."""
    s, inp = _small_layer(E=4, k=1, seed=10)
    idx = (np.arange(s.T) % 3).astype(np.int32).reshape(-1, 1)        # expert 3 unused
    w = np.ones((s.T, 1))
    args = lambda W1: (_bits(inp["x"]), _bits(W1), _bits(inp["W3"]), _bits(inp["W2"]), idx, w)
    y0 = oracle.moe_ffn(*args(inp["W1"]))
    W1b = inp["W1"].clone()
    W1b[3] = W1b[3] * 3 + 1
    y1 = oracle.moe_ffn(*args(W1b))
    assert np.array_equal(y0, y1)
    per = [_bits(inp["W1"][e]) if e < 3 else None for e in range(4)]
    y2 = oracle.moe_ffn(_bits(inp["x"]), per, [_bits(inp["W3"][e]) for e in range(4)],
                        [_bits(inp["W2"][e]) for e in range(4)], idx, w)
    assert np.array_equal(y0, y2)


def pin_ffn_token_subset_and_threads():
    """A token subset returns the same rows; the thread count does not change a bit."""
    s, inp = _small_layer(E=5, k=2, T=13, seed=12)
    idx = wl.random_routing(s.T, s.E, s.k, 1.0, 2).numpy()
    w = wl.random_gates(s.T, s.k, 2).numpy().astype(np.float64)
    a = (_bits(inp["x"]), _bits(inp["W1"]), _bits(inp["W3"]), _bits(inp["W2"]), idx, w)
    y1 = oracle.moe_ffn(*a, nthreads=1)
    y4 = oracle.moe_ffn(*a, nthreads=4)
    assert np.array_equal(y1, y4)
    sub = np.array([12, 0, 5], dtype=np.int64)
    ys = oracle.moe_ffn(*a, tokens=sub, nthreads=2)
    assert np.array_equal(ys, y1[sub])
    assert oracle.moe_ffn(*a, tokens=np.zeros(0, dtype=np.int64)).shape == (0, s.d)


def pin_hand_worked_layer():
    """A layer small enough to work by hand (tests/golden/hand_worked_layer.json)."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_layer.json")
    g = json.load(open(path))
    bf = lambda a: torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)
    x, Wg = bf(g["x"]), bf(g["Wg"])
    W1, W3, W2 = bf(g["W1"]), bf(g["W3"]), bf(g["W2"])
    sh = {n: _bits(bf(g[n])) for n in ("Ws1", "Ws3", "Ws2")}
    for n in ("x", "Wg", "W1", "W3", "W2", "Ws1", "Ws3", "Ws2"):      # all exact in bf16
        assert torch.equal(bf(g[n]).to(torch.float64), torch.tensor(g[n], dtype=torch.float64))
    res = oracle.moe_layer(_bits(x), _bits(Wg), np.array(g["bias"], dtype=np.float32),
                           _bits(W1), _bits(W3), _bits(W2), k=g["k"])
    assert res["idx"].tolist() == g["expected_idx"]
    # closed form of the worked example (derivation in the fixture)
    silu = lambda z: z / (1.0 + math.exp(-z))
    g1 = 1.0 / (1.0 + math.exp(-0.5))                  # softmax over logits (2, 1.5)
    g2 = 1.0 - g1
    h1 = silu(1.0) * 2.0                              # expert 1: g = 1, u = 2
    h2 = silu(-2.0) * 3.0                             # expert 2: g = -2, u = 3
    y = [g1 * h1 * 1.0 + g2 * h2 * 2.0, g1 * h1 * -1.0 + g2 * h2 * 0.5]
    assert np.allclose(res["w"][0], [g1, g2], rtol=1e-15)
    assert np.allclose(res["out"][0], y, rtol=1e-14, atol=0)
    # the same token with the shared expert: g = 3, u = -1, W2s = (1, 2), gate 1
    hs = silu(3.0) * -1.0
    out_s = oracle.moe_ffn(_bits(x), _bits(W1), _bits(W3), _bits(W2), res["idx"], res["w"], shared=sh)
    assert np.allclose(out_s[0], [y[0] + hs * 1.0, y[1] + hs * 2.0], rtol=1e-14, atol=0)


def pin_hand_worked_fp8_layer():
    """An FP8 expert FFN small enough to work by hand (tests/golden/hand_worked_fp8_layer.json):
    the scale choice, the round to nearest of h's requantisation and the absolute output."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_fp8_layer.json")
    g = json.load(open(path))
    d, f, split = g["d"], g["f"], g["W2_split_row"]
    bf = lambda a: torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)
    x = bf(np.full((1, d), g["x_fill"]))
    W1 = bf(np.full((f, d), g["W1_fill"]))
    W3 = bf(np.full((f, d), g["W3_fill"]))
    W2 = np.full((d, f), g["W2_rows_lo"])
    W2[split:] = g["W2_rows_hi"]
    W2 = bf(W2)
    xq, sx = oracle.quantize_rows_fp8(_bits(x))
    W1q, s1 = oracle.quantize_blocks_fp8(_bits(W1))
    W3q, s3 = oracle.quantize_blocks_fp8(_bits(W3))
    W2q, s2 = oracle.quantize_blocks_fp8(_bits(W2))
    exp = g["expected_scales"]
    assert (sx[0, 0], s1[0, 0], s3[0, 0], s2[0, 0]) == (exp["x"], exp["W1"], exp["W3"], exp["W2"])
    assert oracle.e4m3_decode(int(xq[0, 0])) == 256.0 and oracle.e4m3_decode(int(W1q[0, 0])) == 256.0
    # h = silu(1) * 2 = 1.4621...; / 2^-8 = 374.3 -> nearest e4m3 value 384 -> 1.5
    assert oracle.fp8_block_scale(2.0 / (1.0 + math.exp(-1.0))) == 2.0 ** -8
    y = oracle.moe_ffn_fp8(xq, sx, [W1q], [s1], [W3q], [s3], [W2q], [s2], np.zeros((1, 1), dtype=np.int32),
                           np.ones((1, 1)))
    assert np.all(y[0, :split] == g["expected_y_lo"]) and np.all(y[0, split:] == g["expected_y_hi"])


def pin_empty_batch():
    s, inp = _small_layer(T=0, E=3, k=2, seed=13)
    res = oracle.moe_layer(_bits(inp["x"]), _bits(inp["Wg"]), inp["bias"].numpy(), _bits(inp["W1"]),
                           _bits(inp["W3"]), _bits(inp["W2"]), k=2)
    assert res["out"].shape == (0, s.d) and res["counts"].sum() == 0 and res["offsets"][-1] == 0


# --------------------------------------------------------------------------- FP8

def _torch_e4m3(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def pin_e4m3_decode_matches_library():
    """Every one of the 256 codes decodes like torch's float8_e4m3fn (NaN codes included)."""
    codes = np.arange(256, dtype=np.uint8)
    mine = np.array([oracle.e4m3_decode(c) for c in codes])
    ref = _torch_e4m3(codes)
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(0x01) == 2.0 ** -9


def _e4m3_grid() -> np.ndarray:
    """Every finite code value, every midpoint between neighbours, tiny offsets around
    them, random values across the range, both signs."""
    vals = np.array(sorted({oracle.e4m3_decode(c) for c in range(0x7F)}))
    mids = (vals[1:] + vals[:-1]) / 2
    rng = np.random.default_rng(5)
    rnd = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(460.0), 4000))
    g = np.concatenate([vals, mids, mids * (1 + 1e-9), mids * (1 - 1e-9), rnd])
    return np.concatenate([g, -g])


def pin_e4m3_encode_matches_library():
    """Round to nearest, ties to even, against torch's float -> float8_e4m3fn cast (|v| < 464,
    where torch also saturates to 448); above that the reading saturates to 448."""
    g = _e4m3_grid()
    g = g[np.abs(g) < 464]
    mine = np.array([oracle.e4m3_encode(v) for v in g], dtype=np.uint8)
    ref = torch.from_numpy(g).to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # the fp64 -> fp32 step is exact for the grid's code values and midpoints; compare on those
    # and on values whose fp32 rounding cannot cross a midpoint
    exact = g.astype(np.float32).astype(np.float64) == g
    assert np.array_equal(mine[exact], ref[exact])
    for v in (500.0, 1e6, -3e4):
        assert oracle.e4m3_decode(oracle.e4m3_encode(v)) == np.sign(v) * 448.0


def pin_e4m3_fast_encoder_equals_definition():
    g = _e4m3_grid()
    g = np.concatenate([g, [0.0, -0.0, 448.0, 470.0, 1e9, 2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -6 - 2.0 ** -10]])
    a = np.array([oracle.e4m3_encode(v) for v in g])
    b = np.array([oracle.e4m3_encode_fast(v) for v in g])
    assert np.array_equal(a, b)


def pin_fp8_block_scale():
    rng = np.random.default_rng(6)
    for amax in np.concatenate([np.exp(rng.uniform(-30, 30, 500)), [448.0, 449.0, 447.9, 896.0, 1.0, 2.0 ** -20]]):
        s = oracle.fp8_block_scale(amax)
        m, e = np.frexp(s)
        assert m == 0.5                              # a power of two
        assert amax / s <= 448.0 < amax / (s / 2)    # the smallest such
    assert oracle.fp8_block_scale(0.0) == 1.0
    # the UE8M0 range ends at 2^-127: every smaller amax gets that scale
    assert oracle.fp8_block_scale(448.0 * 2.0 ** -127) == 2.0 ** -127
    assert oracle.fp8_block_scale(448.0 * 2.0 ** -127 * 0.75) == 2.0 ** -127
    for amax in (2.0 ** -133, 1e-40, 448.0 * 2.0 ** -140):
        assert oracle.fp8_block_scale(amax) == 2.0 ** -127
    assert oracle.fp8_block_scale(448.0 * 2.0 ** -126 * 0.75) == 2.0 ** -126
    # a row whose block holds only values near the bottom of bf16: codes are x / 2^-127
    xb = np.zeros((1, 128), dtype=np.uint16)
    xb[0, 0] = 0x0001                                 # 2^-133, the smallest bf16 subnormal
    xb[0, 1] = 0x0008                                 # 2^-130
    q, sc = oracle.quantize_rows_fp8(xb)
    assert sc[0, 0] == 2.0 ** -127
    assert oracle.e4m3_decode(int(q[0, 1])) == 0.125  # 2^-130 / 2^-127
    assert oracle.e4m3_decode(int(q[0, 0])) == 2.0 ** -6         # 2^-133 / 2^-127: the smallest e4m3 normal


def pin_fp8_quantize_rows_and_blocks():
    gen = torch.Generator().manual_seed(21)
    x = (torch.randn(6, 384, generator=gen) * torch.logspace(-3, 3, 6)[:, None]).to(torch.bfloat16)
    x[2, 128:256] = 0
    xb = _bits(x)
    q, sc = oracle.quantize_rows_fp8(xb)
    xv = x.to(torch.float64).numpy()
    for r in range(6):
        for b in range(3):
            blk = xv[r, 128 * b:128 * (b + 1)]
            s_ = sc[r, b]
            assert s_ == oracle.fp8_block_scale(np.abs(blk).max())
            ref = torch.from_numpy(blk / s_).to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(q[r, 128 * b:128 * (b + 1)], ref)
    W = (torch.randn(256, 384, generator=gen) * 0.02).to(torch.bfloat16)
    W[:128, 256:] *= 1000
    Wq, Ws = oracle.quantize_blocks_fp8(_bits(W))
    Wv = W.to(torch.float64).numpy()
    for br in range(2):
        for bc in range(3):
            blk = Wv[128 * br:128 * (br + 1), 128 * bc:128 * (bc + 1)]
            assert Ws[br, bc] == oracle.fp8_block_scale(np.abs(blk).max())
            ref = torch.from_numpy(blk / Ws[br, bc]).to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
            assert np.array_equal(Wq[128 * br:128 * (br + 1), 128 * bc:128 * (bc + 1)], ref.numpy())


def _skew_blocks(t: torch.Tensor, row_scale: float, col_scale: float) -> torch.Tensor:
    """Scale the second 128-row block by row_scale and the second 128-column block by
    col_scale (powers of two: exact in bf16), so neighbouring blocks get different,
    asymmetric scales and a block-index slip changes the result."""
    t = t.clone()
    t[..., 128:256, :] *= row_scale
    t[..., :, 128:256] *= col_scale
    return t


def _fp8_layer(E=3, k=2, T=5, d=256, f=256, fs=0, seed=30, skew=False):
    s = wl.LayerShape("p8", T=T, d=d, f=f, E=E, k=k, alpha=1.0, f_shared=fs)
    inp = wl.make_inputs(s, seed=seed)
    if skew:
        inp["x"] = inp["x"].clone()
        inp["x"][:, 128:256] *= 32.0
        for n in ("W1", "W3", "Ws1", "Ws3"):
            if inp.get(n) is not None:
                inp[n] = _skew_blocks(inp[n], 0.125, 4.0)
        for n in ("W2", "Ws2"):
            if inp.get(n) is not None:
                inp[n] = _skew_blocks(inp[n], 0.0625, 8.0)
    xq, sx = oracle.quantize_rows_fp8(_bits(inp["x"]))
    Q = {}
    for n in ("W1", "W3", "W2"):
        Q[n] = [oracle.quantize_blocks_fp8(_bits(inp[n][e])) for e in range(E)]
    sh = None
    if fs:
        sh = {}
        for n, key in (("Ws1", "1"), ("Ws3", "3"), ("Ws2", "2")):
            q_, s_ = oracle.quantize_blocks_fp8(_bits(inp[n]))
            sh["W%sq" % key], sh["s%s" % key] = q_, s_
    return s, inp, xq, sx, Q, sh


def _dq(q, s, rows_per=128, cols_per=128):
    v = _torch_e4m3(q)
    return v * np.repeat(np.repeat(s, rows_per, axis=0), cols_per, axis=1)


def _requant_h(h):
    """1 x 128 requantisation of h rows with the library cast (|h / s| <= 448 by construction)."""
    out = np.empty_like(h)
    for b in range(h.shape[1] // 128):
        blk = h[:, 128 * b:128 * (b + 1)]
        sc = np.array([oracle.fp8_block_scale(a) for a in np.abs(blk).max(axis=1)])
        c = torch.from_numpy(blk / sc[:, None]).to(torch.float8_e4m3fn)   # direct fp64 -> e4m3 cast
        out[:, 128 * b:128 * (b + 1)] = c.to(torch.float64).numpy() * sc[:, None]
    return out


def pin_fp8_ffn_expert_major():
    """Expert-major evaluation with the library's e4m3 decode, float64 matmuls, and the
    library cast for the requantisation of h; shared expert included.  Neighbouring
    128-wide blocks of x and of every weight differ by powers of two, so each block
    scale is used where it belongs."""
    s, inp, xq, sx, Q, sh = _fp8_layer(fs=128, skew=True)
    assert len(np.unique(sx[:, :2])) > 1 and not np.allclose(Q["W2"][0][1], Q["W2"][0][1].T)
    idx = wl.random_routing(s.T, s.E, s.k, 1.0, 3).numpy()
    w = wl.random_gates(s.T, s.k, 3).numpy().astype(np.float64)
    y = oracle.moe_ffn_fp8(xq, sx, [q for q, _ in Q["W1"]], [c for _, c in Q["W1"]], [q for q, _ in Q["W3"]],
                           [c for _, c in Q["W3"]], [q for q, _ in Q["W2"]], [c for _, c in Q["W2"]], idx, w,
                           shared=sh)
    xh = _dq(xq, sx, 1, 128)

    def ffn(W1q, s1, W3q, s3, W2q, s2):
        g = xh @ _dq(W1q, s1).T
        u = xh @ _dq(W3q, s3).T
        h = torch.nn.functional.silu(torch.from_numpy(g)).numpy() * u
        return _requant_h(h) @ _dq(W2q, s2).T

    ref = np.zeros((s.T, s.d))
    for e in range(s.E):
        gate = np.array([w[t][list(idx[t]).index(e)] if e in idx[t] else 0.0 for t in range(s.T)])
        ref += gate[:, None] * ffn(*Q["W1"][e], *Q["W3"][e], *Q["W2"][e])
    ref += ffn(sh["W1q"], sh["s1"], sh["W3q"], sh["s3"], sh["W2q"], sh["s2"])
    assert np.allclose(y, ref, rtol=1e-10, atol=1e-12)


def pin_fp8_expert_h():
    """The requantised h of one FP8 expert on one token (what the down projection reads):
    codes and scales against float64 matmuls on the library's e4m3 decode and the library's
    fp64 -> e4m3 cast, on skewed blocks; and the hand-worked fixture's h = 1.5 exactly."""
    s, inp, xq, sx, Q, _ = _fp8_layer(skew=True)
    xh = _dq(xq, sx, 1, 128)
    for e in range(s.E):
        (W1q, s1), (W3q, s3) = Q["W1"][e], Q["W3"][e]
        g = xh @ _dq(W1q, s1).T
        u = xh @ _dq(W3q, s3).T
        h = torch.nn.functional.silu(torch.from_numpy(g)).numpy() * u
        for t in range(s.T):
            hq, sh = oracle.expert_h_fp8(xq[t], sx[t], W1q, s1, W3q, s3)
            for b in range(s.f // 128):
                blk = h[t, 128 * b:128 * (b + 1)]
                sc = oracle.fp8_block_scale(np.abs(blk).max())
                assert sh[b] == sc
                ref = torch.from_numpy(blk / sc).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
                assert np.array_equal(hq[128 * b:128 * (b + 1)], ref), (e, t, b)
    # the hand-worked layer: h = 2 silu(1) = 1.462..., scale 2^-8, code of 384
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked_fp8_layer.json")))
    d, f = g["d"], g["f"]
    bf = lambda a: torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)
    xq, sx = oracle.quantize_rows_fp8(_bits(bf(np.full((1, d), g["x_fill"]))))
    W1q, s1 = oracle.quantize_blocks_fp8(_bits(bf(np.full((f, d), g["W1_fill"]))))
    W3q, s3 = oracle.quantize_blocks_fp8(_bits(bf(np.full((f, d), g["W3_fill"]))))
    hq, sh = oracle.expert_h_fp8(xq[0], sx[0], W1q, s1, W3q, s3)
    assert np.all(sh == 2.0 ** -8)
    assert all(oracle.e4m3_decode(int(c)) * sh[0] == g["expected_h_after_requant"] for c in hq)


def pin_fp8_ffn_exact_operands_match_bf16_path():
    """With weights and activations that e4m3 holds exactly (scales 1) and h values that the
    requantisation keeps exactly, the FP8 FFN equals the bf16 FFN on the same values."""
    E, T, d, f = 2, 3, 128, 128
    rng = np.random.default_rng(8)
    pick = lambda shape: rng.choice([0.0, 0.5, -0.5, 0.25, -0.25, 0.125], size=shape)
    x = torch.from_numpy(pick((T, d))).to(torch.bfloat16)
    W1 = torch.from_numpy(pick((E, f, d)) / 8).to(torch.bfloat16)
    W3 = torch.zeros(E, f, d, dtype=torch.bfloat16)
    W3[:, :, 0] = 1.0                                    # u = x[:, 0], one of the exact values above
    W2 = torch.from_numpy(pick((E, d, f))).to(torch.bfloat16)
    idx = np.array([[0, 1], [1, 0], [0, 1]], dtype=np.int32)
    w = np.array([[0.75, 0.25], [0.5, 0.5], [1.0, 0.0]])
    y16 = oracle.moe_ffn(_bits(x), _bits(W1), _bits(W3), _bits(W2), idx, w)
    xq, sx = oracle.quantize_rows_fp8(_bits(x))
    assert np.array_equal(_dq(xq, sx, 1, 128), x.to(torch.float64).numpy())
    Qs = {n: [oracle.quantize_blocks_fp8(_bits(t[e])) for e in range(E)] for n, t in (("1", W1), ("3", W3), ("2", W2))}
    y8 = oracle.moe_ffn_fp8(xq, sx, [q for q, _ in Qs["1"]], [c for _, c in Qs["1"]], [q for q, _ in Qs["3"]],
                            [c for _, c in Qs["3"]], [q for q, _ in Qs["2"]], [c for _, c in Qs["2"]], idx, w)
    # h = silu(g) * u is not exact in e4m3, so the two differ only by the requantisation of h:
    # bound it by the e4m3 half-step (2^-4 relative) times sum |W2| |h|
    h_bound = np.zeros_like(y16)
    xv = x.to(torch.float64).numpy()
    for t in range(T):
        for j in range(2):
            e = idx[t, j]
            g = W1[e].double().numpy() @ xv[t]
            u = W3[e].double().numpy() @ xv[t]
            h = torch.nn.functional.silu(torch.from_numpy(g)).numpy() * u
            h_bound[t] += w[t, j] * (np.abs(W2[e].double().numpy()) @ np.abs(h)) * 2.0 ** -4
    assert np.all(np.abs(y8 - y16) <= h_bound + 1e-12)
    assert np.abs(y8 - y16).max() > 0 or np.allclose(h_bound, 0)


def _e2m1_lib():
    import ml_dtypes
    return ml_dtypes.float4_e2m1fn


def _fp4_dq(q, s):
    """e2m1 codes [R, C] (one per byte) with 1 x 32 scales [R, C/32] through the library decode."""
    v = q.astype(np.uint8).view(_e2m1_lib()).astype(np.float64)
    return v * np.repeat(s, 32, axis=1)


def pin_e2m1_codec_matches_library():
    """e2m1 decode of all 16 codes and encode of a dense grid (every midpoint, past +-6,
    signed zeros) against the ml_dtypes float4_e2m1fn conversions."""
    lib = _e2m1_lib()
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(lib).astype(np.float64)
    ours = np.array([oracle.e2m1_decode(int(c)) for c in codes])
    assert np.array_equal(ours, ref) and np.array_equal(np.signbit(ours), np.signbit(ref))
    mags = np.unique(np.abs(ref))
    mids = (mags[1:] + mags[:-1]) / 2
    grid = np.concatenate([np.linspace(-9, 9, 7201), mids, -mids, [6.0001, 100.0, -100.0, -0.0, 1e-9, -1e-9]])
    want = grid.astype(np.float32).astype(lib).view(np.uint8)
    got = np.array([oracle.e2m1_encode(float(v)) for v in grid], dtype=np.uint8)
    assert np.array_equal(got, want)


def pin_fp4_block_scale():
    """A power of two, the smallest with amax / s <= 6, 1 for an all-zero block, inside UE8M0."""
    rng = np.random.default_rng(11)
    for amax in np.concatenate([10.0 ** rng.uniform(-30, 30, 300), [6.0, 6.0001, 3.0, 1.5, 12.0]]):
        sc = oracle.fp4_block_scale(float(amax))
        m, e = math.frexp(sc)
        assert m == 0.5
        assert amax / sc <= 6.0 and amax / (sc / 2) > 6.0
    assert oracle.fp4_block_scale(0.0) == 1.0
    assert oracle.fp4_block_scale(1e-45) == 2.0 ** -127


def pin_fp4_quantize_rows():
    """1 x 32 blocks: each block's scale from its amax, codes the library cast of v / s."""
    gen = torch.Generator().manual_seed(12)
    W = (torch.randn(9, 256, generator=gen) * torch.logspace(-3, 3, 9)[:, None]).to(torch.bfloat16)
    W[0, :32] = 0.0
    W[1, 40] = 1e30
    q, sc = oracle.quantize_rows_fp4(_bits(W))
    Wf = W.to(torch.float64).numpy()
    for r in range(W.shape[0]):
        for b in range(W.shape[1] // 32):
            blk = Wf[r, 32 * b:32 * (b + 1)]
            s_ = oracle.fp4_block_scale(float(np.abs(blk).max()))
            assert sc[r, b] == s_
            want = (blk / s_).astype(np.float32).astype(_e2m1_lib()).view(np.uint8)
            assert np.array_equal(q[r, 32 * b:32 * (b + 1)], want), (r, b)


def _fp4_layer(E=3, k=2, T=5, d=256, f=256, fs=0, seed=31):
    s = wl.LayerShape("p4", T=T, d=d, f=f, E=E, k=k, alpha=1.0, f_shared=fs)
    inp = wl.make_inputs(s, seed=seed)
    inp["x"] = inp["x"].clone()
    inp["x"][:, 128:256] *= 32.0
    xq, sx = oracle.quantize_rows_fp8(_bits(inp["x"]))
    Q = {n: [oracle.quantize_rows_fp4(_bits(inp[n][e])) for e in range(E)] for n in ("W1", "W3", "W2")}
    sh = None
    if fs:
        sh = {}
        for n, key in (("Ws1", "1"), ("Ws3", "3"), ("Ws2", "2")):
            q_, s_ = oracle.quantize_rows_fp4(_bits(inp[n]))
            sh["W%sq" % key], sh["s%s" % key] = q_, s_
    return s, inp, xq, sx, Q, sh


def pin_fp4_ffn_expert_major():
    """Expert-major float64 evaluation on library-decoded e2m1 weights (1 x 32 scales) and e4m3
    activations, h requantised with the library e4m3 cast; shared expert included."""
    s, inp, xq, sx, Q, sh = _fp4_layer(fs=128)
    assert len(np.unique(Q["W1"][0][1][:, :4])) > 1      # distinct per-row block scales are exercised
    idx = wl.random_routing(s.T, s.E, s.k, 1.0, 4).numpy()
    w = wl.random_gates(s.T, s.k, 4).numpy().astype(np.float64)
    y = oracle.moe_ffn_fp4(xq, sx, [q for q, _ in Q["W1"]], [c for _, c in Q["W1"]], [q for q, _ in Q["W3"]],
                           [c for _, c in Q["W3"]], [q for q, _ in Q["W2"]], [c for _, c in Q["W2"]], idx, w,
                           shared=sh)
    xh = _dq(xq, sx, 1, 128)

    def ffn(W1q, s1, W3q, s3, W2q, s2):
        g = xh @ _fp4_dq(W1q, s1).T
        u = xh @ _fp4_dq(W3q, s3).T
        h = torch.nn.functional.silu(torch.from_numpy(g)).numpy() * u
        return _requant_h(h) @ _fp4_dq(W2q, s2).T

    ref = np.zeros((s.T, s.d))
    for e in range(s.E):
        gate = np.array([w[t][list(idx[t]).index(e)] if e in idx[t] else 0.0 for t in range(s.T)])
        ref += gate[:, None] * ffn(*Q["W1"][e], *Q["W3"][e], *Q["W2"][e])
    ref += ffn(sh["W1q"], sh["s1"], sh["W3q"], sh["s3"], sh["W2q"], sh["s2"])
    assert np.allclose(y, ref, rtol=1e-10, atol=1e-12)


def pin_fp4_exact_weights_match_fp8_path():
    """Weights on the e2m1 grid times 2^-4 with every 32-block holding +-6 * 2^-4: the FP4 and the
    FP8 quantisations both keep them exactly, so the FP4 FFN equals the (pinned) FP8 FFN."""
    E, T, d, f = 2, 3, 128, 128
    rng = np.random.default_rng(13)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.5, -1, -1.5, -2, -3, -4, -6]) * 2.0 ** -4

    def weights(rows, cols):
        W = rng.choice(grid, size=(E, rows, cols))
        W[:, :, ::32] = 6 * 2.0 ** -4
        return torch.from_numpy(W).to(torch.bfloat16)

    W1, W3, W2 = weights(f, d), weights(f, d), weights(d, f)
    x = torch.from_numpy(rng.standard_normal((T, d))).to(torch.bfloat16)
    xq, sx = oracle.quantize_rows_fp8(_bits(x))
    idx = np.array([[0, 1], [1, 0], [0, 1]], dtype=np.int32)
    w = np.array([[0.75, 0.25], [0.5, 0.5], [1.0, 0.0]])
    Q4 = {n: [oracle.quantize_rows_fp4(_bits(t[e])) for e in range(E)] for n, t in (("1", W1), ("3", W3), ("2", W2))}
    Q8 = {n: [oracle.quantize_blocks_fp8(_bits(t[e])) for e in range(E)] for n, t in (("1", W1), ("3", W3), ("2", W2))}
    assert np.array_equal(_fp4_dq(*Q4["1"][0]), W1[0].to(torch.float64).numpy())
    args = lambda Q: ([q for q, _ in Q["1"]], [c for _, c in Q["1"]], [q for q, _ in Q["3"]], [c for _, c in Q["3"]],
                      [q for q, _ in Q["2"]], [c for _, c in Q["2"]])
    y4 = oracle.moe_ffn_fp4(xq, sx, *args(Q4), idx, w)
    y8 = oracle.moe_ffn_fp8(xq, sx, *args(Q8), idx, w)
    assert np.array_equal(y4, y8)


ALL_PINS = [v for n, v in sorted(globals().items()) if n.startswith("pin_")]
