"""CUDA path against the CPU oracle, through the C ABI (marked gpu)."""

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


@pytest.fixture(scope="module", autouse=True)
def _lib():
    moe.lib()
    yield
    torch.cuda.synchronize()


def small_ws(T, d, f, E, k, fs=0):
    return moe.new_workspace(T, d, f, E, k, fs)


# ------------------------------------------------------------------ top-k (identical fp32 logits)

@pytest.mark.parametrize("E,k", [(1, 1), (8, 2), (8, 8), (64, 8), (256, 8), (384, 8), (512, 1), (512, 8), (33, 3)])
@pytest.mark.parametrize("ties", [False, True])
def test_topk_bit_exact(E, k, ties):
    T = 1000
    L = wl.random_logits(T, E, seed=E * 10 + k, ties=ties)
    if ties:
        L[0, :] = 0.0           # a whole row of ties
        L[1, ::2] = -0.0        # signed zeros tie with +0
    ws = small_ws(T, 64, 64, E, k)
    idx, w = moe.moe_topk(L.to(DEV), k, ws)
    ref_idx, ref_w = oracle.topk(L.numpy(), k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert np.max(np.abs(w.cpu().numpy() - ref_w)) <= 1e-6
    assert moe.moe_get_device_error(ws) == 0


def test_topk_nan_ranks_last_and_is_reported():
    T, E, k = 64, 16, 4
    L = wl.random_logits(T, E, seed=3)
    L[5, 3] = float("nan")
    L[6, :] = L[6, :].clone()
    L[6, 0] = float("nan")
    ws = small_ws(T, 64, 64, E, k)
    idx, _ = moe.moe_topk(L.to(DEV), k, ws)
    ref_idx, _ = oracle.topk(L.numpy(), k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert moe.moe_get_device_error(ws) & moe.DEVERR_NAN_LOGIT


# ------------------------------------------------------------------ router logits

@pytest.mark.parametrize("name", ["tiny", "decode64", "kimi_k2"])
def test_router_logits(name):
    s = wl.shape(name, T=37)
    inp = wl.make_inputs(s, seed=1, weights=False)
    ws = small_ws(s.T, s.d, 64, s.E, s.k)
    L, idx, w = moe.moe_route(inp["x"].to(DEV), inp["Wg"].to(DEV), inp["bias"].to(DEV), s.k, ws)
    ref = oracle.router_logits(H.bits(inp["x"]), H.bits(inp["Wg"]), inp["bias"].numpy())
    Lh = L.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(Lh - ref) <= 1e-3 + 1e-3 * np.abs(ref))
    # the top-k of those very logits is bit-exact against the oracle's top-k of the same fp32 values
    ref_idx, ref_w = oracle.topk(L.cpu().numpy(), s.k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert np.max(np.abs(w.cpu().numpy() - ref_w)) <= 1e-6


# ------------------------------------------------------------------ histogram / permutation

@pytest.mark.parametrize("T,E,k,alpha", [(1, 1, 1, 1.0), (64, 8, 2, 1.0), (32, 64, 8, 0.1), (333, 64, 8, 10.0),
                                         (5000, 256, 8, 0.05), (2049, 384, 8, 0.02), (700, 512, 3, 1.0)])
def test_permute_bit_exact(T, E, k, alpha):
    d = 128
    idx = wl.random_routing(T, E, k, alpha, seed=T + E)
    x = wl.make_inputs(wl.LayerShape("p", T=T, d=d, f=64, E=E, k=k, alpha=1.0), seed=2, weights=False)["x"]
    ws = small_ws(T, d, 64, E, k)
    counts, offsets, perm, inv, xp = moe.moe_permute(idx.to(DEV), x.to(DEV), E, ws)
    rc, ro, rp, ri = oracle.permutation(idx.numpy(), E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    assert np.array_equal(inv.cpu().numpy(), ri)
    assert torch.equal(xp.cpu(), x[torch.from_numpy(rp).long() // k])
    assert moe.moe_get_device_error(ws) == 0


def test_permute_drops_out_of_range_expert():
    T, E, k, d = 40, 8, 2, 64
    idx = wl.random_routing(T, E, k, 1.0, seed=9)
    idx[3, 1] = E + 5
    idx[7, 0] = -1
    x = wl.make_inputs(wl.LayerShape("p", T=T, d=d, f=64, E=E, k=k, alpha=1.0), seed=2, weights=False)["x"]
    ws = small_ws(T, d, 64, E, k)
    counts, offsets, perm, inv, xp = moe.moe_permute(idx.to(DEV), x.to(DEV), E, ws)
    assert moe.moe_get_device_error(ws) & moe.DEVERR_EXPERT_RANGE
    inv = inv.cpu().numpy()
    assert inv[3 * k + 1] == -1 and inv[7 * k + 0] == -1
    valid = np.ones(T * k, dtype=bool)
    valid[[3 * k + 1, 7 * k]] = False
    assert offsets.cpu().numpy()[-1] == valid.sum()
    # the surviving pairs form the oracle's permutation of the surviving ids
    flat = idx.numpy().ravel()
    keep = np.nonzero(valid)[0]
    order = keep[np.argsort(flat[keep], kind="stable")]
    assert np.array_equal(perm.cpu().numpy()[:valid.sum()], order)
    moe.moe_clear_device_error(ws)
    assert moe.moe_get_device_error(ws) == 0


# ------------------------------------------------------------------ grouped GEMM + combine on given routing

def _gemm_case(s: wl.LayerShape, seed: int, alpha: float):
    inp = wl.make_inputs(s, seed=seed)
    idx = wl.random_routing(s.T, s.E, s.k, alpha, seed)
    gw = wl.random_gates(s.T, s.k, seed)
    ws = small_ws(s.T, s.d, s.f, s.E, s.k)
    d = {n: v.to(DEV) for n, v in inp.items()}
    counts, offsets, perm, inv, xp = moe.moe_permute(idx.to(DEV), d["x"], s.E, ws)
    h, y_p = moe.moe_grouped_gemm(xp, counts, offsets, perm, gw.to(DEV), d["W1"], d["W3"], d["W2"], s.T, s.k, ws)
    out = moe.moe_combine(y_p, inv, s.T, s.k)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    ref = oracle.moe_ffn(H.bits(inp["x"]), H.bits(inp["W1"]), H.bits(inp["W3"]), H.bits(inp["W2"]),
                         idx.numpy(), gw.numpy().astype(np.float64))
    return out.float().cpu().numpy(), ref


@pytest.mark.parametrize("T,d,f,E,k,alpha", [
    (16, 64, 64, 1, 1, 1.0),        # one tile, one k-block
    (3, 128, 128, 2, 1, 1.0),       # ragged N
    (64, 256, 512, 8, 2, 1.0),      # the tiny layer's shape
    (300, 256, 192, 4, 2, 1.0),     # units > 1 (n > 256), f not a multiple of 128
    (600, 320, 256, 8, 4, 0.1),     # skewed, several units per hot expert, d % 128 == 64
    (32, 2048, 1024, 64, 8, 1.0),   # decode shape
])
def test_grouped_gemm_vs_oracle(T, d, f, E, k, alpha):
    s = wl.LayerShape("g", T=T, d=d, f=f, E=E, k=k, alpha=alpha, x_std=1.0)
    out, ref = _gemm_case(s, seed=T + d, alpha=alpha)
    H.assert_close(out, ref, f"grouped GEMM T={T} d={d} f={f} E={E} k={k}")


# ------------------------------------------------------------------ whole layer

def _layer_check(s: wl.LayerShape, seed: int, n_sample=None, device_inputs=False):
    dev_inp = wl.make_inputs(s, seed=seed, device=DEV if device_inputs else "cpu")
    d_inp = {n: v.to(DEV) for n, v in dev_inp.items()}
    ws = small_ws(s.T, s.d, s.f, s.E, s.k, s.f_shared)
    shared = dict(Ws1=d_inp.get("Ws1"), Ws3=d_inp.get("Ws3"), Ws2=d_inp.get("Ws2"))
    out = moe.moe_layer_forward(d_inp["x"], d_inp["Wg"], d_inp["bias"], d_inp["W1"], d_inp["W3"], d_inp["W2"],
                                s.k, ws, **shared)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    views = moe.workspace_views(ws, s.T, s.d, s.f, s.E, s.k, s.f_shared)
    what = f"layer {s}"
    g_L, o_idx, o_w, counts, offsets = H.check_routing(views, s, what)
    H.check_layer_plan(views, s, counts, offsets, what)
    out_h = out.float().cpu().numpy()

    x_h = dev_inp["x"].cpu()
    tokens = np.arange(s.T) if n_sample is None else H.sample_tokens(o_idx, s.E, n_sample, seed)
    # the GPU's router logits against the fp64 definition, on the sampled tokens
    L64 = oracle.router_logits(H.bits(x_h[tokens]), H.bits(dev_inp["Wg"].cpu()), dev_inp["bias"].cpu().numpy())
    dL = np.abs(g_L[tokens].astype(np.float64) - L64)
    assert np.all(dL <= 1e-3 + 1e-3 * np.abs(L64)), f"router logits off by {dL.max()}"
    # the expert FFNs of the sampled tokens under that (bit-exact) routing
    used = np.unique(o_idx[tokens])
    W1 = H.expert_weights_host(dev_inp["W1"], used)
    W3 = H.expert_weights_host(dev_inp["W3"], used)
    W2 = H.expert_weights_host(dev_inp["W2"], used)
    sh = None
    if s.f_shared:
        sh = {n: H.bits(dev_inp[n].cpu()) for n in ("Ws1", "Ws3", "Ws2")}
    ref = oracle.moe_ffn(H.bits(x_h[tokens]), W1, W3, W2, o_idx[tokens], o_w[tokens], shared=sh)
    H.assert_close(out_h[tokens], ref, what)
    return out, ws


@pytest.mark.parametrize("name,kw", [
    ("tiny", dict()),
    ("decode64", dict(alpha=0.1)),
    ("decode64", dict(alpha=1.0)),
    ("decode64", dict(alpha=10.0)),
    ("mixtral", dict(T=1)),
    ("mixtral", dict(T=16)),
    ("kimi_k2", dict(T=8)),
    ("deepseek_v3", dict(T=16, alpha=0.05)),    # one launch for both GEMMs, with the shared expert
    ("deepseek_v3", dict(T=64, alpha=0.05)),
])
def test_layer_small(name, kw):
    s = wl.shape(name, **kw)
    sample = None if s.T * s.k * s.f * s.d <= 32 * 8 * 2048 * 2048 else 24
    _layer_check(s, seed=0, n_sample=sample)


@pytest.mark.parametrize("name,kw", [
    ("mixtral", dict(T=256)),
    ("mixtral", dict(T=4096)),
    ("deepseek_v3", dict(T=1024, alpha=0.5)),
    ("deepseek_v3", dict(T=16384, alpha=5.0)),
    ("kimi_k2", dict(T=256)),
    ("kimi_k2", dict(T=8192)),
])
def test_layer_full_size_sampled(name, kw):
    s = wl.shape(name, **kw)
    _layer_check(s, seed=0, n_sample=16, device_inputs=True)
    torch.cuda.empty_cache()


def test_layer_deterministic_and_steps_match():
    s = wl.DECODE64.with_(alpha=0.1)
    inp = {n: v.to(DEV) for n, v in wl.make_inputs(s, seed=4).items()}
    ws = small_ws(s.T, s.d, s.f, s.E, s.k)
    a = moe.moe_layer_forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], s.k, ws)
    b = moe.moe_layer_forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], s.k, ws)
    assert torch.equal(a, b)
    # the same layer through the separate entry points
    ws2 = small_ws(s.T, s.d, s.f, s.E, s.k)
    L, idx, w = moe.moe_route(inp["x"], inp["Wg"], inp["bias"], s.k, ws2)
    counts, offsets, perm, inv, xp = moe.moe_permute(idx, inp["x"], s.E, ws2)
    h, y_p = moe.moe_grouped_gemm(xp, counts, offsets, perm, w, inp["W1"], inp["W3"], inp["W2"], s.T, s.k, ws2)
    c = moe.moe_combine(y_p, inv, s.T, s.k)
    assert torch.equal(a, c)


def test_layer_identical_experts_closed_form():
    """All experts equal: the layer is the dense SwiGLU FFN of x (gates sum to 1)."""
    s = wl.TINY.with_(T=48, x_std=1.0)
    inp = wl.make_inputs(s, seed=6)
    for n in ("W1", "W3", "W2"):
        inp[n] = inp[n][:1].expand_as(inp[n]).contiguous()
    d = {n: v.to(DEV) for n, v in inp.items()}
    ws = small_ws(s.T, s.d, s.f, s.E, s.k)
    out = moe.moe_layer_forward(d["x"], d["Wg"], d["bias"], d["W1"], d["W3"], d["W2"], s.k, ws)
    x64 = inp["x"].double()
    g = x64 @ inp["W1"][0].double().T
    u = x64 @ inp["W3"][0].double().T
    ref = (torch.nn.functional.silu(g) * u) @ inp["W2"][0].double().T
    H.assert_close(out.float().cpu().numpy(), ref.numpy(), "identical experts")


def test_empty_and_single_token():
    s = wl.TINY.with_(T=1)
    inp = {n: v.to(DEV) for n, v in wl.make_inputs(s, seed=7).items()}
    ws = small_ws(1, s.d, s.f, s.E, s.k)
    out = moe.moe_layer_forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], s.k, ws)
    assert out.shape == (1, s.d) and torch.isfinite(out.float()).all()
    x0 = inp["x"][:0]
    out0 = moe.moe_layer_forward(x0, inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], s.k, ws)
    assert out0.shape == (0, s.d)


FORMS = [(1, 0), (0, 0), (1, 1), (0, 1)]     # (one launch, CTA pairs)
# more token rows per expert (and in the shared expert) than weight rows: the GEMMs
# take such a block's tiles unit-major
TALL = wl.LayerShape("tall", T=2048, d=256, f=128, E=4, k=2, alpha=1.0, f_shared=128)


@pytest.mark.parametrize("gather", [0, 1])
@pytest.mark.parametrize("one_launch,pairs", FORMS)
@pytest.mark.parametrize("name,kw", [
    ("decode64", dict(alpha=0.1)),
    ("deepseek_v3", dict(T=64, alpha=0.05)),     # shared expert
    ("kimi_k2", dict(T=256)),                    # hot experts with units of up to 256 tokens
    ("tall", dict()),                            # unit-major tile order
])
def test_layer_every_launch_form(name, kw, one_launch, pairs, gather):
    """Both expert-GEMM launch forms on single CTAs and on CTA pairs, with the gather pass or
    the TMA row gathers inside the GEMM, each checked against the oracle (routing bit-exact,
    plan invariants, outputs in tolerance)."""
    s = TALL if name == "tall" else wl.shape(name, **kw)
    with H.policy(one_launch=one_launch, pairs=pairs, gather=gather):
        _layer_check(s, seed=3, n_sample=None if name == "tall" else 12, device_inputs=s.d * s.f * s.E > 2**31)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("one_launch,pairs", FORMS)
@pytest.mark.parametrize("T,d,f,E,k,alpha", [
    (300, 256, 192, 4, 2, 1.0),     # f % 128 == 64: a pair's second CTA is past f on the last tile
    (600, 320, 256, 8, 4, 0.1),     # d % 256 == 64: the same for the down tiles
    (45, 128, 128, 3, 2, 1.0),      # widths of 16..48 rounded to 32 for pairs
])
def test_grouped_gemm_every_launch_form(T, d, f, E, k, alpha, one_launch, pairs):
    s = wl.LayerShape("g", T=T, d=d, f=f, E=E, k=k, alpha=alpha, x_std=1.0)
    with H.policy(one_launch=one_launch, pairs=pairs):
        out, ref = _gemm_case(s, seed=T + d + f, alpha=alpha)
    H.assert_close(out, ref, f"grouped GEMM T={T} d={d} f={f} E={E} k={k} one={one_launch} pairs={pairs}")


@pytest.mark.parametrize("tiles,cap", [(1, -1), (-1, 64), (-1, 128), (0, -1)])
@pytest.mark.parametrize("name,kw", [
    ("decode64", dict(alpha=0.1)),
    ("deepseek_v3", dict(T=64, alpha=0.05)),
    ("kimi_k2", dict(T=256)),
    ("mixtral", dict(T=16)),
])
def test_layer_tile_policies(name, kw, tiles, cap):
    """Token-bucket tiles (one width from T, padded), forced caps and the histogram-matched
    table all compute the same layer: routing bit-exact, plan of the policy's shape, outputs
    in tolerance."""
    s = wl.shape(name, **kw)
    with H.policy(tiles=tiles, cap=cap):
        _layer_check(s, seed=5, n_sample=12, device_inputs=s.d * s.f * s.E > 2**31)
    torch.cuda.empty_cache()
