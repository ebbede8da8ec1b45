"""Shared helpers for the GPU parity tests: host copies for the oracle, the
output tolerance, and the routing-margin rule for comparing top-k decisions
taken on differently rounded logits."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from grouped_gemm_02_b200 import workload as wl

# Output tolerance for the BF16 path: |y - y_ref| <= ATOL + RTOL * |y_ref| per element.
ATOL = 1e-2
RTOL = 1e-2
# The per-element bound above is loose when |y| << 1 (the tiny layer's outputs
# are ~1e-3), so every comparison also bounds the relative Frobenius error.
# h, y_p and out are each rounded once to bf16 (relative error <= 2^-9 each,
# independent across elements), which puts the expected relative error near
# 3e-3; 1e-2 leaves a 3x margin.
FROB = 1e-2


def bits(t: torch.Tensor) -> np.ndarray:
    return wl.bf16_bits(t)


def assert_close(y: np.ndarray, y_ref: np.ndarray, what: str, atol=ATOL, rtol=RTOL, frob=FROB):
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == y_ref.shape, (what, y.shape, y_ref.shape)
    if y.size == 0:
        return
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = np.abs(y - y_ref)
    bad = err > atol + rtol * np.abs(y_ref)
    i = np.unravel_index(np.argmax(err), err.shape)
    assert not bad.any(), (f"{what}: {int(bad.sum())}/{y.size} elements out of tolerance; "
                           f"max |err| {err.max():.3e} at {i} (y={y[i]:.5e}, ref={y_ref[i]:.5e})")
    nref = np.linalg.norm(y_ref)
    if nref > 0:
        rel = np.linalg.norm(y - y_ref) / nref
        assert rel <= frob, f"{what}: relative Frobenius error {rel:.3e} > {frob}"


def expert_weights_host(W: torch.Tensor, experts) -> list:
    """Per-expert host bit arrays for the experts listed (None elsewhere)."""
    out = [None] * W.shape[0]
    for e in sorted(set(int(v) for v in experts)):
        out[e] = bits(W[e])
    return out


def clear_margin_tokens(L: np.ndarray, k: int, delta: np.ndarray) -> np.ndarray:
    """Tokens whose top-(k+1) logits are pairwise separated by more than delta,
    so the descending top-k list is the same under any perturbation < delta/2."""
    E = L.shape[1]
    srt = -np.sort(-L, axis=1)
    m = min(k + 1, E)
    gaps = srt[:, :m - 1] - srt[:, 1:m]
    if gaps.shape[1] == 0:
        return np.ones(L.shape[0], dtype=bool)
    return np.all(gaps > delta[:, None], axis=1)


def valid_topk(L: np.ndarray, idx: np.ndarray, delta: np.ndarray) -> bool:
    """Every chosen logit is >= every unchosen one, up to delta."""
    T, E = L.shape
    for t in range(T):
        chosen = np.zeros(E, dtype=bool)
        chosen[idx[t]] = True
        if len(set(idx[t].tolist())) != idx.shape[1]:
            return False
        if (~chosen).any() and L[t, chosen].min() < L[t, ~chosen].max() - delta[t]:
            return False
    return True


def sample_tokens(idx: np.ndarray, E: int, n_random: int, seed: int) -> np.ndarray:
    """A bounded token sample: random tokens plus tokens routed to the hottest and
    the coldest non-empty experts."""
    T = idx.shape[0]
    rng = np.random.default_rng(seed)
    counts = np.bincount(idx.ravel(), minlength=E)
    pick = set(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    nz = np.nonzero(counts)[0]
    if nz.size:
        hot = nz[np.argmax(counts[nz])]
        cold = nz[np.argmin(counts[nz])]
        for e in (hot, cold):
            toks = np.nonzero((idx == e).any(axis=1))[0][:4]
            pick.update(toks.tolist())
    return np.array(sorted(pick), dtype=np.int64)


PLAN_GROUPS = 513          # kMaxGroups: routed experts (<= 512) + the shared expert


def decode_plan(plan) -> dict:
    """The tile plan a layer leaves in its workspace (int32 [MOE_PLAN_INTS]) as host arrays."""
    p = plan.cpu().numpy() if hasattr(plan, "cpu") else np.asarray(plan)
    G = PLAN_GROUPS
    nb, tiles1, tiles2, n_max, pairs, pair, cls, cap = (int(v) for v in p[:8])
    o = 8
    out = {"n_blocks": nb, "tiles1": tiles1, "tiles2": tiles2, "n_max": n_max, "pairs": pairs, "pair": pair,
           "cls": cls, "cap": cap}
    for name in ("group", "row0", "rows", "chunk", "units"):
        out[name] = p[o:o + nb].astype(np.int64)
        o += G
    out["tb1"] = p[o:o + nb + 1].astype(np.int64)
    o += G + 1
    out["tb2"] = p[o:o + nb + 1].astype(np.int64)
    o += G + 1
    out["dep"] = p[o:o + nb].astype(np.int64)
    return out


def check_plan(plan: dict, counts: np.ndarray, offsets: np.ndarray, T: int, f: int, d: int, f_shared: int,
               unit_max: int, m1_rows: int, what: str = "", m2_rows: int = 128, align: int = 16,
               merge: int = 1) -> None:
    """The invariants of a tile plan built from the live histogram:
    * one block per expert with tokens (+ the shared expert over all T tokens),
      heaviest first (ties: lower group id);
    * each block's rows [row0, row0 + rows) are cut into `units` chunks of
      `chunk` rows, a multiple of `align` and at most unit_max, every chunk non-empty,
      so the tiles of a block cover its rows exactly once;
    * the routed blocks' rows tile [0, offsets[E]) exactly once;
    * the tile prefixes count units x M-tiles of the gate/up GEMM and
      ceil(units / merge) x M-tiles of the down GEMM (a down tile spanning
      `merge` units), and n_max is the widest chunk."""
    E = counts.size
    active = np.nonzero(counts > 0)[0]
    n_blocks = active.size + (1 if f_shared else 0)
    assert plan["n_blocks"] == n_blocks, (what, plan["n_blocks"], n_blocks)
    g, r0, rows, ch, un = plan["group"], plan["row0"], plan["rows"], plan["chunk"], plan["units"]
    assert sorted(g.tolist()) == sorted(active.tolist() + ([E] if f_shared else [])), what
    for i in range(n_blocks):
        if g[i] < E:
            assert rows[i] == counts[g[i]] and r0[i] == offsets[g[i]], (what, i)
        else:
            assert rows[i] == T and r0[i] == 0, (what, i)
    key = [(-int(rows[i]), int(g[i])) for i in range(n_blocks)]
    assert key == sorted(key), f"{what}: blocks not heaviest first"
    assert np.all(ch % align == 0) and np.all(ch >= align) and np.all(ch <= unit_max), what
    assert np.all(ch <= plan["cap"]), f"{what}: a tile wider than the plan's cap"
    if plan["cls"] == -2:                       # token buckets: one width for every expert
        assert np.all(ch == plan["cap"]), f"{what}: token-bucket plan with widths {np.unique(ch)}"
    assert np.all(ch * un >= rows) and np.all(ch * (un - 1) < rows), f"{what}: an empty or missing unit"
    cover = np.zeros(int(offsets[-1]), dtype=np.int64)
    for i in range(n_blocks):
        if g[i] == E:
            continue
        for u in range(int(un[i])):
            a = r0[i] + u * ch[i]
            b = r0[i] + min((u + 1) * ch[i], rows[i])
            cover[a:b] += 1
    assert np.all(cover == 1), f"{what}: routed rows not covered exactly once"
    m1 = np.array([-(-(f if gi < E else f_shared) // m1_rows) for gi in g], dtype=np.int64)
    m2 = -(-d // m2_rows)
    assert np.array_equal(plan["tb1"], np.concatenate([[0], np.cumsum(un * m1)])), what
    assert np.array_equal(plan["tb2"], np.concatenate([[0], np.cumsum(-(-un // merge) * m2)])), what
    assert plan["tiles1"] == plan["tb1"][-1] and plan["tiles2"] == plan["tb2"][-1], what
    assert plan["n_max"] == (int(ch.max()) if n_blocks else 0), what
    assert plan["pairs"] == int(offsets[-1]), what


# The launch-form switches the tests have set through moe_set_policy (-1: the library's rule).
POLICY = {"one_launch": -1, "pairs": -1, "tiles": -1, "cap": -1, "gather": -1}


def _apply(pol):
    from grouped_gemm_02_b200 import moe
    moe.moe_set_policy(moe.POLICY_ONE_LAUNCH, pol["one_launch"])
    moe.moe_set_policy(moe.POLICY_CTA_PAIRS, pol["pairs"])
    moe.moe_set_policy(moe.POLICY_TILES, pol["tiles"])
    moe.moe_set_policy(moe.POLICY_TILE_CAP, pol["cap"])
    moe.moe_set_policy(moe.POLICY_GATHER, pol["gather"])


class policy:
    """Context manager: force the library's launch-form and tile-policy switches, restore them after."""

    def __init__(self, one_launch: int = -1, pairs: int = -1, tiles: int = -1, cap: int = -1, gather: int = -1):
        self.want = {"one_launch": one_launch, "pairs": pairs, "tiles": tiles, "cap": cap, "gather": gather}

    def __enter__(self):
        self.prev = dict(POLICY)
        _apply(self.want)
        POLICY.update(self.want)
        return self

    def __exit__(self, *exc):
        _apply(self.prev)
        POLICY.update(self.prev)
        return False


def tile_tables():
    """(cap per histogram class, fixed width per token bucket) as the library was built with."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "grouped_gemm_02_b200",
                            "csrc", "tile_table.h")).read()
    cap = [int(v) for v in re.search(r"#define MOE_TILE_CAP_TABLE \{([^}]*)\}", src).group(1).split(",")]
    width = [int(v) for v in re.search(r"#define MOE_TOKEN_BUCKET_WIDTH \{([^}]*)\}", src).group(1).split(",")]
    return cap, width


def token_bucket(T: int) -> int:
    return 0 if T <= 16 else 1 if T <= 64 else 2 if T <= 256 else 3 if T <= 1024 else 4 if T <= 4096 else 5


def histogram_class(counts: np.ndarray):
    """(class, distance of its features from the nearest bucket edge, relative) of a routing,
    as the plan step defines it: tokens per effective expert, and the hottest expert against it."""
    c = counts[counts > 0].astype(np.float64)
    P = c.sum()
    if P <= 0:
        return 0, 1.0
    eff = np.exp(np.log(P) - (c * np.log(c)).sum() / P)
    m = P / eff
    r = c.max() / m
    e1, e2 = [8, 32, 128, 512], [1.5, 4.0]
    b1 = sum(m >= e for e in e1)
    b2 = sum(r >= e for e in e2)
    margin = min([abs(m / e - 1) for e in e1] + [abs(r / e - 1) for e in e2])
    return 3 * b1 + b2, margin


def fused_gemms(P: int, f: int) -> bool:
    """One launch for both expert GEMMs: the library's rule (P <= 256 pairs and f <= 4096) or the forced switch."""
    if POLICY["one_launch"] >= 0:
        return POLICY["one_launch"] == 1
    return P <= 256 and f <= 4096


def pair_gemms(P: int, f: int) -> bool:
    """CTA-pair tiles (bf16 path): whenever two launches run, unless forced."""
    if POLICY["pairs"] >= 0:
        return POLICY["pairs"] == 1
    return not fused_gemms(P, f)


def pair_gemms_lowp(P: int, f: int) -> bool:
    """CTA-pair tiles (FP8 / FP4 path): only when forced on and two launches run
    (the single launch has no pair form)."""
    return not fused_gemms(P, f) and POLICY["pairs"] == 1


def check_routing(views, s: wl.LayerShape, what: str):
    """Routing on identical fp32 logits: the oracle's top-k of the GPU's own logits
    equals the GPU's indices for every token (gates within 1e-6), and counts,
    offsets, perm and inv_perm equal the oracle's permutation of those indices."""
    g_L = views["logits"].cpu().numpy()
    g_idx = views["topk_idx"].cpu().numpy()
    o_idx, o_w = oracle.topk(g_L, s.k)
    assert np.array_equal(g_idx, o_idx), f"{what}: top-k differs on identical logits"
    assert np.max(np.abs(views["topk_w"].cpu().numpy() - o_w)) <= 1e-6, what
    rc, ro, rp, ri = oracle.permutation(g_idx, s.E)
    assert np.array_equal(views["counts"].cpu().numpy(), rc), what
    assert np.array_equal(views["offsets"].cpu().numpy(), ro), what
    assert np.array_equal(views["perm"].cpu().numpy(), rp), what
    assert np.array_equal(views["inv_perm"].cpu().numpy(), ri), what
    return g_L, o_idx, o_w, rc, ro


def check_layer_plan(views, s: wl.LayerShape, counts, offsets, what, fp8: bool = False):
    """The plan the layer left in its workspace: invariants for the tile shape its
    launch form uses, and (single launch) every gate/up tile's epilogue warps
    published their h rows: 4 per tile and CTA."""
    plan = decode_plan(views["plan"])
    pair = pair_gemms_lowp(s.P, s.f) if fp8 else pair_gemms(s.P, s.f)
    # FP8 / FP4 on single CTAs in two launches: a down tile spans two units (header bit 1)
    merge = 2 if fp8 and not pair and not fused_gemms(s.P, s.f) else 1
    want = int(pair) | (2 if merge == 2 else 0)
    assert plan["pair"] == want, f"{what}: plan header pair={plan['pair']}, expected {want}"
    if fp8 and pair:
        unit_max, m1_rows, m2_rows, align = 224, 128, 256, 32
    elif fp8:
        unit_max, m1_rows, m2_rows, align = 112, 128, 128, 16
    elif pair:
        unit_max, m1_rows, m2_rows, align = 256, 128, 256, 32
    else:
        unit_max, m1_rows, m2_rows, align = 256, 64, 128, 16
    check_plan(plan, counts, offsets, s.T, s.f, s.d, s.f_shared, unit_max, m1_rows, what, m2_rows, align, merge)
    # the tile policy: a forced cap, token buckets, or the table's cap for the histogram class
    rnd = lambda v: max(align, min(v, unit_max) // align * align)
    caps, widths = tile_tables()
    if POLICY["tiles"] == 1:
        w = POLICY["cap"] if POLICY["cap"] > 0 else widths[token_bucket(s.T)]
        assert (plan["cls"], plan["cap"]) == (-2, rnd(w)), what
    elif POLICY["cap"] > 0:
        assert (plan["cls"], plan["cap"]) == (-1, rnd(POLICY["cap"])), what
    else:
        cls, margin = histogram_class(counts)
        if margin > 1e-3:     # features on a bucket edge may round either way in fp32
            assert plan["cls"] == cls, f"{what}: histogram class {plan['cls']}, expected {cls}"
        assert 0 <= plan["cls"] < len(caps) and plan["cap"] == rnd(caps[plan["cls"]]), what
    m1 = np.array([-(-(s.f if g < s.E else s.f_shared) // m1_rows) for g in plan["group"]], dtype=np.int64)
    warps = 8 if pair else 4
    need = warps * plan["units"] * m1 if fused_gemms(s.P, s.f) else np.zeros_like(m1)
    assert np.array_equal(plan["dep"], need), f"{what}: gate/up tiles published {plan['dep']} != {need}"
