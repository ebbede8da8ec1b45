"""The persistent GEMM's tile deal (the skew-aware scheduler's order), on the
CPU: schedule.h is the function the kernels call, built here with g++.

For every (gate/up tiles G, down tiles D, grid, comp) of a sweep, the deal is a
partition (every tile taken by exactly one CTA, none invented), each CTA takes
its tiles in ascending order within each GEMM and all its gate/up tiles before
any down tile, and in the balanced deal the CTAs one gate/up tile short take
their `comp` compensating down tiles first."""

from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("deal") / "libdeal.so")
    subprocess.run(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-o", out,
                    os.path.join(HERE, "deal_harness.cpp")], check=True)
    return C.CDLL(out)


@pytest.fixture(scope="module")
def deal(harness):
    L = harness
    L.deal_all.argtypes = [C.c_int] * 6 + [C.POINTER(C.c_int)]
    L.deal_all.restype = C.c_int

    def run(grid, total, G, comp, balanced):
        max_per = total + 1
        buf = np.full(grid * max_per, -2, dtype=np.int32)
        most = L.deal_all(grid, total, G, comp, int(balanced), max_per, buf.ctypes.data_as(C.POINTER(C.c_int)))
        assert most >= 0
        return buf.reshape(grid, max_per)
    return run


SWEEP = [(G, D, grid, comp)
         for G in (0, 1, 5, 147, 148, 149, 300, 1037)
         for D in (0, 1, 16, 148, 500, 2113)
         for grid in (1, 7, 148)
         for comp in (1, 2, 3, 8)]


@pytest.mark.parametrize("balanced", [False, True])
def test_deal_is_a_partition(deal, balanced):
    for G, D, grid, comp in SWEEP:
        total = G + D
        tiles = deal(grid, total, G, comp, balanced)
        taken = tiles[tiles >= 0]
        assert np.array_equal(np.sort(taken), np.arange(total)), (G, D, grid, comp)
        for b in range(grid):
            seq = tiles[b][tiles[b] >= 0]
            assert np.all(tiles[b][seq.size:] == -1)
            gate = seq[seq < G]
            down = seq[seq >= G]
            assert np.array_equal(seq[:gate.size], gate), f"CTA {b}: a down tile before a gate/up tile"
            assert np.all(np.diff(gate) > 0)
            if not balanced:
                assert np.all(np.diff(seq) == grid)
                assert seq.size == 0 or seq[0] == b


def test_balanced_deal_compensates_short_ctas(deal):
    for G, D, grid, comp in SWEEP:
        if grid == 1 or G % grid == 0:
            continue
        tiles = deal(grid, G + D, G, comp, True)
        grem = G % grid
        comp_total = min(D, (grid - grem) * comp)
        for b in range(grid):
            seq = tiles[b][tiles[b] >= 0]
            n_gate = G // grid + (1 if b < grem else 0)
            assert np.count_nonzero(seq < G) == n_gate
            if b >= grem:
                c0 = (b - grem) * comp
                mine = max(0, min(comp, comp_total - c0))
                assert np.array_equal(seq[n_gate:n_gate + mine], G + c0 + np.arange(mine)), (G, D, grid, comp, b)
        # the largest per-CTA load in units of down tiles is below the round-robin deal's
        # whenever some CTAs end up a gate/up tile short and there are down tiles to give them
        if D >= (grid - grem) * comp:
            loads = [np.count_nonzero(t[t >= 0] < G) * comp + np.count_nonzero(t[t >= 0] >= G) for t in tiles]
            rr = deal(grid, G + D, G, comp, False)
            loads_rr = [np.count_nonzero(t[t >= 0] < G) * comp + np.count_nonzero(t[t >= 0] >= G) for t in rr]
            assert max(loads) <= max(loads_rr), (G, D, grid, comp)


def test_tile_class_and_token_buckets(harness):
    """The histogram class and token bucket (schedule.h, compiled here) against their definition."""
    lib = harness
    lib.tile_class_of.argtypes = [C.c_float, C.c_float, C.c_float]
    lib.token_bucket_of.argtypes = [C.c_longlong]
    from tests import gpu_helpers as H
    rng = np.random.default_rng(0)
    for _ in range(400):
        E = int(rng.integers(1, 512))
        counts = rng.multinomial(int(rng.integers(1, 20000)), rng.dirichlet(np.full(E, 10 ** rng.uniform(-2, 1))))
        cls, margin = H.histogram_class(counts)
        c = counts[counts > 0].astype(np.float64)
        P = c.sum()
        eff = np.exp(np.log(P) - (c * np.log(c)).sum() / P)
        if margin > 1e-4:
            assert lib.tile_class_of(P, eff, c.max()) == cls
    assert lib.tile_class_of(0, 1, 0) == 0
    for T, b in [(1, 0), (16, 0), (17, 1), (64, 1), (65, 2), (256, 2), (1024, 3), (4096, 4), (4097, 5), (10**6, 5)]:
        assert lib.token_bucket_of(T) == b == H.token_bucket(T)
    caps, widths = H.tile_tables()
    assert len(caps) == 15 and len(widths) == 6
    assert all(16 <= v <= 256 and v % 16 == 0 for v in caps + widths)
