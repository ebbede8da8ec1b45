"""moe_permute_noalloc: the permutation step for callers that cannot allocate
device memory (a host framework that owns all device memory, or a loop that
cannot afford cudaMalloc's implicit synchronisation).  It keeps its scratch in
a static device array instead of a caller-provided workspace.

The test calls it through the C ABI twice in a row, on different routings,
and checks each result against moe_permute (the workspace entry point) --
bit-exact, the tolerance the tests use for integer and copy work.  The file
name makes pytest collect it last, so a run that stops at the first failure
has already run every other test.
"""

import ctypes as C

import numpy as np
import pytest
import torch

from grouped_gemm_02_b200 import moe
from grouped_gemm_02_b200 import workload as wl

pytestmark = pytest.mark.gpu


def _noalloc(L, idx, x, E, k):
    T, d = x.shape
    P = T * k
    dev = x.device
    counts = torch.full((E,), -7, dtype=torch.int32, device=dev)
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
    perm = torch.full((P,), -7, dtype=torch.int32, device=dev)
    inv = torch.full((P,), -7, dtype=torch.int32, device=dev)
    xp = torch.zeros(P, d, dtype=torch.bfloat16, device=dev)
    vp = lambda t: C.c_void_p(t.data_ptr())
    rc = L.moe_permute_noalloc(vp(idx), vp(x), T, d, E, k, vp(counts), vp(offsets), vp(perm), vp(inv), vp(xp),
                               C.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, (counts, offsets, perm, inv, xp)


def test_permute_noalloc_matches_workspace_entry_point():
    L = moe.lib()
    i64, vp = C.c_int64, C.c_void_p
    L.moe_permute_noalloc.argtypes = [vp, vp, i64, i64, i64, i64, vp, vp, vp, vp, vp, vp]
    L.moe_permute_noalloc.restype = C.c_int
    cases = [(333, 64, 8, 0.1, 1), (2049, 384, 8, 0.02, 2)]   # two calls in a row, different routings
    for T, E, k, alpha, seed in cases:
        d = 128
        idx = wl.random_routing(T, E, k, alpha, seed=seed).cuda()
        x = wl.make_inputs(wl.LayerShape("p", T=T, d=d, f=64, E=E, k=k, alpha=1.0), seed=seed,
                           weights=False)["x"].cuda()
        rc, got = _noalloc(L, idx, x, E, k)
        assert rc == 0, moe.moe_status_string(rc)
        ws = moe.new_workspace(T, d, 64, E, k)
        ref = moe.moe_permute(idx, x, E, ws)
        torch.cuda.synchronize()
        for name, a, b in zip(("counts", "offsets", "perm", "inv_perm", "xp"), got, ref):
            assert torch.equal(a, b), f"{name} differs from moe_permute (T={T} E={E})"
    # out-of-range expert ids are dropped as moe_permute drops them: no error word to read,
    # so the drop shows as offsets[E] == T*k - (dropped pairs) and inv_perm == -1 there
    T, E, k, d = 300, 64, 4, 128
    idx = wl.random_routing(T, E, k, 1.0, seed=5)
    bad = [(3, 1, E + 2), (17, 0, -1), (299, 3, 1 << 20)]
    for t, j, v in bad:
        idx[t, j] = v
    idx = idx.cuda()
    x = wl.make_inputs(wl.LayerShape("p", T=T, d=d, f=64, E=E, k=k, alpha=1.0), seed=5,
                       weights=False)["x"].cuda()
    rc, got = _noalloc(L, idx, x, E, k)
    assert rc == 0, moe.moe_status_string(rc)
    ws = moe.new_workspace(T, d, 64, E, k)
    ref = moe.moe_permute(idx, x, E, ws)
    torch.cuda.synchronize()
    counts, offsets, perm, inv, xp = got
    n_valid = T * k - len(bad)
    assert int(offsets[E]) == n_valid
    assert all(int(inv[t * k + j]) == -1 for t, j, _ in bad)
    assert torch.equal(counts, ref[0]) and torch.equal(offsets, ref[1]) and torch.equal(inv, ref[3])
    assert torch.equal(perm[:n_valid], ref[2][:n_valid]) and torch.equal(xp, ref[4])
    # a size beyond the static scratch is refused on the host, before any work
    big_T = (65536 // 512 + 1) * 4096 // 8
    rc, _ = _noalloc(L, torch.zeros(big_T, 8, dtype=torch.int32, device="cuda"),
                     torch.zeros(big_T, 64, dtype=torch.bfloat16, device="cuda"), 512, 8)
    assert rc == -3
