"""The failure path of the kernels' bounded waits, without a GPU fault (marked gpu).

The GEMM kernels never spin without a deadline: a wait on an mbarrier or on a
cross-CTA counter that is not satisfied within 1 s sets the sticky
DEVERR_TIMEOUT bit in the workspace's error word and the kernel returns.  The
diagnostic entry point runs both waits against a barrier and a counter that
nothing will complete; this test checks the bit, that no wait ended early, and
that the same context then computes the layer bit-identically to before.
"""

from __future__ import annotations

import pytest
import torch

from grouped_gemm_02_b200 import moe
from grouped_gemm_02_b200 import workload as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(s, inp, ws):
    shared = dict(Ws1=inp.get("Ws1"), Ws3=inp.get("Ws3"), Ws2=inp.get("Ws2"))
    return moe.moe_layer_forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], s.k, ws,
                                 **shared)


def test_bounded_waits_give_up_and_the_context_survives():
    s = wl.TINY
    inp = {n: v.to(DEV) for n, v in wl.make_inputs(s, seed=3).items()}
    ws = moe.new_workspace(s.T, s.d, s.f, s.E, s.k, s.f_shared)
    before = _layer(s, inp, ws).clone()
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0

    moe.moe_selftest_wait_timeout(ws)
    code = moe.moe_get_device_error(ws)
    assert code & moe.DEVERR_TIMEOUT
    assert not code & moe.DEVERR_PLAN            # neither wait ended before its deadline

    moe.moe_clear_device_error(ws)
    after = _layer(s, inp, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    assert torch.equal(before, after)
