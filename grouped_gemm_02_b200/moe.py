"""Python binding of the C ABI in include/moe.h (argument marshalling only).

Every function here takes torch tensors that already live on the current CUDA
device, checks their dtype/shape/contiguity, and passes raw pointers to the
entry point of the same name in libmoe_b200.so.  All arithmetic runs in the
library's kernels; there is no fallback: if the library is missing or the
device is not a B200, the call raises.
"""

from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import torch

from . import build as _build

MOE_OK = 0
STATUS = {0: "ok", -1: "invalid argument", -2: "size or pointer alignment", -3: "workspace too small",
          -4: "CUDA launch or runtime error", -5: "device is not sm_100 (B200)"}
DEVERR_EXPERT_RANGE, DEVERR_TIMEOUT, DEVERR_NAN_LOGIT, DEVERR_PLAN = 1, 2, 4, 8

_lib: Optional[C.CDLL] = None

EXPORTS = ("moe_workspace_size", "moe_workspace_init", "moe_route", "moe_topk", "moe_permute",
           "moe_permute_noalloc", "moe_grouped_gemm", "moe_combine", "moe_layer_forward", "moe_workspace_tensor",
           "moe_record_phase_events", "moe_launch_counter", "moe_get_device_error", "moe_clear_device_error",
           "moe_selftest_wait_timeout",
           "moe_status_string", "moe_set_policy", "moe_quantize_fp8_rows", "moe_quantize_fp8_blocks", "moe_workspace_size_fp8",
           "moe_workspace_tensor_fp8", "moe_layer_forward_fp8", "moe_quantize_fp4_rows", "moe_layer_forward_fp4")


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {status} ({STATUS.get(status, 'unknown')})")
        self.status = status


def library_path() -> str:
    return _build.LIB


def lib() -> C.CDLL:
    """Load libmoe_b200.so (it must have been built: grouped_gemm_02_b200/build.py)."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library {path} is missing; build it with grouped_gemm_02_b200/build.py")
        L = C.CDLL(path)
        i64, vp, sz = C.c_int64, C.c_void_p, C.c_size_t
        sig = {
            "moe_workspace_size": [i64, i64, i64, i64, i64, i64, C.POINTER(sz)],
            "moe_workspace_init": [vp, sz, i64, i64, i64, vp],
            "moe_route": [vp, vp, vp, i64, i64, i64, i64, vp, vp, vp, vp, sz, vp],
            "moe_topk": [vp, i64, i64, i64, vp, vp, vp, vp],
            "moe_permute": [vp, vp, i64, i64, i64, i64, vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_grouped_gemm": [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, vp, vp, vp, sz, vp],
            "moe_combine": [vp, vp, vp, i64, i64, i64, vp, vp],
            "moe_layer_forward": [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, vp, vp, sz, vp],
            "moe_workspace_tensor": [vp, i64, i64, i64, i64, i64, i64, C.c_int, C.POINTER(vp)],
            "moe_get_device_error": [vp, C.POINTER(C.c_uint32), vp],
            "moe_clear_device_error": [vp, vp],
            "moe_selftest_wait_timeout": [vp, vp],
            "moe_status_string": [C.c_int],
            "moe_record_phase_events": [C.POINTER(vp), C.c_int],
            "moe_launch_counter": [],
            "moe_set_policy": [C.c_int, C.c_int],
            "moe_quantize_fp8_rows": [vp, i64, i64, vp, vp, vp],
            "moe_quantize_fp8_blocks": [vp, i64, i64, vp, vp, vp],
            "moe_workspace_size_fp8": [i64, i64, i64, i64, i64, i64, C.POINTER(sz)],
            "moe_workspace_tensor_fp8": [vp, i64, i64, i64, i64, i64, i64, C.c_int, C.POINTER(vp)],
            "moe_layer_forward_fp8": [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                      i64, i64, vp, vp, sz, vp],
            "moe_quantize_fp4_rows": [vp, i64, i64, vp, vp, vp],
            "moe_layer_forward_fp4": [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                      i64, i64, vp, vp, sz, vp],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = {"moe_status_string": C.c_char_p, "moe_launch_counter": C.c_int64}.get(name, C.c_int)
        _lib = L
    return _lib


def _call(name: str, *args) -> None:
    rc = getattr(lib(), name)(*args)
    if rc != MOE_OK:
        raise MoEError(name, rc)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors"
    return C.c_void_p(t.data_ptr())


def _stream(stream) -> C.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _bf16(t: torch.Tensor, shape=None) -> torch.Tensor:
    assert t.dtype == torch.bfloat16, f"expected bf16, got {t.dtype}"
    if shape is not None:
        assert tuple(t.shape) == tuple(shape), f"expected shape {shape}, got {tuple(t.shape)}"
    return t


# ---------------------------------------------------------------- workspace

def moe_workspace_size(T: int, d: int, f: int, E: int, k: int, f_shared: int = 0) -> int:
    n = C.c_size_t(0)
    _call("moe_workspace_size", T, d, f, E, k, f_shared, C.byref(n))
    return int(n.value)


def moe_workspace_init(ws: torch.Tensor, T: int, E: int, k: int, stream=None) -> None:
    _call("moe_workspace_init", _p(ws), ws.numel(), T, E, k, _stream(stream))


def new_workspace(T: int, d: int, f: int, E: int, k: int, f_shared: int = 0, device=None, stream=None) -> torch.Tensor:
    """A layer-sized workspace (a torch uint8 tensor owned by the caller), initialised."""
    n = moe_workspace_size(T, d, f, E, k, f_shared)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device or torch.device("cuda"))
    moe_workspace_init(ws, T, E, k, stream)
    return ws


def moe_workspace_tensor(ws: torch.Tensor, T: int, d: int, f: int, E: int, k: int, f_shared: int, which: int) -> int:
    out = C.c_void_p(0)
    _call("moe_workspace_tensor", _p(ws), T, d, f, E, k, f_shared, which, C.byref(out))
    return int(out.value or 0)


def moe_get_device_error(ws: torch.Tensor, stream=None) -> int:
    code = C.c_uint32(0)
    _call("moe_get_device_error", _p(ws), C.byref(code), _stream(stream))
    return int(code.value)


def moe_clear_device_error(ws: torch.Tensor, stream=None) -> None:
    _call("moe_clear_device_error", _p(ws), _stream(stream))


def moe_selftest_wait_timeout(ws: torch.Tensor, stream=None) -> None:
    """Run the bounded-wait diagnostic (about 2 s); read the result with moe_get_device_error."""
    _call("moe_selftest_wait_timeout", _p(ws), _stream(stream))


def moe_record_phase_events(events) -> None:
    """Arm per-phase timing of the next moe_layer_forward on this thread: six
    torch.cuda.Event(enable_timing=True) recorded before the router, the
    permutation, the gate/up GEMM, the down GEMM and the combine, and after it."""
    if not events:
        _call("moe_record_phase_events", None, 0)
        return
    for e in events:
        if not e.cuda_event:        # torch creates the CUDA event lazily, on its first record
            e.record()
    arr = (C.c_void_p * len(events))(*[C.c_void_p(e.cuda_event) for e in events])
    _call("moe_record_phase_events", arr, len(events))


POLICY_ONE_LAUNCH, POLICY_CTA_PAIRS, POLICY_TILES, POLICY_TILE_CAP, POLICY_GATHER = 1, 2, 3, 4, 5


def moe_set_policy(what: int, value: int) -> None:
    """Force or restore (-1) one of the library's launch-form or tile-policy choices for the process."""
    _call("moe_set_policy", what, value)


def moe_launch_counter() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib().moe_launch_counter())


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


# ---------------------------------------------------------------- steps

def moe_route(x: torch.Tensor, Wg: torch.Tensor, bias: Optional[torch.Tensor], k: int, ws: torch.Tensor,
              logits=None, topk_idx=None, topk_w=None, stream=None):
    T, d = x.shape
    E = Wg.shape[0]
    _bf16(x), _bf16(Wg, (E, d))
    if bias is not None:
        assert bias.dtype == torch.float32 and bias.shape == (E,)
    dev = x.device
    logits = torch.empty(T, E, dtype=torch.float32, device=dev) if logits is None else logits
    topk_idx = torch.empty(T, k, dtype=torch.int32, device=dev) if topk_idx is None else topk_idx
    topk_w = torch.empty(T, k, dtype=torch.float32, device=dev) if topk_w is None else topk_w
    _call("moe_route", _p(x), _p(Wg), _p(bias), T, d, E, k, _p(logits), _p(topk_idx), _p(topk_w), _p(ws),
          ws.numel(), _stream(stream))
    return logits, topk_idx, topk_w


def moe_topk(logits: torch.Tensor, k: int, ws: torch.Tensor, topk_idx=None, topk_w=None, stream=None):
    T, E = logits.shape
    assert logits.dtype == torch.float32
    topk_idx = torch.empty(T, k, dtype=torch.int32, device=logits.device) if topk_idx is None else topk_idx
    topk_w = torch.empty(T, k, dtype=torch.float32, device=logits.device) if topk_w is None else topk_w
    _call("moe_topk", _p(logits), T, E, k, _p(topk_idx), _p(topk_w), _p(ws), _stream(stream))
    return topk_idx, topk_w


def moe_permute(topk_idx: torch.Tensor, x: torch.Tensor, E: int, ws: torch.Tensor, stream=None):
    T, k = topk_idx.shape
    d = x.shape[1]
    assert topk_idx.dtype == torch.int32
    _bf16(x, (T, d))
    dev = x.device
    P = T * k
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(P, 1), dtype=torch.int32, device=dev)[:P]
    inv = torch.empty(max(P, 1), dtype=torch.int32, device=dev)[:P]
    xp = torch.zeros(P, d, dtype=torch.bfloat16, device=dev)
    _call("moe_permute", _p(topk_idx), _p(x), T, d, E, k, _p(counts), _p(offsets), _p(perm), _p(inv), _p(xp),
          _p(ws), ws.numel(), _stream(stream))
    return counts, offsets, perm, inv, xp


def moe_grouped_gemm(xp, counts, offsets, perm, topk_w, W1, W3, W2, T: int, k: int, ws: torch.Tensor,
                     h=None, y_p=None, stream=None):
    E, f, d = W1.shape
    _bf16(W1), _bf16(W3, (E, f, d)), _bf16(W2, (E, d, f)), _bf16(xp, (T * k, d))
    dev = xp.device
    h = torch.zeros(T * k, f, dtype=torch.bfloat16, device=dev) if h is None else h
    y_p = torch.zeros(T * k, d, dtype=torch.bfloat16, device=dev) if y_p is None else y_p
    _call("moe_grouped_gemm", _p(xp), _p(counts), _p(offsets), _p(perm), _p(topk_w.reshape(-1)), _p(W1), _p(W3),
          _p(W2), T, d, f, E, k, _p(h), _p(y_p), _p(ws), ws.numel(), _stream(stream))
    return h, y_p


def moe_combine(y_p, inv_perm, T: int, k: int, shared_out=None, out=None, stream=None):
    d = y_p.shape[1]
    out = torch.empty(T, d, dtype=torch.bfloat16, device=y_p.device) if out is None else out
    _call("moe_combine", _p(y_p), _p(inv_perm), _p(shared_out), T, k, d, _p(out), _stream(stream))
    return out


def moe_layer_forward(x, Wg, bias, W1, W3, W2, k: int, ws: torch.Tensor, Ws1=None, Ws3=None, Ws2=None,
                      out=None, stream=None):
    T, d = x.shape
    E, f, _ = W1.shape
    fs = 0 if Ws1 is None else Ws1.shape[0]
    _bf16(x), _bf16(Wg, (E, d)), _bf16(W1, (E, f, d)), _bf16(W3, (E, f, d)), _bf16(W2, (E, d, f))
    out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device) if out is None else out
    _call("moe_layer_forward", _p(x), _p(Wg), _p(bias), _p(W1), _p(W3), _p(W2), _p(Ws1), _p(Ws3), _p(Ws2), fs,
          T, d, f, E, k, _p(out), _p(ws), ws.numel(), _stream(stream))
    return out


WS_TENSORS = ("logits", "topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm", "xp", "h", "y_p", "hs", "ys",
              "plan")
PLAN_INTS = 8 + 6 * 513 + 2 * 514       # MOE_PLAN_INTS


def workspace_views(ws: torch.Tensor, T: int, d: int, f: int, E: int, k: int, f_shared: int = 0):
    """Torch views of the layer intermediates that moe_layer_forward leaves in ``ws``."""
    P = T * k
    shapes = {"logits": ((T, E), torch.float32), "topk_idx": ((T, k), torch.int32), "topk_w": ((T, k), torch.float32),
              "counts": ((E,), torch.int32), "offsets": ((E + 1,), torch.int32), "perm": ((P,), torch.int32),
              "inv_perm": ((P,), torch.int32), "xp": ((P, d), torch.bfloat16), "h": ((P, f), torch.bfloat16),
              "y_p": ((P, d), torch.bfloat16), "hs": ((T if f_shared else 0, f_shared), torch.bfloat16),
              "ys": ((T if f_shared else 0, d), torch.bfloat16), "plan": ((PLAN_INTS,), torch.int32)}
    base = ws.data_ptr()
    views = {}
    for i, name in enumerate(WS_TENSORS):
        ptr = moe_workspace_tensor(ws, T, d, f, E, k, f_shared, i)
        shape, dt = shapes[name]
        n = 1
        for s in shape:
            n *= s
        off = ptr - base
        nbytes = n * torch.tensor([], dtype=dt).element_size()
        views[name] = ws[off:off + nbytes].view(dt).view(shape)
    return views


# ---------------------------------------------------------------- FP8 path

def moe_quantize_fp8_rows(x: torch.Tensor, stream=None):
    """1 x 128 blocks along rows: bf16 [R, C] -> (e4m3 codes uint8 [R, C], fp32 scales [R, C/128])."""
    R, Cc = x.shape
    _bf16(x)
    q = torch.empty(R, Cc, dtype=torch.uint8, device=x.device)
    sc = torch.empty(R, Cc // 128, dtype=torch.float32, device=x.device)
    _call("moe_quantize_fp8_rows", _p(x), R, Cc, _p(q), _p(sc), _stream(stream))
    return q, sc


def moe_quantize_fp8_blocks(W: torch.Tensor, stream=None):
    """128 x 128 blocks: bf16 [R, C] (or [E, R', C], taken as [E*R', C]) -> (codes, scales [R/128, C/128])."""
    W2d = W.reshape(-1, W.shape[-1])
    _bf16(W2d)
    R, Cc = W2d.shape
    q = torch.empty(W.shape, dtype=torch.uint8, device=W.device)
    sc = torch.empty(R // 128, Cc // 128, dtype=torch.float32, device=W.device)
    _call("moe_quantize_fp8_blocks", _p(W2d), R, Cc, _p(q), _p(sc), _stream(stream))
    return q, sc


def quantize_layer_fp8(w: dict, stream=None) -> dict:
    """The expert weights of a layer (W1, W3, W2 and optionally Ws1, Ws3, Ws2) in e4m3 with 128 x 128 scales."""
    out = {}
    for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2"):
        if w.get(n) is not None:
            out[n + "q"], out[n + "s"] = moe_quantize_fp8_blocks(w[n], stream)
    return out


def moe_workspace_size_fp8(T: int, d: int, f: int, E: int, k: int, f_shared: int = 0) -> int:
    n = C.c_size_t(0)
    _call("moe_workspace_size_fp8", T, d, f, E, k, f_shared, C.byref(n))
    return int(n.value)


def new_workspace_fp8(T: int, d: int, f: int, E: int, k: int, f_shared: int = 0, device=None, stream=None):
    n = moe_workspace_size_fp8(T, d, f, E, k, f_shared)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device or torch.device("cuda"))
    moe_workspace_init(ws, T, E, k, stream)
    return ws


def moe_layer_forward_fp8(x, Wg, bias, Q: dict, k: int, ws: torch.Tensor, out=None, stream=None):
    """FP8 layer; Q holds W1q/W1s, W3q/W3s, W2q/W2s (and Ws1q/Ws1s, ... for the shared expert)."""
    T, d = x.shape
    E, f, _ = Q["W1q"].shape
    fs = 0 if Q.get("Ws1q") is None else Q["Ws1q"].shape[0]
    _bf16(x), _bf16(Wg, (E, d))
    out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device) if out is None else out
    g = lambda n: _p(Q.get(n))
    _call("moe_layer_forward_fp8", _p(x), _p(Wg), _p(bias), g("W1q"), g("W1s"), g("W3q"), g("W3s"), g("W2q"),
          g("W2s"), g("Ws1q"), g("Ws1s"), g("Ws3q"), g("Ws3s"), g("Ws2q"), g("Ws2s"), fs, T, d, f, E, k, _p(out),
          _p(ws), ws.numel(), _stream(stream))
    return out


# ---------------------------------------------------------------- FP4 weights

def moe_quantize_fp4_rows(W: torch.Tensor, stream=None):
    """1 x 32 blocks along rows: bf16 [R, C] (or [E, R', C], taken as [E*R', C]) -> (packed e2m1
    codes uint8 [..., C/2], UE8M0 scale atoms uint8 [R/128, C/128, 512])."""
    W2d = W.reshape(-1, W.shape[-1])
    _bf16(W2d)
    R, Cc = W2d.shape
    q = torch.empty(*W.shape[:-1], Cc // 2, dtype=torch.uint8, device=W.device)
    atoms = torch.empty(R // 128, Cc // 128, 512, dtype=torch.uint8, device=W.device)
    _call("moe_quantize_fp4_rows", _p(W2d), R, Cc, _p(q), _p(atoms), _stream(stream))
    return q, atoms


def quantize_layer_fp4(w: dict, stream=None) -> dict:
    """The expert weights of a layer (W1, W3, W2 and optionally Ws1, Ws3, Ws2) as packed e2m1 with scale atoms."""
    out = {}
    for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2"):
        if w.get(n) is not None:
            out[n + "q"], out[n + "sf"] = moe_quantize_fp4_rows(w[n], stream)
    return out


def moe_layer_forward_fp4(x, Wg, bias, Q: dict, k: int, ws: torch.Tensor, out=None, stream=None):
    """FP4-weight layer; Q holds W1q/W1sf, W3q/W3sf, W2q/W2sf (and Ws1q/Ws1sf, ... for the shared expert)."""
    T, d = x.shape
    E, f, _ = Q["W1q"].shape
    fs = 0 if Q.get("Ws1q") is None else Q["Ws1q"].shape[0]
    _bf16(x), _bf16(Wg, (E, d))
    out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device) if out is None else out
    g = lambda n: _p(Q.get(n))
    _call("moe_layer_forward_fp4", _p(x), _p(Wg), _p(bias), g("W1q"), g("W1sf"), g("W3q"), g("W3sf"), g("W2q"),
          g("W2sf"), g("Ws1q"), g("Ws1sf"), g("Ws3q"), g("Ws3sf"), g("Ws2q"), g("Ws2sf"), fs, T, d, f, E, k, _p(out),
          _p(ws), ws.numel(), _stream(stream))
    return out


WS_TENSORS_FP8 = ("logits", "topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm", "x8", "sx", "xp8", "sxp",
                  "h8", "sh", "y_p", "hs8", "shs", "ys", "sxT", "plan")


def workspace_views_fp8(ws: torch.Tensor, T: int, d: int, f: int, E: int, k: int, f_shared: int = 0):
    P, Ts = T * k, (T if f_shared else 0)
    P4, T4 = (P + 3) // 4 * 4, (T + 3) // 4 * 4     # K-block-major scale rows are padded to 4 entries
    shapes = {"logits": ((T, E), torch.float32), "topk_idx": ((T, k), torch.int32), "topk_w": ((T, k), torch.float32),
              "counts": ((E,), torch.int32), "offsets": ((E + 1,), torch.int32), "perm": ((P,), torch.int32),
              "inv_perm": ((P,), torch.int32), "x8": ((T, d), torch.uint8), "sx": ((T, d // 128), torch.float32),
              "xp8": ((P, d), torch.uint8), "sxp": ((d // 128, P4), torch.float32), "h8": ((P, f), torch.uint8),
              "sh": ((f // 128, P4), torch.float32), "y_p": ((P, d), torch.bfloat16),
              "hs8": ((Ts, f_shared), torch.uint8), "shs": ((f_shared // 128, T4 if Ts else 0), torch.float32),
              "ys": ((Ts, d), torch.bfloat16), "sxT": ((d // 128, T4 if Ts else 0), torch.float32),
              "plan": ((PLAN_INTS,), torch.int32)}
    base = ws.data_ptr()
    views = {}
    for i, name in enumerate(WS_TENSORS_FP8):
        out = C.c_void_p(0)
        _call("moe_workspace_tensor_fp8", _p(ws), T, d, f, E, k, f_shared, i, C.byref(out))
        shape, dt = shapes[name]
        n = 1
        for s_ in shape:
            n *= s_
        off = int(out.value or 0) - base
        nbytes = n * torch.tensor([], dtype=dt).element_size()
        views[name] = ws[off:off + nbytes].view(dt).view(shape)
    return views
