"""fp64 CPU oracle for the fused MoE layer forward (ctypes wrapper of moe_oracle.c).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  It shares no
code with the CUDA path and never imports it; inputs come from the seeded
generator module, never from the CUDA path.

Functions follow the steps of the layer as the pages describe it (Decoding the
Skew, abstract; GC-MoE, abstract); the C source states each step's definition
and every reading taken where the pages are silent.  All arrays are numpy; bf16
tensors travel as their raw uint16 bit patterns.
"""

from __future__ import annotations

import ctypes as C
import os
from typing import Dict, Optional, Sequence

import numpy as np

from . import build as _build

_lib = None


def load(path: str) -> C.CDLL:
    """Open an oracle build at ``path`` and declare its entry points."""
    L = C.CDLL(path)
    i64, i32p = C.c_int64, C.POINTER(C.c_int32)
    u16p, f32p, f64p = C.POINTER(C.c_uint16), C.POINTER(C.c_float), C.POINTER(C.c_double)
    u16pp = C.POINTER(u16p)
    L.oracle_default_threads.restype = C.c_int
    L.oracle_router_logits.argtypes = [u16p, u16p, f32p, i64, i64, i64, f64p]
    L.oracle_topk.argtypes = [f32p, i64, i64, i64, i32p, f64p]
    L.oracle_permutation.argtypes = [i32p, i64, i64, i64, i32p, i32p, i32p, i32p]
    L.oracle_moe_ffn.argtypes = [u16p, u16pp, u16pp, u16pp, i64, i64, i64, i32p, f64p, i64,
                                 u16p, u16p, u16p, i64, C.POINTER(i64), i64, f64p, C.c_int]
    for fn in ("oracle_router_logits", "oracle_topk", "oracle_permutation", "oracle_moe_ffn"):
        getattr(L, fn).restype = C.c_int
    u8p = C.POINTER(C.c_uint8)
    u8pp, f64pp = C.POINTER(u8p), C.POINTER(f64p)
    L.oracle_e4m3_decode.argtypes = [C.c_uint8]
    L.oracle_e4m3_decode.restype = C.c_double
    L.oracle_e4m3_encode.argtypes = [C.c_double]
    L.oracle_e4m3_encode.restype = C.c_uint8
    L.oracle_e4m3_encode_fast.argtypes = [C.c_double]
    L.oracle_e4m3_encode_fast.restype = C.c_uint8
    L.oracle_fp8_block_scale.argtypes = [C.c_double]
    L.oracle_fp8_block_scale.restype = C.c_double
    L.oracle_quantize_rows_fp8.argtypes = [u16p, i64, i64, u8p, f64p]
    L.oracle_quantize_blocks_fp8.argtypes = [u16p, i64, i64, u8p, f64p]
    L.oracle_moe_ffn_fp8.argtypes = [u8p, f64p, u8pp, f64pp, u8pp, f64pp, u8pp, f64pp, i64, i64, i64, i32p, f64p,
                                     i64, u8p, f64p, u8p, f64p, u8p, f64p, i64, C.POINTER(i64), i64, f64p, C.c_int]
    L.oracle_expert_h_fp8.argtypes = [u8p, f64p, u8p, f64p, u8p, f64p, i64, i64, u8p, f64p]
    L.oracle_e2m1_decode.argtypes = [C.c_uint8]
    L.oracle_e2m1_decode.restype = C.c_double
    L.oracle_e2m1_encode.argtypes = [C.c_double]
    L.oracle_e2m1_encode.restype = C.c_uint8
    L.oracle_fp4_block_scale.argtypes = [C.c_double]
    L.oracle_fp4_block_scale.restype = C.c_double
    L.oracle_quantize_rows_fp4.argtypes = [u16p, i64, i64, u8p, f64p]
    L.oracle_quantize_rows_fp4.restype = C.c_int
    L.oracle_moe_ffn_fp4.argtypes = L.oracle_moe_ffn_fp8.argtypes
    L.oracle_moe_ffn_fp4.restype = C.c_int
    for fn in ("oracle_quantize_rows_fp8", "oracle_quantize_blocks_fp8", "oracle_moe_ffn_fp8",
               "oracle_expert_h_fp8"):
        getattr(L, fn).restype = C.c_int
    return L


def lib() -> C.CDLL:
    """The oracle library in use (built from moe_oracle.c on first call)."""
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


def use(L: C.CDLL) -> C.CDLL:
    """Swap the library the module functions call; returns the previous one."""
    global _lib
    prev, _lib = _lib, L
    return prev


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise OracleError(f"{what} failed with status {rc}")


def _ptr(a: Optional[np.ndarray], ct):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(C.POINTER(ct))


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 inputs travel as uint16 bit patterns"
    return a


def default_threads() -> int:
    return int(lib().oracle_default_threads())


def router_logits(x: np.ndarray, Wg: np.ndarray, bias: Optional[np.ndarray]) -> np.ndarray:
    """fp64 logits L[t,e] = sum_c x[t,c] Wg[e,c] + b[e]."""
    x, Wg = _u16(x), _u16(Wg)
    T, d = x.shape
    E = Wg.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    L = np.empty((T, E), dtype=np.float64)
    _check(lib().oracle_router_logits(_ptr(x, C.c_uint16), _ptr(Wg, C.c_uint16), _ptr(b, C.c_float),
                                      T, d, E, _ptr(L, C.c_double)), "router_logits")
    return L


def topk(L32: np.ndarray, k: int):
    """Top-k of fp32 logits (descending, ties to the lower index) and fp64 softmax gates."""
    L32 = np.ascontiguousarray(L32, dtype=np.float32)
    T, E = L32.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    _check(lib().oracle_topk(_ptr(L32, C.c_float), T, E, k, _ptr(idx, C.c_int32), _ptr(w, C.c_double)),
           "topk")
    return idx, w


def permutation(idx: np.ndarray, E: int):
    """counts [E], offsets [E+1], perm [P], inv_perm [P] of the stable expert-major order."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    P = T * k
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(P, dtype=np.int32)
    inv = np.empty(P, dtype=np.int32)
    _check(lib().oracle_permutation(_ptr(idx, C.c_int32), T, k, E, _ptr(counts, C.c_int32),
                                    _ptr(offsets, C.c_int32), _ptr(perm, C.c_int32), _ptr(inv, C.c_int32)),
           "permutation")
    return counts, offsets, perm, inv


def moe_ffn(x: np.ndarray, W1: Sequence, W3: Sequence, W2: Sequence, idx: np.ndarray, w: np.ndarray,
            shared: Optional[Dict[str, np.ndarray]] = None, tokens: Optional[np.ndarray] = None,
            nthreads: int = 0) -> np.ndarray:
    """fp64 y[t] = sum_j w[t,j] FFN_{idx[t,j]}(x_t) (+ shared FFN(x_t)) for the listed tokens.

    W1/W3/W2 are either stacked arrays [E,f,d]/[E,f,d]/[E,d,f] or per-expert
    sequences whose entries may be None for experts no listed token uses.
    """
    x = _u16(x)
    T, d = x.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    k = idx.shape[1]
    E = len(W1)
    W1l = [None if a is None else _u16(a) for a in W1]
    W3l = [None if a is None else _u16(a) for a in W3]
    W2l = [None if a is None else _u16(a) for a in W2]
    f = next(a.shape[0] for a in W1l if a is not None)
    ptr_t = C.POINTER(C.c_uint16)
    arr = lambda lst: (ptr_t * E)(*[ptr_t() if a is None else _ptr(a, C.c_uint16) for a in lst])
    p1, p3, p2 = arr(W1l), arr(W3l), arr(W2l)
    fs = 0
    s1 = s3 = s2 = None
    if shared is not None:
        s1, s3, s2 = _u16(shared["Ws1"]), _u16(shared["Ws3"]), _u16(shared["Ws2"])
        fs = s1.shape[0]
    if tokens is None:
        tok = None
        ntok = T
    else:
        tok = np.ascontiguousarray(tokens, dtype=np.int64)
        assert tok.size == 0 or (tok.min() >= 0 and tok.max() < T)
        ntok = tok.size
    out = np.empty((ntok, d), dtype=np.float64)
    _check(lib().oracle_moe_ffn(_ptr(x, C.c_uint16), p1, p3, p2, d, f, E, _ptr(idx, C.c_int32),
                                _ptr(w, C.c_double), k, _ptr(s1, C.c_uint16), _ptr(s3, C.c_uint16),
                                _ptr(s2, C.c_uint16), fs, _ptr(tok, C.c_int64), ntok,
                                _ptr(out, C.c_double), int(nthreads)), "moe_ffn")
    return out


def moe_layer(x, Wg, bias, W1, W3, W2, k: int, shared=None, tokens=None, nthreads: int = 0):
    """The whole layer: fp64 logits, rounded once to fp32 for the top-k decision,
    fp64 gates, the stable permutation, and the fp64 expert FFNs of ``tokens``."""
    L64 = router_logits(x, Wg, bias)
    L32 = L64.astype(np.float32)
    idx, w = topk(L32, k)
    counts, offsets, perm, inv = permutation(idx, len(W1))
    out = moe_ffn(x, W1, W3, W2, idx, w, shared=shared, tokens=tokens, nthreads=nthreads)
    return dict(L64=L64, L32=L32, idx=idx, w=w, counts=counts, offsets=offsets, perm=perm,
                inv_perm=inv, out=out)


# ---------------------------------------------------------------- FP8 (e4m3, power-of-two block scales)

def e4m3_decode(code: int) -> float:
    return float(lib().oracle_e4m3_decode(int(code)))


def e4m3_encode(v: float) -> int:
    """Nearest e4m3 code (ties to even), saturating to +-448: the definition (walks every code)."""
    return int(lib().oracle_e4m3_encode(float(v)))


def e4m3_encode_fast(v: float) -> int:
    """The same rounding computed from the binary exponent (used by the quantisers)."""
    return int(lib().oracle_e4m3_encode_fast(float(v)))


def fp8_block_scale(amax: float) -> float:
    """Smallest power of two s with amax / s <= 448 (1 for amax = 0)."""
    return float(lib().oracle_fp8_block_scale(float(amax)))


def quantize_rows_fp8(x: np.ndarray):
    """1 x 128 blocks along rows: bf16 bits [R, C] -> (e4m3 codes [R, C], scales [R, C/128])."""
    x = _u16(x)
    R, Cc = x.shape
    q = np.empty((R, Cc), dtype=np.uint8)
    sc = np.empty((R, Cc // 128), dtype=np.float64)
    _check(lib().oracle_quantize_rows_fp8(_ptr(x, C.c_uint16), R, Cc, _ptr(q, C.c_uint8), _ptr(sc, C.c_double)),
           "quantize_rows_fp8")
    return q, sc


def quantize_blocks_fp8(W: np.ndarray):
    """128 x 128 blocks: bf16 bits [R, C] -> (e4m3 codes [R, C], scales [R/128, C/128])."""
    W = _u16(W)
    R, Cc = W.shape
    q = np.empty((R, Cc), dtype=np.uint8)
    sc = np.empty((R // 128, Cc // 128), dtype=np.float64)
    _check(lib().oracle_quantize_blocks_fp8(_ptr(W, C.c_uint16), R, Cc, _ptr(q, C.c_uint8), _ptr(sc, C.c_double)),
           "quantize_blocks_fp8")
    return q, sc


def moe_ffn_fp8(xq, sx, W1q, s1, W3q, s3, W2q, s2, idx, w, shared=None, tokens=None, nthreads: int = 0):
    """fp64 y[t] = sum_j w[t,j] FFN8_e(x^_t) (+ shared) on dequantised e4m3 operands, with h
    requantised in 1 x 128 blocks before the down projection.  Per-expert lists may hold None
    for experts no listed token uses; shared = dict(W1q, s1, W3q, s3, W2q, s2)."""
    return _moe_ffn_lowp(lib().oracle_moe_ffn_fp8, "moe_ffn_fp8", xq, sx, W1q, s1, W3q, s3, W2q, s2, idx, w, shared,
                         tokens, nthreads)


def _moe_ffn_lowp(fn, what, xq, sx, W1q, s1, W3q, s3, W2q, s2, idx, w, shared, tokens, nthreads):
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    sx = np.ascontiguousarray(sx, dtype=np.float64)
    T, d = xq.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    k = idx.shape[1]
    E = len(W1q)
    f = next(a.shape[0] for a in W1q if a is not None)
    keep = []

    def arr(lst, ct, dt):
        vals = []
        for a in lst:
            if a is None:
                vals.append(C.POINTER(ct)())
            else:
                a = np.ascontiguousarray(a, dtype=dt)
                keep.append(a)
                vals.append(_ptr(a, ct))
        return (C.POINTER(ct) * E)(*vals)

    pw1, pw3, pw2 = arr(W1q, C.c_uint8, np.uint8), arr(W3q, C.c_uint8, np.uint8), arr(W2q, C.c_uint8, np.uint8)
    ps1, ps3, ps2 = arr(s1, C.c_double, np.float64), arr(s3, C.c_double, np.float64), arr(s2, C.c_double, np.float64)
    fs = 0
    sh = [None] * 6
    if shared is not None:
        sh = [np.ascontiguousarray(shared[n], dtype=(np.uint8 if n.endswith("q") else np.float64))
              for n in ("W1q", "s1", "W3q", "s3", "W2q", "s2")]
        fs = sh[0].shape[0]
    if tokens is None:
        tok, ntok = None, T
    else:
        tok = np.ascontiguousarray(tokens, dtype=np.int64)
        ntok = tok.size
    out = np.empty((ntok, d), dtype=np.float64)
    _check(fn(_ptr(xq, C.c_uint8), _ptr(sx, C.c_double), pw1, ps1, pw3, ps3, pw2, ps2, d, f, E,
              _ptr(idx, C.c_int32), _ptr(w, C.c_double), k,
              _ptr(sh[0], C.c_uint8), _ptr(sh[1], C.c_double), _ptr(sh[2], C.c_uint8),
              _ptr(sh[3], C.c_double), _ptr(sh[4], C.c_uint8), _ptr(sh[5], C.c_double), fs,
              _ptr(tok, C.c_int64), ntok, _ptr(out, C.c_double), int(nthreads)), what)
    return out


def expert_h_fp8(xq, sx, W1q, s1, W3q, s3):
    """The requantised h of one FP8 expert on one token: h = silu(W1^ x^) * (W3^ x^) in fp64
    on dequantised operands, then 1 x 128 blocks along f -> (codes [f], scales [f/128]).
    xq [d] codes with sx [d/128]; W1q/W3q [f, d] with s1/s3 [f/128, d/128]."""
    xq = np.ascontiguousarray(xq, dtype=np.uint8).ravel()
    sx = np.ascontiguousarray(sx, dtype=np.float64).ravel()
    W1q = np.ascontiguousarray(W1q, dtype=np.uint8)
    W3q = np.ascontiguousarray(W3q, dtype=np.uint8)
    s1 = np.ascontiguousarray(s1, dtype=np.float64)
    s3 = np.ascontiguousarray(s3, dtype=np.float64)
    f, d = W1q.shape
    hq = np.empty(f, dtype=np.uint8)
    sh = np.empty(f // 128, dtype=np.float64)
    _check(lib().oracle_expert_h_fp8(_ptr(W1q, C.c_uint8), _ptr(s1, C.c_double), _ptr(W3q, C.c_uint8),
                                     _ptr(s3, C.c_double), _ptr(xq, C.c_uint8), _ptr(sx, C.c_double), d, f,
                                     _ptr(hq, C.c_uint8), _ptr(sh, C.c_double)), "expert_h_fp8")
    return hq, sh


# ---------------------------------------------------------------- FP4 weights (e2m1, 1 x 32 power-of-two scales)

def e2m1_decode(code: int) -> float:
    return float(lib().oracle_e2m1_decode(int(code)))


def e2m1_encode(v: float) -> int:
    """Nearest e2m1 code (ties to even), saturating to +-6."""
    return int(lib().oracle_e2m1_encode(float(v)))


def fp4_block_scale(amax: float) -> float:
    """Smallest power of two s with amax / s <= 6 (1 for amax = 0)."""
    return float(lib().oracle_fp4_block_scale(float(amax)))


def quantize_rows_fp4(W: np.ndarray):
    """1 x 32 blocks along rows: bf16 bits [R, C] -> (e2m1 codes [R, C], one per byte; scales [R, C/32])."""
    W = _u16(W)
    R, Cc = W.shape
    q = np.empty((R, Cc), dtype=np.uint8)
    sc = np.empty((R, Cc // 32), dtype=np.float64)
    _check(lib().oracle_quantize_rows_fp4(_ptr(W, C.c_uint16), R, Cc, _ptr(q, C.c_uint8), _ptr(sc, C.c_double)),
           "quantize_rows_fp4")
    return q, sc


def moe_ffn_fp4(xq, sx, W1q, s1, W3q, s3, W2q, s2, idx, w, shared=None, tokens=None, nthreads: int = 0):
    """fp64 y[t] = sum_j w[t,j] FFN4_e(x^_t) (+ shared): e4m3 activations (1 x 128 scales), e2m1 weights
    (one code per byte) with 1 x 32 scales ([f, d/32] for W1/W3, [d, f/32] for W2), h requantised to
    e4m3 in 1 x 128 blocks before the down projection.  Per-expert lists may hold None for experts no
    listed token uses; shared = dict(W1q, s1, W3q, s3, W2q, s2)."""
    return _moe_ffn_lowp(lib().oracle_moe_ffn_fp4, "moe_ffn_fp4", xq, sx, W1q, s1, W3q, s3, W2q, s2, idx, w, shared,
                         tokens, nthreads)
