"""The C-ABI library without a GPU: it loads, exports every declared entry
point, sizes workspaces, and rejects bad arguments on the host before any
CUDA call."""

import ctypes as C
import os
import re

import pytest

from grouped_gemm_02_b200 import build, moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return moe.lib()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src)))


def test_header_declares_the_api():
    names = declared_symbols()
    assert set(moe.EXPORTS) == set(names), names


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), f"{name} missing from {moe.library_path()}"
    out = os.popen(f"nm -D --defined-only {moe.library_path()}").read()
    exported = set(re.findall(r" T (moe_\w+)", out))
    assert exported == set(declared_symbols())


def test_status_strings(L):
    assert moe.moe_status_string(0) == "ok"
    assert "workspace" in moe.moe_status_string(-3)


def test_workspace_size_monotone(L):
    a = moe.moe_workspace_size(32, 2048, 1024, 64, 8)
    b = moe.moe_workspace_size(64, 2048, 1024, 64, 8)
    c = moe.moe_workspace_size(32, 2048, 1024, 64, 8, 2048)
    assert 0 < a < b and a < c
    assert a % 256 == 0
    # the big intermediates are counted: xp, y_p [P,d] and h [P,f] in bf16
    P = 32 * 8
    assert a >= P * 2048 * 2 * 2 + P * 1024 * 2
    with pytest.raises(moe.MoEError):
        moe.moe_workspace_size(-1, 2048, 1024, 64, 8)
    with pytest.raises(moe.MoEError):
        moe.moe_workspace_size(1, 2048, 1024, 513, 8)


FAKE = C.c_void_p(0x10000)   # never dereferenced: every call below fails its host checks first


def _layer(L, **kw):
    a = dict(x=FAKE, Wg=FAKE, bias=None, W1=FAKE, W3=FAKE, W2=FAKE, Ws1=None, Ws3=None, Ws2=None, fs=0,
             T=4, d=128, f=128, E=4, k=2, out=FAKE, ws=FAKE, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return L.moe_layer_forward(a["x"], a["Wg"], a["bias"], a["W1"], a["W3"], a["W2"], a["Ws1"], a["Ws3"],
                               a["Ws2"], a["fs"], a["T"], a["d"], a["f"], a["E"], a["k"], a["out"], a["ws"],
                               a["ws_bytes"], a["stream"])


def test_host_argument_checks(L):
    assert _layer(L, x=None) == -1
    assert _layer(L, k=5, E=4) == -1          # k > E
    assert _layer(L, k=9, E=16) == -1         # k > 8
    assert _layer(L, E=513) == -1
    assert _layer(L, T=-1) == -1
    assert _layer(L, d=100) == -2             # d not a multiple of 64
    assert _layer(L, f=96) == -2
    assert _layer(L, x=C.c_void_p(0x10008)) == -2   # misaligned pointer
    assert _layer(L, ws_bytes=1024) == -3
    assert _layer(L, fs=64) == -1             # shared expert without weights
    assert _layer(L, T=0) == 0                # empty batch: nothing to do
    assert L.moe_combine(None, FAKE, None, 4, 2, 128, FAKE, None) == -1
    assert L.moe_topk(FAKE, 4, 8, 9, FAKE, FAKE, FAKE, None) == -1
    assert L.moe_permute(FAKE, FAKE, 4, 128, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None) == -3


def _layer_fp8(L, **kw):
    a = dict(x=FAKE, Wg=FAKE, bias=None, W1q=FAKE, W1s=FAKE, W3q=FAKE, W3s=FAKE, W2q=FAKE, W2s=FAKE, Ws1q=None,
             Ws1s=None, Ws3q=None, Ws3s=None, Ws2q=None, Ws2s=None, fs=0, T=4, d=256, f=256, E=4, k=2, out=FAKE,
             ws=FAKE, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return L.moe_layer_forward_fp8(a["x"], a["Wg"], a["bias"], a["W1q"], a["W1s"], a["W3q"], a["W3s"], a["W2q"],
                                   a["W2s"], a["Ws1q"], a["Ws1s"], a["Ws3q"], a["Ws3s"], a["Ws2q"], a["Ws2s"], a["fs"],
                                   a["T"], a["d"], a["f"], a["E"], a["k"], a["out"], a["ws"], a["ws_bytes"],
                                   a["stream"])


def test_fp8_host_argument_checks(L):
    assert _layer_fp8(L, d=192) == -2          # a multiple of 64 but not of 128
    assert _layer_fp8(L, f=64) == -2
    assert _layer_fp8(L, fs=64) == -2
    assert _layer_fp8(L, d=16512) == -1        # past the 16384 limit of the weight-scale registers
    assert _layer_fp8(L, f=16512) == -1
    assert _layer_fp8(L, W2s=None) == -1
    assert _layer_fp8(L, fs=128) == -1         # shared expert without weights
    assert _layer_fp8(L, x=C.c_void_p(0x10008)) == -2
    assert _layer_fp8(L, ws_bytes=1024) == -3
    assert _layer_fp8(L, T=0) == 0
    assert L.moe_quantize_fp8_rows(FAKE, 4, 100, FAKE, FAKE, None) == -2
    assert L.moe_quantize_fp8_rows(FAKE, -1, 128, FAKE, FAKE, None) == -1
    assert L.moe_quantize_fp8_rows(FAKE, 4, 128, None, FAKE, None) == -1
    assert L.moe_quantize_fp8_rows(FAKE, 0, 128, FAKE, FAKE, None) == 0
    assert L.moe_quantize_fp8_blocks(FAKE, 100, 128, FAKE, FAKE, None) == -2
    assert L.moe_quantize_fp8_blocks(FAKE, 128, 128, FAKE, None, None) == -1


def _layer_fp4(L, **kw):
    a = dict(x=FAKE, Wg=FAKE, bias=None, W1q=FAKE, W1sf=FAKE, W3q=FAKE, W3sf=FAKE, W2q=FAKE, W2sf=FAKE, Ws1q=None,
             Ws1sf=None, Ws3q=None, Ws3sf=None, Ws2q=None, Ws2sf=None, fs=0, T=4, d=256, f=256, E=4, k=2, out=FAKE,
             ws=FAKE, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return L.moe_layer_forward_fp4(a["x"], a["Wg"], a["bias"], a["W1q"], a["W1sf"], a["W3q"], a["W3sf"], a["W2q"],
                                   a["W2sf"], a["Ws1q"], a["Ws1sf"], a["Ws3q"], a["Ws3sf"], a["Ws2q"], a["Ws2sf"],
                                   a["fs"], a["T"], a["d"], a["f"], a["E"], a["k"], a["out"], a["ws"], a["ws_bytes"],
                                   a["stream"])


def test_fp4_host_argument_checks(L):
    """The FP4-weight layer and row quantiser refuse bad arguments on the host, before any device work."""
    assert _layer_fp4(L, d=192) == -2          # a multiple of 64 but not of 128
    assert _layer_fp4(L, f=64) == -2
    assert _layer_fp4(L, fs=64) == -2
    assert _layer_fp4(L, d=16512) == -1
    assert _layer_fp4(L, W2sf=None) == -1      # a weight's scale atoms missing
    assert _layer_fp4(L, fs=128) == -1         # shared expert without weights
    assert _layer_fp4(L, fs=128, Ws1q=FAKE, Ws3q=FAKE, Ws2q=FAKE, Ws1sf=FAKE, Ws3sf=FAKE, Ws2sf=None) == -1
    assert _layer_fp4(L, W1sf=C.c_void_p(0x10008)) == -2   # scale atoms not 16-byte aligned
    assert _layer_fp4(L, x=C.c_void_p(0x10008)) == -2
    assert _layer_fp4(L, ws_bytes=1024) == -3
    assert _layer_fp4(L, T=0) == 0
    assert L.moe_quantize_fp4_rows(FAKE, 100, 128, FAKE, FAKE, None) == -2    # rows not a multiple of 128
    assert L.moe_quantize_fp4_rows(FAKE, 128, 96, FAKE, FAKE, None) == -2     # cols not a multiple of 128
    assert L.moe_quantize_fp4_rows(FAKE, -128, 128, FAKE, FAKE, None) == -1
    assert L.moe_quantize_fp4_rows(FAKE, 128, 128, None, FAKE, None) == -1
    assert L.moe_quantize_fp4_rows(FAKE, 128, 128, FAKE, C.c_void_p(0x10008), None) == -2
    assert L.moe_quantize_fp4_rows(FAKE, 0, 128, FAKE, FAKE, None) == 0


def test_product_path_refuses_missing_library(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "library_path", lambda: str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        moe.lib()


# ------------------------------------------------------------------ workspace layout (host arithmetic only)

PLAN_BYTES = moe.PLAN_INTS * 4


def _bf16_layout(T, d, f, E, k, fs):
    """Byte sizes and alignments of the layer intermediates, from the header's shapes."""
    P, Ts = T * k, (T if fs else 0)
    return [("logits", T * E * 4, 4), ("topk_idx", P * 4, 4), ("topk_w", P * 4, 4), ("counts", E * 4, 4),
            ("offsets", (E + 1) * 4, 4), ("perm", P * 4, 4), ("inv_perm", P * 4, 4), ("xp", P * d * 2, 256),
            ("h", P * f * 2, 256), ("y_p", P * d * 2, 256), ("hs", Ts * fs * 2, 256), ("ys", Ts * d * 2, 256),
            ("plan", PLAN_BYTES, 256)]


def _fp8_layout(T, d, f, E, k, fs):
    P, Ts = T * k, (T if fs else 0)
    P4, T4 = (P + 3) // 4 * 4, (T + 3) // 4 * 4
    return [("logits", T * E * 4, 4), ("topk_idx", P * 4, 4), ("topk_w", P * 4, 4), ("counts", E * 4, 4),
            ("offsets", (E + 1) * 4, 4), ("perm", P * 4, 4), ("inv_perm", P * 4, 4), ("x8", T * d, 256),
            ("sx", T * (d // 128) * 4, 16), ("xp8", P * d, 256), ("sxp", (d // 128) * P4 * 4, 16),
            ("h8", P * f, 256), ("sh", (f // 128) * P4 * 4, 16), ("y_p", P * d * 2, 256),
            ("hs8", Ts * fs, 256), ("shs", (fs // 128) * (T4 if Ts else 0) * 4, 16), ("ys", Ts * d * 2, 256),
            ("sxT", (d // 128) * (T4 if Ts else 0) * 4, 16), ("plan", PLAN_BYTES, 256)]


@pytest.mark.parametrize("T,d,f,E,k,fs", [(32, 2048, 1024, 64, 8, 0), (1, 256, 512, 8, 2, 0), (37, 7168, 2048, 256, 8, 2048),
                                          (16384, 7168, 2048, 256, 8, 2048), (5, 4096, 14336, 8, 2, 0)])
@pytest.mark.parametrize("fp8", [False, True])
def test_workspace_tensors_disjoint_aligned_inside(L, T, d, f, E, k, fs, fp8):
    layout = (_fp8_layout if fp8 else _bf16_layout)(T, d, f, E, k, fs)
    total = C.c_size_t(0)
    rc = (L.moe_workspace_size_fp8 if fp8 else L.moe_workspace_size)(T, d, f, E, k, fs, C.byref(total))
    assert rc == 0
    base = 1 << 40                      # any 1 KiB-aligned address: the call only adds offsets
    fn = L.moe_workspace_tensor_fp8 if fp8 else L.moe_workspace_tensor
    spans = []
    for which, (name, nbytes, align) in enumerate(layout):
        out = C.c_void_p(0)
        assert fn(C.c_void_p(base), T, d, f, E, k, fs, which, C.byref(out)) == 0
        off = out.value - base
        assert off % align == 0, name
        assert 0 <= off and off + nbytes <= total.value, name
        if nbytes:
            spans.append((off, off + nbytes, name))
    spans.sort()
    for (a0, a1, an), (b0, b1, bn) in zip(spans, spans[1:]):
        assert a1 <= b0, f"{an} overlaps {bn}"
    out = C.c_void_p(0)
    assert fn(C.c_void_p(base), T, d, f, E, k, fs, len(layout), C.byref(out)) != 0   # past the last tensor


def test_status_and_error_codes_agree_across_header_binding_and_library(L):
    src = open(HEADER).read()
    defs = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define (MOE_(?:OK|ERR_\w+|DEVERR_\w+))\s+\(?(-?\d+)u?\)?", src)}
    assert defs["MOE_OK"] == moe.MOE_OK
    for name, val in defs.items():
        if name.startswith("MOE_ERR") or name == "MOE_OK":
            assert val in moe.STATUS, name
            assert L.moe_status_string(val).decode() == moe.STATUS[val], name
        else:
            assert getattr(moe, name[len("MOE_"):]) == val, name
    kernel = open(os.path.join(ROOT, "grouped_gemm_02_b200", "csrc", "common.cuh")).read()
    for name, val in defs.items():
        if name.startswith("MOE_DEVERR"):
            m = re.search(name[len("MOE_"):] + r"\s*=\s*(\d+)", kernel)
            assert m and int(m.group(1)) == val, name


def test_plan_size_agrees_across_header_binding_and_kernels():
    src = open(HEADER).read()
    m = re.search(r"#define MOE_PLAN_INTS \((\d+) \+ (\d+) \* (\d+) \+ (\d+) \* (\d+)\)", src)
    assert m
    a, b, c, d_, e = (int(v) for v in m.groups())
    assert a + b * c + d_ * e == moe.PLAN_INTS
    common = open(os.path.join(ROOT, "grouped_gemm_02_b200", "csrc", "common.cuh")).read()
    assert "constexpr int kMaxExperts = 512;" in common
    assert "kPlanInts = 8 + 6 * kMaxGroups + 2 * (kMaxGroups + 1)" in common
    assert moe.PLAN_INTS == 8 + 6 * 513 + 2 * 514
