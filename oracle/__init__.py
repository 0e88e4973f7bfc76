"""ctypes wrapper around the plain-C MoE oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg use it.  The CUDA library never imports, links or
calls anything here; the two share no code.  Inputs are numpy arrays; bf16
tensors travel as their uint16 storage.

Parity pins (tests/test_oracle.py): bf16 rounding against torch's own
conversion and hand-worked ties; logits against a float64 matrix product;
top-k against a full lexicographic sort; dispatch against numpy's stable
argsort and the pages' 156-token, 8-expert, top-2 worked example (mean 39 rows
per expert); the expert FFN against a dense float64 matrix statement; combine
against dense-masked evaluation (every expert on every token); the E=1, k=1
reduction to a dense SwiGLU FFN; a hand-derived tiny layer; relabelling and
scaling invariants; e4m3 decoding against the format's own table of special
values and every code, encoding against nearest-value search over all codes with
ties to the even code, the quantizer's per-row scale and error bounds, and the
fp8 layer against the bf16 layer on weights that the quantizer represents
exactly; with activations quantized too, the experts against the weight-only
experts on rows the quantizer represents exactly, against a float64 BLAS
statement fed the quantizer's dequantized rows, and against exact per-row
power-of-two scaling, and the layer against its pinned steps.  No function is
left unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_LIB_MT = os.path.join(_HERE, "libmoe_oracle_mt.so")
_libs = {}
_use_mt = False


def _compile(path: str, extra) -> None:
    if not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(_SRC):
        tmp = path + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", *extra,
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, path)


def build(force: bool = False) -> str:
    """Compile the oracle with plain gcc (no vector intrinsics, no fast-math): the
    serial library, and the same source with -fopenmp, whose loops over independent
    tokens and rows run on several threads (same arithmetic per row, same bits)."""
    if force:
        for p in (_LIB, _LIB_MT):
            if os.path.exists(p):
                os.utime(p, (0, 0))
    _compile(_LIB, [])
    _compile(_LIB_MT, ["-fopenmp"])
    return _LIB


def set_threads(n: int) -> int:
    """n > 1: later calls run on the OpenMP build with n threads; n <= 1: the serial
    build.  Returns the thread count now in use."""
    global _use_mt
    _use_mt = n > 1
    return int(lib().oracle_threads(n if n > 1 else 0))


def threads() -> int:
    """Threads the oracle's calls use now."""
    return int(lib().oracle_threads(0))


def _P(t):
    return ctypes.POINTER(t)


def lib():
    path = _LIB_MT if _use_mt else _LIB
    if path not in _libs:
        build()
        _libs[path] = _load(path)
    return _libs[path]


def _load(path):
    L = ctypes.CDLL(path)
    u16, i32, f32, f64, i64 = (ctypes.c_uint16, ctypes.c_int32, ctypes.c_float,
                               ctypes.c_double, ctypes.c_int64)
    c_int = ctypes.c_int
    L.oracle_bf16_to_double.argtypes = [u16]
    L.oracle_bf16_to_double.restype = f64
    L.oracle_round_to_bf16.argtypes = [f64]
    L.oracle_round_to_bf16.restype = u16
    L.oracle_router_logits.argtypes = [_P(u16), _P(f32), _P(f32), i64, c_int, c_int, _P(f64)]
    L.oracle_router_logits.restype = None
    L.oracle_topk.argtypes = [_P(f32), i64, c_int, c_int, _P(i32), _P(f64)]
    L.oracle_topk.restype = c_int
    L.oracle_dispatch.argtypes = [_P(i32), i64, c_int, c_int, _P(i32), _P(i32), _P(i32), _P(i32)]
    L.oracle_dispatch.restype = c_int
    L.oracle_permute_rows.argtypes = [_P(u16), _P(i32), i64, c_int, _P(u16)]
    L.oracle_permute_rows.restype = None
    L.oracle_swiglu_ffn.argtypes = [_P(u16), _P(u16), _P(u16), _P(u16), c_int, c_int, _P(f64)]
    L.oracle_swiglu_ffn.restype = None
    L.oracle_expert_ffn.argtypes = [_P(u16), _P(i32), _P(u16), _P(u16), _P(u16), c_int, c_int,
                                    c_int, _P(f64)]
    L.oracle_expert_ffn.restype = None
    L.oracle_combine.argtypes = [_P(f64), _P(i32), _P(f64), _P(f64), i64, c_int, c_int, _P(u16)]
    L.oracle_combine.restype = None
    L.oracle_layer_given_logits.argtypes = (
        [_P(u16), _P(f32), _P(u16), _P(u16), _P(u16), _P(u16), _P(u16), _P(u16), i64] +
        [c_int] * 5 + [_P(u16), _P(i32), _P(f64), _P(i32), _P(i32), _P(i32), _P(i32), _P(f64)])
    L.oracle_layer_given_logits.restype = c_int
    L.oracle_layer.argtypes = ([_P(u16), _P(f32), _P(f32), _P(u16), _P(u16), _P(u16), _P(u16),
                                _P(u16), _P(u16), i64] + [c_int] * 5 + [_P(u16), _P(f32)])
    L.oracle_layer.restype = c_int
    u8 = ctypes.c_uint8
    L.oracle_fp8_e4m3_to_double.argtypes = [u8]
    L.oracle_fp8_e4m3_to_double.restype = f64
    L.oracle_fp8_e4m3_from_float.argtypes = [f32]
    L.oracle_fp8_e4m3_from_float.restype = u8
    L.oracle_quantize_rows_fp8.argtypes = [_P(u16), i64, c_int, _P(u8), _P(f32)]
    L.oracle_quantize_rows_fp8.restype = None
    L.oracle_expert_ffn_fp8.argtypes = [_P(u16), _P(i32), _P(u8), _P(f32), _P(u8), _P(f32), _P(u8),
                                        _P(f32), c_int, c_int, c_int, _P(f64)]
    L.oracle_expert_ffn_fp8.restype = None
    L.oracle_layer_given_logits_fp8.argtypes = (
        [_P(u16), _P(f32), _P(u8), _P(f32), _P(u8), _P(f32), _P(u8), _P(f32), _P(u16), _P(u16),
         _P(u16), i64] + [c_int] * 5 + [_P(u16), _P(f64)])
    L.oracle_layer_given_logits_fp8.restype = c_int
    L.oracle_expert_ffn_fp8_ex.argtypes = [_P(u16), _P(i32), _P(u8), _P(f32), _P(u8), _P(f32), _P(u8),
                                           _P(f32), c_int, c_int, c_int, c_int, _P(u16), _P(f64), _P(u16)]
    L.oracle_expert_ffn_fp8_ex.restype = None
    L.oracle_layer_given_logits_fp8_ex.argtypes = (
        [_P(u16), _P(f32), _P(u8), _P(f32), _P(u8), _P(f32), _P(u8), _P(f32), _P(u16), _P(u16),
         _P(u16), i64] + [c_int] * 6 + [_P(u16), _P(u16), _P(f64)])
    L.oracle_layer_given_logits_fp8_ex.restype = c_int
    L.oracle_threads.argtypes = [c_int]
    L.oracle_threads.restype = c_int
    return L


def _ptr(a, ctype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _u16(a):
    return None if a is None else np.ascontiguousarray(a).view(np.uint16)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.int32)


U16, I32, F32, F64, U8 = ctypes.c_uint16, ctypes.c_int32, ctypes.c_float, ctypes.c_double, ctypes.c_uint8


def _u8(a):
    return None if a is None else np.ascontiguousarray(a).view(np.uint8)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 storage (uint16) -> float64, element by element through the oracle."""
    f = lib().oracle_bf16_to_double
    b = np.asarray(bits).view(np.uint16).ravel()
    return np.array([f(int(v)) for v in b], dtype=np.float64).reshape(np.shape(bits))


def round_to_bf16(values) -> np.ndarray:
    """float64 -> bf16 storage (uint16), element by element through the oracle."""
    f = lib().oracle_round_to_bf16
    v = np.asarray(values, dtype=np.float64)
    return np.array([f(float(a)) for a in v.ravel()], dtype=np.uint16).reshape(v.shape)


def router_logits(x, W_gate, bias=None):
    """fp64 logits [N,E] of bf16 x [N,H] (uint16) against fp32 W_gate [H,E]."""
    x = _u16(x); W = _f32(W_gate); b = _f32(bias)
    N, H = x.shape
    E = W.shape[1]
    out = np.zeros((N, E), dtype=np.float64)
    lib().oracle_router_logits(_ptr(x, U16), _ptr(W, F32), _ptr(b, F32), N, H, E, _ptr(out, F64))
    return out


def topk(logits32, k):
    """(idx int32 [N,k], w float64 [N,k]) from fp32 logits [N,E]."""
    l = _f32(logits32)
    N, E = l.shape
    idx = np.zeros((N, k), dtype=np.int32)
    w = np.zeros((N, k), dtype=np.float64)
    rc = lib().oracle_topk(_ptr(l, F32), N, E, k, _ptr(idx, I32), _ptr(w, F64))
    if rc:
        raise ValueError("oracle_topk: bad sizes")
    return idx, w


def dispatch(idx, E):
    """(counts [E], offsets [E+1], row_to_token [R], token_to_row [N,k])."""
    idx = _i32(idx)
    N, k = idx.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    r2t = np.zeros(N * k, np.int32)
    t2r = np.zeros((N, k), np.int32)
    rc = lib().oracle_dispatch(_ptr(idx, I32), N, E, k, _ptr(counts, I32), _ptr(offsets, I32),
                               _ptr(r2t, I32), _ptr(t2r, I32))
    if rc:
        raise ValueError("oracle_dispatch: expert index outside [0, E)")
    return counts, offsets, r2t, t2r


def permute_rows(x, row_to_token):
    x = _u16(x); r2t = _i32(row_to_token)
    R = r2t.shape[0]
    H = x.shape[1]
    out = np.zeros((R, H), np.uint16)
    lib().oracle_permute_rows(_ptr(x, U16), _ptr(r2t, I32), R, H, _ptr(out, U16))
    return out


def swiglu_ffn(xrow, W1e, W3e, W2e):
    """One token row through one SwiGLU expert -> float64 row (h rounded to bf16 inside)."""
    xrow = _u16(xrow); W1e = _u16(W1e); W3e = _u16(W3e); W2e = _u16(W2e)
    I, H = W1e.shape
    y = np.zeros(H, np.float64)
    lib().oracle_swiglu_ffn(_ptr(xrow, U16), _ptr(W1e, U16), _ptr(W3e, U16), _ptr(W2e, U16),
                            H, I, _ptr(y, F64))
    return y


def expert_ffn(x_perm, offsets, W1, W3, W2):
    x_perm = _u16(x_perm); offsets = _i32(offsets)
    W1 = _u16(W1); W3 = _u16(W3); W2 = _u16(W2)
    E, I, H = W1.shape
    y = np.zeros(x_perm.shape, np.float64)
    lib().oracle_expert_ffn(_ptr(x_perm, U16), _ptr(offsets, I32), _ptr(W1, U16), _ptr(W3, U16),
                            _ptr(W2, U16), E, H, I, _ptr(y, F64))
    return y


def combine(y_perm, token_to_row, w, s=None):
    """y_perm [R,H] and s [N,H] as float64 (unrounded expert outputs)."""
    y_perm = np.ascontiguousarray(y_perm, dtype=np.float64); t2r = _i32(token_to_row)
    w = np.ascontiguousarray(w, dtype=np.float64)
    s = None if s is None else np.ascontiguousarray(s, dtype=np.float64)
    N, k = t2r.shape
    H = y_perm.shape[1]
    out = np.zeros((N, H), np.uint16)
    lib().oracle_combine(_ptr(y_perm, F64), _ptr(t2r, I32), _ptr(w, F64), _ptr(s, F64), N, H, k,
                         _ptr(out, U16))
    return out


def layer_given_logits(x, logits32, W1, W3, W2, k, Ws1=None, Ws3=None, Ws2=None, extras=False):
    """The sparse layer from fp32 logits; returns out (uint16 [N,H]) or a dict."""
    x = _u16(x); l = _f32(logits32)
    W1 = _u16(W1); W3 = _u16(W3); W2 = _u16(W2)
    Ws1 = _u16(Ws1); Ws3 = _u16(Ws3); Ws2 = _u16(Ws2)
    N, H = x.shape
    E, I, _ = W1.shape
    Is = 0 if Ws1 is None else Ws1.shape[0]
    R = N * k
    out = np.zeros((N, H), np.uint16)
    idx = np.zeros((N, k), np.int32); w = np.zeros((N, k), np.float64)
    counts = np.zeros(E, np.int32); offsets = np.zeros(E + 1, np.int32)
    r2t = np.zeros(R, np.int32); t2r = np.zeros((N, k), np.int32)
    yp = np.zeros((R, H), np.float64)
    rc = lib().oracle_layer_given_logits(
        _ptr(x, U16), _ptr(l, F32), _ptr(W1, U16), _ptr(W3, U16), _ptr(W2, U16),
        _ptr(Ws1, U16), _ptr(Ws3, U16), _ptr(Ws2, U16), N, H, I, E, k, Is, _ptr(out, U16),
        _ptr(idx, I32), _ptr(w, F64), _ptr(counts, I32), _ptr(offsets, I32), _ptr(r2t, I32),
        _ptr(t2r, I32), _ptr(yp, F64))
    if rc:
        raise ValueError("oracle_layer_given_logits failed")
    if not extras:
        return out
    return dict(out=out, idx=idx, w=w, counts=counts, offsets=offsets, row_to_token=r2t,
                token_to_row=t2r, y_perm=yp)


def layer(x, W_gate, W1, W3, W2, k, bias=None, Ws1=None, Ws3=None, Ws2=None):
    """The whole layer from x; returns (out uint16 [N,H], fp32 logits [N,E])."""
    x = _u16(x); Wg = _f32(W_gate); b = _f32(bias)
    W1 = _u16(W1); W3 = _u16(W3); W2 = _u16(W2)
    Ws1 = _u16(Ws1); Ws3 = _u16(Ws3); Ws2 = _u16(Ws2)
    N, H = x.shape
    E, I, _ = W1.shape
    Is = 0 if Ws1 is None else Ws1.shape[0]
    out = np.zeros((N, H), np.uint16)
    logits = np.zeros((N, E), np.float32)
    rc = lib().oracle_layer(_ptr(x, U16), _ptr(Wg, F32), _ptr(b, F32), _ptr(W1, U16),
                            _ptr(W3, U16), _ptr(W2, U16), _ptr(Ws1, U16), _ptr(Ws3, U16),
                            _ptr(Ws2, U16), N, H, I, E, k, Is, _ptr(out, U16), _ptr(logits, F32))
    if rc:
        raise ValueError("oracle_layer failed")
    return out, logits


# ------------------------------------------------------------------ fp8 weights

def fp8_to_f64(codes) -> np.ndarray:
    """e4m3 codes (uint8) -> float64, element by element through the oracle."""
    f = lib().oracle_fp8_e4m3_to_double
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([f(int(v)) for v in c.ravel()], dtype=np.float64).reshape(c.shape)


def fp8_from_f32(values) -> np.ndarray:
    """float32 -> e4m3 codes, element by element (nearest, ties to even, 448 at most)."""
    f = lib().oracle_fp8_e4m3_from_float
    v = np.asarray(values, dtype=np.float32)
    return np.array([f(float(a)) for a in v.ravel()], dtype=np.uint8).reshape(v.shape)


def quantize_rows_fp8(W):
    """bf16 weights [..., K] (uint16) -> (e4m3 codes [..., K] uint8, fp32 scale per row [...])."""
    W = _u16(W)
    K = W.shape[-1]
    rows = int(np.prod(W.shape[:-1]))
    q = np.zeros(W.shape, np.uint8)
    sc = np.zeros(W.shape[:-1], np.float32)
    lib().oracle_quantize_rows_fp8(_ptr(W, U16), rows, K, _ptr(q, U8), _ptr(sc, F32))
    return q, sc


def expert_ffn_fp8(x_perm, offsets, q1, s1, q3, s3, q2, s2):
    x_perm = _u16(x_perm); offsets = _i32(offsets)
    q1, q3, q2 = _u8(q1), _u8(q3), _u8(q2)
    s1, s3, s2 = _f32(s1), _f32(s3), _f32(s2)
    E, I, H = q1.shape
    y = np.zeros(x_perm.shape, np.float64)
    lib().oracle_expert_ffn_fp8(_ptr(x_perm, U16), _ptr(offsets, I32), _ptr(q1, U8), _ptr(s1, F32),
                                _ptr(q3, U8), _ptr(s3, F32), _ptr(q2, U8), _ptr(s2, F32), E, H, I,
                                _ptr(y, F64))
    return y


def layer_given_logits_fp8(x, logits32, q1, s1, q3, s3, q2, s2, k, Ws1=None, Ws3=None, Ws2=None):
    """The sparse layer from fp32 logits with e4m3 routed-expert weights; returns out (uint16 [N,H])."""
    x = _u16(x); l = _f32(logits32)
    q1, q3, q2 = _u8(q1), _u8(q3), _u8(q2)
    s1, s3, s2 = _f32(s1), _f32(s3), _f32(s2)
    Ws1 = _u16(Ws1); Ws3 = _u16(Ws3); Ws2 = _u16(Ws2)
    N, H = x.shape
    E, I, _ = q1.shape
    Is = 0 if Ws1 is None else Ws1.shape[0]
    out = np.zeros((N, H), np.uint16)
    rc = lib().oracle_layer_given_logits_fp8(
        _ptr(x, U16), _ptr(l, F32), _ptr(q1, U8), _ptr(s1, F32), _ptr(q3, U8), _ptr(s3, F32),
        _ptr(q2, U8), _ptr(s2, F32), _ptr(Ws1, U16), _ptr(Ws3, U16), _ptr(Ws2, U16), N, H, I, E, k, Is,
        _ptr(out, U16), None)
    if rc:
        raise ValueError("oracle_layer_given_logits_fp8 failed")
    return out


# ------------------------------------------------ fp8 weights and fp8 activations

def expert_ffn_fp8_ex(x_perm, offsets, q1, s1, q3, s3, q2, s2, quantize_acts, h_given=None):
    """e4m3-weight experts; quantize_acts also quantizes each row of x_perm and of h
    per row.  h_given [R,I] bf16 (uint16) replaces the computed h as the second GEMM's
    input.  Returns (y_perm float64 [R,H], the computed h uint16 [R,I])."""
    x_perm = _u16(x_perm); offsets = _i32(offsets)
    q1, q3, q2 = _u8(q1), _u8(q3), _u8(q2)
    s1, s3, s2 = _f32(s1), _f32(s3), _f32(s2)
    h_given = _u16(h_given)
    E, I, H = q1.shape
    R = x_perm.shape[0]
    y = np.zeros((R, H), np.float64)
    h = np.zeros((R, I), np.uint16)
    lib().oracle_expert_ffn_fp8_ex(_ptr(x_perm, U16), _ptr(offsets, I32), _ptr(q1, U8), _ptr(s1, F32),
                                   _ptr(q3, U8), _ptr(s3, F32), _ptr(q2, U8), _ptr(s2, F32), E, H, I,
                                   1 if quantize_acts else 0, _ptr(h_given, U16), _ptr(y, F64), _ptr(h, U16))
    return y, h


def layer_given_logits_fp8_ex(x, logits32, q1, s1, q3, s3, q2, s2, k, quantize_acts, h_given=None,
                              Ws1=None, Ws3=None, Ws2=None, want_y=False):
    """The e4m3-weight layer from fp32 logits with the activation options above;
    h_given [N*k, I] bf16 is in assignment order (row t*k + j: token t's j-th pick).
    Returns out (uint16 [N,H]), and y_perm (float64 [N*k,H]) with want_y."""
    x = _u16(x); l = _f32(logits32)
    q1, q3, q2 = _u8(q1), _u8(q3), _u8(q2)
    s1, s3, s2 = _f32(s1), _f32(s3), _f32(s2)
    Ws1 = _u16(Ws1); Ws3 = _u16(Ws3); Ws2 = _u16(Ws2)
    h_given = _u16(h_given)
    N, H = x.shape
    E, I, _ = q1.shape
    Is = 0 if Ws1 is None else Ws1.shape[0]
    out = np.zeros((N, H), np.uint16)
    y = np.zeros((N * k, H), np.float64) if want_y else None
    rc = lib().oracle_layer_given_logits_fp8_ex(
        _ptr(x, U16), _ptr(l, F32), _ptr(q1, U8), _ptr(s1, F32), _ptr(q3, U8), _ptr(s3, F32),
        _ptr(q2, U8), _ptr(s2, F32), _ptr(Ws1, U16), _ptr(Ws3, U16), _ptr(Ws2, U16), N, H, I, E, k, Is,
        1 if quantize_acts else 0, _ptr(h_given, U16), _ptr(out, U16), _ptr(y, F64))
    if rc:
        raise ValueError("oracle_layer_given_logits_fp8_ex failed")
    return (out, y) if want_y else out
