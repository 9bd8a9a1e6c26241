"""CPU oracle for the MoE layer forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``moe_oracle.c`` (plain C,
double-precision sums, OpenMP over independent rows) with ctypes and numpy.
It shares no code with the CUDA path and never imports it.

bf16 tensors are numpy ``uint16`` arrays of bf16 bit patterns.

Parity pins (tests/test_oracle_pins.py) tie every function here to something
other than itself: brute force, the pages' permutation example, closed forms
and textbook special cases.  No function is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CAP_NONE, CAP_PER_TOKEN, CAP_PER_ASSIGNMENT = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile liboracle.so (gcc -O2, OpenMP; no fast-math, so sums keep C order)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        L.oracle_bf16_round.argtypes = [dbl]
        L.oracle_bf16_round.restype = ctypes.c_uint16
        L.oracle_router_logits.argtypes = [vp, vp, i32, i32, i32, vp]
        L.oracle_route.argtypes = [vp, vp, i32, i32, i32, vp, vp]
        L.oracle_route.restype = i32
        L.oracle_capacity.argtypes = [i32, i32, i32, dbl, i32]
        L.oracle_capacity.restype = i64
        L.oracle_dispatch.argtypes = [vp, i32, i32, i32, i64, vp, vp, vp, vp, vp]
        L.oracle_dispatch.restype = i32
        L.oracle_gather.argtypes = [vp, vp, i32, i32, i32, vp]
        L.oracle_update_bias.argtypes = [vp, i32, i64, vp]
        L.oracle_update_bias.restype = i32
        L.oracle_expert_ffn.argtypes = [vp, i32, vp, vp, vp, i32, i32, vp, vp]
        L.oracle_combine.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp]
        L.oracle_e4m3.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3.restype = dbl
        L.oracle_expert_ffn_q8.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp]
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_quantize_rows_e4m3.argtypes = [vp, i32, i32, vp, vp]
        L.oracle_expert_ffn_w8a8.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp]
        L.oracle_expert_gate_up_w8a8.argtypes = [vp, i32, vp, vp, vp, vp, i32, i32, vp]
        L.oracle_expert_down_w8a8.argtypes = [vp, i32, vp, vp, i32, i32, vp]
        L.oracle_layer_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32,
                                           i32, i32, i32, i32, i32, i64,
                                           vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.oracle_layer_forward.restype = i32
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def bf16_round(v: float) -> int:
    return int(lib().oracle_bf16_round(float(v)))


def router_logits(x: np.ndarray, wg: np.ndarray) -> np.ndarray:
    x = _c(x, np.uint16); wg = _c(wg, np.uint16)
    T, d = x.shape
    E = wg.shape[0]
    out = np.empty((T, E), dtype=np.float32)
    lib().oracle_router_logits(_p(x), _p(wg), T, d, E, _p(out))
    return out


def route(logits: np.ndarray, k: int, bias: Optional[np.ndarray] = None):
    """-> (idx [T,k] int32, w [T,k] float32)."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    if bias is not None:
        bias = _c(bias, np.float32)
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float32)
    rc = lib().oracle_route(_p(logits), _p(bias), T, E, k, _p(idx), _p(w))
    if rc != 0:
        raise ValueError("non-finite router logits or keys")
    return idx, w


def capacity(T: int, E: int, k: int, cf: float, mode: int) -> int:
    return int(lib().oracle_capacity(T, E, k, float(cf), mode))


def dispatch(idx: np.ndarray, E: int, C: int):
    """-> dict(counts_raw, counts, offsets, dest, src_token, N)."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    craw = np.empty(E, np.int32); cnt = np.empty(E, np.int32); off = np.empty(E + 1, np.int32)
    dest = np.empty((T, k), np.int32); src = np.empty(max(T * k, 1), np.int32)
    N = lib().oracle_dispatch(_p(idx), T, E, k, int(C), _p(craw), _p(cnt), _p(off), _p(dest), _p(src))
    return dict(counts_raw=craw, counts=cnt, offsets=off, dest=dest, src_token=src[:N].copy(), N=N)


def update_bias(counts_raw: np.ndarray, C: int) -> np.ndarray:
    """Selection bias from the last batch's overflow: -clamp((c - C) / C, -1, 1), fp32."""
    counts_raw = _c(counts_raw, np.int32)
    out = np.empty(counts_raw.size, np.float32)
    if lib().oracle_update_bias(_p(counts_raw), counts_raw.size, int(C), _p(out)) != 0:
        raise ValueError("capacity must be positive")
    return out


def gather(x: np.ndarray, dest: np.ndarray, N: int) -> np.ndarray:
    x = _c(x, np.uint16); dest = _c(dest, np.int32)
    T, d = x.shape
    k = dest.shape[1]
    xp = np.zeros((max(N, 1), d), np.uint16)
    lib().oracle_gather(_p(x), _p(dest), T, d, k, _p(xp))
    return xp[:N]


def expert_ffn(x: np.ndarray, W1: np.ndarray, W3: np.ndarray, W2: np.ndarray):
    """One expert on rows of x: -> (h [rows,f] bf16, y [rows,d] bf16)."""
    x = _c(x, np.uint16); W1 = _c(W1, np.uint16); W3 = _c(W3, np.uint16); W2 = _c(W2, np.uint16)
    rows, d = x.shape
    f = W1.shape[0]
    assert W1.shape == (f, d) and W3.shape == (f, d) and W2.shape == (d, f)
    h = np.empty((rows, f), np.uint16)
    y = np.empty((rows, d), np.uint16)
    lib().oracle_expert_ffn(_p(x), rows, _p(W1), _p(W3), _p(W2), d, f, _p(h), _p(y))
    return h, y


def e4m3(b: int) -> float:
    return float(lib().oracle_e4m3(int(b)))


def expert_ffn_q8(x, W1q, s1, W3q, s3, W2q, s2):
    """One expert with fp8 e4m3 weights and fp32 row scales: -> (h, y) bf16."""
    x = _c(x, np.uint16)
    W1q = _c(W1q, np.uint8); W3q = _c(W3q, np.uint8); W2q = _c(W2q, np.uint8)
    s1 = _c(s1, np.float32); s3 = _c(s3, np.float32); s2 = _c(s2, np.float32)
    rows, d = x.shape
    f = W1q.shape[0]
    assert W1q.shape == (f, d) and W3q.shape == (f, d) and W2q.shape == (d, f)
    assert s1.shape == (f,) and s3.shape == (f,) and s2.shape == (d,)
    h = np.empty((rows, f), np.uint16)
    y = np.empty((rows, d), np.uint16)
    lib().oracle_expert_ffn_q8(_p(x), rows, _p(W1q), _p(s1), _p(W3q), _p(s3), _p(W2q), _p(s2), d, f, _p(h), _p(y))
    return h, y


def e4m3_encode(v: float) -> int:
    return int(lib().oracle_e4m3_encode(float(v)))


def quantize_rows_e4m3(x: np.ndarray):
    """bf16 rows [rows, K] -> (e4m3 codes uint8 [rows, K], fp32 scale per row): s = amax / 448."""
    x = _c(x, np.uint16)
    rows, K = x.shape
    q = np.empty((rows, K), np.uint8)
    s = np.empty(rows, np.float32)
    lib().oracle_quantize_rows_e4m3(_p(x), rows, K, _p(q), _p(s))
    return q, s


def expert_ffn_w8a8(x, W1q, s1, W3q, s3, W2q, s2):
    """One expert with fp8 weights and fp8 activations (rows quantised per row): -> (h, y) bf16."""
    x = _c(x, np.uint16)
    W1q = _c(W1q, np.uint8); W3q = _c(W3q, np.uint8); W2q = _c(W2q, np.uint8)
    s1 = _c(s1, np.float32); s3 = _c(s3, np.float32); s2 = _c(s2, np.float32)
    rows, d = x.shape
    f = W1q.shape[0]
    h = np.empty((rows, f), np.uint16)
    y = np.empty((rows, d), np.uint16)
    lib().oracle_expert_ffn_w8a8(_p(x), rows, _p(W1q), _p(s1), _p(W3q), _p(s3), _p(W2q), _p(s2), d, f, _p(h), _p(y))
    return h, y


def expert_gate_up_w8a8(x, W1q, s1, W3q, s3):
    """First GEMM of the fp8 x fp8 expert: -> h bf16 [rows, f]."""
    x = _c(x, np.uint16); W1q = _c(W1q, np.uint8); W3q = _c(W3q, np.uint8)
    s1 = _c(s1, np.float32); s3 = _c(s3, np.float32)
    rows, d = x.shape
    f = W1q.shape[0]
    h = np.empty((rows, f), np.uint16)
    lib().oracle_expert_gate_up_w8a8(_p(x), rows, _p(W1q), _p(s1), _p(W3q), _p(s3), d, f, _p(h))
    return h


def expert_down_w8a8(h, W2q, s2):
    """Second GEMM of the fp8 x fp8 expert on given bf16 h rows: -> y bf16 [rows, d]."""
    h = _c(h, np.uint16); W2q = _c(W2q, np.uint8); s2 = _c(s2, np.float32)
    rows, f = h.shape
    d = W2q.shape[0]
    y = np.empty((rows, d), np.uint16)
    lib().oracle_expert_down_w8a8(_p(h), rows, _p(W2q), _p(s2), d, f, _p(y))
    return y


def combine(y_perm: np.ndarray, dest: np.ndarray, w: np.ndarray, y_shared: Optional[np.ndarray] = None) -> np.ndarray:
    y_perm = _c(y_perm, np.uint16); dest = _c(dest, np.int32); w = _c(w, np.float32)
    T, k = dest.shape
    d = y_perm.shape[1] if y_perm.ndim == 2 else (y_shared.shape[1])
    if y_perm.size == 0:
        y_perm = np.zeros((1, d), np.uint16)
    if y_shared is not None:
        y_shared = _c(y_shared, np.uint16)
    out = np.empty((T, d), np.uint16)
    lib().oracle_combine(_p(y_perm), _p(dest), _p(w), _p(y_shared), T, d, k, _p(out))
    return out


def layer_forward(x, wg, W1, W3, W2, k, C=-1, bias=None, logits_in=None, W1s=None, W3s=None, W2s=None):
    """Whole layer; returns a dict of out and every intermediate the CUDA path exports."""
    x = _c(x, np.uint16); wg = _c(wg, np.uint16)
    W1 = _c(W1, np.uint16); W3 = _c(W3, np.uint16); W2 = _c(W2, np.uint16)
    T, d = x.shape
    E, f, _ = W1.shape
    if bias is not None:
        bias = _c(bias, np.float32)
    if logits_in is not None:
        logits_in = _c(logits_in, np.float32)
    f_s = 0
    if W1s is not None:
        W1s = _c(W1s, np.uint16); W3s = _c(W3s, np.uint16); W2s = _c(W2s, np.uint16)
        f_s = W1s.shape[0]
    out = np.empty((T, d), np.uint16)
    logits = np.empty((T, E), np.float32)
    idx = np.empty((T, k), np.int32); w = np.empty((T, k), np.float32)
    craw = np.empty(E, np.int32); cnt = np.empty(E, np.int32); off = np.empty(E + 1, np.int32)
    dest = np.empty((T, k), np.int32); src = np.empty(max(T * k, 1), np.int32)
    ysh = np.empty((T, d), np.uint16) if f_s else None
    N = lib().oracle_layer_forward(_p(x), _p(wg), _p(bias), _p(logits_in), _p(W1), _p(W3), _p(W2),
                                   _p(W1s), _p(W3s), _p(W2s), f_s, T, d, E, k, f, int(C),
                                   _p(out), _p(logits), _p(idx), _p(w), _p(craw), _p(cnt), _p(off),
                                   _p(dest), _p(src), _p(ysh))
    if N < 0:
        raise ValueError("non-finite router logits or keys")
    return dict(out=out, logits=logits, idx=idx, w=w, counts_raw=craw, counts=cnt, offsets=off,
                dest=dest, src_token=src[:N].copy(), N=N, y_shared=ysh)
