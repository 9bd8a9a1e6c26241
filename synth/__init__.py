"""Seeded synthetic inputs for the MoE layer forward (shared by oracle tests and the CUDA path).

This module holds the workload definitions (shapes, distributions, seeds) and a
counter-based generator (Philox4x32-10 + Box-Muller, see ``synth.c``).  It holds
none of the MoE layer's arithmetic.  Every tensor is addressed by
(seed, tensor id, flat element index), so any slice (one expert's weights, one
token's hidden state) can be regenerated on its own.

Workloads (weights and hidden states bf16, seed 0):

* ``tiny``      T=128,   d=256,  E=8,   k=2, f=512
* ``mixtral``   T=4096,  d=4096, E=8,   k=2, f=14336            (prefill)
* ``qwen3``     T=16384, d=4096, E=128, k=8, f=1536             (prefill)
* ``dsv3``      T=256,   d=7168, E=256, k=8, f=2048, shared f_s=2048,
                selection bias ~U(-0.1, 0.1)                    (decode)
* ``skew``      T=32768, d=4096, E=64,  k=2, f=2048, Zipf(1.2) popularity,
                capacity int(T*k/E*1.25)

Distributions: X ~ N(0,1); W_g, W1, W3 ~ N(0, 1/d) (1/d is the variance);
W2 ~ N(0, 1/f).  The skewed workload shifts router row e by b_e*u and every
hidden state by mu*u along one random unit vector u (mu = 4), with b_e
calibrated on a Gaussian model of the router scores.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

# tensor ids (the Philox key's second word)
TID = dict(x=1, wg=2, w1=3, w3=4, w2=5, w1s=6, w3s=7, w2s=8, bias=9, u=10, zipf_g=11, zipf_s=12)

CAP_NONE, CAP_PER_TOKEN, CAP_PER_ASSIGNMENT = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile libsynth.so with gcc (OpenMP)."""
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
        u32, u64, dbl, vp, i32 = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
        L.synth_philox4x32_10.argtypes = [vp, vp, vp]
        L.synth_normal_bf16.argtypes = [u32, u32, u64, u64, dbl, vp]
        L.synth_normal_f64.argtypes = [u32, u32, u64, u64, vp]
        L.synth_uniform_f32.argtypes = [u32, u32, u64, u64, dbl, dbl, vp]
        L.synth_shifted_bf16.argtypes = [u32, u32, u64, u64, u64, dbl, vp, vp, vp]
        L.synth_zipf_shift.argtypes = [u32, u32, u32, i32, i32, dbl, dbl, vp, vp, i32, i32, vp]
        L.synth_quantize_e4m3_rows.argtypes = [vp, u64, u64, vp, vp]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def philox4x32_10(ctr, key):
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().synth_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def normal_bf16(seed: int, tid: int, offset: int, count: int, std: float, out: Optional[np.ndarray] = None) -> np.ndarray:
    """bf16 bit patterns (uint16) of std*N(0,1) draws [offset, offset+count)."""
    if out is None:
        out = np.empty(count, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == count
    lib().synth_normal_bf16(seed, tid, offset, count, float(std), _p(out))
    return out


def normal_f64(seed: int, tid: int, offset: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.float64)
    lib().synth_normal_f64(seed, tid, offset, count, _p(out))
    return out


def uniform_f32(seed: int, tid: int, offset: int, count: int, lo: float, hi: float) -> np.ndarray:
    out = np.empty(count, dtype=np.float32)
    lib().synth_uniform_f32(seed, tid, offset, count, float(lo), float(hi), _p(out))
    return out


def shifted_bf16(seed: int, tid: int, row0: int, nrows: int, ncols: int, std: float,
                 shift: np.ndarray, u: np.ndarray, out: Optional[np.ndarray] = None) -> np.ndarray:
    shift = np.ascontiguousarray(shift, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    assert u.size == ncols and shift.size >= row0 + nrows
    if out is None:
        out = np.empty(nrows * ncols, dtype=np.uint16)
    lib().synth_shifted_bf16(seed, tid, row0, nrows, ncols, float(std), _p(shift), _p(u), _p(out))
    return out


def quantize_e4m3_rows(w: np.ndarray, K: int):
    """bf16 rows [rows, K] -> (fp8 e4m3 bytes [rows, K] uint8, fp32 scale per row)."""
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1, K)
    rows = w.shape[0]
    q = np.empty((rows, K), dtype=np.uint8)
    s = np.empty(rows, dtype=np.float32)
    lib().synth_quantize_e4m3_rows(_p(w), rows, K, _p(q), _p(s))
    return q, s


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    f_shared: int = 0
    bias_range: float = 0.0          # selection bias ~U(-r, r); 0 = no bias
    cap_mode: int = CAP_NONE
    capacity_factor: float = 1.0
    zipf_s: float = 0.0              # >0: skewed router (Zipf popularity)
    zipf_mu: float = 4.0
    seed: int = 0

    @property
    def has_shared(self) -> bool:
        return self.f_shared > 0


WORKLOADS = {
    "tiny": Workload("tiny", 128, 256, 8, 2, 512),
    "mixtral": Workload("mixtral", 4096, 4096, 8, 2, 14336),
    "qwen3": Workload("qwen3", 16384, 4096, 128, 8, 1536),
    "dsv3": Workload("dsv3", 256, 7168, 256, 8, 2048, f_shared=2048, bias_range=0.1),
    "skew": Workload("skew", 32768, 4096, 64, 2, 2048, cap_mode=CAP_PER_ASSIGNMENT, capacity_factor=1.25, zipf_s=1.2),
}
WORKLOAD_ORDER = ["tiny", "mixtral", "qwen3", "dsv3", "skew"]
# Smaller cases with the same per-tile shapes, for profiler captures that must stay small.
PROFILE_WORKLOADS = {
    "mixtral2e": Workload("mixtral2e", 2048, 4096, 2, 2, 14336),
    "dsv3_32e": Workload("dsv3_32e", 32, 7168, 32, 8, 2048, f_shared=2048, bias_range=0.1),
    "qwen3_16e": Workload("qwen3_16e", 2048, 4096, 16, 8, 1536),
    # the Qwen3-like batch (same x, router and routing) with experts cut to f = 128: the router
    # GEMM, top-k, permutation, gather and combine at their full size, ~2.5 GB on the device
    "qwen3_f128": Workload("qwen3_f128", 16384, 4096, 128, 8, 128),
}
WORKLOADS.update(PROFILE_WORKLOADS)


class Inputs:
    """Lazy, sliceable generator of one workload's tensors (bf16 as uint16 bit patterns)."""

    def __init__(self, wl: Workload):
        self.wl = wl
        self._u = None
        self._b = None

    # --- skewed-router helpers -------------------------------------------------
    def u(self) -> np.ndarray:
        """Random unit vector along which router rows and hidden states are shifted."""
        if self._u is None:
            v = normal_f64(self.wl.seed, TID["u"], 0, self.wl.d)
            self._u = v / math.sqrt(float(np.dot(v, v)))
        return self._u

    def zipf_shift(self) -> np.ndarray:
        """Per-expert shifts b_e (calibrated on a Gaussian score model, not on the layer)."""
        wl = self.wl
        if self._b is None:
            std = 1.0 / math.sqrt(wl.d)
            w0 = normal_f64(wl.seed, TID["wg"], 0, wl.E * wl.d).reshape(wl.E, wl.d) * std
            nrm = np.ascontiguousarray(np.sqrt((w0 * w0).sum(axis=1)))
            off = np.ascontiguousarray(wl.zipf_mu * (w0 @ self.u()))
            b = np.zeros(wl.E, dtype=np.float64)
            lib().synth_zipf_shift(wl.seed, TID["zipf_g"], TID["zipf_s"], wl.E, wl.k, float(wl.zipf_s),
                                   float(wl.zipf_mu), _p(nrm), _p(off), 40, 65536, _p(b))
            self._b = b
        return self._b

    def zipf_target(self) -> np.ndarray:
        p = np.arange(1, self.wl.E + 1, dtype=np.float64) ** (-self.wl.zipf_s)
        return p / p.sum()

    # --- tensors ------------------------------------------------------------------
    def x_rows(self, t0: int, n: int, out: Optional[np.ndarray] = None) -> np.ndarray:
        wl = self.wl
        if wl.zipf_s > 0:
            shift = np.full(t0 + n, wl.zipf_mu)
            return shifted_bf16(wl.seed, TID["x"], t0, n, wl.d, 1.0, shift, self.u(), out)
        return normal_bf16(wl.seed, TID["x"], t0 * wl.d, n * wl.d, 1.0, out)

    def x(self) -> np.ndarray:
        return self.x_rows(0, self.wl.T).reshape(self.wl.T, self.wl.d)

    def wg(self) -> np.ndarray:
        wl = self.wl
        std = 1.0 / math.sqrt(wl.d)
        if wl.zipf_s > 0:
            return shifted_bf16(wl.seed, TID["wg"], 0, wl.E, wl.d, std, self.zipf_shift(), self.u()).reshape(wl.E, wl.d)
        return normal_bf16(wl.seed, TID["wg"], 0, wl.E * wl.d, std).reshape(wl.E, wl.d)

    def expert_rows(self, name: str, e0: int, ne: int, out: Optional[np.ndarray] = None) -> np.ndarray:
        """Experts [e0, e0+ne) of W1/W3 ([E,f,d]) or W2 ([E,d,f]), flat."""
        wl = self.wl
        per = wl.f * wl.d
        std = 1.0 / math.sqrt(wl.f if name == "w2" else wl.d)
        return normal_bf16(wl.seed, TID[name], e0 * per, ne * per, std, out)

    def w1(self) -> np.ndarray:
        return self.expert_rows("w1", 0, self.wl.E).reshape(self.wl.E, self.wl.f, self.wl.d)

    def w3(self) -> np.ndarray:
        return self.expert_rows("w3", 0, self.wl.E).reshape(self.wl.E, self.wl.f, self.wl.d)

    def w2(self) -> np.ndarray:
        return self.expert_rows("w2", 0, self.wl.E).reshape(self.wl.E, self.wl.d, self.wl.f)

    def shared(self, name: str) -> Optional[np.ndarray]:
        """W1s/W3s [f_s, d] or W2s [d, f_s]; None if the workload has no shared expert."""
        wl = self.wl
        if not wl.has_shared:
            return None
        n = wl.f_shared * wl.d
        std = 1.0 / math.sqrt(wl.f_shared if name == "w2s" else wl.d)
        a = normal_bf16(wl.seed, TID[name], 0, n, std)
        return a.reshape(wl.d, wl.f_shared) if name == "w2s" else a.reshape(wl.f_shared, wl.d)

    def bias(self) -> Optional[np.ndarray]:
        wl = self.wl
        if wl.bias_range <= 0:
            return None
        return uniform_f32(wl.seed, TID["bias"], 0, wl.E, -wl.bias_range, wl.bias_range)


def device_tensors(wl: Workload, device, names=None, chunk_elems: int = 1 << 27) -> dict:
    """Generate the workload's tensors on the host and copy them to `device` (torch).

    Large expert tensors are produced in chunks of whole experts into pinned staging
    buffers, so host memory stays bounded.  bf16 tensors come back as torch.bfloat16.
    Keys: x, wg, w1, w3, w2, [w1s, w3s, w2s], [bias].
    """
    import torch

    inp = Inputs(wl)
    want = names or ["x", "wg", "w1", "w3", "w2", "w1s", "w3s", "w2s", "bias"]
    out = {}

    def to_dev_bf16(a: np.ndarray, shape):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).reshape(shape)
        return t.to(device)

    if "x" in want:
        out["x"] = to_dev_bf16(inp.x_rows(0, wl.T), (wl.T, wl.d))
    if "wg" in want:
        out["wg"] = to_dev_bf16(inp.wg().ravel(), (wl.E, wl.d))
    per = wl.f * wl.d
    ne = max(1, min(wl.E, chunk_elems // per))
    stage = [torch.empty(ne * per, dtype=torch.int16).pin_memory() for _ in range(2)]
    for name in ("w1", "w3", "w2"):
        if name not in want:
            continue
        shape = (wl.E, wl.d, wl.f) if name == "w2" else (wl.E, wl.f, wl.d)
        dst = torch.empty(shape, dtype=torch.bfloat16, device=device)
        flat = dst.view(-1).view(torch.int16)
        i = 0
        for e0 in range(0, wl.E, ne):
            n = min(ne, wl.E - e0)
            buf = stage[i & 1]
            torch.cuda.current_stream(device).synchronize()   # buffer free again
            inp.expert_rows(name, e0, n, out=buf.numpy()[: n * per].view(np.uint16))
            flat[e0 * per:(e0 + n) * per].copy_(buf[: n * per], non_blocking=True)
            i += 1
        torch.cuda.current_stream(device).synchronize()
        out[name] = dst
    if wl.has_shared:
        for name in ("w1s", "w3s", "w2s"):
            if name in want:
                a = inp.shared(name)
                out[name] = to_dev_bf16(a.ravel(), a.shape)
    if "bias" in want:
        b = inp.bias()
        out["bias"] = torch.from_numpy(b).to(device) if b is not None else None
    return out


def device_tensors_q8(wl: Workload, device, chunk_rows: int = 1 << 16, host: Optional[dict] = None) -> dict:
    """fp8 e4m3 expert weights with fp32 row scales, quantised from the workload's bf16 weights
    (quantize_e4m3_rows) chunk by chunk on the host and copied to `device`.
    Keys: w1q, w3q [E,f,d] uint8, s1, s3 [E,f]; w2q [E,d,f], s2 [E,d]; w1sq, w3sq, w2sq, s1s,
    s3s, s2s for the shared expert.  host: a dict that receives the same arrays as numpy
    (host copies, e.g. for a checker that needs every expert's codes)."""
    import torch

    inp = Inputs(wl)
    out = {}
    per = wl.f * wl.d
    for name, K, rows_per_e in (("w1", wl.d, wl.f), ("w3", wl.d, wl.f), ("w2", wl.f, wl.d)):
        q_dev = torch.empty((wl.E * rows_per_e, K), dtype=torch.uint8, device=device)
        s_dev = torch.empty(wl.E * rows_per_e, dtype=torch.float32, device=device)
        ne = max(1, min(wl.E, chunk_rows // rows_per_e))
        if host is not None:
            host[name + "q"] = np.empty((wl.E, rows_per_e, K), np.uint8)
            host["s" + name[1]] = np.empty((wl.E, rows_per_e), np.float32)
        for e0 in range(0, wl.E, ne):
            n = min(ne, wl.E - e0)
            w = inp.expert_rows(name, e0, n)
            q, sc = quantize_e4m3_rows(w, K)
            q_dev[e0 * rows_per_e:(e0 + n) * rows_per_e].copy_(torch.from_numpy(q))
            s_dev[e0 * rows_per_e:(e0 + n) * rows_per_e].copy_(torch.from_numpy(sc))
            if host is not None:
                host[name + "q"][e0:e0 + n] = q.reshape(n, rows_per_e, K)
                host["s" + name[1]][e0:e0 + n] = sc.reshape(n, rows_per_e)
        out[name + "q"] = q_dev.view(wl.E, rows_per_e, K)
        out["s" + name[1]] = s_dev.view(wl.E, rows_per_e)
    if wl.has_shared:
        for name in ("w1s", "w3s", "w2s"):
            a = inp.shared(name)
            q, sc = quantize_e4m3_rows(a, a.shape[1])
            out[name[:2] + "sq"] = torch.from_numpy(q).to(device)
            out["s" + name[1] + "s"] = torch.from_numpy(sc).to(device)
            if host is not None:
                host[name[:2] + "sq"] = q
                host["s" + name[1] + "s"] = sc
    return out

