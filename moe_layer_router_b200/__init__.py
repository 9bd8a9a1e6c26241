"""B200 (sm_100a) MoE layer forward: Python binding of the C ABI in include/moe.h.

Argument marshalling only.  Every step of the layer runs in the CUDA kernels of
``libmoe_b200.so``; this module passes device pointers, sizes and the current
torch stream, and turns a non-zero status into ``MoeError``.  There is no CPU
fallback: if the library is missing, importing the binding raises.

Names follow the C ABI: ``moe_route``, ``moe_permute``, ``moe_expert_ffn``,
``moe_combine``, ``moe_layer_forward``, plus the helpers ``moe_capacity``,
``moe_workspace_bytes``, ``moe_workspace_layout``, ``moe_get_error``,
``moe_strerror``.  Tensors are torch tensors (bf16 / fp32 / int32, contiguous);
``None`` passes NULL.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_SHAPE = -2
MOE_ERR_ALIGN = -3
MOE_ERR_WORKSPACE = -4
MOE_ERR_CUDA = -5
MOE_ERR_TIMEOUT = -6
MOE_ERR_CHECK = -7
MOE_ERR_DEVICE = -8

MOE_CAP_NONE, MOE_CAP_PER_TOKEN, MOE_CAP_PER_ASSIGNMENT = 0, 1, 2

# Names of the intermediates moe_layer_forward leaves in its workspace (moe_workspace_layout order).
WS_NAMES = ["logits", "idx", "w", "counts_raw", "counts", "offsets", "dest", "src_token",
            "x_perm", "h", "y_perm", "y_shared", "h_shared"]


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} ({code})")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                      "(python moe_layer_router_b200/build.py)")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i32, _i64, _dbl, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t

_lib.moe_capacity.argtypes = [_i32, _i32, _i32, _dbl, _i32]
_lib.moe_capacity.restype = _i64
_lib.moe_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz)]
_lib.moe_workspace_layout.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz)]
_lib.moe_route.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.moe_permute.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.moe_permute_noalloc.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.moe_permute_noalloc.restype = _i32
_lib.moe_expert_ffn.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.moe_combine.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp]
_lib.moe_layer_forward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                                   _i32, _i32, _i32, _i32, _i32, _dbl, _i32, _vp, _vp, _sz, _vp]
_lib.moe_layer_forward_ex.argtypes = _lib.moe_layer_forward.argtypes + [_vp]
_lib.moe_layer_forward_w8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                                      _i32, _i32, _i32, _i32, _i32, _dbl, _i32, _vp, _vp, _sz, _vp, _vp]
_lib.moe_layer_forward_w8.restype = _i32
_lib.moe_cache_state_bytes.argtypes = [_i32, _i32, ctypes.POINTER(_sz)]
_lib.moe_cache_state_bytes.restype = _i32
_lib.moe_cache_layout.argtypes = [_i32, _i32, ctypes.POINTER(_sz)]
_lib.moe_cache_layout.restype = _i32
_lib.moe_cache_reset.argtypes = [_vp, _i32, _i32, _vp]
_lib.moe_cache_reset.restype = _i32
_lib.moe_layer_forward_cached.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _i32,
                                          _i32, _i32, _i32, _i32, _i32, _dbl, _i32, _vp, _vp, _sz, _vp, _vp]
_lib.moe_layer_forward_cached.restype = _i32
class moe_w8_experts(ctypes.Structure):
    _fields_ = [("W1q", _vp), ("W3q", _vp), ("W2q", _vp), ("s1", _vp), ("s3", _vp), ("s2", _vp)]


_lib.moe_layer_forward_cached_w8.argtypes = [_vp, _vp, _vp, ctypes.POINTER(moe_w8_experts),
                                             ctypes.POINTER(moe_w8_experts), _i32, _vp,
                                             ctypes.POINTER(moe_w8_experts), _i32, _i32, _i32, _i32, _i32, _i32,
                                             _dbl, _i32, _vp, _vp, _sz, _vp, _vp]
_lib.moe_layer_forward_cached_w8.restype = _i32
_lib.moe_workspace_bytes_a8.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz)]
_lib.moe_workspace_bytes_a8.restype = _i32
_lib.moe_layer_forward_w8a8.argtypes = _lib.moe_layer_forward_w8.argtypes
_lib.moe_layer_forward_w8a8.restype = _i32
_lib.moe_layer_permute.argtypes = [_vp, _i32, _i32, _i32, _i32, _i32, _i32, _i64, _vp, _vp, _sz, _vp]
_lib.moe_layer_permute.restype = _i32
_lib.moe_ep_workspace_bytes.argtypes = [_i32, _i32, ctypes.POINTER(_sz)]
_lib.moe_ep_workspace_bytes.restype = _i32
_lib.moe_ep_plan.argtypes = [_vp, _i32, _i32, _i32, _i64, _i32, _vp, _sz, _vp]
_lib.moe_ep_plan.restype = _i32
_lib.moe_ep_dispatch.argtypes = [_vp, _i32, _i32, _i32, _i32, ctypes.POINTER(_vp), _vp, _sz, _vp]
_lib.moe_ep_dispatch.restype = _i32
_lib.moe_ep_expert_ffn.argtypes = [_vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp,
                                   _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp]
_lib.moe_ep_expert_ffn.restype = _i32
_lib.moe_ep_return.argtypes = [_vp, _i32, _i32, _i32, _i32, ctypes.POINTER(_vp), _vp, _sz, _vp]
_lib.moe_ep_return.restype = _i32
_lib.moe_ep_expert_ffn_return.argtypes = [_vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp,
                                          _vp, _vp, _i32, _vp, _vp, ctypes.POINTER(_vp), _vp, _vp, _sz, _vp]
_lib.moe_ep_expert_ffn_return.restype = _i32
_lib.moe_ep_dispatch_gather.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, ctypes.POINTER(_vp), _vp, _sz, _vp]
_lib.moe_ep_dispatch_gather.restype = _i32
_lib.moe_layer_permute_indices.argtypes = _lib.moe_layer_permute.argtypes
_lib.moe_layer_permute_indices.restype = _i32
_lib.moe_ep_splits_offset.argtypes = [_i32, _i32, ctypes.POINTER(_sz)]
_lib.moe_ep_splits_offset.restype = _i32
_lib.moe_ipc_export.argtypes = [_vp, _vp]
_lib.moe_ipc_export.restype = _i32
_lib.moe_ipc_import.argtypes = [_vp, ctypes.POINTER(_vp)]
_lib.moe_ipc_import.restype = _i32
_lib.moe_ipc_close.argtypes = [_vp, _vp]
_lib.moe_ipc_close.restype = _i32
MOE_IPC_HANDLE_BYTES = 96
_lib.moe_layer_route_count.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp]
_lib.moe_layer_route_count.restype = _i32
_lib.moe_fill_base.argtypes = [_vp, _i32, _i32, _i32, _vp, _vp]
_lib.moe_fill_base.restype = _i32
_lib.moe_layer_finish.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i64, _vp,
                                  _vp, _vp, _sz, _vp]
_lib.moe_layer_finish.restype = _i32
_lib.moe_pipeline_bytes.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz)]
_lib.moe_pipeline_create.argtypes = [_vp, _vp, _sz, ctypes.POINTER(_vp)]
_lib.moe_pipeline_submit.argtypes = [_vp, _vp, _vp]
_lib.moe_pipeline_sync.argtypes = [_vp]
_lib.moe_pipeline_streams.argtypes = [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp)]
_lib.moe_pipeline_destroy.argtypes = [_vp]
_lib.moe_pipeline_bytes_w8.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz)]
_lib.moe_pipeline_create_w8.argtypes = [_vp, ctypes.POINTER(moe_w8_experts), ctypes.POINTER(moe_w8_experts), _i32,
                                        _vp, _sz, ctypes.POINTER(_vp)]
for _n in ("moe_pipeline_bytes", "moe_pipeline_create", "moe_pipeline_submit", "moe_pipeline_sync",
           "moe_pipeline_streams", "moe_pipeline_destroy", "moe_pipeline_bytes_w8", "moe_pipeline_create_w8"):
    getattr(_lib, _n).restype = _i32
_lib.moe_update_bias.argtypes = [_vp, _i32, _i64, _vp, _vp]
_lib.moe_update_bias.restype = _i32
_lib.moe_get_error.argtypes = [_vp]
_lib.moe_selftest_wait_timeout.argtypes = [_vp]
_lib.moe_selftest_wait_timeout.restype = _i32
_lib.moe_strerror.argtypes = [_i32]
_lib.moe_strerror.restype = ctypes.c_char_p
for _n in ("moe_workspace_bytes", "moe_workspace_layout", "moe_route", "moe_permute", "moe_expert_ffn",
           "moe_combine", "moe_layer_forward", "moe_layer_forward_ex", "moe_get_error"):
    getattr(_lib, _n).restype = _i32


def lib() -> ctypes.CDLL:
    return _lib


def strerror(code: int) -> str:
    return _lib.moe_strerror(int(code)).decode()


moe_strerror = strerror


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(rc: int, where: str) -> None:
    if rc != MOE_OK:
        raise MoeError(rc, where)


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def moe_capacity(T: int, E: int, k: int, capacity_factor: float, cap_mode: int) -> int:
    return int(_lib.moe_capacity(T, E, k, float(capacity_factor), cap_mode))


def moe_workspace_bytes(T: int, d: int, E: int, k: int, f: int, f_shared: int = 0) -> int:
    out = _sz(0)
    _check(_lib.moe_workspace_bytes(T, d, E, k, f, f_shared, ctypes.byref(out)), "moe_workspace_bytes")
    return int(out.value)


def moe_workspace_layout(T: int, d: int, E: int, k: int, f: int, f_shared: int = 0) -> dict:
    arr = (_sz * 13)()
    _check(_lib.moe_workspace_layout(T, d, E, k, f, f_shared, arr), "moe_workspace_layout")
    return {n: int(arr[i]) for i, n in enumerate(WS_NAMES)}


def moe_route(x, Wg, bias, logits_in, T, d, E, k, logits_out, idx, w, ws, stream=None) -> None:
    _check(_lib.moe_route(_ptr(x), _ptr(Wg), _ptr(bias), _ptr(logits_in), T, d, E, k, _ptr(logits_out),
                          _ptr(idx), _ptr(w), _ptr(ws), _nbytes(ws), _stream(stream)), "moe_route")


def moe_permute(x, idx, T, d, E, k, capacity, counts_raw, counts, offsets, dest, src_token, x_perm, ws,
                stream=None) -> None:
    _check(_lib.moe_permute(_ptr(x), _ptr(idx), T, d, E, k, int(capacity), _ptr(counts_raw), _ptr(counts),
                            _ptr(offsets), _ptr(dest), _ptr(src_token), _ptr(x_perm), _ptr(ws), _nbytes(ws),
                            _stream(stream)), "moe_permute")


MOE_NOALLOC_SCRATCH_BYTES = 4 << 20


def moe_permute_noalloc(x, idx, T, d, E, k, capacity, counts_raw, counts, offsets, dest, src_token, x_perm,
                        stream=None) -> None:
    """moe_permute without a workspace, for callers that cannot allocate device memory: the
    scratch is a fixed 4 MiB array inside the library (shared by all calls on a device)."""
    _check(_lib.moe_permute_noalloc(_ptr(x), _ptr(idx), T, d, E, k, int(capacity), _ptr(counts_raw), _ptr(counts),
                                    _ptr(offsets), _ptr(dest), _ptr(src_token), _ptr(x_perm), _stream(stream)),
           "moe_permute_noalloc")


def moe_expert_ffn(x_perm, offsets, max_rows, E, d, f, W1, W3, W2, h, y_perm, ws, stream=None) -> None:
    _check(_lib.moe_expert_ffn(_ptr(x_perm), _ptr(offsets), max_rows, E, d, f, _ptr(W1), _ptr(W3), _ptr(W2),
                               _ptr(h), _ptr(y_perm), _ptr(ws), _nbytes(ws), _stream(stream)), "moe_expert_ffn")


def moe_combine(y_perm, dest, w, y_shared, T, d, k, out, stream=None) -> None:
    _check(_lib.moe_combine(_ptr(y_perm), _ptr(dest), _ptr(w), _ptr(y_shared), T, d, k, _ptr(out),
                            _stream(stream)), "moe_combine")


def moe_layer_forward(x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, f_shared, T, d, E, k, f, capacity_factor, cap_mode,
                      out, ws, stream=None) -> None:
    _check(_lib.moe_layer_forward(_ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(W1s),
                                  _ptr(W3s), _ptr(W2s), f_shared, T, d, E, k, f, float(capacity_factor), cap_mode,
                                  _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream)), "moe_layer_forward")


STAGES = ["route", "topk", "permute", "gate_up", "down", "combine", "end"]   # timeline of one layer call
# struct order; "cache" marks the expert cache kernels (between "permute" and "gate_up") in
# moe_layer_forward_cached; "gemm1" / "gemm2" mark the grouped GEMM kernels themselves in the
# fp8-activation layer (after the quantisation of their rows, inside "gate_up" / "down")
_EVENT_FIELDS = STAGES + ["cache", "gemm1", "gemm2", "copy_start", "copy_end"]


class moe_stage_events(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _EVENT_FIELDS]


def _events(events: Optional[dict]):
    if not events:
        return None
    return moe_stage_events(*[events[n].cuda_event if n in events and events[n] is not None else None
                              for n in _EVENT_FIELDS])


def moe_layer_forward_ex(x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, f_shared, T, d, E, k, f, capacity_factor,
                         cap_mode, out, ws, events: Optional[dict] = None, stream=None) -> None:
    """moe_layer_forward with optional stage markers: events = {stage name: torch.cuda.Event}."""
    ev = _events(events)
    _check(_lib.moe_layer_forward_ex(_ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(W1s),
                                     _ptr(W3s), _ptr(W2s), f_shared, T, d, E, k, f, float(capacity_factor),
                                     cap_mode, _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream),
                                     ctypes.byref(ev) if ev is not None else None), "moe_layer_forward_ex")


def moe_layer_route_count(x, Wg, bias, f_shared, T, d, E, k, f, ws, stream=None) -> None:
    _check(_lib.moe_layer_route_count(_ptr(x), _ptr(Wg), _ptr(bias), f_shared, T, d, E, k, f, _ptr(ws), _nbytes(ws),
                                      _stream(stream)), "moe_layer_route_count")


def moe_fill_base(all_counts, G, rank, E, fill_base, stream=None) -> None:
    _check(_lib.moe_fill_base(_ptr(all_counts), G, rank, E, _ptr(fill_base), _stream(stream)), "moe_fill_base")


def moe_layer_finish(x, W1, W3, W2, W1s, W3s, W2s, f_shared, T, d, E, k, f, capacity, fill_base, out, ws,
                     stream=None) -> None:
    _check(_lib.moe_layer_finish(_ptr(x), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(W1s), _ptr(W3s), _ptr(W2s), f_shared, T,
                                 d, E, k, f, int(capacity), _ptr(fill_base), _ptr(out), _ptr(ws), _nbytes(ws),
                                 _stream(stream)), "moe_layer_finish")


def moe_update_bias(counts_raw, E, capacity, bias, stream=None) -> None:
    _check(_lib.moe_update_bias(_ptr(counts_raw), E, int(capacity), _ptr(bias), _stream(stream)), "moe_update_bias")


class moe_pipeline_params(ctypes.Structure):
    _fields_ = [("Wg", _vp), ("W1", _vp), ("W3", _vp), ("W2", _vp), ("W1s", _vp), ("W3s", _vp), ("W2s", _vp),
                ("bias", _vp), ("T", _i32), ("d", _i32), ("E", _i32), ("k", _i32), ("f", _i32), ("f_shared", _i32),
                ("capacity_factor", _dbl), ("cap_mode", _i32)]


def moe_pipeline_bytes(T, d, E, k, f, f_shared=0) -> int:
    out = _sz(0)
    _check(_lib.moe_pipeline_bytes(T, d, E, k, f, f_shared, ctypes.byref(out)), "moe_pipeline_bytes")
    return int(out.value)


def moe_pipeline_bytes_w8(T, d, E, k, f, f_shared=0, activations_fp8=False) -> int:
    out = _sz(0)
    _check(_lib.moe_pipeline_bytes_w8(T, d, E, k, f, f_shared, int(bool(activations_fp8)), ctypes.byref(out)),
           "moe_pipeline_bytes_w8")
    return int(out.value)


class Pipeline:
    """moe_pipeline_* as an object: submit(x_host, out_host) per batch, sync() to wait.
    dev_mem is a caller-owned device buffer of moe_pipeline_bytes() bytes (moe_pipeline_bytes_w8()
    for fp8 experts); weights stay referenced (keep the tensors alive).  fp8: pass W1 = W3 = W2 =
    None and routed (and, with a shared expert, shared) as dicts of W1q, W3q, W2q, s1, s3, s2
    tensors; activations_fp8 selects moe_layer_forward_w8a8 over moe_layer_forward_w8."""

    def __init__(self, Wg, bias, W1, W3, W2, W1s, W3s, W2s, f_shared, T, d, E, k, f, capacity_factor, cap_mode,
                 dev_mem, routed: Optional[dict] = None, shared: Optional[dict] = None, activations_fp8=False):
        self._keep = (Wg, bias, W1, W3, W2, W1s, W3s, W2s, dev_mem, routed, shared)
        self.params = moe_pipeline_params(_ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(W1s), _ptr(W3s), _ptr(W2s),
                                          _ptr(bias), T, d, E, k, f, f_shared, float(capacity_factor), cap_mode)
        h = _vp()
        if routed is None:
            _check(_lib.moe_pipeline_create(ctypes.byref(self.params), _ptr(dev_mem), _nbytes(dev_mem),
                                            ctypes.byref(h)), "moe_pipeline_create")
        else:
            self._q, self._qs = _w8(routed), _w8(shared)
            _check(_lib.moe_pipeline_create_w8(ctypes.byref(self.params), ctypes.byref(self._q),
                                               ctypes.byref(self._qs) if self._qs is not None else None,
                                               int(bool(activations_fp8)), _ptr(dev_mem), _nbytes(dev_mem),
                                               ctypes.byref(h)), "moe_pipeline_create_w8")
        self.handle = h

    def submit(self, x_host, out_host) -> None:
        _check(_lib.moe_pipeline_submit(self.handle, _ptr(x_host), _ptr(out_host)), "moe_pipeline_submit")

    def sync(self) -> None:
        _check(_lib.moe_pipeline_sync(self.handle), "moe_pipeline_sync")

    def streams(self):
        a, b, c = _vp(), _vp(), _vp()
        _check(_lib.moe_pipeline_streams(self.handle, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
               "moe_pipeline_streams")
        return a.value, b.value, c.value

    def close(self) -> None:
        if self.handle:
            _lib.moe_pipeline_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_layer_forward_w8(x, Wg, bias, W1q, s1, W3q, s3, W2q, s2, W1sq, s1s, W3sq, s3s, W2sq, s2s, f_shared, T, d, E,
                         k, f, capacity_factor, cap_mode, out, ws, events: Optional[dict] = None, stream=None) -> None:
    """The layer with fp8 e4m3 expert weights (uint8 tensors) and fp32 per-row scales."""
    ev = _events(events)
    _check(_lib.moe_layer_forward_w8(_ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1q), _ptr(s1), _ptr(W3q), _ptr(s3),
                                     _ptr(W2q), _ptr(s2), _ptr(W1sq), _ptr(s1s), _ptr(W3sq), _ptr(s3s), _ptr(W2sq),
                                     _ptr(s2s), f_shared, T, d, E, k, f, float(capacity_factor), cap_mode, _ptr(out),
                                     _ptr(ws), _nbytes(ws), _stream(stream), ctypes.byref(ev) if ev is not None else None),
           "moe_layer_forward_w8")


def moe_cache_state_bytes(E: int, S: int) -> int:
    out = _sz(0)
    _check(_lib.moe_cache_state_bytes(E, S, ctypes.byref(out)), "moe_cache_state_bytes")
    return int(out.value)


CACHE_FIELDS = ["counters", "slot_of", "expert_in", "stamp", "load_expert", "load_slot"]


def moe_cache_layout(E: int, S: int) -> dict:
    off = (_sz * 6)()
    _check(_lib.moe_cache_layout(E, S, off), "moe_cache_layout")
    return dict(zip(CACHE_FIELDS, [int(v) for v in off]))


def moe_cache_reset(state, E: int, S: int, stream=None) -> None:
    _check(_lib.moe_cache_reset(_ptr(state), E, S, _stream(stream)), "moe_cache_reset")


def moe_layer_forward_cached(x, Wg, bias, W1_src, W3_src, W2_src, W1_slots, W3_slots, W2_slots, S, state, W1s, W3s,
                             W2s, f_shared, T, d, E, k, f, capacity_factor, cap_mode, out, ws,
                             events: Optional[dict] = None, stream=None) -> None:
    """The layer with routed experts served from the expert cache.  W*_src: page-locked host
    tensors (pin_memory) or device tensors; W*_slots: device tensors [S, ...]; state: a device
    uint8 tensor of moe_cache_state_bytes(E, S) bytes, emptied once by moe_cache_reset."""
    ev = _events(events)
    _check(_lib.moe_layer_forward_cached(_ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1_src), _ptr(W3_src), _ptr(W2_src),
                                         _ptr(W1_slots), _ptr(W3_slots), _ptr(W2_slots), S, _ptr(state), _ptr(W1s),
                                         _ptr(W3s), _ptr(W2s), f_shared, T, d, E, k, f, float(capacity_factor),
                                         cap_mode, _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream),
                                         ctypes.byref(ev) if ev is not None else None), "moe_layer_forward_cached")


def _w8(d):
    """dict with W1q, W3q, W2q, s1, s3, s2 tensors (or None) -> moe_w8_experts."""
    if d is None:
        return None
    return moe_w8_experts(*[_ptr(d[n]) for n in ("W1q", "W3q", "W2q", "s1", "s3", "s2")])


def moe_layer_forward_cached_w8(x, Wg, bias, src: dict, slots: dict, S, state, shared: Optional[dict], f_shared, T, d,
                                E, k, f, capacity_factor, cap_mode, out, ws, events: Optional[dict] = None,
                                stream=None) -> None:
    """The cached layer with fp8 experts.  src / slots / shared: dicts of W1q, W3q, W2q (uint8)
    and s1, s3, s2 (fp32) tensors; src may be page-locked host tensors."""
    ev = _events(events)
    a, b, c = _w8(src), _w8(slots), _w8(shared)
    _check(_lib.moe_layer_forward_cached_w8(_ptr(x), _ptr(Wg), _ptr(bias), ctypes.byref(a), ctypes.byref(b), S,
                                            _ptr(state), ctypes.byref(c) if c is not None else None, f_shared, T, d,
                                            E, k, f, float(capacity_factor), cap_mode, _ptr(out), _ptr(ws),
                                            _nbytes(ws), _stream(stream), ctypes.byref(ev) if ev is not None else None),
           "moe_layer_forward_cached_w8")


def cache_counters(state) -> dict:
    """The cache counters of a state tensor (copies 32 bytes to the host)."""
    v = state[:32].view(__import__("torch").int64).cpu().tolist()
    return dict(step=v[0], hits=v[1], misses=v[2], loads_last=v[3])


def moe_layer_permute(x, f_shared, T, d, E, k, f, capacity, fill_base, ws, stream=None) -> None:
    _check(_lib.moe_layer_permute(_ptr(x), f_shared, T, d, E, k, f, int(capacity), _ptr(fill_base), _ptr(ws),
                                  _nbytes(ws), _stream(stream)), "moe_layer_permute")


def moe_ep_workspace_bytes(R: int, E: int) -> int:
    out = _sz(0)
    _check(_lib.moe_ep_workspace_bytes(R, E, ctypes.byref(out)), "moe_ep_workspace_bytes")
    return int(out.value)


def _addr_array(bufs):
    arr = (_vp * len(bufs))()
    for i, b in enumerate(bufs):
        arr[i] = _ptr(b)
    return arr


def moe_ep_plan(all_counts_raw, R, rank, E, capacity, max_recv_rows, ep_ws, stream=None) -> None:
    _check(_lib.moe_ep_plan(_ptr(all_counts_raw), R, rank, E, int(capacity), max_recv_rows, _ptr(ep_ws),
                            _nbytes(ep_ws), _stream(stream)), "moe_ep_plan")


def moe_ep_dispatch(x_perm, R, rank, E, d, recv_bufs, ep_ws, stream=None) -> None:
    """recv_bufs: R tensors (or device addresses), rank q's receive buffer [max_recv_rows, d] bf16."""
    _check(_lib.moe_ep_dispatch(_ptr(x_perm), R, rank, E, d, _addr_array(recv_bufs), _ptr(ep_ws), _nbytes(ep_ws),
                                _stream(stream)), "moe_ep_dispatch")


def moe_ep_expert_ffn(recv_x, max_recv_rows, R, rank, E, d, f, W1_local, W3_local, W2_local, h, y_recv, x, T, W1s, W3s,
                      W2s, f_shared, h_shared, y_shared, ep_ws, source_major=False, stream=None) -> None:
    """source_major: the received rows came by an all-to-all-v (source-major) rather than by
    moe_ep_dispatch (expert-major)."""
    _check(_lib.moe_ep_expert_ffn(_ptr(recv_x), max_recv_rows, int(bool(source_major)), R, rank, E, d, f,
                                  _ptr(W1_local), _ptr(W3_local),
                                  _ptr(W2_local), _ptr(h), _ptr(y_recv), _ptr(x), T, _ptr(W1s), _ptr(W3s), _ptr(W2s),
                                  f_shared, _ptr(h_shared), _ptr(y_shared), _ptr(ep_ws), _nbytes(ep_ws),
                                  _stream(stream)), "moe_ep_expert_ffn")


def moe_ep_return(y_recv, R, rank, E, d, y_perm_bufs, ep_ws, stream=None) -> None:
    """y_perm_bufs: R tensors (or device addresses), rank s's y_perm (in its layer workspace)."""
    _check(_lib.moe_ep_return(_ptr(y_recv), R, rank, E, d, _addr_array(y_perm_bufs), _ptr(ep_ws), _nbytes(ep_ws),
                              _stream(stream)), "moe_ep_return")


def moe_layer_permute_indices(x, f_shared, T, d, E, k, f, capacity, fill_base, ws, stream=None) -> None:
    """moe_layer_permute without the gather: dest and src_token only (x_perm unwritten)."""
    _check(_lib.moe_layer_permute_indices(_ptr(x), f_shared, T, d, E, k, f, int(capacity), _ptr(fill_base), _ptr(ws),
                                          _nbytes(ws), _stream(stream)), "moe_layer_permute_indices")


def moe_ep_dispatch_gather(x, src_token, R, rank, E, d, recv_bufs, ep_ws, stream=None) -> None:
    """The dispatch fused with the gather: x's kept rows straight into the receive buffers."""
    _check(_lib.moe_ep_dispatch_gather(_ptr(x), _ptr(src_token), R, rank, E, d, _addr_array(recv_bufs), _ptr(ep_ws),
                                       _nbytes(ep_ws), _stream(stream)), "moe_ep_dispatch_gather")


def moe_ep_expert_ffn_return(recv_x, max_recv_rows, R, rank, E, d, f, W1_local, W3_local, W2_local, h, x, T, W1s,
                             W3s, W2s, f_shared, h_shared, y_shared, y_perm_bufs, row_dest, ep_ws,
                             stream=None) -> None:
    """The local experts with the return exchange fused into GEMM2's stores: result rows go straight
    to y_perm_bufs[source rank] (R tensors or device addresses); row_dest: int64 scratch
    [max_recv_rows]."""
    _check(_lib.moe_ep_expert_ffn_return(_ptr(recv_x), max_recv_rows, R, rank, E, d, f, _ptr(W1_local),
                                         _ptr(W3_local), _ptr(W2_local), _ptr(h), _ptr(x), T, _ptr(W1s), _ptr(W3s),
                                         _ptr(W2s), f_shared, _ptr(h_shared), _ptr(y_shared),
                                         _addr_array(y_perm_bufs), _ptr(row_dest), _ptr(ep_ws), _nbytes(ep_ws),
                                         _stream(stream)), "moe_ep_expert_ffn_return")


def moe_ep_splits(ep_ws, R: int, E: int):
    """The [2, R] int32 split table moe_ep_plan wrote into ep_ws (a view, on the device): row 0 the
    rows this rank sends to each rank, row 1 the rows it receives from each rank."""
    import torch
    off = _sz(0)
    _check(_lib.moe_ep_splits_offset(R, E, ctypes.byref(off)), "moe_ep_splits_offset")
    o = int(off.value)
    return ep_ws[o:o + 8 * R].view(torch.int32).view(2, R)


def moe_ipc_export(t) -> bytes:
    """IPC handle (MOE_IPC_HANDLE_BYTES bytes) of the device allocation holding tensor t."""
    buf = ctypes.create_string_buffer(MOE_IPC_HANDLE_BYTES)
    _check(_lib.moe_ipc_export(_ptr(t), buf), "moe_ipc_export")
    return buf.raw


def moe_ipc_import(handle: bytes) -> int:
    """Device address, in this process, of another process's exported pointer."""
    if len(handle) != MOE_IPC_HANDLE_BYTES:
        raise ValueError("IPC handle of the wrong size")
    out = _vp(0)
    _check(_lib.moe_ipc_import(handle, ctypes.byref(out)), "moe_ipc_import")
    return int(out.value)


def moe_ipc_close(addr: int, handle: bytes) -> None:
    _check(_lib.moe_ipc_close(_vp(addr), handle), "moe_ipc_close")


def moe_workspace_bytes_a8(T: int, d: int, E: int, k: int, f: int, f_shared: int = 0) -> int:
    out = _sz(0)
    _check(_lib.moe_workspace_bytes_a8(T, d, E, k, f, f_shared, ctypes.byref(out)), "moe_workspace_bytes_a8")
    return int(out.value)


def moe_layer_forward_w8a8(x, Wg, bias, W1q, s1, W3q, s3, W2q, s2, W1sq, s1s, W3sq, s3s, W2sq, s2s, f_shared, T, d,
                           E, k, f, capacity_factor, cap_mode, out, ws, events: Optional[dict] = None,
                           stream=None) -> None:
    """The layer with fp8 e4m3 weights and fp8 activations (per-row scales); ws: a uint8 tensor of
    moe_workspace_bytes_a8() bytes."""
    ev = _events(events)
    _check(_lib.moe_layer_forward_w8a8(_ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1q), _ptr(s1), _ptr(W3q), _ptr(s3),
                                       _ptr(W2q), _ptr(s2), _ptr(W1sq), _ptr(s1s), _ptr(W3sq), _ptr(s3s),
                                       _ptr(W2sq), _ptr(s2s), f_shared, T, d, E, k, f, float(capacity_factor),
                                       cap_mode, _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream),
                                       ctypes.byref(ev) if ev is not None else None), "moe_layer_forward_w8a8")


def moe_get_error(stream=None) -> int:
    return int(_lib.moe_get_error(_stream(stream)))


def moe_selftest_wait_timeout(stream=None) -> None:
    """Enqueue the bounded-wait self-test (about 2 s; MOE_ERR_TIMEOUT in the error word)."""
    _check(_lib.moe_selftest_wait_timeout(_stream(stream)), "moe_selftest_wait_timeout")


def workspace_view(ws, layout: dict, name: str, shape, dtype):
    """A typed view of one intermediate inside a moe_layer_forward workspace (uint8 tensor)."""
    import torch
    n = 1
    for s in shape:
        n *= s
    nb = n * torch.empty((), dtype=dtype).element_size()
    o = layout[name]
    return ws[o:o + nb].view(dtype).view(*shape)
