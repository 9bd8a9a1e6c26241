"""The C-ABI library without a GPU: it loads, exports every symbol the header declares,
and its host-only logic (capacity, workspace sizes, argument validation) behaves."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")
LIB = os.path.join(ROOT, "moe_layer_router_b200", "libmoe_b200.so")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        import __graft_entry__
        __graft_entry__.build()
    return ctypes.CDLL(LIB)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+\**(moe_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_layer_entry_points():
    names = declared_functions()
    for n in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward"):
        assert n in names
    assert len(names) >= 10


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(declared_functions()) <= exported


def test_capacity_host(lib):
    lib.moe_capacity.restype = ctypes.c_int64
    lib.moe_capacity.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int]
    assert lib.moe_capacity(32768, 64, 2, 1.25, 2) == 1280
    assert lib.moe_capacity(32768, 64, 2, 1.25, 1) == 640
    assert lib.moe_capacity(4096, 8, 2, 2.0, 1) == 1024
    assert lib.moe_capacity(10, 3, 1, 0.9, 1) == 3
    assert lib.moe_capacity(10, 3, 1, 0.9, 0) == -1
    for T, E, k, cf in [(1000, 7, 3, 1.1), (999, 10, 1, 0.3), (16384, 128, 8, 1.0)]:
        assert lib.moe_capacity(T, E, k, cf, 1) == int(T / E * cf)
        assert lib.moe_capacity(T, E, k, cf, 2) == int(T * k / E * cf)


def test_workspace_sizes_and_layout(lib):
    sz = ctypes.c_size_t(0)
    lib.moe_workspace_bytes.argtypes = [ctypes.c_int] * 6 + [ctypes.POINTER(ctypes.c_size_t)]
    assert lib.moe_workspace_bytes(4096, 4096, 8, 2, 14336, 0, ctypes.byref(sz)) == 0
    T, d, E, k, f = 4096, 4096, 8, 2, 14336
    big = T * k * d * 2 * 2 + T * k * f * 2
    assert big < sz.value < big * 1.05
    off = (ctypes.c_size_t * 13)()
    lib.moe_workspace_layout.argtypes = [ctypes.c_int] * 6 + [ctypes.c_size_t * 13]
    assert lib.moe_workspace_layout(T, d, E, k, f, 0, off) == 0
    offs = list(off)
    assert all(o % 256 == 0 for o in offs)
    assert offs[:11] == sorted(offs[:11]) and offs[10] + T * k * d * 2 <= sz.value
    # with a shared expert: y_shared [T, d] then h_shared [T, f_s] follow y_perm
    assert lib.moe_workspace_layout(T, d, E, k, f, 2048, off) == 0
    offs = list(off)
    assert offs[10] < offs[11] < offs[12] and offs[11] + T * d * 2 <= offs[12]
    # shape checks: d % 64, k <= 32, k <= E, E <= 1024
    for args in [(128, 100, 8, 2, 512), (128, 256, 8, 33, 512), (128, 256, 4, 8, 512), (128, 256, 2000, 2, 512),
                 (0, 256, 8, 2, 512), (128, 256, 8, 2, 500)]:
        assert lib.moe_workspace_bytes(*args, 0, ctypes.byref(sz)) == -2


def test_entry_points_validate_before_touching_the_device(lib):
    vp = ctypes.c_void_p
    # a bad shape is rejected on the host, without a GPU
    lib.moe_layer_forward.argtypes = [vp] * 9 + [ctypes.c_int] * 6 + [ctypes.c_double, ctypes.c_int, vp, vp,
                                                                         ctypes.c_size_t, vp]
    assert lib.moe_layer_forward(*([None] * 9), 0, 128, 100, 8, 2, 512, 1.0, 0, None, None, 0, None) == -2
    assert lib.moe_layer_forward(*([None] * 9), 0, 128, 256, 8, 2, 512, 1.0, 0, None, None, 0, None) == -1
    assert lib.moe_layer_forward(*([None] * 9), 0, 128, 256, 8, 2, 512, 1.0, 7, None, None, 0, None) == -1
    lib.moe_combine.argtypes = [vp, vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]
    assert lib.moe_combine(None, None, None, None, 8, 64, 2, None, None) == -1
    assert lib.moe_combine(16, 16, 16, None, 8, 65, 2, 16, None) == -2
    assert lib.moe_combine(16, 16, 16, None, 8, 64, 2, 17, None) == -3     # misaligned out
    lib.moe_strerror.restype = ctypes.c_char_p
    assert lib.moe_strerror(-4) == b"workspace too small"


def test_expert_cache_host_checks(lib):
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.moe_cache_state_bytes.argtypes = [i32, i32, ctypes.POINTER(sz)]
    lib.moe_cache_layout.argtypes = [i32, i32, ctypes.POINTER(sz)]
    b = sz(0)
    assert lib.moe_cache_state_bytes(256, 128, ctypes.byref(b)) == 0
    # 64-byte counters, then slot_of [256] and four [128] int32 arrays
    assert b.value == 64 + 256 * 4 + 4 * 128 * 4
    off = (sz * 6)()
    assert lib.moe_cache_layout(10, 3, off) == 0
    assert list(off) == [0, 64, 64 + 48, 64 + 48 + 16, 64 + 48 + 32, 64 + 48 + 48]   # padded to 16 bytes
    assert lib.moe_cache_state_bytes(8, 9, ctypes.byref(b)) == -2      # more slots than experts
    assert lib.moe_cache_state_bytes(2048, 16, ctypes.byref(b)) == -2  # more than 1024 experts
    assert lib.moe_cache_state_bytes(8, 0, ctypes.byref(b)) == -2
    # the layer needs S >= min(E, T*k) slots; checked before any device call
    lib.moe_layer_forward_cached.argtypes = [vp] * 9 + [i32, vp, vp, vp, vp] + [i32] * 6 + \
        [ctypes.c_double, i32, vp, vp, sz, vp, vp]
    args = [16] * 9
    assert lib.moe_layer_forward_cached(*args, 15, 16, None, None, None, 0, 8, 128, 64, 2, 64, 1.0, 0,
                                        16, 16, 1 << 20, None, None) == -2            # 15 < min(64, 16)
    assert lib.moe_layer_forward_cached(*args, 65, 16, None, None, None, 0, 8, 128, 64, 2, 64, 1.0, 0,
                                        16, 16, 1 << 20, None, None) == -2            # S > E
    assert lib.moe_layer_forward_cached(*([16] * 8 + [None]), 16, 16, None, None, None, 0, 8, 128, 64, 2, 64,
                                        1.0, 0, 16, 16, 1 << 20, None, None) == -1    # missing slots
    assert lib.moe_layer_forward_cached(*([16] * 8 + [24]), 16, 16, None, None, None, 0, 8, 128, 64, 2, 64,
                                        1.0, 0, 16, 16, 1 << 20, None, None) == -3    # misaligned slots


def test_expert_parallel_host_checks(lib):
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.moe_ep_workspace_bytes.argtypes = [i32, i32, ctypes.POINTER(sz)]
    b = sz(0)
    assert lib.moe_ep_workspace_bytes(8, 256, ctypes.byref(b)) == 0 and b.value >= 8 * 256 * 4 + 6 * 256 * 4
    assert lib.moe_ep_workspace_bytes(8, 2048, ctypes.byref(b)) == -2
    assert lib.moe_ep_workspace_bytes(3, 256, ctypes.byref(b)) == -2
    lib.moe_ep_plan.argtypes = [vp, i32, i32, i32, i64, i32, vp, sz, vp]
    ws = 1 << 20
    assert lib.moe_ep_plan(16, 3, 0, 16, -1, 100, 16, ws, None) == -2     # E not a multiple of R
    assert lib.moe_ep_plan(16, 65, 0, 130, -1, 100, 16, ws, None) == -2   # more than 64 ranks
    assert lib.moe_ep_plan(16, 4, 4, 16, -1, 100, 16, ws, None) == -2     # rank out of range
    assert lib.moe_ep_plan(None, 4, 1, 16, -1, 100, 16, ws, None) == -1   # no counts
    assert lib.moe_ep_plan(16, 4, 1, 16, -1, 100, 24, ws, None) == -3     # misaligned workspace
    assert lib.moe_ep_plan(16, 4, 1, 16, -1, 100, 16, 64, None) == -4     # workspace too small
    lib.moe_ep_dispatch.argtypes = [vp, i32, i32, i32, i32, vp, vp, sz, vp]
    assert lib.moe_ep_dispatch(16, 2, 0, 8, 100, 16, 16, ws, None) == -2   # d not a multiple of 64
    lib.moe_layer_permute.argtypes = [vp, i32, i32, i32, i32, i32, i32, i64, vp, vp, sz, vp]
    assert lib.moe_layer_permute(16, 0, 8, 100, 8, 2, 64, -1, None, 16, ws, None) == -2


def test_cached_fp8_entry_host_checks(lib):
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t

    class W8(ctypes.Structure):
        _fields_ = [(n, vp) for n in ("W1q", "W3q", "W2q", "s1", "s3", "s2")]

    lib.moe_layer_forward_cached_w8.argtypes = [vp, vp, vp, ctypes.POINTER(W8), ctypes.POINTER(W8), i32, vp,
                                                ctypes.POINTER(W8), i32, i32, i32, i32, i32, i32,
                                                ctypes.c_double, i32, vp, vp, sz, vp, vp]
    src, slots = W8(*([16] * 6)), W8(*([32] * 6))
    call = lambda S, a, b, T=8, k=2, E=64: lib.moe_layer_forward_cached_w8(
        16, 16, None, a, b, S, 16, None, 0, T, 128, E, k, 64, 1.0, 0, 16, 16, 1 << 20, None, None)
    assert call(15, ctypes.byref(src), ctypes.byref(slots)) == -2          # S < min(E, T*k)
    assert call(16, None, ctypes.byref(slots)) == -1                        # no sources
    bad = W8(16, 16, 16, 16, 16, 24)
    assert call(16, ctypes.byref(src), ctypes.byref(bad)) == -3             # misaligned slot array


def test_fp8_activation_entry_needs_128_byte_k(lib):
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.moe_layer_forward_w8a8.argtypes = [vp] * 15 + [i32] * 6 + [ctypes.c_double, i32, vp, vp, sz, vp, vp]
    args = [16] * 15
    # d = 192 is a multiple of 64 but not of 128: the fp8 stage rows are 128 K-elements
    assert lib.moe_layer_forward_w8a8(*args, 0, 8, 192, 8, 2, 256, 1.0, 0, 16, 16, 1 << 20, None, None) == -2
    assert lib.moe_layer_forward_w8a8(*args, 64, 8, 256, 8, 2, 256, 1.0, 0, 16, 16, 1 << 20, None, None) == -2
    lib.moe_workspace_bytes_a8.argtypes = [i32] * 6 + [ctypes.POINTER(sz)]
    lib.moe_workspace_bytes.argtypes = [i32] * 6 + [ctypes.POINTER(sz)]
    a, b = sz(0), sz(0)
    assert lib.moe_workspace_bytes_a8(256, 7168, 256, 8, 2048, 2048, ctypes.byref(a)) == 0
    assert lib.moe_workspace_bytes(256, 7168, 256, 8, 2048, 2048, ctypes.byref(b)) == 0
    # plus fp8 copies of the permuted rows and of h (routed and shared) and their scales
    assert a.value >= b.value + 2048 * (7168 + 2048) + 256 * (7168 + 2048)


def header_struct_fields(name):
    """Field names of a `typedef struct name { ... } name;` in the header, in order."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    m = re.search(r"typedef struct %s \{(.*?)\} %s;" % (name, name), src, flags=re.S)
    assert m, name
    names = []
    for decl in m.group(1).split(";"):
        for part in decl.split(","):
            ids = re.findall(r"[A-Za-z_][A-Za-z0-9_]*", part)
            if ids:
                names.append(ids[-1])
    return names


def test_binding_stage_events_match_the_header():
    """The ctypes mirror of moe_stage_events has the header's members in the header's order
    (the library reads the whole struct, so a missing trailing member would be read past)."""
    import moe_layer_router_b200 as moe
    fields = header_struct_fields("moe_stage_events")
    assert [n for n, _ in moe.moe_stage_events._fields_] == fields
    assert ctypes.sizeof(moe.moe_stage_events) == len(fields) * ctypes.sizeof(ctypes.c_void_p)
    assert fields[:len(moe.STAGES)] == moe.STAGES


@pytest.mark.parametrize("name", ["moe_pipeline_params", "moe_w8_experts"])
def test_binding_structs_match_the_header(name):
    import moe_layer_router_b200 as moe
    assert [n for n, _ in getattr(moe, name)._fields_] == header_struct_fields(name)


def test_ep_split_table_offset_and_ipc_validation(lib):
    sz = ctypes.c_size_t(0)
    lib.moe_ep_splits_offset.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
    lib.moe_ep_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
    for R, E in [(1, 8), (4, 32), (8, 256), (64, 1024)]:
        assert lib.moe_ep_splits_offset(R, E, ctypes.byref(sz)) == 0
        off = sz.value
        assert lib.moe_ep_workspace_bytes(R, E, ctypes.byref(sz)) == 0
        assert off % 256 == 0 and off + 8 * R <= sz.value          # the [2, R] table fits, aligned
    assert lib.moe_ep_splits_offset(3, 8, ctypes.byref(sz)) == -2     # E not a multiple of R
    assert lib.moe_ep_splits_offset(4, 32, None) == -1
    vp = ctypes.c_void_p
    lib.moe_ipc_export.argtypes = [vp, vp]
    lib.moe_ipc_import.argtypes = [vp, ctypes.POINTER(vp)]
    lib.moe_ipc_close.argtypes = [vp, vp]
    blob = ctypes.create_string_buffer(96)
    out = vp(0)
    assert lib.moe_ipc_export(None, blob) == -1
    assert lib.moe_ipc_export(4096, None) == -1
    assert lib.moe_ipc_import(blob, ctypes.byref(out)) == -1          # not a handle this library wrote
    assert lib.moe_ipc_import(None, ctypes.byref(out)) == -1
    assert lib.moe_ipc_close(None, blob) == -1
    assert lib.moe_ipc_close(4096, blob) == -1
