"""moe_permute_noalloc: the permutation for callers that cannot allocate device memory.

Some callers of this library have no allocator at hand where they run the layer (a
plugin inside a framework that owns all device memory, an engine with a memory plan
fixed at start-up, a program that must not call cudaMalloc because it can synchronise
the device).  moe_permute_noalloc serves them: it takes only inputs and outputs and
keeps its scratch in a fixed array inside the library.  It must return exactly what
moe_permute (which takes a caller-allocated workspace) returns, call after call, even
though its scratch keeps the previous call's contents.

This file is collected last on purpose, so that a run that stops at its first failure
has already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import moe_layer_router_b200 as m
    assert torch.cuda.is_available()
    return m


def _problem(T, d, E, k, tid):
    logits = synth.normal_f64(0, tid, 0, T * E).astype(np.float32).reshape(T, E)
    idx, _ = oracle.route(logits, k)
    x = synth.normal_bf16(0, tid + 1, 0, T * d, 1.0).reshape(T, d)
    return (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda(), torch.from_numpy(idx).cuda())


def _outputs(T, d, E, k):
    i32 = lambda *s: torch.full(s, -7, dtype=torch.int32, device="cuda")
    return dict(counts_raw=i32(E), counts=i32(E), offsets=i32(E + 1), dest=i32(T, k), src_token=i32(T * k),
                x_perm=torch.zeros((T * k, d), dtype=torch.bfloat16, device="cuda"))


def test_noalloc_permute_matches_workspace_permute_on_consecutive_calls(moe):
    # the second call is smaller and has a capacity limit, so stale scratch from the
    # first call would show up if anything depended on it
    for (T, d, E, k, C, tid) in [(3000, 256, 64, 4, -1, 300), (777, 128, 128, 8, 40, 310)]:
        x, idx = _problem(T, d, E, k, tid)
        ref = _outputs(T, d, E, k)
        ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, 64), dtype=torch.uint8, device="cuda")
        moe.moe_permute(x, idx, T, d, E, k, C, ref["counts_raw"], ref["counts"], ref["offsets"], ref["dest"],
                        ref["src_token"], ref["x_perm"], ws)
        got = _outputs(T, d, E, k)
        moe.moe_permute_noalloc(x, idx, T, d, E, k, C, got["counts_raw"], got["counts"], got["offsets"],
                                got["dest"], got["src_token"], got["x_perm"])
        assert moe.moe_get_error() == 0
        N = int(ref["offsets"][E].item())
        assert (N < T * k) == (C >= 0)
        for name in ("counts_raw", "counts", "offsets", "dest"):
            assert torch.equal(got[name], ref[name]), name
        assert torch.equal(got["src_token"][:N], ref["src_token"][:N])
        assert torch.equal(got["x_perm"][:N], ref["x_perm"][:N])


def test_noalloc_permute_rejects_sizes_beyond_its_scratch(moe):
    # 2^20 tokens x 8 experts need 32 MiB of ranks alone; rejected before any launch
    with pytest.raises(moe.MoeError) as e:
        moe.moe_permute_noalloc(256, 256, 1 << 20, 64, 64, 8, -1, 256, 256, 256, 256, 256, 256)
    assert e.value.code == moe.MOE_ERR_WORKSPACE
