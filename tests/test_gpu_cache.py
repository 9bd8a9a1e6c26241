"""Expert cache on the GPU: the cache state against the cache oracle after every batch, the
layer output against the layer oracle and against the uncached layer, and the slot contents
against their source experts."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _util import assert_layer_close, bf16_bits, to_dev_bf16
from oracle.expert_cache import ExpertCacheOracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import moe_layer_router_b200 as m
    assert torch.cuda.is_available()
    return m


def _host_bf16(bits: np.ndarray, pinned: bool) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pinned else t.clone()


def _state(moe, state, E, S):
    lay = moe.moe_cache_layout(E, S)

    def arr(name, n):
        o = lay[name]
        return state[o:o + 4 * n].view(torch.int32).cpu().numpy()

    return dict(slot_of=arr("slot_of", E), expert_in=arr("expert_in", S), stamp=arr("stamp", S),
                load_expert=arr("load_expert", S), load_slot=arr("load_slot", S))


def _bias_towards(E, experts, big=50.0):
    b = np.zeros(E, np.float32)
    b[list(experts)] = big
    return b


# (T, d, E, k, f, S, f_shared, cap_mode, cf, zipf_s, batches, biased first batch)
CASES = {
    "evict": (8, 256, 64, 4, 128, 40, 0, synth.CAP_NONE, 1.0, 1.1, 14, None),
    "evict_shared_cap": (16, 256, 48, 2, 192, 32, 128, synth.CAP_PER_ASSIGNMENT, 2.0, 1.0, 10, None),
    "capacity_zero": (8, 128, 64, 4, 64, 32, 0, synth.CAP_PER_TOKEN, 1.0, 0.0, 3, None),
    "pair_tiles_remapped": (2048, 256, 8, 2, 256, 8, 0, synth.CAP_NONE, 1.0, 0.0, 3, (6, 7)),
}


@pytest.mark.parametrize("src", ["pinned", "device"])
@pytest.mark.parametrize("case", list(CASES))
def test_cached_layer_sequence(moe, case, src):
    T, d, E, k, f, S, fs, cap_mode, cf, zs, nb, first = CASES[case]
    wl = synth.Workload("cache_" + case, T, d, E, k, f, f_shared=fs, cap_mode=cap_mode, capacity_factor=cf,
                        zipf_s=zs, seed=7)
    inp = synth.Inputs(wl)
    wg = inp.wg()
    W1, W3, W2 = inp.w1(), inp.w3(), inp.w2()
    W1s, W3s, W2s = (inp.shared(n) for n in ("w1s", "w3s", "w2s")) if fs else (None, None, None)
    dv = to_dev_bf16
    dW1, dW3, dW2 = dv(W1), dv(W3), dv(W2)
    if src == "pinned":
        sW1, sW3, sW2 = (_host_bf16(a, True) for a in (W1, W3, W2))
    else:
        sW1, sW3, sW2 = dW1, dW3, dW2
    slots = [torch.empty((S,) + tuple(a.shape[1:]), dtype=torch.bfloat16, device="cuda") for a in (W1, W3, W2)]
    state = torch.empty(moe.moe_cache_state_bytes(E, S), dtype=torch.uint8, device="cuda")
    moe.moe_cache_reset(state, E, S)
    dsh = [dv(a) if a is not None else None for a in (W1s, W3s, W2s)]
    ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    ws2 = torch.empty_like(ws)
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    out_plain = torch.empty_like(out)
    C = oracle.capacity(T, E, k, cf, cap_mode)
    ref_cache = ExpertCacheOracle(E, S)
    dwg = dv(wg)
    for b in range(nb):
        x = inp.x_rows(b * T, T).reshape(T, d)
        bias = _bias_towards(E, first) if (first is not None and b == 0) else None
        dx = dv(x)
        dbias = torch.from_numpy(bias).cuda() if bias is not None else None
        moe.moe_layer_forward_cached(dx, dwg, dbias, sW1, sW3, sW2, *slots, S, state, *dsh, fs, T, d, E, k, f, cf,
                                     cap_mode, out, ws)
        moe.moe_layer_forward(dx, dwg, dbias, dW1, dW3, dW2, *dsh, fs, T, d, E, k, f, cf, cap_mode, out_plain, ws2)
        assert moe.moe_get_error() == 0
        logits = moe.workspace_view(ws, L, "logits", (T, E), torch.float32).cpu().numpy()
        r = oracle.layer_forward(x, wg, W1, W3, W2, k=k, C=C, bias=bias, logits_in=logits,
                                 W1s=W1s, W3s=W3s, W2s=W2s)
        # cache decisions: bit-exact against the oracle fed the batch's needed experts
        need = np.nonzero(r["counts"] > 0)[0]
        loads = ref_cache.batch(need)
        st = _state(moe, state, E, S)
        ctr = moe.cache_counters(state)
        assert ctr == dict(step=b + 1, hits=ref_cache.hits, misses=ref_cache.misses, loads_last=len(loads))
        got = list(zip(st["load_expert"][:len(loads)].tolist(), st["load_slot"][:len(loads)].tolist()))
        assert got == loads
        assert st["slot_of"].tolist() == ref_cache.slot_of
        assert st["expert_in"].tolist() == ref_cache.expert_in
        assert st["stamp"].tolist() == ref_cache.stamp
        # the output: the layer's, whichever slot each expert sits in
        assert np.array_equal(bf16_bits(out), bf16_bits(out_plain))
        assert_layer_close(bf16_bits(out), r["out"])
    if case == "capacity_zero":
        assert C == 0 and ref_cache.misses == 0
    else:
        assert ref_cache.misses > 0
        if case != "pair_tiles_remapped":
            assert ref_cache.hits > 0
        else:
            assert ref_cache.slot_of != list(range(E))       # the slot map is not the identity
    # every resident slot holds its expert's weights, bit for bit
    for e, v in enumerate(ref_cache.slot_of):
        if v >= 0:
            for sl, dw in zip(slots, (dW1, dW3, dW2)):
                assert torch.equal(sl[v].view(torch.int16), dw[e].view(torch.int16))


def test_cached_layer_rejects_pageable_source(moe):
    T, d, E, k, f, S = 8, 128, 16, 2, 64, 16
    x = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros((E, d), dtype=torch.bfloat16, device="cuda")
    W1 = torch.zeros((E, f, d), dtype=torch.bfloat16)          # pageable host memory
    slots = [torch.empty((S, f, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    slots.append(torch.empty((S, d, f), dtype=torch.bfloat16, device="cuda"))
    state = torch.empty(moe.moe_cache_state_bytes(E, S), dtype=torch.uint8, device="cuda")
    ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_layer_forward_cached(x, wg, None, W1, W1, W1.transpose(1, 2).contiguous(), *slots, S, state,
                                     None, None, None, 0, T, d, E, k, f, 1.0, moe.MOE_CAP_NONE, out, ws)
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("src", ["pinned", "device"])
def test_cached_layer_fp8_experts(moe, src):
    """fp8 experts through the cache: state against the cache oracle, output bit-identical to the
    uncached fp8 layer, slots equal to their source experts."""
    T, d, E, k, f, S, fs = 8, 256, 48, 4, 192, 32, 128
    wl = synth.Workload("cache_q8", T, d, E, k, f, f_shared=fs, zipf_s=1.1, seed=9)
    inp = synth.Inputs(wl)
    Q = synth.device_tensors_q8(wl, "cuda")
    names = {"W1q": "w1q", "W3q": "w3q", "W2q": "w2q", "s1": "s1", "s3": "s3", "s2": "s2"}
    dev_src = {n: Q[q] for n, q in names.items()}
    srcs = {n: (t.cpu().pin_memory() if src == "pinned" else t) for n, t in dev_src.items()}
    slots = {n: torch.empty((S,) + tuple(t.shape[1:]), dtype=t.dtype, device="cuda") for n, t in dev_src.items()}
    shared = {"W1q": Q["w1sq"], "W3q": Q["w3sq"], "W2q": Q["w2sq"], "s1": Q["s1s"], "s3": Q["s3s"], "s2": Q["s2s"]}
    state = torch.empty(moe.moe_cache_state_bytes(E, S), dtype=torch.uint8, device="cuda")
    moe.moe_cache_reset(state, E, S)
    ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    ws2 = torch.empty_like(ws)
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    out_plain = torch.empty_like(out)
    wg = to_dev_bf16(inp.wg())
    ref_cache = ExpertCacheOracle(E, S)
    for b in range(8):
        x = to_dev_bf16(inp.x_rows(b * T, T).reshape(T, d))
        moe.moe_layer_forward_cached_w8(x, wg, None, srcs, slots, S, state, shared, fs, T, d, E, k, f, 1.0,
                                        moe.MOE_CAP_NONE, out, ws)
        moe.moe_layer_forward_w8(x, wg, None, Q["w1q"], Q["s1"], Q["w3q"], Q["s3"], Q["w2q"], Q["s2"], Q["w1sq"],
                                 Q["s1s"], Q["w3sq"], Q["s3s"], Q["w2sq"], Q["s2s"], fs, T, d, E, k, f, 1.0,
                                 moe.MOE_CAP_NONE, out_plain, ws2)
        assert moe.moe_get_error() == 0
        counts = moe.workspace_view(ws, L, "counts", (E,), torch.int32).cpu().numpy()
        loads = ref_cache.batch(np.nonzero(counts > 0)[0])
        st = _state(moe, state, E, S)
        assert list(zip(st["load_expert"][:len(loads)].tolist(), st["load_slot"][:len(loads)].tolist())) == loads
        assert st["slot_of"].tolist() == ref_cache.slot_of
        assert torch.equal(out.view(torch.int16), out_plain.view(torch.int16))
    assert ref_cache.misses > 0 and ref_cache.hits > 0
    for e, v in enumerate(ref_cache.slot_of):
        if v >= 0:
            for n in names:
                assert torch.equal(slots[n][v], dev_src[n][e]), n
