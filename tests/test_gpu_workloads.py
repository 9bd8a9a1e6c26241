"""Full-size parity: the four large workloads, in the launch configuration bench.py times.

For every token: routing recomputed by the oracle from the GPU's fp32 logits equals the
GPU's routing bit for bit, and so do the histogram, capacity, offsets, dest and src_token.
For a seeded sample of tokens: logits against the oracle's double sums, the oracle's own
routing on tokens without a near tie, x_perm rows, and the layer output against the oracle
(its expert weights regenerated from the seeded generator, never read back from the GPU).
"""
import gc

import numpy as np
import pytest
import torch

import oracle
import synth
from _util import assert_layer_close, bf16_bits, bits_to_f64, logits_tol, ulp_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import moe_layer_router_b200 as m
    assert torch.cuda.is_available()
    return m


SAMPLES = {"mixtral": 12, "qwen3": 12, "dsv3": 6, "skew": 12}


@pytest.mark.parametrize("name", ["mixtral", "qwen3", "dsv3", "skew"])
def test_full_size_layer(moe, name):
    wl = synth.WORKLOADS[name]
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    W = synth.device_tensors(wl, "cuda")
    ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    evs = {n: torch.cuda.Event(enable_timing=True) for n in moe.STAGES}
    for e in evs.values():
        e.record()
    moe.moe_layer_forward_ex(W["x"], W["wg"], W["bias"], W["w1"], W["w3"], W["w2"], W.get("w1s"), W.get("w3s"),
                             W.get("w2s"), fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, out, ws, evs)
    assert moe.moe_get_error() == 0
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    v = lambda n, s, dt: moe.workspace_view(ws, L, n, s, dt).cpu()
    g_logits = v("logits", (T, E), torch.float32).numpy()
    g_idx = v("idx", (T, k), torch.int32).numpy()
    g_w = v("w", (T, k), torch.float32).numpy()
    inp = synth.Inputs(wl)
    bias = inp.bias()

    # (ii) routing from the GPU's logits, every token
    idx_o, w_o = oracle.route(g_logits, k, bias)
    assert np.array_equal(g_idx, idx_o)
    np.testing.assert_allclose(g_w, w_o, rtol=1e-5, atol=1e-7)
    C = oracle.capacity(T, E, k, wl.capacity_factor, wl.cap_mode)
    r = oracle.dispatch(g_idx, E, C)
    for n in ("counts_raw", "counts"):
        assert np.array_equal(v(n, (E,), torch.int32).numpy(), r[n]), n
    assert np.array_equal(v("offsets", (E + 1,), torch.int32).numpy(), r["offsets"])
    g_dest = v("dest", (T, k), torch.int32).numpy()
    assert np.array_equal(g_dest, r["dest"])
    N = r["N"]
    assert np.array_equal(v("src_token", (T * k,), torch.int32).numpy()[:N], r["src_token"])

    # seeded token sample
    rng = np.random.default_rng(7)
    toks = sorted(set([0, T - 1] + list(rng.choice(T, SAMPLES[name] - 2, replace=False))))
    xs = np.stack([inp.x_rows(t, 1) for t in toks])                        # [S, d] bf16 bits
    wg = inp.wg()
    # (i) logits of the sampled rows
    ref_logits = oracle.router_logits(xs, wg)
    assert np.all(np.abs(g_logits[toks].astype(np.float64) - ref_logits) <= logits_tol(xs, wg))
    # (iii) the oracle's own routing on sampled tokens with a clear k-th key
    own_idx, _ = oracle.route(ref_logits.astype(np.float32), k, bias)
    keys = np.sort(ref_logits + (bias if bias is not None else 0), axis=1)[:, ::-1]
    clear = (keys[:, k - 1] - keys[:, k]) >= 1e-5
    assert np.array_equal(own_idx[clear], g_idx[toks][clear])
    # x_perm rows of the sample
    x_perm = moe.workspace_view(ws, L, "x_perm", (T * k, d), torch.bfloat16)
    for i, t in enumerate(toks):
        for j in range(k):
            if g_dest[t, j] >= 0:
                assert np.array_equal(bf16_bits(x_perm[int(g_dest[t, j])]), xs[i])

    # (iv) outputs of the sampled tokens: oracle experts on regenerated weights
    y = {}                                                                  # (i, j) -> y row
    by_expert = {}
    for i, t in enumerate(toks):
        for j in range(k):
            if g_dest[t, j] >= 0:
                by_expert.setdefault(int(g_idx[t, j]), []).append((i, j))
    per = f * d
    for e, items in by_expert.items():
        W1e = inp.expert_rows("w1", e, 1).reshape(f, d)
        W3e = inp.expert_rows("w3", e, 1).reshape(f, d)
        W2e = inp.expert_rows("w2", e, 1).reshape(d, f)
        _, ye = oracle.expert_ffn(np.stack([xs[i] for i, _ in items]), W1e, W3e, W2e)
        for (i, j), row in zip(items, ye):
            y[(i, j)] = row
    ysh = None
    if fs:
        _, ysh = oracle.expert_ffn(xs, inp.shared("w1s"), inp.shared("w3s"), inp.shared("w2s"))
    S = len(toks)
    mini_y = np.zeros((S * k, d), np.uint16)
    mini_dest = np.full((S, k), -1, np.int32)
    for (i, j), row in y.items():
        mini_y[i * k + j] = row
        mini_dest[i, j] = i * k + j
    ref_out = oracle.combine(mini_y, mini_dest, w_o[toks], ysh)
    got = bf16_bits(out[toks])
    assert_layer_close(got, ref_out, f"{name} sampled outputs")
    g64, r64 = bits_to_f64(got), bits_to_f64(ref_out)
    assert np.sqrt(np.mean((g64 - r64) ** 2) / np.mean(r64 ** 2)) < 5e-3      # no systematic drift

    if name == "skew":
        assert C == 1280 and r["counts"].max() <= C
        drop = 1.0 - N / (T * k)
        assert 0.4 < drop < 0.65
        p = r["counts_raw"] / r["counts_raw"].sum()
        assert np.abs(p - inp.zipf_target()).sum() < 0.1
    del W, ws, out, x_perm
    gc.collect()
    torch.cuda.empty_cache()


def test_full_size_decode_fp8_weights(moe):
    """The DeepSeek-V3-like decode layer with fp8 e4m3 expert weights (bench.py --weights fp8):
    routing bit-exact for every token, sampled outputs against the oracle's fp8 experts on
    weights regenerated and quantised on the host."""
    wl = synth.WORKLOADS["dsv3"]
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    W = synth.device_tensors(wl, "cuda", names=["x", "wg", "bias"])
    Q = synth.device_tensors_q8(wl, "cuda")
    ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_w8(W["x"], W["wg"], W["bias"], Q["w1q"], Q["s1"], Q["w3q"], Q["s3"], Q["w2q"], Q["s2"],
                             Q["w1sq"], Q["s1s"], Q["w3sq"], Q["s3s"], Q["w2sq"], Q["s2s"], fs, T, d, E, k, f,
                             wl.capacity_factor, wl.cap_mode, out, ws)
    assert moe.moe_get_error() == 0
    del Q
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    v = lambda n, s, dt: moe.workspace_view(ws, L, n, s, dt).cpu()
    g_logits = v("logits", (T, E), torch.float32).numpy()
    g_idx = v("idx", (T, k), torch.int32).numpy()
    inp = synth.Inputs(wl)
    idx_o, w_o = oracle.route(g_logits, k, inp.bias())
    assert np.array_equal(g_idx, idx_o)
    r = oracle.dispatch(g_idx, E, -1)
    g_dest = v("dest", (T, k), torch.int32).numpy()
    assert np.array_equal(g_dest, r["dest"])

    rng = np.random.default_rng(11)
    toks = sorted(set([0, T - 1] + list(rng.choice(T, 4, replace=False))))
    xs = np.stack([inp.x_rows(t, 1) for t in toks])
    by_expert = {}
    for i, t in enumerate(toks):
        for j in range(k):
            by_expert.setdefault(int(g_idx[t, j]), []).append((i, j))
    y = {}
    for e, items in by_expert.items():
        q1, s1 = synth.quantize_e4m3_rows(inp.expert_rows("w1", e, 1), d)
        q3, s3 = synth.quantize_e4m3_rows(inp.expert_rows("w3", e, 1), d)
        q2, s2 = synth.quantize_e4m3_rows(inp.expert_rows("w2", e, 1), f)
        _, ye = oracle.expert_ffn_q8(np.stack([xs[i] for i, _ in items]), q1, s1, q3, s3, q2, s2)
        for (i, j), row in zip(items, ye):
            y[(i, j)] = row
    qs = {n: synth.quantize_e4m3_rows(inp.shared(n), inp.shared(n).shape[1]) for n in ("w1s", "w3s", "w2s")}
    _, ysh = oracle.expert_ffn_q8(xs, qs["w1s"][0], qs["w1s"][1], qs["w3s"][0], qs["w3s"][1], qs["w2s"][0],
                                  qs["w2s"][1])
    S = len(toks)
    mini_y = np.zeros((S * k, d), np.uint16)
    mini_dest = np.full((S, k), -1, np.int32)
    for (i, j), row in y.items():
        mini_y[i * k + j] = row
        mini_dest[i, j] = i * k + j
    ref_out = oracle.combine(mini_y, mini_dest, w_o[toks], ysh)
    got = bf16_bits(out[toks])
    assert_layer_close(got, ref_out, "dsv3 fp8 sampled outputs")
    g64, r64 = bits_to_f64(got), bits_to_f64(ref_out)
    assert np.sqrt(np.mean((g64 - r64) ** 2) / np.mean(r64 ** 2)) < 5e-3


@pytest.mark.parametrize("name", ["dsv3", "mixtral"])
def test_full_size_fp8_weights_and_activations(moe, name):
    """bench.py --weights fp8a8 at full size (decode on 1-SM tiles, prefill on 2-SM tiles): routing
    bit-exact for every token, sampled outputs against the oracle's fp8 x fp8 experts on weights
    regenerated and quantised on the host."""
    wl = synth.WORKLOADS[name]
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    W = synth.device_tensors(wl, "cuda", names=["x", "wg", "bias"])
    Q = synth.device_tensors_q8(wl, "cuda")
    ws = torch.empty(moe.moe_workspace_bytes_a8(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_w8a8(W["x"], W["wg"], W.get("bias"), Q["w1q"], Q["s1"], Q["w3q"], Q["s3"], Q["w2q"],
                               Q["s2"], Q.get("w1sq"), Q.get("s1s"), Q.get("w3sq"), Q.get("s3s"), Q.get("w2sq"),
                               Q.get("s2s"), fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, out, ws)
    assert moe.moe_get_error() == 0
    del Q
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    v = lambda n, s, dt: moe.workspace_view(ws, L, n, s, dt).cpu()
    g_logits = v("logits", (T, E), torch.float32).numpy()
    g_idx = v("idx", (T, k), torch.int32).numpy()
    inp = synth.Inputs(wl)
    idx_o, w_o = oracle.route(g_logits, k, inp.bias())
    assert np.array_equal(g_idx, idx_o)
    g_dest = v("dest", (T, k), torch.int32).numpy()
    rng = np.random.default_rng(13)
    toks = sorted(set([0, T - 1] + list(rng.choice(T, 4, replace=False))))
    xs = np.stack([inp.x_rows(t, 1) for t in toks])
    h_all = moe.workspace_view(ws, L, "h", (T * k, f), torch.bfloat16)
    # the first GEMM against the oracle; the second on the GPU's h, so both sides quantise the
    # same h rows
    by_expert = {}
    for i, t in enumerate(toks):
        for j in range(k):
            if g_dest[t, j] >= 0:
                by_expert.setdefault(int(g_idx[t, j]), []).append((i, j, int(g_dest[t, j])))
    y = {}
    for e, items in by_expert.items():
        q1, s1 = synth.quantize_e4m3_rows(inp.expert_rows("w1", e, 1), d)
        q3, s3 = synth.quantize_e4m3_rows(inp.expert_rows("w3", e, 1), d)
        q2, s2 = synth.quantize_e4m3_rows(inp.expert_rows("w2", e, 1), f)
        h_ref = oracle.expert_gate_up_w8a8(np.stack([xs[i] for i, _, _ in items]), q1, s1, q3, s3)
        g_h = np.stack([bf16_bits(h_all[r]) for _, _, r in items])
        g64, r64 = bits_to_f64(g_h), bits_to_f64(h_ref)
        assert not (np.abs(g64 - r64) > 1e-3 + 8e-3 * np.abs(r64)).any(), f"h of expert {e}"
        ye = oracle.expert_down_w8a8(g_h, q2, s2)
        for (i, j, _), row in zip(items, ye):
            y[(i, j)] = row
    ysh = None
    if fs:
        qs = {n: synth.quantize_e4m3_rows(inp.shared(n), inp.shared(n).shape[1]) for n in ("w1s", "w3s", "w2s")}
        g_hs = bf16_bits(moe.workspace_view(ws, L, "h_shared", (T, fs), torch.bfloat16)[toks])
        hs_ref = oracle.expert_gate_up_w8a8(xs, qs["w1s"][0], qs["w1s"][1], qs["w3s"][0], qs["w3s"][1])
        g64, r64 = bits_to_f64(g_hs), bits_to_f64(hs_ref)
        assert not (np.abs(g64 - r64) > 1e-3 + 8e-3 * np.abs(r64)).any(), "shared h"
        ysh = oracle.expert_down_w8a8(g_hs, qs["w2s"][0], qs["w2s"][1])
    S = len(toks)
    mini_y = np.zeros((S * k, d), np.uint16)
    mini_dest = np.full((S, k), -1, np.int32)
    for (i, j), row in y.items():
        mini_y[i * k + j] = row
        mini_dest[i, j] = i * k + j
    ref_out = oracle.combine(mini_y, mini_dest, w_o[toks], ysh)
    got = bf16_bits(out[toks])
    assert_layer_close(got, ref_out, f"{name} fp8 x fp8 sampled outputs")
    g64, r64 = bits_to_f64(got), bits_to_f64(ref_out)
    assert np.sqrt(np.mean((g64 - r64) ** 2) / np.mean(r64 ** 2)) < 5e-3
