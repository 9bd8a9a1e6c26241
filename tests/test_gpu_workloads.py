"""Full-size parity: the four large workloads, in the launch configuration bench.py times.

Every token: routing recomputed by the oracle from the GPU's fp32 logits equals the GPU's
routing bit for bit, and so do the histogram, capacity, offsets, dest, src_token and every
x_perm row; the logits are within 1e-5 (absolute) of the oracle's double sums; the oracle's
own routing (from its own logits) matches on every token whose k-th and (k+1)-th keys are at
least 1e-5 apart.

Expert outputs (h, y_perm, y_shared) and the layer output against the oracle, whose expert
weights are regenerated from the seeded generator (never read back from the GPU):
  - every token of the Mixtral-like, DeepSeek-V3-like and skewed layers;
  - for the Qwen3-like layer (131 072 kept rows) the tokens of a covering set of rows: the
    first, the last and one seeded row of every 128-row block of every expert's rows, which
    reaches both halves of every 256-row pair tile, every 128-row tile and every ragged tail.
The fp8 layers (bench.py --weights fp8 / fp8a8) route exactly like the bf16 layer (checked on
every token again); their expert GEMMs are checked on 24-32 seeded tokens of the decode layer and,
for the prefill layer, on the tokens of the first, last and one seeded row of every 256-row tile
of every expert (the fp8 oracle is the slowest part of the suite).
Each test prints the largest logit error and the largest output difference (pytest -rA).
"""
import gc

import numpy as np
import pytest
import torch

import oracle
import synth
from _util import assert_layer_close, bf16_bits, bits_to_f64

pytestmark = pytest.mark.gpu

LOGITS_ATOL = 1e-5           # the router logits bar (absolute)
H_BAR = (1e-3, 8e-3)         # h: |d| <= 1e-3 + 8e-3 |ref|
OUT_BAR = (1e-2, 2e-2)       # expert and layer outputs: |d| <= 1e-2 + 2e-2 |ref|
FULL = {"mixtral": "all", "qwen3": "cover", "dsv3": "all", "skew": "all"}


@pytest.fixture(scope="module")
def moe():
    import moe_layer_router_b200 as m
    assert torch.cuda.is_available()
    return m


def covering_rows(offsets: np.ndarray, seed: int, block: int = 128) -> np.ndarray:
    """First, last and one seeded row of every `block`-row block of every expert's rows."""
    rng = np.random.default_rng(seed)
    rows = []
    for e in range(len(offsets) - 1):
        o0, o1 = int(offsets[e]), int(offsets[e + 1])
        for b in range(o0, o1, block):
            hi = min(b + block, o1)
            rows += [b, hi - 1, int(rng.integers(b, hi))]
    return np.unique(np.asarray(rows, dtype=np.int64))


def _rows(t: torch.Tensor, idx: np.ndarray) -> np.ndarray:
    """Rows idx of a device bf16 tensor as bf16 bit patterns."""
    if len(idx) == 0:
        return np.zeros((0,) + tuple(t.shape[1:]), np.uint16)
    return bf16_bits(t.index_select(0, torch.from_numpy(np.asarray(idx, np.int64)).to(t.device)))


def _max_rel_excess(g_bits, r_bits, bar):
    """max over elements of |g - r| / (a + b |r|): <= 1 inside the bar."""
    g, r = bits_to_f64(g_bits), bits_to_f64(r_bits)
    if g.size == 0:
        return 0.0
    return float(np.max(np.abs(g - r) / (bar[0] + bar[1] * np.abs(r))))


def check_routing(moe, ws, L, wl, inp, label):
    """Routing, dispatch and x_perm of every token; logits of every token against the oracle."""
    T, d, E, k = wl.T, wl.d, wl.E, wl.k
    v = lambda n, s, dt: moe.workspace_view(ws, L, n, s, dt).cpu()
    g_logits = v("logits", (T, E), torch.float32).numpy()
    g_idx = v("idx", (T, k), torch.int32).numpy()
    g_w = v("w", (T, k), torch.float32).numpy()
    bias = inp.bias()
    # routing from the GPU's logits, every token
    idx_o, w_o = oracle.route(g_logits, k, bias)
    assert np.array_equal(g_idx, idx_o)
    np.testing.assert_allclose(g_w, w_o, rtol=1e-5, atol=1e-7)
    C = oracle.capacity(T, E, k, wl.capacity_factor, wl.cap_mode)
    r = oracle.dispatch(g_idx, E, C)
    for n in ("counts_raw", "counts"):
        assert np.array_equal(v(n, (E,), torch.int32).numpy(), r[n]), n
    assert np.array_equal(v("offsets", (E + 1,), torch.int32).numpy(), r["offsets"])
    assert np.array_equal(v("dest", (T, k), torch.int32).numpy(), r["dest"])
    N = r["N"]
    assert np.array_equal(v("src_token", (T * k,), torch.int32).numpy()[:N], r["src_token"])
    # logits of every token against the oracle's double sums
    x = inp.x()
    ref_logits = oracle.router_logits(x, inp.wg())
    err = np.abs(g_logits.astype(np.float64) - ref_logits.astype(np.float64))
    print(f"{label}: max |logit - oracle| = {err.max():.3e} over {T} x {E}")
    assert err.max() <= LOGITS_ATOL, f"{label}: logits off by {err.max():.3e} (bar {LOGITS_ATOL})"
    # the oracle's own routing on every token with a clear k-th key
    own_idx, _ = oracle.route(ref_logits, k, bias)
    keys = np.sort(ref_logits.astype(np.float64) + (bias if bias is not None else 0), axis=1)[:, ::-1]
    clear = (keys[:, k - 1] - keys[:, k]) >= 1e-5 if k < E else np.ones(T, bool)
    assert np.array_equal(own_idx[clear], g_idx[clear])
    print(f"{label}: {int((~clear).sum())} near-tie tokens excluded from the own-routing check")
    return x, g_idx, r, w_o


def check_x_perm(moe, ws, L, wl, x, r):
    xp = moe.workspace_view(ws, L, "x_perm", (wl.T * wl.k, wl.d), torch.bfloat16)[: r["N"]]
    assert np.array_equal(bf16_bits(xp), oracle.gather(x, r["dest"], r["N"]))


def check_experts_and_out(moe, ws, L, wl, x, toks, g_idx, dest, w_o, out, expert, shared, label, own=None):
    """h, y_perm (and y_shared) of every assignment of the tokens `toks`, and their outputs.

    expert(e, xe, g_h) -> (h_ref, y_ref) of expert e on rows xe; g_h is the GPU's h of those rows
    (used by the fp8-activation oracle for its second GEMM).  shared(xs, g_h) likewise.
    own: optional (expert_own(e, xe) -> y, shared_own(xs) -> y), an oracle that does not take the
    GPU's h; the outputs it gives are reported against the bar (printed, not asserted)."""
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    toks = np.asarray(sorted(toks), dtype=np.int64)
    S = len(toks)
    tt = np.repeat(toks, k)
    jj = np.tile(np.arange(k), S)
    dd = dest[tt, jj]
    keep = dd >= 0
    tt, jj, dd = tt[keep], jj[keep], dd[keep].astype(np.int64)
    ee = g_idx[tt, jj]
    h_dev = moe.workspace_view(ws, L, "h", (T * k, f), torch.bfloat16)
    y_dev = moe.workspace_view(ws, L, "y_perm", (T * k, d), torch.bfloat16)
    y_ref = np.zeros((len(tt), d), np.uint16)
    y_own = np.zeros((len(tt), d), np.uint16) if own else None
    worst_h = worst_y = 0.0
    for e in np.unique(ee):
        sel = np.nonzero(ee == e)[0]
        g_h = _rows(h_dev, dd[sel])
        h_ref, ye = expert(int(e), x[tt[sel]], g_h)
        worst_h = max(worst_h, _max_rel_excess(g_h, h_ref, H_BAR))
        worst_y = max(worst_y, _max_rel_excess(_rows(y_dev, dd[sel]), ye, OUT_BAR))
        y_ref[sel] = ye
        if own:
            y_own[sel] = own[0](int(e), x[tt[sel]])
    assert worst_h <= 1.0, f"{label}: h outside its bar (worst |d| / bar = {worst_h:.3f})"
    assert worst_y <= 1.0, f"{label}: y_perm outside its bar (worst |d| / bar = {worst_y:.3f})"
    ysh = None
    if fs:
        hs_dev = moe.workspace_view(ws, L, "h_shared", (T, fs), torch.bfloat16)
        g_hs = _rows(hs_dev, toks)
        hs_ref, ysh = shared(x[toks], g_hs)
        assert _max_rel_excess(g_hs, hs_ref, H_BAR) <= 1.0, f"{label}: shared h"
        ys_dev = moe.workspace_view(ws, L, "y_shared", (T, d), torch.bfloat16)
        assert _max_rel_excess(_rows(ys_dev, toks), ysh, OUT_BAR) <= 1.0, f"{label}: y_shared"
    mini_dest = np.full((S, k), -1, np.int32)
    mini_dest[np.searchsorted(toks, tt), jj] = np.arange(len(tt), dtype=np.int32)
    ref_out = oracle.combine(y_ref, mini_dest, w_o[toks], ysh)
    got = _rows(out, toks)
    assert_layer_close(got, ref_out, f"{label} outputs")
    g64, r64 = bits_to_f64(got), bits_to_f64(ref_out)
    rel_rms = float(np.sqrt(np.mean((g64 - r64) ** 2) / max(np.mean(r64 ** 2), 1e-30)))
    print(f"{label}: {S} tokens ({len(tt)} expert rows) checked; max |out - oracle| = {np.abs(g64 - r64).max():.3e}, "
          f"worst |d|/bar: out {_max_rel_excess(got, ref_out, OUT_BAR):.3f}, y_perm {worst_y:.3f}, h {worst_h:.3f}; "
          f"relative rms {rel_rms:.2e}")
    assert rel_rms < 5e-3                                                  # no systematic drift
    if own:      # the oracle with its own h throughout: how many outputs leave the bar
        ref_own = oracle.combine(y_own, mini_dest, w_o[toks], own[1](x[toks]) if fs else None)
        o64 = bits_to_f64(ref_own)
        bad = np.abs(g64 - o64) > OUT_BAR[0] + OUT_BAR[1] * np.abs(o64)
        print(f"{label}: against the oracle with its own h: {int(bad.sum())} of {bad.size} outputs outside the "
              f"bar, max |d| = {np.abs(g64 - o64).max():.3e}")


def token_set(wl, r, mode, seed, block=128, min_tokens=512):
    """"all": every token; "cover": the tokens of covering_rows (first, last and one seeded row of
    every `block`-row block of every expert), padded with seeded tokens to min_tokens;
    "sample:N": N seeded tokens including the first and the last."""
    if mode == "all":
        return np.arange(wl.T)
    rng = np.random.default_rng(seed + 1)
    if mode.startswith("sample:"):
        n = int(mode.split(":")[1])
        return np.union1d([0, wl.T - 1], rng.choice(wl.T, n - 2, replace=False))
    rows = covering_rows(r["offsets"], seed, block)
    toks = np.unique(r["src_token"][rows])
    if len(toks) < min_tokens:                      # seeded extra tokens
        extra = rng.choice(np.setdiff1d(np.arange(wl.T), toks), min_tokens - len(toks), replace=False)
        toks = np.union1d(toks, extra)
    return toks


def bf16_expert(inp, wl):
    def expert(e, xe, g_h):
        return oracle.expert_ffn(xe, inp.expert_rows("w1", e, 1).reshape(wl.f, wl.d),
                                 inp.expert_rows("w3", e, 1).reshape(wl.f, wl.d),
                                 inp.expert_rows("w2", e, 1).reshape(wl.d, wl.f))

    def shared(xs, g_h):
        return oracle.expert_ffn(xs, inp.shared("w1s"), inp.shared("w3s"), inp.shared("w2s"))
    return expert, shared


def q8_weights(host, e):
    """Expert e's fp8 codes and row scales (the same arrays the GPU was given)."""
    return ((host["w1q"][e], host["s1"][e]), (host["w3q"][e], host["s3"][e]), (host["w2q"][e], host["s2"][e]))


def q8_shared(host):
    return [(host["w1sq"], host["s1s"]), (host["w3sq"], host["s3s"]), (host["w2sq"], host["s2s"])]


@pytest.fixture(scope="module")
def dsv3_q8():
    """The DeepSeek-V3-like layer's fp8 weights, quantised once for both fp8 decode tests: device
    tensors for the layer and the same codes on the host for the oracle."""
    wl = synth.WORKLOADS["dsv3"]
    host = {}
    W = synth.device_tensors(wl, "cuda", names=["x", "wg", "bias"])
    Q = synth.device_tensors_q8(wl, "cuda", host=host)
    yield wl, W, Q, host
    del W, Q
    gc.collect()
    torch.cuda.empty_cache()


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
    del W
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    inp = synth.Inputs(wl)
    x, g_idx, r, w_o = check_routing(moe, ws, L, wl, inp, name)
    check_x_perm(moe, ws, L, wl, x, r)
    toks = token_set(wl, r, FULL[name], seed=7)
    expert, shared = bf16_expert(inp, wl)
    check_experts_and_out(moe, ws, L, wl, x, toks, g_idx, r["dest"], w_o, out, expert, shared, name)

    if name == "skew":
        C = oracle.capacity(T, E, k, wl.capacity_factor, wl.cap_mode)
        assert C == 1280 and r["counts"].max() <= C
        drop = 1.0 - r["N"] / (T * k)
        assert 0.4 < drop < 0.65
        p = r["counts_raw"] / r["counts_raw"].sum()
        assert np.abs(p - inp.zipf_target()).sum() < 0.1
    del ws, out
    gc.collect()
    torch.cuda.empty_cache()


def test_full_size_decode_fp8_weights(moe, dsv3_q8):
    """The DeepSeek-V3-like decode layer with fp8 e4m3 expert weights (bench.py --weights fp8):
    routing bit-exact for every token; h, y_perm, the shared expert and the outputs of 32 seeded
    tokens against the oracle's fp8 experts on the same codes."""
    wl, W, Q, host = dsv3_q8
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_w8(W["x"], W["wg"], W["bias"], Q["w1q"], Q["s1"], Q["w3q"], Q["s3"], Q["w2q"], Q["s2"],
                             Q["w1sq"], Q["s1s"], Q["w3sq"], Q["s3s"], Q["w2sq"], Q["s2s"], fs, T, d, E, k, f,
                             wl.capacity_factor, wl.cap_mode, out, ws)
    assert moe.moe_get_error() == 0
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    inp = synth.Inputs(wl)
    x, g_idx, r, w_o = check_routing(moe, ws, L, wl, inp, "dsv3 fp8 weights")

    def expert(e, xe, g_h):
        (q1, s1), (q3, s3), (q2, s2) = q8_weights(host, e)
        return oracle.expert_ffn_q8(xe, q1, s1, q3, s3, q2, s2)

    qs = q8_shared(host)

    def shared(xs, g_h):
        return oracle.expert_ffn_q8(xs, qs[0][0], qs[0][1], qs[1][0], qs[1][1], qs[2][0], qs[2][1])

    check_experts_and_out(moe, ws, L, wl, x, token_set(wl, r, "sample:32", seed=11), g_idx, r["dest"], w_o, out,
                          expert, shared, "dsv3 fp8 weights")


def _run_w8a8(moe, wl, W, Q, host, mode, own):
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    ws = torch.empty(moe.moe_workspace_bytes_a8(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_w8a8(W["x"], W["wg"], W.get("bias"), Q["w1q"], Q["s1"], Q["w3q"], Q["s3"], Q["w2q"],
                               Q["s2"], Q.get("w1sq"), Q.get("s1s"), Q.get("w3sq"), Q.get("s3s"), Q.get("w2sq"),
                               Q.get("s2s"), fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, out, ws)
    assert moe.moe_get_error() == 0
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    inp = synth.Inputs(wl)
    label = f"{wl.name} fp8 x fp8"
    x, g_idx, r, w_o = check_routing(moe, ws, L, wl, inp, label)

    def expert(e, xe, g_h):
        (q1, s1), (q3, s3), (q2, s2) = q8_weights(host, e)
        return oracle.expert_gate_up_w8a8(xe, q1, s1, q3, s3), oracle.expert_down_w8a8(g_h, q2, s2)

    qs = q8_shared(host) if fs else None

    def shared(xs, g_h):
        h = oracle.expert_gate_up_w8a8(xs, qs[0][0], qs[0][1], qs[1][0], qs[1][1])
        return h, oracle.expert_down_w8a8(g_h, qs[2][0], qs[2][1])

    def expert_own(e, xe):
        (q1, s1), (q3, s3), (q2, s2) = q8_weights(host, e)
        return oracle.expert_ffn_w8a8(xe, q1, s1, q3, s3, q2, s2)[1]

    def shared_own(xs):
        return oracle.expert_ffn_w8a8(xs, qs[0][0], qs[0][1], qs[1][0], qs[1][1], qs[2][0], qs[2][1])[1]

    check_experts_and_out(moe, ws, L, wl, x, mode(r), g_idx, r["dest"], w_o, out, expert, shared, label,
                          own=(expert_own, shared_own) if own else None)


def test_full_size_fp8_weights_and_activations_decode(moe, dsv3_q8):
    """bench.py --weights fp8a8 on the DeepSeek-V3-like decode layer (1-SM tiles): routing bit-exact
    for every token; h against the oracle's fp8 x fp8 first GEMM; the oracle's second GEMM is given
    the kernel's h, so both sides quantise the same h rows (the quantised codes are a decision
    taken on h, like the routing on the logits); 24 seeded tokens.  Also reported: the outputs
    against the oracle that quantises its own h."""
    wl, W, Q, host = dsv3_q8
    _run_w8a8(moe, wl, W, Q, host, lambda r: token_set(wl, r, "sample:24", seed=13), own=True)


def test_full_size_fp8_weights_and_activations_prefill(moe):
    """The same on the Mixtral-like prefill layer (2-SM tiles, swapped tail tiles): the tokens of
    the first, last and one seeded row of every 256-row tile of every expert."""
    wl = synth.WORKLOADS["mixtral"]
    host = {}
    W = synth.device_tensors(wl, "cuda", names=["x", "wg", "bias"])
    Q = synth.device_tensors_q8(wl, "cuda", host=host)
    _run_w8a8(moe, wl, W, Q, host, lambda r: token_set(wl, r, "cover", seed=13, block=256, min_tokens=0), own=False)
    del W, Q
    gc.collect()
    torch.cuda.empty_cache()
