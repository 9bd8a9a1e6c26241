"""Pins for the CPU oracle (no GPU).

Each test ties an oracle function to something other than the oracle itself:
brute force on tiny inputs, the pages' own sort-by-expert example, closed
forms, invariants, and special cases that reduce to textbook routines computed
with torch / scipy on the CPU.  A plausible slip in the oracle (a dropped
term, a wrong sign or index, a transposed operand, an unstable order, a wrong
rounding) fails at least one of them.

Pages cited (titles):
  "MoE 推理中的 Expert Parallel、KV Cache 与大规模专家并行架构解析" (§1, §2, §7, §8)
  "MoE 推理架构深度实战：从 Expert Parallelism 到 DeepSeek-V3 的工程落地" (§2.1 router code, §3.1)
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
RNG = np.random.default_rng(1234)


# --------------------------------------------------------------------------- helpers (test side)

def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float -> bf16 bit patterns via torch (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rand_bf16(shape, std=1.0):
    return bf16_bits((RNG.standard_normal(shape) * std).astype(np.float32))


def ulp_diff_bf16(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two bf16 bit arrays (same-sign finite values)."""
    def key(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x & 0x7FFF)
    return np.abs(key(a) - key(b))


def torch_bf16_round_f64(v: torch.Tensor) -> torch.Tensor:
    return v.to(torch.float32).to(torch.bfloat16)


# --------------------------------------------------------------------------- bf16 rounding

def test_bf16_round_closed_forms():
    # exact ties round to the even mantissa
    assert oracle.bf16_round(1.0 + 2.0 ** -8) == 0x3F80          # tie between 1 and 1+2^-7 -> 1
    assert oracle.bf16_round(1.0 + 3 * 2.0 ** -8) == 0x3F82      # tie -> 1+2^-6 (even)
    assert oracle.bf16_round(-(1.0 + 2.0 ** -8)) == 0xBF80
    # one rounding from double: just above a tie rounds up (an fp32 detour would round to even)
    assert oracle.bf16_round(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert oracle.bf16_round(0.0) == 0x0000
    assert oracle.bf16_round(-2.5) == 0xC020
    assert oracle.bf16_round(3.0e38) == 0x7F62


def test_bf16_round_matches_torch_on_fp32_values():
    v = (RNG.standard_normal(4000) * np.exp(RNG.uniform(-20, 20, 4000))).astype(np.float32)
    ours = np.array([oracle.bf16_round(float(x)) for x in v], dtype=np.uint16)
    assert np.array_equal(ours, bf16_bits(v))


# --------------------------------------------------------------------------- router logits

def test_router_logits_vs_torch_matmul():
    T, d, E = 37, 192, 13
    x, wg = rand_bf16((T, d)), rand_bf16((E, d), 1 / math.sqrt(d))
    ours = oracle.router_logits(x, wg)
    ref = (torch.from_numpy(bf16_to_f64(x)) @ torch.from_numpy(bf16_to_f64(wg)).T).to(torch.float32).numpy()
    # both sum exact bf16 products in double; only the order differs -> at most 1 fp32 ulp
    assert np.all(np.abs(ours - ref) <= np.spacing(np.abs(ref)))
    assert np.mean(ours == ref) > 0.99


# --------------------------------------------------------------------------- routing

def brute_topk(keys: np.ndarray, k: int) -> np.ndarray:
    """k rounds of argmax, removing the winner; np.argmax breaks ties to the lowest index."""
    T = keys.shape[0]
    out = np.empty((T, k), np.int32)
    for t in range(T):
        kk = keys[t].astype(np.float64).copy()
        for j in range(k):
            e = int(np.argmax(kk))
            out[t, j] = e
            kk[e] = -np.inf
    return out


@pytest.mark.parametrize("E,k", [(8, 1), (8, 2), (13, 4), (64, 2), (256, 8), (5, 5)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_route_vs_bruteforce(E, k, with_bias):
    T = 150
    logits = RNG.standard_normal((T, E)).astype(np.float32)
    bias = RNG.uniform(-0.1, 0.1, E).astype(np.float32) if with_bias else None
    idx, w = oracle.route(logits, k, bias)
    keys = logits + (bias if bias is not None else np.float32(0))      # fp32 add
    assert np.array_equal(idx, brute_topk(keys, k))
    # weights: softmax over the chosen subset of the UNBIASED logits (equal to the
    # renormalised full softmax by shift/scale invariance)
    for t in range(T):
        ref = scipy.special.softmax(logits[t, idx[t]].astype(np.float64))
        np.testing.assert_allclose(w[t], ref, rtol=2e-7, atol=1e-9)
    np.testing.assert_allclose(w.astype(np.float64).sum(1), 1.0, atol=1e-6)


def test_route_ties_break_to_lower_expert():
    T, E, k = 300, 16, 4
    logits = RNG.integers(-3, 3, (T, E)).astype(np.float32)     # many exact ties
    logits[0, :] = 0.0                                          # all tied
    logits[1, :] = -0.0
    logits[1, 5] = 0.0                                          # -0 == +0
    idx, w = oracle.route(logits, k)
    assert np.array_equal(idx, brute_topk(logits, k))
    assert list(idx[0]) == [0, 1, 2, 3]
    assert list(idx[1]) == [0, 1, 2, 3]
    np.testing.assert_allclose(w[0], 0.25, rtol=1e-7)


def test_route_k1_is_argmax_with_unit_weight():
    logits = RNG.standard_normal((500, 32)).astype(np.float32)
    idx, w = oracle.route(logits, 1)
    assert np.array_equal(idx[:, 0], np.argmax(logits, axis=1))
    assert np.all(w == 1.0)


def test_route_k_equals_E_gives_full_softmax():
    logits = (RNG.standard_normal((64, 12)) * 3).astype(np.float32)
    idx, w = oracle.route(logits, 12)
    p = scipy.special.softmax(logits.astype(np.float64), axis=1)
    for t in range(64):
        assert np.all(np.diff(logits[t, idx[t]]) <= 0)         # descending
        np.testing.assert_allclose(w[t], p[t, idx[t]], rtol=2e-7)


def test_route_bias_selects_but_does_not_weight():
    T, E, k = 50, 32, 3
    logits = RNG.standard_normal((T, E)).astype(np.float32)
    forced = [4, 9, 30]
    bias = np.zeros(E, np.float32)
    bias[forced] = 100.0
    idx, w = oracle.route(logits, k, bias)
    for t in range(T):
        assert sorted(idx[t]) == forced
        ref = scipy.special.softmax(logits[t, idx[t]].astype(np.float64))
        np.testing.assert_allclose(w[t], ref, rtol=2e-7)


def test_route_shift_invariance():
    logits = RNG.standard_normal((80, 24)).astype(np.float32)
    i1, w1 = oracle.route(logits, 3)
    i2, w2 = oracle.route(logits + np.float32(8.0), 3)
    assert np.array_equal(i1, i2)
    np.testing.assert_allclose(w1, w2, rtol=3e-6)


def test_route_rejects_nonfinite():
    logits = np.zeros((4, 8), np.float32)
    logits[2, 3] = np.inf
    with pytest.raises(ValueError):
        oracle.route(logits, 2)


# --------------------------------------------------------------------------- capacity

def test_capacity_values():
    # router formula int(num_tokens / num_experts * factor), Python int() truncation
    for T, E, k, cf in [(4096, 8, 2, 1.25), (4096, 8, 2, 2.0), (1000, 7, 3, 1.1), (1, 64, 2, 1.25),
                        (16384, 128, 8, 1.0), (999, 10, 1, 0.3)]:
        assert oracle.capacity(T, E, k, cf, oracle.CAP_PER_TOKEN) == int(T / E * cf)
        assert oracle.capacity(T, E, k, cf, oracle.CAP_PER_ASSIGNMENT) == int(T * k / E * cf)
    assert oracle.capacity(32768, 64, 2, 1.25, oracle.CAP_PER_ASSIGNMENT) == 1280
    assert oracle.capacity(32768, 64, 2, 1.25, oracle.CAP_PER_TOKEN) == 640
    assert oracle.capacity(4096, 8, 2, 2.0, oracle.CAP_PER_TOKEN) == 1024      # eval factor 2.0
    assert oracle.capacity(10, 3, 1, 0.9, oracle.CAP_PER_TOKEN) == 3            # 3.0000000000000004 -> 3
    assert oracle.capacity(10, 3, 1, 1.0, oracle.CAP_NONE) == -1


# --------------------------------------------------------------------------- dispatch

def random_idx(T, E, k):
    return np.stack([RNG.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)


def brute_dispatch(idx, E, C):
    """Per expert: the ascending list of tokens routed to it; keep its first C."""
    T, k = idx.shape
    lists = [[t for t in range(T) if e in idx[t]] for e in range(E)]
    kept = [l if C < 0 else l[:C] for l in lists]
    offsets = np.concatenate([[0], np.cumsum([len(l) for l in kept])]).astype(np.int32)
    dest = np.full((T, k), -1, np.int32)
    src = np.empty(offsets[-1], np.int32)
    for e in range(E):
        for pos, t in enumerate(kept[e]):
            j = int(np.where(idx[t] == e)[0][0])
            dest[t, j] = offsets[e] + pos
            src[offsets[e] + pos] = t
    return [len(l) for l in lists], [len(l) for l in kept], offsets, dest, src


@pytest.mark.parametrize("T,E,k,C", [(200, 8, 2, -1), (200, 8, 2, 30), (333, 16, 4, 50), (64, 8, 8, 5),
                                     (100, 4, 1, 0), (257, 32, 3, 1000), (1, 8, 2, -1)])
def test_dispatch_vs_bruteforce(T, E, k, C):
    idx = random_idx(T, E, k)
    r = oracle.dispatch(idx, E, C)
    craw, cnt, off, dest, src = brute_dispatch(idx, E, C)
    assert np.array_equal(r["counts_raw"], craw)
    assert np.array_equal(r["counts"], cnt)
    assert np.array_equal(r["offsets"], off)
    assert np.array_equal(r["dest"], dest)
    assert np.array_equal(r["src_token"], src)
    # invariants
    assert r["counts_raw"].sum() == T * k
    assert np.array_equal(r["counts_raw"], np.bincount(idx.ravel(), minlength=E))
    drops = int((r["dest"] < 0).sum())
    assert r["counts"].sum() == T * k - drops == r["N"]
    if C >= 0:
        assert np.array_equal(r["counts"], np.minimum(r["counts_raw"], C))
    else:
        assert drops == 0
    assert np.all(np.diff(r["offsets"]) >= 0)
    kept = r["dest"] >= 0
    tt = np.repeat(np.arange(T)[:, None], k, 1)
    assert np.array_equal(r["src_token"][r["dest"][kept]], tt[kept])


def test_dispatch_zero_capacity_drops_everything():
    idx = random_idx(40, 8, 2)
    r = oracle.dispatch(idx, 8, 0)
    assert r["N"] == 0 and np.all(r["dest"] == -1) and np.all(r["offsets"] == 0)


def test_permutation_matches_pages_example():
    rows = [l.split() for l in open(os.path.join(HERE, "golden", "permutation_example.txt"))
            if l.strip() and not l.startswith("#")]
    experts, sorted_ids, src_expected = ([int(v) for v in r] for r in rows)
    idx = np.array(experts, np.int32)[:, None]
    r = oracle.dispatch(idx, 8, -1)
    assert list(r["src_token"]) == src_expected
    assert [experts[t] for t in r["src_token"]] == sorted_ids


# --------------------------------------------------------------------------- permute / combine

def test_unpermute_identity_k1():
    T, d, E = 90, 64, 8
    x = rand_bf16((T, d))
    idx = random_idx(T, E, 1)
    r = oracle.dispatch(idx, E, -1)
    xp = oracle.gather(x, r["dest"], r["N"])
    out = oracle.combine(xp, r["dest"], np.ones((T, 1), np.float32))
    assert np.array_equal(out, x)


def test_unpermute_identity_k4_weights_sum_to_one():
    T, d, E, k = 70, 32, 16, 4
    x = rand_bf16((T, d))
    logits = RNG.standard_normal((T, E)).astype(np.float32)
    idx, w = oracle.route(logits, k)
    r = oracle.dispatch(idx, E, -1)
    xp = oracle.gather(x, r["dest"], r["N"])
    out = oracle.combine(xp, r["dest"], w)
    assert np.array_equal(out, x)


def test_combine_dropped_slots_contribute_zero_and_shared_added():
    T, d, k = 3, 8, 2
    y = bf16_bits(np.arange(4 * d, dtype=np.float32).reshape(4, d) / 8)
    dest = np.array([[0, -1], [-1, -1], [2, 3]], np.int32)
    w = np.array([[0.75, 0.25], [0.5, 0.5], [0.5, 0.5]], np.float32)
    ysh = bf16_bits(np.full((T, d), 0.5, np.float32))
    out = bf16_to_f64(oracle.combine(y, dest, w, ysh))
    yf = bf16_to_f64(y)
    np.testing.assert_array_equal(out[0], 0.75 * yf[0] + 0.5)
    np.testing.assert_array_equal(out[1], 0.5)
    np.testing.assert_allclose(out[2], bf16_to_f64(bf16_bits((0.5 * yf[2] + 0.5 * yf[3] + 0.5).astype(np.float32))))


# --------------------------------------------------------------------------- experts

def textbook_swiglu(x, W1, W3, W2):
    """torch float64 dense SwiGLU FFN, W2 (silu(W1 x) * (W3 x)), with bf16 stores of h and y."""
    X = torch.from_numpy(bf16_to_f64(x))
    g = X @ torch.from_numpy(bf16_to_f64(W1)).T
    u = X @ torch.from_numpy(bf16_to_f64(W3)).T
    h = torch_bf16_round_f64(torch.nn.functional.silu(g) * u)
    y = torch_bf16_round_f64(h.to(torch.float64) @ torch.from_numpy(bf16_to_f64(W2)).T)
    to_bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    return to_bits(h), to_bits(y)


def test_expert_ffn_vs_textbook():
    rows, d, f = 24, 96, 160
    x = rand_bf16((rows, d))
    W1, W3 = rand_bf16((f, d), d ** -0.5), rand_bf16((f, d), d ** -0.5)
    W2 = rand_bf16((d, f), f ** -0.5)
    h, y = oracle.expert_ffn(x, W1, W3, W2)
    h_ref, y_ref = textbook_swiglu(x, W1, W3, W2)
    # only summation order (and torch's fp32 detour when rounding) differ: <= 1 bf16 ulp, nearly all exact
    assert ulp_diff_bf16(h, h_ref).max() <= 1 and np.mean(h == h_ref) > 0.99
    assert ulp_diff_bf16(y, y_ref).max() <= 1 and np.mean(y == y_ref) > 0.97


def test_layer_single_expert_is_dense_swiglu():
    T, d, f = 40, 64, 128
    x = rand_bf16((T, d))
    wg = rand_bf16((1, d), d ** -0.5)
    W1, W3 = rand_bf16((1, f, d), d ** -0.5), rand_bf16((1, f, d), d ** -0.5)
    W2 = rand_bf16((1, d, f), f ** -0.5)
    r = oracle.layer_forward(x, wg, W1, W3, W2, k=1)
    _, y_ref = textbook_swiglu(x, W1[0], W3[0], W2[0])
    assert np.all(r["w"] == 1.0) and np.all(r["idx"] == 0)
    assert ulp_diff_bf16(r["out"], y_ref).max() <= 1 and np.mean(r["out"] == y_ref) > 0.97


def test_layer_equals_dense_weighted_sum_over_all_experts():
    T, d, E, k, f = 48, 64, 8, 2, 96
    x = rand_bf16((T, d))
    wg = rand_bf16((E, d), d ** -0.5)
    W1, W3 = rand_bf16((E, f, d), d ** -0.5), rand_bf16((E, f, d), d ** -0.5)
    W2 = rand_bf16((E, d, f), f ** -0.5)
    r = oracle.layer_forward(x, wg, W1, W3, W2, k=k)
    # every expert on every token (textbook), gates zero off the selected set
    G = np.zeros((T, E))
    for t in range(T):
        G[t, r["idx"][t]] = r["w"][t]
    acc = np.zeros((T, d))
    for e in range(E):
        _, ye = textbook_swiglu(x, W1[e], W3[e], W2[e])
        acc += G[:, e:e + 1] * bf16_to_f64(ye)
    ref = bf16_bits(acc.astype(np.float32))
    assert ulp_diff_bf16(r["out"], ref).max() <= 2 and np.mean(r["out"] == ref) > 0.95


def test_shared_expert_alone_when_routed_outputs_vanish():
    T, d, E, k, f, fs = 32, 64, 4, 2, 64, 128
    x = rand_bf16((T, d))
    wg = rand_bf16((E, d), d ** -0.5)
    W1, W3 = rand_bf16((E, f, d), d ** -0.5), rand_bf16((E, f, d), d ** -0.5)
    W2 = np.zeros((E, d, f), np.uint16)                                    # routed experts output 0
    W1s, W3s, W2s = rand_bf16((fs, d), d ** -0.5), rand_bf16((fs, d), d ** -0.5), rand_bf16((d, fs), fs ** -0.5)
    r = oracle.layer_forward(x, wg, W1, W3, W2, k=k, W1s=W1s, W3s=W3s, W2s=W2s)
    _, ysh = textbook_swiglu(x, W1s, W3s, W2s)
    assert ulp_diff_bf16(r["out"], ysh).max() <= 1
    assert np.array_equal(r["out"], r["y_shared"])


def test_layer_zero_capacity_outputs_zero():
    T, d, E, k, f = 16, 32, 4, 2, 64
    x = rand_bf16((T, d))
    wg = rand_bf16((E, d), d ** -0.5)
    W1, W3, W2 = rand_bf16((E, f, d)), rand_bf16((E, f, d)), rand_bf16((E, d, f))
    r = oracle.layer_forward(x, wg, W1, W3, W2, k=k, C=0)
    assert r["N"] == 0 and np.all(bf16_to_f64(r["out"]) == 0)


def test_layer_routes_supplied_logits():
    T, d, E, k, f = 20, 32, 8, 2, 64
    x = rand_bf16((T, d))
    wg = rand_bf16((E, d), d ** -0.5)
    W1, W3, W2 = rand_bf16((E, f, d)), rand_bf16((E, f, d)), rand_bf16((E, d, f))
    logits = RNG.standard_normal((T, E)).astype(np.float32)
    r = oracle.layer_forward(x, wg, W1, W3, W2, k=k, logits_in=logits)
    i2, _ = oracle.route(logits, k)
    assert np.array_equal(r["idx"], i2) and np.array_equal(r["logits"], logits)


# --------------------------------------------------------------------------- overflow bias update

def test_update_bias_closed_forms():
    C = 200
    counts = np.array([0, 100, 200, 300, 400, 1000, 50], np.int32)
    b = oracle.update_bias(counts, C)
    assert list(b) == [1.0, 0.5, 0.0, -0.5, -1.0, -1.0, 0.75]      # -clamp((c - C) / C, -1, 1)
    assert np.signbit(b[2])                                          # -(+0) in fp32
    with pytest.raises(ValueError):
        oracle.update_bias(counts, 0)


def test_update_bias_steers_load_away_from_overloaded_experts():
    # route a batch, derive the bias from its overflow, route the next batch with it:
    # the expert that overflowed most loses assignments, the idlest one gains
    T, E, k = 4000, 16, 2
    skew = np.linspace(1.0, -1.0, E).astype(np.float32)             # expert 0 popular, 15 idle
    l1 = (RNG.standard_normal((T, E)) * 0.5 + skew).astype(np.float32)
    l2 = (RNG.standard_normal((T, E)) * 0.5 + skew).astype(np.float32)
    C = oracle.capacity(T, E, k, 2.0, oracle.CAP_PER_TOKEN)         # eval capacity factor 2.0
    i1, _ = oracle.route(l1, k)
    c1 = oracle.dispatch(i1, E, C)["counts_raw"]
    bias = oracle.update_bias(c1, C)
    i2, _ = oracle.route(l2, k, bias)
    c2 = oracle.dispatch(i2, E, C)["counts_raw"]
    i2n, _ = oracle.route(l2, k)
    c2n = oracle.dispatch(i2n, E, C)["counts_raw"]
    assert c1[0] > C and bias[0] < 0 and bias[-1] > 0
    assert c2[0] < c2n[0] and c2[-1] > c2n[-1]


# --------------------------------------------------------------------------- fp8 e4m3 expert weights

def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([oracle.e4m3(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2          # 0x7F, 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])
    assert oracle.e4m3(0x7E) == 448.0 and oracle.e4m3(0x01) == 2.0 ** -9 and oracle.e4m3(0x38) == 1.0


def test_q8_expert_equals_bf16_expert_on_representable_weights():
    # scales that are powers of two make e4m3(q) * s exactly a bf16 value: the fp8 expert must
    # then equal the (pinned) bf16 expert bit for bit
    rows, d, f = 12, 64, 96
    x = rand_bf16((rows, d))
    q = lambda shape: RNG.integers(0, 256, shape).astype(np.uint8)
    W1q, W3q, W2q = q((f, d)), q((f, d)), q((d, f))
    for W in (W1q, W3q, W2q):
        W[(W & 0x7F) == 0x7F] = 0x38                                       # no NaN codes
    s1 = (2.0 ** RNG.integers(-12, -6, f)).astype(np.float32)
    s3 = (2.0 ** RNG.integers(-12, -6, f)).astype(np.float32)
    s2 = (2.0 ** RNG.integers(-12, -6, d)).astype(np.float32)
    deq = lambda Wq, s: bf16_bits((torch.from_numpy(Wq).view(torch.float8_e4m3fn).to(torch.float64).numpy()
                                   * s[:, None]).astype(np.float32))
    h_q, y_q = oracle.expert_ffn_q8(x, W1q, s1, W3q, s3, W2q, s2)
    h_b, y_b = oracle.expert_ffn(x, deq(W1q, s1), deq(W3q, s3), deq(W2q, s2))
    assert np.array_equal(h_q, h_b) and np.array_equal(y_q, y_b)


def test_q8_expert_vs_textbook_dequantised():
    rows, d, f = 10, 128, 64
    x = rand_bf16((rows, d))
    w = lambda shape, std: rand_bf16(shape, std)
    import synth
    W1q, s1 = synth.quantize_e4m3_rows(w((f, d), d ** -0.5), d)
    W3q, s3 = synth.quantize_e4m3_rows(w((f, d), d ** -0.5), d)
    W2q, s2 = synth.quantize_e4m3_rows(w((d, f), f ** -0.5), f)
    h, y = oracle.expert_ffn_q8(x, W1q, s1, W3q, s3, W2q, s2)
    deq = lambda Wq, s: torch.from_numpy(Wq).view(torch.float8_e4m3fn).to(torch.float64) * torch.from_numpy(s).double()[:, None]
    X = torch.from_numpy(bf16_to_f64(x))
    g, u = X @ deq(W1q, s1).T, X @ deq(W3q, s3).T
    hh = torch_bf16_round_f64(torch.nn.functional.silu(g) * u)
    yy = torch_bf16_round_f64(hh.double() @ deq(W2q, s2).T)
    to_bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    assert ulp_diff_bf16(h, to_bits(hh)).max() <= 1 and ulp_diff_bf16(y, to_bits(yy)).max() <= 1


# --------------------------------------------------------------------------- fp8 activations


def test_e4m3_encode_matches_torch_rne():
    # every code, every midpoint between neighbouring codes (ties go to the even code), random
    # fp32 values across the range, and saturation beyond 448
    pos = np.array([oracle.e4m3(c) for c in range(0x7F)], np.float64)          # 0 .. 448
    mids = (pos[:-1] + pos[1:]) / 2
    rng = np.random.default_rng(3)
    rand = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(400.0), 4000))
    vals = np.concatenate([pos, mids, rand, [0.0, 2.0 ** -11, 2.0 ** -10, 460.0, 1e6]]).astype(np.float32)
    vals = np.concatenate([vals, -vals])
    ours = np.array([oracle.e4m3_encode(float(v)) for v in vals], np.uint8)
    clipped = np.clip(vals, -448.0, 448.0)               # saturating conversion
    ref = torch.from_numpy(clipped).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    # ties: the midpoint of codes 0x38 (1.0) and 0x39 (1.125) goes to the even code 0x38
    assert oracle.e4m3_encode(1.0625) == 0x38 and oracle.e4m3_encode(1.1875) == 0x3A


def test_quantize_rows_matches_torch_fp32_recipe():
    # rows across magnitudes, one row scaled into the tiny range, and an all-zero row
    x = np.concatenate([rand_bf16((1, 512), std) for std in (1e-6, 1e-3, 1.0, 37.0, 3e4)]
                       + [np.zeros((1, 512), np.uint16)])
    q, s = oracle.quantize_rows_e4m3(x)
    xf = torch.from_numpy((x.astype(np.uint32) << 16).view(np.float32))
    amax = xf.abs().amax(dim=1)
    s_ref = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    assert np.array_equal(s.view(np.uint32), s_ref.numpy().view(np.uint32))
    q_ref = (xf / s_ref[:, None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, q_ref)
    assert (q[-1] == 0).all() and s[-1] == 1.0
    # the largest magnitude of each nonzero row lands on +-448
    for r in range(len(x) - 1):
        assert np.abs(np.array([oracle.e4m3(c) for c in q[r]])).max() == 448.0


def test_w8a8_expert_equals_weight_only_expert_when_activations_are_exact():
    # x rows made of e4m3 values times a power of two, each row reaching 448 * 2^k: quantising them
    # is exact, so the first GEMM (h) must equal the weight-only fp8 expert's h bit for bit
    import synth
    rng = np.random.default_rng(11)
    d, f, rows = 128, 64, 5
    codes = rng.integers(0, 0x7F, size=(rows, d)).astype(np.uint8)
    codes[rng.random((rows, d)) < 0.5] |= 0x80
    codes[:, 0] = 0x7E                                              # amax = 448 in every row
    vals = np.array([[oracle.e4m3(c) for c in row] for row in codes]) * (2.0 ** rng.integers(-8, 4, (rows, 1)))
    x = bf16_bits(vals.astype(np.float32))
    assert np.array_equal((x.astype(np.uint32) << 16).view(np.float32), vals.astype(np.float32))   # exact in bf16
    W1q, s1 = synth.quantize_e4m3_rows(rand_bf16((f, d), d ** -0.5), d)
    W3q, s3 = synth.quantize_e4m3_rows(rand_bf16((f, d), d ** -0.5), d)
    W2q, s2 = synth.quantize_e4m3_rows(rand_bf16((d, f), f ** -0.5), f)
    h_a8, y_a8 = oracle.expert_ffn_w8a8(x, W1q, s1, W3q, s3, W2q, s2)
    h_w8, _ = oracle.expert_ffn_q8(x, W1q, s1, W3q, s3, W2q, s2)
    assert np.array_equal(h_a8, h_w8)
    # the second GEMM: dequantise h with the pinned quantiser and multiply in float64 (torch)
    hq, sh = oracle.quantize_rows_e4m3(h_a8)
    deq = lambda qq: torch.from_numpy(qq).view(torch.float8_e4m3fn).to(torch.float64)
    hd = deq(hq) * torch.from_numpy(sh.astype(np.float64))[:, None]
    Wd = deq(W2q) * torch.from_numpy(s2.astype(np.float64))[:, None]
    y_ref = bf16_bits((hd @ Wd.T).numpy().astype(np.float32))
    assert np.max(ulp_diff_bf16(y_a8, y_ref)) <= 1
    assert np.mean(y_a8 == y_ref) > 0.95
