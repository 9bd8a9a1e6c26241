"""GPU parity of each stage of the CUDA path against the CPU oracle (through the C ABI).

Bars: routing indices, counts, offsets, dest, src_token and x_perm bit-exact given the
same fp32 logits; routing weights rel 1e-5; logits within the fp32-accumulation bound of
_util.logits_tol; h within 1e-3 + 8e-3|ref| (one bf16 ulp plus cancellation floor);
expert outputs and layer outputs within 1e-2 + 2e-2|ref|.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _util import assert_layer_close, bf16_bits, bits_to_f64, logits_tol, to_dev_bf16, ulp_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import moe_layer_router_b200 as m
    assert torch.cuda.is_available()
    return m


def _logits(T, E, tid=100, scale=1.0):
    return (synth.normal_f64(0, tid, 0, T * E) * scale).astype(np.float32).reshape(T, E)


def _bf16(n_rows, n_cols, tid, std=1.0):
    return synth.normal_bf16(0, tid, 0, n_rows * n_cols, std).reshape(n_rows, n_cols)


def _ws(moe, T, d, E, k, f=64, f_shared=0):
    return torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, f_shared), dtype=torch.uint8, device="cuda")


# ----------------------------------------------------------------------------- routing

@pytest.mark.parametrize("T,E,k,with_bias", [(128, 8, 2, False), (1000, 8, 2, False), (777, 128, 8, False),
                                             (256, 256, 8, True), (300, 64, 2, False), (100, 1024, 32, True),
                                             (50, 5, 5, False), (33, 40, 1, True)])
def test_route_on_supplied_logits_bit_exact(moe, T, E, k, with_bias):
    logits = _logits(T, E)
    bias = synth.uniform_f32(0, 101, 0, E, -0.1, 0.1) if with_bias else None
    idx_o, w_o = oracle.route(logits, k, bias)
    lg = torch.from_numpy(logits).cuda()
    b = torch.from_numpy(bias).cuda() if bias is not None else None
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(None, None, b, lg, T, 64, E, k, None, idx, w, None)
    assert moe.moe_get_error() == 0
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    np.testing.assert_allclose(w.cpu().numpy(), w_o, rtol=1e-5, atol=1e-7)


def test_route_ties_break_to_lower_expert(moe):
    T, E, k = 512, 64, 8
    logits = np.round(_logits(T, E, tid=103) * 1.5).astype(np.float32)   # many exact ties
    logits[0] = 0.0
    idx_o, w_o = oracle.route(logits, k)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(None, None, None, torch.from_numpy(logits).cuda(), T, 64, E, k, None, idx, w, None)
    assert moe.moe_get_error() == 0
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert list(idx_o[0]) == list(range(8))
    np.testing.assert_allclose(w.cpu().numpy(), w_o, rtol=1e-5, atol=1e-7)


def test_route_nonfinite_score_sets_check_error(moe):
    T, E, k = 16, 8, 2
    logits = _logits(T, E)
    logits[3, 5] = np.nan
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(None, None, None, torch.from_numpy(logits).cuda(), T, 64, E, k, None, idx, w, None)
    assert moe.moe_get_error() == moe.MOE_ERR_CHECK
    assert moe.moe_get_error() == 0          # cleared by the read


# ----------------------------------------------------------------------------- permutation

@pytest.mark.parametrize("T,d,E,k,C", [(128, 256, 8, 2, -1), (1000, 128, 8, 2, 100), (777, 64, 128, 8, -1),
                                       (777, 64, 128, 8, 40), (2000, 192, 64, 2, 0), (513, 64, 16, 4, 70),
                                       (1, 64, 8, 2, -1), (300, 64, 1024, 32, 5), (4099, 128, 32, 3, 300)])
def test_permute_bit_exact(moe, T, d, E, k, C):
    idx, _ = oracle.route(_logits(T, E, tid=104), k)
    x = _bf16(T, d, 105)
    r = oracle.dispatch(idx, E, C)
    xp = oracle.gather(x, r["dest"], r["N"])
    dev = lambda a: torch.from_numpy(a).cuda()
    craw = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    dest = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    src = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    x_perm = torch.zeros((T * k, d), dtype=torch.bfloat16, device="cuda")
    ws = _ws(moe, T, d, E, k)
    moe.moe_permute(to_dev_bf16(x), dev(idx), T, d, E, k, C, craw, cnt, off, dest, src, x_perm, ws)
    assert moe.moe_get_error() == 0
    N = r["N"]
    assert np.array_equal(craw.cpu().numpy(), r["counts_raw"])
    assert np.array_equal(cnt.cpu().numpy(), r["counts"])
    assert np.array_equal(off.cpu().numpy(), r["offsets"])
    assert np.array_equal(dest.cpu().numpy(), r["dest"])
    assert np.array_equal(src.cpu().numpy()[:N], r["src_token"])
    assert np.array_equal(bf16_bits(x_perm)[:N], xp)


# ----------------------------------------------------------------------------- combine

@pytest.mark.parametrize("with_shared", [False, True])
def test_combine(moe, with_shared):
    T, d, E, k, C = 300, 256, 16, 4, 50
    idx, w = oracle.route(_logits(T, E, tid=106), k)
    r = oracle.dispatch(idx, E, C)
    y_perm = _bf16(T * k, d, 107)
    ysh = _bf16(T, d, 108) if with_shared else None
    ref = oracle.combine(y_perm[: max(r["N"], 1)], r["dest"], w, ysh)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(to_dev_bf16(y_perm), torch.from_numpy(r["dest"]).cuda(), torch.from_numpy(w).cuda(),
                    to_dev_bf16(ysh) if ysh is not None else None, T, d, k, out)
    assert moe.moe_get_error() == 0
    got = bf16_bits(out)
    assert_layer_close(got, ref)
    assert np.mean(ulp_bf16(got, ref) <= 1) > 0.999
    assert (r["dest"] < 0).any()                  # drops exercised


# ----------------------------------------------------------------------------- router GEMM

@pytest.mark.parametrize("T,d,E", [(128, 256, 8), (300, 512, 128), (129, 1024, 256), (200, 256, 300), (64, 7168, 256),
                                   (1000, 4096, 64), (17, 64, 40), (130, 128, 1024)])
def test_router_gemm(moe, T, d, E):
    k = min(2, E)
    x = _bf16(T, d, 109)
    wg = _bf16(E, d, 110, std=d ** -0.5)
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(to_dev_bf16(x), to_dev_bf16(wg), None, None, T, d, E, k, logits, idx, w, _ws(moe, T, d, E, k))
    assert moe.moe_get_error() == 0
    g = logits.cpu().numpy()
    ref = oracle.router_logits(x, wg)
    tol = logits_tol(x, wg)
    assert np.all(np.abs(g.astype(np.float64) - ref) <= tol), float(np.max(np.abs(g - ref) / tol))
    i2, w2 = oracle.route(g, k)
    assert np.array_equal(idx.cpu().numpy(), i2)
    np.testing.assert_allclose(w.cpu().numpy(), w2, rtol=1e-5, atol=1e-7)


# ----------------------------------------------------------------------------- expert FFN

# groups averaging >= 256 rows run on CTA-pair (2-SM) tiles, the others on 1-SM tiles
@pytest.mark.parametrize("counts,d,f", [([0, 1, 127, 128, 129, 300, 5, 0], 256, 512), ([200, 200, 200], 128, 320),
                                        ([1], 64, 64), ([0, 0, 0], 128, 128), ([17, 260, 3, 64], 448, 192),
                                        ([513, 1, 700], 1024, 1536),
                                        ([0, 1, 255, 256, 257, 700, 5, 1000], 256, 512),
                                        ([300, 0, 600], 448, 192), ([2000], 128, 128)])
def test_expert_ffn(moe, counts, d, f):
    E = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    N = int(off[-1])
    max_rows = N + 37
    x_perm = _bf16(max_rows, d, 111)
    W1 = _bf16(E * f, d, 112, d ** -0.5).reshape(E, f, d)
    W3 = _bf16(E * f, d, 113, d ** -0.5).reshape(E, f, d)
    W2 = _bf16(E * d, f, 114, f ** -0.5).reshape(E, d, f)
    h = torch.full((max_rows, f), 7.0, dtype=torch.bfloat16, device="cuda")
    y = torch.full((max_rows, d), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(4096 * 4, dtype=torch.uint8, device="cuda")
    moe.moe_expert_ffn(to_dev_bf16(x_perm), torch.from_numpy(off).cuda(), max_rows, E, d, f, to_dev_bf16(W1),
                       to_dev_bf16(W3), to_dev_bf16(W2), h, y, ws)
    assert moe.moe_get_error() == 0
    hg, yg = bf16_bits(h), bf16_bits(y)
    for e in range(E):
        a, b = off[e], off[e + 1]
        if a == b:
            continue
        ho, yo = oracle.expert_ffn(x_perm[a:b], W1[e], W3[e], W2[e])
        dh = np.abs(bits_to_f64(hg[a:b]) - bits_to_f64(ho))
        assert np.all(dh <= 1e-3 + 8e-3 * np.abs(bits_to_f64(ho))), f"h of expert {e}"
        assert_layer_close(yg[a:b], yo, f"y of expert {e}")
        assert np.mean(ulp_bf16(yg[a:b], yo) <= 1) > 0.99
    # rows past the last group are never written (tiles straddling a group edge are masked)
    assert np.all(bits_to_f64(hg[N:]) == 7.0) and np.all(bits_to_f64(yg[N:]) == 7.0)


def test_expert_ffn_rejects_bad_offsets(moe):
    E, d, f, max_rows = 4, 64, 64, 100
    off = np.array([0, 10, 5, 20, 30], np.int32)          # not monotone
    z = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device="cuda")
    y = torch.full((max_rows, d), 3.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    moe.moe_expert_ffn(z(max_rows, d), torch.from_numpy(off).cuda(), max_rows, E, d, f, z(E, f, d), z(E, f, d),
                       z(E, d, f), z(max_rows, f), y, ws)
    assert moe.moe_get_error() == moe.MOE_ERR_CHECK
    assert torch.all(y == 3.0)                             # no tile ran


# ----------------------------------------------------------------------------- whole layer, small

SMALL = [
    dict(name="tiny", wl=synth.WORKLOADS["tiny"]),
    dict(name="all-options", wl=synth.Workload("all", 300, 256, 16, 4, 320, f_shared=192, bias_range=0.1,
                                               cap_mode=synth.CAP_PER_TOKEN, capacity_factor=1.25)),
    dict(name="per-assignment-cap", wl=synth.Workload("cap", 513, 128, 8, 2, 128, cap_mode=synth.CAP_PER_ASSIGNMENT,
                                                      capacity_factor=0.8)),
    dict(name="single-expert", wl=synth.Workload("one", 200, 128, 1, 1, 256)),
    dict(name="pair-tiles-shared-cap", wl=synth.Workload("pairs", 1500, 256, 4, 2, 384, f_shared=256, bias_range=0.1,
                                                         cap_mode=synth.CAP_PER_TOKEN, capacity_factor=1.5)),
    dict(name="pair-tail-tiles-shared", wl=synth.Workload("tails", 1400, 256, 4, 2, 448, f_shared=192, bias_range=0.1)),
]


@pytest.mark.parametrize("case", SMALL, ids=[c["name"] for c in SMALL])
def test_layer_small_all_intermediates(moe, case):
    wl = case["wl"]
    inp = synth.Inputs(wl)
    x, wg, W1, W3, W2 = inp.x(), inp.wg(), inp.w1(), inp.w3(), inp.w2()
    bias = inp.bias()
    W1s, W3s, W2s = inp.shared("w1s"), inp.shared("w3s"), inp.shared("w2s")
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    C = oracle.capacity(T, E, k, wl.capacity_factor, wl.cap_mode)
    assert moe.moe_capacity(T, E, k, wl.capacity_factor, wl.cap_mode) == C
    dv = lambda a: to_dev_bf16(a) if a is not None else None
    ws = _ws(moe, T, d, E, k, f, fs)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(dv(x), dv(wg), torch.from_numpy(bias).cuda() if bias is not None else None, dv(W1), dv(W3),
                          dv(W2), dv(W1s), dv(W3s), dv(W2s), fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, out, ws)
    assert moe.moe_get_error() == 0
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    v = lambda n, s, dt: moe.workspace_view(ws, L, n, s, dt).cpu()
    g_logits = v("logits", (T, E), torch.float32).numpy()
    # (i) logits
    ref_logits = oracle.router_logits(x, wg)
    assert np.all(np.abs(g_logits.astype(np.float64) - ref_logits) <= logits_tol(x, wg))
    # (ii) routing from the GPU's logits: bit-exact; everything downstream fed the same logits
    ref = oracle.layer_forward(x, wg, W1, W3, W2, k=k, C=C, bias=bias, logits_in=g_logits, W1s=W1s, W3s=W3s, W2s=W2s)
    assert np.array_equal(v("idx", (T, k), torch.int32).numpy(), ref["idx"])
    np.testing.assert_allclose(v("w", (T, k), torch.float32).numpy(), ref["w"], rtol=1e-5, atol=1e-7)
    for n in ("counts_raw", "counts"):
        assert np.array_equal(v(n, (E,), torch.int32).numpy(), ref[n])
    assert np.array_equal(v("offsets", (E + 1,), torch.int32).numpy(), ref["offsets"])
    assert np.array_equal(v("dest", (T, k), torch.int32).numpy(), ref["dest"])
    N = ref["N"]
    assert np.array_equal(v("src_token", (T * k,), torch.int32).numpy()[:N], ref["src_token"])
    xp = bf16_bits(v("x_perm", (T * k, d), torch.bfloat16))[:N]
    assert np.array_equal(xp, oracle.gather(x, ref["dest"], N))
    # (iii) routing from the oracle's own logits, on tokens without a near tie at the k-th key
    own_idx, _ = oracle.route(ref_logits.astype(np.float32), k, bias)
    keys = np.sort(ref_logits + (bias if bias is not None else 0), axis=1)[:, ::-1]
    clear = (keys[:, k - 1] - keys[:, k]) >= 1e-5 if k < E else np.ones(T, bool)
    assert np.array_equal(own_idx[clear], ref["idx"][clear])
    # (iv) outputs
    got = bf16_bits(out)
    assert_layer_close(got, ref["out"])
    assert np.mean(ulp_bf16(got, ref["out"]) <= 1) > 0.99
    if fs:
        assert_layer_close(bf16_bits(v("y_shared", (T, d), torch.bfloat16)), ref["y_shared"], "y_shared")


# ----------------------------------------------------------------------------- overflow bias update

def test_update_bias_bit_exact(moe):
    E = 300
    counts = (synth.uniform_f32(0, 120, 0, E, 0, 5000)).astype(np.int32)
    for C in (1, 640, 1280, 4999):
        ref = oracle.update_bias(counts, C)
        b = torch.full((E,), 9.0, dtype=torch.float32, device="cuda")
        moe.moe_update_bias(torch.from_numpy(counts).cuda(), E, C, b)
        got = b.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    with pytest.raises(moe.MoeError):
        moe.moe_update_bias(torch.from_numpy(counts).cuda(), E, 0, b)


def test_two_batches_with_overflow_bias_and_eval_capacity(moe):
    # batch 1 routes without bias; its overflow sets the bias for batch 2 (eval factor 2.0)
    wl = synth.Workload("bias", 1024, 256, 16, 2, 256, cap_mode=synth.CAP_PER_TOKEN, capacity_factor=2.0)
    T, d, E, k, f = wl.T, wl.d, wl.E, wl.k, wl.f
    inp = synth.Inputs(wl)
    x1 = inp.x()
    x2 = inp.x_rows(T, T).reshape(T, d)
    wg = _bf16(E, d, 121, d ** -0.5)
    wg[:4] = _bf16(4, d, 122, 3 * d ** -0.5)          # a few hot experts
    W1, W3, W2 = inp.w1(), inp.w3(), inp.w2()
    C = oracle.capacity(T, E, k, 2.0, oracle.CAP_PER_TOKEN)
    dv = to_dev_bf16
    ws = _ws(moe, T, d, E, k, f)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros(E, dtype=torch.float32, device="cuda")
    L = moe.moe_workspace_layout(T, d, E, k, f)
    outs, logits = [], []
    for xb, b in ((x1, None), (x2, bias)):
        moe.moe_layer_forward(dv(xb), dv(wg), b, dv(W1), dv(W3), dv(W2), None, None, None, 0, T, d, E, k, f, 2.0,
                              moe.MOE_CAP_PER_TOKEN, out, ws)
        logits.append(moe.workspace_view(ws, L, "logits", (T, E), torch.float32).cpu().numpy())
        outs.append(bf16_bits(out))
        if b is None:     # bias for the next batch, from this batch's raw counts
            craw = moe.workspace_view(ws, L, "counts_raw", (E,), torch.int32)
            moe.moe_update_bias(craw, E, C, bias)
    assert moe.moe_get_error() == 0
    r1 = oracle.layer_forward(x1, wg, W1, W3, W2, k=k, C=C, logits_in=logits[0])
    b_ref = oracle.update_bias(r1["counts_raw"], C)
    assert np.array_equal(bias.cpu().numpy().view(np.uint32), b_ref.view(np.uint32))
    assert r1["counts_raw"].max() > C                  # the first batch did overflow
    r2 = oracle.layer_forward(x2, wg, W1, W3, W2, k=k, C=C, bias=b_ref, logits_in=logits[1])
    assert_layer_close(outs[0], r1["out"])
    assert_layer_close(outs[1], r2["out"])
    assert np.array_equal(moe.workspace_view(ws, L, "idx", (T, k), torch.int32).cpu().numpy(), r2["idx"])


# ----------------------------------------------------------------------------- one batch over two shards

def test_sharded_batch_with_global_capacity_matches_whole_batch(moe):
    # two shards of one batch run one after the other on this GPU (no kernel waits on another):
    # shard 1's fill_base comes from shard 0's counts, exactly as the all-gather would give it
    G, T, d, E, k, f = 2, 1024, 256, 16, 2, 256
    wl = synth.Workload("shards", G * T, d, E, k, f)
    inp = synth.Inputs(wl)
    x = inp.x()
    wg = _bf16(E, d, 131, d ** -0.5)
    wg[:3] = _bf16(3, d, 132, 3 * d ** -0.5)                # hot experts: the capacity binds
    W1, W3, W2 = inp.w1(), inp.w3(), inp.w2()
    C = moe.moe_capacity(G * T, E, k, 1.0, moe.MOE_CAP_PER_ASSIGNMENT)
    dv = to_dev_bf16
    Wd = [dv(W1), dv(W3), dv(W2)]
    ws = [_ws(moe, T, d, E, k, f) for _ in range(G)]
    xs = [dv(x[g * T:(g + 1) * T]) for g in range(G)]
    outs = [torch.empty((T, d), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    L = moe.moe_workspace_layout(T, d, E, k, f)
    for g in range(G):
        moe.moe_layer_route_count(xs[g], dv(wg), None, 0, T, d, E, k, f, ws[g])
    all_counts = torch.stack([moe.workspace_view(ws[g], L, "counts_raw", (E,), torch.int32) for g in range(G)])
    fill = torch.empty((G, E), dtype=torch.int32, device="cuda")
    for g in range(G):
        moe.moe_fill_base(all_counts, G, g, E, fill[g])
        moe.moe_layer_finish(xs[g], *Wd, None, None, None, 0, T, d, E, k, f, C, fill[g], outs[g], ws[g])
    assert moe.moe_get_error() == 0
    logits = np.concatenate([moe.workspace_view(ws[g], L, "logits", (T, E), torch.float32).cpu().numpy()
                             for g in range(G)])
    ref = oracle.layer_forward(x, wg, W1, W3, W2, k=k, C=C, logits_in=logits)
    assert (ref["counts_raw"] > C).any()
    assert np.array_equal(fill[1].cpu().numpy(), all_counts[0].cpu().numpy())
    kept = 0
    for g in range(G):
        dest = moe.workspace_view(ws[g], L, "dest", (T, k), torch.int32).cpu().numpy()
        assert np.array_equal(dest >= 0, ref["dest"][g * T:(g + 1) * T] >= 0)
        kept += int((dest >= 0).sum())
        assert_layer_close(bf16_bits(outs[g]), ref["out"][g * T:(g + 1) * T], f"shard {g}")
    assert kept == ref["N"]


# ----------------------------------------------------------------------------- host-buffer pipeline

def test_pipeline_matches_layer_forward_batch_by_batch(moe):
    wl = synth.Workload("pipe", 512, 256, 8, 2, 384, f_shared=128, bias_range=0.1,
                        cap_mode=synth.CAP_PER_TOKEN, capacity_factor=1.5)
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    inp = synth.Inputs(wl)
    dv = to_dev_bf16
    Wg, W1, W3, W2 = dv(inp.wg()), dv(inp.w1()), dv(inp.w3()), dv(inp.w2())
    W1s, W3s, W2s = dv(inp.shared("w1s")), dv(inp.shared("w3s")), dv(inp.shared("w2s"))
    bias = torch.from_numpy(inp.bias()).cuda()
    nb = 5
    xs = [torch.from_numpy(inp.x_rows(b * T, T).view(np.int16)).view(torch.bfloat16).reshape(T, d).pin_memory()
          for b in range(nb)]
    outs = [torch.zeros((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(nb)]
    mem = torch.empty(moe.moe_pipeline_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    pl = moe.Pipeline(Wg, bias, W1, W3, W2, W1s, W3s, W2s, fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, mem)
    for b in range(nb):
        pl.submit(xs[b], outs[b])
    pl.sync()
    pl.close()
    ws = _ws(moe, T, d, E, k, f, fs)
    ref = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    for b in range(nb):
        moe.moe_layer_forward(xs[b].cuda(), Wg, bias, W1, W3, W2, W1s, W3s, W2s, fs, T, d, E, k, f,
                              wl.capacity_factor, wl.cap_mode, ref, ws)
        assert torch.equal(outs[b].view(torch.int16), ref.cpu().view(torch.int16)), f"batch {b}"
    assert moe.moe_get_error() == 0


@pytest.mark.parametrize("a8", [False, True], ids=["fp8-weights", "fp8-weights-and-activations"])
def test_fp8_pipeline_matches_layer_forward_batch_by_batch(moe, a8):
    """moe_pipeline_create_w8: the fp8 layers through the host-buffer pipeline, bit for bit the
    same as the layer called on each batch."""
    wl = synth.Workload("pipe8", 384, 256, 8, 2, 256, f_shared=128, bias_range=0.1,
                        cap_mode=synth.CAP_PER_TOKEN, capacity_factor=1.5)
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    inp = synth.Inputs(wl)
    Wg = to_dev_bf16(inp.wg())
    bias = torch.from_numpy(inp.bias()).cuda()
    Q = synth.device_tensors_q8(wl, "cuda")
    routed = {"W1q": Q["w1q"], "W3q": Q["w3q"], "W2q": Q["w2q"], "s1": Q["s1"], "s3": Q["s3"], "s2": Q["s2"]}
    shared = {"W1q": Q["w1sq"], "W3q": Q["w3sq"], "W2q": Q["w2sq"], "s1": Q["s1s"], "s3": Q["s3s"], "s2": Q["s2s"]}
    nb = 4
    xs = [torch.from_numpy(inp.x_rows(b * T, T).view(np.int16)).view(torch.bfloat16).reshape(T, d).pin_memory()
          for b in range(nb)]
    outs = [torch.zeros((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(nb)]
    mem = torch.empty(moe.moe_pipeline_bytes_w8(T, d, E, k, f, fs, a8), dtype=torch.uint8, device="cuda")
    pl = moe.Pipeline(Wg, bias, None, None, None, None, None, None, fs, T, d, E, k, f, wl.capacity_factor,
                      wl.cap_mode, mem, routed=routed, shared=shared, activations_fp8=a8)
    for b in range(nb):
        pl.submit(xs[b], outs[b])
    pl.sync()
    pl.close()
    call = moe.moe_layer_forward_w8a8 if a8 else moe.moe_layer_forward_w8
    ws_bytes = moe.moe_workspace_bytes_a8(T, d, E, k, f, fs) if a8 else moe.moe_workspace_bytes(T, d, E, k, f, fs)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    ref = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    for b in range(nb):
        call(xs[b].cuda(), Wg, bias, Q["w1q"], Q["s1"], Q["w3q"], Q["s3"], Q["w2q"], Q["s2"], Q["w1sq"], Q["s1s"],
             Q["w3sq"], Q["s3s"], Q["w2sq"], Q["s2s"], fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, ref, ws)
        assert torch.equal(outs[b].view(torch.int16), ref.cpu().view(torch.int16)), f"batch {b}"
    assert moe.moe_get_error() == 0


# ----------------------------------------------------------------------------- fp8 expert weights

def _q8_reference(wl, x, logits, inp, k, C):
    """Oracle layer with fp8 experts: route the GPU's logits, dispatch, fp8 experts, combine."""
    E, d, f = wl.E, wl.d, wl.f
    idx, w = oracle.route(logits, k, inp.bias())
    r = oracle.dispatch(idx, E, C)
    y_perm = np.zeros((max(r["N"], 1), d), np.uint16)
    for e in range(E):
        a, b = r["offsets"][e], r["offsets"][e + 1]
        if a == b:
            continue
        q1, s1 = synth.quantize_e4m3_rows(inp.expert_rows("w1", e, 1), d)
        q3, s3 = synth.quantize_e4m3_rows(inp.expert_rows("w3", e, 1), d)
        q2, s2 = synth.quantize_e4m3_rows(inp.expert_rows("w2", e, 1), f)
        _, y_perm[a:b] = oracle.expert_ffn_q8(oracle.gather(x, r["dest"], r["N"])[a:b], q1, s1, q3, s3, q2, s2)
    ysh = None
    if wl.has_shared:
        qs = {n: synth.quantize_e4m3_rows(inp.shared(n), inp.shared(n).shape[1]) for n in ("w1s", "w3s", "w2s")}
        _, ysh = oracle.expert_ffn_q8(x, qs["w1s"][0], qs["w1s"][1], qs["w3s"][0], qs["w3s"][1], qs["w2s"][0],
                                      qs["w2s"][1])
    return idx, r, oracle.combine(y_perm, r["dest"], w, ysh)


@pytest.mark.parametrize("wl", [synth.Workload("q8", 300, 256, 16, 4, 320, f_shared=192, bias_range=0.1,
                                               cap_mode=synth.CAP_PER_TOKEN, capacity_factor=1.5),
                                synth.Workload("q8dec", 40, 448, 32, 8, 192, f_shared=128, bias_range=0.1),
                                synth.Workload("q8mix", 512, 256, 16, 2, 192, zipf_s=1.2)],
                         ids=["shared-cap-bias", "decode-shaped", "skewed-mixed-tiles"])
def test_layer_fp8_weights(moe, wl):
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    inp = synth.Inputs(wl)
    x = inp.x()
    Q = synth.device_tensors_q8(wl, "cuda")
    ws = _ws(moe, T, d, E, k, f, fs)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    bias = torch.from_numpy(inp.bias()).cuda() if inp.bias() is not None else None
    moe.moe_layer_forward_w8(to_dev_bf16(x), to_dev_bf16(inp.wg()), bias, Q["w1q"], Q["s1"], Q["w3q"], Q["s3"],
                             Q["w2q"], Q["s2"], Q.get("w1sq"), Q.get("s1s"), Q.get("w3sq"), Q.get("s3s"),
                             Q.get("w2sq"), Q.get("s2s"), fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, out, ws)
    assert moe.moe_get_error() == 0
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    logits = moe.workspace_view(ws, L, "logits", (T, E), torch.float32).cpu().numpy()
    C = oracle.capacity(T, E, k, wl.capacity_factor, wl.cap_mode)
    idx, r, ref = _q8_reference(wl, x, logits, inp, k, C)
    assert np.array_equal(moe.workspace_view(ws, L, "idx", (T, k), torch.int32).cpu().numpy(), idx)
    assert np.array_equal(moe.workspace_view(ws, L, "dest", (T, k), torch.int32).cpu().numpy(), r["dest"])
    got = bf16_bits(out)
    assert_layer_close(got, ref, "fp8-weight layer")
    assert np.mean(ulp_bf16(got, ref) <= 1) > 0.98


def _a8_reference(wl, x, logits, inp, k, C, g_h, g_hs):
    """Oracle layer with fp8 weights and fp8 activations on the GPU's logits.  The first expert
    GEMM runs on the oracle's own quantised x; the second on the GPU's h (g_h, g_hs), so that
    both sides quantise the same h rows (h itself is checked against the oracle's h).
    -> idx, dispatch, permuted x, oracle h, oracle h of the shared expert, output."""
    E, d, f = wl.E, wl.d, wl.f
    idx, w = oracle.route(logits, k, inp.bias())
    r = oracle.dispatch(idx, E, C)
    xp = oracle.gather(x, r["dest"], r["N"])
    h_ref = np.zeros((max(r["N"], 1), f), np.uint16)
    y_perm = np.zeros((max(r["N"], 1), d), np.uint16)
    for e in range(E):
        a, b = r["offsets"][e], r["offsets"][e + 1]
        if a == b:
            continue
        q1, s1 = synth.quantize_e4m3_rows(inp.expert_rows("w1", e, 1), d)
        q3, s3 = synth.quantize_e4m3_rows(inp.expert_rows("w3", e, 1), d)
        q2, s2 = synth.quantize_e4m3_rows(inp.expert_rows("w2", e, 1), f)
        h_ref[a:b] = oracle.expert_gate_up_w8a8(xp[a:b], q1, s1, q3, s3)
        y_perm[a:b] = oracle.expert_down_w8a8(g_h[a:b], q2, s2)
    hs_ref, ysh = None, None
    if wl.has_shared:
        qs = {n: synth.quantize_e4m3_rows(inp.shared(n), inp.shared(n).shape[1]) for n in ("w1s", "w3s", "w2s")}
        hs_ref = oracle.expert_gate_up_w8a8(x, qs["w1s"][0], qs["w1s"][1], qs["w3s"][0], qs["w3s"][1])
        ysh = oracle.expert_down_w8a8(g_hs, qs["w2s"][0], qs["w2s"][1])
    return idx, r, xp, h_ref[:r["N"]], hs_ref, oracle.combine(y_perm, r["dest"], w, ysh)


def _assert_h_close(g, r, what):
    """h bar: |d| <= 1e-3 + 8e-3 |ref| (one bf16 ulp plus a floor for cancellation in g, u)."""
    g64, r64 = bits_to_f64(g), bits_to_f64(r)
    bad = np.abs(g64 - r64) > 1e-3 + 8e-3 * np.abs(r64)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside 1e-3 + 8e-3|ref|"


@pytest.mark.parametrize("wl", [synth.Workload("a8", 300, 256, 16, 4, 384, f_shared=256, bias_range=0.1,
                                               cap_mode=synth.CAP_PER_TOKEN, capacity_factor=1.5),
                                synth.Workload("a8dec", 40, 512, 32, 8, 256, f_shared=128, bias_range=0.1),
                                synth.Workload("a8mix", 512, 256, 16, 2, 128, zipf_s=1.2),
                                synth.Workload("a8pair", 1024, 256, 4, 2, 256, f_shared=128,
                                               cap_mode=synth.CAP_PER_ASSIGNMENT, capacity_factor=1.1)],
                         ids=["shared-cap-bias", "decode-shaped", "skewed-mixed-tiles", "pair-tiles-shared-cap"])
def test_layer_fp8_weights_and_activations(moe, wl):
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    inp = synth.Inputs(wl)
    x = inp.x()
    Q = synth.device_tensors_q8(wl, "cuda")
    ws = torch.empty(moe.moe_workspace_bytes_a8(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    bias = torch.from_numpy(inp.bias()).cuda() if inp.bias() is not None else None
    moe.moe_layer_forward_w8a8(to_dev_bf16(x), to_dev_bf16(inp.wg()), bias, Q["w1q"], Q["s1"], Q["w3q"], Q["s3"],
                               Q["w2q"], Q["s2"], Q.get("w1sq"), Q.get("s1s"), Q.get("w3sq"), Q.get("s3s"),
                               Q.get("w2sq"), Q.get("s2s"), fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode,
                               out, ws)
    assert moe.moe_get_error() == 0
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    logits = moe.workspace_view(ws, L, "logits", (T, E), torch.float32).cpu().numpy()
    C = oracle.capacity(T, E, k, wl.capacity_factor, wl.cap_mode)
    g_h = bf16_bits(moe.workspace_view(ws, L, "h", (T * k, f), torch.bfloat16))
    g_hs = bf16_bits(moe.workspace_view(ws, L, "h_shared", (T, fs), torch.bfloat16)) if fs else None
    idx, r, xp, h_ref, hs_ref, ref = _a8_reference(wl, x, logits, inp, k, C, g_h, g_hs)
    assert np.array_equal(moe.workspace_view(ws, L, "idx", (T, k), torch.int32).cpu().numpy(), idx)
    _assert_h_close(g_h[:r["N"]], h_ref, "fp8 x fp8 h")
    if fs:
        _assert_h_close(g_hs, hs_ref, "fp8 x fp8 shared h")
    xq_ref, sx_ref = oracle.quantize_rows_e4m3(xp)
    got = bf16_bits(out)
    assert_layer_close(got, ref, "fp8 x fp8 layer")
    g64, r64 = bits_to_f64(got), bits_to_f64(ref)
    assert np.sqrt(np.mean((g64 - r64) ** 2) / max(np.mean(r64 ** 2), 1e-30)) < 5e-3
    assert xq_ref.shape[0] == r["N"] and np.isfinite(sx_ref).all()


def _a8_regions(T, d, k, f, fs, base):
    """Byte offsets of the fp8 rows and scales that follow the layer workspace (256-byte aligned,
    in the order xq, sx, hq, sh, xqs, sxs, hqs, shs)."""
    al = lambda v: (v + 255) // 256 * 256
    sizes = [("xq", T * k * d), ("sx", T * k * 4), ("hq", T * k * f), ("sh", T * k * 4),
             ("xqs", T * d if fs else 0), ("sxs", T * 4 if fs else 0), ("hqs", T * fs), ("shs", T * 4 if fs else 0)]
    off, cur = {}, al(base)
    for n, b in sizes:
        off[n] = cur
        cur = al(cur + b)
    return off


@pytest.mark.parametrize("wl", [synth.Workload("a8q", 64, 512, 4, 2, 768),
                                synth.Workload("a8q1", 32, 1024, 8, 3, 256),
                                synth.Workload("a8q2", 48, 2048, 8, 2, 6144),
                                synth.Workload("a8qm", 40, 4096, 16, 4, 2048, f_shared=128),
                                synth.Workload("a8qs", 24, 7168, 2, 2, 9216, f_shared=1536)],
                         ids=["d512", "d1024", "d2048-f6144", "d4096-shared", "d7168-f9216-shared"])
def test_quantised_rows_bit_exact(moe, wl):
    """The layer's activation quantisers against the oracle's: the routed rows (each token row
    quantised once and written to its permuted rows), the shared expert's rows, and h before
    GEMM2 (the kernel's own h, read back), bit for bit.  The row lengths reach every variant:
    a warp per row with 2, 4 or 8 chunks a lane (d = 512, 1024, 2048), 128 threads with 4 or 8
    (d = 4096, 7168; h of 6144), 256 threads (h of 9216), and the two-pass kernel (h <= 2048)."""
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    inp = synth.Inputs(wl)
    x = inp.x()
    Q = synth.device_tensors_q8(wl, "cuda")
    ws = torch.zeros(moe.moe_workspace_bytes_a8(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_w8a8(to_dev_bf16(x), to_dev_bf16(inp.wg()), None, Q["w1q"], Q["s1"], Q["w3q"], Q["s3"],
                               Q["w2q"], Q["s2"], Q.get("w1sq"), Q.get("s1s"), Q.get("w3sq"), Q.get("s3s"),
                               Q.get("w2sq"), Q.get("s2s"), fs, T, d, E, k, f, 1.0, moe.MOE_CAP_NONE, out, ws)
    assert moe.moe_get_error() == 0
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    o = _a8_regions(T, d, k, f, fs, moe.moe_workspace_bytes(T, d, E, k, f, fs))
    N = T * k
    rows = lambda n, r, c: ws[o[n]:o[n] + r * c].cpu().numpy().reshape(r, c)
    scales = lambda n, r: ws[o[n]:o[n] + 4 * r].view(torch.float32).cpu().numpy()
    dest = moe.workspace_view(ws, L, "dest", (T, k), torch.int32).cpu().numpy()
    xq_ref, sx_ref = oracle.quantize_rows_e4m3(oracle.gather(x, dest, N))
    assert np.array_equal(scales("sx", N).view(np.uint32), sx_ref.view(np.uint32))
    assert np.array_equal(rows("xq", N, d), xq_ref)
    h = bf16_bits(moe.workspace_view(ws, L, "h", (N, f), torch.bfloat16))
    hq_ref, sh_ref = oracle.quantize_rows_e4m3(h)
    assert np.array_equal(scales("sh", N).view(np.uint32), sh_ref.view(np.uint32))
    assert np.array_equal(rows("hq", N, f), hq_ref)
    if fs:
        xqs_ref, sxs_ref = oracle.quantize_rows_e4m3(x)
        assert np.array_equal(scales("sxs", T).view(np.uint32), sxs_ref.view(np.uint32))
        assert np.array_equal(rows("xqs", T, d), xqs_ref)
        hs = bf16_bits(moe.workspace_view(ws, L, "h_shared", (T, fs), torch.bfloat16))
        hqs_ref, shs_ref = oracle.quantize_rows_e4m3(hs)
        assert np.array_equal(scales("shs", T).view(np.uint32), shs_ref.view(np.uint32))
        assert np.array_equal(rows("hqs", T, fs), hqs_ref)


@pytest.mark.parametrize("wl", [synth.Workload("a8c0", 64, 256, 16, 4, 128, f_shared=128, cap_mode=synth.CAP_PER_TOKEN,
                                               capacity_factor=0.2),
                                synth.Workload("a8t1", 1, 256, 8, 2, 128)],
                         ids=["capacity-zero-shared-only", "one-token"])
def test_fp8_activation_layer_edge_cases(moe, wl):
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    inp = synth.Inputs(wl)
    x = inp.x()
    Q = synth.device_tensors_q8(wl, "cuda")
    ws = torch.empty(moe.moe_workspace_bytes_a8(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_w8a8(to_dev_bf16(x), to_dev_bf16(inp.wg()), None, Q["w1q"], Q["s1"], Q["w3q"], Q["s3"],
                               Q["w2q"], Q["s2"], Q.get("w1sq"), Q.get("s1s"), Q.get("w3sq"), Q.get("s3s"),
                               Q.get("w2sq"), Q.get("s2s"), fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode,
                               out, ws)
    assert moe.moe_get_error() == 0
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    logits = moe.workspace_view(ws, L, "logits", (T, E), torch.float32).cpu().numpy()
    C = oracle.capacity(T, E, k, wl.capacity_factor, wl.cap_mode)
    g_h = bf16_bits(moe.workspace_view(ws, L, "h", (T * k, f), torch.bfloat16))
    g_hs = bf16_bits(moe.workspace_view(ws, L, "h_shared", (T, fs), torch.bfloat16)) if fs else None
    idx, r, xp, h_ref, hs_ref, ref = _a8_reference(wl, x, logits, inp, k, C, g_h, g_hs)
    if wl.name == "a8c0":
        assert C == 0 and r["N"] == 0          # every routed row dropped: the shared expert alone
    assert_layer_close(bf16_bits(out), ref, "fp8 x fp8 edge case")
