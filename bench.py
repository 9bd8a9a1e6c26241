#!/usr/bin/env python
"""Benchmark: MoE-layer tokens/s on B200 (Router -> Permutation -> Expert GEMM -> Combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral] [--impl ours|reference]

One step = one moe_layer_forward over one batch of T tokens whose inputs already sit in
HBM (router GEMM, top-k, histogram/scan/permute, grouped GEMM1 + SwiGLU, grouped GEMM2,
combine).  Under torchrun each rank runs its own token batch against replicated weights
(no collective on the data path: weak scaling) and the time is the max over ranks.

Rank 0 prints one JSON line: value (tokens/s over all ranks), the dominant kernel's
roofline (its CUDA-event duration inside the timed region vs MEASURED_PEAKS.json),
an end-to-end number through the public API with host buffers, the SM clocks seen,
and (at N=1) the CPU oracle timed on a bounded sample.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200; % of BF16 tensor or HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS_PER_STEP = 9   # router GEMM, top-k, count, scan, scatter, gather, GEMM1, GEMM2, combine


def launches_per_step(a8: bool, shared: bool) -> int:
    """Kernels one layer call launches.  fp8 activations: no gather (one quantiser writes each x
    row's codes to its permuted rows and, with a shared expert, its own row), a quantiser of h
    before GEMM2 and one more for the shared expert's h."""
    if not a8:
        return KERNELS_PER_STEP
    return KERNELS_PER_STEP - 1 + 2 + (1 if shared else 0)

DESCR = {
    "tiny": "tiny MoE layer T=128 d=256 E=8 top-2 f=512",
    "mixtral": "Mixtral-like prefill T=4096 d=4096 E=8 top-2 SwiGLU f=14336",
    "qwen3": "Qwen3-235B-A22B-like prefill T=16384 d=4096 E=128 top-8 f=1536",
    "dsv3": "DeepSeek-V3-like decode T=256 d=7168 E=256 top-8 f=2048 + shared f=2048, selection bias",
    "skew": "skewed routing T=32768 d=4096 E=64 top-2 f=2048 Zipf(1.2), capacity int(T*k/E*1.25)",
    "mixtral2e": "profiling case: Mixtral-like layer cut to T=2048, E=2 (same tile shapes)",
    "dsv3_32e": "profiling case: DeepSeek-V3-like decode cut to T=32, E=32 (same tile shapes)",
    "qwen3_16e": "profiling case: Qwen3-like prefill cut to T=2048, E=16 (same tile shapes)",
    "qwen3_f128": "profiling case: Qwen3-like batch and routing (T=16384 E=128 top-8) with experts cut to f=128",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mixtral", choices=list(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--weights", default="bf16", choices=["bf16", "fp8", "fp8a8"],
                    help="expert weight format: bf16; fp8 e4m3 with fp32 row scales (moe_layer_forward_w8); "
                         "fp8a8: fp8 weights and fp8 activations with per-row scales (moe_layer_forward_w8a8)")
    ap.add_argument("--cache-slots", type=int, default=0,
                    help="> 0: decode through the expert cache (moe_layer_forward_cached) with this many HBM "
                         "slots; expert weights in page-locked host memory; a fresh token batch every step")
    ap.add_argument("--cache-tokens", type=int, default=16, help="decode batch (tokens per step) with --cache-slots")
    ap.add_argument("--cache-zipf", type=float, default=1.0, help="Zipf exponent of expert popularity (cache runs)")
    ap.add_argument("--ep-ranks", type=int, default=0,
                    help="> 0: expert parallelism with this many ranks emulated on one GPU (the workload's batch "
                         "split over the ranks, experts split contiguously); prints its own line")
    ap.add_argument("--ep-exchange", default="fused", choices=["put", "fused", "a2a"],
                    help="with --ep-ranks: put kernels both ways; put dispatch + return from GEMM2's own stores "
                         "(fused); or all-to-all-v style copies")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="at N=1 with bf16 weights the line also carries per_config: every workload of the "
                         "task timed in the same run (tokens/s, roofline, oracle sample); this skips it")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(fp8: bool = False) -> str:
    """Hash of the sources of the grouped GEMM kernels (bf16, or the fp8-weight one)."""
    h = hashlib.sha256()
    files = ("grouped_gemm.cuh", "grouped_gemm_pair.cuh", "ptx.cuh") + (("grouped_gemm_w8.cuh",) if fp8 else ())
    for n in files:
        h.update(open(os.path.join(ROOT, "moe_layer_router_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this kernel source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    src = kernel_source_hash(kernel.endswith("_fp8"))   # "_fp8a8" kernels live in the bf16 sources
    for line in open(p):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload \
                and parts[2] == src:
            return float(parts[3])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.dev)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            p = [s.strip() for s in line.split(",")]
            if len(p) < 8:
                continue
            try:
                rows.append((float(p[0]), float(p[1]), p[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = np.array([r[0] for r in rows])
        mx = max(r[1] for r in rows)
        loaded = sm[sm >= 0.5 * np.max(sm)]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[2][i].lower() == "active"})
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------ oracle (CPU) legs

def host_weights(wl):
    inp = synth.Inputs(wl)
    w = dict(wg=inp.wg(), w1=inp.w1(), w3=inp.w3(), w2=inp.w2(), bias=inp.bias(),
             w1s=inp.shared("w1s"), w3s=inp.shared("w3s"), w2s=inp.shared("w2s"))
    return inp, w


def oracle_step(oracle, wl, inp, w, t0, S):
    x = inp.x_rows(t0, S).reshape(S, wl.d)
    C = oracle.capacity(wl.T, wl.E, wl.k, wl.capacity_factor, wl.cap_mode)
    if C >= 0:   # the capacity of the full batch, scaled to the sample
        C = max(0, int(C * S / wl.T))
    t = time.perf_counter()
    oracle.layer_forward(x, w["wg"], w["w1"], w["w3"], w["w2"], k=wl.k, C=C, bias=w["bias"],
                         W1s=w["w1s"], W3s=w["w3s"], W2s=w["w2s"])
    return time.perf_counter() - t


def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def sample_size(oracle, wl, inp, w, seconds):
    """Tokens in one oracle sample so that it takes about `seconds` (calibrated on a small run)."""
    s0 = min(wl.T, 16)
    dt = oracle_step(oracle, wl, inp, w, 0, s0)
    S = int(s0 * seconds / max(dt, 1e-3))
    return max(1, min(wl.T, S)), dt, s0


def cpu_baseline(wl, seconds, inp=None, w=None):
    import oracle
    if inp is None:
        inp, w = host_weights(wl)
    S, _, _ = sample_size(oracle, wl, inp, w, seconds)
    dt = oracle_step(oracle, wl, inp, w, 0, S)
    if dt < 0.6 * seconds and S < wl.T:          # parallel efficiency grows with the sample: rescale once
        S = max(1, min(wl.T, int(S * seconds / max(dt, 1e-3))))
        dt = oracle_step(oracle, wl, inp, w, 0, S)
    return {"value": S / dt, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"oracle layer forward on the first {S} of {wl.T} tokens ({dt:.1f} s, capacity scaled to "
                      f"the sample), double-precision sums, OpenMP over rows"}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    import oracle
    inp, w = host_weights(wl)
    per_step = min(8.0, 150.0 / max(1, args.steps + args.warmup))
    S, _, _ = sample_size(oracle, wl, inp, w, per_step)
    for i in range(args.warmup):
        oracle_step(oracle, wl, inp, w, 0, S)
    tot = 0.0
    for i in range(args.steps):
        tot += oracle_step(oracle, wl, inp, w, (i * S) % max(1, wl.T - S + 1), S)
    value = S * args.steps / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": DESCR[wl.name], "global_batch": S, "sample_tokens_per_step": S},
            "cpu_baseline": {"kind": "oracle", "cores": cpu_threads(), "value": value, "unit": "tokens/s",
                             "sample": f"{S} of {wl.T} tokens per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ GPU leg

def gemm1_work(wl, N):
    """Algorithmic FLOPs and bytes of one launch of the first grouped GEMM (W1/W3 + SwiGLU)."""
    flops = 4.0 * N * wl.d * wl.f + 4.0 * wl.T * wl.d * wl.f_shared
    return flops


def gemm1_bytes(wl, N, touched, wbytes=2, abytes=2):
    """Algorithmic bytes of one launch of the first grouped GEMM: weights of the touched experts
    (wbytes per element, + fp32 row scales for fp8), its A rows (abytes per element, + a row
    scale for fp8 activations), h written in bf16; the same for the shared expert."""
    b = touched * 2.0 * wl.f * wl.d * wbytes        # W1, W3 of touched experts
    if wbytes == 1:
        b += touched * 2.0 * wl.f * 4                # row scales
    b += N * wl.d * abytes + N * wl.f * 2           # A rows read, h write
    if abytes == 1:
        b += N * 4.0
    if wl.f_shared:
        b += 2.0 * wl.f_shared * wl.d * wbytes + wl.T * wl.d * abytes + wl.T * wl.f_shared * 2
        if wbytes == 1:
            b += 2.0 * wl.f_shared * 4
        if abytes == 1:
            b += wl.T * 4.0
    return b


def gemms_work(wl, N):
    """FLOPs of both grouped GEMMs of one layer call (routed + shared)."""
    return 6.0 * N * wl.d * wl.f + 6.0 * wl.T * wl.d * wl.f_shared


def layer_work(wl, N, touched, wbytes=2):
    flops = 6.0 * N * wl.d * wl.f + 2.0 * wl.T * wl.d * wl.E + 6.0 * wl.T * wl.d * wl.f_shared
    b = touched * 3.0 * wl.f * wl.d * wbytes + wl.E * wl.d * 2 + 3.0 * wl.f_shared * wl.d * wbytes
    b += wl.T * wl.d * 2 + 2 * N * wl.d * 2 + 2 * N * wl.f * 2 + 2 * N * wl.d * 2 + wl.T * wl.d * 2
    if wl.f_shared:
        b += 2 * wl.T * wl.f_shared * 2 + 2 * wl.T * wl.d * 2
    return flops, b


L2_BYTES = 126 * 10**6          # B200 L2


def working_set_bytes(wl, wbytes: int = 2) -> float:
    """Upper bound of the bytes one layer step touches: every expert's weights, the shared expert,
    the router, x and out, and the permuted rows / h / y_perm of all T k assignments."""
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    return (3.0 * E * f * d * wbytes + 3.0 * fs * d * wbytes + E * d * 2 + 2.0 * T * d * 2 +
            T * k * (2.0 * d + f) * 2 + (T * (d + fs) * 2 if fs else 0))


class L2Flush:
    """Writes a buffer twice the size of L2 between timed steps whose working set fits in L2, so
    that every step starts with cold caches."""

    def __init__(self, dev):
        import torch
        self.buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.buf.zero_()


def timed_steps(fwd, evs, flush, sync=None):
    """Run len(evs) timed layer steps; with `flush`, L2 is flushed before each step and the step
    time is the sum of the per-step (route -> end) intervals, so the flushes stay outside it;
    without, it is the span from the first step's start to the last step's end."""
    K = len(evs)
    for i in range(K):
        if flush is not None:
            flush()
        fwd(evs[i])
    if sync is None:
        import torch
        sync = torch.cuda.synchronize
    sync()
    if flush is not None:
        return float(sum(e["route"].elapsed_time(e["end"]) for e in evs))
    return evs[0]["route"].elapsed_time(evs[K - 1]["end"])


def l2_note(wl, flush, wbytes: int = 2) -> str:
    ws = working_set_bytes(wl, wbytes)
    if flush is not None:
        return "L2 flushed before every timed step (a %d MB write; working set %.1f MB < L2)" % (
            2 * L2_BYTES // 10**6, ws / 1e6)
    return "working set larger than L2 (%.2f GB per step)" % (ws / 1e9)


def roofline_and_layer(wl, N, touched, counts, craw, gemm_ms, step_ms, fp8, a8, peaks, peak_src):
    """The dominant kernel's roofline (GEMM1: tensor-bound for prefill, HBM-bound for decode) and
    the layer's totals for one timed configuration.  gemm_ms: mean kernel times of the two grouped
    GEMMs; step_ms: mean layer time."""
    T, k, E = wl.T, wl.k, wl.E
    g1_ms = gemm_ms["gate_up"]
    decode = wl.name.startswith("dsv3")
    tc_ratio = 2.0 if a8 else 1.0     # fp8 tensor peak = measured bf16 peak x the nominal 4.5 / 2.25
    if decode:
        alg = gemm1_bytes(wl, N, touched, 1 if fp8 else 2, 1 if a8 else 2)
        achieved = alg / (g1_ms / 1000.0) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    else:
        alg = gemm1_work(wl, N)
        achieved = alg / (g1_ms / 1000.0) / 1e12
        roof = {"bound": "latency" if wl.name == "tiny" else "tensor", "achieved": achieved,
                "peak": peaks["bf16_tflops"] * tc_ratio, "unit": "TFLOP/s",
                "frac": achieved / (peaks["bf16_tflops"] * tc_ratio)}
        # the same achieved rate against the power-capped sustained GEMM rate, for context
        roof["frac_of_sustained"] = achieved / (peaks["bf16_tflops_sustained"] * tc_ratio)
    roof["traffic"] = recorded_traffic("gate_up" + ("_fp8a8" if a8 else "_fp8" if fp8 else ""), wl.name)
    pair = T * k >= 256 * E
    roof["kernel"] = (("grouped_gemm_pair_kernel" if pair else "grouped_gemm_kernel") + "<EPI_SWIGLU, F8> (fp8 x fp8)"
                      if a8 else
                      "grouped_gemm_w8_kernel<EPI_SWIGLU>" if fp8 else
                      "grouped_gemm_pair_kernel<EPI_SWIGLU>" if pair else "grouped_gemm_kernel<EPI_SWIGLU>") + \
        " (gate_up: W1/W3 + SwiGLU)"
    roof["peak_source"] = f"{peak_src} ({'hbm_gbs' if decode else 'bf16_tflops'}, burst)" + \
        ("" if decode or not a8 else " x 2 (nominal fp8 / bf16 dense ratio)")
    roof["algorithmic_per_launch"] = alg
    lf, lb = layer_work(wl, N, touched, 1 if fp8 else 2)
    step_s = step_ms / 1000.0
    layer = {"tflops": lf / step_s / 1e12, "gbs": lb / step_s / 1e9,
             # both grouped GEMMs' FLOPs over their kernel times, against the tensor peak
             # of their operand type (bf16, or fp8 = measured bf16 x 2)
             "gemms_tensor_frac": gemms_work(wl, N) / ((gemm_ms["gate_up"] + gemm_ms["down"]) / 1e3) / 1e12
             / (peaks["bf16_tflops"] * tc_ratio),
             "tensor_frac": lf / step_s / 1e12 / peaks["bf16_tflops"],
             "hbm_frac": lb / step_s / 1e9 / peaks["hbm_gbs"], "kept_rows": N, "touched_experts": touched,
             "drop_rate": 1.0 - N / float(T * k), "load_var_raw": float(np.var(craw)),
             "load_var_kept": float(np.var(counts)), "max_rows": int(counts.max()),
             "min_rows": int(counts.min())}
    if wl.zipf_s > 0:
        p = craw / craw.sum()
        layer["zipf_l1_error"] = float(np.abs(p - synth.Inputs(wl).zipf_target()).sum())
    return roof, layer



PER_CONFIG_STEPS = {"tiny": 50, "mixtral": 20, "qwen3": 20, "dsv3": 20, "skew": 20}


def config_entry(wl, value, ms_per_step, steps, roof, layer, stage_ms, gemm_ms, clocks, cpu, l2=None):
    """One workload's record in per_config."""
    r = {k: roof[k] for k in ("bound", "kernel", "achieved", "unit", "peak", "frac", "peak_source")}
    if "frac_of_sustained" in roof:
        r["frac_of_sustained"] = roof["frac_of_sustained"]
    e = {"workload": DESCR[wl.name], "tokens_per_s": value, "ms_per_step": ms_per_step, "steps": steps,
         "roofline": r, "gemms_tensor_frac": layer["gemms_tensor_frac"], "tensor_frac": layer["tensor_frac"],
         "hbm_frac": layer["hbm_frac"], "kept_rows": layer["kept_rows"], "drop_rate": layer["drop_rate"],
         "load_var_raw": layer["load_var_raw"], "load_var_kept": layer["load_var_kept"],
         "stages_ms": stage_ms, "gemm_ms": gemm_ms, "clocks": clocks, "cpu_baseline": cpu}
    if l2 is not None:
        e["l2"] = l2
    if "zipf_l1_error" in layer:
        e["zipf_l1_error"] = layer["zipf_l1_error"]
    return e


def measure_config(name, dev, warmup, peaks, peak_src, cpu_seconds):
    """Time one workload at N = 1 (bf16 weights; inputs resident in HBM), and the oracle on a sample
    of it, for per_config.  The host copy of the weights serves both."""
    import torch
    import moe_layer_router_b200 as moe

    wl = synth.WORKLOADS[name]
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    inp, w = host_weights(wl)
    dv = lambda a: None if a is None else \
        torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    W = {n: dv(w[n]) for n in ("wg", "w1", "w3", "w2", "w1s", "w3s", "w2s")}
    bias = None if w["bias"] is None else torch.from_numpy(w["bias"]).to(dev)
    x = dv(inp.x())
    ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device=dev)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)

    def fwd(events=None):
        moe.moe_layer_forward_ex(x, W["wg"], bias, W["w1"], W["w3"], W["w2"], W["w1s"], W["w3s"], W["w2s"], fs,
                                 T, d, E, k, f, wl.capacity_factor, wl.cap_mode, out, ws, events)

    for _ in range(max(3, warmup)):
        fwd()
    torch.cuda.synchronize()
    rc = moe.moe_get_error()
    if rc != 0:
        raise RuntimeError(f"{name}: device error after warm-up: {moe.strerror(rc)}")
    K = PER_CONFIG_STEPS[name]
    evs = [{n: torch.cuda.Event(enable_timing=True) for n in moe.STAGES} for _ in range(K)]
    for e in evs:
        for ev in e.values():
            ev.record()
    flush = L2Flush(dev) if working_set_bytes(wl) < L2_BYTES else None
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        total_ms = timed_steps(fwd, evs, flush)
    rc = moe.moe_get_error()
    if rc != 0:
        raise RuntimeError(f"{name}: device error: {moe.strerror(rc)}")
    l2 = l2_note(wl, flush)
    del flush
    stage_ms = {a: float(np.mean([e[a].elapsed_time(e[b]) for e in evs]))
                for a, b in zip(moe.STAGES[:-1], moe.STAGES[1:])}
    gemm_ms = {"gate_up": stage_ms["gate_up"], "down": stage_ms["down"]}
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    counts = moe.workspace_view(ws, L, "counts", (E,), torch.int32).cpu().numpy()
    craw = moe.workspace_view(ws, L, "counts_raw", (E,), torch.int32).cpu().numpy()
    N = int(counts.sum())
    touched = int((counts > 0).sum())
    roof, layer = roofline_and_layer(wl, N, touched, counts, craw, gemm_ms, total_ms / K, False, False, peaks,
                                     peak_src)
    del W, bias, x, ws, out
    torch.cuda.empty_cache()
    cpu = cpu_baseline(wl, cpu_seconds, inp, w) if cpu_seconds > 0 else None
    return config_entry(wl, T * K / (total_ms / 1e3), total_ms / K, K, roof, layer, stage_ms, gemm_ms,
                        clk.summary(), cpu, l2)



def run_cached(args, base, rank, world, local):
    """Decode with the routed experts in page-locked host memory and an LRU of S HBM slots.

    One step = one moe_layer_forward_cached over a fresh batch of `--cache-tokens` tokens (the
    router sees new tokens every step, so the cache sees real misses); the expert popularity
    follows Zipf(`--cache-zipf`).  The dominant kernel is the copy of the missed experts over the
    host link, so its roofline is that link: the bytes it moved over its event time, against a
    pinned cudaMemcpyAsync host-to-device copy of 1 GiB measured in the same run."""
    import dataclasses

    import torch
    import torch.distributed as dist
    import moe_layer_router_b200 as moe
    from moe_layer_router_b200 import dp

    wl = dataclasses.replace(base, name=base.name + "_cached", T=args.cache_tokens, zipf_s=args.cache_zipf)
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    S = args.cache_slots
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    fp8 = args.weights == "fp8"
    if fp8:
        W = synth.device_tensors(wl, dev, names=["wg", "bias"])
        Q = synth.device_tensors_q8(wl, dev)
        routed = {"W1q": "w1q", "W3q": "w3q", "W2q": "w2q", "s1": "s1", "s3": "s3", "s2": "s2"}
        shared = {"W1q": Q["w1sq"], "W3q": Q["w3sq"], "W2q": Q["w2sq"], "s1": Q["s1s"], "s3": Q["s3s"], "s2": Q["s2s"]}
        W.update({n: Q[q] for n, q in routed.items()})
        names = list(routed)
    else:
        W = synth.device_tensors(wl, dev, names=["wg", "w1", "w3", "w2", "w1s", "w3s", "w2s", "bias"])
        names = ["w1", "w3", "w2"]
    host = {}
    for n in names:                        # the routed experts live in page-locked host memory
        host[n] = torch.empty(W[n].shape, dtype=W[n].dtype, pin_memory=True)
        host[n].copy_(W[n])
        del W[n]
    if fp8:
        del Q
    torch.cuda.empty_cache()
    slots = {n: torch.empty((S,) + tuple(host[n].shape[1:]), dtype=host[n].dtype, device=dev) for n in names}
    state = torch.empty(moe.moe_cache_state_bytes(E, S), dtype=torch.uint8, device=dev)
    moe.moe_cache_reset(state, E, S)
    inp = synth.Inputs(wl)
    nb = max(3, args.warmup) + args.steps
    row0 = rank * nb * T
    xs = torch.from_numpy(inp.x_rows(row0, nb * T).view(np.int16)).view(torch.bfloat16).reshape(nb, T, d).to(dev)
    ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device=dev)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)

    def fwd(i, events=None, xin=None):
        xi = xs[i] if xin is None else xin
        if fp8:
            moe.moe_layer_forward_cached_w8(xi, W["wg"], W["bias"], host, slots, S, state, shared, fs, T, d, E, k, f,
                                            wl.capacity_factor, wl.cap_mode, out, ws, events)
        else:
            moe.moe_layer_forward_cached(xi, W["wg"], W["bias"], host["w1"], host["w3"], host["w2"], slots["w1"],
                                         slots["w3"], slots["w2"], S, state, W.get("w1s"), W.get("w3s"), W.get("w2s"),
                                         fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, out, ws, events)

    nw = max(3, args.warmup)
    for i in range(nw):
        fwd(i)
    torch.cuda.synchronize()
    if moe.moe_get_error() != 0:
        raise RuntimeError("device error after warm-up")
    c0 = moe.cache_counters(state)
    K = args.steps
    names = moe.STAGES + ["cache", "copy_start", "copy_end"]
    evs = [{n: torch.cuda.Event(enable_timing=True) for n in names} for _ in range(K)]
    for e in evs:
        for ev in e.values():
            ev.record()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(K):
            fwd(nw + i, evs[i])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = dp.max_over_ranks(evs[0]["route"].elapsed_time(evs[K - 1]["end"]), device=dev)
    order = ["route", "topk", "permute", "cache", "gate_up", "down", "combine", "end"]
    stage_ms = {a: float(np.mean([e[a].elapsed_time(e[b]) for e in evs])) for a, b in zip(order[:-1], order[1:])}
    c1 = moe.cache_counters(state)
    expert_bytes = 3 * f * d + 4 * (2 * f + d) if fp8 else 3 * f * d * 2
    hits, misses = c1["hits"] - c0["hits"], c1["misses"] - c0["misses"]
    # the copy kernel on the cache's copy stream (it overlaps the resident experts' GEMMs)
    copy_ms = sum(e["copy_start"].elapsed_time(e["copy_end"]) for e in evs)
    link_gbs = misses * expert_bytes / 1e9 / (copy_ms / 1e3)
    # end to end: every step copies its tokens from page-locked host memory and its output back
    x_pin = xs.cpu().pin_memory()
    out_pin = torch.empty((T, d), dtype=torch.bfloat16, pin_memory=True)
    xin = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for i in range(K):
        xin.copy_(x_pin[nw + i], non_blocking=True)
        fwd(0, None, xin)
        out_pin.copy_(out, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = dp.max_over_ranks(e0.elapsed_time(e1), device=dev)
    # the host link as a plain DMA copy sees it: 1 GiB page-locked -> device, 5 times
    hsrc = torch.empty(1 << 30, dtype=torch.uint8, pin_memory=True)
    ddst = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    ddst.copy_(hsrc, non_blocking=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(5):
        ddst.copy_(hsrc, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    dma_gbs = 5 * (1 << 30) / 1e9 / (e0.elapsed_time(e1) / 1e3)
    if moe.moe_get_error() != 0:
        raise RuntimeError("device error")
    value = dp.job_throughput(T, world, K, total_ms)
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    line = {
        "metric": "MoE-layer tokens/s on 1 B200, routed experts served from an HBM expert cache",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": nw,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 activations, fp8 e4m3 expert weights" if fp8 else "bf16",
        "data": "synthetic (seeded Philox4x32-10 + Box-Muller; random-init weights)",
        "config": {"workload": f"DeepSeek-V3-like decode T={T} d={d} E={E} top-{k} f={f} + shared f={fs}, "
                               f"Zipf({wl.zipf_s}) expert popularity, fresh tokens every step; routed experts in "
                               f"page-locked host memory ({E * expert_bytes / 1e9:.1f} GB), {S} HBM slots",
                   "global_batch": world * T, "seq_len": T, "parallelism": f"dp{world}", "cache_slots": S,
                   "l2": "working set larger than L2 (expert weights streamed from host memory and HBM)"},
        "roofline": {"bound": "host_link", "achieved": link_gbs, "peak": dma_gbs, "unit": "GB/s",
                     "frac": link_gbs / dma_gbs if dma_gbs else None, "traffic": None,
                     "kernel": "cache_load_kernel (missed experts' W1/W3/W2, host memory -> HBM slots)",
                     "peak_source": "measured in this run (cudaMemcpyAsync page-locked -> device, 1 GiB x 5)",
                     "algorithmic_per_launch": misses / K * expert_bytes},
        "cache": {"hits": hits, "misses": misses, "hit_rate": hits / max(1, hits + misses),
                  "loads_per_step": misses / K, "expert_mb": expert_bytes / 1e6,
                  "copy_ms_per_step": copy_ms / K, "step_over_copy": total_ms / max(copy_ms, 1e-9)},
        "stages_ms": stage_ms,
        "e2e": {"value": dp.job_throughput(T, world, K, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": T * d * 2,
                "d2h_bytes_per_step": T * d * 2},
        "gpu_launches": (KERNELS_PER_STEP + 4) * K,   # + cache plan, copy, the loaded experts' two GEMMs
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_ep(args, wl, local):
    """The workload's batch split over R expert-parallel ranks emulated on one GPU (ep.EmulatedEP):
    every rank routes its T / R tokens, the row ranges move between the ranks' buffers by the
    library's put kernels, each rank runs its E / R experts.  Timed beside the single-GPU layer
    on the same batch.  The exchange kernels' roofline is the HBM copy bandwidth here (on several
    GPUs it would be the NVLink bandwidth); bytes = rows moved x d x 2 B, read + written, both ways."""
    import torch
    import moe_layer_router_b200 as moe
    from moe_layer_router_b200.ep import EmulatedEP

    R = args.ep_ranks
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    if T % R or E % R:
        raise SystemExit("--ep-ranks must divide T and E")
    Tr = T // R
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    W = synth.device_tensors(wl, dev, names=["x", "wg", "w1", "w3", "w2", "w1s", "w3s", "w2s", "bias"])
    xs = [W["x"][r * Tr:(r + 1) * Tr] for r in range(R)]
    outs = [torch.empty((Tr, d), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    ep = EmulatedEP(R, Tr, d, E, k, f, fs, device=dev, exchange=args.ep_exchange)

    def step(events=None):
        ep.forward(xs, W["wg"], W["bias"], W["w1"], W["w3"], W["w2"], W.get("w1s"), W.get("w3s"), W.get("w2s"),
                   wl.capacity_factor, wl.cap_mode, outs, events)

    ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device=dev)
    out1 = torch.empty((T, d), dtype=torch.bfloat16, device=dev)

    def single():
        moe.moe_layer_forward(W["x"], W["wg"], W["bias"], W["w1"], W["w3"], W["w2"], W.get("w1s"), W.get("w3s"),
                              W.get("w2s"), fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, out1, ws)

    for _ in range(max(3, args.warmup)):
        step()
        single()
    torch.cuda.synchronize()
    if moe.moe_get_error() != 0:
        raise RuntimeError("device error after warm-up")
    K = args.steps
    evs = [{n: torch.cuda.Event(enable_timing=True) for n in EmulatedEP.STAGES} for _ in range(K)]
    for e in evs:
        for ev in e.values():
            ev.record()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(K):
            step(evs[i])
        torch.cuda.synchronize()
    total_ms = evs[0]["route"].elapsed_time(evs[K - 1]["end"])
    st = EmulatedEP.STAGES
    stage_ms = {a: float(np.mean([e[a].elapsed_time(e[b]) for e in evs])) for a, b in zip(st[:-1], st[1:])}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K):
        single()
    e1.record()
    torch.cuda.synchronize()
    single_ms = e0.elapsed_time(e1)
    if moe.moe_get_error() != 0:
        raise RuntimeError("device error")
    N = sum(int(moe.workspace_view(b.ws, b.layout, "counts", (E,), torch.int32).sum()) for b in ep.ranks)
    fused = args.ep_exchange == "fused"
    moved = (1 if fused else 2) * N * d * 2     # rows out (and back, unless GEMM2 returns them), bf16
    put_ms = stage_ms["dispatch"] + (0.0 if fused else stage_ms["return"])
    achieved = 2 * moved / 1e9 / (put_ms / 1e3)  # read + write
    put_kernel = ("ep_put_rows_kernel (dispatch row ranges; GEMM2's epilogue stores the results into the "
                  "tokens' ranks' y_perm)" if fused else
                  "ep_put_rows_kernel (dispatch + return row ranges between the ranks' buffers)")
    peaks, peak_src = load_peaks()
    line = {
        "metric": "MoE-layer tokens/s on 1 B200, experts split over R expert-parallel ranks emulated on the GPU",
        "value": T * K / (total_ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": max(3, args.warmup),
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded Philox4x32-10 + Box-Muller; random-init weights)",
        "config": {"workload": DESCR.get(wl.name, wl.name) + f", split over {R} emulated expert-parallel ranks "
                               f"({Tr} tokens and {E // R} experts each)",
                   "global_batch": T, "seq_len": T, "parallelism": f"ep{R} (emulated on one GPU)",
                   "l2": "working set larger than L2 (expert weights streamed every step)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "kernel": put_kernel,
                     "peak_source": f"{peak_src} (hbm_gbs, burst)",
                     "algorithmic_per_launch": 2 * moved / ((1 if fused else 2) * R)},
        "exchange": args.ep_exchange,
        "single_gpu_layer_ms": single_ms / K,
        "stages_ms": stage_ms,
        "e2e": None,
        "gpu_launches": None,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    wl = synth.WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, wl, rank, world)
    if args.cache_slots > 0:
        return run_cached(args, wl, rank, world, local)
    if args.ep_ranks > 0:
        return run_ep(args, wl, local)

    import torch
    import torch.distributed as dist
    import moe_layer_router_b200 as moe
    from moe_layer_router_b200 import dp

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    # inputs: replicated weights, a distinct token batch per rank
    fp8 = args.weights in ("fp8", "fp8a8")
    a8 = args.weights == "fp8a8"
    tensors = synth.device_tensors(wl, dev, names=["wg", "bias"] if fp8 else
                                   ["wg", "w1", "w3", "w2", "w1s", "w3s", "w2s", "bias"])
    if fp8:
        tensors.update(synth.device_tensors_q8(wl, dev))
    inp = synth.Inputs(wl)
    row0, nrows = dp.token_rows(rank, world, wl.T)
    x_host = torch.from_numpy(inp.x_rows(row0, nrows).view(np.int16)).view(torch.bfloat16).reshape(wl.T, wl.d)
    x = x_host.to(dev)
    T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
    ws_bytes = moe.moe_workspace_bytes_a8(T, d, E, k, f, fs) if a8 else moe.moe_workspace_bytes(T, d, E, k, f, fs)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    W = tensors

    def fwd(xin, o, events=None):
        if fp8:
            call = moe.moe_layer_forward_w8a8 if a8 else moe.moe_layer_forward_w8
            call(xin, W["wg"], W["bias"], W["w1q"], W["s1"], W["w3q"], W["s3"], W["w2q"], W["s2"], W.get("w1sq"),
                 W.get("s1s"), W.get("w3sq"), W.get("s3s"), W.get("w2sq"), W.get("s2s"), fs, T, d, E, k, f,
                 wl.capacity_factor, wl.cap_mode, o, ws, events)
        else:
            moe.moe_layer_forward_ex(xin, W["wg"], W["bias"], W["w1"], W["w3"], W["w2"], W.get("w1s"), W.get("w3s"),
                                     W.get("w2s"), fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, o, ws, events)

    for _ in range(max(3, args.warmup)):
        fwd(x, out)
    torch.cuda.synchronize()
    rc = moe.moe_get_error()
    if rc != 0:
        raise RuntimeError(f"device error after warm-up: {moe.strerror(rc)}")

    K = args.steps
    ev_names = moe.STAGES + (["gemm1", "gemm2"] if a8 else [])
    evs = [{n: torch.cuda.Event(enable_timing=True) for n in ev_names} for _ in range(K)]
    for e in evs:               # torch creates the CUDA event on its first record
        for ev in e.values():
            ev.record()
    flush = L2Flush(dev) if working_set_bytes(wl, 1 if fp8 else 2) < L2_BYTES else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        total_ms = timed_steps(lambda e: fwd(x, out, e), evs, flush)
    if world > 1:
        dist.barrier()
    l2 = l2_note(wl, flush, 1 if fp8 else 2)
    del flush
    stage_ms = {}
    for a, b in zip(moe.STAGES[:-1], moe.STAGES[1:]):
        stage_ms[a] = float(np.mean([e[a].elapsed_time(e[b]) for e in evs]))
    # the grouped GEMM kernels alone (fp8 activations: the stages also hold the row quantisers)
    gemm_ms = {"gate_up": stage_ms["gate_up"], "down": stage_ms["down"]}
    if a8:
        gemm_ms = {"gate_up": float(np.mean([e["gemm1"].elapsed_time(e["down"]) for e in evs])),
                   "down": float(np.mean([e["gemm2"].elapsed_time(e["combine"]) for e in evs]))}
        stage_ms["quant_x"] = float(np.mean([e["gate_up"].elapsed_time(e["gemm1"]) for e in evs]))
        stage_ms["quant_h"] = float(np.mean([e["down"].elapsed_time(e["gemm2"]) for e in evs]))
    total_ms = dp.max_over_ranks(total_ms, device=dev)
    value = dp.job_throughput(T, world, K, total_ms)

    # kept rows and touched experts of the (deterministic) routing
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    counts = moe.workspace_view(ws, L, "counts", (E,), torch.int32).cpu().numpy()
    craw = moe.workspace_view(ws, L, "counts_raw", (E,), torch.int32).cpu().numpy()
    N = int(counts.sum())
    touched = int((counts > 0).sum())

    # end to end through the public API: every step copies its batch from pinned host memory to
    # the device and its output back, in the library's host-buffer pipeline (the copies of the
    # neighbouring batches overlap the layer); timed from the first copy in to the last copy out
    x_pin = x_host.pin_memory()
    out_pin = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
    if fp8:
        routed = {n: W[w] for n, w in (("W1q", "w1q"), ("W3q", "w3q"), ("W2q", "w2q"), ("s1", "s1"), ("s3", "s3"),
                                       ("s2", "s2"))}
        shared = {n: W[w] for n, w in (("W1q", "w1sq"), ("W3q", "w3sq"), ("W2q", "w2sq"), ("s1", "s1s"),
                                       ("s3", "s3s"), ("s2", "s2s"))} if fs else None
        pmem = torch.empty(moe.moe_pipeline_bytes_w8(T, d, E, k, f, fs, a8), dtype=torch.uint8, device=dev)
        pl = moe.Pipeline(W["wg"], W["bias"], None, None, None, None, None, None, fs, T, d, E, k, f,
                          wl.capacity_factor, wl.cap_mode, pmem, routed=routed, shared=shared, activations_fp8=a8)
    else:
        pmem = torch.empty(moe.moe_pipeline_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device=dev)
        pl = moe.Pipeline(W["wg"], W["bias"], W["w1"], W["w3"], W["w2"], W.get("w1s"), W.get("w3s"), W.get("w2s"),
                          fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, pmem)
    s_h2d, _, s_d2h = pl.streams()
    for _ in range(3):
        pl.submit(x_pin, out_pin)
    pl.sync()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(torch.cuda.ExternalStream(s_h2d))
    for _ in range(K):
        pl.submit(x_pin, out_pin)
    e1.record(torch.cuda.ExternalStream(s_d2h))
    pl.sync()
    torch.cuda.synchronize()
    pl.close()
    e2e_ms = dp.max_over_ranks(e0.elapsed_time(e1), device=dev)
    if world > 1:
        dist.barrier()
    e2e_value = dp.job_throughput(T, world, K, e2e_ms)
    rc = moe.moe_get_error()
    if rc != 0:
        raise RuntimeError(f"device error: {moe.strerror(rc)}")

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    peaks, peak_src = load_peaks()
    roof, layer = roofline_and_layer(wl, N, touched, counts, craw, gemm_ms, total_ms / K, fp8, a8, peaks,
                                     peak_src)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("fp8 e4m3 activations and expert weights (per-row scales), bf16 in/out" if a8 else
                  "bf16 activations, fp8 e4m3 expert weights" if fp8 else "bf16"),
        "data": "synthetic (seeded Philox4x32-10 + Box-Muller; random-init weights)",
        "config": {"workload": DESCR[wl.name], "global_batch": world * T, "seq_len": T, "parallelism": f"dp{world}",
                   "l2": l2},
        "roofline": roof,
        "layer": layer,
        "stages_ms": stage_ms,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * d * 2,
                "d2h_bytes_per_step": T * d * 2},
        "gemm_ms": gemm_ms,
        "gpu_launches": launches_per_step(a8, wl.has_shared) * K,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    if world == 1 and args.weights == "bf16" and not args.no_per_config and wl.name in synth.WORKLOAD_ORDER:
        # every workload of the task in the same run, one after the other on this GPU
        del W, tensors, x, ws, out, pmem
        torch.cuda.empty_cache()
        per = {}
        for name in synth.WORKLOAD_ORDER:
            if name == wl.name:
                per[name] = config_entry(wl, value, total_ms / K, K, roof, layer, stage_ms, gemm_ms, line["clocks"],
                                         line.get("cpu_baseline"), l2)
            else:
                per[name] = measure_config(name, dev, 3, peaks, peak_src,
                                           0.0 if args.no_cpu_baseline else min(args.cpu_seconds, 6.0))
        line["per_config"] = per
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
