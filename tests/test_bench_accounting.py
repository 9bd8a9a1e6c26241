"""The work and launch accounting behind bench.py's roofline line, against closed forms written
from the layer's shapes (CPU only)."""
import bench
import synth


def test_gemm1_flops_and_both_gemms():
    wl = synth.WORKLOADS["mixtral"]
    N = wl.T * wl.k
    assert bench.gemm1_work(wl, N) == 4.0 * 8192 * 4096 * 14336
    assert bench.gemms_work(wl, N) == 6.0 * 8192 * 4096 * 14336
    ds = synth.WORKLOADS["dsv3"]
    assert bench.gemms_work(ds, 2048) == 6.0 * 2048 * 7168 * 2048 + 6.0 * 256 * 7168 * 2048


def test_decode_gemm1_bytes():
    wl = synth.WORKLOADS["dsv3"]
    N, touched = 2048, 256
    d, f, fs, T = 7168, 2048, 2048, 256
    bf16 = touched * 2 * f * d * 2 + N * d * 2 + N * f * 2 + 2 * fs * d * 2 + T * d * 2 + T * fs * 2
    assert bench.gemm1_bytes(wl, N, touched) == bf16
    # fp8 weights (+ fp32 row scales) with bf16 activations
    w8 = touched * 2 * f * d + touched * 2 * f * 4 + N * d * 2 + N * f * 2 + 2 * fs * d + 2 * fs * 4 \
        + T * d * 2 + T * fs * 2
    assert bench.gemm1_bytes(wl, N, touched, 1) == w8
    # fp8 weights and fp8 activation rows (+ one fp32 scale per row)
    a8 = touched * 2 * f * d + touched * 2 * f * 4 + N * d + N * 4 + N * f * 2 + 2 * fs * d + 2 * fs * 4 \
        + T * d + T * 4 + T * fs * 2
    assert bench.gemm1_bytes(wl, N, touched, 1, 1) == a8
    assert abs(bf16 / 1e9 - 15.13) < 0.01          # the figure the DRAM captures are read against


def test_layer_flops_follow_the_scope_formula():
    wl = synth.WORKLOADS["qwen3"]
    N = wl.T * wl.k
    flops, _ = bench.layer_work(wl, N, wl.E)
    assert flops == 6.0 * wl.d * wl.f * N + 2.0 * wl.T * wl.d * wl.E


def test_launches_per_step():
    # router GEMM, top-k, count, scan, scatter, gather, GEMM1, GEMM2, combine
    assert bench.launches_per_step(False, False) == 9
    assert bench.launches_per_step(False, True) == 9
    # fp8 activations: no gather; x quantiser (routed + shared rows in one), h quantiser, shared h
    assert bench.launches_per_step(True, False) == 10      # 70 launches over 7 layer steps in the ncu list
    assert bench.launches_per_step(True, True) == 11


class _Ev:
    """Stand-in for a timed CUDA event: a timestamp in ms."""

    def __init__(self, t):
        self.t = t

    def elapsed_time(self, other):
        return other.t - self.t


def test_timed_steps_keeps_l2_flushes_outside_the_timed_steps():
    # step i runs from 10 i to 10 i + 3 (ms); a flush, when asked for, sits in the gaps
    evs = [{"route": _Ev(10.0 * i), "end": _Ev(10.0 * i + 3.0)} for i in range(4)]
    calls = []
    ran = []
    t = bench.timed_steps(lambda e: ran.append(e), evs, lambda: calls.append(1), sync=lambda: None)
    assert t == 4 * 3.0 and len(calls) == 4 and ran == evs
    # without a flush: the span from the first start to the last end
    assert bench.timed_steps(lambda e: None, evs, None, sync=lambda: None) == 33.0


def test_only_workloads_smaller_than_l2_are_flushed():
    import synth
    small = [n for n in ("tiny", "mixtral", "qwen3", "dsv3", "skew")
             if bench.working_set_bytes(synth.WORKLOADS[n]) < bench.L2_BYTES]
    assert small == ["tiny"]
    # the weights alone bound the estimate from below
    wl = synth.WORKLOADS["mixtral"]
    assert bench.working_set_bytes(wl) >= 3.0 * wl.E * wl.f * wl.d * 2
