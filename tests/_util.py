"""Test helpers: bf16 bit patterns <-> torch tensors, tolerances."""
import numpy as np
import torch


def to_dev_bf16(a: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 on device."""
    a = np.ascontiguousarray(a, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """torch.bfloat16 (any device) -> uint16 bit patterns (numpy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(a: np.ndarray) -> np.ndarray:
    return (np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_layer_close(gpu_bits: np.ndarray, ref_bits: np.ndarray, what: str = "out"):
    """The layer-output bar: |gpu - oracle| <= 1e-2 + 2e-2 |oracle| per element."""
    g, r = bits_to_f64(gpu_bits), bits_to_f64(ref_bits)
    bad = np.abs(g - r) > 1e-2 + 2e-2 * np.abs(r)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} elements outside 1e-2 + 2e-2|ref|; " \
                          f"max |d| = {np.abs(g - r).max():.3e}"


def ulp_bf16(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    def key(x):
        x = np.asarray(x, dtype=np.uint16).astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x & 0x7FFF)
    return np.abs(key(a) - key(b))


def logits_tol(x_bits: np.ndarray, wg_bits: np.ndarray) -> np.ndarray:
    """Per-element bound for fp32 tensor-core logits vs the double-sum oracle:
    16 * 2^-24 * sum_i |x_i w_i| + 1e-6 (fp32 partial sums over d/16 K-steps)."""
    ax = np.abs(bits_to_f64(x_bits))
    aw = np.abs(bits_to_f64(wg_bits))
    return 16 * 2.0 ** -24 * (ax @ aw.T) + 1e-6
