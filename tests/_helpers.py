"""Shared helpers of the GPU tests: moving seeded inputs to the device and the
error metrics the tolerances are stated in."""
import numpy as np

# tolerances (fixed by the workloads' statement of the target)
F32_O_MAX_ABS = 1e-4          # fp32 workload: max abs error on O
BF16_MAX_ABS = 2e-2           # bf16 inputs, fp32 accumulation: O, dQ, dK, dV
BF16_REL_FRO = 1e-2
LSE_MAX_ABS = 1e-3


def to_dev(x, dtype):
    """float32 numpy array (bf16-exact when dtype is bf16) -> CUDA tensor."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(device="cuda", dtype=dtype).contiguous()


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def max_abs(x, y):
    return float(np.max(np.abs(x - y))) if x.size else 0.0


def rel_fro(x, y):
    den = float(np.linalg.norm(y))
    return float(np.linalg.norm(x - y)) / den if den > 0 else float(np.linalg.norm(x - y))


def lse_err(got, want):
    """Max abs LSE difference; -inf entries must match exactly."""
    ninf_g, ninf_w = np.isneginf(got), np.isneginf(want)
    assert np.array_equal(ninf_g, ninf_w), "rows with no visible key differ"
    fin = ~ninf_w
    return max_abs(got[fin], want[fin])


def assert_close_bf16(name, got, want):
    ma, rf = max_abs(got, want), rel_fro(got, want)
    assert ma <= BF16_MAX_ABS and rf <= BF16_REL_FRO, f"{name}: max abs {ma:.3e} rel-F {rf:.3e}"
    return ma, rf
