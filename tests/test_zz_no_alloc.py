"""GPU test of fa_bwd_noalloc, the backward entry point for callers that
cannot allocate device memory (no workspace; its scratch is a fixed array in
the library). Called through the C ABI and compared with fa_bwd on the same
inputs, twice in a row (the second call runs on the array the first one left
behind). Kept in its own file so that it is collected last."""
import ctypes

import numpy as np
import pytest

from _helpers import BF16_MAX_ABS, BF16_REL_FRO, max_abs, rel_fro, to_dev, to_np
from exact_io_aware_45_b200 import fa, inputs

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    L = fa.lib()
    f = L.fa_bwd_noalloc
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    f.argtypes = [P] * 9 + [I, I, I, I, I, F, I, P, I, P, P]
    f.restype = I
    return f


@pytest.mark.parametrize("case", [
    # B, Hq, Hkv, N, d, causal, mask density, input dtype
    (2, 4, 2, 300, 64, True, None, "bf16"),      # tensor-core kernels
    (1, 2, 1, 640, 128, False, 0.5, "bf16"),     # tensor-core kernels, block mask
    (1, 2, 1, 200, 32, True, None, "f32"),       # CUDA-core kernels, fp32 inputs
    (1, 4, 2, 257, 32, False, 0.5, "bf16"),      # CUDA-core kernels (d = 32), bf16 inputs
])
def test_bwd_noalloc_matches_fa_bwd(case):
    import torch
    B, Hq, Hkv, N, d, causal, dens, dt_name = case
    dt = torch.bfloat16 if dt_name == "bf16" else torch.float32
    x = inputs.random_case(B, Hq, Hkv, N, d, seed=21 + N, mask_density=dens, dtype=dt_name)
    q, k, v, do = (to_dev(x[n], dt) for n in ("q", "k", "v", "do"))
    mask = None if x["mask"] is None else torch.from_numpy(x["mask"]).cuda()
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.forward(q, k, v, scale, causal, mask)
    ref = fa.backward(q, k, v, o, do, lse, scale, causal, mask, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    f = _noalloc_fn()
    err_word = torch.zeros(4, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    P = lambda t: 0 if t is None else t.data_ptr()  # noqa: E731
    for call in range(2):
        dq = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        dk = torch.full(k.shape, float("nan"), dtype=torch.float32, device="cuda")
        dv = torch.full(v.shape, float("nan"), dtype=torch.float32, device="cuda")
        s = f(P(q), P(k), P(v), P(o), P(do), P(lse), P(dq), P(dk), P(dv), B, Hq, Hkv, N, d,
              float(scale), int(causal), P(mask), fa.FA_BF16 if dt_name == "bf16" else fa.FA_F32,
              P(err_word) if call == 0 else 0, stream)
        assert s == fa.FA_OK, fa.status_string(s)
        torch.cuda.synchronize()
        for name, got, want in (("dQ", dq, ref[0]), ("dK", dk, ref[1]), ("dV", dv, ref[2])):
            g, w = to_np(got), to_np(want)
            assert np.isfinite(g).all(), f"call {call}: {name} not fully written"
            ma, rf = max_abs(g, w), rel_fro(g, w)
            assert ma <= BF16_MAX_ABS and rf <= BF16_REL_FRO, f"call {call} {name}: {ma} {rf}"
    assert int(err_word[0].item()) == 0


def test_bwd_noalloc_rejects_oversize():
    """More rows than the fixed array holds: refused before any launch."""
    f = _noalloc_fn()
    good = 1 << 20  # fake aligned pointers; never dereferenced
    s = f(good, good, good, good, good, good, good, good, good, 1, 64, 64, 16384 + 1, 64, 0.125,
          0, 0, fa.FA_BF16, 0, 0)
    assert s == fa.FA_ERR_UNSUPPORTED
