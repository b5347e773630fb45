"""GPU test of the bounded-wait contract of the tensor-core kernels.

A kernel whose wait runs out must record FA_ERR_TIMEOUT in the workspace's
error word and return without faulting; the CUDA context stays usable;
launches made while the word is set do no work; and once fa_get_device_error
has cleared the word the next call on the same workspace is correct.

The wait is made to run out with the library's test hook fa_debug_set_stall:
the chosen kernel's MMA-issuing thread first waits, with a limit of a few
milliseconds, on a barrier that nothing signals. Nothing traps, faults or
hangs; the abort path that follows is the one a real stall would take.
"""
import time

import numpy as np
import pytest

from _helpers import LSE_MAX_ABS, assert_close_bf16, lse_err, to_dev, to_np
from exact_io_aware_45_b200 import fa, inputs
from oracle import attention as orc

pytestmark = pytest.mark.gpu

STALL_CYCLES = 4_000_000   # about 2 ms of SM clock
B, HQ, HKV, N, D = 1, 4, 2, 640, 128
SCALE = 1.0 / np.sqrt(D)


@pytest.fixture(autouse=True)
def _hook_off():
    import torch
    assert torch.cuda.is_available(), "GPU tests need CUDA"
    fa.lib()
    fa.fa_debug_set_stall(0, 0)
    yield
    fa.fa_debug_set_stall(0, 0)


@pytest.fixture(scope="module")
def case():
    import torch
    x = inputs.random_case(B, HQ, HKV, N, D, seed=31)
    dev = {n: to_dev(x[n], torch.bfloat16) for n in ("q", "k", "v", "do")}
    O, L = orc.forward(x["q"], x["k"], x["v"], SCALE, True)
    grads = orc.backward(x["q"], x["k"], x["v"], x["do"], SCALE, True, O=O)
    return dev, (O, L), grads


def _context_usable():
    import torch
    a = torch.arange(1000, device="cuda", dtype=torch.float32)
    assert float(a.sum().item()) == 499500.0
    torch.cuda.synchronize()


def _stalled(kernels, fn):
    """Runs fn() with the hook on for `kernels`; returns its wall time."""
    import torch
    torch.cuda.synchronize()
    assert fa.fa_debug_set_stall(kernels, STALL_CYCLES) == fa.FA_OK
    try:
        t0 = time.perf_counter()
        fn()
        torch.cuda.synchronize()
        return time.perf_counter() - t0
    finally:
        fa.fa_debug_set_stall(0, 0)


# Every form of the tensor-core forward, each with its own MMA-issue loop and
# abort path: form -> (B, Hq, Hkv, N, d, causal, left window edge (-1: none),
# block-mask density (None: no mask))
FWD_FORMS = {
    "persistent-d128": (1, 4, 2, 640, 128, True, -1, None),
    "persistent-d64": (1, 4, 2, 640, 64, True, -1, None),
    "one-item": (1, 2, 1, 4300, 128, True, -1, None),   # above the persistent form's 4096 keys
    "skipping": (1, 4, 2, 640, 128, True, 200, None),    # a left window edge
    "split": (1, 4, 2, 640, 64, False, -1, 0.5),         # a block mask
}


@pytest.mark.parametrize("form", list(FWD_FORMS))
def test_forward_wait_runs_out(form):
    import torch
    b, hq, hkv, n, d, causal, wl, density = FWD_FORMS[form]
    x = inputs.random_case(b, hq, hkv, n, d, seed=41 + n + d)
    q, k, v = (to_dev(x[name], torch.bfloat16) for name in ("q", "k", "v"))
    scale = 1.0 / np.sqrt(d)
    mask_np = inputs.random_block_mask(n, density, 5) if density else None
    mask = torch.from_numpy(mask_np).to("cuda") if density else None
    mods = fa.mods(window_left=wl)
    ws = fa.new_workspace(fa.fa_fwd_workspace_size(), "cuda")

    def run(o=None, lse=None):
        return fa.forward_mod(q, k, v, mods, scale, causal, mask, workspace=ws, out=o, lse=lse)

    dt = _stalled(fa.FA_STALL_FWD, run)
    assert dt < 1.0
    # a launch while the word is still set does nothing: O keeps its poison
    o = torch.full_like(q, float("nan"))
    lse = torch.full((b, hq, n), float("nan"), device="cuda")
    run(o, lse)
    torch.cuda.synchronize()
    assert torch.isnan(o).all() and torch.isnan(lse).all()
    assert fa.device_error(ws) == fa.FA_ERR_TIMEOUT
    assert fa.device_error(ws) == fa.FA_OK          # read and cleared
    _context_usable()
    o, lse = run()
    torch.cuda.synchronize()
    assert fa.device_error(ws) == fa.FA_OK
    O, L = orc.forward(x["q"], x["k"], x["v"], scale, causal, mask_np,
                       (wl, -1) if wl >= 0 else None)
    assert_close_bf16("O", to_np(o), O)
    assert lse_err(to_np(lse), L) <= LSE_MAX_ABS


@pytest.mark.parametrize("which,d", [("main", 128), ("dq", 128), ("main", 64)])
def test_backward_wait_runs_out(case, which, d):
    """The main backward kernel (its d = 128 and d = 64 schedules differ) and
    the deterministic path's dQ kernel."""
    import torch
    if d == D:
        dev, _, (dQ, dK, dV) = case
    else:
        x = inputs.random_case(B, HQ, HKV, N, d, seed=32)
        dev = {n: to_dev(x[n], torch.bfloat16) for n in ("q", "k", "v", "do")}
        O, _ = orc.forward(x["q"], x["k"], x["v"], 1.0 / np.sqrt(d), True)
        dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], 1.0 / np.sqrt(d), True, O=O)
    scale = 1.0 / np.sqrt(d)
    q, k, v, do = dev["q"], dev["k"], dev["v"], dev["do"]
    o, lse = fa.forward(q, k, v, scale, True)
    ws = fa.new_workspace(fa.fa_bwd_workspace_size(B, HQ, N, d), "cuda")
    det = which == "dq"
    kernels = fa.FA_STALL_DQ if det else fa.FA_STALL_BWD
    dt = _stalled(kernels, lambda: fa.backward(q, k, v, o, do, lse, scale, True, workspace=ws,
                                               deterministic=det))
    assert dt < 1.0
    assert fa.device_error(ws) == fa.FA_ERR_TIMEOUT
    assert fa.device_error(ws) == fa.FA_OK
    _context_usable()
    dq, dk, dv = fa.backward(q, k, v, o, do, lse, scale, True, workspace=ws, deterministic=det)
    torch.cuda.synchronize()
    assert fa.device_error(ws) == fa.FA_OK
    assert_close_bf16("dQ", to_np(dq), dQ)
    assert_close_bf16("dK", to_np(dk), dK)
    assert_close_bf16("dV", to_np(dv), dV)
