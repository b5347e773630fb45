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


def test_forward_wait_runs_out(case):
    import torch
    dev, (O, L), _ = case
    q, k, v = dev["q"], dev["k"], dev["v"]
    ws = fa.new_workspace(fa.fa_fwd_workspace_size(), "cuda")
    dt = _stalled(fa.FA_STALL_FWD, lambda: fa.forward(q, k, v, SCALE, True, workspace=ws))
    assert dt < 1.0
    # a launch while the word is still set does nothing: O keeps its poison
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, HQ, N), float("nan"), device="cuda")
    fa.forward(q, k, v, SCALE, True, out=o, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isnan(o).all() and torch.isnan(lse).all()
    assert fa.device_error(ws) == fa.FA_ERR_TIMEOUT
    assert fa.device_error(ws) == fa.FA_OK          # read and cleared
    _context_usable()
    o, lse = fa.forward(q, k, v, SCALE, True, workspace=ws)
    torch.cuda.synchronize()
    assert fa.device_error(ws) == fa.FA_OK
    assert_close_bf16("O", to_np(o), O)
    assert lse_err(to_np(lse), L) <= LSE_MAX_ABS


@pytest.mark.parametrize("which", ["main", "dq"])
def test_backward_wait_runs_out(case, which):
    import torch
    dev, _, (dQ, dK, dV) = case
    q, k, v, do = dev["q"], dev["k"], dev["v"], dev["do"]
    o, lse = fa.forward(q, k, v, SCALE, True)
    ws = fa.new_workspace(fa.fa_bwd_workspace_size(B, HQ, N, D), "cuda")
    det = which == "dq"
    kernels = fa.FA_STALL_DQ if det else fa.FA_STALL_BWD
    dt = _stalled(kernels, lambda: fa.backward(q, k, v, o, do, lse, SCALE, True, workspace=ws,
                                               deterministic=det))
    assert dt < 1.0
    assert fa.device_error(ws) == fa.FA_ERR_TIMEOUT
    assert fa.device_error(ws) == fa.FA_OK
    _context_usable()
    dq, dk, dv = fa.backward(q, k, v, o, do, lse, SCALE, True, workspace=ws, deterministic=det)
    torch.cuda.synchronize()
    assert fa.device_error(ws) == fa.FA_OK
    assert_close_bf16("dQ", to_np(dq), dQ)
    assert_close_bf16("dK", to_np(dk), dK)
    assert_close_bf16("dV", to_np(dv), dV)
