"""The FMA-pipe exponential the forward kernel uses for part of its softmax
terms: its constants come from the fit script beside the kernels, its float32
steps (modelled in NumPy) meet the stated bound, and the device version,
called through the C ABI, meets the same bound against fp64 exp2."""
import importlib.util
import os
import re

import numpy as np
import pytest

from exact_io_aware_45_b200 import fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_io_aware_45_b200", "csrc")
REL_BOUND = 1e-4   # relative error of the cubic on |f| <= 1/2 is 7.7e-5


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit",
                                                  os.path.join(CSRC, "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_constants():
    text = open(os.path.join(CSRC, "sm100_common.cuh")).read()
    vals = dict(re.findall(r"(kExp2P[0-3]) = ([-+0-9.e]+)f", text))
    return np.array([float(vals[f"kExp2P{i}"]) for i in range(4)], dtype=np.float32)


def test_kernel_constants_are_the_fit():
    fit = _fit_module().fit()
    assert np.array_equal(_kernel_constants(), fit)


def test_float32_model_meets_bound():
    m = _fit_module()
    c = _kernel_constants()
    x = np.concatenate([np.linspace(-125.0, 64.0, 1_000_001, dtype=np.float32),
                        np.float32([-125.0, -0.5, 0.5, 0.0, 1.0, -1.0, 8.0])])
    got = m.eval_f32(x, c).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= REL_BOUND
    # below the clamp the result is 2^-125 (within the same bound)
    low = m.eval_f32(np.float32([-126.0, -300.0]), c).astype(np.float64)
    assert np.all(np.abs(low / 2.0 ** -125 - 1.0) <= REL_BOUND)


def test_abi_argument_checks():
    assert fa.fa_exp2_fma(0, 0, -1, 0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_exp2_fma(0, 0, 5, 0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_exp2_fma(0, 0, 0, 0) == fa.FA_OK


@pytest.mark.gpu
def test_device_exp2_meets_bound():
    import torch
    assert torch.cuda.is_available()
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.0, 64.0, 2_000_001, dtype=np.float32),
                        rng.uniform(-30.0, 8.0, 1_000_001).astype(np.float32),
                        np.float32([-126.0, -1e4])])
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    s = fa.fa_exp2_fma(xd.data_ptr(), yd.data_ptr(), x.size,
                       torch.cuda.current_stream().cuda_stream)
    assert s == fa.FA_OK
    torch.cuda.synchronize()
    y = yd.cpu().numpy().astype(np.float64)
    ref = np.exp2(np.maximum(x.astype(np.float64), -125.0))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= REL_BOUND, float(rel.max())
    # the device steps are the float32 model's steps
    model = _fit_module().eval_f32(x, _kernel_constants()).astype(np.float64)
    assert np.max(np.abs(y / model - 1.0)) <= 2 ** -22
