"""Sliding-window (local) attention: key j visible to query i iff
i - left <= j <= i + right (a negative bound: unbounded), on top of the causal
flag and the block mask (the lesson's FlexAttention note: one tiled kernel,
many masks).

CPU tests pin the oracle's window against the causal flag, a brute-force
softmax over each row's window written with math.exp, the one-key closed
form and central finite differences; GPU tests compare fa_fwd_window /
fa_bwd_window with the oracle on seeded cases whose windows cut tiles in
every way (left only, right only, both, with causal, GQA, block mask), and
the (unbounded, 0) window with the causal kernel bit for bit."""
import math

import numpy as np
import pytest

from _helpers import LSE_MAX_ABS, assert_close_bf16, lse_err, to_dev, to_np
from exact_io_aware_45_b200 import fa, inputs
from oracle import attention as orc


# ------------------------------------------------------------------ oracle pins (CPU)

def test_window_right_zero_is_causal():
    x = inputs.random_case(1, 2, 1, 70, 8, seed=1)
    O1, L1 = orc.forward(x["q"], x["k"], x["v"], 0.4, False, None, (-1, 0))
    O2, L2 = orc.forward(x["q"], x["k"], x["v"], 0.4, True)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


@pytest.mark.parametrize("window,causal", [((5, -1), False), ((-1, 3), False), ((4, 2), False),
                                           ((6, -1), True)])
def test_window_brute_force(window, causal):
    x = inputs.random_case(1, 1, 1, 23, 4, seed=2)
    scale = 0.7
    O, L = orc.forward(x["q"], x["k"], x["v"], scale, causal, None, window)
    q, k, v = (x[n][0, 0].astype(np.float64) for n in ("q", "k", "v"))
    left, right = window
    for i in range(23):
        js = [j for j in range(23) if (left < 0 or j >= i - left) and (right < 0 or j <= i + right)
              and (not causal or j <= i)]
        s = [scale * float(np.dot(q[i], k[j])) for j in js]
        m = max(s)
        e = [math.exp(t - m) for t in s]
        z = sum(e)
        o = sum(ej * v[j] for ej, j in zip(e, js)) / z
        assert np.allclose(O[0, 0, i], o, atol=1e-12)
        assert abs(L[0, 0, i] - (m + math.log(z))) < 1e-12


def test_window_zero_sees_only_itself():
    x = inputs.random_case(1, 2, 2, 16, 8, seed=3)
    O, L = orc.forward(x["q"], x["k"], x["v"], 0.5, False, None, (0, 0))
    assert np.allclose(O, x["v"], atol=1e-12)
    qk = np.einsum("bhnd,bhnd->bhn", x["q"].astype(np.float64), x["k"].astype(np.float64))
    assert np.allclose(L, 0.5 * qk, atol=1e-12)


def test_window_backward_finite_differences():
    rng = np.random.default_rng(4)
    B, H, N, d = 1, 1, 12, 4
    Q, K, V, dO = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    win = (3, 1)
    dQ, dK, dV = orc.backward(Q, K, V, dO, 0.6, False, None, window=win)
    loss = lambda Q_, K_, V_: float(np.sum(orc.forward(Q_, K_, V_, 0.6, False, None, win)[0] * dO))  # noqa: E731
    eps = 1e-6
    for name, X, G in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += eps
            Xm[idx] -= eps
            args = {"Q": (Q, K, V), "K": (Q, K, V), "V": (Q, K, V)}[name]
            ap = [Xp if a is X else a for a in args]
            am = [Xm if a is X else a for a in args]
            num[idx] = (loss(*ap) - loss(*am)) / (2 * eps)
        assert np.allclose(num, G, rtol=1e-6, atol=1e-8), name


def test_window_argument_checks():
    G = 0x10000
    args = [G, G, G, G, G, 1, 2, 1, 64, 64, 0.125, 0, -2, -1, 0, fa.FA_BF16, G, 0]
    assert fa.fa_fwd_window(*args) == fa.FA_ERR_INVALID_ARG
    args[12], args[13] = 4, -1
    args[15] = fa.FA_F32
    assert fa.fa_fwd_window(*args) == fa.FA_ERR_UNSUPPORTED


# ------------------------------------------------------------------ GPU parity

CASES = [
    # B, Hq, Hkv, N, d, causal, window, mask density
    (1, 2, 1, 700, 128, False, (200, -1), None),
    (1, 2, 2, 700, 64, False, (-1, 150), None),
    (2, 4, 2, 513, 128, False, (100, 60), None),
    (1, 4, 1, 900, 128, True, (300, -1), None),
    (1, 2, 2, 1024, 64, False, (257, 257), 0.5),
    (1, 2, 1, 300, 128, True, (0, -1), None),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: "N{}d{}{}w{}_{}{}".format(
    c[3], c[4], "c" if c[5] else "", c[6][0], c[6][1], "m" if c[7] else ""))
def test_window_matches_oracle(case):
    import torch
    B, Hq, Hkv, N, d, causal, win, dens = case
    x = inputs.random_case(B, Hq, Hkv, N, d, seed=N + d, mask_density=dens)
    scale = 1.0 / np.sqrt(d)
    bf = torch.bfloat16
    q, k, v, do = (to_dev(x[n], bf) for n in ("q", "k", "v", "do"))
    mask = None if x["mask"] is None else torch.from_numpy(x["mask"]).cuda()
    o, lse = fa.forward_window(q, k, v, win[0], win[1], scale, causal, mask)
    g = fa.backward_window(q, k, v, o, do, lse, win[0], win[1], scale, causal, mask)
    torch.cuda.synchronize()
    O, L = orc.forward(x["q"], x["k"], x["v"], scale, causal, x["mask"], win)
    G = orc.backward(x["q"], x["k"], x["v"], x["do"], scale, causal, x["mask"], O=O, window=win)
    assert_close_bf16("O", to_np(o), O)
    assert lse_err(to_np(lse), L) <= LSE_MAX_ABS
    for name, got, want in zip(("dQ", "dK", "dV"), g, G):
        assert_close_bf16(name, to_np(got), want)


@pytest.mark.gpu
def test_window_unbounded_left_zero_right_is_causal_kernel():
    import torch
    x = inputs.random_case(1, 4, 2, 640, 128, seed=9)
    bf = torch.bfloat16
    q, k, v = (to_dev(x[n], bf) for n in ("q", "k", "v"))
    o1, l1 = fa.forward_window(q, k, v, -1, 0, None, False)
    o2, l2 = fa.forward(q, k, v, None, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
