"""Pins of the fp64 oracle against what the FlashAttention pages and the
mathematics fix (no GPU).

Each test is chosen so that a plausible slip in the oracle (a dropped scale, a
wrong sign, a transposed operand, a mask applied to the wrong index, a missing
sum over the heads of a KV group) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as orc
from exact_io_aware_45_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "numpy_lesson_fp32.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split(None, 1)
        vals[k] = v
    return vals


def _pages_inputs():
    w = inputs.WORKLOADS["fp32_n512_d32"]
    x = inputs.make_inputs(w)
    return x["q"][0, 0], x["k"][0, 0], x["v"][0, 0], w.scale


# ---------------------------------------------------------------- the pages' worked example

def test_pages_example_tiled_matches_naive_fp32():
    """The lesson's own run: tiled fp32 loop vs one-shot fp32 at atol 1e-5."""
    g = _golden()
    Q, K, V, scale = _pages_inputs()
    naive = orc.naive_forward_f32(Q, K, V, scale)
    tiled = orc.tiled_forward(Q, K, V, scale, block=128, dtype=np.float32)
    diff = float(np.abs(naive - tiled).max())
    assert np.allclose(naive, tiled, atol=float(g["atol"])) == (g["outputs_match"] == "True")
    # the printed difference is float32 rounding: same order of magnitude
    printed = float(g["largest_abs_difference"])
    assert diff <= float(g["atol"])
    assert printed / 30 <= diff <= printed * 30
    # score buffers held: N x N vs N x block float32 values
    N = Q.shape[0]
    assert N * N * 4 == int(g["naive_score_bytes"])
    assert N * 128 * 4 == int(g["tiled_score_bytes"])
    assert int(g["naive_score_bytes"]) // int(g["tiled_score_bytes"]) == int(g["ratio"])


def test_oracle_matches_pages_example_fp32():
    """The fp64 oracle agrees with the lesson's fp32 result within fp32 rounding."""
    Q, K, V, scale = _pages_inputs()
    O, L = orc.forward(Q[None, None], K[None, None], V[None, None], scale)
    naive = orc.naive_forward_f32(Q, K, V, scale)
    assert np.abs(O[0, 0] - naive).max() < 1e-5


@pytest.mark.parametrize("block", [16, 128, 512])
@pytest.mark.parametrize("N", [512, 300, 77])
def test_oracle_equals_online_softmax_loop_fp64(block, N):
    """Tile sizes the lesson suggests (one tile of 512, tiles of 16 where the
    correction fires often) and lengths that are not tile multiples: the
    running-max recurrence and the one-shot definition agree to fp64 rounding."""
    rng = np.random.default_rng(N + block)
    Q, K, V = (rng.standard_normal((N, 32)) * 2 for _ in range(3))
    trace = []
    tiled = orc.tiled_forward(Q, K, V, 0.3, block=block, trace=trace)
    O, _ = orc.forward(Q[None, None], K[None, None], V[None, None], 0.3)
    assert np.abs(O[0, 0] - tiled).max() < 1e-12
    if block == 16:
        assert sum(trace[1:]) > 0  # the correction step really fired


def test_single_tile_is_the_one_shot_result():
    """Block = N: the loop runs once, so its result equals the definition."""
    Q, K, V, scale = _pages_inputs()
    a = orc.tiled_forward(Q, K, V, scale, block=512)
    O, _ = orc.forward(Q[None, None], K[None, None], V[None, None], scale)
    assert np.abs(a - O[0, 0]).max() < 1e-14


# ---------------------------------------------------------------- closed forms of the definition

def test_softmax_rows_sum_to_one_and_shift():
    rng = np.random.default_rng(1)
    S = rng.standard_normal((50, 70)) * 5
    S[3, :10] = -np.inf
    P, lse = orc.softmax_rows(S)
    assert np.abs(P.sum(axis=1) - 1).max() < 1e-12
    assert np.all(P[3, :10] == 0)
    c = rng.standard_normal(50)[:, None] * 100
    P2, lse2 = orc.softmax_rows(S + c)
    assert np.abs(P2 - P).max() < 1e-12
    assert np.abs(lse2 - (lse + c[:, 0])).max() < 1e-9
    # LSE is log of the sum of exponentials, computed directly
    ref = np.log(np.exp(S[5]).sum())
    assert abs(lse[5] - ref) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_give_mean_of_values(causal):
    """Q = 0 makes every allowed score equal, so O_i is the mean of the
    visible V rows and LSE_i = ln(number of visible keys)."""
    rng = np.random.default_rng(2)
    N, d = 200, 8
    Q = np.zeros((1, 1, N, d))
    K = rng.standard_normal((1, 1, N, d))
    V = rng.standard_normal((1, 1, N, d))
    O, L = orc.forward(Q, K, V, 0.5, causal=causal)
    if causal:
        want = np.cumsum(V[0, 0], axis=0) / np.arange(1, N + 1)[:, None]
        assert np.abs(L[0, 0] - np.log(np.arange(1, N + 1))).max() < 1e-12
    else:
        want = np.broadcast_to(V[0, 0].mean(axis=0), (N, d))
        assert np.abs(L[0, 0] - np.log(N)).max() < 1e-12
    assert np.abs(O[0, 0] - want).max() < 1e-12


def test_constant_values_give_constant_output():
    rng = np.random.default_rng(3)
    N, d = 150, 16
    Q = rng.standard_normal((1, 2, N, d))
    K = rng.standard_normal((1, 2, N, d))
    V = np.full((1, 2, N, d), 1.75)
    for causal in (False, True):
        O, _ = orc.forward(Q, K, V, 0.25, causal=causal)
        assert np.abs(O - 1.75).max() < 1e-12


def test_causal_first_row():
    """Row 0 under the causal flag sees only key 0: O_0 = V_0 and
    LSE_0 = scale * q_0 . k_0."""
    rng = np.random.default_rng(4)
    Q, K, V = (rng.standard_normal((1, 1, 64, 8)) for _ in range(3))
    O, L = orc.forward(Q, K, V, 0.7, causal=True)
    assert np.abs(O[0, 0, 0] - V[0, 0, 0]).max() < 1e-14
    assert abs(L[0, 0, 0] - 0.7 * Q[0, 0, 0] @ K[0, 0, 0]) < 1e-13


def _brute_force_row(q, K, V, scale, keys):
    """Softmax over an explicit list of keys with math.exp, one row."""
    s = [scale * float(np.dot(q, K[j])) for j in keys]
    mx = max(s)
    e = [math.exp(x - mx) for x in s]
    tot = sum(e)
    o = sum(ei * V[j] for ei, j in zip(e, keys)) / tot
    return o, mx + math.log(tot)


@pytest.mark.parametrize("causal", [False, True])
def test_block_mask_against_brute_force(causal):
    """A 3x3 block mask with blocks off: every row equals a softmax over
    exactly the keys the mask (and causal flag) leave visible."""
    rng = np.random.default_rng(5)
    N, d = 300, 4
    Q, K, V = (rng.standard_normal((1, 1, N, d)) for _ in range(3))
    mask = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 1]], dtype=np.uint8)
    O, L = orc.forward(Q, K, V, 0.9, causal=causal, block_mask=mask)
    for i in range(0, N, 7):
        keys = [j for j in range(N) if mask[i // 128, j // 128] and (not causal or j <= i)]
        o, lse = _brute_force_row(Q[0, 0, i], K[0, 0], V[0, 0], 0.9, keys)
        assert np.abs(O[0, 0, i] - o).max() < 1e-12
        assert abs(L[0, 0, i] - lse) < 1e-12


def test_all_ones_mask_is_no_mask():
    rng = np.random.default_rng(6)
    N = 260
    Q, K, V = (rng.standard_normal((1, 1, N, 8)) for _ in range(3))
    ones = np.ones((3, 3), dtype=np.uint8)
    for causal in (False, True):
        a = orc.forward(Q, K, V, 0.5, causal=causal)
        b = orc.forward(Q, K, V, 0.5, causal=causal, block_mask=ones)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_masked_block_contributes_nothing():
    """Turning one block off changes exactly the rows of that block row, and
    they equal attention over the remaining keys."""
    rng = np.random.default_rng(7)
    N = 384
    Q, K, V = (rng.standard_normal((1, 1, N, 8)) for _ in range(3))
    full = np.ones((3, 3), dtype=np.uint8)
    off = full.copy()
    off[1, 2] = 0
    a, _ = orc.forward(Q, K, V, 0.5, block_mask=full)
    b, _ = orc.forward(Q, K, V, 0.5, block_mask=off)
    assert np.array_equal(a[0, 0, :128], b[0, 0, :128])
    assert np.array_equal(a[0, 0, 256:], b[0, 0, 256:])
    sub, _ = orc.forward(Q[:, :, 128:256], K[:, :, :256], V[:, :, :256], 0.5)
    assert np.abs(b[0, 0, 128:256] - sub[0, 0]).max() < 1e-12


def test_empty_row_is_zero():
    """A block row with no visible block: O = 0, LSE = -inf, zero gradients."""
    rng = np.random.default_rng(8)
    N = 256
    Q, K, V, dO = (rng.standard_normal((1, 1, N, 8)) for _ in range(4))
    mask = np.array([[1, 1], [0, 0]], dtype=np.uint8)
    O, L = orc.forward(Q, K, V, 0.5, block_mask=mask)
    assert np.all(O[0, 0, 128:] == 0) and np.all(np.isneginf(L[0, 0, 128:]))
    dQ, dK, dV = orc.backward(Q, K, V, dO, 0.5, block_mask=mask)
    assert np.all(dQ[0, 0, 128:] == 0)
    # the empty rows send nothing to any key: changing their Q and dO leaves
    # dK and dV unchanged
    Q2, dO2 = Q.copy(), dO.copy()
    Q2[0, 0, 128:] = rng.standard_normal((128, 8)) * 3
    dO2[0, 0, 128:] = rng.standard_normal((128, 8)) * 3
    _, dK2, dV2 = orc.backward(Q2, K, V, dO2, 0.5, block_mask=mask)
    assert np.abs(dK - dK2).max() < 1e-12 and np.abs(dV - dV2).max() < 1e-12


# ---------------------------------------------------------------- GQA

def test_gqa_equals_repeated_heads():
    rng = np.random.default_rng(9)
    B, Hq, Hkv, N, d = 2, 6, 2, 40, 8
    Q = rng.standard_normal((B, Hq, N, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    dO = rng.standard_normal((B, Hq, N, d))
    g = Hq // Hkv
    Kr, Vr = np.repeat(K, g, axis=1), np.repeat(V, g, axis=1)
    for causal in (False, True):
        a = orc.forward(Q, K, V, 0.3, causal=causal)
        b = orc.forward(Q, Kr, Vr, 0.3, causal=causal)
        assert np.abs(a[0] - b[0]).max() < 1e-13
        ga = orc.backward(Q, K, V, dO, 0.3, causal=causal)
        gb = orc.backward(Q, Kr, Vr, dO, 0.3, causal=causal)
        assert np.abs(ga[0] - gb[0]).max() < 1e-12
        for x, y in ((ga[1], gb[1]), (ga[2], gb[2])):
            ysum = y.reshape(B, Hkv, g, N, d).sum(axis=2)
            assert np.abs(x - ysum).max() < 1e-12


# ---------------------------------------------------------------- backward

def _loss(Q, K, V, dO, scale, causal, mask):
    O, _ = orc.forward(Q, K, V, scale, causal, mask)
    return float(np.sum(O * dO))


@pytest.mark.parametrize("causal,N,d,Hq,Hkv,mask", [
    (False, 12, 5, 1, 1, None),
    (True, 16, 4, 2, 1, None),
    (False, 140, 2, 1, 1, np.array([[1, 0], [1, 1]], dtype=np.uint8)),
])
def test_backward_finite_differences(causal, N, d, Hq, Hkv, mask):
    """Central differences of L = sum(O * dO): gradient of every input element."""
    rng = np.random.default_rng(10 + N)
    Q = rng.standard_normal((1, Hq, N, d))
    K = rng.standard_normal((1, Hkv, N, d))
    V = rng.standard_normal((1, Hkv, N, d))
    dO = rng.standard_normal((1, Hq, N, d))
    scale = 0.6
    dQ, dK, dV = orc.backward(Q, K, V, dO, scale, causal, mask)
    h = 1e-6
    sel = rng.choice(Q.size, size=min(Q.size, 60), replace=False)
    for X, G in ((Q, dQ), (K, dK), (V, dV)):
        num = np.zeros(sel.size)
        for t, idx in enumerate(sel[sel < X.size]):
            old = X.flat[idx]
            X.flat[idx] = old + h
            lp = _loss(Q, K, V, dO, scale, causal, mask)
            X.flat[idx] = old - h
            lm = _loss(Q, K, V, dO, scale, causal, mask)
            X.flat[idx] = old
            num[t] = (lp - lm) / (2 * h)
        ana = G.flat[sel[sel < X.size]]
        num = num[:ana.size]
        assert np.abs(ana - num).max() <= 1e-6 * max(1.0, np.abs(num).max())


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_torch_autograd(causal):
    """An independent implementation: torch fp64 autograd of the naive formula."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, N, d = 1, 4, 2, 33, 8
    Q = rng.standard_normal((B, Hq, N, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    dO = rng.standard_normal((B, Hq, N, d))
    scale = 0.35
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    g = Hq // Hkv
    S = torch.einsum("bhnd,bhmd->bhnm", tq, tk.repeat_interleave(g, 1)) * scale
    if causal:
        S = S.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    O = torch.softmax(S, dim=-1) @ tv.repeat_interleave(g, 1)
    O.backward(torch.tensor(dO))
    dQ, dK, dV = orc.backward(Q, K, V, dO, scale, causal)
    Oo, L = orc.forward(Q, K, V, scale, causal)
    assert np.abs(Oo - O.detach().numpy()).max() < 1e-12
    assert np.abs(L - torch.logsumexp(S, -1).detach().numpy()).max() < 1e-12
    for a, t in ((dQ, tq), (dK, tk), (dV, tv)):
        assert np.abs(a - t.grad.numpy()).max() < 1e-12


def test_backward_closed_forms():
    """Q = 0 (non-causal): P is uniform, so dV_j = mean_i dO_i for every j.
    Constant K rows: every row of dS sums to zero, so dQ = 0."""
    rng = np.random.default_rng(12)
    N, d = 50, 6
    K, V, dO = (rng.standard_normal((1, 1, N, d)) for _ in range(3))
    Q = np.zeros((1, 1, N, d))
    _, _, dV = orc.backward(Q, K, V, dO, 0.4)
    assert np.abs(dV[0, 0] - dO[0, 0].mean(axis=0)).max() < 1e-12
    Q = rng.standard_normal((1, 1, N, d))
    Kc = np.broadcast_to(rng.standard_normal(d), (1, 1, N, d)).copy()
    dQ, _, _ = orc.backward(Q, Kc, V, dO, 0.4)
    assert np.abs(dQ).max() < 1e-12


def test_row_sampled_pieces_equal_full_backward():
    """The row-sampled functions used at full sizes reproduce the full oracle."""
    rng = np.random.default_rng(13)
    B, Hq, Hkv, N, d = 1, 4, 2, 300, 8
    Q = rng.standard_normal((B, Hq, N, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    dO = rng.standard_normal((B, Hq, N, d))
    mask = np.array([[1, 0, 1], [1, 1, 0], [0, 1, 1]], dtype=np.uint8)
    for causal in (False, True):
        O, L = orc.forward(Q, K, V, 0.5, causal, mask)
        dQ, dK, dV = orc.backward(Q, K, V, dO, 0.5, causal, mask)
        rows = np.array([0, 5, 130, 299])
        o, l = orc.forward_rows(Q, K, V, 0.5, causal, mask, 0, 3, rows)
        assert np.abs(o - O[0, 3, rows]).max() < 1e-13
        assert np.array_equal(np.isinf(l), np.isinf(L[0, 3, rows]))
        dq = orc.dq_rows(Q, K, V, dO, 0.5, causal, mask, 0, 3, rows)
        assert np.abs(dq - dQ[0, 3, rows]).max() < 1e-12
        krows = np.array([1, 127, 128, 260])
        dk, dv = orc.dkdv_rows(Q, K, V, dO, 0.5, causal, mask, 0, 1, krows)
        assert np.abs(dk - dK[0, 1, krows]).max() < 1e-12
        assert np.abs(dv - dV[0, 1, krows]).max() < 1e-12


# ---------------------------------------------------------------- inputs and FLOP counting

def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 1 + 2 ** -7 + 2 ** -9],
                 dtype=np.float32)
    r = inputs.bf16_round(x)
    assert r[0] == 1.0
    assert r[1] == 1.0                  # tie -> even (mantissa 0)
    assert r[2] == 1.0 + 2 ** -7        # above half -> up
    assert r[3] == -2.5
    assert r[4] == 1 + 2 ** -7          # below half -> down
    t = torch.tensor(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(t, r)


def test_allowed_count_brute_force():
    mask = inputs.random_block_mask(300, 0.5, seed=3)
    for causal in (False, True):
        for m in (None, mask):
            ok = orc.allowed(np.arange(300), 300, causal, m)
            assert inputs.allowed_count(300, causal, m) == int(ok.sum())


def test_block_mask_recipe():
    m = inputs.random_block_mask(65536)
    nb = 512
    assert m.shape == (nb, nb) and np.all(np.diag(m) == 1)
    assert int(m.sum()) == nb + int(round(0.25 * (nb * nb - nb)))


# ---------------------------------------------------------------- mask and score modifiers

def _visible_brute(i, j, causal, window, prefix, doc):
    """Whether key j is visible to query i, from the modifier rules one by one."""
    right_ok = (not causal or j <= i)
    left_ok = True
    if window is not None:
        if window[1] >= 0 and j > i + window[1]:
            right_ok = False
        if window[0] >= 0 and j < i - window[0]:
            left_ok = False
    if j < prefix:
        right_ok = True
    return right_ok and left_ok and (doc is None or doc[i] == doc[j])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("window", [None, (5, -1), (3, 2), (-1, 4)])
@pytest.mark.parametrize("prefix", [0, 1, 7])
@pytest.mark.parametrize("with_doc", [False, True])
def test_modifier_visibility_brute_force(causal, window, prefix, with_doc):
    N = 23
    doc = np.repeat([0, 1, 2, 3], [6, 1, 9, 7]) if with_doc else None
    got = orc.allowed(np.arange(N), N, causal, None, window, prefix, doc)
    for i in range(N):
        for j in range(N):
            assert got[i, j] == _visible_brute(i, j, causal, window, prefix, doc), (i, j)


def _doc_case(seed, N=150, Hq=2, Hkv=1, d=16):
    rng = np.random.default_rng(seed)
    lengths = [37, 1, 64, 48]
    doc = np.repeat(np.arange(len(lengths)), lengths)
    assert doc.size == N
    Q = rng.standard_normal((1, Hq, N, d))
    K = rng.standard_normal((1, Hkv, N, d))
    V = rng.standard_normal((1, Hkv, N, d))
    dO = rng.standard_normal((1, Hq, N, d))
    return Q, K, V, dO, doc, lengths


@pytest.mark.parametrize("causal", [False, True])
def test_document_mask_is_attention_per_document(causal):
    """A document-id mask over packed documents gives, for every document,
    exactly the attention of that document on its own (forward and
    gradients)."""
    Q, K, V, dO, doc, lengths = _doc_case(5)
    O, L = orc.forward(Q, K, V, 0.3, causal, doc=doc)
    dQ, dK, dV = orc.backward(Q, K, V, dO, 0.3, causal, doc=doc)
    s0 = 0
    for n in lengths:
        sl = slice(s0, s0 + n)
        o, lse = orc.forward(Q[:, :, sl], K[:, :, sl], V[:, :, sl], 0.3, causal)
        dq, dk, dv = orc.backward(Q[:, :, sl], K[:, :, sl], V[:, :, sl], dO[:, :, sl], 0.3, causal)
        assert np.abs(O[:, :, sl] - o).max() < 1e-12
        assert np.abs(L[:, :, sl] - lse).max() < 1e-12
        for a, b_ in ((dQ[:, :, sl], dq), (dK[:, :, sl], dk), (dV[:, :, sl], dv)):
            assert np.abs(a - b_).max() < 1e-12
        s0 += n


def test_prefix_lm_special_cases():
    """Prefix LM: a prefix of N or more is full (non-causal) attention, a
    prefix of 0 or 1 is plain causal attention (key 0 is visible to every
    query already), and rows inside the prefix see exactly the prefix in both
    directions (bidirectional attention over the first P tokens alone)."""
    rng = np.random.default_rng(6)
    N, d, P = 90, 8, 33
    Q, K, V = (rng.standard_normal((1, 1, N, d)) for _ in range(3))
    full, _ = orc.forward(Q, K, V, 0.4, False)
    causal, _ = orc.forward(Q, K, V, 0.4, True)
    assert np.abs(orc.forward(Q, K, V, 0.4, True, prefix=N)[0] - full).max() < 1e-12
    assert np.abs(orc.forward(Q, K, V, 0.4, True, prefix=N + 50)[0] - full).max() < 1e-12
    for p in (0, 1):
        assert np.abs(orc.forward(Q, K, V, 0.4, True, prefix=p)[0] - causal).max() < 1e-12
    O, _ = orc.forward(Q, K, V, 0.4, True, prefix=P)
    head, _ = orc.forward(Q[:, :, :P], K[:, :, :P], V[:, :, :P], 0.4, False)
    assert np.abs(O[:, :, :P] - head).max() < 1e-12
    # a row past the prefix sees keys 0..i: the causal result
    assert np.abs(O[:, :, P:] - causal[:, :, P:]).max() < 1e-12


def test_softcap_limits():
    """Soft-capping with a huge cap is the plain score; with Q = 0 every score
    is cap * tanh(0) = 0, so O is the mean of V whatever the cap."""
    rng = np.random.default_rng(7)
    Q, K, V = (rng.standard_normal((1, 1, 64, 8)) for _ in range(3))
    plain, Lp = orc.forward(Q, K, V, 0.5, True)
    big, Lb = orc.forward(Q, K, V, 0.5, True, softcap=1e7)
    assert np.abs(plain - big).max() < 1e-9 and np.abs(Lp - Lb).max() < 1e-9
    O0, _ = orc.forward(np.zeros_like(Q), K, V, 0.5, False, softcap=2.0)
    assert np.abs(O0[0, 0] - V[0, 0].mean(axis=0)).max() < 1e-12


def test_softcap_gradients_finite_differences():
    """Gradients through the soft-cap chain rule against central differences
    of sum(O * dO), with a cap small enough to bend the scores."""
    rng = np.random.default_rng(8)
    N, d, cap = 9, 4, 1.5
    Q, K, V, dO = (rng.standard_normal((1, 1, N, d)) * 1.5 for _ in range(4))
    doc = np.array([0, 0, 0, 0, 1, 1, 1, 1, 1])
    kw = dict(causal=True, softcap=cap, prefix=2, doc=doc)
    dQ, dK, dV = orc.backward(Q, K, V, dO, 0.7, **kw)

    def f(Q_, K_, V_):
        return float(np.sum(orc.forward(Q_, K_, V_, 0.7, **kw)[0] * dO))

    eps = 1e-6
    for X, G, which in ((Q, dQ, 0), (K, dK, 1), (V, dV, 2)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += eps
            Xm[idx] -= eps
            args_p, args_m = [Q, K, V], [Q, K, V]
            args_p[which], args_m[which] = Xp, Xm
            num[idx] = (f(*args_p) - f(*args_m)) / (2 * eps)
        assert np.abs(num - G).max() < 1e-6 * max(1.0, np.abs(G).max())


def test_softcap_gradients_match_torch_autograd():
    """The oracle's hand-derived backward with soft-capping and a document
    mask equals torch fp64 autograd of the forward formula."""
    rng = np.random.default_rng(9)
    N, d, cap, scale = 40, 8, 2.0, 0.6
    Q, K, V, dO = (rng.standard_normal((1, 1, N, d)) for _ in range(4))
    doc = np.repeat([0, 1, 2], [10, 18, 12])
    dQ, dK, dV = orc.backward(Q, K, V, dO, scale, True, softcap=cap, doc=doc)
    q, k, v = (torch.tensor(a[0, 0], dtype=torch.float64, requires_grad=True) for a in (Q, K, V))
    x = scale * (q @ k.T)
    s = cap * torch.tanh(x / cap)
    i = torch.arange(N)
    dt = torch.tensor(doc)
    vis = (i[None, :] <= i[:, None]) & (dt[:, None] == dt[None, :])
    s = s.masked_fill(~vis, float("-inf"))
    o = torch.softmax(s, dim=1) @ v
    (o * torch.tensor(dO[0, 0])).sum().backward()
    for got, ref in ((dQ, q.grad), (dK, k.grad), (dV, v.grad)):
        assert np.abs(got[0, 0] - ref.numpy()).max() < 1e-12
