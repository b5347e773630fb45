"""Variable-length (padding-free) batches: sequences packed back to back,
each attending only to itself (glossary page, "Sequence Length Flexibility").

CPU tests pin the oracle's variable-length wrapper (it must equal the batched
oracle when all lengths are equal, keep sequences independent, and reduce to
closed forms on one-token sequences) and check the C ABI's argument handling;
GPU tests compare fa_fwd_varlen / fa_bwd_varlen with the oracle on seeded
length mixes that span several tiles, ragged tails and empty sequences, and
with the dense kernels on an equal-length batch."""
import numpy as np
import pytest

from _helpers import BF16_MAX_ABS, LSE_MAX_ABS, assert_close_bf16, lse_err, to_dev, to_np
from exact_io_aware_45_b200 import fa, inputs
from oracle import attention as orc


def _dense_from_packed(x, B, N):
    total, H, d = x.shape
    return np.ascontiguousarray(np.transpose(x.reshape(B, N, H, d), (0, 2, 1, 3)))


# ------------------------------------------------------------------ oracle pins (CPU)

@pytest.mark.parametrize("causal", [False, True])
def test_oracle_varlen_equals_batched_oracle(causal):
    B, N, Hq, Hkv, d = 3, 40, 4, 2, 16
    x = inputs.varlen_case([N] * B, Hq, Hkv, d, seed=5)
    scale = 0.3
    O, L = orc.forward_varlen(x["q"], x["k"], x["v"], x["cu"], scale, causal)
    dQ, dK, dV = orc.backward_varlen(x["q"], x["k"], x["v"], x["do"], x["cu"], scale, causal)
    q, k, v, do = (_dense_from_packed(x[n], B, N) for n in ("q", "k", "v", "do"))
    Od, Ld = orc.forward(q, k, v, scale, causal)
    gd = orc.backward(q, k, v, do, scale, causal, O=Od)
    assert np.allclose(_dense_from_packed(O, B, N), Od, atol=1e-12)
    assert np.allclose(np.transpose(L.reshape(Hq, B, N), (1, 0, 2)), Ld, atol=1e-12)
    for got, want in zip((dQ, dK, dV), gd):
        assert np.allclose(_dense_from_packed(got, B, N), want, atol=1e-12)


def test_oracle_varlen_sequences_are_independent():
    lengths = [17, 0, 33, 5]
    x = inputs.varlen_case(lengths, 2, 1, 8, seed=2)
    O1, L1 = orc.forward_varlen(x["q"], x["k"], x["v"], x["cu"], 0.5, True)
    cu = x["cu"]
    y = {n: x[n].copy() for n in ("q", "k", "v")}
    for n in y:                       # change every token of the third sequence
        y[n][cu[2]:cu[3]] += 1.0
    O2, L2 = orc.forward_varlen(y["q"], y["k"], y["v"], cu, 0.5, True)
    keep = np.r_[0:cu[2], cu[3]:cu[4]]
    assert np.array_equal(O1[keep], O2[keep]) and np.array_equal(L1[:, keep], L2[:, keep])
    assert not np.allclose(O1[cu[2]:cu[3]], O2[cu[2]:cu[3]])


def test_oracle_varlen_one_token_sequences():
    """A one-token sequence attends to itself only: O = V, LSE = scale * q.k."""
    x = inputs.varlen_case([1, 1, 1], 2, 2, 8, seed=3)
    O, L = orc.forward_varlen(x["q"], x["k"], x["v"], x["cu"], 0.25, False)
    assert np.allclose(O, x["v"], atol=1e-12)
    qk = np.einsum("thd,thd->ht", x["q"].astype(np.float64), x["k"].astype(np.float64))
    assert np.allclose(L, 0.25 * qk, atol=1e-12)


def test_varlen_lengths_recipe():
    lens = inputs.varlen_lengths(10000, 100, 900, seed=0)
    assert sum(lens) == 10000 and all(0 < n <= 900 for n in lens)
    assert lens == inputs.varlen_lengths(10000, 100, 900, seed=0)


# ------------------------------------------------------------------ ABI checks (no launch)

GOOD = 0x10000


def _fwd(**kw):
    a = dict(Q=GOOD, K=GOOD, V=GOOD, O=GOOD, LSE=GOOD, cu=GOOD, B=2, maxlen=64, total=100, Hq=2,
             Hkv=1, d=64, scale=0.125, causal=0, dtype=fa.FA_BF16, ws=GOOD, stream=0)
    a.update(kw)
    return fa.fa_fwd_varlen(a["Q"], a["K"], a["V"], a["O"], a["LSE"], a["cu"], a["B"],
                            a["maxlen"], a["total"], a["Hq"], a["Hkv"], a["d"], a["scale"],
                            a["causal"], a["dtype"], a["ws"], a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(cu=0), fa.FA_ERR_INVALID_ARG),
    (dict(cu=GOOD + 2), fa.FA_ERR_INVALID_ARG),
    (dict(B=-1), fa.FA_ERR_INVALID_ARG),
    (dict(total=-1), fa.FA_ERR_INVALID_ARG),
    (dict(maxlen=0), fa.FA_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), fa.FA_ERR_INVALID_ARG),
    (dict(causal=2), fa.FA_ERR_INVALID_ARG),
    (dict(Q=GOOD + 8), fa.FA_ERR_INVALID_ARG),
    (dict(dtype=fa.FA_F32), fa.FA_ERR_UNSUPPORTED),
    (dict(d=32), fa.FA_ERR_UNSUPPORTED),
    (dict(scale=-1.0), fa.FA_ERR_UNSUPPORTED),
    (dict(B=0), fa.FA_OK),
    (dict(total=0), fa.FA_OK),
])
def test_fwd_varlen_argument_checks(kw, want):
    assert _fwd(**kw) == want


def test_bwd_varlen_workspace_size():
    B, Hq, maxlen, total, d = 3, 4, 300, 700, 64
    npad = 384
    vec = (4 * B * Hq * npad + 255) // 256 * 256
    acc = (4 * total * Hq * d + 255) // 256 * 256
    assert fa.fa_bwd_varlen_workspace_size(B, Hq, maxlen, total, d) == 256 + 2 * vec + acc
    assert fa.fa_bwd_varlen_workspace_size(-1, 1, 1, 1, 1) == 0


# ------------------------------------------------------------------ GPU parity

CASES = [
    # lengths, Hq, Hkv, d, causal
    ([1, 127, 128, 129, 300], 4, 2, 128, True),
    ([1, 127, 128, 129, 300], 2, 2, 64, False),
    ([513, 1000, 64], 4, 1, 128, False),
    ([100, 0, 200, 257], 2, 1, 64, True),
    ([700], 3, 3, 128, True),
]


@pytest.mark.gpu
@pytest.mark.parametrize("lengths,Hq,Hkv,d,causal", CASES)
def test_varlen_matches_oracle(lengths, Hq, Hkv, d, causal):
    import torch
    x = inputs.varlen_case(lengths, Hq, Hkv, d, seed=11)
    scale = 1.0 / np.sqrt(d)
    bf = torch.bfloat16
    q, k, v, do = (to_dev(x[n], bf) for n in ("q", "k", "v", "do"))
    cu = torch.from_numpy(x["cu"]).cuda()
    o, lse = fa.forward_varlen(q, k, v, cu, x["max_seqlen"], scale, causal)
    dq, dk, dv = fa.backward_varlen(q, k, v, o, do, lse, cu, x["max_seqlen"], scale, causal)
    torch.cuda.synchronize()
    O, L = orc.forward_varlen(x["q"], x["k"], x["v"], x["cu"], scale, causal)
    dQ, dK, dV = orc.backward_varlen(x["q"], x["k"], x["v"], x["do"], x["cu"], scale, causal)
    assert_close_bf16("O", to_np(o), O)
    assert lse_err(to_np(lse), L) <= LSE_MAX_ABS
    for name, got, want in (("dQ", dq, dQ), ("dK", dk, dK), ("dV", dv, dV)):
        assert_close_bf16(name, to_np(got), want)


@pytest.mark.gpu
def test_varlen_bf16_gradients():
    import torch
    x = inputs.varlen_case([200, 333], 2, 2, 128, seed=12)
    bf = torch.bfloat16
    q, k, v, do = (to_dev(x[n], bf) for n in ("q", "k", "v", "do"))
    cu = torch.from_numpy(x["cu"]).cuda()
    o, lse = fa.forward_varlen(q, k, v, cu, x["max_seqlen"], None, True)
    g = fa.backward_varlen(q, k, v, o, do, lse, cu, x["max_seqlen"], None, True, grad_dtype=bf)
    torch.cuda.synchronize()
    scale = 1.0 / np.sqrt(128)
    want = orc.backward_varlen(x["q"], x["k"], x["v"], x["do"], x["cu"], scale, True)
    for name, got, w in zip(("dQ", "dK", "dV"), g, want):
        assert got.dtype == bf
        assert_close_bf16(name, to_np(got), w)


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
def test_varlen_equal_lengths_equals_dense(d):
    """Equal lengths: the packed layout must give the dense kernel's result
    (forward bit for bit; gradients within the fp32 accumulation order)."""
    import torch
    B, N, Hq, Hkv = 3, 384, 4, 2
    x = inputs.varlen_case([N] * B, Hq, Hkv, d, seed=13)
    bf = torch.bfloat16
    q, k, v, do = (to_dev(x[n], bf) for n in ("q", "k", "v", "do"))
    cu = torch.from_numpy(x["cu"]).cuda()
    o, lse = fa.forward_varlen(q, k, v, cu, N, None, True)
    g = fa.backward_varlen(q, k, v, o, do, lse, cu, N, None, True)
    dense = {n: to_dev(_dense_from_packed(x[n], B, N), bf) for n in ("q", "k", "v", "do")}
    od, ld = fa.forward(dense["q"], dense["k"], dense["v"], None, True)
    gd = fa.backward(dense["q"], dense["k"], dense["v"], od, dense["do"], ld, None, True)
    torch.cuda.synchronize()
    assert np.array_equal(_dense_from_packed(to_np(o), B, N), to_np(od))
    assert np.array_equal(np.transpose(to_np(lse).reshape(Hq, B, N), (1, 0, 2)), to_np(ld))
    for got, want in zip(g, gd):
        assert np.max(np.abs(_dense_from_packed(to_np(got), B, N) - to_np(want))) <= 1e-4
