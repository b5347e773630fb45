"""GPU parity: the CUDA library (called through the C ABI) against the fp64
oracle on the same seeded inputs.

Small cases span several 128-row tiles and ragged tails and run the whole
oracle; the four bf16 workloads run at full size in the launch configuration
the benchmark times and are compared on sampled rows the oracle computes one by
one (plus properties that hold at any size).
"""
import numpy as np
import pytest

from _helpers import (F32_O_MAX_ABS, LSE_MAX_ABS, assert_close_bf16, lse_err, max_abs, to_dev,
                      to_np)
from exact_io_aware_45_b200 import fa, inputs
from oracle import attention as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need CUDA"
    fa.lib()


def _run(x, scale, causal, path, dtype_name="bf16", grad="f32", backward=True):
    import torch
    dt = torch.bfloat16 if dtype_name == "bf16" else torch.float32
    q, k, v = (to_dev(x[n], dt) for n in ("q", "k", "v"))
    mask = None if x["mask"] is None else torch.from_numpy(x["mask"]).cuda()
    o, lse = fa.forward(q, k, v, scale, causal, mask, path=path)
    out = {"o": o, "lse": lse}
    if backward:
        do = to_dev(x["do"], dt)
        gdt = torch.float32 if grad == "f32" else torch.bfloat16
        dq, dk, dv = fa.backward(q, k, v, o, do, lse, scale, causal, mask, grad_dtype=gdt,
                                 path=path)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    return out


# ------------------------------------------------------------------ fp32 workload (the lesson's example)

@pytest.mark.parametrize("path", [fa.PATH_AUTO, fa.PATH_SIMT])
def test_fp32_lesson_example(path):
    w = inputs.WORKLOADS["fp32_n512_d32"]
    x = inputs.make_inputs(w)
    r = _run(x, w.scale, False, path, "f32", backward=False)
    O, L = orc.forward(x["q"], x["k"], x["v"], w.scale)
    assert max_abs(to_np(r["o"]), O) <= F32_O_MAX_ABS
    assert lse_err(to_np(r["lse"]), L) <= F32_O_MAX_ABS


def test_fp32_backward_small():
    """fp32 inputs and gradients on the CUDA-core path (derived bound: fp32
    rounding of sums over <= 300 terms stays far below 1e-4)."""
    x = inputs.random_case(1, 2, 1, 300, 32, seed=3, dtype="f32")
    r = _run(x, 0.2, True, fa.PATH_AUTO, "f32")
    O, L = orc.forward(x["q"], x["k"], x["v"], 0.2, True)
    dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], 0.2, True, O=O)
    assert max_abs(to_np(r["o"]), O) <= 1e-4
    for g, ref in ((r["dq"], dQ), (r["dk"], dK), (r["dv"], dV)):
        assert max_abs(to_np(g), ref) <= 1e-4


# ------------------------------------------------------------------ small bf16 cases

SMALL = [
    # B, Hq, Hkv, N, d, causal, mask density
    (1, 1, 1, 1, 64, False, None),
    (1, 1, 1, 17, 128, True, None),
    (2, 2, 2, 127, 64, False, None),
    (1, 2, 1, 128, 128, True, None),
    (1, 4, 2, 129, 64, True, None),
    (2, 2, 1, 255, 128, False, None),
    (1, 8, 2, 300, 64, False, 0.5),
    (1, 4, 4, 384, 128, True, 0.5),
    (1, 3, 1, 513, 128, False, None),
    (2, 4, 1, 640, 64, True, None),
    (1, 2, 2, 1000, 128, False, 0.3),
    (1, 2, 2, 1024, 64, True, 0.3),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "B{}H{}x{}N{}d{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], "c" if c[5] else "", "m" if c[6] else ""))
@pytest.mark.parametrize("path", [fa.PATH_AUTO, fa.PATH_SIMT], ids=["auto", "simt"])
def test_small_parity(case, path):
    B, Hq, Hkv, N, d, causal, dens = case
    x = inputs.random_case(B, Hq, Hkv, N, d, seed=N + d, mask_density=dens)
    scale = 1.0 / np.sqrt(d)
    r = _run(x, scale, causal, path)
    O, L = orc.forward(x["q"], x["k"], x["v"], scale, causal, x["mask"])
    assert_close_bf16("O", to_np(r["o"]), O)
    assert lse_err(to_np(r["lse"]), L) <= LSE_MAX_ABS
    dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], scale, causal, x["mask"], O=O)
    assert_close_bf16("dQ", to_np(r["dq"]), dQ)
    assert_close_bf16("dK", to_np(r["dk"]), dK)
    assert_close_bf16("dV", to_np(r["dv"]), dV)


def test_bf16_gradients_output():
    """bf16 gradient outputs: the oracle rounded to bf16 is within the bound."""
    x = inputs.random_case(1, 2, 1, 256, 64, seed=5)
    r = _run(x, 0.125, True, fa.PATH_AUTO, grad="bf16")
    O, _ = orc.forward(x["q"], x["k"], x["v"], 0.125, True)
    dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], 0.125, True, O=O)
    assert r["dq"].dtype.__str__().endswith("bfloat16")
    for n, g, ref in (("dQ", r["dq"], dQ), ("dK", r["dk"], dK), ("dV", r["dv"], dV)):
        assert_close_bf16(n, to_np(g), ref)


def test_empty_block_row():
    """A block row with no visible block: O = 0, LSE = -inf, dQ = 0."""
    x = inputs.random_case(1, 2, 2, 256, 64, seed=6)
    x["mask"] = np.array([[1, 1], [0, 0]], dtype=np.uint8)
    for path in (fa.PATH_AUTO, fa.PATH_SIMT):
        r = _run(x, 0.125, False, path)
        o, lse, dq = to_np(r["o"]), to_np(r["lse"]), to_np(r["dq"])
        assert np.all(o[:, :, 128:] == 0) and np.all(np.isneginf(lse[:, :, 128:]))
        assert np.all(dq[:, :, 128:] == 0)
        O, L = orc.forward(x["q"], x["k"], x["v"], 0.125, False, x["mask"])
        assert_close_bf16("O", o, O)
        dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], 0.125, False, x["mask"], O=O)
        assert_close_bf16("dK", to_np(r["dk"]), dK)
        assert_close_bf16("dV", to_np(r["dv"]), dV)


BLOCK_PATTERNS = {
    # the second query tile of the pair sees nothing
    "lower_off": [[1, 1], [0, 0]],
    # the first query tile of the pair sees nothing
    "upper_off": [[0, 0], [1, 1]],
    # every key tile is seen by exactly one tile of the first pair; the second
    # pair has one empty row and one row with a gap
    "alternating": [[1, 0, 1, 0], [0, 1, 0, 1], [0, 0, 0, 0], [1, 1, 0, 1]],
    # query tiles that see exactly one key tile (one softmax stream of the
    # split form has nothing), and one that sees all three
    "single": [[1, 0, 0], [0, 0, 1], [1, 1, 1]],
}


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("pattern", sorted(BLOCK_PATTERNS))
def test_block_mask_patterns(pattern, d):
    """Block masks under which a query tile sees only some, or none, of the key
    tiles its partner tile sees; rows with nothing visible give O = 0 and
    LSE = -inf, the rest match the oracle."""
    mask = np.array(BLOCK_PATTERNS[pattern], dtype=np.uint8)
    N = 128 * mask.shape[0]
    x = inputs.random_case(1, 2, 1, N, d, seed=11 + d)
    x["mask"] = mask
    scale = 1.0 / np.sqrt(d)
    r = _run(x, scale, False, fa.PATH_AUTO)
    o, lse = to_np(r["o"]), to_np(r["lse"])
    O, L = orc.forward(x["q"], x["k"], x["v"], scale, False, mask)
    empty = np.repeat(mask.sum(axis=1) == 0, 128)
    assert np.all(o[:, :, empty] == 0) and np.all(np.isneginf(lse[:, :, empty]))
    assert_close_bf16("O", o, O)
    assert lse_err(lse[:, :, ~empty], L[:, :, ~empty]) <= LSE_MAX_ABS
    dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], scale, False, mask, O=O)
    assert_close_bf16("dQ", to_np(r["dq"]), dQ)
    assert_close_bf16("dK", to_np(r["dk"]), dK)
    assert_close_bf16("dV", to_np(r["dv"]), dV)


def test_forward_deterministic_and_fully_written():
    """Outputs are poisoned with NaN first; two runs agree bit for bit."""
    import torch
    x = inputs.random_case(2, 4, 2, 700, 128, seed=7)
    q, k, v = (to_dev(x[n], torch.bfloat16) for n in ("q", "k", "v"))
    outs = []
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:3], float("nan"), device="cuda")
        fa.forward(q, k, v, 0.1, True, out=o, lse=lse)
        torch.cuda.synchronize()
        assert not torch.isnan(o).any() and not torch.isnan(lse).any()
        outs.append((o.clone(), lse.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_no_device_error_after_runs():
    import torch
    x = inputs.random_case(1, 2, 1, 200, 64, seed=8)
    q, k, v, do = (to_dev(x[n], torch.bfloat16) for n in ("q", "k", "v", "do"))
    ws = fa.new_workspace(fa.fa_bwd_workspace_size(1, 2, 200, 64), "cuda")
    o, lse = fa.forward(q, k, v, 0.125, True, workspace=ws)
    fa.backward(q, k, v, o, do, lse, 0.125, True, workspace=ws)
    assert fa.device_error(ws) == fa.FA_OK


# ------------------------------------------------------------------ full-size workloads (sampled)

def _sample_rows(rng, N, n):
    return np.unique(np.concatenate([[0, 1, 127, 128, N - 1], rng.choice(N, n, replace=False)]))


# (batch, query head) pairs sampled at full size: first, last and interior heads
QUERY_HEADS = {
    "llama7b_causal": [(0, 0), (1, 7), (2, 19), (3, 31), (0, 16), (3, 1)],
    "gqa16k_causal": [(0, 0), (0, 5), (0, 13), (0, 18), (0, 26), (0, 31)],
    "sparse64k": [(0, 0), (0, 3), (0, 7), (0, 9), (0, 12), (0, 15)],
}
# (batch, KV head) pairs whose dK / dV rows are compared; for the grouped
# workload every KV head collects the gradients of its 4 query heads, which
# the oracle sums over the group
KV_HEADS = {
    "llama7b_causal": [(0, 0), (2, 13), (3, 31)],
    "gqa16k_causal": [(0, 0), (0, 7)],
    "sparse64k": [(0, 0), (0, 9)],
}


def _key_rows(rng, w, mask):
    """Key rows whose dK / dV are compared at full size.

    Causal workloads: key tile 0 (key 0 sees every query, so its dK / dV sum
    the longest accumulation and hold the largest values), a tile in the
    middle of the sequence and the last one. Block-sparse: block column 3 and
    the block column with the most active cells."""
    N = w.N
    if w.causal:
        mid = (N // 2 // 128) * 128
        parts = [[0, 1, 127], rng.choice(128, 21, replace=False),
                 [mid, mid + 127], mid + rng.choice(128, 14, replace=False),
                 [N - 1], rng.choice(np.arange(N - 128, N), 12, replace=False)]
    else:
        dense_col = int(np.argmax(mask.sum(axis=0)))
        parts = []
        for kb in sorted({3, dense_col}):
            parts += [[kb * 128, kb * 128 + 127], kb * 128 + rng.choice(128, 20, replace=False)]
    return np.unique(np.concatenate([np.asarray(p, dtype=np.int64) for p in parts]))


@pytest.mark.parametrize("name", ["gpt2_small", "llama7b_causal", "gqa16k_causal", "sparse64k"])
def test_workload_parity(name):
    w = inputs.WORKLOADS[name]
    x = inputs.make_inputs(w)
    r = _run(x, w.scale, w.causal, fa.PATH_AUTO)
    o, lse = r["o"], r["lse"]
    import torch
    for t in (o, lse, r["dq"], r["dk"], r["dv"]):
        assert torch.isfinite(t).all()
    rng = np.random.default_rng(123)
    mask = x["mask"]
    if name == "gpt2_small":
        # small enough for the whole oracle
        O, L = orc.forward(x["q"], x["k"], x["v"], w.scale, w.causal, mask)
        assert_close_bf16("O", to_np(o), O)
        assert lse_err(to_np(lse), L) <= LSE_MAX_ABS
        dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal, mask, O=O)
        assert_close_bf16("dQ", to_np(r["dq"]), dQ)
        assert_close_bf16("dK", to_np(r["dk"]), dK)
        assert_close_bf16("dV", to_np(r["dv"]), dV)
        return
    got_o, want_o, got_q, want_q = [], [], [], []
    for b, h in QUERY_HEADS[name]:
        rows = _sample_rows(rng, w.N, 96)
        Orow, Lrow = orc.forward_rows(x["q"], x["k"], x["v"], w.scale, w.causal, mask, b, h, rows)
        got_o.append(to_np(o[b, h, rows]))
        want_o.append(Orow)
        assert lse_err(to_np(lse[b, h, rows]), Lrow) <= LSE_MAX_ABS
        got_q.append(to_np(r["dq"][b, h, rows]))
        want_q.append(orc.dq_rows(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal, mask, b, h,
                                  rows))
    assert_close_bf16("O rows", np.concatenate(got_o), np.concatenate(want_o))
    assert_close_bf16("dQ rows", np.concatenate(got_q), np.concatenate(want_q))
    keys = _key_rows(rng, w, mask)
    for b, hk in KV_HEADS[name]:
        dk, dv = orc.dkdv_rows(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal, mask, b, hk,
                               keys)
        # each KV head on its own, so a wrong head or group sum cannot hide
        # behind the others
        assert_close_bf16(f"dK rows (b={b}, kv head {hk})", to_np(r["dk"][b, hk, keys]), dk)
        assert_close_bf16(f"dV rows (b={b}, kv head {hk})", to_np(r["dv"][b, hk, keys]), dv)


@pytest.mark.parametrize("dt_name", ["bf16", "f32"])
def test_autograd_attention(dt_name):
    """fa.attention through torch autograd: O from the forward, and the
    gradients of sum(O * dO) (returned in the input dtype) against the oracle."""
    import torch
    dt = torch.bfloat16 if dt_name == "bf16" else torch.float32
    x = inputs.random_case(1, 4, 2, 300, 64, seed=17, dtype=dt_name)
    q, k, v = (to_dev(x[n], dt).requires_grad_(True) for n in ("q", "k", "v"))
    do = to_dev(x["do"], dt)
    scale = 0.125
    o = fa.attention(q, k, v, scale, causal=True)
    (o.float() * do.float()).sum().backward()
    torch.cuda.synchronize()
    O, _ = orc.forward(x["q"], x["k"], x["v"], scale, True)
    dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], scale, True, O=O)
    for name, got, want in (("O", o, O), ("dQ", q.grad, dQ), ("dK", k.grad, dK),
                            ("dV", v.grad, dV)):
        assert got.dtype == dt
        if dt_name == "bf16":
            assert_close_bf16(name, to_np(got), want)
        else:
            assert max_abs(to_np(got), want) <= 1e-4, name


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_block_mask_ragged(causal, d):
    """Random block masks with a ragged last tile (N = 700): the split form's
    last query tile has rows past N and its last key tile keys past N."""
    x = inputs.random_case(1, 2, 1, 700, d, seed=23 + d + int(causal), mask_density=0.5)
    scale = 1.0 / np.sqrt(d)
    r = _run(x, scale, causal, fa.PATH_AUTO)
    O, L = orc.forward(x["q"], x["k"], x["v"], scale, causal, x["mask"])
    o, lse = to_np(r["o"]), to_np(r["lse"])
    assert_close_bf16("O", o, O)
    assert lse_err(lse, L) <= LSE_MAX_ABS
    dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], scale, causal, x["mask"], O=O)
    assert_close_bf16("dQ", to_np(r["dq"]), dQ)
    assert_close_bf16("dK", to_np(r["dk"]), dK)
    assert_close_bf16("dV", to_np(r["dv"]), dV)
