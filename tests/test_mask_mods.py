"""Mask modifiers (fa_fwd_mod / fa_bwd_mod): prefix LM, per-token document ids
and their combinations with the causal flag, a sliding window and the block
mask, against the fp64 oracle on the same seeded inputs. The GPU cases span
several tiles with ragged tails; the argument checks run on the CPU."""
import ctypes

import numpy as np
import pytest

from _helpers import LSE_MAX_ABS, assert_close_bf16, lse_err, to_dev, to_np
from exact_io_aware_45_b200 import fa, inputs
from oracle import attention as orc


def _docs(lengths):
    return np.repeat(np.arange(len(lengths)), lengths).astype(np.int32)


CASES = [
    # name, B, Hq, Hkv, N, d, causal, window, prefix, doc lengths, mask density, softcap
    ("prefix_lm", 1, 4, 2, 700, 128, True, None, 300, None, None),
    ("prefix_lm_d64", 2, 2, 1, 513, 64, True, None, 129, None, None),
    ("prefix_past_tiles", 1, 2, 2, 384, 64, True, None, 383, None, None),
    ("docs_causal", 1, 4, 2, 700, 128, True, None, 0, [100, 1, 260, 139, 200], None),
    ("docs_full", 1, 2, 1, 700, 64, False, None, 0, [100, 1, 260, 139, 200], None),
    ("docs_one_doc", 1, 2, 2, 300, 128, True, None, 0, [300], None),
    ("docs_window", 1, 2, 1, 640, 128, True, (64, -1), 0, [129, 383, 128], None),
    ("prefix_window_mask", 1, 2, 2, 640, 64, True, (200, -1), 100, None, 0.5),
    ("right_window_prefix", 1, 2, 1, 500, 128, False, (-1, 40), 70, None, None),
    ("docs_prefix_mask", 1, 2, 1, 768, 128, True, None, 64, [64, 300, 404], 0.6),
    # soft-capping (score modifier), alone and with masks; caps small enough
    # to bend the N(0, 1) scores
    ("softcap", 1, 2, 1, 600, 128, False, None, 0, None, None, 1.5),
    ("softcap_causal_d64", 2, 2, 2, 300, 64, True, None, 0, None, None, 0.8),
    ("softcap_docs_mask", 1, 2, 1, 640, 64, True, (100, -1), 0, [300, 340], 0.5, 2.0),
    # the capped variant of each remaining forward form: skipping (a left
    # window edge, no block mask), split at d = 128 (a block mask), one-item
    # (above the persistent form's 4,096 keys)
    ("softcap_window_d128", 1, 2, 1, 640, 128, True, (150, -1), 0, [200, 440], None, 1.7),
    ("softcap_mask_d128", 1, 2, 1, 520, 128, False, None, 0, None, 0.5, 1.0),
    ("softcap_long_d64", 1, 1, 1, 4200, 64, True, None, 0, None, None, 1.2),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_mask_mod_parity(case):
    import torch
    _, B, Hq, Hkv, N, d, causal, window, prefix, lengths, dens = case[:11]
    cap = case[11] if len(case) > 11 else 0.0
    fa.lib()
    x = inputs.random_case(B, Hq, Hkv, N, d, seed=N + d + prefix, mask_density=dens)
    doc = None if lengths is None else _docs(lengths)
    q, k, v, do = (to_dev(x[n], torch.bfloat16) for n in ("q", "k", "v", "do"))
    mask = None if x["mask"] is None else torch.from_numpy(x["mask"]).cuda()
    doc_t = None if doc is None else torch.from_numpy(doc).cuda()
    wl, wr = window if window is not None else (-1, -1)
    m = fa.mods(wl, wr, prefix, doc_t, cap)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.forward_mod(q, k, v, m, scale, causal, mask)
    dq, dk, dv = fa.backward_mod(q, k, v, o, do, lse, m, scale, causal, mask)
    torch.cuda.synchronize()
    kw = dict(window=window, prefix=prefix, doc=doc, softcap=cap)
    O, L = orc.forward(x["q"], x["k"], x["v"], scale, causal, x["mask"], **kw)
    assert_close_bf16("O", to_np(o), O)
    assert lse_err(to_np(lse), L) <= LSE_MAX_ABS
    dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], scale, causal, x["mask"], O=O,
                              **kw)
    assert_close_bf16("dQ", to_np(dq), dQ)
    assert_close_bf16("dK", to_np(dk), dK)
    assert_close_bf16("dV", to_np(dv), dV)


@pytest.mark.gpu
def test_mods_off_is_plain_attention():
    """All modifier fields off: bit-identical to fa_fwd (same kernel form)."""
    import torch
    fa.lib()
    x = inputs.random_case(1, 2, 1, 400, 128, seed=44)
    q, k, v = (to_dev(x[n], torch.bfloat16) for n in ("q", "k", "v"))
    o1, l1 = fa.forward(q, k, v, 0.1, True)
    o2, l2 = fa.forward_mod(q, k, v, fa.mods(), 0.1, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _call_fwd(m, dtype=fa.FA_BF16, d=128):
    g = 1 << 20   # aligned fake pointers: every case below is refused before any launch
    return fa.fa_fwd_mod(g, g, g, g, g, 1, 2, 1, 256, d, 0.1, 1, 0, ctypes.byref(m), dtype, g, 0)


def test_mod_arguments_checked_on_host():
    assert _call_fwd(fa.mods(prefix=-1)) == fa.FA_ERR_INVALID_ARG
    assert _call_fwd(fa.mods(window_left=-2)) == fa.FA_ERR_INVALID_ARG
    m = fa.mods()
    m.doc_ids = (1 << 20) + 2   # not 4-byte aligned
    assert _call_fwd(m) == fa.FA_ERR_INVALID_ARG
    assert _call_fwd(fa.mods(softcap=-1.0)) == fa.FA_ERR_INVALID_ARG
    # modifiers run on the tensor-core kernels only
    assert _call_fwd(fa.mods(prefix=3), dtype=fa.FA_F32) == fa.FA_ERR_UNSUPPORTED
    assert _call_fwd(fa.mods(prefix=3), d=32) == fa.FA_ERR_UNSUPPORTED
