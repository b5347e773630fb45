"""Host-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before launching anything (these
calls never reach the GPU, so they run without one)."""
import ctypes
import os
import re

import pytest

from exact_io_aware_45_b200 import fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def _declared():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    L = fa.lib()
    declared = _declared()
    assert declared, "no declarations found"
    for n in declared:
        assert hasattr(L, n), n
    assert set(fa.EXPORTS) <= declared


def test_status_strings_and_version():
    assert fa.status_string(0) == "FA_OK"
    assert fa.status_string(4) == "FA_ERR_TIMEOUT"
    assert fa.status_string(99) == "FA_ERR_UNKNOWN"
    assert fa.fa_version() >= 10000


def test_workspace_sizes():
    assert fa.fa_fwd_workspace_size() == 256
    B, Hq, N, d = 2, 3, 300, 64
    npad = 384
    vec = (4 * B * Hq * npad + 255) // 256 * 256
    acc = (4 * B * Hq * N * d + 255) // 256 * 256
    assert fa.fa_bwd_workspace_size(B, Hq, N, d) == 256 + 2 * vec + acc
    assert fa.fa_bwd_workspace_size(-1, 1, 1, 1) == 0


# fake device pointers: never dereferenced, validation fails or returns first
GOOD = 0x10000


def fwd(**kw):
    a = dict(Q=GOOD, K=GOOD, V=GOOD, O=GOOD, LSE=GOOD, B=1, Hq=2, Hkv=1, N=64, d=64,
             scale=0.125, causal=0, mask=0, dtype=fa.FA_BF16, ws=GOOD, stream=0, path=0)
    a.update(kw)
    return fa.fa_fwd_ex(a["Q"], a["K"], a["V"], a["O"], a["LSE"], a["B"], a["Hq"], a["Hkv"],
                        a["N"], a["d"], a["scale"], a["causal"], a["mask"], a["dtype"],
                        a["ws"], a["stream"], a["path"])


def bwd(**kw):
    a = dict(B=1, Hq=2, Hkv=1, N=64, d=64, scale=0.125, causal=0, mask=0, dtype=fa.FA_BF16,
             gdtype=fa.FA_F32, ws=GOOD, wsb=1 << 30, path=0)
    a.update(kw)
    ptr = {k: a.pop(k, GOOD) for k in ("Q", "K", "V", "O", "dO", "LSE", "dQ", "dK", "dV")}
    return fa.fa_bwd_ex(ptr["Q"], ptr["K"], ptr["V"], ptr["O"], ptr["dO"], ptr["LSE"], ptr["dQ"],
                        ptr["dK"], ptr["dV"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"],
                        a["scale"], a["causal"], a["mask"], a["dtype"], a["gdtype"], a["ws"],
                        a["wsb"], 0, a["path"])


@pytest.mark.parametrize("kw,want", [
    (dict(Hq=3, Hkv=2), fa.FA_ERR_INVALID_ARG),       # Hq % Hkv != 0
    (dict(Hkv=0), fa.FA_ERR_INVALID_ARG),
    (dict(B=-1), fa.FA_ERR_INVALID_ARG),
    (dict(N=-5), fa.FA_ERR_INVALID_ARG),
    (dict(causal=2), fa.FA_ERR_INVALID_ARG),
    (dict(dtype=7), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(path=9), fa.FA_ERR_INVALID_ARG),
    (dict(d=48), fa.FA_ERR_UNSUPPORTED),
    (dict(d=256), fa.FA_ERR_UNSUPPORTED),
    (dict(Q=0), fa.FA_ERR_INVALID_ARG),
    (dict(LSE=0), fa.FA_ERR_INVALID_ARG),
    (dict(ws=0), fa.FA_ERR_INVALID_ARG),
    (dict(K=GOOD + 8), fa.FA_ERR_INVALID_ARG),        # not 16-byte aligned
    (dict(O=GOOD + 2), fa.FA_ERR_INVALID_ARG),
    (dict(N=0, Q=0), fa.FA_OK),                       # empty problem: no launch
    (dict(B=0, Q=0, K=0), fa.FA_OK),
    (dict(dtype=fa.FA_F32, path=fa.PATH_TC), fa.FA_ERR_UNSUPPORTED),
    (dict(d=32, path=fa.PATH_TC), fa.FA_ERR_UNSUPPORTED),
])
def test_fwd_argument_checks(kw, want):
    assert fwd(**kw) == want
    if want != fa.FA_OK:
        assert fa.fa_last_launch_count() == 0


@pytest.mark.parametrize("kw,want", [
    (dict(Hq=4, Hkv=3), fa.FA_ERR_INVALID_ARG),
    (dict(gdtype=5), fa.FA_ERR_INVALID_ARG),
    (dict(dO=0), fa.FA_ERR_INVALID_ARG),
    (dict(dV=GOOD + 4), fa.FA_ERR_INVALID_ARG),
    (dict(wsb=100), fa.FA_ERR_INVALID_ARG),           # workspace too small
    (dict(d=80), fa.FA_ERR_UNSUPPORTED),
    (dict(N=0), fa.FA_OK),
    (dict(dtype=fa.FA_F32, path=fa.PATH_TC), fa.FA_ERR_UNSUPPORTED),
])
def test_bwd_argument_checks(kw, want):
    assert bwd(**kw) == want
    assert fa.fa_last_launch_count() == 0


def test_device_error_null_workspace():
    assert fa.fa_get_device_error(0, 0) == fa.FA_ERR_INVALID_ARG


def test_debug_stall_hook_arguments():
    """The wait-limit test hook validates its arguments and can be switched
    off again (no kernel runs here)."""
    assert fa.fa_debug_set_stall(0, 0) == fa.FA_OK
    assert fa.fa_debug_set_stall(-1, 10_000) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_set_stall(8, 10_000) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_set_stall(fa.FA_STALL_FWD, 10) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_set_stall(fa.FA_STALL_FWD, 3_000_000_000) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_set_stall(fa.FA_STALL_FWD | fa.FA_STALL_DQ, 10_000) == fa.FA_OK
    assert fa.fa_debug_set_stall(0, 0) == fa.FA_OK
