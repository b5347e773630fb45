"""Seeded synthetic inputs for the attention workloads.

This module holds no attention arithmetic. It draws the input tensors, rounds
them to bfloat16 where a workload asks for it, builds the block mask of the
block-sparse workload and counts the score elements a mask allows (the unit
the TFLOP/s figures are quoted in). Both the CUDA path and the fp64 oracle
consume exactly the arrays produced here.

Workloads (FlashAttention pages: the NumPy example of the "Developer" lesson,
and the GPT-2 / 16K / 64K block-sparse points of the paper summary):

* ``fp32_n512_d32``   -- one head, Q, K, V fp32 [512, 32] drawn the way the
  NumPy lesson draws them: ``default_rng(0)``, ``normal(size=(N, d))`` cast to
  float32, in the order Q, K, V. Forward only.
* ``gpt2_small``      -- B=8, H=12, N=1024, d=64, dense.
* ``llama7b_causal``  -- B=4, H=32, N=4096, d=128, causal.
* ``gqa16k_causal``   -- B=1, Hq=32, Hkv=8, N=16384, d=128, causal.
* ``sparse64k``       -- B=1, H=16, N=65536, d=64, 128x128 block mask with
  every diagonal block on and a seeded random quarter of the off-diagonal
  blocks on.

For the bf16 workloads ``default_rng(seed)`` draws Q, K, V and dO in that order
as float32 standard normals of the full [B, H, N, d] shape (K and V with the
KV head count), each then rounded to bfloat16 with round-to-nearest-even.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

BLOCK = 128  # block-mask granularity (rows and columns of one mask cell)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    sparse: bool
    dtype: str          # "f32" or "bf16"
    backward: bool      # does the workload include the backward pass
    scale: float

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv


WORKLOADS = {
    "fp32_n512_d32": Workload("fp32_n512_d32", 1, 1, 1, 512, 32, False, False,
                              "f32", False, 1.0 / np.sqrt(32.0)),
    "gpt2_small": Workload("gpt2_small", 8, 12, 12, 1024, 64, False, False,
                           "bf16", True, 1.0 / 8.0),
    "llama7b_causal": Workload("llama7b_causal", 4, 32, 32, 4096, 128, True,
                               False, "bf16", True, 1.0 / np.sqrt(128.0)),
    "gqa16k_causal": Workload("gqa16k_causal", 1, 32, 8, 16384, 128, True,
                              False, "bf16", True, 1.0 / np.sqrt(128.0)),
    "sparse64k": Workload("sparse64k", 1, 16, 16, 65536, 64, False, True,
                          "bf16", True, 1.0 / 8.0),
}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even).

    Returns the rounded values as float32 (exactly representable in bf16).
    Inputs here are finite normals, so no NaN handling is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (r & np.uint32(0xFFFF0000)).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The uint16 bit patterns of values that are already bf16-exact."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def random_block_mask(N: int, density: float = 0.25, seed: int = 0) -> np.ndarray:
    """uint8 [nb, nb] block mask: diagonal on, round(density * (nb^2 - nb))
    off-diagonal blocks chosen without replacement by ``default_rng(seed)``
    over the row-major list of off-diagonal blocks."""
    nb = (N + BLOCK - 1) // BLOCK
    mask = np.zeros((nb, nb), dtype=np.uint8)
    np.fill_diagonal(mask, 1)
    off = np.flatnonzero(~np.eye(nb, dtype=bool))
    k = int(round(density * off.size))
    if k:
        pick = np.random.default_rng(seed).choice(off.size, size=k, replace=False)
        mask.flat[off[pick]] = 1
    return mask


def make_inputs(w: Workload, seed: int = 0, N: Optional[int] = None,
                B: Optional[int] = None, Hq: Optional[int] = None,
                Hkv: Optional[int] = None):
    """Draw the inputs of workload ``w`` (sizes overridable for small cases).

    Returns a dict with float32 arrays ``q, k, v`` (and ``do`` when the
    workload has a backward pass) holding bf16-exact values for bf16
    workloads, plus ``mask`` (uint8 block mask or None).
    """
    N = w.N if N is None else N
    B = w.B if B is None else B
    Hq = w.Hq if Hq is None else Hq
    Hkv = w.Hkv if Hkv is None else Hkv
    if w.dtype == "f32":
        rng = np.random.default_rng(seed)
        q = rng.normal(size=(N, w.d)).astype(np.float32)
        k = rng.normal(size=(N, w.d)).astype(np.float32)
        v = rng.normal(size=(N, w.d)).astype(np.float32)
        out = {"q": q.reshape(1, 1, N, w.d), "k": k.reshape(1, 1, N, w.d),
               "v": v.reshape(1, 1, N, w.d)}
        if w.backward:
            out["do"] = rng.normal(size=(1, 1, N, w.d)).astype(np.float32)
    else:
        rng = np.random.default_rng(seed)
        shq = (B, Hq, N, w.d)
        shk = (B, Hkv, N, w.d)
        out = {"q": bf16_round(rng.standard_normal(shq, dtype=np.float32)),
               "k": bf16_round(rng.standard_normal(shk, dtype=np.float32)),
               "v": bf16_round(rng.standard_normal(shk, dtype=np.float32))}
        if w.backward:
            out["do"] = bf16_round(rng.standard_normal(shq, dtype=np.float32))
    out["mask"] = random_block_mask(N) if w.sparse else None
    return out


def random_case(B: int, Hq: int, Hkv: int, N: int, d: int, seed: int,
                dtype: str = "bf16", mask_density: Optional[float] = None):
    """Small seeded case for edge tests: same recipe as the bf16 workloads
    (or plain float32 normals for ``dtype='f32'``)."""
    rng = np.random.default_rng(seed)
    shq, shk = (B, Hq, N, d), (B, Hkv, N, d)
    draw = (lambda s: bf16_round(rng.standard_normal(s, dtype=np.float32))) \
        if dtype == "bf16" else (lambda s: rng.standard_normal(s, dtype=np.float32))
    out = {"q": draw(shq), "k": draw(shk), "v": draw(shk), "do": draw(shq)}
    out["mask"] = None if mask_density is None else random_block_mask(N, mask_density, seed)
    return out


def allowed_count(N: int, causal: bool, mask: Optional[np.ndarray]) -> int:
    """Number of (query, key) pairs the causal flag and block mask allow for
    one head: N^2 dense, N(N+1)/2 causal, 128^2 per active block (clipped to
    N and to the causal triangle) otherwise. This is the element count the
    FLOP convention multiplies: forward 4*d per element, backward 10*d."""
    if mask is None:
        return N * (N + 1) // 2 if causal else N * N
    nb = mask.shape[0]
    total = 0
    for qb in range(nb):
        r0, r1 = qb * BLOCK, min(N, (qb + 1) * BLOCK)
        for kb in np.flatnonzero(mask[qb]):
            c0, c1 = kb * BLOCK, min(N, (kb + 1) * BLOCK)
            if not causal or c1 - 1 <= r0:
                total += (r1 - r0) * (c1 - c0)
            elif c0 > r1 - 1:
                continue
            else:
                for r in range(r0, r1):
                    total += max(0, min(c1, r + 1) - c0)
    return int(total)


def flops(w_or_dims, N=None, causal=None, mask=None, backward=False) -> float:
    """Algorithmic FLOPs: 4*d per allowed score element forward (two
    matmuls), 10*d backward (five matmuls, the recompute of S included),
    times B*Hq."""
    if isinstance(w_or_dims, Workload):
        w = w_or_dims
        B, Hq, d = w.B, w.Hq, w.d
        N = w.N if N is None else N
        causal = w.causal
    else:
        B, Hq, d = w_or_dims
    per = 10 * d if backward else 4 * d
    return float(per) * allowed_count(N, causal, mask) * B * Hq


def varlen_case(lengths, Hq: int, Hkv: int, d: int, seed: int = 0):
    """A variable-length batch: sequences of the given lengths packed back to
    back. ``default_rng(seed)`` draws Q, K, V, dO in that order as float32
    standard normals of shape [total, H, d] (K and V with Hkv heads), each
    rounded to bfloat16. Returns the arrays, the int32 offsets cu [B + 1]
    and max(lengths)."""
    lengths = [int(n) for n in lengths]
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    total = int(cu[-1])
    rng = np.random.default_rng(seed)
    out = {}
    for name, h in (("q", Hq), ("k", Hkv), ("v", Hkv), ("do", Hq)):
        out[name] = bf16_round(rng.standard_normal((total, h, d), dtype=np.float32))
    out["cu"] = cu
    out["max_seqlen"] = max(lengths) if lengths else 0
    return out


def varlen_lengths(total_target: int, lo: int, hi: int, seed: int = 0):
    """Seeded sequence lengths drawn uniformly from [lo, hi] until their sum
    reaches total_target (the last one is cut so the sum is exact)."""
    rng = np.random.default_rng(seed)
    lengths, s = [], 0
    while s < total_target:
        n = int(min(rng.integers(lo, hi + 1), total_target - s))
        lengths.append(n)
        s += n
    return lengths


def varlen_allowed_count(lengths, causal: bool) -> int:
    """Score elements a variable-length batch computes (per head)."""
    return sum(allowed_count(n, causal, None) for n in lengths)


def window_allowed_count(N: int, causal: bool, left: int, right: int) -> int:
    """Score elements per head under a sliding window (key j visible to
    query i iff i - left <= j <= i + right, -1 unbounded, and j <= i when
    causal), without materialising the N x N pattern."""
    i = np.arange(N, dtype=np.int64)
    lo = np.zeros(N, dtype=np.int64) if left < 0 else np.maximum(i - left, 0)
    hi = np.full(N, N - 1, dtype=np.int64) if right < 0 else np.minimum(i + right, N - 1)
    if causal:
        hi = np.minimum(hi, i)
    return int(np.maximum(hi - lo + 1, 0).sum())
