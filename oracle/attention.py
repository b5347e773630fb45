"""fp64 CPU oracle for exact scaled-dot-product attention (test infrastructure).

THIS IS TEST INFRASTRUCTURE. Only the tests, the smoke check of
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it. The
CUDA path never calls it and shares no code with it.

What it computes follows the FlashAttention pages:

* the definition O = softmax(Q K^T * scale) V of one head (Pranay Mahendrakar,
  "FlashAttention", Researcher section "The problem being solved"), with the
  softmax taken safely by subtracting the row maximum (Developer section,
  "The three running quantities");
* the per-row statistic the forward pass keeps for the backward pass (paper
  summary, "Core Idea" item 3, and Researcher section "IO complexity"): the
  natural-log logsumexp LSE_i = m_i + ln(l_i) of the scaled scores, from which
  P = exp(S - LSE);
* the causal flag (Developer section, "Common mistakes": use the flag rather
  than a dense mask), the 128x128 block-sparse mask (paper summary, "Key Method
  Details": block-sparse extension) and grouped-query heads (glossary page,
  "FlashAttention-2 Improvements / Multi-Query Attention Support").

The pages give no backward formulas; the oracle takes the textbook gradient of
softmax(S) V: dV = P^T dO, dP = dO V^T, D_i = sum_k dO_ik O_ik, dS = P*(dP - D),
dQ = scale * dS K, dK = scale * dS^T Q, with dK and dV summed over the query
heads that share a KV head.

Everything is the plain definition: full rows of scores are formed (in row
chunks only so that memory stays bounded; every row is complete before it is
normalised). Disallowed pairs are set to -inf; a row with no allowed key gets
O = 0, LSE = -inf and zero gradients. ``tiled_forward`` restates the pages'
online-softmax recurrence separately (as a fold of per-tile summaries); it is
used only to pin ``forward`` against the pages' own worked example.

Layouts: Q, dO, O [B, Hq, N, d]; K, V [B, Hkv, N, d]; LSE [B, Hq, N];
block_mask uint8 [ceil(N/128), ceil(N/128)] shared by every (batch, head).
"""
from __future__ import annotations

import functools

import numpy as np

BLOCK = 128
ROW_CHUNK = 512


def allowed(rows: np.ndarray, N: int, causal: bool, block_mask, window=None, prefix: int = 0,
            doc=None) -> np.ndarray:
    """Boolean [len(rows), N]: whether key j is visible to query i.

    Key j is visible to query i iff all of these hold:
      * right bound: (not causal or j <= i) and, for a sliding window
        (left, right) with right >= 0, j <= i + right -- unless j < prefix:
        the first ``prefix`` keys are visible to every query whatever the
        causal flag and the right bound say (a prefix language model: the
        prefix attends to itself in both directions);
      * left bound: for a window with left >= 0, j >= i - left;
      * documents: ``doc`` (int array [N] of per-token document ids, or None)
        has doc[j] == doc[i];
      * block mask: mask[i // 128, j // 128] is non-zero (no mask: all on).
    A negative window bound means unbounded. The prefix and document rules are
    mask modifiers in the sense of the lesson's Researcher section ("Beyond
    hand-written kernels"): one tiled kernel, many masks."""
    rows = np.asarray(rows)
    cols = np.arange(N)
    right = np.ones((rows.size, N), dtype=bool)
    left = np.ones((rows.size, N), dtype=bool)
    if causal:
        right &= cols[None, :] <= rows[:, None]
    if window is not None:
        wl, wr = window
        if wl >= 0:
            left &= cols[None, :] >= rows[:, None] - wl
        if wr >= 0:
            right &= cols[None, :] <= rows[:, None] + wr
    if prefix > 0:
        right |= cols[None, :] < prefix
    ok = left & right
    if doc is not None:
        doc = np.asarray(doc)
        ok &= doc[rows][:, None] == doc[None, :N]
    if block_mask is not None:
        ok &= block_mask[(rows // BLOCK)[:, None], (cols // BLOCK)[None, :]].astype(bool)
    return ok


def scores(Qr, Kh, scale, softcap: float = 0.0):
    """Scores of query rows Qr against keys Kh and the scaled products they
    come from: X = scale * Qr Kh^T, and S = X, or S = softcap * tanh(X / softcap)
    when softcap > 0 (soft-capping, a score modifier in the FlexAttention
    sense of the lesson's Researcher section, "Beyond hand-written kernels").
    Returns (S, X)."""
    X = scale * (Qr @ Kh.T)
    if softcap > 0:
        return softcap * np.tanh(X / softcap), X
    return X, X


def score_grad(dS, X, softcap: float = 0.0):
    """Chain rule through the score modifier: the gradient with respect to
    X = scale * Q K^T of a gradient dS with respect to S(X). Soft-capping has
    dS/dX = 1 - tanh(X / softcap)^2."""
    if softcap > 0:
        t = np.tanh(X / softcap)
        return dS * (1.0 - t * t)
    return dS


def softmax_rows(S: np.ndarray):
    """Safe softmax of each row of S (entries -inf are excluded).

    Returns (P, LSE). Rows that are entirely -inf give P = 0, LSE = -inf.
    """
    m = S.max(axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    E = np.exp(S - m_safe[:, None])
    l = E.sum(axis=1)
    l_safe = np.where(empty, 1.0, l)
    P = E / l_safe[:, None]
    lse = np.where(empty, -np.inf, m_safe + np.log(l_safe))
    return P, lse


def _kv_head(h: int, Hq: int, Hkv: int) -> int:
    return h // (Hq // Hkv)


def forward_rows(Q, K, V, scale, causal, block_mask, b, h, rows, window=None, prefix=0,
                 doc=None, softcap=0.0):
    """O and LSE of query rows ``rows`` of head (b, h), in fp64. The mask and
    score modifiers (window, prefix, doc, softcap) are those of ``allowed`` and
    ``scores``; LSE is the logsumexp of the (modified) scores."""
    Hq, Hkv, N = Q.shape[1], K.shape[1], K.shape[2]
    hk = _kv_head(h, Hq, Hkv)
    Kh = K[b, hk].astype(np.float64)
    Vh = V[b, hk].astype(np.float64)
    rows = np.asarray(rows)
    O = np.empty((rows.size, Q.shape[3]))
    L = np.empty(rows.size)
    for c in range(0, rows.size, ROW_CHUNK):
        r = rows[c:c + ROW_CHUNK]
        S, _ = scores(Q[b, h, r].astype(np.float64), Kh, scale, softcap)
        S[~allowed(r, N, causal, block_mask, window, prefix, doc)] = -np.inf
        P, lse = softmax_rows(S)
        O[c:c + r.size] = P @ Vh
        L[c:c + r.size] = lse
    return O, L


def forward(Q, K, V, scale, causal=False, block_mask=None, window=None, prefix=0, doc=None,
            softcap=0.0):
    """O [B,Hq,N,d] and LSE [B,Hq,N] in fp64 for all heads."""
    B, Hq, N, d = Q.shape
    O = np.empty((B, Hq, N, d))
    L = np.empty((B, Hq, N))
    rows = np.arange(N)
    for b in range(B):
        for h in range(Hq):
            O[b, h], L[b, h] = forward_rows(Q, K, V, scale, causal, block_mask, b, h, rows,
                                            window, prefix, doc, softcap)
    return O, L


def _head_grads(Qh, Kh, Vh, dOh, Oh, scale, causal, block_mask, rows, want_dq=True,
                window=None, prefix=0, doc=None, softcap=0.0):
    """Gradient pieces of one query head restricted to query rows ``rows``.

    Returns (dQ_rows or None, dK contribution [N,d], dV contribution [N,d]).
    """
    N = Kh.shape[0]
    dK = np.zeros_like(Kh)
    dV = np.zeros_like(Vh)
    dQ = np.zeros((rows.size, Qh.shape[1])) if want_dq else None
    for c in range(0, rows.size, ROW_CHUNK):
        r = rows[c:c + ROW_CHUNK]
        S, X = scores(Qh[r], Kh, scale, softcap)
        S[~allowed(r, N, causal, block_mask, window, prefix, doc)] = -np.inf
        P, _ = softmax_rows(S)
        dP = dOh[r] @ Vh.T
        D = np.sum(dOh[r] * Oh[r], axis=1)
        dS = score_grad(P * (dP - D[:, None]), X, softcap)
        dV += P.T @ dOh[r]
        dK += scale * (dS.T @ Qh[r])
        if want_dq:
            dQ[c:c + r.size] = scale * (dS @ Kh)
    return dQ, dK, dV


def backward(Q, K, V, dO, scale, causal=False, block_mask=None, O=None, window=None, prefix=0,
             doc=None, softcap=0.0):
    """dQ [B,Hq,N,d], dK and dV [B,Hkv,N,d] in fp64.

    O is the oracle's own forward output (recomputed here when not given).
    """
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    if O is None:
        O, _ = forward(Q, K, V, scale, causal, block_mask, window, prefix, doc, softcap)
    dQ = np.zeros((B, Hq, N, d))
    dK = np.zeros((B, Hkv, N, d))
    dV = np.zeros((B, Hkv, N, d))
    rows = np.arange(N)
    for b in range(B):
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            dq, dk, dv = _head_grads(Q[b, h].astype(np.float64), K[b, hk].astype(np.float64),
                                     V[b, hk].astype(np.float64), dO[b, h].astype(np.float64),
                                     O[b, h], scale, causal, block_mask, rows,
                                     window=window, prefix=prefix, doc=doc, softcap=softcap)
            dQ[b, h] = dq
            dK[b, hk] += dk
            dV[b, hk] += dv
    return dQ, dK, dV


def dq_rows(Q, K, V, dO, scale, causal, block_mask, b, h, rows, window=None, prefix=0,
            doc=None, softcap=0.0):
    """dQ of query rows ``rows`` of head (b, h) (needs only those rows)."""
    Hq, Hkv = Q.shape[1], K.shape[1]
    hk = _kv_head(h, Hq, Hkv)
    rows = np.asarray(rows)
    O, _ = forward_rows(Q, K, V, scale, causal, block_mask, b, h, rows, window, prefix, doc,
                        softcap)
    Oh = np.zeros((Q.shape[2], Q.shape[3]))
    Oh[rows] = O
    dq, _, _ = _head_grads(Q[b, h].astype(np.float64), K[b, hk].astype(np.float64),
                           V[b, hk].astype(np.float64), dO[b, h].astype(np.float64),
                           Oh, scale, causal, block_mask, rows, window=window, prefix=prefix,
                           doc=doc, softcap=softcap)
    return dq


def dkdv_rows(Q, K, V, dO, scale, causal, block_mask, b, hk, key_rows, window=None, prefix=0,
              doc=None, softcap=0.0):
    """dK and dV of key rows ``key_rows`` of KV head (b, hk).

    Every query row that can see one of those keys contributes; for each one
    the full score row is formed (its LSE and O need all keys).
    """
    Hq, Hkv, N = Q.shape[1], K.shape[1], K.shape[2]
    g = Hq // Hkv
    key_rows = np.asarray(key_rows)
    dK = np.zeros((key_rows.size, K.shape[3]))
    dV = np.zeros((key_rows.size, K.shape[3]))
    qrows = np.flatnonzero(np.concatenate([
        allowed(np.arange(c, min(N, c + ROW_CHUNK)), N, causal, block_mask, window, prefix,
                doc)[:, key_rows].any(axis=1) for c in range(0, N, ROW_CHUNK)]))
    Kh = K[b, hk].astype(np.float64)
    Vh = V[b, hk].astype(np.float64)
    for h in range(hk * g, (hk + 1) * g):
        Qh = Q[b, h].astype(np.float64)
        dOh = dO[b, h].astype(np.float64)
        for c in range(0, qrows.size, ROW_CHUNK):
            r = qrows[c:c + ROW_CHUNK]
            S, X = scores(Qh[r], Kh, scale, softcap)
            S[~allowed(r, N, causal, block_mask, window, prefix, doc)] = -np.inf
            P, _ = softmax_rows(S)
            O = P @ Vh
            D = np.sum(dOh[r] * O, axis=1)
            Pk = P[:, key_rows]
            dPk = dOh[r] @ Vh[key_rows].T
            dSk = score_grad(Pk * (dPk - D[:, None]), X[:, key_rows], softcap)
            dV += Pk.T @ dOh[r]
            dK += scale * (dSk.T @ Qh[r])
    return dK, dV


def tiled_forward(Q2, K2, V2, scale, block, dtype=np.float64, trace=None):
    """The online-softmax recurrence for one head (lesson, Researcher section
    "Online softmax", after Milakov and Gimelshein), written as a left fold of
    per-tile summaries.

    Key tile j (``block`` keys wide) is first summarised on its own as a
    triple: its row maxima M_j, the row sums L_j of exp(S^(j) - M_j) and the
    unnormalised partial output U_j = exp(S^(j) - M_j) V^(j). The running state
    after tile j, (m^(j), l^(j), O^(j)), merges the state after tile j - 1 with
    that triple: m^(j) = max(m^(j-1), M_j), and each side is carried onto the
    new maximum by its own factor, exp(m^(j-1) - m^(j)) or exp(M_j - m^(j)),
    before the two are added. Since rowsum(exp(S^(j) - m^(j))) equals
    exp(M_j - m^(j)) L_j, this is the page's recurrence term for term; the
    result is O^(T) / l^(T). All arithmetic is done in ``dtype``. If ``trace``
    is a list, the number of rows whose running maximum grew is appended for
    each tile.
    """
    Q2, K2, V2 = (np.asarray(a_, dtype=dtype) for a_ in (Q2, K2, V2))
    sc = dtype(scale)

    def summary(j0):
        S = (Q2 @ K2[j0:j0 + block].T) * sc
        M = S.max(axis=1)
        E = np.exp(S - M[:, None])
        return M, E.sum(axis=1), E @ V2[j0:j0 + block]

    def merge(state, tile):
        m_prev, l_prev, O_prev = state
        M, L, U = tile
        m_next = np.maximum(m_prev, M)
        if trace is not None:
            trace.append(int(np.count_nonzero(m_next > m_prev)))
        keep = np.exp(m_prev - m_next)     # 0 while nothing has been accumulated
        bring = np.exp(M - m_next)
        return m_next, keep * l_prev + bring * L, keep[:, None] * O_prev + bring[:, None] * U

    rows = Q2.shape[0]
    empty = (np.full(rows, -np.inf, dtype=dtype), np.zeros(rows, dtype=dtype),
             np.zeros((rows, V2.shape[1]), dtype=dtype))
    _, l_fin, O_fin = functools.reduce(merge, map(summary, range(0, K2.shape[0], block)), empty)
    return O_fin / l_fin[:, None]


def naive_forward_f32(Q2, K2, V2, scale):
    """The one-shot float32 result for one head that the lesson checks its
    loop against: the whole N x N score matrix is formed and every row is
    normalised by its logsumexp (taken about the row maximum so that no
    exponential overflows) before the product with V."""
    f32 = np.float32
    S = np.matmul(np.asarray(Q2, dtype=f32), np.asarray(K2, dtype=f32).T) * f32(scale)
    top = S.max(axis=1, keepdims=True)
    lse = top + np.log(np.exp(S - top).sum(axis=1, keepdims=True))
    return np.exp(S - lse) @ np.asarray(V2, dtype=f32)


# ---------------------------------------------------------------- variable-length batches
#
# A packed batch of B sequences (glossary page, "Sequence Length Flexibility"):
# sequence b is rows cu[b] .. cu[b+1]-1 of Q, K, V [total, H, d] and attends
# only to itself. By definition it is the per-sequence attention above, so
# the oracle applies forward / backward to each slice (as a batch of one) and
# writes the results back in the packed layout; LSE is [Hq, total].

def _seq(x, s0, s1):
    """[s1 - s0, H, d] slice -> [1, H, n, d]."""
    return np.ascontiguousarray(np.transpose(x[s0:s1], (1, 0, 2))[None])


def forward_varlen(Q, K, V, cu, scale, causal=False):
    total, Hq, d = Q.shape
    O = np.zeros((total, Hq, d))
    L = np.full((Hq, total), -np.inf)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        if s1 == s0:
            continue
        Ob, Lb = forward(_seq(Q, s0, s1), _seq(K, s0, s1), _seq(V, s0, s1), scale, causal)
        O[s0:s1] = np.transpose(Ob[0], (1, 0, 2))
        L[:, s0:s1] = Lb[0]
    return O, L


def backward_varlen(Q, K, V, dO, cu, scale, causal=False):
    dQ = np.zeros(Q.shape)
    dK = np.zeros(K.shape)
    dV = np.zeros(V.shape)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        if s1 == s0:
            continue
        g = backward(_seq(Q, s0, s1), _seq(K, s0, s1), _seq(V, s0, s1), _seq(dO, s0, s1), scale,
                     causal)
        for dst, src in zip((dQ, dK, dV), g):
            dst[s0:s1] = np.transpose(src[0], (1, 0, 2))
    return dQ, dK, dV
