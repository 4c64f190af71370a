"""Float64 CPU oracle for exact masked attention with log-sum-exp.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, header, table or helper with the CUDA library and imports nothing
from it.

What it computes is the plain definition, not the tiled algorithm, because the
pages state that the tiled method reaches that definition exactly:

* "Flash Attention" (dileepadev learn-ai), section "The Problem with Standard
  Attention": Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V; section
  "Mathematical Equivalence": the tiled form gives the same output, it is not
  an approximation.
* "Tiled attention with online softmax" (Lab 3): the ``reference`` function
  forms the whole score matrix, masks the future with a lower-triangular keep
  mask, subtracts the row max, exponentiates and normalises.
* "Hands-On Build Guide: Flash Attention Implementation from Scratch in
  NumPy", Step 2 (causal mask, True = keep on and below the diagonal) and
  Step 7 (the naive full-matrix check).
* "USAAIO Lesson 91", slide 32 (MQA: H query heads share one K/V head; GQA:
  G groups of query heads share one K/V head each).
* "USAAIO Lesson 91", slides 20-23 (ALiBi position bias): the logit of query i
  and key j gets -m_h * |i - j| added before the softmax, with one slope per
  head, m_h = 2^(-h * 8 / H) for h = 1 .. H.

Readings taken where the pages are open:

* keep(i, j) = (not causal or j <= i) and (window == 0 or i - j < window or
  j < n_sink).  The window counts the query itself; sink keys are the first
  ``n_sink`` positions and stay subject to causality (Lab 3, exercise 4 poses
  sinks plus a sliding window without defining them).
* ``scale`` multiplies Q K^T before masking; 0 is a legal scale.
* LSE_i = ln sum_{j kept} exp(scale * q_i . k_j), natural log, per query row
  (the Hands-On Build Guide, Step 5, names a log-sum-exp carried across tiles
  without defining it).
* Query head h reads K/V head h // (H // H_kv).
* A row with no kept key is an error here (the API never produces one: the
  diagonal is always kept).
* With ALiBi the bias is added to the scaled logits, scale * q.k - m_h |i - j|
  (slide 20 writes the scale as 1 / sqrt(d)), before masking; LSE is then the
  log-sum-exp of the biased logits.

All arithmetic is float64.  Inputs are expected to be the exact float64
upcast of the 16-bit values the GPU consumes.
"""
from __future__ import annotations

import numpy as np

# Rows per chunk when the full score matrix of one head would exceed this many
# float64 entries (1 GiB).  Each chunk holds complete score rows, so the
# softmax of every row is still the plain one.
_MAX_SCORE_ENTRIES = (1 << 30) // 8
_ROW_CHUNK = 2048


def keep_mask(n_q: int, n_k: int, causal: bool, window: int = 0, n_sink: int = 0,
              rows: np.ndarray | None = None) -> np.ndarray:
    """Boolean keep mask (True = the key is attended), shape [len(rows), n_k].

    Causal rule as in the Hands-On Build Guide, Step 2 (``np.tri``: on and
    below the diagonal is kept) and Lab 3's per-block ``i >= j`` test; window
    and sink rule as read above.
    """
    i = (np.arange(n_q) if rows is None else np.asarray(rows))[:, None]
    j = np.arange(n_k)[None, :]
    keep = np.ones((i.shape[0], n_k), dtype=bool)
    if causal:
        keep &= j <= i
    if window > 0:
        keep &= (i - j < window) | (j < n_sink)
    return keep


def alibi_slopes(H: int) -> np.ndarray:
    """ALiBi slopes of H heads: the geometric sequence m_h = 2^(-h * 8 / H),
    h = 1 .. H ("USAAIO Lesson 91", slide 23), in float64."""
    if H < 1:
        raise ValueError("H must be positive")
    return np.array([2.0 ** (-h * 8.0 / H) for h in range(1, H + 1)])


def alibi_bias(n_k: int, slope: float, rows: np.ndarray) -> np.ndarray:
    """-slope * |i - j| for query rows ``rows`` and keys 0 .. n_k - 1
    ("USAAIO Lesson 91", slide 20: logit(i, j) = q_i.k_j / sqrt(d) - m_h |i - j|)."""
    i = np.asarray(rows, np.float64)[:, None]
    j = np.arange(n_k, dtype=np.float64)[None, :]
    return -float(slope) * np.abs(i - j)


def scores(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """scale * q k^T in float64 (the logits before masking)."""
    return float(scale) * (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T)


def attention_weights(q, k, scale, causal, window=0, n_sink=0, rows=None):
    """The explicit softmax matrix P (rows of it), masked entries exactly 0."""
    s = scores(q, k, scale)
    keep = keep_mask(k.shape[0], k.shape[0], causal, window, n_sink, rows)
    if not keep.any(axis=1).all():
        raise ValueError("a query row has no kept key")
    s = np.where(keep, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return p / p.sum(axis=1, keepdims=True)


def attention_head(q, k, v, scale, causal, window=0, n_sink=0, rows=None, slope=0.0):
    """O and LSE for one head.

    q: [n_rows, d] (the query rows ``rows`` of the head, or all of them),
    k, v: [N, d]; ``slope``: the head's ALiBi slope (0 = no bias).
    Returns (O [n_rows, d], LSE [n_rows]).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n = k.shape[0]
    if rows is None:
        rows = np.arange(q.shape[0])
    rows = np.asarray(rows)
    s = scores(q, k, scale)
    if slope:
        s = s + alibi_bias(n, slope, rows)
    keep = keep_mask(n, n, causal, window, n_sink, rows)
    if not keep.any(axis=1).all():
        raise ValueError("a query row has no kept key")
    s = np.where(keep, s, -np.inf)
    m = s.max(axis=1)
    p = np.exp(s - m[:, None])
    l = p.sum(axis=1)
    o = (p @ v) / l[:, None]
    lse = m + np.log(l)
    return o, lse


def kv_head_of(h: int, H: int, H_kv: int) -> int:
    """K/V head read by query head h (USAAIO Lesson 91, slide 32, GQA/MQA)."""
    if H % H_kv:
        raise ValueError("H must be a multiple of H_kv")
    return h // (H // H_kv)


def attention(Q, K, V, scale, causal=False, window=0, n_sink=0, slopes=None):
    """Full forward for [B, H, N, d] queries and [B, H_kv, N, d] keys/values.

    ``slopes``: optional ALiBi slope per query head ([H]).
    Returns (O [B, H, N, d] float64, LSE [B, H, N] float64).
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    B, H, N, d = Q.shape
    H_kv = K.shape[1]
    O = np.empty((B, H, N, V.shape[3]))
    L = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            O[b, h], L[b, h] = attention_bh(Q, K, V, b, h, scale, causal, window, n_sink,
                                            slopes=slopes)
    return O, L


def attention_bh(Q, K, V, b, h, scale, causal=False, window=0, n_sink=0, rows=None,
                 slopes=None):
    """O and LSE of head (b, h) for all query rows, or the given ``rows``."""
    slope = 0.0 if slopes is None else float(slopes[h])
    H, N = Q.shape[1], Q.shape[2]
    g = kv_head_of(h, H, K.shape[1])
    q_all = Q[b, h]
    k = np.asarray(K[b, g], np.float64)
    v = np.asarray(V[b, g], np.float64)
    if rows is None:
        rows = np.arange(N)
    rows = np.asarray(rows)
    if rows.size * N <= _MAX_SCORE_ENTRIES:
        return attention_head(np.asarray(q_all[rows], np.float64), k, v, scale,
                              causal, window, n_sink, rows, slope)
    o = np.empty((rows.size, V.shape[3]))
    lse = np.empty(rows.size)
    for c0 in range(0, rows.size, _ROW_CHUNK):
        r = rows[c0:c0 + _ROW_CHUNK]
        o[c0:c0 + r.size], lse[c0:c0 + r.size] = attention_head(
            np.asarray(q_all[r], np.float64), k, v, scale, causal, window, n_sink, r, slope)
    return o, lse


def kept_pairs(N: int, causal: bool, window: int = 0, n_sink: int = 0) -> int:
    """Number of kept (query, key) pairs of one head, by enumerating the mask."""
    total = 0
    for c0 in range(0, N, _ROW_CHUNK):
        r = np.arange(c0, min(N, c0 + _ROW_CHUNK))
        total += int(keep_mask(N, N, causal, window, n_sink, r).sum())
    return total
