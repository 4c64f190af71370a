"""Float64 tiled online-softmax attention, in the two loop orders the pages show.

TEST INFRASTRUCTURE ONLY (see ``oracle/definition.py``).  These functions exist
to pin the plain-definition oracle: the pages claim the tiled computation and
the full-matrix computation agree, so each is checked against the other on the
CPU.  Neither is used to produce an expected value for the GPU.

* ``tiled_q_outer`` follows "Tiled attention with online softmax" (Lab 3):
  query blocks outside, key blocks inside, per-row running max m, running
  denominator l and running numerator o, rescaled by exp(m_old - m_new) when a
  block raises the max, key blocks after the query block skipped when causal,
  and o / l written once per query block.
* ``tiled_kv_outer`` follows "USAAIO Lesson 91", slide 11 ("Online softmax:
  tiled update equations"): key blocks outside, query blocks inside, m, l and O
  for every row kept across the whole pass, normalised at the end.

Both accept a ragged last block (Lab 3, exercise 1: the block size need not
divide N).  One reading is added to the pages' update: when every key seen so
far in a row is masked, m_new is -inf and exp(m_old - m_new) would be
exp(-inf + inf) = NaN, so the rescale factor is taken as 0 there (nothing has
been accumulated yet) and the exponent reference is taken as 0.

With ALiBi ("USAAIO Lesson 91", slides 20-23) each tile's logits get
-slope * |i - j| added before masking, exactly as in the full matrix.
"""
from __future__ import annotations

import numpy as np

from .definition import keep_mask, kv_head_of


def _block_update(m, l, o, s, v):
    """One online-softmax step for a block of rows.

    m, l: [r]; o: [r, d]; s: [r, c] masked scores (-inf = dropped); v: [c, d].
    """
    m_new = np.maximum(m, s.max(axis=1))
    ref = np.where(np.isneginf(m_new), 0.0, m_new)
    alpha = np.where(np.isneginf(m), 0.0, np.exp(m - ref))
    p = np.exp(s - ref[:, None])
    l = alpha * l + p.sum(axis=1)
    o = alpha[:, None] * o + p @ v
    return m_new, l, o


def tiled_q_outer(q, k, v, scale, causal, window=0, n_sink=0, bs=16, slope=0.0):
    """Q-outer / KV-inner tiled attention of one head; returns (O, LSE)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n, d = q.shape[0], v.shape[1]
    out = np.zeros((n, d))
    lse = np.zeros(n)
    for i in range(0, n, bs):
        qi = q[i:i + bs]
        rows = np.arange(i, i + qi.shape[0])
        m = np.full(qi.shape[0], -np.inf)
        l = np.zeros(qi.shape[0])
        o = np.zeros((qi.shape[0], d))
        # With a causal mask no key after the last row of this block is kept.
        j_end = min(n, i + qi.shape[0]) if causal else n
        for j in range(0, j_end, bs):
            kj, vj = k[j:j + bs], v[j:j + bs]
            s = scale * (qi @ kj.T)
            if slope:
                s = s - slope * np.abs(rows[:, None] - np.arange(j, j + kj.shape[0])[None, :])
            keep = keep_mask(n, n, causal, window, n_sink, rows)[:, j:j + kj.shape[0]]
            s = np.where(keep, s, -np.inf)
            m, l, o = _block_update(m, l, o, s, vj)
        out[i:i + qi.shape[0]] = o / l[:, None]
        lse[i:i + qi.shape[0]] = m + np.log(l)
    return out, lse


def tiled_kv_outer(q, k, v, scale, causal, window=0, n_sink=0, bs=16, slope=0.0):
    """KV-outer / Q-inner tiled attention of one head; returns (O, LSE)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n, d = q.shape[0], v.shape[1]
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    o = np.zeros((n, d))
    for j in range(0, n, bs):
        kj, vj = k[j:j + bs], v[j:j + bs]
        for i in range(0, n, bs):
            rows = np.arange(i, min(n, i + bs))
            s = scale * (q[i:i + bs] @ kj.T)
            if slope:
                s = s - slope * np.abs(rows[:, None] - np.arange(j, j + kj.shape[0])[None, :])
            keep = keep_mask(n, n, causal, window, n_sink, rows)[:, j:j + kj.shape[0]]
            s = np.where(keep, s, -np.inf)
            m[rows], l[rows], o[rows] = _block_update(m[rows], l[rows], o[rows], s, vj)
    return o / l[:, None], m + np.log(l)


def tiled_attention(Q, K, V, scale, causal=False, window=0, n_sink=0, bs=16, order="q",
                    slopes=None):
    """Batched wrapper over [B, H, N, d] / [B, H_kv, N, d] inputs."""
    fn = tiled_q_outer if order == "q" else tiled_kv_outer
    B, H, N = Q.shape[:3]
    O = np.empty((B, H, N, V.shape[3]))
    L = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            g = kv_head_of(h, H, K.shape[1])
            sl = 0.0 if slopes is None else float(slopes[h])
            O[b, h], L[b, h] = fn(Q[b, h], K[b, g], V[b, g], scale, causal, window, n_sink, bs,
                                  sl)
    return O, L
