"""Float64 tiled online-softmax attention, in the two loop orders the pages show.

TEST INFRASTRUCTURE ONLY (see ``oracle/definition.py``).  These functions exist
to pin the plain-definition oracle: the pages claim the tiled computation and
the full-matrix computation agree, so each is checked against the other on the
CPU.  Neither is used to produce an expected value for the GPU.

* ``tiled_q_outer`` takes query blocks outside and key blocks inside, as
  "Tiled attention with online softmax" (Lab 3) does, but is written from the
  statement in "Flash Attention", section "Mathematical Equivalence": the
  softmax statistics of disjoint key sets combine exactly, because
  exp(x - m) = exp(x - m') exp(m' - m).  Each key block of a query block gives
  a partial result on its own (row max, row sum of exponentials, unnormalised
  output); the partials are folded together with that identity, and blocks
  holding no kept pair are left out (which, for a causal mask, is Lab 3's
  skipping of key blocks after the query block).
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

import functools

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


def _partial(s, v):
    """Statistics of one block of masked scores s [r, c] taken alone: the row
    max, the row sum of exp(s - max) and the unnormalised output (rows whose
    keys are all masked give max -inf, sum 0 and output 0)."""
    m = s.max(axis=1)
    ref = np.where(np.isneginf(m), 0.0, m)
    e = np.exp(s - ref[:, None])
    return m, e.sum(axis=1), e @ v


def _combine(a, b):
    """Partial results over two disjoint key sets, brought to the larger max."""
    (m1, l1, o1), (m2, l2, o2) = a, b
    m = np.maximum(m1, m2)
    ref = np.where(np.isneginf(m), 0.0, m)
    w1 = np.where(np.isneginf(m1), 0.0, np.exp(m1 - ref))
    w2 = np.where(np.isneginf(m2), 0.0, np.exp(m2 - ref))
    return m, w1 * l1 + w2 * l2, w1[:, None] * o1 + w2[:, None] * o2


def tiled_q_outer(q, k, v, scale, causal, window=0, n_sink=0, bs=16, slope=0.0):
    """Q-outer / KV-inner tiled attention of one head; returns (O, LSE)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n, d = q.shape[0], v.shape[1]
    out = np.zeros((n, d))
    lse = np.zeros(n)
    starts = range(0, n, bs)
    for i in starts:
        rows = np.arange(i, min(n, i + bs))
        keep = keep_mask(n, n, causal, window, n_sink, rows)
        parts = []
        for j in starts:
            cols = np.arange(j, min(n, j + bs))
            kb = keep[:, cols]
            if not kb.any():
                continue                      # no kept pair: the block is skipped
            s = scale * (q[rows] @ k[cols].T)
            if slope:
                s = s - slope * np.abs(rows[:, None] - cols[None, :])
            parts.append(_partial(np.where(kb, s, -np.inf), v[cols]))
        m, l, o = functools.reduce(_combine, parts)
        out[rows] = o / l[:, None]
        lse[rows] = m + np.log(l)
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
