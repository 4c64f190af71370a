"""Float64 oracle for the gradients of exact masked attention.

TEST INFRASTRUCTURE ONLY (see ``oracle/definition.py``).

* "USAAIO Lesson 91", slide 9 (backward pass): the backward of Flash
  Attention 2 recomputes the attention tiles from saved statistics instead of
  storing the N x N matrix; the FLOPs are those of standard attention.

The pages give no gradient formulas, so this module takes the plainest
reading: the backward pass returns dQ, dK and dV, the gradients of the scalar
sum(O * dO) for a given upstream gradient dO of the forward's output O
(LSE, a saved statistic, receives no gradient).  They follow from the chain
rule through the definition of ``definition.attention_head``:

    s_ij  = scale * q_i . k_j + bias_ij     (bias: ALiBi, a constant)
    P_ij  = softmax over the kept keys of row i (0 where masked)
    O_i   = sum_j P_ij v_j
    dV_j  = sum_i P_ij dO_i
    dP_ij = dO_i . v_j
    dS_ij = P_ij (dP_ij - D_i),   D_i = sum_j P_ij dP_ij = dO_i . O_i
    dQ_i  = scale sum_j dS_ij k_j
    dK_j  = scale sum_i dS_ij q_i

With grouped K/V heads (slide 32) a K/V head's gradient is the sum over the
query heads that read it.  P is formed by the plain softmax of the
definition, not from a saved LSE, so nothing here borrows the tiled method's
steps.  The tests pin these formulas against central finite differences of
``definition.attention`` and against torch autograd of the same definition.
"""
from __future__ import annotations

import numpy as np

from .definition import alibi_bias, keep_mask, kv_head_of, scores


def backward_head(q, k, v, do, scale, causal, window=0, n_sink=0, slope=0.0):
    """dQ [N, d], dK [N, d], dV [N, d] of one head, all rows at once."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    n = k.shape[0]
    rows = np.arange(q.shape[0])
    s = scores(q, k, scale)
    if slope:
        s = s + alibi_bias(n, slope, rows)
    keep = keep_mask(n, n, causal, window, n_sink, rows)
    if not keep.any(axis=1).all():
        raise ValueError("a query row has no kept key")
    s = np.where(keep, s, -np.inf)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    d_row = (do * o).sum(axis=1)
    ds = p * (dp - d_row[:, None])
    dq = float(scale) * (ds @ k)
    dk = float(scale) * (ds.T @ q)
    return dq, dk, dv


def attention_backward(Q, K, V, dO, scale, causal=False, window=0, n_sink=0, slopes=None):
    """dQ [B, H, N, d], dK and dV [B, H_kv, N, d] (float64) for [B, H, N, d]
    queries, [B, H_kv, N, d] keys/values and upstream gradient dO [B, H, N, d].
    ``slopes``: optional ALiBi slope per query head."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    dO = np.asarray(dO, np.float64)
    B, H, N, d = Q.shape
    H_kv = K.shape[1]
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for b in range(B):
        for h in range(H):
            g = kv_head_of(h, H, H_kv)
            slope = 0.0 if slopes is None else float(slopes[h])
            dq, dk, dv = backward_head(Q[b, h], K[b, g], V[b, g], dO[b, h], scale, causal,
                                       window, n_sink, slope)
            dQ[b, h] = dq
            dK[b, g] += dk
            dV[b, g] += dv
    return dQ, dK, dV


def row_dot(O, dO):
    """D_i = dO_i . O_i per query row ([B, H, N]): the row term of dS."""
    return (np.asarray(O, np.float64) * np.asarray(dO, np.float64)).sum(axis=-1)


def tiled_backward_head(q, k, v, o, do, lse, scale, causal, window=0, n_sink=0, slope=0.0,
                        bs=16):
    """dQ, dK, dV of one head by the tiled recomputation the pages name for
    the Flash Attention 2 backward ("USAAIO Lesson 91", slide 9: the attention
    tiles are recomputed from saved statistics instead of being stored).

    Key blocks outside, query blocks inside.  The saved statistics are the
    forward's output ``o`` and natural-log ``lse``; for each block pair the
    probabilities are recomputed as P = exp(s - LSE) (0 where masked), and
    D_i = dO_i . o_i.  dK and dV of a key block are complete after its inner
    loop; dQ is summed over key blocks.  Ragged last blocks are allowed.
    Float64 throughout.  Used only to pin ``backward_head`` (and to state the
    recomputation in code); it produces no expected value for the GPU.
    """
    q, k, v, o, do = (np.asarray(x, np.float64) for x in (q, k, v, o, do))
    lse = np.asarray(lse, np.float64)
    n = k.shape[0]
    d_row = (do * o).sum(axis=1)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for c0 in range(0, n, bs):
        cols = np.arange(c0, min(n, c0 + bs))
        for r0 in range(0, q.shape[0], bs):
            rows = np.arange(r0, min(q.shape[0], r0 + bs))
            keep = keep_mask(n, n, causal, window, n_sink, rows)[:, cols]
            if not keep.any():
                continue
            s = float(scale) * (q[rows] @ k[cols].T)
            if slope:
                s = s - float(slope) * np.abs(rows[:, None] - cols[None, :])
            p = np.exp(np.where(keep, s - lse[rows][:, None], -np.inf))
            dv[cols] += p.T @ do[rows]
            dp = do[rows] @ v[cols].T
            ds = p * (dp - d_row[rows][:, None])
            dq[rows] += float(scale) * (ds @ k[cols])
            dk[cols] += float(scale) * (ds.T @ q[rows])
    return dq, dk, dv
