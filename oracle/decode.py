"""Float64 oracle for attention of a few new query rows against a K/V cache,
and for the split-KV form that reduces per-split partial results.

TEST INFRASTRUCTURE ONLY (see ``oracle/definition.py``).

* "USAAIO Lesson 91", slide 31 ("MHA KV cache is the inference bottleneck"):
  during autoregressive decoding every new token attends to the whole cache of
  past keys and values; slide 32: with MQA / GQA the query heads share K/V heads.
* "Building a FlashAttention-style tiled self-attention block in pure NumPy",
  "Extending It", item 6: split the sequence dimension across workers, each
  handling a subset of tiles, then reduce the partial outputs.

Readings taken where the pages are open:

* The N_q new query rows of a head sit at cache positions N_kv - N_q + i
  (i = 0 .. N_q - 1): they are the last N_q tokens of the sequence.  The keep
  rule of the forward applies with that position as the query index (causal:
  key j is kept iff j <= N_kv - N_q + i; the window and sinks likewise).
* The reduction of partial outputs is the log-sum-exp merge: a split s over
  key range [lo_s, hi_s) yields O_s (softmax-normalised over its own kept
  keys) and LSE_s; then LSE = ln sum_s exp(LSE_s) and
  O = sum_s exp(LSE_s - LSE) O_s.  A split with no kept key has LSE_s = -inf
  and weight 0.  This is exact: it regroups the sums of the plain softmax.
"""
from __future__ import annotations

import numpy as np

from .definition import attention_head, keep_mask, kv_head_of, scores


def positions(n_q: int, n_kv: int) -> np.ndarray:
    """Cache positions of the new query rows (the last n_q tokens)."""
    if not 1 <= n_q <= n_kv:
        raise ValueError("need 1 <= n_q <= n_kv")
    return np.arange(n_kv - n_q, n_kv)


def decode(Q, K, V, scale, causal=True, window=0, n_sink=0):
    """O [B, H, N_q, d] and LSE [B, H, N_q] of the new rows, plain definition."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    B, H, n_q, _ = Q.shape
    H_kv, n_kv = K.shape[1], K.shape[2]
    rows = positions(n_q, n_kv)
    O = np.empty((B, H, n_q, V.shape[3]))
    L = np.empty((B, H, n_q))
    for b in range(B):
        for h in range(H):
            g = kv_head_of(h, H, H_kv)
            O[b, h], L[b, h] = attention_head(Q[b, h], K[b, g], V[b, g], scale, causal, window,
                                              n_sink, rows)
    return O, L


def partial_head(q, k, v, scale, causal, window, n_sink, rows, lo, hi):
    """(O_s, LSE_s) of query rows ``rows`` over the kept keys in [lo, hi) only.
    O_s is normalised over those keys; a row with none gets O_s = 0, LSE_s = -inf."""
    s = scores(q, k, scale)
    n = k.shape[0]
    keep = keep_mask(n, n, causal, window, n_sink, rows)
    inside = np.zeros(n, bool)
    inside[lo:hi] = True
    keep &= inside[None, :]
    s = np.where(keep, s, -np.inf)
    m = s.max(axis=1)
    has = np.isfinite(m)
    ref = np.where(has, m, 0.0)
    p = np.exp(s - ref[:, None])
    l = p.sum(axis=1)
    o = np.where(has[:, None], (p @ np.asarray(v, np.float64)) / np.where(has, l, 1.0)[:, None], 0.0)
    lse = np.where(has, ref + np.log(np.where(has, l, 1.0)), -np.inf)
    return o, lse


def merge_partials(O_parts, LSE_parts):
    """Log-sum-exp merge of per-split partial results.

    O_parts: [S, ..., d]; LSE_parts: [S, ...].  Returns (O [..., d], LSE [...]).
    """
    O_parts = np.asarray(O_parts, np.float64)
    L = np.asarray(LSE_parts, np.float64)
    m = L.max(axis=0)
    w = np.exp(L - m[None])                      # exp(-inf) = 0 for empty splits
    tot = w.sum(axis=0)
    lse = m + np.log(tot)
    o = (w[..., None] * O_parts).sum(axis=0) / tot[..., None]
    return o, lse


def decode_split(Q, K, V, scale, causal=True, window=0, n_sink=0, bounds=(0,)):
    """The split-KV form: key ranges [bounds[s], bounds[s+1]) (the last range ends at
    N_kv), partial results per range, then the log-sum-exp merge."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    B, H, n_q, _ = Q.shape
    H_kv, n_kv = K.shape[1], K.shape[2]
    rows = positions(n_q, n_kv)
    edges = list(bounds) + [n_kv]
    O = np.empty((B, H, n_q, V.shape[3]))
    L = np.empty((B, H, n_q))
    for b in range(B):
        for h in range(H):
            g = kv_head_of(h, H, H_kv)
            parts = [partial_head(Q[b, h], K[b, g], V[b, g], scale, causal, window, n_sink, rows,
                                  edges[s], edges[s + 1]) for s in range(len(edges) - 1)]
            O[b, h], L[b, h] = merge_partials([p[0] for p in parts], [p[1] for p in parts])
    return O, L
