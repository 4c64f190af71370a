"""The backward kernel's work list, restated on the host: for key tile j it
visits query tiles i_lo .. i_hi with i_lo = j under causality (else 0), and,
with a window and no sink key in the tile, i_hi = the tile holding query
128 j + 127 + window - 1 (bw_unit in bwd_kernel.cuh).  These must be exactly
the (query tile, key tile) pairs that hold a kept pair under the mask rule, so
no gradient term is missed and no empty tile is computed; their number per
head equals the forward's attn_visited_blocks."""
import numpy as np
import pytest

import exact_tiled_attention_44_b200 as A


def bw_pairs(N, causal, window, n_sink):
    W = 0 if window >= N else window
    S = min(n_sink, N) if W > 0 else 0
    nt = (N + 127) // 128
    out = set()
    for j in range(nt):
        i_lo = j if causal else 0
        i_hi = nt - 1
        if W > 0 and j * 128 >= S:
            i_hi = min(i_hi, (j * 128 + 127 + W - 1) // 128)
        out |= {(i, j) for i in range(i_lo, i_hi + 1)}
    return out, W, S


def kept_block_pairs(N, causal, W, S):
    q = np.arange(N)[:, None]
    k = np.arange(N)[None, :]
    keep = np.ones((N, N), bool)
    if causal:
        keep &= k <= q
    if W > 0:
        keep &= (q - k < W) | (k < S)
    nt = (N + 127) // 128
    return {(i, j) for i in range(nt) for j in range(nt)
            if keep[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128].any()}


CASES = [(N, 0, 0, 0) for N in (1, 127, 128, 129, 300, 640)] + [
    (N, 1, W, S) for N in (1, 129, 257, 500, 1000)
    for W, S in ((0, 0), (1, 0), (2, 1), (127, 0), (128, 64), (129, 3), (300, 129), (2000, 5))]


@pytest.mark.parametrize("N,causal,window,n_sink", CASES)
def test_backward_visits_exactly_the_kept_block_pairs(N, causal, window, n_sink):
    pairs, W, S = bw_pairs(N, causal, window, n_sink)
    assert pairs == kept_block_pairs(N, causal, W, S)
    assert len(pairs) == A.visited_blocks(N, causal, window, n_sink)
