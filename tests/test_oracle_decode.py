"""Pins of the decode / split-KV oracle ("USAAIO Lesson 91", slides 31-32;
"Building a FlashAttention-style tiled self-attention block in pure NumPy",
"Extending It", item 6).

The decode rows are checked against the full forward computed on a sequence
whose last rows are those queries, against brute-force loops, and the
split-and-merge form against the unsplit one; planted mistakes must be caught.
"""
import math

import numpy as np
import pytest

import oracle
from exact_tiled_attention_44_b200.inputs import random_qkv, to_f64


def _qkv(B, H, H_kv, n_q, n_kv, d, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, n_q, d))
    k = rng.standard_normal((B, H_kv, n_kv, d))
    v = rng.standard_normal((B, H_kv, n_kv, d))
    return q, k, v


CASES = [(True, 0, 0), (False, 0, 0), (True, 37, 5), (True, 1, 0), (True, 400, 3)]


# impl(Q, K, V, scale, causal, window, n_sink) -> (O, LSE)   [decode semantics]

def pin_last_rows_of_full_forward(impl):
    """The decode rows are the last rows of the ordinary forward over the whole
    sequence (same keys, queries placed at the end)."""
    for causal, w, ns in CASES:
        q, k, v = _qkv(2, 4, 2, 3, 150, 16, seed=1)
        O, L = impl(q, k, v, 0.25, causal, w, ns)
        qf = np.random.default_rng(2).standard_normal((2, 4, 150, 16))
        qf[:, :, -3:] = q
        Of, Lf = oracle.attention(qf, k, v, 0.25, causal, w, ns)
        assert np.abs(O - Of[:, :, -3:]).max() < 1e-13 and np.abs(L - Lf[:, :, -3:]).max() < 1e-13


def pin_brute_force(impl):
    q, k, v = _qkv(1, 2, 1, 2, 6, 3, seed=4)
    for causal, w, ns in [(True, 0, 0), (False, 0, 0), (True, 2, 1)]:
        O, L = impl(q, k, v, 0.6, causal, w, ns)
        for h in range(2):
            for i in range(2):
                pos = 6 - 2 + i
                logits = {j: 0.6 * float(np.dot(q[0, h, i], k[0, 0, j])) for j in range(6)
                          if (not causal or j <= pos) and (w == 0 or pos - j < w or j < ns)}
                mx = max(logits.values())
                den = sum(math.exp(x - mx) for x in logits.values())
                assert abs(L[0, h, i] - (mx + math.log(den))) < 1e-12
                num = sum(math.exp(x - mx) * v[0, 0, j] for j, x in logits.items())
                assert np.abs(O[0, h, i] - num / den).max() < 1e-12


def pin_split_merge_matches(impl):
    """Splitting the keys into ranges and merging the partial results by
    log-sum-exp reproduces the unsplit result, including ranges with no kept
    key (a short window leaves the early ranges empty)."""
    q, k, v = _qkv(1, 4, 1, 2, 300, 8, seed=6)
    for causal, w, ns in CASES:
        O, L = impl(q, k, v, 0.4, causal, w, ns)
        for bounds in [(0,), (0, 64, 128, 192, 256), (0, 1, 299), (0, 150)]:
            Os, Ls = oracle.decode_split(q, k, v, 0.4, causal, w, ns, bounds)
            assert np.abs(O - Os).max() < 1e-13 and np.abs(L - Ls).max() < 1e-13


PINS = [pin_last_rows_of_full_forward, pin_brute_force, pin_split_merge_matches]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_decode_oracle_pin(pin):
    pin(oracle.decode)


def test_merge_of_one_part_is_identity_and_empty_parts_weigh_nothing():
    rng = np.random.default_rng(0)
    o, l = rng.standard_normal((3, 5)), rng.standard_normal(3)
    O, L = oracle.merge_partials(o[None], l[None])
    assert np.array_equal(O, o) and np.allclose(L, l, atol=1e-15, rtol=0)
    O2, L2 = oracle.merge_partials(np.stack([o, np.zeros_like(o)]),
                                   np.stack([l, np.full(3, -np.inf)]))
    assert np.array_equal(O2, o) and np.array_equal(L2, L)


def test_positions_are_the_last_rows():
    assert oracle.positions(1, 10).tolist() == [9]
    assert oracle.positions(3, 3).tolist() == [0, 1, 2]
    with pytest.raises(ValueError):
        oracle.positions(4, 3)


def _mutant(kind):
    def impl(Q, K, V, scale, causal, window, n_sink):
        B, H, n_q, _ = Q.shape
        H_kv, n_kv = K.shape[1], K.shape[2]
        rows = np.arange(n_q) if kind == "top_aligned" else np.arange(n_kv - n_q, n_kv)
        O = np.empty((B, H, n_q, V.shape[3]))
        L = np.empty((B, H, n_q))
        for b in range(B):
            for h in range(H):
                g = h // (H // H_kv)
                if kind == "merge_plain_mean":
                    # split in two halves and average the normalised partials
                    half = n_kv // 2
                    parts = [oracle.partial_head(Q[b, h], K[b, g], V[b, g], scale, causal, window,
                                                 n_sink, rows, lo, hi)
                             for lo, hi in ((0, half), (half, n_kv))]
                    ok = [np.isfinite(p[1]) for p in parts]
                    cnt = ok[0].astype(float) + ok[1].astype(float)
                    O[b, h] = (parts[0][0] * ok[0][:, None] + parts[1][0] * ok[1][:, None]) / cnt[:, None]
                    L[b, h] = np.logaddexp(parts[0][1], parts[1][1])
                    continue
                O[b, h], L[b, h] = oracle.attention_head(Q[b, h], K[b, g], V[b, g], scale, causal,
                                                         window, n_sink, rows)
        return O, L
    return impl


@pytest.mark.parametrize("kind", ["top_aligned", "merge_plain_mean"])
def test_planted_decode_mistakes_are_caught(kind):
    impl = _mutant(kind)
    failed = []
    with np.errstate(all="ignore"):
        for pin in PINS:
            try:
                pin(impl)
            except (AssertionError, ValueError, FloatingPointError, IndexError):
                failed.append(pin.__name__)
    assert failed, kind


def test_unplanted_decode_mutant_passes():
    for pin in PINS:
        pin(_mutant("none"))
