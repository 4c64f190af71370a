"""Pins of the oracle's ALiBi position bias ("USAAIO Lesson 91", slides 20-23).

Each pin checks the oracle against something other than itself: the slides'
slope formula and worked-example bias rows, closed-form geometric sums, a
brute-force loop, the plain definition at slope 0, and both tiled loop
orders.  Planted mistakes in a copy of the biased definition must each be
caught by at least one pin.
"""
import math

import numpy as np
import pytest

import oracle
from exact_tiled_attention_44_b200.inputs import random_qkv, to_f64


# ------------------------------------------------------------------ slopes and bias


def test_slopes_pages_formula():
    """Slide 23: m_h = 2^(-h 8 / H), h = 1..H.  For H = 4 and H = 8 these are
    exact powers of two; in general consecutive slopes have the ratio 2^(-8/H)."""
    assert oracle.alibi_slopes(4).tolist() == [0.25, 0.0625, 0.015625, 0.00390625]
    assert oracle.alibi_slopes(8).tolist() == [2.0 ** -e for e in range(1, 9)]
    for H in (1, 3, 12, 16, 32):
        s = oracle.alibi_slopes(H)
        assert s.shape == (H,)
        assert abs(s[0] - 2.0 ** (-8.0 / H)) < 1e-15
        assert abs(s[-1] - 2.0 ** -8) < 1e-15
        assert np.allclose(s[1:] / s[:-1], 2.0 ** (-8.0 / H), rtol=1e-14, atol=0)


def test_bias_rows_of_the_worked_example():
    """Slide 23's example (N = 6, H = 4): head 0 has slope 1/4, so its bias row
    0 is -|0 - j| / 4 and row 2 is -|2 - j| / 4."""
    m0 = oracle.alibi_slopes(4)[0]
    b = oracle.alibi_bias(6, m0, np.array([0, 2]))
    assert b[0].tolist() == [0.0, -0.25, -0.5, -0.75, -1.0, -1.25]
    assert b[1].tolist() == [-0.5, -0.25, 0.0, -0.25, -0.5, -0.75]


# ------------------------------------------------------------------ pins on an implementation
# impl(Q, K, V, scale, causal, window, n_sink, slopes) -> (O, LSE)


def pin_zero_slope_is_plain(impl):
    q, k, v = (to_f64(t) for t in random_qkv(1, 2, 1, 40, 16, seed=3))
    for causal, w, ns in [(True, 0, 0), (False, 0, 0), (True, 9, 2)]:
        O0, L0 = oracle.attention(q, k, v, 0.3, causal, w, ns)
        O1, L1 = impl(q, k, v, 0.3, causal, w, ns, np.zeros(2))
        assert np.abs(O0 - O1).max() < 1e-12 and np.abs(L0 - L1).max() < 1e-12


def _geometric(m, n):
    """sum_{t=0}^{n-1} e^{-m t} in closed form."""
    return n if m == 0 else (1.0 - math.exp(-m * n)) / (1.0 - math.exp(-m))


def pin_identical_keys_closed_form(impl):
    """All keys equal: the logit of (i, j) is c - m |i - j|, so the weights are
    e^{-m |i - j|} and LSE_i = c + ln(sum of a geometric series); with V rows
    v_j = e_j (one-hot), O_i is those weights normalised."""
    N, scale = 24, 0.5
    rng = np.random.default_rng(5)
    q = rng.normal(size=(1, 2, N, 8))
    k = np.broadcast_to(rng.normal(size=8), (1, 1, N, 8)).copy()
    v = np.zeros((1, 1, N, N)); v[0, 0] = np.eye(N)
    slopes = np.array([0.3, 1.7])
    for causal in (True, False):
        O, L = impl(q, k, v, scale, causal, 0, 0, slopes)
        for h in range(2):
            m = slopes[h]
            c = scale * (q[0, h] @ k[0, 0, 0])
            for i in range(N):
                tot = _geometric(m, i + 1) + (0.0 if causal else _geometric(m, N - i) - 1.0)
                assert abs(L[0, h, i] - (c[i] + math.log(tot))) < 1e-12
                w = np.array([math.exp(-m * abs(i - j)) if (j <= i or not causal) else 0.0
                              for j in range(N)])
                assert np.abs(O[0, h, i] - w / w.sum()).max() < 1e-12


def pin_brute_force_loops(impl):
    """Tiny cases against explicit Python loops over (i, j)."""
    for causal, w, ns in [(True, 0, 0), (False, 0, 0), (True, 3, 1)]:
        q, k, v = (to_f64(t) for t in random_qkv(1, 2, 2, 7, 4, seed=11))
        slopes = np.array([0.4, 0.05])
        O, L = impl(q, k, v, 0.7, causal, w, ns, slopes)
        for h in range(2):
            for i in range(7):
                logits = {}
                for j in range(7):
                    kept = (not causal or j <= i) and (w == 0 or i - j < w or j < ns)
                    if kept:
                        dot = sum(q[0, h, i, t] * k[0, h, j, t] for t in range(4))
                        logits[j] = 0.7 * dot - slopes[h] * abs(i - j)
                mx = max(logits.values())
                den = sum(math.exp(x - mx) for x in logits.values())
                assert abs(L[0, h, i] - (mx + math.log(den))) < 1e-12
                for t in range(4):
                    num = sum(math.exp(x - mx) * v[0, h, j, t] for j, x in logits.items())
                    assert abs(O[0, h, i, t] - num / den) < 1e-12


def pin_tiled_orders_agree(impl):
    """Both tiled loop orders of the pages, with the bias added per tile, reach
    the same result as the implementation under test."""
    q, k, v = (to_f64(t) for t in random_qkv(1, 4, 2, 45, 8, seed=7))
    slopes = oracle.alibi_slopes(4)
    for causal, w, ns in [(True, 0, 0), (False, 0, 0), (True, 11, 3)]:
        O, L = impl(q, k, v, 0.35, causal, w, ns, slopes)
        for order in ("q", "kv"):
            Ot, Lt = oracle.tiled_attention(q, k, v, 0.35, causal, w, ns, bs=7, order=order,
                                            slopes=slopes)
            assert np.abs(O - Ot).max() < 1e-12 and np.abs(L - Lt).max() < 1e-12


PINS = [pin_zero_slope_is_plain, pin_identical_keys_closed_form, pin_brute_force_loops,
        pin_tiled_orders_agree]


def _definition(Q, K, V, scale, causal, window, n_sink, slopes):
    return oracle.attention(Q, K, V, scale, causal, window, n_sink, slopes=slopes)


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_alibi_pin(pin):
    pin(_definition)


def _mutant(kind):
    """A copy of the biased definition with one plausible mistake planted."""
    def impl(Q, K, V, scale, causal, window, n_sink, slopes):
        B, H, N = Q.shape[:3]
        H_kv = K.shape[1]
        O = np.empty((B, H, N, V.shape[3]))
        L = np.empty((B, H, N))
        i = np.arange(N)[:, None]
        j = np.arange(N)[None, :]
        for b in range(B):
            for h in range(H):
                g = h // (H // H_kv)
                s = scale * (Q[b, h] @ K[b, g].T)
                m = slopes[h + 1] if (kind == "slope_of_next_head" and h + 1 < H) else slopes[h]
                dist = (i - j) if kind == "signed_distance" else np.abs(i - j)
                sign = 1.0 if kind == "bias_sign" else -1.0
                if kind != "bias_dropped":
                    s = s + sign * m * dist
                keep = np.ones((N, N), bool)
                if causal:
                    keep &= j <= i
                if window > 0:
                    keep &= (i - j < window) | (j < n_sink)
                s = np.where(keep, s, -np.inf)
                mx = s.max(1)
                p = np.exp(s - mx[:, None])
                l = p.sum(1)
                O[b, h] = (p @ V[b, g]) / l[:, None]
                L[b, h] = mx + np.log(l)
        return O, L
    return impl


MUTANTS = ["bias_sign", "signed_distance", "slope_of_next_head", "bias_dropped"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_alibi_mistakes_are_caught(kind):
    impl = _mutant(kind)
    failed = []
    with np.errstate(all="ignore"):
        for pin in PINS:
            try:
                pin(impl)
            except (AssertionError, ValueError, FloatingPointError, IndexError):
                failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake {kind!r}"


def test_unplanted_alibi_mutant_copy_passes():
    for pin in PINS:
        pin(_mutant("none"))


def test_alibi_rows_and_chunking():
    """The row-subset and row-chunk paths carry the head's slope."""
    q, k, v = (to_f64(t) for t in random_qkv(1, 2, 1, 300, 16, seed=9))
    slopes = np.array([0.02, 0.3])
    O, L = oracle.attention(q, k, v, 0.25, True, slopes=slopes)
    rows = np.array([0, 17, 150, 299])
    for h in range(2):
        o, l = oracle.attention_bh(q, k, v, 0, h, 0.25, True, rows=rows, slopes=slopes)
        assert np.abs(o - O[0, h, rows]).max() < 1e-14 and np.abs(l - L[0, h, rows]).max() < 1e-14
