"""Pins of the oracle's attention gradients (the backward pass that "USAAIO
Lesson 91", slide 9, says Flash Attention 2 recomputes tile by tile).

The gradients are pinned against things other than their own formulas:
central finite differences of the forward definition, torch autograd of the
definition written with torch ops, invariants that the mathematics fixes
(softmax rows sum to one, so the key gradients sum to zero and dQ ignores a
shift shared by all keys), and closed forms for one key, constant values and
identical keys.  Planted mistakes in a copy of the formulas must each be caught
by at least one pin.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_44_b200.inputs import random_qkv, to_f64

CASES = [  # (causal, window, n_sink, with ALiBi)
    (True, 0, 0, False),
    (False, 0, 0, False),
    (True, 3, 1, False),
    (False, 4, 0, True),
    (True, 0, 0, True),
]


def _inputs(B, H, H_kv, N, d, seed):
    q, k, v = (to_f64(t) for t in random_qkv(B, H, H_kv, N, d, seed=seed))
    rng = np.random.default_rng(seed + 100)
    do = rng.standard_normal(q.shape)
    return q, k, v, do


def _slopes(H, alibi):
    return oracle.alibi_slopes(H) if alibi else None


def pin_finite_differences(impl):
    """Every gradient entry against the central difference of
    sum(O * dO) with O from the forward definition (step 1e-6)."""
    q, k, v, do = _inputs(1, 2, 1, 6, 3, seed=11)
    scale = 0.7
    for causal, w, ns, alibi in CASES:
        sl = _slopes(2, alibi)

        def loss(Q, K, V):
            O, _ = oracle.attention(Q, K, V, scale, causal, w, ns, slopes=sl)
            return float((O * do).sum())

        dQ, dK, dV = impl(q, k, v, do, scale, causal, w, ns, sl)
        for which, x, g in ((0, q, dQ), (1, k, dK), (2, v, dV)):
            for idx in np.ndindex(x.shape):
                args = [q.copy(), k.copy(), v.copy()]
                args[which][idx] += 1e-6
                up = loss(*args)
                args[which][idx] -= 2e-6
                dn = loss(*args)
                fd = (up - dn) / 2e-6
                assert abs(g[idx] - fd) < 1e-7 * max(1.0, abs(fd)), (which, idx, g[idx], fd)


def _torch_grads(q, k, v, do, scale, causal, w, ns, slopes):
    """Autograd of the definition written in torch float64 ops."""
    Q, K, V = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    B, H, N, _ = q.shape
    G = H // k.shape[1]
    Ke = K.repeat_interleave(G, dim=1)
    Ve = V.repeat_interleave(G, dim=1)
    s = scale * Q @ Ke.transpose(-1, -2)
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    if slopes is not None:
        s = s - torch.tensor(slopes)[None, :, None, None] * (i - j).abs()
    keep = torch.ones(N, N, dtype=torch.bool)
    if causal:
        keep &= j <= i
    if w > 0:
        keep &= (i - j < w) | (j < ns)
    s = s.masked_fill(~keep, float("-inf"))
    O = torch.softmax(s, dim=-1) @ Ve
    (O * torch.tensor(do)).sum().backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


def pin_torch_autograd(impl):
    """Grouped heads (H = 4 over H_kv = 2), several tiles' worth of rows."""
    q, k, v, do = _inputs(2, 4, 2, 37, 8, seed=12)
    for causal, w, ns, alibi in CASES:
        sl = _slopes(4, alibi)
        got = impl(q, k, v, do, 0.3, causal, w, ns, sl)
        ref = _torch_grads(q, k, v, do, 0.3, causal, w, ns, sl)
        for a, b in zip(got, ref):
            assert np.abs(a - b).max() < 1e-11 * max(1.0, np.abs(b).max())


def pin_invariants(impl):
    """Rows of dS sum to zero, so sum_j dK_j = 0 and dQ ignores a shift c added
    to every key; rows of P sum to one, so sum_j dV_j = sum over the group's
    query heads of sum_i dO_i; the gradients are linear in dO."""
    q, k, v, do = _inputs(1, 4, 2, 23, 5, seed=13)
    c = np.random.default_rng(5).standard_normal(5)
    for causal, w, ns, alibi in CASES:
        sl = _slopes(4, alibi)
        dQ, dK, dV = impl(q, k, v, do, 0.45, causal, w, ns, sl)
        assert np.abs(dK.sum(axis=2)).max() < 1e-11
        sum_do = do.reshape(1, 2, 2, 23, 5).sum(axis=(2, 3))
        assert np.abs(dV.sum(axis=2) - sum_do).max() < 1e-11
        dQs, _, _ = impl(q, k + c, v, do, 0.45, causal, w, ns, sl)
        assert np.abs(dQs - dQ).max() < 1e-10
        g2 = impl(q, k, v, 2.0 * do - 0.5 * do[..., ::-1], 0.45, causal, w, ns, sl)
        ga = impl(q, k, v, do[..., ::-1].copy(), 0.45, causal, w, ns, sl)
        for x2, x1, xa in zip(g2, (dQ, dK, dV), ga):
            assert np.abs(x2 - (2.0 * x1 - 0.5 * xa)).max() < 1e-10


def pin_closed_forms(impl):
    """One key: P = 1, so dV = dO and dQ = dK = 0.  Constant value rows: O does
    not depend on P, so dQ = dK = 0 and dV_j = sum_i P_ij dO_i with P uniform
    when every key is identical: dV_j = sum over rows i keeping j of dO_i / n_i."""
    q, k, v, do = _inputs(1, 1, 1, 1, 4, seed=14)
    dQ, dK, dV = impl(q, k, v, do, 0.5, True, 0, 0, None)
    assert np.abs(dQ).max() == 0 and np.abs(dK).max() == 0
    assert np.array_equal(dV, do)
    N = 9
    q, k, v, do = _inputs(1, 1, 1, N, 4, seed=15)
    k_same = np.broadcast_to(k[:, :, :1], k.shape).copy()
    v_same = np.broadcast_to(v[:, :, :1], v.shape).copy()
    for causal, w, ns in [(True, 0, 0), (False, 0, 0), (True, 3, 2)]:
        dQ, dK, dV = impl(q, k_same, v_same, do, 0.8, causal, w, ns, None)
        assert np.abs(dQ).max() < 1e-12 and np.abs(dK).max() < 1e-12
        keep = oracle.keep_mask(N, N, causal, w, ns)
        n_i = keep.sum(axis=1)
        want = (keep / n_i[:, None]).T @ do[0, 0]
        assert np.abs(dV[0, 0] - want).max() < 1e-12


def pin_two_keys_by_hand(impl):
    """One query q = 1 and two keys k = (0, ln 3), values v = (1, 5), scale 1,
    dO = 1, no mask: P = (1/4, 3/4), O = 4, so dV = P = (1/4, 3/4),
    dS_j = P_j (v_j - O) = (-3/4, 3/4), dK_j = dS_j q = (-3/4, 3/4) and
    dQ = sum_j dS_j k_j = P_1 P_2 (v_1 - v_2)(k_1 - k_2) = (3/4) ln 3, worked out
    by hand.  Posed as a 2-row non-causal problem whose second row has q = 0
    and dO = 0, so that it adds nothing to dK and dV and its dQ is 0."""
    import math
    q = np.array([[[[1.0], [0.0]]]])
    k = np.array([[[[0.0], [math.log(3.0)]]]])
    v = np.array([[[[1.0], [5.0]]]])
    do = np.array([[[[1.0], [0.0]]]])
    dQ, dK, dV = impl(q, k, v, do, 1.0, False, 0, 0, None)
    assert abs(dQ[0, 0, 0, 0] - 0.75 * math.log(3.0)) < 1e-14
    assert abs(dQ[0, 0, 1, 0]) < 1e-14
    assert np.abs(dK[0, 0, :, 0] - np.array([-0.75, 0.75])).max() < 1e-14
    assert np.abs(dV[0, 0, :, 0] - np.array([0.25, 0.75])).max() < 1e-14


PINS = [pin_finite_differences, pin_torch_autograd, pin_invariants, pin_closed_forms,
        pin_two_keys_by_hand]


def _oracle_impl(Q, K, V, dO, scale, causal, window, n_sink, slopes):
    return oracle.attention_backward(Q, K, V, dO, scale, causal, window, n_sink, slopes)


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_backward_pin(pin):
    pin(_oracle_impl)


def _mutant(kind):
    """A copy of the gradient formulas with one plausible mistake planted."""
    def impl(Q, K, V, dO, scale, causal, window, n_sink, slopes):
        B, H, N, d = Q.shape
        H_kv = K.shape[1]
        dQ = np.zeros_like(Q)
        dK = np.zeros_like(K)
        dV = np.zeros_like(V)
        i = np.arange(N)[:, None]
        j = np.arange(N)[None, :]
        for b in range(B):
            for h in range(H):
                g = h // (H // H_kv)
                q, k, v, do = Q[b, h], K[b, g], V[b, g], dO[b, h]
                s = scale * (q @ k.T)
                if slopes is not None:
                    s = s - slopes[h] * np.abs(i - j)
                keep = np.ones((N, N), bool)
                if causal:
                    keep &= j <= i
                if window > 0:
                    keep &= (i - j < window) | (j < n_sink)
                s = np.where(keep, s, -np.inf)
                p = np.exp(s - s.max(1, keepdims=True))
                p /= p.sum(1, keepdims=True)
                o = p @ v
                dv = (p @ do) if kind == "p_not_transposed" else (p.T @ do)
                dp = do @ v.T
                D = (do * o).sum(1)
                if kind == "row_term_dropped":
                    ds = p * dp
                elif kind == "row_term_sign":
                    ds = p * (dp + D[:, None])
                elif kind == "row_term_from_dp_rowsum":
                    ds = p * (dp - dp.sum(1, keepdims=True))
                else:
                    ds = p * (dp - D[:, None])
                dq = scale * (ds @ k)
                dk = (ds.T @ q) if kind == "dk_scale_dropped" else scale * (ds.T @ q)
                if kind == "dk_from_keys":
                    dk = scale * (ds.T @ k)
                dQ[b, h] = dq
                if kind == "group_overwrites":
                    dK[b, g] = dk
                    dV[b, g] = dv
                else:
                    dK[b, g] += dk
                    dV[b, g] += dv
        return dQ, dK, dV
    return impl


MUTANTS = ["p_not_transposed", "row_term_dropped", "row_term_sign", "row_term_from_dp_rowsum",
           "dk_scale_dropped", "dk_from_keys", "group_overwrites"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_backward_mistakes_are_caught(kind):
    impl = _mutant(kind)
    failed = []
    with np.errstate(all="ignore"):
        for pin in PINS:
            try:
                pin(impl)
            except (AssertionError, ValueError, FloatingPointError, IndexError):
                failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake {kind!r}"


def test_unplanted_backward_mutant_copy_passes():
    for pin in PINS:
        pin(_mutant("none"))


def test_row_dot_matches_forward():
    """D_i = dO_i . O_i equals sum_j P_ij dP_ij (the two forms the formulas use)."""
    q, k, v, do = _inputs(1, 2, 2, 17, 6, seed=16)
    O, _ = oracle.attention(q, k, v, 0.4, True)
    D = oracle.row_dot(O, do)
    for h in range(2):
        P = oracle.attention_weights(q[0, h], k[0, h], 0.4, True)
        dP = do[0, h] @ v[0, h].T
        assert np.abs((P * dP).sum(1) - D[0, h]).max() < 1e-12


@pytest.mark.parametrize("bs", [1, 5, 16, 64])
def test_tiled_recomputation_equals_the_definition(bs):
    """The tiled recomputation from the saved (O, LSE) of the forward (slide 9)
    reaches the plain gradients to rounding, for every mask kind, ALiBi and a
    block size that does not divide N."""
    q, k, v, do = _inputs(1, 2, 1, 41, 6, seed=17)
    sl = oracle.alibi_slopes(2)
    for causal, w, ns, alibi in CASES:
        for h in range(2):
            slope = float(sl[h]) if alibi else 0.0
            O, L = oracle.attention_head(q[0, h], k[0, 0], v[0, 0], 0.6, causal, w, ns,
                                         slope=slope)
            want = oracle.backward_head(q[0, h], k[0, 0], v[0, 0], do[0, h], 0.6, causal, w, ns,
                                        slope)
            got = oracle.tiled_backward_head(q[0, h], k[0, 0], v[0, 0], O, do[0, h], L, 0.6,
                                             causal, w, ns, slope, bs=bs)
            for a, b in zip(got, want):
                assert np.abs(a - b).max() < 1e-12 * max(1.0, np.abs(b).max())


def test_random_configurations_against_autograd():
    """Random shapes, group sizes, masks, scales (any sign) and slopes: the
    oracle's gradients equal torch autograd of the definition."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=40, deadline=None, derandomize=True)
    @given(st.integers(1, 2), st.sampled_from([(1, 1), (2, 1), (4, 2), (3, 3), (6, 2)]),
           st.integers(1, 23), st.sampled_from([2, 4, 8]), st.booleans(),
           st.integers(0, 6), st.integers(0, 3), st.booleans(),
           st.floats(-1.5, 1.5, allow_nan=False), st.integers(0, 10_000))
    def check(B, heads, N, d, causal, window, n_sink, alibi, scale, seed):
        H, H_kv = heads
        if window and not causal:
            window = 0
        q, k, v, do = _inputs(B, H, H_kv, N, d, seed)
        sl = _slopes(H, alibi)
        got = oracle.attention_backward(q, k, v, do, scale, causal, window, n_sink, sl)
        ref = _torch_grads(q, k, v, do, scale, causal, window, n_sink, sl)
        for a, b in zip(got, ref):
            assert np.abs(a - b).max() <= 1e-10 * max(1.0, np.abs(b).max())

    check()
