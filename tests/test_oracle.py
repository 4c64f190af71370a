"""Pins for the float64 oracle, checked against what the pages and mathematics fix.

None of these use the CUDA library.  Every pin is a function of an attention
implementation ``impl(Q, K, V, scale, causal, window, n_sink) -> (O, LSE)`` so
that ``test_planted_mistakes_are_caught`` can run the same pins against copies
of the oracle with one mistake planted each, and show that each mistake fails
at least one pin.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import definition as oatt
from exact_tiled_attention_44_b200.inputs import WORKLOADS, make_inputs, to_f64

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages.json")))
RNG = np.random.default_rng(1234)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _c1_inputs():
    q, k, v = make_inputs(WORKLOADS["c1"])
    return to_f64(q), to_f64(k), to_f64(v)


# --------------------------------------------------------------------------- pins


def pin_tiled_equivalence(impl):
    """Lab 3: tiled and full computations agree (printed: about 1e-16)."""
    Q, K, V = _c1_inputs()
    sc = WORKLOADS["c1"].scale
    O, L = impl(Q, K, V, sc, True, 0, 0)
    for order in ("q", "kv"):
        Ot, Lt = oracle.tiled_attention(Q, K, V, sc, True, bs=16, order=order)
        assert np.abs(O - Ot).max() <= 1e-14, order
        assert np.abs(L - Lt).max() <= 1e-13, order


def pin_block_sizes(impl):
    """Lab 3 exercise 1: block size (1, 7, 16, 64; ragged) does not change the result."""
    N, d = 50, 8
    Q, K, V = (_rand((1, 2, N, d), s) for s in (1, 2, 3))
    for causal, window, n_sink in ((True, 0, 0), (False, 0, 0), (True, 9, 3), (True, 4, 0)):
        O, L = impl(Q, K, V, 0.37, causal, window, n_sink)
        for bs in GOLDEN["lab3_block_sizes"]["block_sizes"]:
            for order in ("q", "kv"):
                Ot, Lt = oracle.tiled_attention(Q, K, V, 0.37, causal, window, n_sink, bs, order)
                assert np.abs(O - Ot).max() <= 1e-13, (causal, window, n_sink, bs, order)
                assert np.abs(L - Lt).max() <= 1e-12, (causal, window, n_sink, bs, order)


def pin_softmax_rows(impl):
    """The softmax weights are a probability distribution over the kept keys; O = P V."""
    N, d = 40, 6
    Q, K, V = (_rand((1, 1, N, d), s) for s in (4, 5, 6))
    for causal, window, n_sink in ((True, 0, 0), (False, 0, 0), (True, 7, 2)):
        P = oracle.attention_weights(Q[0, 0], K[0, 0], 0.5, causal, window, n_sink)
        keep = oracle.keep_mask(N, N, causal, window, n_sink)
        assert np.abs(P.sum(1) - 1).max() <= 1e-15 * N
        assert (P >= 0).all() and (P[~keep] == 0).all() and (P[keep] > 0).all()
        O, _ = impl(Q, K, V, 0.5, causal, window, n_sink)
        assert np.abs(O[0, 0] - P @ V[0, 0]).max() <= 1e-14


def pin_causal_row0(impl):
    """Causal row 0 sees only key 0: O[0] = V[0] and LSE[0] = scale * q0 . k0."""
    Q, K, V = (_rand((2, 3, 17, 5), s) for s in (7, 8, 9))
    O, L = impl(Q, K, V, 0.3, True, 0, 0)
    assert (O[:, :, 0] == V[:, :, 0]).all()
    expect = 0.3 * np.einsum("bhd,bhd->bh", Q[:, :, 0], K[:, :, 0])
    assert np.abs(L[:, :, 0] - expect).max() <= 1e-15


def _kept_lists(N, causal, window, n_sink):
    """Kept key indices per row, written out from the mask rule with plain loops."""
    out = []
    for i in range(N):
        js = []
        for j in range(N):
            if causal and j > i:
                continue
            if window > 0 and not (i - j < window or j < n_sink):
                continue
            js.append(j)
        out.append(js)
    return out


def pin_identical_keys(impl):
    """Equal logits in a row: O_i is the mean of the kept V rows, LSE_i = s + ln(#kept)."""
    N, d = 23, 4
    Q = _rand((1, 2, N, d), 10)
    V = _rand((1, 2, N, d), 11)
    krow = _rand((d,), 12)
    K = np.broadcast_to(krow, (1, 2, N, d)).copy()
    for causal, window, n_sink in ((True, 0, 0), (False, 0, 0), (True, 5, 3)):
        kept = _kept_lists(N, causal, window, n_sink)
        for scale in (0.0, 0.7):
            O, L = impl(Q, K, V, scale, causal, window, n_sink)
            for h in range(2):
                for i in range(N):
                    js = kept[i]
                    np.testing.assert_allclose(O[0, h, i], V[0, h, js].mean(0), rtol=0, atol=1e-14)
                    s = scale * float(Q[0, h, i] @ krow)
                    assert abs(L[0, h, i] - (s + math.log(len(js)))) <= 1e-13


def _brute(q, k, v, scale, causal, window, n_sink):
    """Scalar pure-Python attention: lists, math.exp, no numpy arithmetic."""
    n, d = len(q), len(q[0])
    kept = _kept_lists(n, causal, window, n_sink)
    O, L = [], []
    for i in range(n):
        s = {j: scale * sum(q[i][t] * k[j][t] for t in range(d)) for j in kept[i]}
        mx = max(s.values())
        w = {j: math.exp(s[j] - mx) for j in s}
        tot = sum(w.values())
        O.append([sum(w[j] * v[j][t] for j in w) / tot for t in range(d)])
        L.append(mx + math.log(tot))
    return O, L


def pin_brute_force(impl):
    """Brute force on tiny inputs (Lesson 91 Milestone 1 size N=8, d=4, and smaller)."""
    for N in (1, 2, 3, 5, 8):
        for d in (1, 4):
            Q, K, V = (_rand((1, 1, N, d), 100 * N + 10 * d + s) for s in (1, 2, 3))
            for causal, window, n_sink in ((True, 0, 0), (False, 0, 0), (True, 3, 1), (True, 2, 0)):
                O, L = impl(Q, K, V, 0.61, causal, window, n_sink)
                Ob, Lb = _brute(Q[0, 0].tolist(), K[0, 0].tolist(), V[0, 0].tolist(), 0.61,
                                causal, window, n_sink)
                assert np.abs(O[0, 0] - np.array(Ob)).max() <= 1e-13, (N, d, causal, window)
                assert np.abs(L[0, 0] - np.array(Lb)).max() <= 1e-13, (N, d, causal, window)


def pin_library(impl):
    """torch's float64 CPU scaled_dot_product_attention and scipy's logsumexp."""
    B, H, H_kv, N, d = 2, 4, 2, 37, 16
    Q, K, V = _rand((B, H, N, d), 20), _rand((B, H_kv, N, d), 21), _rand((B, H_kv, N, d), 22)
    rep = H // H_kv
    Kr, Vr = np.repeat(K, rep, axis=1), np.repeat(V, rep, axis=1)
    for causal, window, n_sink in ((True, 0, 0), (False, 0, 0), (True, 6, 2)):
        keep = oracle.keep_mask(N, N, causal, window, n_sink)
        O, L = impl(Q, K, V, 0.29, causal, window, n_sink)
        Ot = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q), torch.from_numpy(Kr), torch.from_numpy(Vr),
            attn_mask=torch.from_numpy(keep), scale=0.29).numpy()
        assert np.abs(O - Ot).max() <= 1e-13
        logits = 0.29 * torch.matmul(torch.from_numpy(Q), torch.from_numpy(Kr).transpose(-1, -2)).numpy()
        Ls = scipy.special.logsumexp(np.where(keep, logits, -np.inf), axis=-1)
        assert np.abs(L - Ls).max() <= 1e-13


def pin_mqa(impl):
    """MQA/GQA (Lesson 91 slide 32): H_kv shared heads == MHA on repeated K/V."""
    B, H, N, d = 1, 8, 19, 4
    Q = _rand((B, H, N, d), 30)
    for H_kv in (1, 2, 4):
        K, V = _rand((B, H_kv, N, d), 31 + H_kv), _rand((B, H_kv, N, d), 41 + H_kv)
        rep = H // H_kv
        O, L = impl(Q, K, V, 0.5, True, 0, 0)
        Om, Lm = impl(Q, np.repeat(K, rep, 1), np.repeat(V, rep, 1), 0.5, True, 0, 0)
        assert np.abs(O - Om).max() == 0 and np.abs(L - Lm).max() == 0
        # each query head must read its own group's K/V, not another group's
        for h in range(H):
            g = h // rep
            Oh, _ = impl(Q[:, h:h + 1], K[:, g:g + 1], V[:, g:g + 1], 0.5, True, 0, 0)
            assert np.abs(O[:, h] - Oh[:, 0]).max() == 0


def pin_permutation(impl):
    """Non-causal: permuting key and value rows together leaves O and LSE unchanged."""
    N, d = 31, 5
    Q, K, V = (_rand((1, 1, N, d), s) for s in (50, 51, 52))
    perm = np.random.default_rng(53).permutation(N)
    O, L = impl(Q, K, V, 0.4, False, 0, 0)
    Op, Lp = impl(Q, K[:, :, perm], V[:, :, perm], 0.4, False, 0, 0)
    assert np.abs(O - Op).max() <= 1e-14 and np.abs(L - Lp).max() <= 1e-13


def pin_shift(impl):
    """Adding c to every logit (an extra q/k column) leaves O unchanged and adds c to LSE."""
    N, d, c, scale = 21, 4, 2.5, 0.5
    Q, K, V = (_rand((1, 1, N, d), s) for s in (60, 61, 62))
    Qa = np.concatenate([Q, np.full((1, 1, N, 1), c / scale)], axis=-1)
    Ka = np.concatenate([K, np.ones((1, 1, N, 1))], axis=-1)
    for causal, window, n_sink in ((True, 0, 0), (False, 0, 0), (True, 4, 2)):
        O, L = impl(Q, K, V, scale, causal, window, n_sink)
        Oa, La = impl(Qa, Ka, V, scale, causal, window, n_sink)
        assert np.abs(O - Oa).max() <= 1e-14
        assert np.abs(La - L - c).max() <= 1e-13


def pin_scale_applied(impl):
    """Scale multiplies the logits: scale s on (Q, K) equals scale 1 on (s*Q, K)."""
    N, d = 15, 4
    Q, K, V = (_rand((1, 1, N, d), s) for s in (70, 71, 72))
    O, L = impl(Q, K, V, 0.25, True, 0, 0)
    O1, L1 = impl(0.25 * Q, K, V, 1.0, True, 0, 0)
    assert np.abs(O - O1).max() <= 1e-14 and np.abs(L - L1).max() <= 1e-14
    O2, _ = impl(Q, K, V, 0.0, False, 0, 0)
    assert np.abs(O2[0, 0] - V[0, 0].mean(0)).max() <= 1e-14


PINS = [pin_tiled_equivalence, pin_block_sizes, pin_softmax_rows, pin_causal_row0,
        pin_identical_keys, pin_brute_force, pin_library, pin_mqa, pin_permutation,
        pin_shift, pin_scale_applied]


def _oracle_impl(Q, K, V, scale, causal, window, n_sink):
    return oracle.attention(Q, K, V, scale, causal, window, n_sink)


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(_oracle_impl)


# ------------------------------------------------------------ planted mistakes


def _mutant(kind):
    """A copy of the oracle's definition with one plausible mistake planted."""
    def impl(Q, K, V, scale, causal, window, n_sink):
        B, H, N = Q.shape[:3]
        H_kv = K.shape[1]
        O = np.empty((B, H, N, V.shape[3]))
        L = np.empty((B, H, N))
        i = np.arange(N)[:, None]
        j = np.arange(N)[None, :]
        for b in range(B):
            for h in range(H):
                g = h % H_kv if kind == "kv_head_modulo" else h // (H // H_kv)
                q, k, v = Q[b, h], K[b, g], V[b, g]
                sc = 1.0 if kind == "scale_dropped" else scale
                s = sc * (q @ k.T)
                keep = np.ones((N, N), bool)
                if causal:
                    keep &= (j >= i) if kind == "mask_transposed" else (j <= i)
                    if kind == "causal_strict":
                        keep &= j < i
                        keep[0, 0] = True
                if window > 0:
                    w = window + 1 if kind == "window_off_by_one" else window
                    ns = 0 if kind == "sinks_ignored" else n_sink
                    keep &= (i - j < w) | (j < ns)
                s = np.where(keep, s, -np.inf)
                m = s.max(1)
                p = np.exp(s - m[:, None])
                l = p.sum(1)
                vv = k if kind == "v_is_k" else v
                if kind == "unnormalised":
                    O[b, h] = p @ vv
                else:
                    O[b, h] = (p @ vv) / l[:, None]
                if kind == "lse_log2":
                    L[b, h] = m + np.log2(l)
                elif kind == "lse_no_max":
                    L[b, h] = np.log(l)
                else:
                    L[b, h] = m + np.log(l)
        return O, L
    return impl


MUTANTS = ["kv_head_modulo", "scale_dropped", "mask_transposed", "causal_strict",
           "window_off_by_one", "sinks_ignored", "v_is_k", "unnormalised", "lse_log2",
           "lse_no_max"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_mistakes_are_caught(kind):
    impl = _mutant(kind)
    failed = []
    with np.errstate(all="ignore"):
        for pin in PINS:
            try:
                pin(impl)
            except (AssertionError, ValueError, FloatingPointError, IndexError):
                failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake {kind!r}"


def test_unplanted_mutant_copy_passes():
    """The mutant scaffold itself, with no mistake planted, passes every pin."""
    for pin in PINS:
        pin(_mutant("none"))


# ------------------------------------------------------------------ page facts


def test_lab3_printed_difference():
    """Lab 3 in float64 exactly as drawn there: tiled vs full differ by ~1e-16."""
    g = GOLDEN["lab3_tiled_equals_reference"]
    rng = np.random.default_rng(g["seed"])
    q, k, v = (rng.normal(size=(g["n"], g["d"])) for _ in range(3))
    sc = 1 / np.sqrt(g["d"])
    O, _ = oracle.attention_head(q, k, v, sc, True)
    Ot, _ = oracle.tiled_q_outer(q, k, v, sc, True, bs=g["bs"])
    assert np.abs(O - Ot).max() <= g["bound_used"]


def test_hands_on_mask_semantics():
    g = GOLDEN["hands_on_causal_mask"]
    assert (oracle.keep_mask(g["N"], g["N"], True).astype(int) == np.array(g["keep"])).all()
    # the property the guide's unit test meant: nothing above the diagonal is kept
    assert not np.triu(oracle.keep_mask(16, 16, True), k=1).any()


def test_score_matrix_size_16384():
    g = GOLDEN["score_matrix_entries_16384"]
    assert g["N"] ** 2 == g["entries"]
    assert abs(g["entries"] * 4 - g["approx_bytes_fp32"]) / g["approx_bytes_fp32"] < 0.1


def test_lesson91_milestone_bound():
    """Milestone 1 size: the KV-outer tiled loop matches standard attention to < 1e-6."""
    g = GOLDEN["lesson91_milestone_shape"]
    Q, K, V = (_rand((1, 1, g["N"], g["d"]), s) for s in (80, 81, 82))
    O, _ = oracle.attention(Q, K, V, g["d"] ** -0.5, False)
    Ot, _ = oracle.tiled_attention(Q, K, V, g["d"] ** -0.5, False, bs=g["block"], order="kv")
    assert np.abs(O - Ot).max() < g["bound"]


# --------------------------------------------------------------- mask counting


def _closed_form_pairs(N, causal, window, n_sink):
    if not causal:
        return N * N
    if window <= 0:
        return N * (N + 1) // 2
    tot = 0
    for i in range(N):
        tot += min(i + 1, window) + max(0, min(n_sink, i - window + 1))
    return tot


@pytest.mark.parametrize("N,causal,window,n_sink", [
    (1, True, 0, 0), (7, False, 0, 0), (64, True, 0, 0), (200, True, 17, 5),
    (300, True, 128, 64), (129, True, 1, 0), (50, True, 60, 10), (90, True, 8, 100)])
def test_kept_pairs_closed_form(N, causal, window, n_sink):
    assert oracle.kept_pairs(N, causal, window, n_sink) == _closed_form_pairs(N, causal, window, n_sink)


def test_kept_pairs_c5():
    """The MQA window/sink workload keeps 8,321,568 pairs per head (enumerated)."""
    w = WORKLOADS["c5"]
    assert oracle.kept_pairs(w.N, True, w.window, w.n_sink) == 8321568
    assert _closed_form_pairs(w.N, True, w.window, w.n_sink) == 8321568


def test_row_chunking_matches_whole():
    """Chunked rows (used when N^2 float64 would exceed 1 GiB) give the same result."""
    Q, K, V = (_rand((1, 1, 300, 8), s) for s in (90, 91, 92))
    O, L = oracle.attention_bh(Q, K, V, 0, 0, 0.3, True, 40, 4)
    saved = (oatt._MAX_SCORE_ENTRIES, oatt._ROW_CHUNK)
    try:
        oatt._MAX_SCORE_ENTRIES, oatt._ROW_CHUNK = 1000, 37
        Oc, Lc = oracle.attention_bh(Q, K, V, 0, 0, 0.3, True, 40, 4)
    finally:
        oatt._MAX_SCORE_ENTRIES, oatt._ROW_CHUNK = saved
    assert np.abs(O - Oc).max() <= 1e-14 and np.abs(L - Lc).max() <= 1e-14


def test_rows_subset_matches_whole():
    Q, K, V = (_rand((1, 2, 70, 8), s) for s in (93, 94, 95))
    O, L = oracle.attention(Q, K, V, 0.3, True, 9, 2)
    rows = np.array([0, 5, 33, 69])
    Or, Lr = oracle.attention_bh(Q, K, V, 0, 1, 0.3, True, 9, 2, rows=rows)
    assert np.abs(O[0, 1, rows] - Or).max() <= 1e-14 and np.abs(L[0, 1, rows] - Lr).max() <= 1e-14


def test_empty_row_is_rejected():
    """A query row with no kept key has no defined softmax: the oracle refuses it."""
    with pytest.raises(ValueError):
        oracle.attention_weights(np.ones((3, 2)), np.ones((3, 2)), 1.0, True, rows=np.array([-5]))


# ------------------------------------------------------------- input recipe


def test_c1_is_lab3_draw_rounded_to_bf16():
    rng = np.random.default_rng(0)
    q, k, v = (rng.normal(size=(64, 16)) for _ in range(3))
    tq, tk, tv = make_inputs(WORKLOADS["c1"])
    for a, t in ((q, tq), (k, tk), (v, tv)):
        assert t.dtype == torch.bfloat16 and tuple(t.shape) == (1, 1, 64, 16)
        assert (to_f64(t)[0, 0] == torch.from_numpy(a).to(torch.bfloat16).double().numpy()).all()


def test_outlier_rows_scaled():
    w = WORKLOADS["c4"].with_(N=1000, H=2, H_kv=2)
    q, k, v = make_inputs(w)
    w0 = w.with_(outlier_frac=0.0)
    _, k0, _ = make_inputs(w0)
    ratio = to_f64(k) / np.where(to_f64(k0) == 0, 1, to_f64(k0))
    big = (np.abs(ratio - 8) < 0.1).all(-1)
    assert (big.sum(-1) == 10).all()
