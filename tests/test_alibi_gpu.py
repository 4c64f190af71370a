"""GPU parity of attn_fwd_alibi (ALiBi position bias, "USAAIO Lesson 91",
slides 20-23) against the float64 oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A
import oracle
from exact_tiled_attention_44_b200.inputs import WORKLOADS, make_inputs, random_qkv, to_f64
from parity_utils import assert_parity, errors, round_floor

pytestmark = pytest.mark.gpu

BF, FP = torch.bfloat16, torch.float16


def run_alibi(q, k, v, slopes, causal, window, n_sink, scale, out_f32):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = A.attention(qd, kd, vd, causal=causal, window=window, n_sink=n_sink, scale=scale,
                         out_f32=out_f32, alibi_slopes=slopes.cuda())
    torch.cuda.synchronize()
    return o, lse


def oracle_alibi(q, k, v, slopes, causal, window, n_sink, scale):
    return oracle.attention(to_f64(q), to_f64(k), to_f64(v), scale, causal, window, n_sink,
                            slopes=slopes.double().numpy())


# (B, H, H_kv, N, d, dtype, causal, window, n_sink)
SWEEP = [
    (1, 1, 1, 1, 64, BF, 1, 0, 0),
    (1, 4, 1, 77, 128, BF, 1, 0, 0),
    (1, 2, 2, 129, 64, FP, 0, 0, 0),
    (2, 4, 2, 255, 128, BF, 1, 0, 0),
    (1, 8, 8, 300, 32, BF, 0, 0, 0),
    (1, 4, 4, 520, 16, FP, 1, 0, 0),
    (1, 8, 2, 700, 128, BF, 1, 130, 3),
    (1, 4, 4, 900, 128, FP, 1, 128, 64),
    (1, 16, 16, 1024, 128, BF, 1, 0, 0),
]


def _id(c):
    B, H, Hk, N, d, dt, ca, w, s = c
    return f"B{B}H{H}k{Hk}N{N}d{d}{'bf' if dt == BF else 'fp'}{'c' if ca else 'n'}w{w}s{s}"


@pytest.mark.parametrize("case", SWEEP, ids=[_id(c) for c in SWEEP])
def test_alibi_sweep_pages_slopes(case):
    B, H, Hk, N, d, dt, causal, window, n_sink = case
    q, k, v = random_qkv(B, H, Hk, N, d, dt, seed=N * 7 + d)
    slopes = A.alibi_slopes(H)
    scale = A.default_scale(d)
    Or, Lr = oracle_alibi(q, k, v, slopes, bool(causal), window, n_sink, scale)
    o32, l32 = run_alibi(q, k, v, slopes, bool(causal), window, n_sink, scale, True)
    assert_parity(errors(o32, l32, Or, Lr), what="fp32 out")
    o16, l16 = run_alibi(q, k, v, slopes, bool(causal), window, n_sink, scale, False)
    assert_parity(errors(o16, l16, Or, Lr), round_floor(Or, dt), what="16-bit out")
    assert torch.equal(o16, o32.to(dt)) and torch.equal(l16, l32)


@pytest.mark.parametrize("slope_set", ["zero", "negative", "steep", "mixed"])
def test_alibi_slope_values(slope_set):
    B, H, Hk, N, d = 1, 4, 2, 333, 128
    q, k, v = random_qkv(B, H, Hk, N, d, BF, seed=21)
    slopes = {"zero": [0.0] * 4, "negative": [-0.01, -0.002, 0.0, -0.0005],
              "steep": [4.0, 1.0, 0.5, 2.0], "mixed": [0.3, -0.001, 0.0, 1.5]}[slope_set]
    slopes = torch.tensor(slopes, dtype=torch.float32)
    for causal in (True, False):
        Or, Lr = oracle_alibi(q, k, v, slopes, causal, 0, 0, 0.088)
        o, l = run_alibi(q, k, v, slopes, causal, 0, 0, 0.088, True)
        assert_parity(errors(o, l, Or, Lr), what=f"{slope_set} causal={causal}")


def test_zero_slopes_match_the_plain_kernel():
    """Zero slopes give the plain attention.  The biased path scales S before
    its row max while the plain path scales after it, so a probability may
    round to the neighbouring 16-bit value: O may differ by about one bf16
    ulp of a weight (2^-8 relative), LSE (fp32 sums) only in the last bits."""
    q, k, v = random_qkv(2, 4, 4, 600, 128, BF, seed=4)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o0, l0 = A.attention(qd, kd, vd, causal=True, out_f32=True)
    o1, l1 = A.attention(qd, kd, vd, causal=True, out_f32=True,
                         alibi_slopes=torch.zeros(4, device="cuda"))
    torch.cuda.synchronize()
    Or, Lr = oracle_alibi(q, k, v, torch.zeros(4), True, 0, 0, A.default_scale(128))
    assert_parity(errors(o1, l1, Or, Lr), what="zero slopes")
    assert (o0 - o1).abs().max().item() < 1e-2
    assert (l0 - l1).abs().max().item() < 1e-5


def test_identical_keys_geometric_closed_form():
    """All keys equal: the weights are e^{-m |i - j|}, so LSE_i is the scaled
    dot product plus ln of a geometric series, and O_i with one-hot V rows is
    the normalised weight vector."""
    N, d, H = 128, 128, 2
    g = torch.Generator().manual_seed(3)
    q = (torch.randn(1, H, N, d, generator=g) * 0.5).to(BF)
    k = torch.randn(1, 1, 1, d, generator=g).to(BF).expand(1, 1, N, d).contiguous()
    v = torch.zeros(1, 1, N, d, dtype=BF)
    v[0, 0, :, :] = torch.eye(N, d, dtype=BF)
    slopes = torch.tensor([0.25, 1.0], dtype=torch.float32)
    scale = 0.1
    o, l = run_alibi(q, k, v, slopes, True, 0, 0, scale, True)
    qd, kd = to_f64(q), to_f64(k)
    for h in range(H):
        m = float(slopes[h])
        c = scale * (qd[0, h] @ kd[0, 0, 0])
        for i in range(N):
            tot = (1.0 - math.exp(-m * (i + 1))) / (1.0 - math.exp(-m))
            assert abs(l[0, h, i].item() - (c[i] + math.log(tot))) < 1e-3
            w = np.exp(-m * (i - np.arange(i + 1)))
            got = o[0, h, i, :i + 1].double().cpu().numpy()
            assert np.abs(got - w / w.sum()).max() < 1e-2


def test_alibi_headline_shape_sampled_rows():
    """The headline workload shape (causal bf16 B4 H16 N4096 d128) with the
    pages' slopes, sampled rows of every (b, h) against the oracle."""
    w = WORKLOADS["c3"]
    q, k, v = make_inputs(w)
    slopes = A.alibi_slopes(w.H)
    o, l = run_alibi(q, k, v, slopes, True, 0, 0, w.scale, True)
    rng = np.random.default_rng(0)
    sl = slopes.double().numpy()
    worst = 0.0
    for b in range(w.B):
        for h in range(w.H):
            rows = np.unique(np.concatenate([[0, 127, 128, w.N - 1], rng.integers(0, w.N, 4)]))
            Q = to_f64(q[b:b + 1, h:h + 1]); K = to_f64(k[b:b + 1, h:h + 1]); V = to_f64(v[b:b + 1, h:h + 1])
            Or, Lr = oracle.attention_bh(Q, K, V, 0, 0, w.scale, True, rows=rows, slopes=sl[h:h + 1])
            og = o[b, h, rows].double().cpu().numpy()
            lg = l[b, h, rows].double().cpu().numpy()
            assert np.abs(og - Or).max() <= 1e-2 and np.abs(lg - Lr).max() <= 1e-3, (b, h)
            worst = max(worst, float(np.abs(og - Or).max()))
    assert worst < 1e-2


def test_alibi_deterministic_and_lse_optional():
    q, k, v = random_qkv(1, 8, 1, 1000, 128, BF, seed=8)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    s = A.alibi_slopes(8, "cuda")
    o1, l1 = A.attention(qd, kd, vd, causal=True, alibi_slopes=s)
    o2, l2 = A.attention(qd, kd, vd, causal=True, alibi_slopes=s)
    o3, l3 = A.attention(qd, kd, vd, causal=True, alibi_slopes=s, return_lse=False)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and torch.equal(o1, o3) and l3 is None
    assert A.get_status() == A.ATTN_OK


def test_binding_validates_slopes():
    q, k, v = (t.cuda() for t in random_qkv(1, 4, 4, 64, 64, BF, seed=1))
    for bad in (torch.zeros(3, device="cuda"), torch.zeros(4, dtype=torch.float64, device="cuda"),
                torch.zeros(4)):
        with pytest.raises(ValueError):
            A.attention(q, k, v, causal=True, alibi_slopes=bad)
