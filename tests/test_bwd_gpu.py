"""GPU parity of attn_bwd (dQ, dK, dV through the C ABI) against the float64
gradient oracle.

Tolerance, derived from the arithmetic: the kernel rounds P and dS to 16 bits
before the products that consume them (unit roundoff 2^-9 for bf16) and
accumulates in fp32, and D is formed from the 16-bit O.  Each gradient entry
is a sum of many such rounded terms whose errors partly cancel, so the error
of a whole gradient tensor is bounded here relative to its own size:
    max |G - G_ref| <= 2e-2 * max |G_ref|   and   ||G - G_ref||_2 <= 1e-2 * ||G_ref||_2
(about five unit roundoffs).  The fp16 bars are the same.  Inputs of the
backward (O as a 16-bit tensor and LSE) come from the oracle's forward unless
a test says otherwise, so that the backward is judged on its own.
"""
import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A
import oracle
from exact_tiled_attention_44_b200.inputs import make_grad_output, random_qkv, to_f64

pytestmark = pytest.mark.gpu

BF, FP = torch.bfloat16, torch.float16
REL_MAX, REL_L2 = 2e-2, 1e-2


def rel_errors(got, ref):
    g = got.detach().double().cpu().numpy()
    d = g - ref
    return (float(np.abs(d).max() / max(np.abs(ref).max(), 1e-30)),
            float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30)))


# A gradient that is exactly zero in the reference (dQ and dK when every row
# keeps a single key: P = 1 and dP - D cancels) is compared absolutely: what is
# left is fp32 rounding of that cancellation.
ZERO_ABS = 1e-5


def assert_grads(got, ref, what=""):
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        if np.abs(r).max() == 0:
            e = float(g.detach().abs().max().item())
            assert e <= ZERO_ABS, f"{what} {name}: max {e:.3e} where the reference is 0"
            continue
        em, e2 = rel_errors(g, r)
        assert em <= REL_MAX and e2 <= REL_L2, f"{what} {name}: rel max {em:.3e}, rel L2 {e2:.3e}"


def run_case(B, H, H_kv, N, d, dt, causal, window, n_sink, alibi, out_f32, seed):
    q, k, v = random_qkv(B, H, H_kv, N, d, dtype=dt, seed=seed)
    do = make_grad_output(B, H, N, d, dtype=dt, seed=seed)
    scale = A.default_scale(d)
    slopes = A.alibi_slopes(H) if alibi else None
    sl64 = slopes.double().numpy() if alibi else None
    Q, K, V, DO = (to_f64(t) for t in (q, k, v, do))
    O, L = oracle.attention(Q, K, V, scale, causal, window, n_sink, slopes=sl64)
    ref = oracle.attention_backward(Q, K, V, DO, scale, causal, window, n_sink, slopes=sl64)
    dev = torch.device("cuda")
    o16 = torch.from_numpy(O).to(dt).to(dev)
    lse = torch.from_numpy(L).float().to(dev)
    got = A.attention_backward(q.to(dev), k.to(dev), v.to(dev), o16, do.to(dev), lse,
                               causal=causal, window=window, n_sink=n_sink, scale=scale,
                               alibi_slopes=slopes.to(dev) if alibi else None, out_f32=out_f32)
    torch.cuda.synchronize()
    assert A.get_status() == A.ATTN_OK
    return got, ref


# (B, H, H_kv, N, d, dtype, causal, window, n_sink, alibi, out_f32)
SWEEP = [
    (1, 1, 1, 128, 64, BF, 1, 0, 0, 0, 1),
    (1, 2, 2, 300, 64, BF, 1, 0, 0, 0, 1),
    (1, 2, 2, 300, 128, BF, 1, 0, 0, 0, 1),
    (1, 4, 2, 256, 128, BF, 0, 0, 0, 0, 1),
    (2, 2, 1, 200, 32, BF, 1, 0, 0, 0, 1),
    (1, 2, 2, 130, 16, BF, 1, 0, 0, 0, 1),
    (1, 2, 2, 77, 128, FP, 0, 0, 0, 0, 1),
    (1, 2, 2, 400, 64, BF, 1, 100, 4, 0, 1),
    (1, 2, 1, 520, 128, FP, 1, 130, 0, 0, 1),
    (1, 4, 4, 257, 128, BF, 1, 0, 0, 1, 1),
    (1, 4, 2, 190, 64, BF, 0, 0, 0, 1, 1),
    (1, 2, 2, 300, 128, BF, 1, 0, 0, 0, 0),
    (1, 4, 1, 333, 64, FP, 1, 0, 0, 0, 0),
    (1, 8, 8, 1, 128, BF, 1, 0, 0, 0, 1),
]


def _id(c):
    B, H, Hk, N, d, dt, ca, w, s, al, f = c
    return (f"B{B}H{H}k{Hk}N{N}d{d}{'bf' if dt == BF else 'fp'}{'c' if ca else 'n'}w{w}s{s}"
            f"{'A' if al else ''}{'f32' if f else 'o16'}")


@pytest.mark.parametrize("case", SWEEP, ids=[_id(c) for c in SWEEP])
def test_bwd_sweep(case):
    B, H, Hk, N, d, dt, causal, window, n_sink, alibi, out_f32 = case
    got, ref = run_case(B, H, Hk, N, d, dt, causal, window, n_sink, alibi, out_f32,
                        seed=N + 7 * d + H)
    assert_grads(got, ref, _id(case))
    if not out_f32:
        assert all(g.dtype == dt for g in got)


def test_bwd_after_gpu_forward():
    """End to end: the backward fed with this library's own forward output."""
    q, k, v = random_qkv(2, 4, 2, 384, 128, dtype=BF, seed=5)
    do = make_grad_output(2, 4, 384, 128, dtype=BF, seed=5)
    scale = A.default_scale(128)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = A.attention(qd, kd, vd, causal=True, scale=scale)
    got = A.attention_backward(qd, kd, vd, o, dod, lse, causal=True, scale=scale, out_f32=True)
    torch.cuda.synchronize()
    ref = oracle.attention_backward(*(to_f64(t) for t in (q, k, v, do)), scale, True)
    assert_grads(got, ref, "after forward")


def test_bwd_dk_dv_deterministic():
    """dK and dV are written once per key tile (bitwise repeatable); dQ is
    summed with atomics and only agrees to rounding."""
    q, k, v = random_qkv(1, 4, 2, 640, 64, dtype=BF, seed=9)
    do = make_grad_output(1, 4, 640, 64, dtype=BF, seed=9)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = A.attention(qd, kd, vd, causal=True)
    a = A.attention_backward(qd, kd, vd, o, dod, lse, causal=True, out_f32=True)
    b = A.attention_backward(qd, kd, vd, o, dod, lse, causal=True, out_f32=True)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert (a[0] - b[0]).abs().max().item() <= 1e-4 * a[0].abs().max().item()


def test_bwd_empty_is_a_no_op():
    dev = torch.device("cuda")
    z = torch.empty((1, 2, 0, 64), dtype=BF, device=dev)
    lse = torch.empty((1, 2, 0), dtype=torch.float32, device=dev)
    dq, dk, dv = A.attention_backward(z, z, z, z, z, lse, causal=True)
    assert dq.shape == (1, 2, 0, 64) and dk.shape == (1, 2, 0, 64)


@pytest.mark.slow
def test_bwd_full_size_c3_sampled_heads():
    """B4 H16 N4096 d128 causal bf16 (the benchmark shape), as bench.py runs
    it: two heads against the oracle's per-head gradients, and the invariant
    sum_j dK_j = 0 (rows of dS sum to zero) for every head."""
    B, H, N, d = 4, 16, 4096, 128
    q, k, v = random_qkv(B, H, H, N, d, dtype=BF, seed=0)
    do = make_grad_output(B, H, N, d, dtype=BF, seed=0)
    scale = A.default_scale(d)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = A.attention(qd, kd, vd, causal=True, scale=scale)
    dq, dk, dv = A.attention_backward(qd, kd, vd, o, dod, lse, causal=True, scale=scale,
                                      out_f32=True)
    torch.cuda.synchronize()
    assert A.get_status() == A.ATTN_OK
    for b, h in ((0, 0), (B - 1, H - 1)):
        ref = oracle.backward_head(to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h]),
                                   to_f64(do[b, h]), scale, True)
        assert_grads((dq[b, h], dk[b, h], dv[b, h]), ref, f"head ({b}, {h})")
    s = dk.double().sum(dim=2).abs().max().item()
    assert s <= 1e-3 * dk.double().abs().sum(dim=2).max().item()
