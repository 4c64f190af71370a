"""GPU parity of attn_decode (new query rows against a K/V cache, split across
the cache and merged by log-sum-exp) against the float64 decode oracle."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A
import oracle
from exact_tiled_attention_44_b200.inputs import to_f64
from parity_utils import assert_parity, errors, round_floor

pytestmark = pytest.mark.gpu

BF, FP = torch.bfloat16, torch.float16


def _inputs(B, H, H_kv, N_q, N_kv, d, dt, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, N_q, d), dtype=np.float32)
    k = rng.standard_normal((B, H_kv, N_kv, d), dtype=np.float32)
    v = rng.standard_normal((B, H_kv, N_kv, d), dtype=np.float32)
    return tuple(torch.from_numpy(x).to(dt).contiguous() for x in (q, k, v))


def run_decode(q, k, v, causal, window, n_sink, scale, out_f32):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, l = A.decode(qd, kd, vd, causal=causal, window=window, n_sink=n_sink, scale=scale,
                    out_f32=out_f32)
    torch.cuda.synchronize()
    assert A.get_status() == A.ATTN_OK
    return o, l


# (B, H, H_kv, N_q, N_kv, d, dtype, causal, window, n_sink)
SWEEP = [
    (1, 1, 1, 1, 1, 64, BF, 1, 0, 0),
    (1, 4, 4, 1, 63, 128, BF, 1, 0, 0),
    (2, 8, 2, 1, 300, 128, FP, 1, 0, 0),
    (1, 8, 1, 2, 1000, 64, BF, 1, 0, 0),
    (2, 32, 8, 1, 4096, 128, BF, 1, 0, 0),
    (1, 16, 1, 4, 2500, 128, BF, 0, 0, 0),
    (1, 32, 1, 2, 8192 + 77, 128, BF, 1, 0, 0),
    (1, 4, 2, 16, 3000, 64, FP, 1, 0, 0),
    (1, 8, 8, 3, 5000, 128, BF, 1, 1024, 64),
    (1, 32, 1, 1, 8192, 128, BF, 1, 1024, 64),
    (2, 2, 1, 8, 777, 128, FP, 1, 100, 3),
    (1, 64, 1, 1, 20000, 64, BF, 1, 0, 0),
]


def _id(c):
    B, H, Hk, Nq, Nkv, d, dt, ca, w, s = c
    return f"B{B}H{H}k{Hk}q{Nq}kv{Nkv}d{d}{'bf' if dt == BF else 'fp'}{'c' if ca else 'n'}w{w}s{s}"


@pytest.mark.parametrize("case", SWEEP, ids=[_id(c) for c in SWEEP])
def test_decode_sweep(case):
    B, H, Hk, Nq, Nkv, d, dt, causal, window, n_sink = case
    q, k, v = _inputs(B, H, Hk, Nq, Nkv, d, dt, seed=Nkv + 17 * d + Nq)
    scale = A.default_scale(d)
    Or, Lr = oracle.decode(to_f64(q), to_f64(k), to_f64(v), scale, bool(causal), window, n_sink)
    o32, l32 = run_decode(q, k, v, bool(causal), window, n_sink, scale, True)
    assert_parity(errors(o32, l32, Or, Lr), what="fp32 out")
    o16, l16 = run_decode(q, k, v, bool(causal), window, n_sink, scale, False)
    assert_parity(errors(o16, l16, Or, Lr), round_floor(Or, dt), what="16-bit out")
    assert torch.equal(l16, l32)


def test_decode_deterministic_and_workspace_reuse():
    q, k, v = (t.cuda() for t in _inputs(2, 32, 8, 1, 6000, 128, BF, seed=1))
    ws = torch.empty(A.decode_workspace_bytes(2, 32, 8, 1, 6000, 128), dtype=torch.uint8,
                     device="cuda")
    outs = [A.decode(q, k, v, workspace=ws) for _ in range(3)]
    torch.cuda.synchronize()
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])


def test_decode_matches_the_forward_last_rows():
    """Decode of the last N_q rows equals the forward over the whole sequence
    on those rows (both against the oracle, and within the tolerance of each
    other)."""
    B, H, Hk, N, d = 1, 8, 2, 1500, 128
    rng = np.random.default_rng(5)
    qf = torch.from_numpy(rng.standard_normal((B, H, N, d), dtype=np.float32)).to(BF)
    k = torch.from_numpy(rng.standard_normal((B, Hk, N, d), dtype=np.float32)).to(BF)
    v = torch.from_numpy(rng.standard_normal((B, Hk, N, d), dtype=np.float32)).to(BF)
    of, lf = A.attention(qf.cuda(), k.cuda(), v.cuda(), causal=True, out_f32=True)
    qd = qf[:, :, -4:].contiguous()
    od, ld = run_decode(qd, k, v, True, 0, 0, A.default_scale(d), True)
    assert (od - of[:, :, -4:]).abs().max().item() < 1e-2
    assert (ld - lf[:, :, -4:]).abs().max().item() < 1e-3


def test_decode_lse_optional_and_binding_checks():
    q, k, v = (t.cuda() for t in _inputs(1, 8, 2, 1, 3000, 64, BF, seed=2))
    o1, l1 = A.decode(q, k, v)
    o2, l2 = A.decode(q, k, v, return_lse=False)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and l2 is None
    with pytest.raises(A.AttnError):
        A.decode(q, k, v, workspace=torch.empty(8, dtype=torch.uint8, device="cuda"))
