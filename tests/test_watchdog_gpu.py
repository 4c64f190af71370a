"""Failure detection on the GPU without a fault: a launch whose copy warp
issues nothing makes every other wait run into the watchdog; the kernel must
report ATTN_ERR_DEVICE_TIMEOUT through the status word, release its resources
and return, leaving the context usable for the next, correct launch.  Covered
for the three kernels: the forward, the tiled backward and the split-KV
decoding step."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A
import oracle
from exact_tiled_attention_44_b200.inputs import make_decode_inputs, make_grad_output, random_qkv, to_f64
from parity_utils import assert_parity, errors, oracle_full

pytestmark = pytest.mark.gpu


def test_expired_waits_report_timeout_and_context_survives():
    q, k, v = random_qkv(1, 2, 2, 300, 64, torch.bfloat16, seed=2)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    assert A.get_status() == A.ATTN_OK
    old = A.set_watchdog_ns(1_000_000)          # 1 ms per wait
    try:
        assert A.test_withhold_loads(1) == A.ATTN_OK
        A.attention(qd, kd, vd, causal=True)
        torch.cuda.synchronize()
        assert A.get_status() == A.ATTN_ERR_DEVICE_TIMEOUT
        assert A.get_status() == A.ATTN_OK      # read-and-clear
    finally:
        A.test_withhold_loads(0)
        A.set_watchdog_ns(old)
    # the next launch runs normally and is correct
    o, l = A.attention(qd, kd, vd, causal=True, out_f32=True)
    torch.cuda.synchronize()
    assert A.get_status() == A.ATTN_OK
    Or, Lr = oracle_full(q, k, v, True, 0, 0, A.default_scale(64))
    assert_parity(errors(o, l, Or, Lr), what="after a timed-out launch")


def test_hook_counts_launches():
    q, k, v = (t.cuda() for t in random_qkv(1, 1, 1, 130, 128, torch.bfloat16, seed=3))
    old = A.set_watchdog_ns(1_000_000)
    try:
        A.test_withhold_loads(2)
        for _ in range(2):
            A.attention(q, k, v, causal=True)
            torch.cuda.synchronize()
            assert A.get_status() == A.ATTN_ERR_DEVICE_TIMEOUT
        A.attention(q, k, v, causal=True)
        torch.cuda.synchronize()
        assert A.get_status() == A.ATTN_OK
    finally:
        A.test_withhold_loads(0)
        A.set_watchdog_ns(old)


def _withheld(call):
    """Runs call() with the next launch's loads withheld and a 1 ms watchdog;
    checks the reported timeout and the read-and-clear of the status word."""
    assert A.get_status() == A.ATTN_OK
    old = A.set_watchdog_ns(1_000_000)
    try:
        assert A.test_withhold_loads(1) == A.ATTN_OK
        call()
        torch.cuda.synchronize()
        assert A.get_status() == A.ATTN_ERR_DEVICE_TIMEOUT
        assert A.get_status() == A.ATTN_OK
    finally:
        A.test_withhold_loads(0)
        A.set_watchdog_ns(old)


def test_backward_expiry_reports_timeout_and_next_call_is_correct():
    B, H, H_kv, N, d = 1, 2, 1, 300, 128
    q, k, v = random_qkv(B, H, H_kv, N, d, torch.bfloat16, seed=5)
    do = make_grad_output(B, H, N, d, seed=5)
    scale = A.default_scale(d)
    Q, K, V, DO = (to_f64(t) for t in (q, k, v, do))
    O, L = oracle.attention(Q, K, V, scale, True)
    dev = torch.device("cuda")
    args = (q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(O).to(q.dtype).to(dev), do.to(dev),
            torch.from_numpy(L).float().to(dev))
    _withheld(lambda: A.attention_backward(*args, causal=True, scale=scale, out_f32=True))
    got = A.attention_backward(*args, causal=True, scale=scale, out_f32=True)
    torch.cuda.synchronize()
    assert A.get_status() == A.ATTN_OK
    ref = oracle.attention_backward(Q, K, V, DO, scale, True)
    for g, r in zip(got, ref):
        dg = g.double().cpu().numpy() - r
        assert np.abs(dg).max() <= 2e-2 * np.abs(r).max()
        assert np.linalg.norm(dg) <= 1e-2 * np.linalg.norm(r)


@pytest.mark.parametrize("H,H_kv,N_q,N_kv", [(8, 2, 1, 3000), (32, 1, 2, 1500)])
def test_decode_expiry_reports_timeout_and_next_call_is_correct(H, H_kv, N_q, N_kv):
    # (8, 2, 1, 3000): 4 query rows per group; (32, 1, 2, 1500): 64 rows, the
    # largest group
    q, k, v = make_decode_inputs(1, H, H_kv, N_q, N_kv, 128, seed=6)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    _withheld(lambda: A.decode(qd, kd, vd, causal=True))
    o, l = A.decode(qd, kd, vd, causal=True, out_f32=True)
    torch.cuda.synchronize()
    assert A.get_status() == A.ATTN_OK
    Or, Lr = oracle.decode(to_f64(q), to_f64(k), to_f64(v), A.default_scale(128), True)
    assert_parity(errors(o, l, Or, Lr), what="decode after a timed-out launch")
