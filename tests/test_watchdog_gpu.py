"""Failure detection on the GPU without a fault: a launch whose copy warp
issues nothing makes every other wait run into the watchdog; the kernel must
report ATTN_ERR_DEVICE_TIMEOUT through the status word, release its resources
and return, leaving the context usable for the next, correct launch."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A
from exact_tiled_attention_44_b200.inputs import random_qkv
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
