"""The kernels' schedule on the GPU: the score tiles the forward computes and
the steps the tiled backward takes, counted on the device through the
attn_test_count_blocks hook, equal attn_visited_blocks() x B x H -- the
(128-row query tile, 128-key block) pairs that hold at least one kept pair
("Tiled attention with online softmax", exercise 3: count the block pairs the
tiled loop visits against the full n^2)."""
import pytest
import torch

import exact_tiled_attention_44_b200 as A
from exact_tiled_attention_44_b200.inputs import WORKLOADS, make_grad_output, random_qkv

pytestmark = pytest.mark.gpu

BF, FP = torch.bfloat16, torch.float16

# (B, H, H_kv, N, d, dtype, causal, window, n_sink)
CASES = [
    (1, 1, 1, 64, 16, BF, 1, 0, 0),          # c1 shape
    (2, 8, 8, 1024, 64, FP, 0, 0, 0),        # c2 shape
    (2, 8, 8, 1024, 64, FP, 1, 0, 0),        # c2c shape
    (1, 2, 2, 4096, 128, BF, 1, 0, 0),       # c3 heads
    (1, 4, 1, 8192, 128, BF, 1, 1024, 64),   # c5 heads (MQA, window + sinks)
    (1, 3, 1, 1000, 64, BF, 1, 300, 200),    # ragged, sinks beyond one block
    (2, 2, 2, 777, 128, BF, 1, 1, 0),        # window 1: the diagonal only
    (1, 2, 1, 1300, 32, FP, 0, 0, 0),        # ragged, non-causal
]


def _count(fn):
    counter = torch.zeros(1, dtype=torch.int64, device="cuda")
    assert A.test_count_blocks(counter) == A.ATTN_OK
    try:
        fn()
        torch.cuda.synchronize()
    finally:
        A.test_count_blocks(None)
    assert A.get_status() == A.ATTN_OK
    return int(counter.item())


@pytest.mark.parametrize("case", CASES)
def test_forward_computes_exactly_the_visited_blocks(case):
    B, H, H_kv, N, d, dt, causal, window, n_sink = case
    q, k, v = (t.cuda() for t in random_qkv(B, H, H_kv, N, d, dt, seed=1))
    got = _count(lambda: A.attention(q, k, v, causal=bool(causal), window=window, n_sink=n_sink))
    assert got == A.visited_blocks(N, bool(causal), window, n_sink) * B * H


@pytest.mark.parametrize("mode", [0, 1, 2], ids=["pairs", "split", "heads"])
@pytest.mark.parametrize("case", CASES)
def test_forward_unit_shapes_compute_exactly_the_visited_blocks(case, mode):
    """Pairs of Q tiles, single Q tiles shared by both softmax warpgroups and
    pairs of query heads of one K/V head compute the same set of score tiles."""
    B, H, H_kv, N, d, dt, causal, window, n_sink = case
    q, k, v = (t.cuda() for t in random_qkv(B, H, H_kv, N, d, dt, seed=1))
    assert A.test_force_units(mode) == A.ATTN_OK
    try:
        got = _count(lambda: A.attention(q, k, v, causal=bool(causal), window=window,
                                         n_sink=n_sink))
    finally:
        A.test_force_units(-1)
    assert got == A.visited_blocks(N, bool(causal), window, n_sink) * B * H


@pytest.mark.parametrize("case", CASES)
def test_forward_with_position_bias_computes_exactly_the_visited_blocks(case):
    """With ALiBi slopes the forward walks every unit's blocks in descending
    order; the set of score tiles it computes is the same."""
    B, H, H_kv, N, d, dt, causal, window, n_sink = case
    q, k, v = (t.cuda() for t in random_qkv(B, H, H_kv, N, d, dt, seed=1))
    s = A.alibi_slopes(H, "cuda")
    got = _count(lambda: A.attention(q, k, v, causal=bool(causal), window=window, n_sink=n_sink,
                                     alibi_slopes=s))
    assert got == A.visited_blocks(N, bool(causal), window, n_sink) * B * H


@pytest.mark.parametrize("case", CASES)
def test_backward_steps_are_exactly_the_visited_blocks(case):
    B, H, H_kv, N, d, dt, causal, window, n_sink = case
    q, k, v = (t.cuda() for t in random_qkv(B, H, H_kv, N, d, dt, seed=1))
    o, lse = A.attention(q, k, v, causal=bool(causal), window=window, n_sink=n_sink)
    do = make_grad_output(B, H, N, d, dtype=dt, seed=1).cuda()
    got = _count(lambda: A.attention_backward(q, k, v, o, do, lse, causal=bool(causal),
                                              window=window, n_sink=n_sink))
    assert got == A.visited_blocks(N, bool(causal), window, n_sink) * B * H


def test_hook_off_by_default_and_counts_accumulate():
    w = WORKLOADS["c2c"]
    q, k, v = (t.cuda() for t in random_qkv(w.B, w.H, w.H_kv, w.N, w.d, w.torch_dtype, seed=2))
    counter = torch.zeros(1, dtype=torch.int64, device="cuda")
    A.test_count_blocks(counter)
    try:
        for _ in range(3):
            A.attention(q, k, v, causal=True)
        torch.cuda.synchronize()
    finally:
        A.test_count_blocks(None)
    A.attention(q, k, v, causal=True)          # not counted
    torch.cuda.synchronize()
    assert int(counter.item()) == 3 * A.visited_blocks(w.N, True) * w.B * w.H
