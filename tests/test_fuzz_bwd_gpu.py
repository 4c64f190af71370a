"""Seeded random configurations of the backward (dQ, dK, dV) against the
float64 gradient oracle, with the bars of the backward sweep (relative to each
gradient's size): sizes, head grouping, d, dtype, mask, ALiBi slopes and
gradient precision are drawn from one fixed generator."""
import numpy as np
import pytest
import torch

from test_bwd_gpu import BF, FP, assert_grads, run_case

pytestmark = pytest.mark.gpu


def _cases(n=16, seed=4242):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        d = int(rng.choice([16, 32, 64, 128]))
        H_kv = int(rng.choice([1, 2]))
        H = H_kv * int(rng.choice([1, 2, 4]))
        B = int(rng.integers(1, 3))
        N = int(rng.integers(1, 700))
        mask = int(rng.integers(0, 3))
        causal = mask >= 1
        window = int(rng.integers(1, 300)) if mask == 2 else 0
        n_sink = int(rng.integers(0, 80)) if mask == 2 else 0
        alibi = bool(rng.random() < 0.3)
        out_f32 = bool(rng.random() < 0.5)
        dt = BF if rng.random() < 0.7 else FP
        out.append((i, B, H, H_kv, N, d, dt, causal, window, n_sink, alibi, out_f32))
    return out


CASES = _cases()


@pytest.mark.parametrize("case", CASES, ids=[f"case{c[0]}" for c in CASES])
def test_random_backward_matches_oracle(case):
    i, B, H, H_kv, N, d, dt, causal, window, n_sink, alibi, out_f32 = case
    got, ref = run_case(B, H, H_kv, N, d, dt, causal, window, n_sink, alibi, out_f32, seed=900 + i)
    assert_grads(got, ref, what=f"backward case {i}")
