"""Seeded random configurations of the forward against the float64 oracle:
sizes, head grouping, head dim, dtype, mask (causal / window / sinks / none),
ALiBi slopes, output precision and the forced work-unit kind are drawn from
one fixed generator, so every run checks the same 40 cases.  Sampled rows of
every head are compared ("Tiled attention with online softmax", Lab 3: the
tiled result equals the reference)."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A
import oracle
from exact_tiled_attention_44_b200.inputs import random_qkv, to_f64
from parity_utils import assert_parity, errors

pytestmark = pytest.mark.gpu


def _cases(n=40, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        d = int(rng.choice([16, 32, 64, 128]))
        H_kv = int(rng.choice([1, 2, 3, 4]))
        G = int(rng.choice([1, 2, 3, 4, 8]))
        H = H_kv * G
        B = int(rng.integers(1, 4))
        N = int(rng.choice([int(rng.integers(1, 300)), int(rng.integers(300, 1500)),
                            int(rng.integers(1500, 3000))]))
        mask = int(rng.integers(0, 3))          # 0 none, 1 causal, 2 causal + window (+ sinks)
        causal = mask >= 1
        window = int(rng.integers(1, 700)) if mask == 2 else 0
        n_sink = int(rng.integers(0, 200)) if mask == 2 else 0
        alibi = bool(rng.random() < 0.25)
        out_f32 = bool(rng.random() < 0.5)
        kind = int(rng.integers(-1, 3))         # -1 automatic, else forced
        dtype = torch.bfloat16 if rng.random() < 0.7 else torch.float16
        out.append((i, B, H, H_kv, N, d, dtype, causal, window, n_sink, alibi, out_f32, kind))
    return out


CASES = _cases()


@pytest.mark.parametrize("case", CASES, ids=[f"case{c[0]}" for c in CASES])
def test_random_configuration_matches_oracle(case):
    i, B, H, H_kv, N, d, dtype, causal, window, n_sink, alibi, out_f32, kind = case
    q, k, v = random_qkv(B, H, H_kv, N, d, dtype, seed=1000 + i)
    scale = A.default_scale(d)
    slopes = A.alibi_slopes(H) if alibi else None
    assert A.test_force_units(kind) == A.ATTN_OK
    try:
        o, lse = A.attention(q.cuda(), k.cuda(), v.cuda(), causal=causal, window=window,
                             n_sink=n_sink, scale=scale, out_f32=out_f32,
                             alibi_slopes=slopes.cuda() if alibi else None)
        torch.cuda.synchronize()
    finally:
        A.test_force_units(-1)
    assert A.get_status() == A.ATTN_OK
    rng = np.random.default_rng(i)
    sl = slopes.double().numpy() if alibi else None
    for b in range(B):
        for h in range(H):
            g = oracle.kv_head_of(h, H, H_kv)
            Qd = to_f64(q[b:b + 1, h:h + 1])
            Kd, Vd = to_f64(k[b:b + 1, g:g + 1]), to_f64(v[b:b + 1, g:g + 1])
            rows = np.unique(np.concatenate([[0, N - 1, min(127, N - 1), min(128, N - 1)],
                                             rng.integers(0, N, 6)]))
            Or, Lr = oracle.attention_bh(Qd, Kd, Vd, 0, 0, scale, causal, window, n_sink,
                                         rows=rows, slopes=sl[h:h + 1] if alibi else None)
            idx = torch.from_numpy(rows)
            og = o[b, h, idx]
            if not out_f32:
                # the 16-bit output: the bars plus its own rounding floor
                r = torch.from_numpy(Or).to(dtype).double().numpy()
                floor = (float(np.abs(r - Or).max()), float(np.abs(r - Or).mean()))
                assert_parity(errors(og, lse[b, h, idx], Or, Lr), floor, what=f"case {i} ({b},{h})")
            else:
                assert_parity(errors(og, lse[b, h, idx], Or, Lr), what=f"case {i} ({b},{h})")
