"""GPU tests of grouped query heads in the forward ("USAAIO Lesson 91", slide
32: GQA / MQA, query head h reads K/V head h / (H / H_kv)).  Every row must come
out bitwise as it does when the K/V heads are repeated to plain multi-head
attention, and within the oracle's tolerance, for even and odd group sizes,
windows with sinks, and ALiBi (each query head its own slope)."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A
import oracle
from exact_tiled_attention_44_b200.inputs import random_qkv, to_f64

pytestmark = pytest.mark.gpu

BF, FP = torch.bfloat16, torch.float16

# (B, H, H_kv, N, d, dtype, causal, window, n_sink, alibi); G = H / H_kv
CASES = [
    (1, 2, 1, 300, 128, BF, 1, 0, 0, 0),       # G = 2, ragged tail
    (2, 8, 2, 257, 64, FP, 1, 0, 0, 0),        # G = 4
    (1, 8, 1, 1000, 128, BF, 1, 200, 4, 0),    # MQA, window + sinks
    (1, 4, 2, 384, 128, BF, 0, 0, 0, 0),       # non-causal
    (1, 6, 3, 500, 64, BF, 1, 0, 0, 0),        # G = 2, three groups
    (1, 6, 2, 333, 128, BF, 1, 0, 0, 0),       # G = 3: odd group
    (1, 4, 1, 640, 128, BF, 1, 0, 0, 1),       # ALiBi: each head its own slope
    (1, 16, 2, 129, 32, FP, 1, 0, 0, 1),       # ALiBi, G = 8
    (2, 32, 1, 77, 16, BF, 1, 0, 0, 0),        # G = 32, one tile
]


def _id(c):
    B, H, Hk, N, d, dt, ca, w, s, al = c
    return f"B{B}H{H}k{Hk}N{N}d{d}{'bf' if dt == BF else 'fp'}{'c' if ca else 'n'}w{w}s{s}{'A' if al else ''}"


def _run(q, k, v, causal, window, n_sink, scale, slopes):
    dev = torch.device("cuda")
    o, l = A.attention(q.to(dev), k.to(dev), v.to(dev), causal=causal, window=window,
                       n_sink=n_sink, scale=scale, out_f32=True,
                       alibi_slopes=slopes.to(dev) if slopes is not None else None)
    torch.cuda.synchronize()
    assert A.get_status() == A.ATTN_OK
    return o, l


@pytest.mark.parametrize("case", CASES, ids=[_id(c) for c in CASES])
def test_grouped_heads_equal_repeated_heads_and_oracle(case):
    B, H, Hk, N, d, dt, causal, window, n_sink, alibi = case
    q, k, v = random_qkv(B, H, Hk, N, d, dtype=dt, seed=N + H + d)
    scale = A.default_scale(d)
    slopes = A.alibi_slopes(H) if alibi else None
    o1, l1 = _run(q, k, v, causal, window, n_sink, scale, slopes)
    G = H // Hk
    kr = k.repeat_interleave(G, 1).contiguous()
    vr = v.repeat_interleave(G, 1).contiguous()
    o2, l2 = _run(q, kr, vr, causal, window, n_sink, scale, slopes)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    O, L = oracle.attention(to_f64(q), to_f64(k), to_f64(v), scale, causal, window, n_sink,
                            slopes=slopes.double().numpy() if alibi else None)
    assert np.abs(o1.double().cpu().numpy() - O).max() <= 1e-2
    assert np.abs(o1.double().cpu().numpy() - O).mean() <= 1e-3
    assert np.abs(l1.double().cpu().numpy() - L).max() <= 1e-3
