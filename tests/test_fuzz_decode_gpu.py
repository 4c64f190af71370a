"""Seeded random decoding steps against the float64 decode oracle: batch, head
grouping (up to 64 query rows per K/V head), new rows, cache length, head
dim, dtype, mask and output precision are drawn from one fixed generator, so
that the split of the cache into ranges and the merge of split groups meet
many plans ("Building a FlashAttention-style tiled self-attention block in
pure NumPy", "Extending It", item 6: split, then reduce the partial outputs)."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A
import oracle
from exact_tiled_attention_44_b200.inputs import to_f64
from parity_utils import assert_parity, errors, round_floor

pytestmark = pytest.mark.gpu


def _cases(n=30, seed=77):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        d = int(rng.choice([64, 128]))
        H_kv = int(rng.choice([1, 2, 4, 8]))
        N_q = int(rng.choice([1, 1, 2, 3, 4, 8]))
        G = int(rng.choice([1, 2, 4, 8]))
        while G * N_q > 64:
            G //= 2
        H = H_kv * max(G, 1)
        B = int(rng.integers(1, 5))
        N_kv = int(rng.integers(N_q, 12000))
        mask = int(rng.integers(0, 3))
        causal = mask >= 1
        window = int(rng.integers(1, 2000)) if mask == 2 else 0
        n_sink = int(rng.integers(0, 300)) if mask == 2 else 0
        out_f32 = bool(rng.random() < 0.5)
        dtype = torch.bfloat16 if rng.random() < 0.7 else torch.float16
        out.append((i, B, H, H_kv, N_q, N_kv, d, dtype, causal, window, n_sink, out_f32))
    return out


CASES = _cases()


@pytest.mark.parametrize("case", CASES, ids=[f"case{c[0]}" for c in CASES])
def test_random_decoding_step_matches_oracle(case):
    i, B, H, H_kv, N_q, N_kv, d, dtype, causal, window, n_sink, out_f32 = case
    rng = np.random.default_rng(500 + i)
    q, k, v = (torch.from_numpy(rng.standard_normal(s, dtype=np.float32)).to(dtype).contiguous()
               for s in ((B, H, N_q, d), (B, H_kv, N_kv, d), (B, H_kv, N_kv, d)))
    scale = A.default_scale(d)
    o, l = A.decode(q.cuda(), k.cuda(), v.cuda(), causal=causal, window=window, n_sink=n_sink,
                    scale=scale, out_f32=out_f32)
    torch.cuda.synchronize()
    assert A.get_status() == A.ATTN_OK
    Or, Lr = oracle.decode(to_f64(q), to_f64(k), to_f64(v), scale, causal, window, n_sink)
    floor = (0.0, 0.0) if out_f32 else round_floor(Or, dtype)
    assert_parity(errors(o, l, Or, Lr), floor, what=f"decode case {i}")
