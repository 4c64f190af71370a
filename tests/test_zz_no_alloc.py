"""attn_decode_noalloc: attn_decode with its scratch in a static device array
(no caller workspace, nothing allocated).  Collected last; passes alone and
after the other GPU tests."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A

BF = torch.bfloat16


def _noalloc(q, k, v, o, lse, causal=True, window=0, n_sink=0, scale=0.088, dtype=A.ATTN_BF16):
    B, H, N_q, d = q.shape
    H_kv, N_kv = k.shape[1], k.shape[2]
    return A.attn_decode_noalloc_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                     lse.data_ptr() if lse is not None else None, B, H, H_kv,
                                     N_q, N_kv, d, causal, window, n_sink, scale, dtype,
                                     torch.cuda.current_stream().cuda_stream)


def test_size_limit_is_rejected_before_launch():
    """A split plan whose scratch exceeds the static array is refused on the
    host (fake, never dereferenced, widely spaced addresses)."""
    assert A.decode_workspace_bytes(1, 64, 1, 1, 65536, 128) > 4 << 20
    rc = A.attn_decode_noalloc_raw(1 << 28, 2 << 28, 3 << 28, 4 << 28, 5 << 28, 1, 64, 1, 1, 65536,
                                   128, 1, 0, 0, 0.088, A.ATTN_BF16, None)
    assert rc == A.ATTN_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_two_calls_match_the_workspace_entry_point():
    rng = np.random.default_rng(11)
    B, H, H_kv, N_q, N_kv, d = 2, 16, 4, 2, 5000, 128
    q = torch.from_numpy(rng.standard_normal((B, H, N_q, d), dtype=np.float32)).to(BF).cuda()
    k = torch.from_numpy(rng.standard_normal((B, H_kv, N_kv, d), dtype=np.float32)).to(BF).cuda()
    v = torch.from_numpy(rng.standard_normal((B, H_kv, N_kv, d), dtype=np.float32)).to(BF).cuda()
    assert A.decode_workspace_bytes(B, H, H_kv, N_q, N_kv, d) > 0      # the cache is split
    o_ref, l_ref = A.decode(q, k, v, scale=0.088)
    outs = []
    for _ in range(2):
        o = torch.empty_like(q)
        l = torch.empty((B, H, N_q), device="cuda")
        assert _noalloc(q, k, v, o, l) == A.ATTN_OK
        outs.append((o, l))
    torch.cuda.synchronize()
    assert A.get_status() == A.ATTN_OK
    for o, l in outs:
        assert torch.equal(o, o_ref) and torch.equal(l, l_ref)
