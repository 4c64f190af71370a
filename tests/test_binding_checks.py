"""The Python binding refuses caller-provided buffers that do not match what
the C ABI will write (it sizes every tensor from B, H, H_kv, N and d), before
any device work.  CPU tensors stand in here: the checks run before the CUDA
check, so a wrong buffer is reported as such, and a right one reaches the
"takes CUDA tensors" refusal."""
import pytest
import torch

import exact_tiled_attention_44_b200 as A

BF = torch.bfloat16


def qkv(B=1, H=4, H_kv=2, N=33, d=64, dt=BF):
    return (torch.zeros(B, H, N, d, dtype=dt), torch.zeros(B, H_kv, N, d, dtype=dt),
            torch.zeros(B, H_kv, N, d, dtype=dt))


def test_attention_out_and_lse_are_checked():
    q, k, v = qkv()
    with pytest.raises(ValueError, match="out must be"):
        A.attention(q, k, v, out=torch.zeros(1, 4, 32, 64, dtype=BF))
    with pytest.raises(ValueError, match="out must be"):
        A.attention(q, k, v, out=torch.zeros(1, 4, 33, 64, dtype=BF), out_f32=True)
    with pytest.raises(ValueError, match="out must be"):
        A.attention(q, k, v, out=torch.zeros(1, 4, 64, 33, dtype=BF).transpose(2, 3))
    with pytest.raises(ValueError, match="lse must be"):
        A.attention(q, k, v, lse=torch.zeros(1, 4, 33, dtype=torch.float16))
    with pytest.raises(ValueError, match="CUDA"):
        A.attention(q, k, v, out=torch.zeros(1, 4, 33, 64, dtype=BF),
                    lse=torch.zeros(1, 4, 33))


def test_decode_buffers_are_checked():
    q = torch.zeros(1, 4, 2, 64, dtype=BF)
    k = torch.zeros(1, 2, 100, 64, dtype=BF)
    with pytest.raises(ValueError, match="out must be"):
        A.decode(q, k, k, out=torch.zeros(1, 4, 1, 64, dtype=BF))
    with pytest.raises(ValueError, match="lse must be"):
        A.decode(q, k, k, lse=torch.zeros(1, 4, 3))
    with pytest.raises(ValueError, match="workspace must be"):
        A.decode(q, k, k, workspace=torch.zeros(64, dtype=torch.float32))
    with pytest.raises(ValueError, match="CUDA"):
        A.decode(q, k, k, out=torch.zeros(1, 4, 2, 64, dtype=BF), lse=torch.zeros(1, 4, 2))


def test_backward_buffers_are_checked():
    q, k, v = qkv()
    lse = torch.zeros(1, 4, 33)
    good = (torch.zeros_like(q), torch.zeros_like(k), torch.zeros_like(v))
    with pytest.raises(ValueError, match="dk must be"):
        A.attention_backward(q, k, v, q, q, lse, grads=(good[0], torch.zeros_like(q), good[2]))
    with pytest.raises(ValueError, match="dq must be"):
        A.attention_backward(q, k, v, q, q, lse, grads=good, out_f32=True)
    with pytest.raises(ValueError, match="grads must be"):
        A.attention_backward(q, k, v, q, q, lse, grads=good[:2])
    with pytest.raises(ValueError, match="workspace must be"):
        A.attention_backward(q, k, v, q, q, lse, workspace=torch.zeros(8, 8, dtype=torch.uint8))
    with pytest.raises(ValueError, match="lse must be"):
        A.attention_backward(q, k, v, q, q, torch.zeros(1, 4, 32))
    with pytest.raises(ValueError, match="dout must be"):
        A.attention_backward(q, k, v, q, q.float(), lse)
    with pytest.raises(ValueError, match="CUDA"):
        A.attention_backward(q, k, v, q, q, lse, grads=good)


def test_host_entry_buffers_are_checked():
    q, k, v = qkv()
    staging = {"q": q.clone(), "k": k.clone(), "v": v.clone(), "o": torch.zeros_like(q)}
    with pytest.raises(ValueError, match="out must be"):
        A.attention_from_host(q, k, v, staging=staging, out=torch.zeros(1, 4, 33, 32, dtype=BF))
    with pytest.raises(ValueError, match="staging needs an 'lse'"):
        A.attention_from_host(q, k, v, staging=staging, out=torch.zeros_like(q),
                              lse=torch.zeros(1, 4, 33))
    bad = dict(staging, k=torch.zeros_like(q))
    with pytest.raises(ValueError, match=r"staging\['k'\]"):
        A.attention_from_host(q, k, v, staging=bad, out=torch.zeros_like(q))
    with pytest.raises(ValueError, match="staging tensors must be CUDA"):
        A.attention_from_host(q, k, v, staging=staging, out=torch.zeros_like(q))


def test_mixed_devices_and_dtypes_are_refused():
    q, k, v = qkv()
    with pytest.raises(TypeError):
        A.attention(q, k.half(), v)
    with pytest.raises(ValueError, match="shape mismatch"):
        A.attention(q, k[:, :, :5], v)
