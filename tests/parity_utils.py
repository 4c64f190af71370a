"""Shared helpers for the GPU parity tests: run the CUDA path, run the oracle on
the same rounded inputs, compare with the tolerances the target fixes.

Tolerances (fp32 accumulation throughout):
  O   : max |err| <= 1e-2 and mean |err| <= 1e-3   (graded on the fp32 output)
  LSE : max |err| <= 1e-3
The 16-bit output adds its own unavoidable rounding: its error is checked
against the same bars plus the rounding floor max|round16(O_oracle) - O_oracle|
(and the mean floor for the mean bar).
"""
from __future__ import annotations

import numpy as np
import torch

import exact_tiled_attention_44_b200 as A
import oracle
from exact_tiled_attention_44_b200.inputs import to_f64

O_MAX, O_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3


def run_gpu(q, k, v, causal, window, n_sink, scale, out_f32):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = A.attention(qd, kd, vd, causal=causal, window=window, n_sink=n_sink, scale=scale,
                         out_f32=out_f32)
    torch.cuda.synchronize()
    return o, lse


def oracle_full(q, k, v, causal, window, n_sink, scale):
    return oracle.attention(to_f64(q), to_f64(k), to_f64(v), scale, causal, window, n_sink)


def oracle_rows(q, k, v, b, h, rows, causal, window, n_sink, scale):
    """Oracle for selected query rows of head (b, h), upcasting only that head."""
    H, H_kv = q.shape[1], k.shape[1]
    g = oracle.kv_head_of(h, H, H_kv)
    Q = to_f64(q[b:b + 1, h:h + 1])
    K = to_f64(k[b:b + 1, g:g + 1])
    V = to_f64(v[b:b + 1, g:g + 1])
    return oracle.attention_bh(Q, K, V, 0, 0, scale, causal, window, n_sink, rows=np.asarray(rows))


def errors(o_gpu, lse_gpu, o_ref, lse_ref):
    o = o_gpu.detach().double().cpu().numpy()
    d = np.abs(o - o_ref)
    out = {"o_max": float(d.max()), "o_mean": float(d.mean())}
    if lse_gpu is not None:
        out["lse_max"] = float(np.abs(lse_gpu.detach().double().cpu().numpy() - lse_ref).max())
    return out


def round_floor(o_ref, dtype):
    r = torch.from_numpy(o_ref).to(dtype).double().numpy()
    d = np.abs(r - o_ref)
    return float(d.max()), float(d.mean())


def assert_parity(err, floor=(0.0, 0.0), what=""):
    assert np.isfinite(err["o_max"]), (what, err)
    assert err["o_max"] <= O_MAX + floor[0], (what, err, floor)
    assert err["o_mean"] <= O_MEAN + floor[1], (what, err, floor)
    if "lse_max" in err:
        assert err["lse_max"] <= LSE_MAX, (what, err)
