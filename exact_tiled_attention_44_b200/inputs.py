"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle legs.

This module only draws random numbers and rounds them to the 16-bit storage
type; it holds none of the attention arithmetic.  Both the CUDA path and the
float64 oracle consume exactly the tensors produced here (the oracle takes
their exact float64 upcast).

Workloads (shapes and mask settings of the pages' examples, scaled to B200
sizes):

* ``c1``: one causal head, B=1 H=1 N=64 d=16, scale 1/sqrt(16), bf16.  The draw
  is the one "Tiled attention with online softmax" (Lab 3) makes: one
  ``numpy.random.default_rng(0)``, then Q, K and V in that order as float64
  standard normals of shape (64, 16); here they are then rounded to bf16.
* ``c2`` / ``c2c``: B=2 H=8 N=1024 d=64 fp16, scale 1/8, non-causal / causal
  on the same inputs (the tensor shape of the PyTorch example in "Flash
  Attention", section "Using Flash Attention in Practice").
* ``c3``: B=4 H=16 N=4096 d=128 bf16 causal, scale 1/sqrt(128).
* ``c4``: B=1 H=32 N=16384 d=128 bf16 causal; in every (b, kv head) 1% of the
  key rows (164 of 16384, drawn without replacement after V) are multiplied by
  8 before rounding, which puts outlier logits in the running max.
* ``c5``: MQA, B=8 H=32 H_kv=1 N=8192 d=128 bf16, causal, sliding window 1024
  plus 64 always-attended sink positions.

For c2..c5: one ``numpy.random.default_rng(seed)`` draws Q, K, V in that order
as float32 standard normals of shape [B, H, N, d] (Q) and [B, H_kv, N, d]
(K, V), then torch rounds them to the 16-bit type (round to nearest even).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    H_kv: int
    N: int
    d: int
    dtype: str            # "bf16" or "fp16"
    causal: bool
    window: int = 0
    n_sink: int = 0
    scale: float = 0.0    # fp32-representable value, fixed once on the host
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    lab3_draw: bool = False

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def f32(x: float) -> float:
    """Round a Python float to the nearest float32 value (the host does this once)."""
    return float(np.float32(x))


WORKLOADS = {
    "c1": Workload("c1", 1, 1, 1, 64, 16, "bf16", True, scale=f32(1 / math.sqrt(16)),
                   lab3_draw=True),
    "c2": Workload("c2", 2, 8, 8, 1024, 64, "fp16", False, scale=f32(1 / 8)),
    "c2c": Workload("c2c", 2, 8, 8, 1024, 64, "fp16", True, scale=f32(1 / 8)),
    "c3": Workload("c3", 4, 16, 16, 4096, 128, "bf16", True, scale=f32(1 / math.sqrt(128))),
    "c4": Workload("c4", 1, 32, 32, 16384, 128, "bf16", True, scale=f32(1 / math.sqrt(128)),
                   outlier_frac=0.01, outlier_mult=8.0),
    "c5": Workload("c5", 8, 32, 1, 8192, 128, "bf16", True, window=1024, n_sink=64,
                   scale=f32(1 / math.sqrt(128))),
}


def make_inputs(w: Workload, seed: int = 0):
    """Return (q, k, v) as contiguous CPU torch tensors of the workload's 16-bit type."""
    if w.lab3_draw:
        if (w.B, w.H, w.H_kv) != (1, 1, 1):
            raise ValueError("the Lab 3 draw is defined for one head")
        rng = np.random.default_rng(seed)
        q, k, v = (rng.normal(size=(w.N, w.d)) for _ in range(3))
        arrs = [a.reshape(1, 1, w.N, w.d) for a in (q, k, v)]
    else:
        rng = np.random.default_rng(seed)
        q = rng.standard_normal((w.B, w.H, w.N, w.d), dtype=np.float32)
        k = rng.standard_normal((w.B, w.H_kv, w.N, w.d), dtype=np.float32)
        v = rng.standard_normal((w.B, w.H_kv, w.N, w.d), dtype=np.float32)
        if w.outlier_frac > 0:
            n_out = int(round(w.outlier_frac * w.N))
            for b in range(w.B):
                for g in range(w.H_kv):
                    idx = rng.choice(w.N, n_out, replace=False)
                    k[b, g, idx, :] *= np.float32(w.outlier_mult)
        arrs = [q, k, v]
    return tuple(torch.from_numpy(np.ascontiguousarray(a)).to(w.torch_dtype).contiguous()
                 for a in arrs)


def random_qkv(B, H, H_kv, N, d, dtype=torch.bfloat16, seed=0, std=1.0):
    """Generic seeded N(0, std^2) inputs rounded to ``dtype`` (parity sweeps)."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, N, d), dtype=np.float32) * np.float32(std)
    k = rng.standard_normal((B, H_kv, N, d), dtype=np.float32) * np.float32(std)
    v = rng.standard_normal((B, H_kv, N, d), dtype=np.float32)
    return tuple(torch.from_numpy(a).to(dtype).contiguous() for a in (q, k, v))


# Decode workload: new query rows against a K/V cache (one decoding step of a
# GQA model; shapes in the range of the pages' KV-cache discussion, "USAAIO
# Lesson 91", slides 31 and 51).
DECODE_WORKLOADS = {
    "dec1": dict(B=8, H=32, H_kv=8, N_q=1, N_kv=8192, d=128, dtype="bf16", causal=True),
}


def make_decode_inputs(B, H, H_kv, N_q, N_kv, d, dtype=torch.bfloat16, seed=0):
    """q [B, H, N_q, d] and the cache k, v [B, H_kv, N_kv, d]: one
    numpy.random.default_rng(seed) draws float32 standard normals for q, k, v in
    that order, rounded to ``dtype``."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, N_q, d), dtype=np.float32)
    k = rng.standard_normal((B, H_kv, N_kv, d), dtype=np.float32)
    v = rng.standard_normal((B, H_kv, N_kv, d), dtype=np.float32)
    return tuple(torch.from_numpy(a).to(dtype).contiguous() for a in (q, k, v))


def make_grad_output(B, H, N, d, dtype=torch.bfloat16, seed=0):
    """Upstream gradient dO [B, H, N, d] for the backward pass: float32
    standard normals from numpy.random.default_rng(seed + 1), rounded to
    ``dtype`` (seed + 1 keeps it independent of the q, k, v draw of ``seed``)."""
    rng = np.random.default_rng(seed + 1)
    g = rng.standard_normal((B, H, N, d), dtype=np.float32)
    return torch.from_numpy(g).to(dtype).contiguous()


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 upcast of a 16-bit tensor (every bf16/fp16 value is a float64 value)."""
    return t.detach().to("cpu", torch.float64).numpy()
