"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded, 16-bit-rounded inputs, plus oracle-free invariants."""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A
from exact_tiled_attention_44_b200.inputs import WORKLOADS, make_inputs, random_qkv, to_f64
from parity_utils import (assert_parity, errors, oracle_full, oracle_rows, round_floor, run_gpu)

pytestmark = pytest.mark.gpu

BF, FP = torch.bfloat16, torch.float16

# (B, H, H_kv, N, d, dtype, causal, window, n_sink)
SWEEP = [
    (1, 1, 1, 1, 64, BF, 1, 0, 0),
    (1, 1, 1, 1, 128, FP, 0, 0, 0),
    (1, 1, 1, 7, 16, BF, 1, 0, 0),
    (1, 2, 1, 63, 128, BF, 1, 0, 0),
    (1, 1, 1, 64, 16, BF, 0, 0, 0),
    (2, 2, 2, 65, 64, FP, 1, 0, 0),
    (1, 3, 1, 127, 32, BF, 0, 0, 0),
    (1, 1, 1, 128, 128, BF, 1, 0, 0),
    (1, 2, 2, 129, 128, FP, 0, 0, 0),
    (1, 2, 2, 200, 64, FP, 1, 0, 0),
    (2, 4, 2, 255, 128, BF, 1, 0, 0),
    (1, 2, 1, 256, 32, FP, 1, 0, 0),
    (1, 2, 2, 257, 16, BF, 0, 0, 0),
    (1, 2, 2, 384, 128, BF, 0, 0, 0),
    (1, 4, 4, 500, 64, BF, 1, 0, 0),
    (1, 2, 1, 640, 128, FP, 1, 0, 0),
    (1, 1, 1, 1100, 128, BF, 1, 0, 0),
    (1, 2, 2, 500, 128, BF, 1, 1, 0),
    (1, 2, 2, 500, 64, BF, 1, 100, 0),
    (1, 2, 1, 700, 128, BF, 1, 130, 3),
    (1, 2, 2, 900, 128, FP, 1, 128, 64),
    (1, 1, 1, 900, 32, BF, 1, 300, 200),
    (1, 2, 2, 300, 128, BF, 1, 1000, 5),
    (1, 2, 1, 1000, 16, BF, 1, 257, 129),
    (2, 8, 1, 600, 128, BF, 1, 256, 64),
]


def _id(c):
    B, H, Hk, N, d, dt, ca, w, s = c
    return f"B{B}H{H}k{Hk}N{N}d{d}{'bf' if dt == BF else 'fp'}{'c' if ca else 'n'}w{w}s{s}"


@pytest.mark.parametrize("case", SWEEP, ids=[_id(c) for c in SWEEP])
def test_sweep_full_parity(case):
    B, H, Hk, N, d, dt, causal, window, n_sink = case
    q, k, v = random_qkv(B, H, Hk, N, d, dt, seed=N * 131 + d)
    scale = A.default_scale(d)
    Or, Lr = oracle_full(q, k, v, bool(causal), window, n_sink, scale)
    o32, l32 = run_gpu(q, k, v, bool(causal), window, n_sink, scale, out_f32=True)
    assert_parity(errors(o32, l32, Or, Lr), what="fp32 out")
    o16, l16 = run_gpu(q, k, v, bool(causal), window, n_sink, scale, out_f32=False)
    assert o16.dtype == dt
    assert_parity(errors(o16, l16, Or, Lr), round_floor(Or, dt), what="16-bit out")
    # the 16-bit output is the fp32 output rounded once
    assert torch.equal(o16, o32.to(dt))
    assert torch.equal(l16, l32)


@pytest.fixture
def units():
    """Runs a test under a forced work-unit shape and restores the automatic choice."""
    def force(mode):
        assert A.test_force_units(mode) == A.ATTN_OK
    yield force
    A.test_force_units(-1)


@pytest.mark.parametrize("mode", [0, 1, 2], ids=["pairs", "split", "heads"])
@pytest.mark.parametrize("case", SWEEP, ids=[_id(c) for c in SWEEP])
def test_sweep_every_unit_shape(case, mode, units):
    """Every sweep case with pairs of Q tiles, with single Q tiles whose key
    blocks the two softmax warpgroups share, and with pairs of query heads
    that share a K/V head (the automatic choice takes one of them by problem
    size): each against the oracle, the 16-bit output the fp32 one rounded
    once."""
    units(mode)
    B, H, Hk, N, d, dt, causal, window, n_sink = case
    q, k, v = random_qkv(B, H, Hk, N, d, dt, seed=N * 131 + d)
    scale = A.default_scale(d)
    Or, Lr = oracle_full(q, k, v, bool(causal), window, n_sink, scale)
    o32, l32 = run_gpu(q, k, v, bool(causal), window, n_sink, scale, out_f32=True)
    assert_parity(errors(o32, l32, Or, Lr), what="fp32 out")
    o16, l16 = run_gpu(q, k, v, bool(causal), window, n_sink, scale, out_f32=False)
    assert_parity(errors(o16, l16, Or, Lr), round_floor(Or, dt), what="16-bit out")
    assert torch.equal(o16, o32.to(dt)) and torch.equal(l16, l32)
    assert A.get_status() == A.ATTN_OK


@pytest.mark.parametrize("case", [(2, 8, 2, 700, 128, BF, 1, 0, 0), (1, 6, 1, 1000, 64, FP, 1, 300, 65),
                                  (1, 5, 1, 300, 32, BF, 0, 0, 0), (2, 4, 4, 257, 128, BF, 1, 0, 0)])
def test_head_pair_units_equal_pair_units_bitwise(case, units):
    """Two query heads of one K/V head per unit compute each row exactly as a
    pair of Q tiles of one head does (same blocks, same order): the outputs
    are bitwise equal, odd head counts and G = 1 included."""
    B, H, Hk, N, d, dt, causal, window, n_sink = case
    q, k, v = random_qkv(B, H, Hk, N, d, dt, seed=N + H)
    scale = A.default_scale(d)
    units(0)
    o0, l0 = run_gpu(q, k, v, bool(causal), window, n_sink, scale, out_f32=False)
    units(2)
    o2, l2 = run_gpu(q, k, v, bool(causal), window, n_sink, scale, out_f32=False)
    assert torch.equal(o0, o2) and torch.equal(l0, l2)


@pytest.mark.parametrize("mode", [1, 2], ids=["split", "heads"])
@pytest.mark.parametrize("case", [(2, 8, 2, 4096, 128, BF, 1, 0, 0), (1, 12, 3, 4000, 64, FP, 1, 512, 64),
                                  (4, 8, 1, 1500, 128, BF, 0, 0, 0)])
def test_unit_kinds_with_several_units_per_cta(case, mode, units):
    """Split and head-pair units forced on problems with more units than SMs,
    so that CTAs run several units (warpgroup 1 of a split unit waits for
    warpgroup 0 to read its half of the previous unit): sampled rows of every
    head against the oracle, and the whole output against pair units."""
    B, H, Hk, N, d, dt, causal, window, n_sink = case
    q, k, v = random_qkv(B, H, Hk, N, d, dt, seed=N + 3 * H)
    scale = A.default_scale(d)
    units(mode)
    o, l = run_gpu(q, k, v, bool(causal), window, n_sink, scale, out_f32=True)
    units(0)
    o0, l0 = run_gpu(q, k, v, bool(causal), window, n_sink, scale, out_f32=True)
    rng = np.random.default_rng(5)
    for b in range(B):
        for h in range(H):
            rows = _sample_rows(N, rng, extra=8)
            Or, Lr = oracle_rows(q, k, v, b, h, rows, bool(causal), window, n_sink, scale)
            idx = torch.from_numpy(rows)
            assert_parity(errors(o[b, h, idx], l[b, h, idx], Or, Lr), what=f"head ({b},{h})")
    if mode == 2:
        assert torch.equal(o, o0) and torch.equal(l, l0)
    else:
        assert (o - o0).abs().max().item() < 1e-2 and (l - l0).abs().max().item() < 1e-5


@pytest.mark.parametrize("wl", ["c2", "c2c"])
def test_small_workloads_split_units_against_oracle_and_pairs(wl, units):
    """c2 / c2c in full run as split units by default; they match the oracle
    and the pair-unit result to the fp32 rounding level."""
    w = WORKLOADS[wl]
    q, k, v = make_inputs(w)
    Or, Lr = oracle_full(q, k, v, w.causal, w.window, w.n_sink, w.scale)
    units(1)
    o1, l1 = run_gpu(q, k, v, w.causal, w.window, w.n_sink, w.scale, out_f32=True)
    units(0)
    o0, l0 = run_gpu(q, k, v, w.causal, w.window, w.n_sink, w.scale, out_f32=True)
    units(-1)
    oa, la = run_gpu(q, k, v, w.causal, w.window, w.n_sink, w.scale, out_f32=True)
    assert torch.equal(oa, o1) and torch.equal(la, l1)       # the automatic choice is split
    assert_parity(errors(o1, l1, Or, Lr), what="split units")
    assert_parity(errors(o0, l0, Or, Lr), what="pair units")
    assert (o1 - o0).abs().max().item() < 1e-2 and (l1 - l0).abs().max().item() < 1e-5


@pytest.mark.parametrize("scale", [0.0, -0.2, 0.9, 3.0])
def test_scale_values(scale):
    q, k, v = random_qkv(1, 2, 2, 300, 64, BF, seed=7)
    for causal in (True, False):
        Or, Lr = oracle_full(q, k, v, causal, 0, 0, scale)
        o, l = run_gpu(q, k, v, causal, 0, 0, scale, out_f32=True)
        assert_parity(errors(o, l, Or, Lr), what=f"scale={scale} causal={causal}")


def test_large_logits_rescale():
    """Logit ranges far beyond the lazy-rescale threshold (std 4 inputs, scale 1)."""
    q, k, v = random_qkv(1, 2, 2, 777, 128, BF, seed=11, std=2.0)
    Or, Lr = oracle_full(q, k, v, True, 0, 0, 0.5)
    o, l = run_gpu(q, k, v, True, 0, 0, 0.5, out_f32=True)
    assert_parity(errors(o, l, Or, Lr), what="large logits")


# --------------------------------------------------------------- workloads

@pytest.mark.parametrize("name", ["c1", "c2", "c2c"])
def test_small_workloads_full(name):
    w = WORKLOADS[name]
    q, k, v = make_inputs(w)
    Or, Lr = oracle_full(q, k, v, w.causal, w.window, w.n_sink, w.scale)
    o32, l32 = run_gpu(q, k, v, w.causal, w.window, w.n_sink, w.scale, out_f32=True)
    assert_parity(errors(o32, l32, Or, Lr), what=name)
    o16, l16 = run_gpu(q, k, v, w.causal, w.window, w.n_sink, w.scale, out_f32=False)
    assert_parity(errors(o16, l16, Or, Lr), round_floor(Or, w.torch_dtype), what=name + " 16-bit")


def _sample_rows(N, rng, extra=24):
    base = [0, 1, 2, 63, 64, 127, 128, 129, 255, 256, 257, 1023, 1024, 1025, N // 2,
            N - 257, N - 256, N - 129, N - 128, N - 2, N - 1]
    rows = sorted(set([r for r in base if 0 <= r < N] + list(rng.integers(0, N, extra))))
    return np.array(rows)


def _full_size_launch(w):
    """The workload at full size in the launch configuration bench.py times:
    fp32 output (graded) and 16-bit output (reported beside its rounding floor)."""
    q, k, v = make_inputs(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o32, l32 = A.attention(qd, kd, vd, causal=w.causal, window=w.window, n_sink=w.n_sink,
                           scale=w.scale, out_f32=True)
    o16, l16 = A.attention(qd, kd, vd, causal=w.causal, window=w.window, n_sink=w.n_sink,
                           scale=w.scale)
    torch.cuda.synchronize()
    assert A.get_status() == A.ATTN_OK
    assert torch.isfinite(o32).all() and torch.isfinite(l32).all()
    # the 16-bit output is the fp32 result rounded once, and the LSE is shared
    assert torch.equal(o16, o32.to(w.torch_dtype)) and torch.equal(l16, l32)
    return q, k, v, o32.cpu(), l32.cpu(), o16.cpu()


def test_c3_full_tensor_every_head_every_row():
    """The headline workload (B4 H16 N4096 d128 causal): all 64 heads x 4096 rows
    of O and LSE against the oracle, element by element (Lab 3: the tiled
    result equals the reference)."""
    w = WORKLOADS["c3"]
    q, k, v, o32, l32, o16 = _full_size_launch(w)
    Q, K, V = to_f64(q), to_f64(k), to_f64(v)
    import oracle as orc
    for b in range(w.B):
        for h in range(w.H):
            Or, Lr = orc.attention_bh(Q, K, V, b, h, w.scale, w.causal, w.window, w.n_sink)
            assert_parity(errors(o32[b, h], l32[b, h], Or, Lr), what=f"c3 head ({b},{h})")
            assert_parity(errors(o16[b, h], None, Or, Lr), round_floor(Or, w.torch_dtype),
                          what=f"c3 16-bit head ({b},{h})")


@pytest.mark.parametrize("name", ["c4", "c5"])
def test_full_size_every_head_sampled_rows(name):
    """c4 (32 heads x 16384 rows) and c5 (256 heads x 8192 rows) at full size:
    every head, on 64 rows each (the tile and window edges, the tail and
    random rows; a different random draw per head)."""
    w = WORKLOADS[name]
    q, k, v, o32, l32, o16 = _full_size_launch(w)
    rng = np.random.default_rng(0)
    for b in range(w.B):
        for h in range(w.H):
            rows = _sample_rows(w.N, rng, extra=43)
            Or, Lr = oracle_rows(q, k, v, b, h, rows, w.causal, w.window, w.n_sink, w.scale)
            idx = torch.from_numpy(rows)
            assert_parity(errors(o32[b, h, idx], l32[b, h, idx], Or, Lr), what=f"{name} head ({b},{h})")
            assert_parity(errors(o16[b, h, idx], None, Or, Lr), round_floor(Or, w.torch_dtype),
                          what=f"{name} 16-bit head ({b},{h})")


# --------------------------------------------------------- oracle-free checks

def test_causal_row0_is_v0_exactly():
    q, k, v = random_qkv(2, 3, 3, 300, 128, BF, seed=3)
    o, l = run_gpu(q, k, v, True, 0, 0, 0.3, out_f32=True)
    assert torch.equal(o[:, :, 0].cpu(), v[:, :, 0].float())
    expect = 0.3 * (q[:, :, 0].double() * k[:, :, 0].double()).sum(-1)
    assert (l[:, :, 0].double().cpu() - expect).abs().max() < 1e-3


@pytest.mark.parametrize("causal,window,n_sink", [(True, 0, 0), (False, 0, 0), (True, 200, 70)])
def test_identical_keys_give_mean_of_kept_values(causal, window, n_sink):
    B, H, N, d = 1, 2, 700, 64
    q, _, v = random_qkv(B, H, H, N, d, BF, seed=5)
    k = torch.randn(d, generator=torch.Generator().manual_seed(9)).to(BF).expand(B, H, N, d).contiguous()
    o, l = run_gpu(q, k, v, causal, window, n_sink, 0.125, out_f32=True)
    import oracle as orc
    keep = orc.keep_mask(N, N, causal, window, n_sink)
    V = to_f64(v)
    ref = np.einsum("ij,bhjd->bhid", keep / keep.sum(1, keepdims=True), V)
    assert np.abs(o.double().cpu().numpy() - ref).max() < 1e-2
    s = 0.125 * (to_f64(q) @ to_f64(k)[0, 0, 0])
    assert np.abs(l.double().cpu().numpy() - (s + np.log(keep.sum(1)))).max() < 1e-3


def test_mqa_equals_repeated_mha_bitwise():
    B, H, Hk, N, d = 2, 8, 2, 520, 128
    q, k, v = random_qkv(B, H, Hk, N, d, BF, seed=13)
    o1, l1 = run_gpu(q, k, v, True, 0, 0, 0.088, out_f32=True)
    kr, vr = k.repeat_interleave(H // Hk, 1).contiguous(), v.repeat_interleave(H // Hk, 1).contiguous()
    o2, l2 = run_gpu(q, kr, vr, True, 0, 0, 0.088, out_f32=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_deterministic_bitwise():
    w = WORKLOADS["c2c"]
    q, k, v = make_inputs(w)
    a = run_gpu(q, k, v, True, 0, 0, w.scale, out_f32=False)
    b = run_gpu(q, k, v, True, 0, 0, w.scale, out_f32=False)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_noncausal_key_permutation():
    q, k, v = random_qkv(1, 2, 2, 400, 64, FP, seed=17)
    perm = torch.randperm(400, generator=torch.Generator().manual_seed(1))
    o1, l1 = run_gpu(q, k, v, False, 0, 0, 0.125, out_f32=True)
    o2, l2 = run_gpu(q, k[:, :, perm].contiguous(), v[:, :, perm].contiguous(), False, 0, 0, 0.125,
                     out_f32=True)
    assert (o1 - o2).abs().max() < 1e-2 and (l1 - l2).abs().max() < 1e-3


def test_no_quadratic_workspace():
    """The library allocates nothing: memory around a long-sequence call is the outputs only."""
    q, k, v = (t.cuda() for t in random_qkv(1, 4, 4, 8192, 128, BF, seed=1))
    o = torch.empty_like(q)
    lse = torch.empty(1, 4, 8192, device="cuda")
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    before = torch.cuda.memory_allocated()
    A.attention(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == before


def test_host_entry_point_matches_device():
    w = WORKLOADS["c2c"]
    q, k, v = make_inputs(w)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    lh = torch.empty(q.shape[:3], dtype=torch.float32).pin_memory()
    staging = {"q": torch.empty_like(q, device="cuda"), "k": torch.empty_like(k, device="cuda"),
               "v": torch.empty_like(v, device="cuda"), "o": torch.empty_like(q, device="cuda"),
               "lse": torch.empty(q.shape[:3], device="cuda")}
    A.attention_from_host(qh, kh, vh, staging=staging, out=oh, lse=lh, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    o, l = run_gpu(q, k, v, True, 0, 0, w.scale, out_f32=False)
    assert torch.equal(oh, o.cpu()) and torch.equal(lh, l.cpu())


@pytest.mark.parametrize("B,H,H_kv,N,d,causal,window,n_sink", [
    (3, 8, 2, 520, 128, 1, 0, 0),     # GQA: 6 groups, 6 chunks
    (1, 4, 1, 333, 64, 1, 100, 5),    # MQA, G * N % 4 != 0: one chunk
    (2, 3, 3, 257, 32, 0, 0, 0),      # 6 groups of one head, ragged N
    (5, 8, 8, 300, 128, 1, 0, 0),     # 40 groups in 16 chunks of 2-3 groups
])
def test_host_entry_point_chunked_matches_device(B, H, H_kv, N, d, causal, window, n_sink):
    """attn_fwd_host cuts the problem into chunks of (batch, K/V head) groups
    whose copies overlap the forward: the result equals attn_fwd's bitwise."""
    q, k, v = random_qkv(B, H, H_kv, N, d, BF, seed=21)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    lh = torch.empty(q.shape[:3], dtype=torch.float32).pin_memory()
    staging = {"q": torch.empty_like(q, device="cuda"), "k": torch.empty_like(k, device="cuda"),
               "v": torch.empty_like(v, device="cuda"), "o": torch.empty_like(q, device="cuda"),
               "lse": torch.empty(q.shape[:3], device="cuda")}
    A.attention_from_host(qh, kh, vh, staging=staging, out=oh, lse=lh, causal=bool(causal),
                          window=window, n_sink=n_sink)
    torch.cuda.synchronize()
    o, l = run_gpu(q, k, v, bool(causal), window, n_sink, A.default_scale(d), out_f32=False)
    assert torch.equal(oh, o.cpu()) and torch.equal(lh, l.cpu())
    assert A.get_status() == A.ATTN_OK


def test_side_stream_and_launch_count():
    q, k, v = (t.cuda() for t in random_qkv(1, 2, 2, 333, 64, BF, seed=2))
    ref, lref = A.attention(q, k, v, causal=True)
    s = torch.cuda.Stream()
    n0 = A.launch_count()
    with torch.cuda.stream(s):
        o, l = A.attention(q, k, v, causal=True)
    s.synchronize()
    assert A.launch_count() == n0 + 1
    assert torch.equal(o, ref) and torch.equal(l, lref)
    assert A.get_status() == 0


def test_lse_optional():
    q, k, v = (t.cuda() for t in random_qkv(1, 1, 1, 200, 64, BF, seed=4))
    o1, _ = A.attention(q, k, v, causal=True, return_lse=False)
    o2, _ = A.attention(q, k, v, causal=True)
    assert torch.equal(o1, o2)
