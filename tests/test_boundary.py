"""C-ABI boundary on the CPU: the library loads, exports what include/attn.h
declares, rejects malformed calls before touching CUDA, and its host-only
schedule helpers agree with the oracle's mask."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import exact_tiled_attention_44_b200 as A
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")

# Fake, 16-byte aligned, never dereferenced addresses (validation runs first).
P_Q, P_K, P_V, P_O, P_L = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = A.load_library()
    decl = declared_functions()
    assert decl == sorted(A.EXPORTED_SYMBOLS)
    for name in decl:
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_error_strings():
    for code in (A.ATTN_OK, A.ATTN_ERR_INVALID_ARG, A.ATTN_ERR_UNSUPPORTED, A.ATTN_ERR_MISALIGNED,
                 A.ATTN_ERR_CUDA, A.ATTN_ERR_DEVICE_TIMEOUT, 12345):
        assert isinstance(A.error_string(code), str) and A.error_string(code)


def call(q=P_Q, k=P_K, v=P_V, o=P_O, lse=P_L, B=1, H=2, H_kv=2, N=100, d=64, causal=1, window=0,
         n_sink=0, scale=0.125, dtype=A.ATTN_BF16):
    return A.attn_fwd_raw(q, k, v, o, lse, B, H, H_kv, N, d, causal, window, n_sink, scale, dtype,
                          None)


@pytest.mark.parametrize("kw,expect", [
    (dict(B=-1), A.ATTN_ERR_INVALID_ARG),
    (dict(N=-5), A.ATTN_ERR_INVALID_ARG),
    (dict(H_kv=0), A.ATTN_ERR_INVALID_ARG),
    (dict(H=6, H_kv=4), A.ATTN_ERR_INVALID_ARG),
    (dict(d=0), A.ATTN_ERR_INVALID_ARG),
    (dict(d=48), A.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), A.ATTN_ERR_UNSUPPORTED),
    (dict(causal=2), A.ATTN_ERR_INVALID_ARG),
    (dict(window=-1), A.ATTN_ERR_INVALID_ARG),
    (dict(n_sink=-1), A.ATTN_ERR_INVALID_ARG),
    (dict(causal=0, window=8), A.ATTN_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), A.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), A.ATTN_ERR_INVALID_ARG),
    (dict(dtype=2), A.ATTN_ERR_INVALID_ARG),
    (dict(dtype=0x20), A.ATTN_ERR_INVALID_ARG),
    (dict(q=None), A.ATTN_ERR_INVALID_ARG),
    (dict(o=None), A.ATTN_ERR_INVALID_ARG),
    (dict(q=P_Q + 8), A.ATTN_ERR_MISALIGNED),
    (dict(v=P_V + 2), A.ATTN_ERR_MISALIGNED),
    (dict(lse=P_L + 4), A.ATTN_ERR_MISALIGNED),
    (dict(o=P_Q + 64), A.ATTN_ERR_INVALID_ARG),          # o overlaps q
    (dict(o=P_K), A.ATTN_ERR_INVALID_ARG),               # o aliases k
    (dict(lse=P_O + 16), A.ATTN_ERR_INVALID_ARG),        # lse overlaps o
])
def test_invalid_calls_are_rejected_before_launch(kw, expect):
    assert call(**kw) == expect


@pytest.mark.parametrize("kw", [dict(B=0), dict(H=0), dict(N=0),
                                dict(B=0, q=None, k=None, v=None, o=None, lse=None)])
def test_empty_problem_is_a_no_op(kw):
    assert call(**kw) == A.ATTN_OK


def test_binding_refuses_cpu_tensors():
    q = torch.zeros(1, 1, 8, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        A.attention(q, q, q)
    with pytest.raises(TypeError):
        A.attention(q.float(), q.float(), q.float())


@pytest.mark.parametrize("N,causal,window,n_sink", [
    (1, 1, 0, 0), (1, 0, 0, 0), (7, 0, 0, 0), (64, 1, 0, 0), (1000, 1, 0, 0),
    (300, 1, 1, 0), (300, 1, 17, 5), (777, 1, 128, 64), (777, 1, 300, 200), (257, 1, 256, 0),
    (200, 1, 500, 10), (1024, 1, 1024, 64), (1500, 1, 129, 130)])
def test_unmasked_pairs_matches_oracle_enumeration(N, causal, window, n_sink):
    assert A.unmasked_pairs(N, causal, window, n_sink) == oracle.kept_pairs(N, bool(causal), window, n_sink)


def test_unmasked_pairs_workloads():
    assert A.unmasked_pairs(4096, 1) == 4096 * 4097 // 2
    assert A.unmasked_pairs(1024, 0) == 1024 * 1024
    assert A.unmasked_pairs(8192, 1, 1024, 64) == 8321568
    assert A.unmasked_pairs(10, 0, 3, 0) == -1
    assert A.unmasked_pairs(-1, 1) == -1


def _visited_by_mask(N, causal, window, n_sink, blk=128):
    keep = oracle.keep_mask(N, N, bool(causal), window, n_sink)
    nb = (N + blk - 1) // blk
    count = 0
    for qb in range(nb):
        for kb in range(nb):
            if keep[qb * blk:(qb + 1) * blk, kb * blk:(kb + 1) * blk].any():
                count += 1
    return count


@pytest.mark.parametrize("N,causal,window,n_sink", [
    (1, 1, 0, 0), (64, 1, 0, 0), (64, 0, 0, 0), (200, 1, 0, 0), (1000, 0, 0, 0),
    (1000, 1, 0, 0), (1000, 1, 1, 0), (1000, 1, 100, 0), (1000, 1, 300, 64),
    (1300, 1, 129, 200), (1300, 1, 257, 1), (900, 1, 2000, 5)])
def test_visited_blocks_is_exactly_the_blocks_with_kept_pairs(N, causal, window, n_sink):
    """Lab 3, exercise 3: count visited block pairs; none is skipped that holds work."""
    assert A.visited_blocks(N, causal, window, n_sink) == _visited_by_mask(N, causal, window, n_sink)


def test_visited_blocks_workloads():
    assert A.visited_blocks(4096, 1) == 528           # 32 * 33 / 2
    assert A.visited_blocks(1024, 0) == 64
    assert A.visited_blocks(1024, 1) == 36
    assert A.visited_blocks(16384, 1) == 128 * 129 // 2
    assert A.visited_blocks(64, 1) == 1


# ------------------------------------------------------------------ ALiBi entry points


P_S = 0x600000   # fake, aligned slopes address


def call_alibi(slopes=P_S, **kw):
    a = dict(q=P_Q, k=P_K, v=P_V, o=P_O, lse=P_L, B=1, H=2, H_kv=2, N=100, d=64, causal=1,
             window=0, n_sink=0, scale=0.125, dtype=A.ATTN_BF16)
    a.update(kw)
    return A.attn_fwd_alibi_raw(a["q"], a["k"], a["v"], a["o"], a["lse"], slopes, a["B"], a["H"],
                                a["H_kv"], a["N"], a["d"], a["causal"], a["window"], a["n_sink"],
                                a["scale"], a["dtype"], None)


@pytest.mark.parametrize("kw,expect", [
    (dict(slopes=None), A.ATTN_ERR_INVALID_ARG),
    (dict(slopes=P_S + 2), A.ATTN_ERR_MISALIGNED),
    (dict(slopes=P_O + 8), A.ATTN_ERR_INVALID_ARG),      # overlaps o
    (dict(d=48), A.ATTN_ERR_UNSUPPORTED),
    (dict(causal=0, window=8), A.ATTN_ERR_UNSUPPORTED),
    (dict(H=6, H_kv=4), A.ATTN_ERR_INVALID_ARG),
    (dict(q=P_Q + 8), A.ATTN_ERR_MISALIGNED),
])
def test_alibi_invalid_calls_are_rejected_before_launch(kw, expect):
    assert call_alibi(**kw) == expect


def test_alibi_empty_problem_is_a_no_op():
    # nothing to compute: OK before any pointer (slopes included) is looked at
    assert call_alibi(B=0, slopes=None) == A.ATTN_OK
    assert call_alibi(N=0) == A.ATTN_OK


@pytest.mark.parametrize("H", [1, 2, 4, 8, 12, 16, 32, 64])
def test_alibi_slopes_helper_matches_pages_formula(H):
    """attn_alibi_slopes (host) against the oracle's slope sequence, rounded once to fp32."""
    got = A.alibi_slopes(H)
    want = torch.tensor(oracle.alibi_slopes(H), dtype=torch.float64).to(torch.float32)
    assert got.dtype == torch.float32 and torch.equal(got, want)


def test_alibi_slopes_helper_rejects_bad_h():
    lib = A.load_library()
    buf = (ctypes.c_float * 4)()
    assert lib.attn_alibi_slopes(0, buf) == A.ATTN_ERR_INVALID_ARG
    assert lib.attn_alibi_slopes(4, None) == A.ATTN_ERR_INVALID_ARG


def test_withhold_hook_arguments():
    assert A.test_withhold_loads(-1) == A.ATTN_ERR_INVALID_ARG
    assert A.test_withhold_loads(0) == A.ATTN_OK


# -------------------------------------------------------- work-unit kind (host only)

@pytest.mark.parametrize("sizes,kind", [
    ((1, 1, 1, 64, 0, False), 1),          # c1: one tile -> split units
    ((2, 8, 8, 1024, 0, False), 1),        # c2 / c2c: 64 pairs < 148 SMs, 128 tiles -> split
    ((4, 16, 16, 4096, 0, False), 0),      # c3: 1024 pairs -> tile pairs
    ((1, 32, 32, 16384, 0, False), 0),     # c4: MHA -> tile pairs
    ((8, 32, 1, 8192, 1024, False), 2),    # c5: MQA, rows see 1024 keys -> head pairs
    ((4, 32, 4, 16384, 0, False), 0),      # GQA with long causal rows -> tile pairs
    ((4, 32, 8, 4096, 0, False), 2),       # GQA, N = 4096 -> head pairs
    ((4, 32, 8, 4097, 0, False), 0),       # one key past the head-pair limit
    ((4, 16, 16, 4096, 0, True), 0),       # a position bias keeps pairs
    ((2, 8, 8, 1024, 0, True), 0),         # ... even where split units would apply
    ((1, 148, 148, 256, 0, False), 0),     # 148 pairs: no SM idle -> pairs
    ((1, 147, 147, 256, 0, False), 1),     # 147 pairs, 294 tiles <= 296 -> split
    ((1, 100, 100, 384, 0, False), 0),     # 200 pairs >= 148 -> pairs
    ((1, 60, 60, 640, 0, False), 0),       # 60 heads x 3 pairs = 180 >= 148 -> pairs
    ((1, 60, 60, 384, 0, False), 1),       # 60 x 2 = 120 pairs, 180 tiles -> split
])
def test_unit_kind_rule(sizes, kind):
    B, H, Hk, N, window, alibi = sizes
    pairs = B * H * ((N + 255) // 256)
    tiles = B * H * ((N + 127) // 128)
    if alibi:
        expect = 0
    elif pairs < 148 and tiles <= 296:
        expect = 1
    elif H // Hk >= 2 and (window if 0 < window < N else N) <= 4096:
        expect = 2
    else:
        expect = 0
    got = A.fwd_unit_kind(B, H, Hk, N, window, alibi, 148)
    assert got == expect == kind


def test_unit_kind_arguments():
    for bad in [(-1, 1, 1, 64, 0, 0, 148), (1, 0, 1, 64, 0, 0, 148), (1, 4, 3, 64, 0, 0, 148),
                (1, 4, 0, 64, 0, 0, 148), (1, 4, 4, -1, 0, 0, 148), (1, 4, 4, 64, -2, 0, 148),
                (1, 4, 4, 64, 0, 0, -1)]:
        assert A.fwd_unit_kind(*bad) == A.ATTN_ERR_INVALID_ARG
    assert A.fwd_unit_kind(0, 4, 4, 64, 0, False, 148) in (0, 1, 2)   # empty problem: any kind


def test_force_units_hook_arguments():
    for bad in (-2, 3, 7):
        assert A.test_force_units(bad) == A.ATTN_ERR_INVALID_ARG
    for mode in (0, 1, 2, -1):
        assert A.test_force_units(mode) == A.ATTN_OK


def test_count_blocks_hook_arguments():
    assert A.test_count_blocks(None) == A.ATTN_OK
    with pytest.raises(ValueError):
        A.test_count_blocks(torch.zeros(1, dtype=torch.int64))         # not on a GPU


# ------------------------------------------------------------------ decode entry points


# fake, aligned, never dereferenced addresses far enough apart for a cache of several MB
D_Q, D_K, D_V, D_O, D_L, D_W = (i << 28 for i in range(1, 7))


def call_decode(ws=D_W, ws_bytes=1 << 26, **kw):
    a = dict(q=D_Q, k=D_K, v=D_V, o=D_O, lse=D_L, B=1, H=8, H_kv=2, N_q=1, N_kv=4096, d=128,
             causal=1, window=0, n_sink=0, scale=0.088, dtype=A.ATTN_BF16)
    a.update(kw)
    return A.attn_decode_raw(a["q"], a["k"], a["v"], a["o"], a["lse"], ws, ws_bytes, a["B"], a["H"],
                             a["H_kv"], a["N_q"], a["N_kv"], a["d"], a["causal"], a["window"],
                             a["n_sink"], a["scale"], a["dtype"], None)


@pytest.mark.parametrize("kw,expect", [
    (dict(N_q=5, N_kv=4), A.ATTN_ERR_INVALID_ARG),
    (dict(d=32), A.ATTN_ERR_UNSUPPORTED),
    (dict(H=64, H_kv=1, N_q=2), A.ATTN_ERR_UNSUPPORTED),      # 128 rows per K/V head
    (dict(causal=0, window=8), A.ATTN_ERR_UNSUPPORTED),
    (dict(H=6, H_kv=4), A.ATTN_ERR_INVALID_ARG),
    (dict(ws=None), A.ATTN_ERR_INVALID_ARG),                  # the cache is split: workspace needed
    (dict(ws_bytes=16), A.ATTN_ERR_INVALID_ARG),
    (dict(ws=D_W + 16), A.ATTN_ERR_MISALIGNED),
    (dict(q=D_Q + 4), A.ATTN_ERR_MISALIGNED),
    (dict(o=D_K + 64), A.ATTN_ERR_INVALID_ARG),               # o overlaps the cache
    (dict(ws=D_O), A.ATTN_ERR_INVALID_ARG),                   # workspace overlaps o
    (dict(ws_bytes=-1), A.ATTN_ERR_INVALID_ARG),
])
def test_decode_invalid_calls_are_rejected_before_launch(kw, expect):
    assert call_decode(**kw) == expect


def test_decode_empty_problem_is_a_no_op():
    assert call_decode(B=0, ws=None, ws_bytes=0) == A.ATTN_OK
    assert call_decode(N_q=0, ws=None, ws_bytes=0) == A.ATTN_OK


def test_decode_workspace_size():
    # The kept tiles of all (batch, K/V head) groups are cut into at most 148
    # ranges, so a group spans at most ceil(148 / groups) + 1 of them; each
    # part keeps an LSE and a D-wide fp32 row per query row of the group.
    for B, H, H_kv, N_q, N_kv, d in ((4, 8, 2, 1, 200, 128), (1, 8, 2, 1, 4096, 128),
                                     (8, 32, 8, 1, 8192, 128), (1, 64, 1, 1, 20000, 64),
                                     (300, 4, 1, 2, 100, 64)):
        groups, rows = B * H_kv, (H // H_kv) * N_q
        parts = -(-148 // groups) + 1
        lse = -(-groups * parts * rows * 4 // 256) * 256
        assert A.decode_workspace_bytes(B, H, H_kv, N_q, N_kv, d) == lse + groups * parts * rows * d * 4
    # it does not depend on the cache length
    assert A.decode_workspace_bytes(1, 8, 2, 1, 4096, 128) == A.decode_workspace_bytes(1, 8, 2, 1, 64, 128)
    assert A.decode_workspace_bytes(1, 8, 2, 5, 4, 128) == -1
    assert A.decode_workspace_bytes(0, 8, 2, 1, 4096, 128) == 0


# ------------------------------------------------------------------ backward entry point


# fake, aligned, never dereferenced addresses (B=1, H=4, N=256, d=64 tensors are 128 KB)
B_Q, B_K, B_V, B_O, B_DO, B_L, B_S, B_DQ, B_DK, B_DV, B_W = (i << 24 for i in range(1, 12))


def call_bwd(**kw):
    a = dict(q=B_Q, k=B_K, v=B_V, o=B_O, dout=B_DO, lse=B_L, slopes=None, dq=B_DQ, dk=B_DK,
             dv=B_DV, ws=B_W, ws_bytes=1 << 22, B=1, H=4, H_kv=2, N=256, d=64, causal=1,
             window=0, n_sink=0, scale=0.125, dtype=A.ATTN_BF16)
    a.update(kw)
    return A.attn_bwd_raw(a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["slopes"],
                          a["dq"], a["dk"], a["dv"], a["ws"], a["ws_bytes"], a["B"], a["H"],
                          a["H_kv"], a["N"], a["d"], a["causal"], a["window"], a["n_sink"],
                          a["scale"], a["dtype"], None)


@pytest.mark.parametrize("kw,expect", [
    (dict(o=None), A.ATTN_ERR_INVALID_ARG),
    (dict(dout=None), A.ATTN_ERR_INVALID_ARG),
    (dict(lse=None), A.ATTN_ERR_INVALID_ARG),
    (dict(dk=None), A.ATTN_ERR_INVALID_ARG),
    (dict(ws=None), A.ATTN_ERR_INVALID_ARG),
    (dict(ws_bytes=1024), A.ATTN_ERR_INVALID_ARG),            # smaller than the dQ accumulator
    (dict(ws_bytes=-1), A.ATTN_ERR_INVALID_ARG),
    (dict(ws=B_W + 16), A.ATTN_ERR_MISALIGNED),               # workspace wants 256 bytes
    (dict(dout=B_DO + 8), A.ATTN_ERR_MISALIGNED),
    (dict(lse=B_L + 4), A.ATTN_ERR_MISALIGNED),
    (dict(slopes=B_S + 2), A.ATTN_ERR_MISALIGNED),
    (dict(d=48), A.ATTN_ERR_UNSUPPORTED),
    (dict(causal=0, window=8), A.ATTN_ERR_UNSUPPORTED),
    (dict(H=6, H_kv=4), A.ATTN_ERR_INVALID_ARG),
    (dict(dq=B_Q + 256), A.ATTN_ERR_INVALID_ARG),             # dQ overlaps q
    (dict(dk=B_DV), A.ATTN_ERR_INVALID_ARG),                  # dK overlaps dV
    (dict(dv=B_L), A.ATTN_ERR_INVALID_ARG),                   # dV overlaps lse
    (dict(ws=B_DQ), A.ATTN_ERR_INVALID_ARG),                  # workspace overlaps dQ
    (dict(dq=B_S, slopes=B_S), A.ATTN_ERR_INVALID_ARG),       # dQ overlaps the slopes
    (dict(scale=float("nan")), A.ATTN_ERR_INVALID_ARG),
])
def test_bwd_invalid_calls_are_rejected_before_launch(kw, expect):
    assert call_bwd(**kw) == expect


def test_bwd_inputs_may_alias_each_other():
    """Read-only inputs may share memory (e.g. o passed as dout); validation
    then goes on to the device query, which fails here without a GPU."""
    rc = call_bwd(dout=B_O)
    assert rc not in (A.ATTN_ERR_INVALID_ARG, A.ATTN_ERR_MISALIGNED, A.ATTN_ERR_UNSUPPORTED)


def test_bwd_empty_problem_is_a_no_op():
    assert call_bwd(B=0, ws=None, ws_bytes=0) == A.ATTN_OK
    assert call_bwd(N=0, ws=None, ws_bytes=0) == A.ATTN_OK


def test_bwd_workspace_size():
    rows = 2 * 8 * 300
    # D per row (rounded to 256 bytes), then the fp32 dQ accumulator
    want = -(-rows * 4 // 256) * 256 + rows * 64 * 4
    assert A.bwd_workspace_bytes(2, 8, 300, 64, A.ATTN_BF16) == want
    # fp32 gradients: dQ is accumulated in place, only D remains
    assert A.bwd_workspace_bytes(2, 8, 300, 64, A.ATTN_BF16 | A.ATTN_OUT_F32) == -(-rows * 4 // 256) * 256
    assert A.bwd_workspace_bytes(0, 8, 300, 64, A.ATTN_BF16) == 0
    assert A.bwd_workspace_bytes(-1, 8, 300, 64, A.ATTN_BF16) == -1
    assert A.bwd_workspace_bytes(1, 8, 300, 64, 0x100) == -1
