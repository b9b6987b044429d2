"""CUDA path vs the fp64 oracle, through the C ABI (ctypes binding).

Small cases span several score chunks, ragged tails, every query-tile width
of the tensor-core scorer (Q*G = 4, 16, 32, 64) and the CUDA-core scorer
(fp32, and bf16 with Q*G > 64); edge cases cover k > visible keys, k = 1,
k = visible keys, one-key sequences, exact ties, the largest k, NaN-poisoned
cache rows past the sequence end, and an out-of-range sequence length.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_block, check_token, to_device

import exact_top_sparse_score_b200 as tka

pytestmark = pytest.mark.gpu


def _seed(case):
    return zlib.crc32(repr(case).encode()) % 100000


def run_token(w, k, scale=0.0):
    q, kc, vc, lens = to_device(w)
    out, idx, tail = tka.topk_attn_decode(q, kc, vc, lens, k, scale=scale)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    return out, idx, tail


TOKEN_CASES = [
    # dtype, B, Q, Hq, Hkv, L_max, seq_lens, k
    ("bf16", 2, 1, 8, 2, 1000, [1000, 517], 100),      # ragged tail, Q*G = 4
    ("bf16", 2, 1, 32, 8, 4133, [4133, 3001], 512),    # Llama-3-8B head layout
    ("bf16", 2, 2, 16, 2, 600, [600, 301], 40),        # Q*G = 16
    ("bf16", 1, 4, 16, 2, 1500, None, 64),             # Q*G = 32
    ("bf16", 2, 16, 32, 8, 2500, [2500, 2000], 300),   # Q*G = 64, causal chunk
    ("bf16", 1, 8, 32, 2, 900, None, 50),              # Q*G = 128: CUDA-core scorer
    ("f32", 2, 3, 8, 4, 777, [777, 200], 50),          # fp32, causal
    ("f32", 1, 1, 4, 4, 3000, None, 1),                # k = 1
    ("bf16", 2, 1, 8, 2, 300, [300, 50], 100),         # k > visible keys for b=1
    ("bf16", 2, 1, 4, 1, 64, [1, 64], 8),              # one-key sequence
    ("bf16", 1, 1, 8, 2, 256, None, 256),              # k = visible keys
    ("bf16", 1, 1, 8, 8, 10000, None, 8192),           # largest k
    ("bf16", 1, 3, 4, 4, 700, None, 30),               # G = 1 (multi-head), Q = 3
    ("bf16", 5, 1, 32, 8, 20000, [20000, 19001, 16384, 17777, 20000], 1024),  # more rows than SMs: 512-thread
                                                       # select, sampled band, segments streamed in two batches
    ("bf16", 1, 1, 8, 2, 40000, None, 2048),           # 1024-thread select, segments streamed in two batches
]


@pytest.mark.parametrize("case", TOKEN_CASES, ids=lambda c: "-".join(map(str, c[:6])) + f"-k{c[7]}")
def test_token_parity_small(case, cuda_device):
    dtype, B, Q, Hq, Hkv, L, lens, k = case
    w = workloads.make_workload(B, Q, Hq, Hkv, L, dtype=dtype, seq_lens=lens, k_mean_std=0.5, seed=_seed(case))
    out, idx, tail = run_token(w, k)
    assert torch.isfinite(out).all() and torch.isfinite(tail).all()
    check_token(w, k, out, idx, tail, oracle.topk_attn(w, k))


def test_token_explicit_scale(cuda_device):
    w = workloads.make_workload(2, 1, 8, 2, 800, dtype="bf16", seed=3)
    out, idx, tail = run_token(w, 64, scale=0.3)
    check_token(w, 64, out, idx, tail, oracle.topk_attn(w, 64, scale=0.3), scale=0.3)


def test_token_exact_ties_go_to_lower_position(cuda_device):
    # many duplicated key rows: exactly equal scores on both sides
    w = workloads.make_workload(1, 1, 8, 2, 2048, dtype="bf16", seed=4)
    src = torch.arange(2048) % 97
    w.k_cache[:] = w.k_cache[:, :, src]
    out, idx, tail = run_token(w, 200)
    ref = oracle.topk_attn(w, 200)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    check_token(w, 200, out, idx, tail, ref)


def test_planted_heavy_tail(cuda_device):
    w = workloads.make_workload(2, 1, 32, 8, 5000, dtype="bf16", seq_len_range=(2500, 5000), plant_count=16,
                                seed=5)
    out, idx, tail = run_token(w, 256)
    check_token(w, 256, out, idx, tail, oracle.topk_attn(w, 256))


@pytest.mark.parametrize("rise", [1.5, 6.0, 30.0])
def test_scores_rising_with_position(rise, cuda_device):
    # a recency-like pattern: keys drift along their group's mean query
    # direction with position, so the kept positions crowd into the last
    # segments of each row (more per warp than its ordered list holds)
    B, Hq, Hkv, L = 5, 32, 8, 20000
    w = workloads.make_workload(B, 1, Hq, Hkv, L, dtype="bf16", seed=7)
    u = w.q.float().reshape(B, Hkv, Hq // Hkv, 128).mean(2)
    u = u / u.norm(dim=-1, keepdim=True)
    ramp = torch.linspace(0.0, rise, L)
    w.k_cache[:] = (w.k_cache.float() + ramp[None, None, :, None] * u[:, :, None, :]).to(w.k_cache.dtype)
    out, idx, tail = run_token(w, 1024)
    check_token(w, 1024, out, idx, tail, oracle.topk_attn(w, 1024))


@pytest.mark.parametrize("B", [1, 5])
def test_all_scores_equal(B, cuda_device):
    # one key row repeated along every sequence: every score of a row ties, the
    # sampled band holds the whole row (more candidates than the per-warp lists
    # take), and the exact multi-pass route keeps the lowest k positions; B = 5
    # gives more rows than SMs (512-thread rows), B = 1 the 1024-thread rows
    L, k = 20000, 1024
    w = workloads.make_workload(B, 1, 32, 8, L, dtype="bf16", seed=8)
    w.k_cache[:] = w.k_cache[:, :, :1].expand_as(w.k_cache)
    out, idx, tail = run_token(w, k)
    ref = oracle.topk_attn(w, k)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    assert (idx.cpu()[..., :] == torch.arange(k, dtype=torch.int32)).all()
    check_token(w, k, out, idx, tail, ref)


@pytest.mark.parametrize("k", [100, 2047])
def test_short_row_all_scores_equal(k, cuda_device):
    # a row its select step samples whole (2048 keys) with every score equal:
    # the k-th score's bin holds more than 32 scores, so the row leaves the
    # register-resident route for the lists and the exact multi-pass route
    w = workloads.make_workload(1, 1, 8, 2, 2048, dtype="bf16", seed=21)
    w.k_cache[:] = w.k_cache[:, :, :1].expand_as(w.k_cache)
    out, idx, tail = run_token(w, k)
    ref = oracle.topk_attn(w, k)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    check_token(w, k, out, idx, tail, ref)


def test_short_row_ties_inside_the_kth_bin(cuda_device):
    # 40 distinct key rows repeated along 1024 positions: the k-th score's
    # value occurs ~26 times, the register-resident route ranks the bin's
    # scores and keeps the lowest-positioned ties
    L = 1024
    w = workloads.make_workload(2, 1, 8, 2, L, dtype="bf16", seed=22)
    src = torch.arange(L) % 40
    w.k_cache[:] = w.k_cache[:, :, src]
    for k in (30, 333):
        out, idx, tail = run_token(w, k)
        ref = oracle.topk_attn(w, k)
        assert np.array_equal(idx.cpu().numpy(), ref["idx"])
        check_token(w, k, out, idx, tail, ref)


def test_repeat_calls_are_bitwise_identical(cuda_device):
    w = workloads.make_workload(2, 1, 32, 8, 3000, dtype="bf16", seed=6)
    q, kc, vc, lens = to_device(w)
    ws = torch.empty(tka.topk_attn_workspace_size(tka._binding.make_shape(q, kc), 300), dtype=torch.uint8,
                     device="cuda")
    a = tka.topk_attn_decode(q, kc, vc, lens, 300, workspace=ws)
    a = [t.clone() for t in a]
    b = tka.topk_attn_decode(q, kc, vc, lens, 300, workspace=ws)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_partial_stage_events(cuda_device):
    # only the after-select event recorded (the idx read-back overlapping the
    # gather): same results as the plain call, and idx is final at the event
    w = workloads.make_workload(4, 1, 32, 8, 6000, dtype="bf16", seed=9)
    q, kc, vc, lens = to_device(w)
    a = [t.clone() for t in tka.topk_attn_decode(q, kc, vc, lens, 512)]
    ev = torch.cuda.Event()
    ev.record()
    side = torch.cuda.Stream()
    out, idx, tail = tka.topk_attn_decode(q, kc, vc, lens, 512, stage_events=[None, None, ev, None])
    side.wait_event(ev)
    with torch.cuda.stream(side):
        idx_copy = idx.clone()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    for x, y in zip(a, (out, idx, tail)):
        assert torch.equal(x, y)
    assert torch.equal(idx_copy, a[1])


def test_non_default_stream(cuda_device):
    w = workloads.make_workload(1, 1, 8, 2, 1200, dtype="bf16", seed=7)
    q, kc, vc, lens = to_device(w)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        out, idx, tail = tka.topk_attn_decode(q, kc, vc, lens, 100)
    st.synchronize()
    check_token(w, 100, out, idx, tail, oracle.topk_attn(w, 100))


def test_bad_seq_len_raises_status_and_skips_sequence(cuda_device):
    w = workloads.make_workload(2, 1, 8, 2, 500, dtype="bf16", seed=8)
    q, kc, vc, lens = to_device(w)
    bad = lens.clone()
    bad[1] = 501  # > L_max
    out = torch.full((2, 1, 8, 128), 7.0, dtype=torch.float32, device="cuda")
    idx = torch.full((2, 1, 8, 40), -7, dtype=torch.int32, device="cuda")
    tail = torch.full((2, 1, 8), 7.0, dtype=torch.float32, device="cuda")
    tka.topk_attn_device_status()
    tka.topk_attn_decode(q, kc, vc, bad, 40, out=out, idx=idx, tail_mass=tail)
    assert tka.topk_attn_device_status() & tka.DEV_BAD_SEQ_LEN
    assert tka.topk_attn_device_status() == 0  # cleared by reading
    assert (out[1] == 7.0).all() and (idx[1] == -7).all() and (tail[1] == 7.0).all()
    ref = oracle.topk_attn(w, 40)
    w1 = workloads.make_workload(1, 1, 8, 2, 500, dtype="bf16", seed=8)
    check_token(w1, 40, out[:1], idx[:1], tail[:1], {k: v[:1] for k, v in ref.items()})


BLOCK_CASES = [
    # dtype, B, Hq, Hkv, L_max, seq_lens, block_size, top_blocks
    ("bf16", 2, 8, 2, 4096, [4096, 3000], 64, 16),
    ("bf16", 2, 32, 8, 2000, [2000, 1111], 32, 5),
    ("f32", 2, 8, 4, 1024, [1024, 70], 16, 7),
    ("bf16", 1, 4, 1, 640, None, 128, 2),
    ("bf16", 2, 8, 2, 700, [700, 64], 64, 30),          # top_blocks >= competing blocks: dense
    ("bf16", 1, 8, 2, 256, [1], 64, 4),                 # one-key sequence
    ("bf16", 2, 8, 2, 3000, [3000, 2500], 32, 0),       # only the current block
    ("bf16", 1, 8, 2, 65536, [65521], 16, 255),         # 4095 blocks, the largest top_blocks
    ("bf16", 2, 8, 2, 32768, [32768, 20000], 16, 40),   # 2048 blocks
    ("bf16", 1, 64, 2, 131072, [131000], 16, 8),        # G = 32 x 8192 blocks: the kv-head's scores exceed the
                                                        # cluster's shared memory -> two launches via the workspace
]


@pytest.mark.parametrize("case", BLOCK_CASES, ids=lambda c: "-".join(map(str, c)))
def test_block_parity_small(case, cuda_device):
    dtype, B, Hq, Hkv, L, lens, bs, top = case
    w = workloads.make_workload(B, 1, Hq, Hkv, L, dtype=dtype, seq_lens=lens, seed=_seed(case))
    q, kc, vc, lens_d = to_device(w)
    bk = tka.topk_block_pool_keys(kc, lens_d, bs)
    ref_bk = oracle.block_pool(w, bs)
    np.testing.assert_allclose(bk.cpu().double().numpy(), ref_bk, atol=2e-5, rtol=1e-5)
    out, bidx = tka.topk_block_attn_decode(q, kc, vc, bk, lens_d, bs, top)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    check_block(w, bs, top, out, bidx, oracle.block_attn(w, bs, top))


def test_block_parity_exact_ties(cuda_device):
    """Blocks repeat with period 4, so every block score is shared by about a
    quarter of the blocks and the top_blocks boundary falls inside a run of
    exactly equal scores: the kept blocks must be the lowest-numbered ones."""
    bs, top, L = 32, 10, 4096
    w = workloads.make_workload(1, 1, 8, 2, L, dtype="bf16", seed=77)
    nblk = L // bs
    for j in range(4, nblk - 1):
        w.k_cache[:, :, j * bs:(j + 1) * bs] = w.k_cache[:, :, (j % 4) * bs:(j % 4 + 1) * bs]
    q, kc, vc, lens_d = to_device(w)
    bk = tka.topk_block_pool_keys(kc, lens_d, bs)
    out, bidx = tka.topk_block_attn_decode(q, kc, vc, bk, lens_d, bs, top)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    ref = oracle.block_attn(w, bs, top)
    # equal block keys give bit-equal scores on both sides, so the lists agree exactly
    assert np.array_equal(bidx.cpu().numpy(), ref["block_idx"])
    assert check_block(w, bs, top, out, bidx, ref) == 0


def test_block_repeat_calls_are_bitwise_identical(cuda_device):
    """Rows split between CTAs are merged in piece order, not arrival order."""
    w = workloads.make_workload(4, 1, 32, 8, 8192, dtype="bf16", seed=79)
    q, kc, vc, lens = to_device(w)
    bk = tka.topk_block_pool_keys(kc, lens, 64)
    a = [t.clone() for t in tka.topk_block_attn_decode(q, kc, vc, bk, lens, 64, 20)]
    b = tka.topk_block_attn_decode(q, kc, vc, bk, lens, 64, 20)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_block_bad_seq_len_raises_status_and_skips_sequence(cuda_device):
    w = workloads.make_workload(2, 1, 8, 2, 2048, dtype="bf16", seed=80)
    q, kc, vc, lens = to_device(w)
    bk = tka.topk_block_pool_keys(kc, lens, 32)
    bad = lens.clone()
    bad[1] = 0
    out = torch.full((2, 1, 8, 128), 7.0, dtype=torch.float32, device="cuda")
    tka.topk_attn_device_status()
    tka.topk_block_attn_decode(q, kc, vc, bk, bad, 32, 6, out=out)
    assert tka.topk_attn_device_status() & tka.DEV_BAD_SEQ_LEN
    assert tka.topk_attn_device_status() == 0
    assert (out[1] == 7.0).all()
    w0 = workloads.make_workload(1, 1, 8, 2, 2048, dtype="bf16", seed=80)
    ref = oracle.block_attn(w0, 32, 6)
    _, bidx0 = tka.topk_block_attn_decode(q[:1], kc[:1], vc[:1], bk[:1], lens[:1], 32, 6)
    check_block(w0, 32, 6, out[:1], bidx0, ref)


def test_one_launch_path_matches_three_launches(cuda_device):
    """Small problems take one cooperative launch (score, grid barrier, select
    and attention per row); the staged call records events between its steps,
    so it takes the three-kernel path.  With an fp32 cache both score on the
    CUDA cores in the same order: identical kept sets, outputs to rounding."""
    w = workloads.make_workload(2, 2, 8, 4, 4096, dtype="f32", seq_lens=[4096, 1777], seed=77)
    q, kc, vc, lens = to_device(w)
    k = 96
    out1, idx1, tail1 = tka.topk_attn_decode(q, kc, vc, lens, k)
    ev = [torch.cuda.Event(), None, None, None]
    out3, idx3, tail3 = tka.topk_attn_decode(q, kc, vc, lens, k, stage_events=ev)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    assert torch.equal(idx1, idx3)
    assert (out1 - out3).abs().max().item() <= 1e-5 and (tail1 - tail3).abs().max().item() <= 1e-6
    check_token(w, k, out1, idx1, tail1, oracle.topk_attn(w, k))
