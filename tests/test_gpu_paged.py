"""Paged KV cache (block tables) on the GPU.

The same workload is laid out as a pool of pages in a random physical order
(with unused pages and -1 table entries past each sequence's end); the paged
call must give exactly what the contiguous call gives on the original cache,
and both what the fp64 oracle gives.  Entries past a sequence's last page
are -1 and pages nobody references hold NaN, so any read of them would show.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_token, to_device

import exact_top_sparse_score_b200 as tka


def paged_copy(w, page_size, extra_pages=5, seed=0):
    """(k_pages, v_pages, block_table) holding w's cache in shuffled pages."""
    rng = np.random.default_rng(seed)
    max_pages = -(-w.L_max // page_size)
    used = [-(-int(w.seq_lens[b]) // page_size) for b in range(w.B)]
    num_pages = sum(used) + extra_pages
    phys = rng.permutation(num_pages)
    kp = torch.full((num_pages, w.Hkv, page_size, w.d), float("nan"), dtype=w.k_cache.dtype)
    vp = torch.full_like(kp, float("nan"))
    table = torch.full((w.B, max_pages), -1, dtype=torch.int32)
    n = 0
    for b in range(w.B):
        for j in range(used[b]):
            pg = int(phys[n])
            n += 1
            table[b, j] = pg
            lo, hi = j * page_size, min((j + 1) * page_size, w.L_max)
            kp[pg, :, :hi - lo] = w.k_cache[b, :, lo:hi]
            vp[pg, :, :hi - lo] = w.v_cache[b, :, lo:hi]
    return kp, vp, table


CASES = [
    # dtype, B, Q, Hq, Hkv, L_max, seq_lens, k, page_size
    ("bf16", 2, 1, 32, 8, 4096, [4096, 2500], 300, 16),
    ("bf16", 2, 1, 8, 2, 3000, [3000, 1333], 256, 64),
    ("bf16", 3, 1, 8, 2, 2048, [2048, 129, 1000], 100, 128),
    ("bf16", 2, 4, 16, 4, 2048, [2048, 700], 128, 256),     # causal chunk of 4 queries
    ("f32", 2, 1, 4, 2, 1500, [1500, 77], 64, 32),           # fp32: the CUDA-core scorer
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_paged_equals_contiguous_and_oracle(case, cuda_device):
    dtype, B, Q, Hq, Hkv, L, lens, k, ps = case
    seed = zlib.crc32(repr(case).encode()) % 100000
    w = workloads.make_workload(B, Q, Hq, Hkv, L, dtype=dtype, seq_lens=lens, seed=seed)
    q, kc, vc, lens_d = to_device(w)
    kp, vp, table = paged_copy(w, ps, seed=seed)
    tka.topk_attn_device_status()
    got = tka.topk_attn_decode_paged(q, kp.cuda(), vp.cuda(), table.cuda(), lens_d, k)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    # the staged call takes the same three-launch path as the paged call (a
    # small contiguous problem otherwise takes the one-launch path, whose
    # CUDA-core scores round differently from the tensor cores')
    want = tka.topk_attn_decode(q, kc, vc, lens_d, k, stage_events=[None] * 4)
    for g, c in zip(got, want):
        assert torch.equal(g, c)
    check_token(w, k, *got, oracle.topk_attn(w, k))


@pytest.mark.gpu
def test_bad_page_entry_is_reported(cuda_device):
    w = workloads.make_workload(1, 1, 8, 2, 1024, dtype="bf16", seed=3)
    q, _, _, lens_d = to_device(w)
    kp, vp, table = paged_copy(w, 64, seed=3)
    table[0, 5] = kp.shape[0] + 7  # names no page
    tka.topk_attn_device_status()
    tka.topk_attn_decode_paged(q, kp.cuda(), vp.cuda(), table.cuda(), lens_d, 50)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() & tka.DEV_BAD_PAGE
