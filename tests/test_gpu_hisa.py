"""Hierarchical block -> token Top-k on the GPU against the fp64 oracle
("Sparse Attention Landscape", section "Hierarchical Sparse Attention")."""
import zlib

import pytest
import torch

import oracle
import workloads
from parity import check_hisa, to_device

import exact_top_sparse_score_b200 as tka

CASES = [
    # dtype, B, Hq, Hkv, L_max, seq_lens, block_size, top_blocks, k
    ("bf16", 2, 8, 2, 4096, [4096, 3000], 64, 16, 256),
    ("bf16", 2, 32, 8, 2000, [2000, 1111], 32, 8, 64),
    ("f32", 2, 8, 4, 1024, [1024, 70], 16, 7, 50),
    ("bf16", 1, 4, 1, 640, None, 128, 2, 300),          # fewer candidates than k: padding
    ("bf16", 2, 8, 2, 700, [700, 64], 64, 30, 100),     # every block kept
    ("bf16", 1, 8, 2, 65536, [65521], 64, 32, 512),     # long row, 1024 blocks
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_hisa_parity(case, cuda_device):
    dtype, B, Hq, Hkv, L, lens, bs, top, k = case
    w = workloads.make_workload(B, 1, Hq, Hkv, L, dtype=dtype, seq_lens=lens,
                                seed=zlib.crc32(repr(case).encode()) % 100000)
    q, kc, vc, lens_d = to_device(w)
    bk = tka.topk_block_pool_keys(kc, lens_d, bs)
    tka.topk_attn_device_status()
    out, idx, tail, bidx = tka.topk_hisa_attn_decode(q, kc, vc, bk, lens_d, bs, top, k)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    ref = oracle.hisa_attn(w, bs, top, k)
    n_band = check_hisa(w, bs, top, k, out, idx, tail, bidx, ref)
    assert n_band <= max(2, B * Hq // 8)
