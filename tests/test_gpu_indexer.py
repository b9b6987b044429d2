"""Lightning-indexer token selection on the GPU against the fp64 oracle
("Sparse Attention Landscape", section "Token Sparse Attention")."""
import zlib

import pytest
import torch

import oracle
import workloads
from parity import check_indexer, index_scores_f64, to_device

import exact_top_sparse_score_b200 as tka

CASES = [
    # dtype, B, Q, Hq, Hkv, L_max, seq_lens, H_I, d_I, k
    ("bf16", 2, 1, 32, 8, 4096, [4096, 2222], 16, 128, 256),
    ("bf16", 2, 4, 8, 2, 2000, [2000, 900], 8, 64, 100),     # causal chunk of 4 queries
    ("f32", 2, 1, 8, 8, 1500, [1500, 40], 4, 64, 64),        # G = 1; fewer tokens than k in batch 1
    ("bf16", 1, 1, 16, 1, 20000, None, 32, 128, 2048),       # G = 16
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_indexer_parity(case, cuda_device):
    dtype, B, Q, Hq, Hkv, L, lens, H_I, d_I, k = case
    seed = zlib.crc32(repr(case).encode()) % 100000
    w = workloads.make_workload(B, Q, Hq, Hkv, L, dtype=dtype, seq_lens=lens, seed=seed)
    qi, wi, ki = workloads.make_indexer_inputs(w, H_I, d_I)
    q, kc, vc, lens_d = to_device(w)
    tka.topk_attn_device_status()
    out, idx = tka.topk_indexer_attn_decode(q, kc, vc, qi.cuda(), wi.cuda(), ki.cuda(), lens_d, k)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    ref = oracle.indexer_attn(w, qi, wi, ki, k)
    n_band = check_indexer(w, k, out, idx, ref, index_scores_f64(w, qi, wi, ki))
    assert n_band <= max(1, B * Q // 4)
