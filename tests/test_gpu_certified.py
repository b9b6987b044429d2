"""Certified adaptive Top-k on the GPU against the fp64 oracle.

Per row the smallest k (at most k_max) whose discarded softmax tail mass is at
most eps ("A Mathematical Theory of Top-k Sparse Attention via Total
Variation Distance", abstract).  tests/parity.py:check_certified states what
must agree.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_certified, to_device

import exact_top_sparse_score_b200 as tka

CASES = [
    # dtype, B, Q, Hq, Hkv, L_max, seq_lens, eps, k_max, k_mean_std, plant_count
    ("bf16", 2, 1, 8, 2, 3000, [3000, 1777], 0.3, 1024, 0.0, 0),
    ("bf16", 2, 1, 8, 2, 3000, [3000, 1777], 0.05, 512, 0.0, 0),    # mostly capped
    ("bf16", 1, 1, 32, 8, 5000, None, 0.75, 2048, 0.5, 0),          # certified well below k_max
    ("bf16", 2, 1, 8, 2, 20000, [20000, 9000], 0.02, 1024, 0.0, 16),  # planted heavy tail
    ("f32", 2, 3, 4, 2, 700, [700, 90], 0.0, 700, 0.0, 0),          # eps 0: every visible key
    ("bf16", 1, 4, 8, 4, 2048, None, 0.5, 4096, 0.0, 0),            # k_max above vis
    ("bf16", 2, 1, 4, 1, 640, [640, 3], 0.999, 64, 0.0, 0),         # eps near 1: the argmax alone
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_certified_parity(case, cuda_device):
    dtype, B, Q, Hq, Hkv, L, lens, eps, k_max, kms, plants = case
    w = workloads.make_workload(B, Q, Hq, Hkv, L, dtype=dtype, seq_lens=lens, k_mean_std=kms,
                                plant_count=plants, seed=zlib.crc32(repr(case).encode()) % 100000)
    q, kc, vc, lens_d = to_device(w)
    out, idx, tail, k_used = tka.topk_attn_decode_certified(q, kc, vc, lens_d, eps, k_max)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    ref = oracle.certified_attn(w, eps, k_max)
    n_diff = check_certified(w, eps, k_max, out, idx, tail, k_used, ref)
    assert n_diff <= max(1, B * Q * Hq // 16), f"{n_diff} rows chose another k than the oracle"


@pytest.mark.gpu
def test_certified_equals_fixed_k_path_at_its_k(cuda_device):
    """At its certified k a row keeps exactly the positions topk_attn_decode keeps
    for that k; out and tail agree up to the summation order (the certified
    path sums the same terms in other groupings)."""
    w = workloads.make_workload(1, 1, 8, 2, 4096, dtype="bf16", seed=91)
    q, kc, vc, lens_d = to_device(w)
    out, idx, tail, k_used = tka.topk_attn_decode_certified(q, kc, vc, lens_d, 0.4, 4096)
    for h in range(8):
        ku = int(k_used[0, 0, h])
        o2, i2, t2 = tka.topk_attn_decode(q, kc, vc, lens_d, ku)
        assert torch.equal(idx[0, 0, h, :ku], i2[0, 0, h])
        torch.testing.assert_close(out[0, 0, h], o2[0, 0, h], rtol=1e-5, atol=1e-6)
        assert abs(float(tail[0, 0, h]) - float(t2[0, 0, h])) <= 1e-5


@pytest.mark.gpu
@pytest.mark.slow
def test_certified_planted_workload_full_size(cuda_device):
    """The planted-retrieval workload at full size (B=4, L up to 131072) with
    k_max = 2048 and eps = 0.01: every row checked against the oracle."""
    w = workloads.config_workload(3)
    q, kc, vc, lens_d = to_device(w)
    out, idx, tail, k_used = tka.topk_attn_decode_certified(q, kc, vc, lens_d, 0.01, 2048)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    del kc, vc
    ref = oracle.certified_attn(w, 0.01, 2048)
    n_diff = check_certified(w, 0.01, 2048, out, idx, tail, k_used, ref)
    assert n_diff <= 4
