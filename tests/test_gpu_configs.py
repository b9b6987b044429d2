"""The five decode workloads at full size: CUDA path vs the fp64 oracle on
every query row, in the launch configuration the benchmark times."""
import pytest
import torch

import oracle
import workloads
from parity import check_block, check_token, to_device

import exact_top_sparse_score_b200 as tka

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("cfg", [1, 2, 3, 5])
def test_token_config_full(cfg, cuda_device):
    w = workloads.config_workload(cfg)
    k = w.k
    q, kc, vc, lens = to_device(w)
    out, idx, tail = tka.topk_attn_decode(q, kc, vc, lens, k)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    del kc, vc
    ref = oracle.topk_attn(w, k)
    n_band = check_token(w, k, out, idx, tail, ref)
    rows = w.B * w.Q * w.Hq
    assert n_band <= max(2, rows // 50), f"{n_band} of {rows} rows differ inside the tie band"


def test_block_config_full(cuda_device):
    w = workloads.config_workload(4)
    q, kc, vc, lens = to_device(w)
    bk = tka.topk_block_pool_keys(kc, lens, w.block_size)
    out, bidx = tka.topk_block_attn_decode(q, kc, vc, bk, lens, w.block_size, w.top_blocks)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    ref = oracle.block_attn(w, w.block_size, w.top_blocks)
    n_band = check_block(w, w.block_size, w.top_blocks, out, bidx, ref)
    assert n_band <= 2
