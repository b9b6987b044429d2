"""The bounded waits inside the tensor-core score kernel and the block
attention kernel: a wait that gives up raises TKA_DEV_TIMEOUT, the kernel
drains what it issued and returns, and the next call on the same workspace is
correct again.  The limit is lowered to a few polls through the library's
diagnostics call (no GPU is hung or faulted: every wait stays bounded and the
drains keep their full bound)."""
import pytest
import torch

import oracle
import workloads
from parity import check_block, check_token, to_device

import exact_top_sparse_score_b200 as tka
from exact_top_sparse_score_b200 import _binding as bd

pytestmark = pytest.mark.gpu

TKA_ERR_TIMEOUT = 5


@pytest.fixture
def short_waits():
    yield lambda polls: bd.topk_attn_debug_set_wait_limit(polls)
    bd.topk_attn_debug_set_wait_limit(0)


def test_score_wait_gives_up_and_the_next_call_is_correct(cuda_device, short_waits):
    w = workloads.make_workload(4, 1, 32, 8, 8192, dtype="bf16", seed=311)
    q, kc, vc, lens = to_device(w)
    ws = torch.empty(tka.topk_attn_workspace_size(bd.make_shape(q, kc), 256), dtype=torch.uint8, device=q.device)
    assert tka.topk_attn_device_status() == 0
    short_waits(1)
    tka.topk_attn_decode(q, kc, vc, lens, 256, workspace=ws)
    assert tka.topk_attn_last_device_status() == TKA_ERR_TIMEOUT  # read and cleared
    assert tka.topk_attn_device_status() == 0
    short_waits(0)
    out, idx, tail = tka.topk_attn_decode(q, kc, vc, lens, 256, workspace=ws)
    assert tka.topk_attn_last_device_status() == 0
    check_token(w, 256, out, idx, tail, oracle.topk_attn(w, 256))


def test_block_attention_wait_gives_up_and_the_next_call_is_correct(cuda_device, short_waits):
    w = workloads.make_workload(2, 1, 32, 8, 4096, dtype="bf16", seed=312)
    q, kc, vc, lens = to_device(w)
    bk = tka.topk_block_pool_keys(kc, lens, 64)
    ws = torch.empty(bd.block_attn_workspace_size(bd.make_shape(q, kc), 64, 8), dtype=torch.uint8,
                     device=q.device)
    torch.cuda.synchronize()
    assert tka.topk_attn_device_status() == 0
    short_waits(1)
    tka.topk_block_attn_decode(q, kc, vc, bk, lens, 64, 8, workspace=ws)
    bits = tka.topk_attn_device_status()
    assert bits & tka.DEV_TIMEOUT and not bits & ~tka.DEV_TIMEOUT
    short_waits(0)
    out, bidx = tka.topk_block_attn_decode(q, kc, vc, bk, lens, 64, 8, workspace=ws)
    assert tka.topk_attn_device_status() == 0
    check_block(w, 64, 8, out, bidx, oracle.block_attn(w, 64, 8))
