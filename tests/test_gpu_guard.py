"""Guard bands and a poisoned workspace for every entry point.

Each output is a view into a larger buffer whose bytes before and after it
hold a sentinel pattern; the workspace is filled with 0xFF bytes (NaN in every
fp32 word, -1 in every int32 word) and framed by sentinel bands too.  After
the call every sentinel byte must be unchanged (nothing is written outside
its buffer) and the results must match the fp64 oracle (nothing reads
workspace it did not write first).  The scratch-array entry point is called
right after a call with a different shape, so its array holds another call's
leftovers."""
import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_block, check_certified, check_hisa, check_indexer, check_token, index_scores_f64, to_device
from test_gpu_paged import paged_copy

import exact_top_sparse_score_b200 as tka
from exact_top_sparse_score_b200 import _binding as bd

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes of sentinel on each side
SENTINEL = 0xA5


class Guarded:
    """A tensor of `shape`/`dtype` framed by sentinel bytes inside one uint8 allocation."""

    def __init__(self, shape, dtype, fill=None):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + n + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        if fill is not None:
            self.raw[GUARD:GUARD + n] = fill
        self.n = n
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape)

    def intact(self):
        return bool((self.raw[:GUARD] == SENTINEL).all()) and bool((self.raw[GUARD + self.n:] == SENTINEL).all())


def poisoned_ws(nbytes):
    return Guarded((nbytes,), torch.uint8, fill=0xFF)


def _seed(tag):
    return zlib.crc32(tag.encode()) % 100000


def test_decode_guard_and_poison(cuda_device):
    w = workloads.make_workload(3, 2, 16, 4, 5000, dtype="bf16", seq_lens=[5000, 3001, 17], seed=_seed("dec"))
    q, kc, vc, lens = to_device(w)
    k = 300
    out = Guarded((w.B, w.Q, w.Hq, 128), torch.float32)
    idx = Guarded((w.B, w.Q, w.Hq, k), torch.int32)
    tail = Guarded((w.B, w.Q, w.Hq), torch.float32)
    ws = poisoned_ws(tka.topk_attn_workspace_size(bd.make_shape(q, kc), k))
    tka.topk_attn_decode(q, kc, vc, lens, k, out=out.t, idx=idx.t, tail_mass=tail.t, workspace=ws.t)
    assert tka.topk_attn_device_status() == 0
    assert out.intact() and idx.intact() and tail.intact() and ws.intact()
    check_token(w, k, out.t, idx.t, tail.t, oracle.topk_attn(w, k))


def test_paged_guard_and_poison(cuda_device):
    w = workloads.make_workload(2, 1, 32, 8, 4096, dtype="bf16", seq_lens=[4096, 2222], seed=_seed("paged"))
    q, _, _, lens = to_device(w)
    kp, vp, table = paged_copy(w, 64, seed=3)
    k = 256
    out = Guarded((w.B, 1, w.Hq, 128), torch.float32)
    idx = Guarded((w.B, 1, w.Hq, k), torch.int32)
    tail = Guarded((w.B, 1, w.Hq), torch.float32)
    ws = poisoned_ws(tka.topk_attn_workspace_size(bd.make_shape(q, w.k_cache.to("cuda")), k))
    tka.topk_attn_decode_paged(q, kp.cuda(), vp.cuda(), table.cuda(), lens, k, out=out.t, idx=idx.t,
                               tail_mass=tail.t, workspace=ws.t)
    assert tka.topk_attn_device_status() == 0
    assert out.intact() and idx.intact() and tail.intact() and ws.intact()
    check_token(w, k, out.t, idx.t, tail.t, oracle.topk_attn(w, k))


def test_certified_guard_and_poison(cuda_device):
    w = workloads.make_workload(2, 1, 32, 8, 6000, dtype="bf16", seq_lens=[6000, 4000], plant_count=16,
                                seed=_seed("cert"))
    q, kc, vc, lens = to_device(w)
    k_max, eps = 512, 0.05
    out = Guarded((w.B, 1, w.Hq, 128), torch.float32)
    idx = Guarded((w.B, 1, w.Hq, k_max), torch.int32)
    tail = Guarded((w.B, 1, w.Hq), torch.float32)
    k_used = Guarded((w.B, 1, w.Hq), torch.int32)
    ws = poisoned_ws(tka.topk_attn_workspace_size(bd.make_shape(q, kc), k_max))
    tka.topk_attn_decode_certified(q, kc, vc, lens, eps, k_max, out=out.t, idx=idx.t, tail_mass=tail.t,
                                   k_used=k_used.t, workspace=ws.t)
    assert tka.topk_attn_device_status() == 0
    assert out.intact() and idx.intact() and tail.intact() and k_used.intact() and ws.intact()
    check_certified(w, eps, k_max, out.t, idx.t, tail.t, k_used.t, oracle.certified_attn(w, eps, k_max))


def test_static_guard_after_another_shape(cuda_device):
    # a bigger call first fills the built-in array with its own scratch
    w0 = workloads.make_workload(4, 1, 32, 8, 9000, dtype="bf16", seed=_seed("static0"))
    q0, kc0, vc0, lens0 = to_device(w0)
    o0 = torch.empty((4, 1, 32, 128), dtype=torch.float32, device="cuda")
    i0 = torch.empty((4, 1, 32, 700), dtype=torch.int32, device="cuda")
    tka.topk_attn_decode_static(q0, kc0, vc0, lens0, 700, out=o0, idx=i0)
    w = workloads.make_workload(2, 3, 8, 2, 3000, dtype="bf16", seq_lens=[3000, 1200], seed=_seed("static"))
    q, kc, vc, lens = to_device(w)
    k = 200
    out = Guarded((w.B, w.Q, w.Hq, 128), torch.float32)
    idx = Guarded((w.B, w.Q, w.Hq, k), torch.int32)
    tail = Guarded((w.B, w.Q, w.Hq), torch.float32)
    tka.topk_attn_decode_static(q, kc, vc, lens, k, out=out.t, idx=idx.t, tail_mass=tail.t)
    assert tka.topk_attn_device_status() == 0
    assert out.intact() and idx.intact() and tail.intact()
    check_token(w, k, out.t, idx.t, tail.t, oracle.topk_attn(w, k))


def test_block_guard_and_poison(cuda_device):
    w = workloads.make_workload(2, 1, 32, 8, 8192, dtype="bf16", seq_lens=[8192, 5000], seed=_seed("block"))
    q, kc, vc, lens = to_device(w)
    bs, top = 64, 16
    nblk = 8192 // bs
    bk = Guarded((w.B, w.Hkv, nblk, 128), torch.float32, fill=0xFF)
    tka.topk_block_pool_keys(kc, lens, bs, block_keys=bk.t)
    out = Guarded((w.B, 1, w.Hq, 128), torch.float32)
    bidx = Guarded((w.B, 1, w.Hq, top + 1), torch.int32)
    ws = poisoned_ws(bd.block_attn_workspace_size(bd.make_shape(q, kc), bs, top))
    tka.topk_block_attn_decode(q, kc, vc, bk.t, lens, bs, top, out=out.t, block_idx=bidx.t, workspace=ws.t)
    assert tka.topk_attn_device_status() == 0
    assert bk.intact() and out.intact() and bidx.intact() and ws.intact()
    np.testing.assert_allclose(bk.t.cpu().double().numpy(), oracle.block_pool(w, bs), atol=2e-5, rtol=1e-5)
    check_block(w, bs, top, out.t, bidx.t, oracle.block_attn(w, bs, top))


def test_hisa_guard_and_poison(cuda_device):
    w = workloads.make_workload(2, 1, 8, 2, 4096, dtype="bf16", seq_lens=[4096, 3000], seed=_seed("hisa"))
    q, kc, vc, lens = to_device(w)
    bs, top, k = 64, 16, 256
    bk = tka.topk_block_pool_keys(kc, lens, bs)
    out = Guarded((w.B, 1, w.Hq, 128), torch.float32)
    idx = Guarded((w.B, 1, w.Hq, k), torch.int32)
    tail = Guarded((w.B, 1, w.Hq), torch.float32)
    bidx = Guarded((w.B, 1, w.Hq, top), torch.int32)
    nbytes = tka.load_library().topk_hisa_attn_workspace_size(bd.make_shape(q, kc), bs, top, k)
    ws = poisoned_ws(nbytes)
    tka.topk_hisa_attn_decode(q, kc, vc, bk, lens, bs, top, k, out=out.t, idx=idx.t, tail_mass=tail.t,
                              block_idx=bidx.t, workspace=ws.t)
    assert tka.topk_attn_device_status() == 0
    assert out.intact() and idx.intact() and tail.intact() and bidx.intact() and ws.intact()
    check_hisa(w, bs, top, k, out.t, idx.t, tail.t, bidx.t, oracle.hisa_attn(w, bs, top, k))


def test_indexer_guard_and_poison(cuda_device):
    w = workloads.make_workload(2, 2, 32, 8, 3000, dtype="bf16", seq_lens=[3000, 1500], seed=_seed("indexer"))
    qi, wi, ki = workloads.make_indexer_inputs(w, 16, 128)
    q, kc, vc, lens = to_device(w)
    k = 200
    out = Guarded((w.B, w.Q, w.Hq, 128), torch.float32)
    idx = Guarded((w.B, w.Q, k), torch.int32)
    nbytes = tka.load_library().topk_indexer_attn_workspace_size(bd.make_shape(q, kc), 16, 128, k)
    ws = poisoned_ws(nbytes)
    tka.topk_indexer_attn_decode(q, kc, vc, qi.cuda(), wi.cuda(), ki.cuda(), lens, k, out=out.t, idx=idx.t,
                                 workspace=ws.t)
    assert tka.topk_attn_device_status() == 0
    assert out.intact() and idx.intact() and ws.intact()
    check_indexer(w, k, out.t, idx.t, oracle.indexer_attn(w, qi, wi, ki, k), index_scores_f64(w, qi, wi, ki))
