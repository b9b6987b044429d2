"""topk_attn_decode_static: the decode call for callers that cannot allocate.

Such callers (an engine that reserves all device memory for its own pool and
forbids other allocations while serving, or a host runtime with no device
allocator) get a variant that uses a scratch array built into the library
instead of a caller-provided workspace.  The GPU test calls it through the C
ABI twice in a row, with different inputs and k, and checks each result
against the regular entry point's on the same inputs, within the parity
tolerances; the host test checks that a shape needing more scratch than the
array holds is rejected before anything is launched.

This file is collected last so that a run stopping at the first failure has
run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from parity import TAIL_TOL, out_tol, to_device

import exact_top_sparse_score_b200 as tka
from exact_top_sparse_score_b200 import _binding as bd

TKA_ERR_WORKSPACE = 3


def _static_call(lib, q, kc, vc, lens, k):
    """One topk_attn_decode_static call through ctypes; outputs preallocated by the caller."""
    B, Q, Hq, d = q.shape
    out = torch.empty((B, Q, Hq, d), dtype=torch.float32, device=q.device)
    idx = torch.empty((B, Q, Hq, k), dtype=torch.int32, device=q.device)
    tail = torch.empty((B, Q, Hq), dtype=torch.float32, device=q.device)
    shape = bd.make_shape(q, kc)
    rc = lib.topk_attn_decode_static(ctypes.byref(shape), q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                     lens.data_ptr(), k, out.data_ptr(), idx.data_ptr(), tail.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
    assert rc == 0, f"topk_attn_decode_static returned {rc}"
    return out, idx, tail


@pytest.mark.gpu
def test_static_workspace_matches_regular_entry_point_twice(cuda_device):
    lib = bd.load_library()
    cases = [
        (workloads.make_workload(2, 1, 32, 8, 20000, dtype="bf16", seq_lens=[20000, 13001], k_mean_std=0.5,
                                 seed=901), 512),
        (workloads.make_workload(3, 2, 16, 4, 9000, dtype="bf16", seq_lens=[9000, 4444, 77], seed=902), 300),
        # fp32 cache: the CUDA-core scorer's scores in the shared array, with another k
        (workloads.make_workload(2, 1, 8, 4, 6000, dtype="f32", seq_lens=[6000, 2500], seed=903), 77),
    ]
    for w, k in cases:
        q, kc, vc, lens = to_device(w)
        got = _static_call(lib, q, kc, vc, lens, k)
        torch.cuda.synchronize()
        assert tka.topk_attn_device_status() == 0
        ref = tka.topk_attn_decode(q, kc, vc, lens, k)
        torch.cuda.synchronize()
        atol, rtol = out_tol(w.dtype)
        np.testing.assert_allclose(got[0].cpu().numpy(), ref[0].cpu().numpy(), atol=atol, rtol=rtol)
        assert torch.equal(got[1], ref[1])
        assert (got[2] - ref[2]).abs().max().item() <= TAIL_TOL


@pytest.mark.gpu
def test_static_call_allocates_nothing(cuda_device):
    """The binding-level call with every output preallocated leaves the torch
    allocator's count of allocated bytes unchanged (and the library itself
    never calls a device allocator)."""
    w = workloads.make_workload(2, 1, 32, 8, 12000, dtype="bf16", seed=904)
    q, kc, vc, lens = to_device(w)
    k = 400
    out = torch.empty((2, 1, 32, 128), dtype=torch.float32, device=q.device)
    idx = torch.empty((2, 1, 32, k), dtype=torch.int32, device=q.device)
    tail = torch.empty((2, 1, 32), dtype=torch.float32, device=q.device)
    tka.topk_attn_decode_static(q, kc, vc, lens, k, out=out, idx=idx, tail_mass=tail)  # first call: address lookup
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    for _ in range(3):
        tka.topk_attn_decode_static(q, kc, vc, lens, k, out=out, idx=idx, tail_mass=tail)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    assert tka.topk_attn_device_status() == 0
    ref = tka.topk_attn_decode(q, kc, vc, lens, k)
    assert torch.equal(idx, ref[1])


def test_static_workspace_rejects_shapes_beyond_its_capacity():
    lib = bd.load_library()
    cap = lib.topk_attn_static_workspace_capacity()
    assert cap == 48 << 20
    # B=8, 32 query heads, L = 65536: 256 rows x 256 KB of scores alone exceeds 48 MiB
    shape = bd.tka_shape(8, 1, 32, 8, 128, 65536, 1, 0.0)
    assert bd.topk_attn_workspace_size(shape, 2048) > cap
    fake = 1 << 20
    rc = lib.topk_attn_decode_static(ctypes.byref(shape), fake, fake, fake, fake, 2048, fake, fake, fake, None)
    assert rc == TKA_ERR_WORKSPACE
