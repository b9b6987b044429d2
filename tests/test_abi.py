"""Host-side checks of the C ABI: the library loads, exports every entry point
that include/topk_attn.h declares, sizes workspaces, and rejects bad
arguments on the host before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

from exact_top_sparse_score_b200 import _binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "topk_attn.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
FAKE = 1 << 20  # a non-null, 256-byte aligned address that is never dereferenced on error paths


def declared_functions():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    return sorted(set(re.findall(r"\b(topk_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from exact_top_sparse_score_b200.build import build
    build()
    return bd.load_library()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["topk_attn_decode", "topk_attn_workspace_size", "topk_block_attn_decode",
              "topk_block_pool_keys", "topk_block_attn_workspace_size", "topk_attn_device_status",
              "topk_attn_status_string", "topk_attn_decode_certified",
              "topk_attn_decode_paged", "topk_hisa_attn_decode", "topk_hisa_attn_workspace_size",
              "topk_indexer_attn_decode", "topk_indexer_attn_workspace_size"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.topk_attn_status_string(0) == b"TKA_OK"
    assert lib.topk_attn_status_string(3) == b"TKA_ERR_WORKSPACE"
    assert lib.topk_attn_status_string(5) == b"TKA_ERR_TIMEOUT"


def test_device_status_calls_are_declared_and_exported(lib):
    names = declared_functions()
    for n in ["topk_attn_device_status", "topk_attn_last_device_status", "topk_attn_debug_set_wait_limit"]:
        assert n in names and hasattr(lib, n)
    # the wait limit is a plain host-side setting: setting and clearing it launches nothing
    bd.topk_attn_debug_set_wait_limit(8)
    bd.topk_attn_debug_set_wait_limit(0)


def shape(B=2, Q=1, Hq=8, Hkv=2, d=128, L=1000, dtype=1, scale=0.0):
    return bd.tka_shape(B, Q, Hq, Hkv, d, L, dtype, scale)


def test_workspace_size_layout(lib):
    s = shape(B=8, Q=1, Hq=32, Hkv=8, L=32768)
    n = bd.topk_attn_workspace_size(s, 2048)
    rows = 8 * 32
    # scores + weights + stats + partial (32 splits of 64 keys) + counters
    want = rows * 32768 * 4 + rows * 2048 * 4 + rows * 16 + rows * 32 * 128 * 4 + 1024
    assert n == want
    assert bd.topk_attn_workspace_size(shape(L=1001), 7) % 256 == 0


@pytest.mark.parametrize("kw,k", [(dict(d=64), 8), (dict(dtype=5), 8), (dict(Q=65, L=100), 8),
                                  (dict(Hq=8, Hkv=3), 8), (dict(B=0), 8), (dict(), 0), (dict(), 8193),
                                  (dict(scale=-1.0), 8), (dict(Q=5, L=4), 2)])
def test_workspace_size_zero_on_bad_shape(lib, kw, k):
    assert bd.topk_attn_workspace_size(shape(**kw), k) == 0


def call_decode(lib, s, k=8, q=FAKE, kc=FAKE, vc=FAKE, lens=FAKE, out=FAKE, idx=FAKE, tail=FAKE, ws=FAKE,
                nbytes=None):
    if nbytes is None:
        nbytes = bd.topk_attn_workspace_size(s, k) if bd.topk_attn_workspace_size(s, k) else 1 << 40
    return lib.topk_attn_decode(ctypes.byref(s), q, kc, vc, lens, k, out, idx, tail, ws, nbytes, None)


def test_decode_rejects_bad_arguments_before_launch(lib):
    s = shape()
    assert call_decode(lib, s, k=0) == INVALID
    assert call_decode(lib, s, k=9000) == UNSUPPORTED
    assert call_decode(lib, s, q=None) == INVALID
    assert call_decode(lib, s, idx=None) == INVALID
    assert call_decode(lib, s, kc=FAKE + 8) == INVALID          # misaligned
    assert call_decode(lib, s, ws=None) == WORKSPACE
    assert call_decode(lib, s, ws=FAKE + 16) == WORKSPACE       # workspace not 256-byte aligned
    assert call_decode(lib, s, nbytes=bd.topk_attn_workspace_size(s, 8) - 1) == WORKSPACE
    assert call_decode(lib, shape(d=64)) == UNSUPPORTED
    assert call_decode(lib, shape(Hkv=3)) == INVALID
    assert call_decode(lib, shape(dtype=2)) == UNSUPPORTED
    assert lib.topk_attn_decode(None, FAKE, FAKE, FAKE, FAKE, 8, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == INVALID


def test_block_decode_rejects_bad_arguments_before_launch(lib):
    def call(s, bs=64, top=16, bk=FAKE, nbytes=None):
        if nbytes is None:
            nbytes = bd.block_attn_workspace_size(s, bs, top) or (1 << 40)
        return lib.topk_block_attn_decode(ctypes.byref(s), FAKE, FAKE, FAKE, bk, FAKE, bs, top, FAKE, FAKE,
                                          FAKE, nbytes, None)
    s = shape(L=65536)
    assert call(s, bs=48) == UNSUPPORTED
    assert call(s, top=-1) == INVALID
    assert call(s, top=256) == UNSUPPORTED
    assert call(shape(Q=2, L=65536)) == UNSUPPORTED
    assert call(shape(L=65536 * 4), bs=16) == UNSUPPORTED          # 16384 blocks > 8192
    assert call(s, bk=None) == INVALID
    assert call(s, nbytes=16) == WORKSPACE
    assert lib.topk_block_pool_keys(ctypes.byref(s), FAKE, FAKE, 0, FAKE, None) == INVALID
    assert lib.topk_block_pool_keys(ctypes.byref(shape(d=96)), FAKE, FAKE, 64, FAKE, None) == UNSUPPORTED


def test_binding_rejects_mismatched_output_buffers(lib):
    import torch
    import exact_top_sparse_score_b200 as tka
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    kc = torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16)
    lens = torch.full((1,), 64, dtype=torch.int32)
    with pytest.raises(TypeError):   # fp64 outputs would be misread: the kernels write fp32
        tka.topk_attn_decode(q, kc, kc, lens, 8, out=torch.zeros(1, 1, 4, 128, dtype=torch.float64))
    with pytest.raises(TypeError):
        tka.topk_attn_decode(q, kc, kc, lens, 8, idx=torch.zeros(1, 1, 4, 8, dtype=torch.int64))
    with pytest.raises(ValueError):
        tka.topk_attn_decode(q, kc, kc, lens, 8, tail_mass=torch.zeros(1, 1, 3, dtype=torch.float32))
    with pytest.raises(ValueError):  # host tensors: there is no CPU path
        tka.topk_attn_decode(q, kc, kc, lens, 8)


def test_static_call_checks_arguments_before_its_capacity(lib):
    # a null pointer is an argument error even on a shape too large for the array
    big = shape(B=8, Q=1, Hq=32, Hkv=8, L=65536)
    assert bd.topk_attn_workspace_size(big, 2048) > lib.topk_attn_static_workspace_capacity()
    assert lib.topk_attn_decode_static(ctypes.byref(big), None, FAKE, FAKE, FAKE, 2048, FAKE, FAKE, FAKE,
                                       None) == INVALID
    assert lib.topk_attn_decode_static(ctypes.byref(big), FAKE + 8, FAKE, FAKE, FAKE, 2048, FAKE, FAKE, FAKE,
                                       None) == INVALID
    assert lib.topk_attn_decode_static(ctypes.byref(big), FAKE, FAKE, FAKE, FAKE, 2048, FAKE, FAKE, FAKE,
                                       None) == WORKSPACE


def test_static_binding_checks_v_cache_before_any_launch(lib):
    import torch
    import exact_top_sparse_score_b200 as tka
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    kc = torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16)
    lens = torch.full((1,), 64, dtype=torch.int32)
    out = torch.zeros(1, 1, 4, 128)
    idx = torch.zeros(1, 1, 4, 8, dtype=torch.int32)
    for vc in (torch.zeros(1, 2, 32, 128, dtype=torch.bfloat16), torch.zeros(1, 2, 64, 128)):
        with pytest.raises(TypeError, match="v_cache"):
            tka.topk_attn_decode_static(q, kc, vc, lens, 8, out=out, idx=idx)


class _FakeCuda:
    """Stands in for a CUDA tensor in the binding's host-side checks (no GPU here)."""

    def __init__(self, index):
        import torch
        self.is_cuda = True
        self.device = torch.device("cuda", index)

    def is_contiguous(self):
        return True


def test_binding_requires_every_tensor_on_one_device():
    bd._check_cuda(q=_FakeCuda(0), k_cache=_FakeCuda(0), out=None)
    with pytest.raises(ValueError, match="k_cache is on cuda:1"):
        bd._check_cuda(q=_FakeCuda(0), k_cache=_FakeCuda(1))


def test_every_entry_point_refuses_host_tensors(lib):
    # there is no CPU path anywhere: each public call raises on host memory
    # (before any launch) instead of computing something on the CPU
    import torch
    import exact_top_sparse_score_b200 as tka
    B, Hq, Hkv, L, d = 1, 4, 2, 64, 128
    q = torch.zeros(B, 1, Hq, d, dtype=torch.bfloat16)
    kc = torch.zeros(B, Hkv, L, d, dtype=torch.bfloat16)
    lens = torch.full((B,), L, dtype=torch.int32)
    bk = torch.zeros(B, Hkv, L // 16, d, dtype=torch.float32)
    pages = torch.zeros(L // 16 * B, Hkv, 16, d, dtype=torch.bfloat16)
    table = torch.arange(L // 16, dtype=torch.int32).view(B, L // 16)
    qi = torch.zeros(B, 1, 4, 64, dtype=torch.bfloat16)
    wi = torch.zeros(B, 1, 4, dtype=torch.float32)
    ki = torch.zeros(B, L, 64, dtype=torch.bfloat16)
    calls = {
        "decode": lambda: tka.topk_attn_decode(q, kc, kc, lens, 8),
        "paged": lambda: tka.topk_attn_decode_paged(q, pages, pages, table, lens, 8),
        "certified": lambda: tka.topk_attn_decode_certified(q, kc, kc, lens, 0.1, 8),
        "static": lambda: tka.topk_attn_decode_static(q, kc, kc, lens, 8, out=torch.zeros(B, 1, Hq, d),
                                                      idx=torch.zeros(B, 1, Hq, 8, dtype=torch.int32)),
        "pool": lambda: tka.topk_block_pool_keys(kc, lens, 16),
        "block": lambda: tka.topk_block_attn_decode(q, kc, kc, bk, lens, 16, 2),
        "hisa": lambda: tka.topk_hisa_attn_decode(q, kc, kc, bk, lens, 16, 2, 8),
        "indexer": lambda: tka.topk_indexer_attn_decode(q, kc, kc, qi, wi, ki, lens, 8),
    }
    for name, call in calls.items():
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()
