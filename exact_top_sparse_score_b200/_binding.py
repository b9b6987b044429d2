"""ctypes binding of the C ABI in include/topk_attn.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libtopk_attn.so"

TKA_F32, TKA_BF16 = 0, 1
DEV_BAD_SEQ_LEN, DEV_INTERNAL, DEV_TIMEOUT, DEV_BAD_PAGE = 0x1, 0x2, 0x4, 0x8
_STATUS = {0: "TKA_OK", 1: "TKA_ERR_INVALID_ARG", 2: "TKA_ERR_UNSUPPORTED", 3: "TKA_ERR_WORKSPACE",
           4: "TKA_ERR_CUDA", 5: "TKA_ERR_TIMEOUT"}


class TopkAttnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {_STATUS.get(code, code)}")
        self.code = code


class tka_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Q", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32), ("L_max", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("scale", ctypes.c_float)]


_lib = None
_vp, _sz, _i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
_shape_p = ctypes.POINTER(tka_shape)


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def load_library() -> ctypes.CDLL:
    """Loads the in-tree CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m exact_top_sparse_score_b200.build` "
                               "(there is no fallback implementation)")
        lib = ctypes.CDLL(path)
        lib.topk_attn_workspace_size.argtypes = [_shape_p, _i32]
        lib.topk_attn_workspace_size.restype = _sz
        lib.topk_attn_decode.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp]
        lib.topk_attn_decode.restype = ctypes.c_int
        lib.topk_attn_decode_staged.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp,
                                                ctypes.POINTER(_vp)]
        lib.topk_attn_decode_staged.restype = ctypes.c_int
        lib.topk_attn_decode_certified.argtypes = [_shape_p, _vp, _vp, _vp, _vp, ctypes.c_float, _i32, _vp, _vp,
                                                   _vp, _vp, _vp, _sz, _vp]
        lib.topk_attn_decode_certified.restype = ctypes.c_int
        lib.topk_attn_decode_paged.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _i32, _vp,
                                               _vp, _vp, _vp, _sz, _vp]
        lib.topk_attn_decode_paged.restype = ctypes.c_int
        lib.topk_hisa_attn_workspace_size.argtypes = [_shape_p, _i32, _i32, _i32]
        lib.topk_hisa_attn_workspace_size.restype = _sz
        lib.topk_hisa_attn_decode.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp,
                                              _vp, _vp, _sz, _vp]
        lib.topk_hisa_attn_decode.restype = ctypes.c_int
        lib.topk_indexer_attn_workspace_size.argtypes = [_shape_p, _i32, _i32, _i32]
        lib.topk_indexer_attn_workspace_size.restype = _sz
        lib.topk_indexer_attn_decode.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i32,
                                                 _vp, _vp, _vp, _sz, _vp]
        lib.topk_indexer_attn_decode.restype = ctypes.c_int
        lib.topk_attn_static_workspace_capacity.argtypes = []
        lib.topk_attn_static_workspace_capacity.restype = _sz
        lib.topk_attn_decode_static.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp]
        lib.topk_attn_decode_static.restype = ctypes.c_int
        lib.topk_block_pool_keys.argtypes = [_shape_p, _vp, _vp, _i32, _vp, _vp]
        lib.topk_block_pool_keys.restype = ctypes.c_int
        lib.topk_block_attn_workspace_size.argtypes = [_shape_p, _i32, _i32]
        lib.topk_block_attn_workspace_size.restype = _sz
        lib.topk_block_attn_decode.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp,
                                               _sz, _vp]
        lib.topk_block_attn_decode.restype = ctypes.c_int
        lib.topk_attn_device_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint32)]
        lib.topk_attn_device_status.restype = ctypes.c_int
        lib.topk_attn_last_device_status.argtypes = [_vp]
        lib.topk_attn_last_device_status.restype = ctypes.c_int
        lib.topk_attn_debug_set_wait_limit.argtypes = [ctypes.c_uint32]
        lib.topk_attn_debug_set_wait_limit.restype = None
        lib.topk_attn_status_string.argtypes = [ctypes.c_int]
        lib.topk_attn_status_string.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TKA_BF16
    if t.dtype == torch.float32:
        return TKA_F32
    raise TypeError(f"unsupported cache dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_cuda(**tensors):
    """Every tensor must be a contiguous CUDA tensor, all on one device (the
    library launches on the current device, which the wrappers set to it)."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other tensors on {dev}")


def _on_device(fn):
    """Runs a wrapper with the device of its first tensor argument current, so
    that the library's kernels, its per-device state and the default stream
    all belong to the device the tensors live on."""
    import functools

    @functools.wraps(fn)
    def run(*args, **kwargs):
        first = args[0] if args else None
        if isinstance(first, torch.Tensor) and first.is_cuda:
            with torch.cuda.device(first.device):
                return fn(*args, **kwargs)
        return fn(*args, **kwargs)
    return run


def _check_out(name: str, t: Optional[torch.Tensor], dtype: torch.dtype, shape: tuple):
    """Caller-supplied output buffers must match what the kernels write."""
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def make_shape(q: torch.Tensor, k_cache: torch.Tensor, scale: float = 0.0) -> tka_shape:
    """Shape struct from q [B,Q,Hq,d] and a cache [B,Hkv,L_max,d]."""
    if q.dim() != 4 or k_cache.dim() != 4:
        raise ValueError("q must be [B,Q,Hq,d] and the caches [B,Hkv,L_max,d]")
    B, Q, Hq, d = q.shape
    Bk, Hkv, L_max, dk = k_cache.shape
    if Bk != B or dk != d:
        raise ValueError("q and cache shapes disagree")
    if q.dtype != k_cache.dtype:
        raise TypeError("q must have the cache dtype")
    return tka_shape(B, Q, Hq, Hkv, d, L_max, _dtype_code(k_cache), float(scale))


def topk_attn_workspace_size(shape: tka_shape, k: int) -> int:
    return int(load_library().topk_attn_workspace_size(ctypes.byref(shape), k))


def block_attn_workspace_size(shape: tka_shape, block_size: int, top_blocks: int) -> int:
    return int(load_library().topk_block_attn_workspace_size(ctypes.byref(shape), block_size, top_blocks))


# Workspaces the binding allocates itself, one per (device, stream), grown on
# demand and kept for the life of the process: a call's kernels may still be
# running when the call returns, so its scratch must not go back to the
# allocator at that point.  Calls on one stream run in order, so they can
# share one buffer.
_cached_ws = {}


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor], stream_handle: int) -> torch.Tensor:
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace needs {nbytes} bytes")
        return workspace
    key = (torch.device(device).index, stream_handle)
    ws = _cached_ws.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        _cached_ws[key] = ws
    return ws


@_on_device
def topk_attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, seq_lens: torch.Tensor,
                     k: int, *, scale: float = 0.0, out: Optional[torch.Tensor] = None,
                     idx: Optional[torch.Tensor] = None, tail_mass: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, want_tail: bool = True,
                     stream=None, stage_events=None) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """Exact Top-k decode attention; returns (out fp32 [B,Q,Hq,d], idx int32 [B,Q,Hq,k], tail fp32 [B,Q,Hq]).

    stage_events: optional four torch.cuda.Event objects (or None entries, not
    recorded) for before score, before select, before gather (idx is final
    there) and after gather (topk_attn_decode_staged)."""
    lib = load_library()
    shape = make_shape(q, k_cache, scale)
    B, Q, Hq, d = q.shape
    dev = q.device
    if out is None:
        out = torch.empty((B, Q, Hq, d), dtype=torch.float32, device=dev)
    if idx is None:
        idx = torch.empty((B, Q, Hq, k), dtype=torch.int32, device=dev)
    if tail_mass is None and want_tail:
        tail_mass = torch.empty((B, Q, Hq), dtype=torch.float32, device=dev)
    if seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise TypeError("seq_lens must be int32 [B]")
    if v_cache.dtype != k_cache.dtype or v_cache.shape != k_cache.shape:
        raise TypeError("v_cache must match k_cache in dtype and shape")
    _check_out("out", out, torch.float32, (B, Q, Hq, d))
    _check_out("idx", idx, torch.int32, (B, Q, Hq, k))
    _check_out("tail_mass", tail_mass, torch.float32, (B, Q, Hq))
    if workspace is not None and workspace.dtype != torch.uint8:
        raise TypeError("workspace must be a uint8 tensor")
    _check_cuda(q=q, k_cache=k_cache, v_cache=v_cache, seq_lens=seq_lens, out=out, idx=idx, tail_mass=tail_mass,
                workspace=workspace)
    nbytes = topk_attn_workspace_size(shape, k)
    if nbytes == 0:
        raise TopkAttnError("topk_attn_workspace_size", 2)
    sh = _stream(stream)
    ws = _workspace(nbytes, dev, workspace, sh)
    args = (ctypes.byref(shape), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seq_lens.data_ptr(), k,
            out.data_ptr(), idx.data_ptr(), _ptr(tail_mass), ws.data_ptr(), nbytes, sh)
    if stage_events is None:
        rc = lib.topk_attn_decode(*args)
    else:
        evs = (_vp * 4)(*[e.cuda_event if e is not None else None for e in stage_events])
        rc = lib.topk_attn_decode_staged(*args, evs)
    if rc:
        raise TopkAttnError("topk_attn_decode", rc)
    return out, idx, tail_mass


@_on_device
def topk_attn_decode_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                           block_table: torch.Tensor, seq_lens: torch.Tensor, k: int, *, scale: float = 0.0,
                           out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                           tail_mass: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Exact Top-k decode attention over a paged cache: k_pages / v_pages
    [num_pages, Hkv, page_size, d], block_table int32 [B, max_pages] (logical
    page j of sequence b -> physical page).  Returns (out, idx, tail) as
    topk_attn_decode does on the equivalent contiguous cache."""
    lib = load_library()
    if q.dim() != 4 or k_pages.dim() != 4 or block_table.dim() != 2:
        raise ValueError("q [B,Q,Hq,d], pages [num_pages,Hkv,page_size,d], block_table [B,max_pages]")
    B, Q, Hq, d = q.shape
    num_pages, Hkv, page_size, dk = k_pages.shape
    max_pages = block_table.shape[1]
    if dk != d or block_table.shape[0] != B:
        raise ValueError("q, pages and block_table shapes disagree")
    if q.dtype != k_pages.dtype or v_pages.dtype != k_pages.dtype or v_pages.shape != k_pages.shape:
        raise TypeError("q, k_pages and v_pages must share dtype and shape")
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise TypeError("block_table and seq_lens must be int32")
    shape = tka_shape(B, Q, Hq, Hkv, d, max_pages * page_size, _dtype_code(k_pages), float(scale))
    dev = q.device
    if out is None:
        out = torch.empty((B, Q, Hq, d), dtype=torch.float32, device=dev)
    if idx is None:
        idx = torch.empty((B, Q, Hq, k), dtype=torch.int32, device=dev)
    if tail_mass is None:
        tail_mass = torch.empty((B, Q, Hq), dtype=torch.float32, device=dev)
    _check_out("out", out, torch.float32, (B, Q, Hq, d))
    _check_out("idx", idx, torch.int32, (B, Q, Hq, k))
    _check_out("tail_mass", tail_mass, torch.float32, (B, Q, Hq))
    if workspace is not None and workspace.dtype != torch.uint8:
        raise TypeError("workspace must be a uint8 tensor")
    _check_cuda(q=q, k_pages=k_pages, v_pages=v_pages, block_table=block_table, seq_lens=seq_lens, out=out,
                idx=idx, tail_mass=tail_mass, workspace=workspace)
    nbytes = topk_attn_workspace_size(shape, k)
    if nbytes == 0:
        raise TopkAttnError("topk_attn_workspace_size", 2)
    sh = _stream(stream)
    ws = _workspace(nbytes, dev, workspace, sh)
    rc = lib.topk_attn_decode_paged(ctypes.byref(shape), q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                    block_table.data_ptr(), max_pages, num_pages, page_size, seq_lens.data_ptr(), k,
                                    out.data_ptr(), idx.data_ptr(), tail_mass.data_ptr(), ws.data_ptr(), nbytes, sh)
    if rc:
        raise TopkAttnError("topk_attn_decode_paged", rc)
    return out, idx, tail_mass


@_on_device
def topk_attn_decode_certified(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                               seq_lens: torch.Tensor, eps: float, k_max: int, *, scale: float = 0.0,
                               out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                               tail_mass: Optional[torch.Tensor] = None, k_used: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None, stream=None):
    """Certified adaptive Top-k decode attention: per row the smallest k (at
    most k_max) whose discarded softmax tail mass is <= eps.  Returns
    (out fp32 [B,Q,Hq,d], idx int32 [B,Q,Hq,k_max], tail fp32 [B,Q,Hq],
    k_used int32 [B,Q,Hq])."""
    lib = load_library()
    shape = make_shape(q, k_cache, scale)
    B, Q, Hq, d = q.shape
    dev = q.device
    if out is None:
        out = torch.empty((B, Q, Hq, d), dtype=torch.float32, device=dev)
    if idx is None:
        idx = torch.empty((B, Q, Hq, k_max), dtype=torch.int32, device=dev)
    if tail_mass is None:
        tail_mass = torch.empty((B, Q, Hq), dtype=torch.float32, device=dev)
    if k_used is None:
        k_used = torch.empty((B, Q, Hq), dtype=torch.int32, device=dev)
    if seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise TypeError("seq_lens must be int32 [B]")
    if v_cache.dtype != k_cache.dtype or v_cache.shape != k_cache.shape:
        raise TypeError("v_cache must match k_cache in dtype and shape")
    _check_out("out", out, torch.float32, (B, Q, Hq, d))
    _check_out("idx", idx, torch.int32, (B, Q, Hq, k_max))
    _check_out("tail_mass", tail_mass, torch.float32, (B, Q, Hq))
    _check_out("k_used", k_used, torch.int32, (B, Q, Hq))
    if workspace is not None and workspace.dtype != torch.uint8:
        raise TypeError("workspace must be a uint8 tensor")
    _check_cuda(q=q, k_cache=k_cache, v_cache=v_cache, seq_lens=seq_lens, out=out, idx=idx, tail_mass=tail_mass,
                k_used=k_used, workspace=workspace)
    nbytes = topk_attn_workspace_size(shape, k_max)
    if nbytes == 0:
        raise TopkAttnError("topk_attn_workspace_size", 2)
    sh = _stream(stream)
    ws = _workspace(nbytes, dev, workspace, sh)
    rc = lib.topk_attn_decode_certified(ctypes.byref(shape), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                        seq_lens.data_ptr(), float(eps), k_max, out.data_ptr(), idx.data_ptr(),
                                        tail_mass.data_ptr(), k_used.data_ptr(), ws.data_ptr(), nbytes, sh)
    if rc:
        raise TopkAttnError("topk_attn_decode_certified", rc)
    return out, idx, tail_mass, k_used


@_on_device
def topk_attn_decode_static(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, seq_lens: torch.Tensor,
                            k: int, *, out: torch.Tensor, idx: torch.Tensor, tail_mass: Optional[torch.Tensor] = None,
                            scale: float = 0.0, stream=None) -> None:
    """topk_attn_decode on the library's built-in scratch array: the caller
    passes every output buffer and nothing is allocated (no torch allocation
    either).  Raises TopkAttnError (TKA_ERR_WORKSPACE) when the shape needs
    more scratch than topk_attn_static_workspace_capacity()."""
    lib = load_library()
    shape = make_shape(q, k_cache, scale)
    B, Q, Hq, d = q.shape
    if seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise TypeError("seq_lens must be int32 [B]")
    if v_cache.dtype != k_cache.dtype or v_cache.shape != k_cache.shape:
        raise TypeError("v_cache must match k_cache in dtype and shape")
    _check_out("out", out, torch.float32, (B, Q, Hq, d))
    _check_out("idx", idx, torch.int32, (B, Q, Hq, k))
    _check_out("tail_mass", tail_mass, torch.float32, (B, Q, Hq))
    _check_cuda(q=q, k_cache=k_cache, v_cache=v_cache, seq_lens=seq_lens, out=out, idx=idx, tail_mass=tail_mass)
    rc = lib.topk_attn_decode_static(ctypes.byref(shape), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                     seq_lens.data_ptr(), k, out.data_ptr(), idx.data_ptr(), _ptr(tail_mass),
                                     _stream(stream))
    if rc:
        raise TopkAttnError("topk_attn_decode_static", rc)


def topk_attn_static_workspace_capacity() -> int:
    return int(load_library().topk_attn_static_workspace_capacity())


@_on_device
def topk_block_pool_keys(k_cache: torch.Tensor, seq_lens: torch.Tensor, block_size: int, *,
                         block_keys: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Mean-pooled block keys fp32 [B, Hkv, ceil(L_max/block_size), d]."""
    lib = load_library()
    B, Hkv, L_max, d = k_cache.shape
    nblk = -(-L_max // block_size)
    if block_keys is None:
        block_keys = torch.empty((B, Hkv, nblk, d), dtype=torch.float32, device=k_cache.device)
    if seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise TypeError("seq_lens must be int32 [B]")
    _check_out("block_keys", block_keys, torch.float32, (B, Hkv, nblk, d))
    _check_cuda(k_cache=k_cache, seq_lens=seq_lens, block_keys=block_keys)
    shape = tka_shape(B, 1, Hkv, Hkv, d, L_max, _dtype_code(k_cache), 0.0)
    rc = lib.topk_block_pool_keys(ctypes.byref(shape), k_cache.data_ptr(), seq_lens.data_ptr(), block_size,
                                  block_keys.data_ptr(), _stream(stream))
    if rc:
        raise TopkAttnError("topk_block_pool_keys", rc)
    return block_keys


@_on_device
def topk_block_attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                           block_keys: torch.Tensor, seq_lens: torch.Tensor, block_size: int, top_blocks: int, *,
                           scale: float = 0.0, out: Optional[torch.Tensor] = None,
                           block_idx: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MoBA block-sparse decode attention; returns (out fp32 [B,1,Hq,d], block_idx int32 [B,1,Hq,top+1])."""
    lib = load_library()
    shape = make_shape(q, k_cache, scale)
    B, Q, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Q, Hq, d), dtype=torch.float32, device=q.device)
    if block_idx is None:
        block_idx = torch.empty((B, Q, Hq, top_blocks + 1), dtype=torch.int32, device=q.device)
    if seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise TypeError("seq_lens must be int32 [B]")
    if v_cache.dtype != k_cache.dtype or v_cache.shape != k_cache.shape:
        raise TypeError("v_cache must match k_cache in dtype and shape")
    _check_out("out", out, torch.float32, (B, Q, Hq, d))
    _check_out("block_idx", block_idx, torch.int32, (B, Q, Hq, top_blocks + 1))
    _check_out("block_keys", block_keys, torch.float32, (B, k_cache.shape[1], -(-k_cache.shape[2] // block_size), d))
    if workspace is not None and workspace.dtype != torch.uint8:
        raise TypeError("workspace must be a uint8 tensor")
    _check_cuda(q=q, k_cache=k_cache, v_cache=v_cache, block_keys=block_keys, seq_lens=seq_lens, out=out,
                block_idx=block_idx, workspace=workspace)
    nbytes = block_attn_workspace_size(shape, block_size, top_blocks)
    if nbytes == 0:
        raise TopkAttnError("topk_block_attn_workspace_size", 2)
    sh = _stream(stream)
    ws = _workspace(nbytes, q.device, workspace, sh)
    rc = lib.topk_block_attn_decode(ctypes.byref(shape), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                    block_keys.data_ptr(), seq_lens.data_ptr(), block_size, top_blocks,
                                    out.data_ptr(), block_idx.data_ptr(), ws.data_ptr(), nbytes, sh)
    if rc:
        raise TopkAttnError("topk_block_attn_decode", rc)
    return out, block_idx


def topk_attn_last_device_status(stream=None) -> int:
    """Synchronises the stream and returns the device status word read as a
    status code (5 = TKA_ERR_TIMEOUT when a bounded wait gave up), clearing it."""
    return int(load_library().topk_attn_last_device_status(_stream(stream)))


def topk_attn_debug_set_wait_limit(polls: int) -> None:
    """Diagnostics: polls before a pipeline wait inside the tensor-core score
    and block-attention kernels gives up (0 restores the default bound)."""
    load_library().topk_attn_debug_set_wait_limit(int(polls))


def topk_attn_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status bits."""
    bits = ctypes.c_uint32(0)
    rc = load_library().topk_attn_device_status(_stream(stream), ctypes.byref(bits))
    if rc:
        raise TopkAttnError("topk_attn_device_status", rc)
    return int(bits.value)


@_on_device
def topk_hisa_attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_keys: torch.Tensor,
                          seq_lens: torch.Tensor, block_size: int, top_blocks: int, k: int, *, scale: float = 0.0,
                          out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                          tail_mass: Optional[torch.Tensor] = None, block_idx: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None, stream=None):
    """Hierarchical block -> token Top-k decode attention (one query per sequence).

    Returns (out fp32 [B,1,Hq,d], idx int32 [B,1,Hq,k], tail fp32 [B,1,Hq],
    block_idx int32 [B,1,Hq,top_blocks])."""
    lib = load_library()
    shape = make_shape(q, k_cache, scale)
    B, Q, Hq, d = q.shape
    dev = q.device
    if out is None:
        out = torch.empty((B, Q, Hq, d), dtype=torch.float32, device=dev)
    if idx is None:
        idx = torch.empty((B, Q, Hq, k), dtype=torch.int32, device=dev)
    if tail_mass is None:
        tail_mass = torch.empty((B, Q, Hq), dtype=torch.float32, device=dev)
    if block_idx is None:
        block_idx = torch.empty((B, Q, Hq, top_blocks), dtype=torch.int32, device=dev)
    if seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise TypeError("seq_lens must be int32 [B]")
    if v_cache.dtype != k_cache.dtype or v_cache.shape != k_cache.shape:
        raise TypeError("v_cache must match k_cache in dtype and shape")
    _check_out("out", out, torch.float32, (B, Q, Hq, d))
    _check_out("idx", idx, torch.int32, (B, Q, Hq, k))
    _check_out("tail_mass", tail_mass, torch.float32, (B, Q, Hq))
    _check_out("block_idx", block_idx, torch.int32, (B, Q, Hq, top_blocks))
    _check_out("block_keys", block_keys, torch.float32, (B, k_cache.shape[1], -(-k_cache.shape[2] // block_size), d))
    if workspace is not None and workspace.dtype != torch.uint8:
        raise TypeError("workspace must be a uint8 tensor")
    _check_cuda(q=q, k_cache=k_cache, v_cache=v_cache, block_keys=block_keys, seq_lens=seq_lens, out=out, idx=idx,
                tail_mass=tail_mass, block_idx=block_idx, workspace=workspace)
    nbytes = int(lib.topk_hisa_attn_workspace_size(ctypes.byref(shape), block_size, top_blocks, k))
    if nbytes == 0:
        raise TopkAttnError("topk_hisa_attn_workspace_size", 2)
    sh = _stream(stream)
    ws = _workspace(nbytes, dev, workspace, sh)
    rc = lib.topk_hisa_attn_decode(ctypes.byref(shape), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                   block_keys.data_ptr(), seq_lens.data_ptr(), block_size, top_blocks, k,
                                   out.data_ptr(), idx.data_ptr(), tail_mass.data_ptr(), block_idx.data_ptr(),
                                   ws.data_ptr(), nbytes, sh)
    if rc:
        raise TopkAttnError("topk_hisa_attn_decode", rc)
    return out, idx, tail_mass, block_idx


@_on_device
def topk_indexer_attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, q_idx: torch.Tensor,
                             w_idx: torch.Tensor, k_idx: torch.Tensor, seq_lens: torch.Tensor, k: int, *,
                             scale: float = 0.0, out: Optional[torch.Tensor] = None,
                             idx: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                             stream=None):
    """Lightning-indexer token selection, then exact attention per head.

    Returns (out fp32 [B,Q,Hq,d], idx int32 [B,Q,k])."""
    lib = load_library()
    shape = make_shape(q, k_cache, scale)
    B, Q, Hq, d = q.shape
    if q_idx.dim() != 4 or tuple(q_idx.shape[:2]) != (B, Q):
        raise ValueError("q_idx must be [B,Q,H_I,d_I]")
    H_I, d_I = q_idx.shape[2], q_idx.shape[3]
    if tuple(k_idx.shape) != (B, k_cache.shape[2], d_I) or tuple(w_idx.shape) != (B, Q, H_I):
        raise ValueError("k_idx must be [B,L_max,d_I] and w_idx [B,Q,H_I]")
    if q_idx.dtype != k_cache.dtype or k_idx.dtype != k_cache.dtype or w_idx.dtype != torch.float32:
        raise TypeError("q_idx and k_idx take the cache dtype, w_idx fp32")
    dev = q.device
    if out is None:
        out = torch.empty((B, Q, Hq, d), dtype=torch.float32, device=dev)
    if idx is None:
        idx = torch.empty((B, Q, k), dtype=torch.int32, device=dev)
    if seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise TypeError("seq_lens must be int32 [B]")
    _check_out("out", out, torch.float32, (B, Q, Hq, d))
    _check_out("idx", idx, torch.int32, (B, Q, k))
    if workspace is not None and workspace.dtype != torch.uint8:
        raise TypeError("workspace must be a uint8 tensor")
    _check_cuda(q=q, k_cache=k_cache, v_cache=v_cache, q_idx=q_idx, w_idx=w_idx, k_idx=k_idx, seq_lens=seq_lens,
                out=out, idx=idx, workspace=workspace)
    nbytes = int(lib.topk_indexer_attn_workspace_size(ctypes.byref(shape), H_I, d_I, k))
    if nbytes == 0:
        raise TopkAttnError("topk_indexer_attn_workspace_size", 2)
    sh = _stream(stream)
    ws = _workspace(nbytes, dev, workspace, sh)
    rc = lib.topk_indexer_attn_decode(ctypes.byref(shape), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                      q_idx.data_ptr(), w_idx.data_ptr(), k_idx.data_ptr(), H_I, d_I,
                                      seq_lens.data_ptr(), k, out.data_ptr(), idx.data_ptr(), ws.data_ptr(), nbytes, sh)
    if rc:
        raise TopkAttnError("topk_indexer_attn_decode", rc)
    return out, idx
