"""fp64 CPU oracle for exact Top-k sparse decode attention -- TEST INFRASTRUCTURE.

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  The C source (``oracle.c``) is a plain, slow,
obviously correct restatement of the method; it shares no code with the CUDA
library.  ``build()`` compiles it with gcc + OpenMP into ``_oracle.so``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "_oracle.so")
_lib = None

_dp = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_ip = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p
_i = ctypes.c_int
_d = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile oracle.c (gcc -O2 -fopenmp, IEEE semantics) into _oracle.so.

    ORACLE_LIB_OVERRIDE names another build of the same source to load instead
    (the mutation test uses it to load copies with planted mistakes).
    """
    override = os.environ.get("ORACLE_LIB_OVERRIDE")
    if override:
        return override
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
                               "-Wall", "-Werror", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_max_threads.restype = _i
        lib.oracle_row_scores.argtypes = [_i] * 7 + [_d, _vp, _vp, _ip, _i, _i, _i, _dp]
        lib.oracle_row_scores.restype = _i
        lib.oracle_topk_attn.argtypes = [_i] * 7 + [_d, _vp, _vp, _vp, _ip, _i, _dp, _ip, _dp, _dp, _i]
        lib.oracle_topk_attn.restype = _i
        lib.oracle_certified_attn.argtypes = [_i] * 7 + [_d, _vp, _vp, _vp, _ip, _d, _i, _dp, _ip, _dp, _ip, _i]
        lib.oracle_certified_attn.restype = _i
        lib.oracle_hisa_attn.argtypes = [_i] * 6 + [_d, _vp, _vp, _vp, _ip, _i, _i, _i, _dp, _ip, _ip, _dp, _i]
        lib.oracle_hisa_attn.restype = _i
        lib.oracle_indexer_attn.argtypes = [_i] * 7 + [_d, _vp, _vp, _vp, _ip, _i, _i, _vp,
                                                       np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS"),
                                                       _vp, _i, _dp, _ip, _dp, _i]
        lib.oracle_indexer_attn.restype = _i
        lib.oracle_block_pool.argtypes = [_i] * 5 + [_vp, _ip, _i, _dp]
        lib.oracle_block_pool.restype = _i
        lib.oracle_block_attn.argtypes = [_i] * 6 + [_d, _vp, _vp, _vp, _ip, _i, _i, _dp, _ip, _dp, _dp, _i]
        lib.oracle_block_attn.restype = _i
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _code(dtype: str) -> int:
    return {"f32": 0, "bf16": 1}[dtype]


def _arr(w, t):
    return np.ascontiguousarray(w.raw(t))


def _lens(w):
    return np.ascontiguousarray(w.seq_lens.numpy().astype(np.int32))


def topk_attn(w, k: int, scale: float = 0.0, nthreads: int = 0) -> dict:
    """Exact Top-k decode attention over every row of workload ``w``.

    Returns out [B,Q,Hq,d] f64, idx [B,Q,Hq,k] int32 (ascending, -1 padded),
    tail [B,Q,Hq] f64 (discarded softmax mass) and kth [B,Q,Hq] f64 (the
    smallest kept score).  scale 0 means 1/sqrt(d).
    """
    lib = _load()
    q, kc, vc, lens = _arr(w, w.q), _arr(w, w.k_cache), _arr(w, w.v_cache), _lens(w)
    out = np.zeros((w.B, w.Q, w.Hq, w.d), np.float64)
    idx = np.zeros((w.B, w.Q, w.Hq, k), np.int32)
    tail = np.zeros((w.B, w.Q, w.Hq), np.float64)
    kth = np.zeros((w.B, w.Q, w.Hq), np.float64)
    rc = lib.oracle_topk_attn(w.B, w.Q, w.Hq, w.Hkv, w.d, w.L_max, _code(w.dtype), scale,
                              q.ctypes.data, kc.ctypes.data, vc.ctypes.data, lens, k,
                              out, idx, tail, kth, nthreads)
    if rc:
        raise ValueError(f"oracle_topk_attn failed with code {rc}")
    return dict(out=out, idx=idx, tail=tail, kth=kth)


def certified_attn(w, eps: float, k_max: int, scale: float = 0.0, nthreads: int = 0) -> dict:
    """Certified adaptive Top-k decode attention over every row of ``w``.

    Per row the smallest k (at most min(k_max, vis)) whose discarded softmax
    tail mass is <= eps.  Returns out [B,Q,Hq,d] f64, idx [B,Q,Hq,k_max]
    int32 (ascending, -1 padded), tail [B,Q,Hq] f64 and k_used [B,Q,Hq] int32.
    """
    lib = _load()
    q, kc, vc, lens = _arr(w, w.q), _arr(w, w.k_cache), _arr(w, w.v_cache), _lens(w)
    out = np.zeros((w.B, w.Q, w.Hq, w.d), np.float64)
    idx = np.zeros((w.B, w.Q, w.Hq, k_max), np.int32)
    tail = np.zeros((w.B, w.Q, w.Hq), np.float64)
    k_used = np.zeros((w.B, w.Q, w.Hq), np.int32)
    rc = lib.oracle_certified_attn(w.B, w.Q, w.Hq, w.Hkv, w.d, w.L_max, _code(w.dtype), scale,
                                   q.ctypes.data, kc.ctypes.data, vc.ctypes.data, lens, eps, k_max,
                                   out, idx, tail, k_used, nthreads)
    if rc:
        raise ValueError(f"oracle_certified_attn failed with code {rc}")
    return dict(out=out, idx=idx, tail=tail, k_used=k_used)


def row_scores(w, b: int, qpos: int, h: int, scale: float = 0.0) -> np.ndarray:
    """fp64 scores of one row over its visible keys."""
    lib = _load()
    q, kc, lens = _arr(w, w.q), _arr(w, w.k_cache), _lens(w)
    s = np.zeros(w.L_max, np.float64)
    vis = lib.oracle_row_scores(w.B, w.Q, w.Hq, w.Hkv, w.d, w.L_max, _code(w.dtype), scale,
                                q.ctypes.data, kc.ctypes.data, lens, b, qpos, h, s)
    if vis < 0:
        raise ValueError("bad row")
    return s[:vis].copy()


def block_pool(w, block_size: int) -> np.ndarray:
    """Mean-pooled block keys [B, Hkv, ceil(L_max/bs), d] in fp64."""
    lib = _load()
    kc, lens = _arr(w, w.k_cache), _lens(w)
    nblk = (w.L_max + block_size - 1) // block_size
    bk = np.zeros((w.B, w.Hkv, nblk, w.d), np.float64)
    rc = lib.oracle_block_pool(w.B, w.Hkv, w.d, w.L_max, _code(w.dtype), kc.ctypes.data, lens,
                               block_size, bk)
    if rc:
        raise ValueError(f"oracle_block_pool failed with code {rc}")
    return bk


def block_attn(w, block_size: int, top_blocks: int, scale: float = 0.0, nthreads: int = 0) -> dict:
    """MoBA block-sparse decode attention (one query per sequence).

    Returns out [B,1,Hq,d], block_idx [B,1,Hq,top_blocks+1] (ascending, -1
    padded), tail [B,1,Hq] (softmax mass outside the kept blocks) and kth
    [B,1,Hq] (smallest kept competing block score, -inf if all kept).
    """
    if w.Q != 1:
        raise ValueError("the block variant takes one query position per sequence")
    lib = _load()
    q, kc, vc, lens = _arr(w, w.q), _arr(w, w.k_cache), _arr(w, w.v_cache), _lens(w)
    out = np.zeros((w.B, 1, w.Hq, w.d), np.float64)
    bidx = np.zeros((w.B, 1, w.Hq, top_blocks + 1), np.int32)
    tail = np.zeros((w.B, 1, w.Hq), np.float64)
    kth = np.zeros((w.B, 1, w.Hq), np.float64)
    rc = lib.oracle_block_attn(w.B, w.Hq, w.Hkv, w.d, w.L_max, _code(w.dtype), scale,
                               q.ctypes.data, kc.ctypes.data, vc.ctypes.data, lens,
                               block_size, top_blocks, out, bidx, tail, kth, nthreads)
    if rc:
        raise ValueError(f"oracle_block_attn failed with code {rc}")
    return dict(out=out, block_idx=bidx, tail=tail, kth=kth)


def hisa_attn(w, block_size: int, top_blocks: int, k: int, scale: float = 0.0, nthreads: int = 0) -> dict:
    """Hierarchical block -> token Top-k decode attention (one query per sequence).

    Returns out [B,1,Hq,d] f64, block_idx [B,1,Hq,top_blocks] and idx [B,1,Hq,k]
    (ascending, -1 padded) and tail [B,1,Hq] (discarded mass among the candidates).
    """
    if w.Q != 1:
        raise ValueError("one query position per sequence")
    lib = _load()
    q, kc, vc, lens = _arr(w, w.q), _arr(w, w.k_cache), _arr(w, w.v_cache), _lens(w)
    out = np.zeros((w.B, 1, w.Hq, w.d), np.float64)
    bidx = np.zeros((w.B, 1, w.Hq, top_blocks), np.int32)
    idx = np.zeros((w.B, 1, w.Hq, k), np.int32)
    tail = np.zeros((w.B, 1, w.Hq), np.float64)
    rc = lib.oracle_hisa_attn(w.B, w.Hq, w.Hkv, w.d, w.L_max, _code(w.dtype), scale,
                              q.ctypes.data, kc.ctypes.data, vc.ctypes.data, lens,
                              block_size, top_blocks, k, out, bidx, idx, tail, nthreads)
    if rc:
        raise ValueError(f"oracle_hisa_attn failed with code {rc}")
    return dict(out=out, block_idx=bidx, idx=idx, tail=tail)


def indexer_attn(w, q_idx, w_idx, k_idx, k: int, scale: float = 0.0, nthreads: int = 0) -> dict:
    """Token selection by a lightning indexer, then exact attention per head.

    q_idx [B,Q,H_I,d_I] and k_idx [B,L_max,d_I] in the cache dtype (torch
    tensors), w_idx [B,Q,H_I] fp32.  Returns out [B,Q,Hq,d] f64, idx [B,Q,k]
    (ascending, -1 padded, shared by all heads of a query position) and kth
    [B,Q] (the smallest kept indexer score).
    """
    lib = _load()
    B, Q, H_I, d_I = q_idx.shape
    q, kc, vc, lens = _arr(w, w.q), _arr(w, w.k_cache), _arr(w, w.v_cache), _lens(w)
    qi, ki = _arr(w, q_idx), _arr(w, k_idx)
    wi = np.ascontiguousarray(w_idx.numpy().astype(np.float32))
    out = np.zeros((w.B, w.Q, w.Hq, w.d), np.float64)
    idx = np.zeros((w.B, w.Q, k), np.int32)
    kth = np.zeros((w.B, w.Q), np.float64)
    rc = lib.oracle_indexer_attn(w.B, w.Q, w.Hq, w.Hkv, w.d, w.L_max, _code(w.dtype), scale,
                                 q.ctypes.data, kc.ctypes.data, vc.ctypes.data, lens, H_I, d_I,
                                 qi.ctypes.data, wi, ki.ctypes.data, k, out, idx, kth, nthreads)
    if rc:
        raise ValueError(f"oracle_indexer_attn failed with code {rc}")
    return dict(out=out, idx=idx, kth=kth)
