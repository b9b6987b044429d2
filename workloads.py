"""Seeded synthetic decode workloads: the only code shared by the oracle side
and the CUDA side.

This module draws random numbers and lays them out; it holds none of the
attention arithmetic (no scores, no selection, no softmax).  Every tensor is
drawn in fp32 from numpy's PCG64, one independent stream per
(tensor, batch, kv-head) slab keyed by ``SeedSequence([seed, tensor, b, h])``,
so a slab's values do not depend on how many threads generated it.  bf16
workloads are rounded once, round-to-nearest-even, and both sides read the
identical rounded values.

Layouts (row-major, contiguous):
  q        [B, Q, Hq, d]
  k_cache  [B, Hkv, L_max, d]
  v_cache  [B, Hkv, L_max, d]
  seq_lens int32 [B]
Cache rows at positions >= seq_lens[b] are filled with NaN so that a kernel
that reads past a sequence's end poisons its output.

The five named workloads follow the decode settings of the pages: a
single-head fp32 case, a Llama-3-8B-shaped GQA layer at 32K context with
k = 2048 (the fixed Top-K budget the Baidu articles quote), a 128K-context
case with planted retrieval keys, a MoBA-style block-sparse case
("Sparse Attention Landscape", block-sparse attention / MoBA) and a 16-query
causal chunk.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch

# stream ids inside a seed
_T_Q, _T_K, _T_V, _T_KMEAN, _T_PLANT_POS, _T_PLANT_NOISE, _T_SEQ, _T_IQ, _T_IW, _T_IK = range(10)


@dataclass
class Workload:
    name: str
    B: int
    Q: int
    Hq: int
    Hkv: int
    d: int
    L_max: int
    dtype: str                      # "f32" | "bf16"
    q: torch.Tensor                 # [B,Q,Hq,d]
    k_cache: torch.Tensor           # [B,Hkv,L_max,d]
    v_cache: torch.Tensor           # [B,Hkv,L_max,d]
    seq_lens: torch.Tensor          # int32 [B]
    k: Optional[int] = None         # token Top-k budget (token variant)
    block_size: Optional[int] = None
    top_blocks: Optional[int] = None
    variant: str = "token"          # "token" | "block"
    seed: int = 0
    recipe: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def raw(self, t: torch.Tensor) -> np.ndarray:
        """Numpy view of a tensor's storage: uint16 bits for bf16, float32 otherwise."""
        if t.dtype == torch.bfloat16:
            return t.contiguous().view(torch.int16).numpy().view(np.uint16)
        return t.contiguous().numpy()


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *key])))


def _normal(seed: int, key: Sequence[int], n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _rng(seed, *key).standard_normal(out=out, dtype=np.float32)
    return out


def _to_dtype(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(x)
    return t.to(torch.bfloat16) if dtype == "bf16" else t.clone()


def _torch_dtype(dtype: str) -> torch.dtype:
    if dtype == "bf16":
        return torch.bfloat16
    if dtype == "f32":
        return torch.float32
    raise ValueError(f"unknown dtype {dtype!r}")


def _threads() -> int:
    return max(1, min(16, len(os.sched_getaffinity(0))))


def make_workload(
    B: int,
    Q: int,
    Hq: int,
    Hkv: int,
    L_max: int,
    dtype: str = "bf16",
    d: int = 128,
    seq_lens: Optional[Sequence[int]] = None,
    seq_len_range: Optional[tuple] = None,
    k_mean_std: float = 0.0,
    plant_count: int = 0,
    plant_scale: Optional[float] = None,
    plant_noise: float = 0.1,
    seed: int = 0,
    k: Optional[int] = None,
    block_size: Optional[int] = None,
    top_blocks: Optional[int] = None,
    name: str = "custom",
) -> Workload:
    """Draw one workload.

    seq_lens / seq_len_range: explicit lengths, or integers uniform on the
      inclusive range; default every sequence full (L_max).
    k_mean_std: one random mean vector per (b, kv-head), entries N(0, std^2),
      added to every key of that head (the "per-head random mean offset").
    plant_count / plant_scale / plant_noise: per (b, kv-head), that many
      distinct positions uniform on [0, L_b) get key = plant_scale * 4 * u + eps,
      u the unit vector of the mean of the group's query vectors (all Q
      positions), eps ~ N(0, plant_noise^2).  plant_scale None means sqrt(d).
    """
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    tdt = _torch_dtype(dtype)
    G = Hq // Hkv
    if seq_lens is not None:
        lens = np.asarray(list(seq_lens), dtype=np.int64)
    elif seq_len_range is not None:
        lo, hi = seq_len_range
        lens = _rng(seed, _T_SEQ).integers(lo, hi, size=B, endpoint=True)
    else:
        lens = np.full(B, L_max, dtype=np.int64)
    if lens.shape != (B,) or (lens < 1).any() or (lens > L_max).any():
        raise ValueError("seq_lens must be B values in [1, L_max]")

    qf = np.empty((B, Q, Hq, d), dtype=np.float32)
    for b in range(B):
        qf[b] = _normal(seed, (_T_Q, b), Q * Hq * d).reshape(Q, Hq, d)
    q = _to_dtype(qf, dtype)

    k_cache = torch.empty((B, Hkv, L_max, d), dtype=tdt)
    v_cache = torch.empty((B, Hkv, L_max, d), dtype=tdt)
    if plant_scale is None:
        plant_scale = math.sqrt(d)

    def slab(job):
        b, h = job
        Lb = int(lens[b])
        kf = _normal(seed, (_T_K, b, h), Lb * d).reshape(Lb, d)
        vf = _normal(seed, (_T_V, b, h), Lb * d).reshape(Lb, d)
        if k_mean_std:
            kf += np.float32(k_mean_std) * _normal(seed, (_T_KMEAN, b, h), d)[None, :]
        if plant_count:
            pos = _rng(seed, _T_PLANT_POS, b, h).choice(Lb, size=min(plant_count, Lb), replace=False)
            qg = qf[b, :, h * G:(h + 1) * G, :].reshape(-1, d).astype(np.float64).mean(axis=0)
            u = qg / np.linalg.norm(qg)
            noise = _normal(seed, (_T_PLANT_NOISE, b, h), len(pos) * d).reshape(len(pos), d)
            kf[pos] = (plant_scale * 4.0 * u)[None, :].astype(np.float32) + np.float32(plant_noise) * noise
        k_cache[b, h, :Lb] = _to_dtype(kf, dtype)
        v_cache[b, h, :Lb] = _to_dtype(vf, dtype)
        if Lb < L_max:
            k_cache[b, h, Lb:] = float("nan")
            v_cache[b, h, Lb:] = float("nan")

    jobs = [(b, h) for b in range(B) for h in range(Hkv)]
    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(slab, jobs))

    recipe = dict(k_mean_std=k_mean_std, plant_count=plant_count,
                  plant_scale=float(plant_scale) if plant_count else None,
                  plant_noise=plant_noise if plant_count else None,
                  seq_len_range=seq_len_range)
    return Workload(name=name, B=B, Q=Q, Hq=Hq, Hkv=Hkv, d=d, L_max=L_max, dtype=dtype,
                    q=q, k_cache=k_cache, v_cache=v_cache,
                    seq_lens=torch.from_numpy(lens.astype(np.int32)),
                    k=k, block_size=block_size, top_blocks=top_blocks,
                    variant="block" if block_size else "token", seed=seed, recipe=recipe)


# The five decode workloads.  Head counts are 32 query / 8 KV heads, so each
# KV head serves a GQA group of 4 query heads.
CONFIGS = {
    1: dict(name="single_head_f32_L4096_k64", B=1, Q=1, Hq=1, Hkv=1, L_max=4096, dtype="f32", k=64),
    2: dict(name="llama3_8b_gqa_bf16_B8_L32768_k2048", B=8, Q=1, Hq=32, Hkv=8, L_max=32768,
            dtype="bf16", k=2048, k_mean_std=0.5),
    3: dict(name="planted_retrieval_bf16_B4_L131072_k2048", B=4, Q=1, Hq=32, Hkv=8, L_max=131072,
            dtype="bf16", k=2048, seq_len_range=(65536, 131072), plant_count=16),
    4: dict(name="moba_block_bf16_B8_L65536_bs64_top16", B=8, Q=1, Hq=32, Hkv=8, L_max=65536,
            dtype="bf16", block_size=64, top_blocks=16),
    5: dict(name="causal_chunk_bf16_B2_Q16_L65536_k1024", B=2, Q=16, Hq=32, Hkv=8, L_max=65536,
            dtype="bf16", k=1024),
}


def config_workload(cfg_id: int, seed: Optional[int] = None, plant_scale: Optional[float] = None,
                    **overrides) -> Workload:
    """One of the five named workloads, seed 1000 + id unless given.

    ``overrides`` replace fields of the recipe (e.g. a smaller B or L_max for a
    quick case); the planted-key scale of workload 3 defaults to sqrt(d)
    (pass plant_scale=1.0 for the literal 4 x unit-direction reading).
    """
    spec = dict(CONFIGS[cfg_id])
    spec.update(overrides)
    if plant_scale is not None:
        spec["plant_scale"] = plant_scale
    if seed is None:
        seed = 1000 + cfg_id
    return make_workload(seed=seed, **spec)


def make_indexer_inputs(w: "Workload", H_I: int = 16, d_I: int = 128, seed: Optional[int] = None):
    """Synthetic lightning-indexer inputs for workload ``w``: projected indexer
    queries q_idx [B, Q, H_I, d_I] and keys k_idx [B, L_max, d_I] (N(0, 1),
    rounded to the cache dtype; keys past a sequence's end NaN) and head
    weights w_idx [B, Q, H_I] (uniform on [0, 1), fp32).  No trained weights
    exist here: the inputs have the shapes, not the statistics, of a trained
    indexer."""
    seed = w.seed if seed is None else seed
    qi = np.stack([_normal(seed, (_T_IQ, b), w.Q * H_I * d_I).reshape(w.Q, H_I, d_I) for b in range(w.B)])
    wi = np.stack([_rng(seed, _T_IW, b).random((w.Q, H_I), dtype=np.float32) for b in range(w.B)])
    ki = np.stack([_normal(seed, (_T_IK, b), w.L_max * d_I).reshape(w.L_max, d_I) for b in range(w.B)])
    q_idx = _to_dtype(np.ascontiguousarray(qi), w.dtype)
    k_idx = _to_dtype(np.ascontiguousarray(ki), w.dtype)
    for b in range(w.B):
        Lb = int(w.seq_lens[b])
        if Lb < w.L_max:
            k_idx[b, Lb:] = float("nan")
    return q_idx, torch.from_numpy(np.ascontiguousarray(wi)), k_idx
