"""bench.py's host-side arithmetic, on CPU."""
import types

import numpy as np
import torch

import bench


def test_unique_kept_rows_counts_each_position_once_per_kv_head():
    # B=2, Q=2, Hq=4, Hkv=2 (G=2), k=3; -1 padding is not a row
    w = types.SimpleNamespace(B=2, Q=2, Hq=4, Hkv=2)
    rng = np.random.default_rng(0)
    idx = rng.integers(-1, 6, size=(2, 2, 4, 3)).astype(np.int32)
    want = 0
    for b in range(2):
        for kvh in range(2):
            heads = range(kvh * 2, kvh * 2 + 2)
            s = {int(x) for q in range(2) for h in heads for x in idx[b, q, h] if x >= 0}
            want += len(s)
    assert bench.unique_kept_rows(torch.from_numpy(idx), w) == want


def test_unique_bytes_never_exceed_the_formula_bytes():
    w = types.SimpleNamespace(B=1, Q=1, Hq=4, Hkv=1, d=128, dtype="bf16", seq_lens=torch.tensor([100]))
    idx = torch.arange(4 * 8, dtype=torch.int32).view(1, 1, 4, 8) % 10  # heavy overlap between heads
    u = bench.unique_kept_rows(idx, w)
    assert u == 10
    assert bench.alg_bytes_unique(w, 8, u) < bench.alg_bytes_token(w, 8, kept=4 * 8)
