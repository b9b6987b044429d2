"""Writes the stored expected values of tests/golden/ by calling only the oracle.

The pages print no worked example with numbers to reproduce ("A Mathematical
Theory of Top-k Sparse Attention via Total Variation Distance" states its
results as identities and bounds; the other pages give no numeric example of
the path), so the oracle is pinned by identities, closed forms, brute force
and planted mistakes in tests/test_oracle.py and tests/test_oracle_mutants.py.
The fixture written here is a regression record of the pinned oracle on small
seeded inputs: tests/test_golden.py checks that the oracle still reproduces it
exactly, so any later change of the oracle's arithmetic shows up and has to be
justified by a passage of the pages.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402

# (name, workload arguments, k, extra): small enough to read by eye; the
# record keeps every index and tail mass and the first 16 output dims of a row
CASES = [
    ("token_bf16_gqa", dict(B=1, Q=1, Hq=4, Hkv=2, L_max=40, dtype="bf16", d=128, seq_lens=[40], seed=11), 5, {}),
    ("token_bf16_ragged", dict(B=2, Q=1, Hq=2, Hkv=1, L_max=24, dtype="bf16", d=128, seq_lens=[24, 9], seed=12), 12,
     {}),
    ("token_f32_causal", dict(B=1, Q=3, Hq=2, Hkv=2, L_max=16, dtype="f32", d=128, seq_lens=[16], seed=13), 4, {}),
    ("block_bf16", dict(B=1, Q=1, Hq=2, Hkv=1, L_max=64, dtype="bf16", d=128, seq_lens=[61], seed=14), None,
     dict(block_size=8, top_blocks=3)),
]


def compute(case):
    name, args, k, extra = case
    w = workloads.make_workload(**args)
    if extra:
        r = oracle.block_attn(w, extra["block_size"], extra["top_blocks"])
        return {"out16": r["out"][..., :16].ravel().tolist(), "block_idx": r["block_idx"].ravel().tolist()}
    r = oracle.topk_attn(w, k)
    return {"out16": r["out"][..., :16].ravel().tolist(), "idx": r["idx"].ravel().tolist(),
            "tail": r["tail"].ravel().tolist()}


def main():
    data = {name: {"args": args, "k": k, "extra": extra, "expected": compute((name, args, k, extra))}
            for name, args, k, extra in CASES}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small_cases.json")
    with open(path, "w") as f:
        json.dump(data, f, indent=1)
        f.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
