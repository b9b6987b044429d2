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


def _run_bench(*args, env_extra=None):
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **(env_extra or {}))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], capture_output=True, text=True,
                       cwd=root, env=env, timeout=300)
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    return r.returncode, [json.loads(l) for l in lines]


def test_reference_arm_prints_one_contract_line():
    rc, out = _run_bench("--impl", "reference", "--config", "1", "--steps", "3", "--warmup", "3")
    assert rc == 0 and len(out) == 1
    r = out[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in r, key
    assert r["impl"] == "reference" and r["steps"] == 3 and r["warmup"] == 3 and r["value"] > 0
    assert r["config"]["workload"]
    assert {"value", "unit", "cores", "kind", "sample"} <= set(r["cpu_baseline"])
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["value"] == r["value"]
    assert r["e2e"] == {"value": r["value"], "unit": r["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    rc, out = _run_bench("--impl", "reference", "--config", "1", "--steps", "3", "--warmup", "3",
                         env_extra={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert rc == 0 and out == []


def test_too_few_warmup_steps_are_refused():
    rc, out = _run_bench("--impl", "reference", "--config", "1", "--steps", "3", "--warmup", "2")
    assert rc != 0 and out == []


def test_both_arms_describe_the_workload_with_one_config_object():
    # the reference arm prints exactly the config object the CUDA arm builds
    import argparse
    import workloads
    rc, out = _run_bench("--impl", "reference", "--config", "1", "--steps", "3", "--warmup", "3")
    assert rc == 0 and len(out) == 1
    w = workloads.config_workload(1, seed=1001)
    args = argparse.Namespace(certified_eps=None, paged=None, hisa=None, indexer=None)
    assert out[0]["config"] == bench.workload_config(w, w.k, 1, args)



def test_launch_accounting_of_the_five_workloads():
    # gpu_launches per step: the one-launch path takes workload 1 only (a
    # 4096-row cache); the MoBA selection fits one cluster launch
    import types

    import bench
    import workloads

    def shape(c):
        spec = dict(workloads.CONFIGS[c])
        return types.SimpleNamespace(B=spec["B"], Q=spec["Q"], Hq=spec["Hq"], Hkv=spec["Hkv"], L_max=spec["L_max"])

    one = {c: bench.one_launch(shape(c), 148) for c in (1, 2, 3, 5)}
    assert one == {1: True, 2: False, 3: False, 5: False}
    G4 = workloads.CONFIGS[4]["Hq"] // workloads.CONFIGS[4]["Hkv"]
    assert bench.block_select_launches(G4, workloads.CONFIGS[4]["L_max"] // workloads.CONFIGS[4]["block_size"]) == 1
    assert bench.block_select_launches(32, 131072 // 16) == 2
