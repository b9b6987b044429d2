"""The N > 1 path on CPU: two gloo ranks, as bench.py runs them on N GPUs.

The path shards by sequence with no exchange step (every (sequence, kv-head)
unit is independent), so a job of N ranks is N replicas on disjoint batches:
- each rank draws its own batch (bench.make_inputs seeds by rank);
- the oracle run on each rank's batch gives exactly the rows of one run over
  the concatenated batch (what sharding must preserve);
- the job's time is the slowest rank's (bench.reduce_over_ranks, a MAX
  all-reduce), and its value counts every rank's rows (bench.job_value).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.timeout(300)

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, errors):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD))
        torch.distributed.init_process_group("gloo", rank=rank, world_size=WORLD,
                                             timeout=datetime.timedelta(seconds=120))
        try:
            import bench
            import oracle
            import workloads

            # per-rank batches of the bench: same shapes, different draws
            w = bench.make_inputs(1, rank)
            sums = [None] * WORLD
            torch.distributed.all_gather_object(sums, (tuple(w.q.shape), float(w.q.double().sum())))
            assert sums[0][0] == sums[1][0] and sums[0][1] != sums[1][1]

            # sharded oracle runs == one run over the concatenated batch
            k = 24
            mine = workloads.make_workload(2, 1, 8, 2, 400, dtype="bf16", seq_lens=[400, 257], seed=300 + rank)
            res = oracle.topk_attn(mine, k)
            parts = [None] * WORLD
            torch.distributed.all_gather_object(parts, (mine, {n: res[n] for n in ("out", "idx", "tail")}))
            if rank == 0:
                ws = [p[0] for p in parts]
                full = workloads.make_workload(2 * WORLD, 1, 8, 2, 400, dtype="bf16", seed=1)
                full.q = torch.cat([x.q for x in ws])
                full.k_cache = torch.cat([x.k_cache for x in ws])
                full.v_cache = torch.cat([x.v_cache for x in ws])
                full.seq_lens = torch.cat([x.seq_lens for x in ws])
                ref = oracle.topk_attn(full, k)
                for n in ("out", "idx", "tail"):
                    got = np.concatenate([p[1][n] for p in parts])
                    assert np.array_equal(got, ref[n]), n

            # the job's time is the slowest rank's; its value counts every rank's rows
            vals = torch.tensor([10.0 + rank, 30.0 - rank, 5.0], dtype=torch.float64)
            bench.reduce_over_ranks(vals, WORLD)
            assert vals.tolist() == [11.0, 30.0, 5.0]
            assert bench.job_value(WORLD, 256, 0.5) == pytest.approx(2 * 256 / 0.5e-3)
            torch.distributed.barrier()
        finally:
            torch.distributed.destroy_process_group()
    except BaseException as e:  # reported to the parent
        errors.put(f"rank {rank}: {type(e).__name__}: {e}")
        raise


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    errors = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, errors)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(240)
    for p in procs:
        if p.is_alive():
            p.kill()
    msgs = []
    while not errors.empty():
        msgs.append(errors.get())
    assert not msgs, msgs
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
