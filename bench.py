#!/usr/bin/env python
"""Benchmark of exact Top-k sparse decode attention on B200.

One step = one decode call over one batch of synthetic input: score every
cached key, select the top k per query head, softmax over the kept keys,
gather P.V, tail mass (token variant, workloads 1/2/3/5), or block select +
attention over kept blocks (workload 4).  The default workload is the
Llama-3-8B-shaped GQA decode layer: B=8, 32 query / 8 KV heads, d=128,
L=32768, k=2048, bf16 cache.

Prints ONE JSON line (rank 0).  Timing: W untimed warm-up steps, then exactly
K timed steps of plain API calls, each bracketed by CUDA events on the
launching stream, with an L2 flush between steps outside the events (a 256 MiB
write, then a 256 MiB read, so that no dirty line of the flush buffer is left
in L2 to be written back inside the timed region); the sum of the K step
times, max over ranks, gives `value`.  The token variant then times a second
pass of K steps with events between its three kernels (`stage_us`, and the
score kernel's roofline).  `e2e` repeats the K steps through the public API
with the step's inputs copied from pinned host memory and its results copied
back inside the events (idx on a side stream while the gather runs).
Multi-GPU (torchrun) runs one independent replica per GPU (the path shards by
sequence with no exchange): weak scaling.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1..5] [--impl ours|reference]
                  [--certified-eps E | --paged P | --hisa BS,TOP | --indexer H_I,D_I]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "Top-k decode attention queries/s and achieved HBM GB/s vs B200 peak, L=32K–128K"
UNIT = "queries/s"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0
L2_FLUSH_BYTES = 256 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (smaller cases for profiling)")
    ap.add_argument("--paged", type=int, default=None, metavar="PAGE_SIZE",
                    help="lay the cache out as shuffled pages of PAGE_SIZE positions (block tables)")
    ap.add_argument("--indexer", type=str, default=None, metavar="H_I,D_I",
                    help="lightning-indexer token selection with H_I indexer heads of D_I dims "
                         "(synthetic indexer inputs)")
    ap.add_argument("--hisa", type=str, default=None, metavar="BLOCK_SIZE,TOP_BLOCKS",
                    help="hierarchical block -> token Top-k: score only the tokens of the best TOP_BLOCKS "
                         "blocks of BLOCK_SIZE (one-query workloads)")
    ap.add_argument("--certified-eps", type=float, default=None,
                    help="certified adaptive Top-k: per row the smallest k (at most the workload's k) "
                         "whose discarded tail mass is <= EPS")
    return ap.parse_args()


# ----------------------------------------------------------------------------- accounting

def elem_bytes(w):
    return 2 if w.dtype == "bf16" else 4


def visible(w, b, qp):
    return int(w.seq_lens[b]) - w.Q + qp + 1


def k_bytes(w):
    """Whole K cache read once: every kv-head's rows below its sequence length."""
    return sum(int(w.seq_lens[b]) for b in range(w.B)) * w.Hkv * w.d * elem_bytes(w)


def alg_bytes_token(w, k, kept=None):
    """Algorithmic bytes of one step: full K read + the k kept K and V rows of
    every query row (or `kept` rows in total) + q, out, idx and tail."""
    row = w.d * elem_bytes(w)
    if kept is None:
        kept = sum(min(k, visible(w, b, qp)) for b in range(w.B) for qp in range(w.Q)) * w.Hq
    rows = w.B * w.Q * w.Hq
    return k_bytes(w) + kept * 2 * row + rows * w.d * (elem_bytes(w) + 4) + rows * (k * 4 + 4)


def unique_kept_rows(idx, w):
    """Kept positions counted once per (sequence, kv-head): the union over the
    G heads and Q positions of the group (what the gather must read at least
    once; -1 padding excluded).  idx [B, Q, Hq, k] on the device."""
    k = idx.shape[-1]
    g = idx.view(w.B, w.Q, w.Hkv, w.Hq // w.Hkv, k).permute(0, 2, 1, 3, 4).reshape(w.B * w.Hkv, -1)
    srt = torch.sort(g, dim=1).values
    new = torch.ones_like(srt, dtype=torch.bool)
    new[:, 1:] = srt[:, 1:] != srt[:, :-1]
    return int((new & (srt >= 0)).sum())


def alg_bytes_unique(w, k, uniq_rows):
    """The stricter algorithmic bytes: K once + every unique kept V row once + q, out, idx and tail."""
    rows = w.B * w.Q * w.Hq
    return k_bytes(w) + uniq_rows * w.d * elem_bytes(w) + rows * w.d * (elem_bytes(w) + 4) + rows * (k * 4 + 4)


def alg_bytes_block(w):
    """Block keys (fp32) of every competing block + the kept blocks' K and V rows + q/out/block_idx."""
    bs, top = w.block_size, w.top_blocks
    total = 0
    for b in range(w.B):
        Lb = int(w.seq_lens[b])
        nblk = -(-Lb // bs)
        comp = nblk - 1
        total += w.Hkv * comp * w.d * 4
        kept_tokens = min(top, comp) * bs + (Lb - (nblk - 1) * bs)
        total += w.Hq * kept_tokens * 2 * w.d * elem_bytes(w)
    rows = w.B * w.Hq
    return total + rows * w.d * (elem_bytes(w) + 4) + rows * (top + 1) * 4


def one_launch(w, num_sms):
    """Whether the library decodes this token workload in one launch (a small
    cache: at most 65536 rows in all, no more query rows or kv-heads than SMs,
    at most 64 query rows per kv-head)."""
    rows, units = w.B * w.Q * w.Hq, w.B * w.Hkv
    return w.B * w.Hkv * w.L_max <= 65536 and rows <= num_sms and units <= num_sms and w.Q * (w.Hq // w.Hkv) <= 64


def block_select_launches(G, nblk_max):
    """Kernels the block selection takes: one on a cluster of 8 CTAs per
    (sequence, kv-head) when a kv-head's block scores fit its shared memory
    (96 KB: queries, G chunks of scores, one head's gathered scores and keys),
    else block scores + one top-k CTA per row."""
    chmax = -(-nblk_max // 8)
    return 1 if G * 32 * 16 + G * chmax * 4 + nblk_max * 8 <= 96 * 1024 else 2


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def score_traffic(source_file):
    """dram bytes per launch of the score kernel from the committed ncu summary,
    if it was taken from the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "score_bf16_llama3_8b_L32768.txt")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_b = re.search(r"^dram_bytes_per_launch_full_workload:\s*([0-9.eE+]+)", text, re.M)
    m_h = re.search(r"^kernel_source_sha256:\s*([0-9a-f]+)", text, re.M)
    if not m_b or not m_h:
        return None
    src = hashlib.sha256(open(source_file, "rb").read()).hexdigest()
    return float(m_b.group(1)) if src == m_h.group(1) else None


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index, period=0.005):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._nv:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- CPU oracle

def time_oracle(w, k, budget_s=10.0, max_reps=50, eps=None, nthreads=0):
    """The oracle as it stands on this host's cores (nthreads = 0: all of
    them), whole workload repeated until `budget_s` has elapsed (at least
    once).  Returns (queries/s, threads used, sample text)."""
    import oracle
    rows = w.B * w.Q * w.Hq
    reps, t0 = 0, time.perf_counter()
    while True:
        if w.variant == "block":
            oracle.block_attn(w, w.block_size, w.top_blocks, nthreads=nthreads)
        elif eps is not None:
            oracle.certified_attn(w, eps, k, nthreads=nthreads)
        else:
            oracle.topk_attn(w, k, nthreads=nthreads)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s or reps >= max_reps:
            break
    sample = f"whole workload ({rows} query rows) x {reps} repetitions, {dt:.1f} s"
    return rows * reps / dt, (nthreads or oracle.max_threads()), sample


def workload_config(w, k, world, args):
    """The `config` object of the JSON line: the same for both arms."""
    certified = args.certified_eps is not None and w.variant != "block"
    paged = args.paged is not None and w.variant != "block" and not certified
    hisa = args.hisa is not None and w.variant != "block" and not certified and not paged
    indexer = args.indexer is not None and w.variant != "block" and not certified and not paged and not hisa
    cfg = {
        "workload": w.name, "B": w.B, "Q": w.Q, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "L_max": w.L_max,
        "k": k, "block_size": w.block_size, "top_blocks": w.top_blocks,
        "seq_lens": "full" if int(w.seq_lens.min()) == w.L_max else [int(x) for x in w.seq_lens],
        "accumulate": "fp32", "parallelism": f"replica x{world} (independent sequences per GPU)",
        "l2": "flushed between timed steps (256 MiB write + 256 MiB read, outside the timed events)",
    }
    if certified:
        cfg.update({"certified_eps": args.certified_eps, "k_max": k})
    if paged:
        cfg.update({"page_size": args.paged, "pages": "shuffled pool, block tables"})
    if hisa:
        h_bs, h_top = (int(x) for x in args.hisa.split(","))
        cfg.update({"hisa_block_size": h_bs, "hisa_top_blocks": h_top})
    if indexer:
        i_h, i_d = (int(x) for x in args.indexer.split(","))
        cfg.update({"indexer_heads": i_h, "indexer_dims": i_d, "indexer_inputs": "synthetic"})
    return cfg


# ----------------------------------------------------------------------------- runs

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def reduce_over_ranks(vals, world):
    """Max over ranks of each entry of vals (timings: the slowest rank sets the job's time)."""
    if world > 1:
        torch.distributed.all_reduce(vals, op=torch.distributed.ReduceOp.MAX)
    return vals


def job_value(world, rows_per_rank, ms_per_step):
    """Whole-job throughput: the query rows of every rank over the slowest rank's step time."""
    return world * rows_per_rank / (ms_per_step / 1e3)


def make_inputs(cfg, rank, batch=None):
    # each rank decodes its own batch (weak scaling); rank 0 draws the tested workload
    over = {} if batch is None else {"B": batch}
    return workloads.config_workload(cfg, seed=1000 + cfg + 7919 * rank, **over)


def page_cache(kc, vc, page_size, rank):
    """The contiguous caches [B, Hkv, L, d] as shuffled pages [num_pages, Hkv, page_size, d] and
    the block table [B, L / page_size] that maps them back."""
    B, Hkv, L, d = kc.shape
    if L % page_size:
        raise SystemExit("--paged: the page size must divide L_max")
    npg = L // page_size
    g = torch.Generator(device=kc.device).manual_seed(4242 + rank)
    perm = torch.randperm(B * npg, generator=g, device=kc.device)
    pages = []
    for c in (kc, vc):
        p = c.reshape(B, Hkv, npg, page_size, d).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, page_size, d)
        out = torch.empty_like(p)
        out[perm] = p
        pages.append(out)
    table = perm.reshape(B, npg).to(torch.int32).contiguous()
    return pages[0], pages[1], table


def run_ours(args, world, rank, local):
    import exact_top_sparse_score_b200 as tka
    from exact_top_sparse_score_b200._binding import block_attn_workspace_size, make_shape

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = make_inputs(args.config, rank, args.batch)
    q, kc, vc, lens = (w.q.to(dev), w.k_cache.to(dev), w.v_cache.to(dev), w.seq_lens.to(dev))
    rows = w.B * w.Q * w.Hq
    block = w.variant == "block"
    certified = args.certified_eps is not None and not block
    paged = args.paged is not None and not block and not certified
    hisa = args.hisa is not None and not block and not certified and not paged
    indexer = args.indexer is not None and not block and not certified and not paged and not hisa
    if indexer:
        i_h, i_d = (int(x) for x in args.indexer.split(","))
        i_q, i_w, i_k = (t.to(dev) for t in workloads.make_indexer_inputs(w, i_h, i_d))
    if hisa:
        h_bs, h_top = (int(x) for x in args.hisa.split(","))
    k = w.k
    if block:
        bk = tka.topk_block_pool_keys(kc, lens, w.block_size)
        ws = torch.empty(block_attn_workspace_size(make_shape(q, kc), w.block_size, w.top_blocks),
                         dtype=torch.uint8, device=dev)
        out = torch.empty((w.B, w.Q, w.Hq, w.d), dtype=torch.float32, device=dev)
        bidx = torch.empty((w.B, w.Q, w.Hq, w.top_blocks + 1), dtype=torch.int32, device=dev)
        launches_per_step = block_select_launches(w.G, -(-w.L_max // w.block_size)) + 1  # + block_attn

        def step(events=None, qq=q):
            if events:
                events[0].record()
            tka.topk_block_attn_decode(qq, kc, vc, bk, lens, w.block_size, w.top_blocks, out=out,
                                       block_idx=bidx, workspace=ws)
            if events:
                events[3].record()
        alg = alg_bytes_block(w)
        dominant_bytes = None
    else:
        ws = torch.empty(tka.topk_attn_workspace_size(make_shape(q, kc), k), dtype=torch.uint8, device=dev)
        out = torch.empty((w.B, w.Q, w.Hq, w.d), dtype=torch.float32, device=dev)
        idx = torch.empty((w.B, w.Q, w.Hq, k), dtype=torch.int32, device=dev)
        tail = torch.empty((w.B, w.Q, w.Hq), dtype=torch.float32, device=dev)
        launches_per_step = 1 if one_launch(w, torch.cuda.get_device_properties(dev).multi_processor_count) else 3
        if certified:
            k_used = torch.empty((w.B, w.Q, w.Hq), dtype=torch.int32, device=dev)
            launches_per_step = 4  # + certify

            def step(events=None, qq=q):
                if events:
                    events[0].record()
                tka.topk_attn_decode_certified(qq, kc, vc, lens, args.certified_eps, k, out=out, idx=idx,
                                               tail_mass=tail, k_used=k_used, workspace=ws)
                if events:
                    events[3].record()
        elif indexer:
            i_idx = torch.empty((w.B, w.Q, k), dtype=torch.int32, device=dev)
            ws = torch.empty(tka._binding.load_library().topk_indexer_attn_workspace_size(
                make_shape(q, kc), i_h, i_d, k), dtype=torch.uint8, device=dev)
            # 128-dim bf16 index keys: the tensor-core scorer + the weighted ReLU combine;
            # otherwise indexer_scores on CUDA cores; then select and indexer_attn
            launches_per_step = 4 if (i_d == 128 and w.dtype == "bf16" and w.Q * i_h <= 128) else 3

            def step(events=None, qq=q):
                if events:
                    events[0].record()
                tka.topk_indexer_attn_decode(qq, kc, vc, i_q, i_w, i_k, lens, k, out=out, idx=i_idx, workspace=ws)
                if events:
                    events[3].record()
        elif hisa:
            h_bk = tka.topk_block_pool_keys(kc, lens, h_bs)
            h_bidx = torch.empty((w.B, 1, w.Hq, h_top), dtype=torch.int32, device=dev)
            ws = torch.empty(tka._binding.load_library().topk_hisa_attn_workspace_size(
                make_shape(q, kc), h_bs, h_top, k), dtype=torch.uint8, device=dev)
            # block selection, hisa_scores, select, gather
            launches_per_step = block_select_launches(w.G, -(-w.L_max // h_bs)) + 3

            def step(events=None, qq=q):
                if events:
                    events[0].record()
                tka.topk_hisa_attn_decode(qq, kc, vc, h_bk, lens, h_bs, h_top, k, out=out, idx=idx,
                                          tail_mass=tail, block_idx=h_bidx, workspace=ws)
                if events:
                    events[3].record()
        elif paged:
            kp, vp, table = page_cache(kc, vc, args.paged, rank)
            launches_per_step = 3

            def step(events=None, qq=q):
                if events:
                    events[0].record()
                tka.topk_attn_decode_paged(qq, kp, vp, table, lens, k, out=out, idx=idx, tail_mass=tail,
                                           workspace=ws)
                if events:
                    events[3].record()
        else:
            def step(events=None, qq=q):
                if events:
                    events[0].record()
                tka.topk_attn_decode(qq, kc, vc, lens, k, out=out, idx=idx, tail_mass=tail, workspace=ws)
                if events:
                    events[3].record()

            def staged_step(events):
                # events between the kernels: the per-stage times (and no early
                # launch of a kernel behind the one before)
                tka.topk_attn_decode(q, kc, vc, lens, k, out=out, idx=idx, tail_mass=tail, workspace=ws,
                                     stage_events=events)
        alg = alg_bytes_token(w, k)
        dominant_bytes = k_bytes(w) + q.numel() * q.element_size()

    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def l2_flush():
        flush_w.zero_()  # evicts everything the step left in L2 ...
        flush_r.amax()   # ... and leaves only clean lines behind

    staged = not (block or certified or paged or hisa or indexer)
    for _ in range(args.warmup):
        step()
        if staged:
            # the stage-timed pass runs the three-kernel path, which a small
            # problem's plain call (one launch) does not: load its kernels too
            staged_step([None] * 4)
    torch.cuda.synchronize()
    if tka.topk_attn_device_status() != 0:
        raise RuntimeError("device status raised during warm-up")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    for e in (x for row in evs for x in row):
        e.record()  # torch creates the CUDA event on its first record
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sevs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)] if staged else []
    for e in (x for row in sevs for x in row):
        e.record()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(K):
            l2_flush()
            step(evs[i])
        torch.cuda.synchronize()
        if staged:
            # a second timed pass, same flushes, with events between the kernels
            for i in range(K):
                l2_flush()
                staged_step(sevs[i])
            torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = [e[0].elapsed_time(e[3]) for e in evs]
    stage_ms = [[e[j].elapsed_time(e[j + 1]) for e in sevs] for j in range(3)] if staged else None
    total_ms = sum(step_ms)

    e2e_ms = None
    h2d = d2h = 0
    if not args.no_e2e:
        # public API with host buffers: H2D of the step's queries and lengths
        # from pinned memory, D2H of every result, all inside the events
        q_host = w.q.pin_memory()
        lens_host = w.seq_lens.pin_memory()
        q_step = torch.empty_like(q)
        lens_step = torch.empty_like(lens)
        outs = [out, bidx] if block else ([out, idx, tail, k_used] if certified else
                                          ([out, i_idx] if indexer else [out, idx, tail]))
        hosts = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
        h2d = q_host.numel() * q_host.element_size() + lens_host.numel() * 4
        d2h = sum(t.numel() * t.element_size() for t in outs)
        e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        idx_ready = [torch.cuda.Event() for _ in range(K)]
        for e in idx_ready:
            e.record()  # torch creates the CUDA event on its first record
        side = torch.cuda.Stream(device=dev)
        for i in range(K):
            l2_flush()
            e2e_ev[i][0].record()
            q_step.copy_(q_host, non_blocking=True)
            lens_step.copy_(lens_host, non_blocking=True)
            if block:
                tka.topk_block_attn_decode(q_step, kc, vc, bk, lens_step, w.block_size, w.top_blocks, out=out,
                                           block_idx=bidx, workspace=ws)
            elif certified:
                tka.topk_attn_decode_certified(q_step, kc, vc, lens_step, args.certified_eps, k, out=out,
                                               idx=idx, tail_mass=tail, k_used=k_used, workspace=ws)
            elif paged:
                tka.topk_attn_decode_paged(q_step, kp, vp, table, lens_step, k, out=out, idx=idx,
                                           tail_mass=tail, workspace=ws)
            elif hisa:
                tka.topk_hisa_attn_decode(q_step, kc, vc, h_bk, lens_step, h_bs, h_top, k, out=out, idx=idx,
                                          tail_mass=tail, block_idx=h_bidx, workspace=ws)
            elif indexer:
                tka.topk_indexer_attn_decode(q_step, kc, vc, i_q, i_w, i_k, lens_step, k, out=out, idx=i_idx,
                                             workspace=ws)
            else:
                # idx is final once the select has run: its read-back (the
                # largest result) overlaps the gather on a side stream
                tka.topk_attn_decode(q_step, kc, vc, lens_step, k, out=out, idx=idx, tail_mass=tail, workspace=ws,
                                     stage_events=[None, None, idx_ready[i], None])
                side.wait_event(idx_ready[i])
                with torch.cuda.stream(side):
                    hosts[1].copy_(idx, non_blocking=True)
            for j, (h, t) in enumerate(zip(hosts, outs)):
                if not (staged and j == 1):
                    h.copy_(t, non_blocking=True)
            if staged:
                torch.cuda.current_stream().wait_stream(side)
            e2e_ev[i][1].record()
        torch.cuda.synchronize()
        e2e_ms = sum(e[0].elapsed_time(e[1]) for e in e2e_ev)
    if tka.topk_attn_device_status() != 0:
        raise RuntimeError("device status raised during timing")

    vals = torch.tensor([total_ms, e2e_ms or 0.0] + ([sum(s) for s in stage_ms] if stage_ms else [0.0] * 3),
                        dtype=torch.float64, device=dev)
    reduce_over_ranks(vals, world)
    total_ms, e2e_ms_max = float(vals[0]), float(vals[1])
    stage_tot = [float(x) for x in vals[2:]]

    # unique kept rows from this rank's last result (token variant): the
    # stricter bytes, counted on the device after the timing
    alg_u = alg_bytes_unique(w, k, unique_kept_rows(idx, w)) if (staged or paged) else None

    if rank != 0:
        return None
    ms = total_ms / K
    peak, peak_src = measured_hbm_peak()
    res = {
        "metric": METRIC,
        "value": job_value(world, rows, ms),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded numpy PCG64, rounded once to the cache dtype)",
        "config": workload_config(w, k, world, args),
        "us_per_step": ms * 1e3,
        "tokens_per_s": world * w.B * w.Q / (ms / 1e3),
        "alg_bytes_per_step": alg,
        "alg_gbs": alg / (ms / 1e3) / 1e9,
        "alg_frac_of_spec_8tbs": alg / (ms / 1e3) / 1e9 / SPEC_HBM_GBS,
        "alg_frac_of_measured_hbm": alg / (ms / 1e3) / 1e9 / peak,
        **({"alg_bytes_unique_rows": alg_u, "unique_gbs": alg_u / (ms / 1e3) / 1e9,
            "unique_frac_of_measured_hbm": alg_u / (ms / 1e3) / 1e9 / peak} if alg_u else {}),
        "gpu_launches": launches_per_step * K,
        "clocks": clocks.summary(),
    }
    if indexer:
        # algorithmic bytes: index keys once per sequence + the k kept K and V rows per kv-head + q/out/idx
        row = w.d * elem_bytes(w)
        kept = sum(min(k, visible(w, b, qp)) for b in range(w.B) for qp in range(w.Q))
        alg = (k_bytes(w) // (w.Hkv * w.d) * i_d) + kept * w.Hkv * 2 * row + rows * w.d * (elem_bytes(w) + 4) \
            + w.B * w.Q * k * 4
        res["alg_bytes_per_step"] = alg
        res["alg_gbs"] = alg / (ms / 1e3) / 1e9
        res["alg_frac_of_spec_8tbs"] = res["alg_gbs"] / SPEC_HBM_GBS
        res["alg_frac_of_measured_hbm"] = res["alg_gbs"] / peak
        res["roofline"] = {"kernel": "whole step (indexer scores + select + attention)", "bound": "hbm",
                           "achieved": res["alg_gbs"], "peak": peak,
                           "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                           else "fallback 6.65 TB/s", "unit": "GB/s", "frac": res["alg_gbs"] / peak,
                           "traffic": None, "alg_bytes_per_launch": alg}
    if hisa:
        # algorithmic bytes: block keys + the kept blocks' K rows + the k kept V rows + q/out/idx
        row = w.d * elem_bytes(w)
        nblk = -(-w.L_max // h_bs)
        alg = rows * (nblk * w.d * 4 // w.G + h_top * h_bs * row + k * row) + rows * w.d * (elem_bytes(w) + 4) + rows * 4 * (k + 1)
        res["alg_bytes_per_step"] = alg
        res["alg_gbs"] = alg / (ms / 1e3) / 1e9
        res["alg_frac_of_spec_8tbs"] = res["alg_gbs"] / SPEC_HBM_GBS
        res["alg_frac_of_measured_hbm"] = res["alg_gbs"] / peak
        res["roofline"] = {"kernel": "whole step (hierarchical: blocks + candidates + select + gather)",
                           "bound": "hbm", "achieved": res["alg_gbs"], "peak": peak,
                           "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                           else "fallback 6.65 TB/s", "unit": "GB/s", "frac": res["alg_gbs"] / peak,
                           "traffic": None, "alg_bytes_per_launch": alg}
    if paged:
        # no per-kernel events on this path: the whole step against the copy peak
        res["roofline"] = {"kernel": "whole step (paged: score + select + gather)", "bound": "hbm",
                           "achieved": res["alg_gbs"], "peak": peak,
                           "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                           else "fallback 6.65 TB/s", "unit": "GB/s", "frac": res["alg_gbs"] / peak,
                           "traffic": None, "alg_bytes_per_launch": alg}
    if certified:
        ku = k_used.cpu().long()
        alg = alg_bytes_token(w, k, kept=int(ku.sum()))
        res["alg_bytes_per_step"] = alg
        res["alg_gbs"] = alg / (ms / 1e3) / 1e9
        res["alg_frac_of_spec_8tbs"] = res["alg_gbs"] / SPEC_HBM_GBS
        res["alg_frac_of_measured_hbm"] = res["alg_gbs"] / peak
        res["certified"] = {"eps": args.certified_eps, "k_max": k, "k_used_mean": float(ku.float().mean()),
                            "k_used_min": int(ku.min()), "k_used_max": int(ku.max()),
                            "rows_at_k_max": int((ku == k).sum()),
                            "tail_max": float(tail.max())}
        # no per-kernel events on this path: the whole step against the copy peak
        res["roofline"] = {"kernel": "whole step (score + select + certify + gather)", "bound": "hbm",
                           "achieved": res["alg_gbs"], "peak": peak,
                           "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                           else "fallback 6.65 TB/s", "unit": "GB/s", "frac": res["alg_gbs"] / peak,
                           "traffic": None, "alg_bytes_per_launch": alg}
    if stage_ms:
        res["stage_us"] = {n: stage_tot[j] / K * 1e3 for j, n in enumerate(["score", "select", "gather"])}
        res["stage_timing"] = ("a second timed pass of the same steps with events between the three kernels "
                               "(which also keeps each kernel from starting early behind the one before)")
        score_s = stage_tot[0] / K / 1e3
        achieved = dominant_bytes / score_s / 1e9
        traffic = score_traffic(os.path.join(ROOT, "exact_top_sparse_score_b200", "csrc", "score_tc.cu"))
        res["roofline"] = {"kernel": "score", "bound": "hbm", "achieved": achieved, "peak": peak,
                           "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                           else "fallback 6.65 TB/s", "unit": "GB/s", "frac": achieved / peak,
                           "traffic": traffic, "alg_bytes_per_launch": dominant_bytes}
    if e2e_ms is not None:
        e2e_step = e2e_ms_max / K
        res["e2e"] = {"value": job_value(world, rows, e2e_step), "unit": UNIT, "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "ms_per_step": e2e_step}
        if staged:
            res["e2e"]["overlap"] = ("idx is read back on a side stream from the event the library records "
                                     "after the select, while the gather runs")
    if world == 1 and not args.no_cpu_baseline:
        eps = args.certified_eps if certified else None
        v, cores, sample = time_oracle(w, k, eps=eps)
        v1, _, sample1 = time_oracle(w, k, budget_s=5.0, eps=eps, nthreads=1)
        res["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                               "value_1thread": v1, "sample_1thread": sample1}
    return res


def run_reference(args, rank):
    """The fp64 CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    w = make_inputs(args.config, 0, args.batch)
    rows = w.B * w.Q * w.Hq
    k = w.k

    def step():
        if w.variant == "block":
            oracle.block_attn(w, w.block_size, w.top_blocks)
        elif args.certified_eps is not None:
            oracle.certified_attn(w, args.certified_eps, k)
        else:
            oracle.topk_attn(w, k)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    ms = dt / args.steps * 1e3
    value = rows / (ms / 1e3)
    cores = oracle.max_threads()
    sample = f"whole workload ({rows} query rows) per step"
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64)",
        "config": workload_config(w, k, args.gpus, args),
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    world, rank, local = dist_setup(args)
    try:
        res = run_reference(args, rank) if args.impl == "reference" else run_ours(args, world, rank, local)
        if res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
