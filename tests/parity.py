"""Comparison of the CUDA path with the fp64 oracle.

Agreement required:
  * kept index sets equal, except for positions whose oracle score lies within
    BAND = 1e-3 of the oracle's k-th (smallest kept) score: near-ties that fp32
    scoring may order either way.  Rows whose sets differ inside the band are
    checked for validity instead: their out and tail must match an fp64
    evaluation over the GPU's own kept set.
  * out within 2e-2 absolute or 1e-2 relative for bf16 inputs, 1e-4 for fp32;
  * tail mass within 1e-3 absolute.
"""
import math

import numpy as np
import torch

import oracle

BAND = 1e-3
TAIL_TOL = 1e-3


def out_tol(dtype):
    return (2e-2, 1e-2) if dtype == "bf16" else (1e-4, 1e-4)


def to_device(w, device="cuda:0"):
    return (w.q.to(device), w.k_cache.to(device), w.v_cache.to(device), w.seq_lens.to(device))


def _close(got, want, atol, rtol):
    return np.abs(got - want) <= atol + rtol * np.abs(want)


def _vis(w, b, qp):
    return int(w.seq_lens[b]) - w.Q + qp + 1


def _set_eval(w, s, sel, b, h):
    """fp64 out and tail over a given kept set (validity check of a tie-band row)."""
    m = s.max()
    e = np.exp(s - m)
    zk = e[sel].sum()
    V = w.v_cache[b, h // w.G].double().numpy()[sel]
    return (e[sel, None] * V).sum(0) / zk, 1.0 - zk / e.sum()


def check_token(w, k, out, idx, tail, ref, scale=0.0, rows_checked=None):
    """Asserts parity of topk_attn_decode outputs with oracle.topk_attn output `ref`.

    rows_checked: optional list of (b, qpos, h) to restrict to (sampled full-size checks;
    `ref` then holds only those rows, in that order)."""
    out = out.detach().cpu().double().numpy()
    idx = idx.detach().cpu().numpy()
    tail = tail.detach().cpu().double().numpy() if tail is not None else None
    atol, rtol = out_tol(w.dtype)
    rows = rows_checked or [(b, qp, h) for b in range(w.B) for qp in range(w.Q) for h in range(w.Hq)]
    n_band = 0
    for r_i, (b, qp, h) in enumerate(rows):
        g = idx[b, qp, h]
        if rows_checked:
            o, ro, rt, kth = ref["idx"][r_i], ref["out"][r_i], ref["tail"][r_i], ref["kth"][r_i]
        else:
            o, ro, rt, kth = ref["idx"][b, qp, h], ref["out"][b, qp, h], ref["tail"][b, qp, h], ref["kth"][b, qp, h]
        vis = _vis(w, b, qp)
        kk = min(k, vis)
        where = f"row (b={b}, q={qp}, h={h})"
        assert np.all(g[kk:] == -1), f"{where}: padding"
        gs = g[:kk]
        assert np.all(gs >= 0) and np.all(gs < vis), f"{where}: position out of range"
        assert np.all(np.diff(gs) > 0), f"{where}: not strictly ascending"
        if np.array_equal(gs, o[:kk]):
            ok = _close(out[b, qp, h], ro, atol, rtol)
            assert ok.all(), f"{where}: out max |diff| {np.abs(out[b, qp, h] - ro).max():.3e}"
            if tail is not None:
                assert abs(tail[b, qp, h] - rt) <= TAIL_TOL, f"{where}: tail {tail[b, qp, h]} vs {rt}"
            continue
        n_band += 1
        s = oracle.row_scores(w, b, qp, h, scale)
        diff = np.setxor1d(gs, o[:kk])
        assert np.all(np.abs(s[diff] - kth) <= BAND), \
            f"{where}: set differs outside the tie band (max {np.abs(s[diff] - kth).max():.3e})"
        vo, vt = _set_eval(w, s, gs, b, h)
        assert _close(out[b, qp, h], vo, atol, rtol).all(), f"{where}: out invalid for its own set"
        if tail is not None:
            assert abs(tail[b, qp, h] - vt) <= TAIL_TOL, f"{where}: tail invalid for its own set"
    return n_band


def oracle_block_scores(w, bk, b, h, scale=0.0):
    sc = scale if scale > 0 else 1.0 / math.sqrt(w.d)
    return bk[b, h // w.G] @ w.q[b, 0, h].double().numpy() * sc


def check_block(w, block_size, top_blocks, out, bidx, ref, scale=0.0):
    out = out.detach().cpu().double().numpy()
    bidx = bidx.detach().cpu().numpy()
    atol, rtol = out_tol(w.dtype)
    bk = None
    n_band = 0
    for b in range(w.B):
        Lb = int(w.seq_lens[b])
        nblk = -(-Lb // block_size)
        nk = min(top_blocks, nblk - 1) + 1
        for h in range(w.Hq):
            where = f"row (b={b}, h={h})"
            g, o = bidx[b, 0, h], ref["block_idx"][b, 0, h]
            assert np.all(g[nk:] == -1), f"{where}: padding"
            gs = g[:nk]
            assert np.all(np.diff(gs) > 0) and gs[-1] == nblk - 1 and gs[0] >= 0, f"{where}: block list"
            if np.array_equal(gs, o[:nk]):
                ok = _close(out[b, 0, h], ref["out"][b, 0, h], atol, rtol)
                assert ok.all(), f"{where}: out max |diff| {np.abs(out[b, 0, h] - ref['out'][b, 0, h]).max():.3e}"
                continue
            n_band += 1
            if bk is None:
                bk = oracle.block_pool(w, block_size)
            r = oracle_block_scores(w, bk, b, h, scale)
            diff = np.setxor1d(gs, o[:nk])
            assert np.all(np.abs(r[diff] - ref["kth"][b, 0, h]) <= BAND), f"{where}: block set outside tie band"
            # validity: dense attention over the GPU's kept blocks
            s = oracle.row_scores(w, b, 0, h, scale)
            sel = np.concatenate([np.arange(j * block_size, min(j * block_size + block_size, Lb)) for j in gs])
            e = np.exp(s[sel] - s[sel].max())
            V = w.v_cache[b, h // w.G].double().numpy()[sel]
            want = (e[:, None] * V).sum(0) / e.sum()
            assert _close(out[b, 0, h], want, atol, rtol).all(), f"{where}: out invalid for its own blocks"
    return n_band


CERT_TOL = 1e-4  # slack on the eps comparison for fp32 scores and masses


def check_certified(w, eps, k_max, out, idx, tail, k_used, ref, scale=0.0, rows_checked=None):
    """Asserts parity of topk_attn_decode_certified with oracle.certified_attn output `ref`.

    Every row: k_used is certified and minimal against the oracle's fp64 tail
    masses (within CERT_TOL of eps, or at the cap); idx holds the top-k_used
    positions (up to the tie band around the k_used-th score), ascending and
    -1 padded; out and tail match an fp64 evaluation over the kept set.  Rows
    whose k_used equals the oracle's compare idx, out and tail with it
    directly.  Returns the number of rows whose k differs from the oracle's."""
    out = out.detach().cpu().double().numpy()
    idx = idx.detach().cpu().numpy()
    tail = tail.detach().cpu().double().numpy()
    k_used = k_used.detach().cpu().numpy()
    atol, rtol = out_tol(w.dtype)
    rows = rows_checked or [(b, qp, h) for b in range(w.B) for qp in range(w.Q) for h in range(w.Hq)]
    n_diff = 0
    for r_i, (b, qp, h) in enumerate(rows):
        if rows_checked:
            ro, ri, rt, rk = ref["out"][r_i], ref["idx"][r_i], ref["tail"][r_i], ref["k_used"][r_i]
        else:
            ro, ri, rt, rk = (ref["out"][b, qp, h], ref["idx"][b, qp, h], ref["tail"][b, qp, h],
                              ref["k_used"][b, qp, h])
        where = f"row (b={b}, q={qp}, h={h})"
        vis = _vis(w, b, qp)
        cap = min(k_max, vis)
        kg = int(k_used[b, qp, h])
        assert 1 <= kg <= cap, f"{where}: k_used {kg} outside [1, {cap}]"
        s = oracle.row_scores(w, b, qp, h, scale)
        order = np.lexsort((np.arange(vis), -s))
        e = np.exp(s[order] - s[order[0]])
        tau = 1.0 - np.cumsum(e) / e.sum()  # tau[j] = tail mass of the top j + 1
        if kg < cap:
            assert tau[kg - 1] <= eps + CERT_TOL, f"{where}: k={kg} leaves {tau[kg - 1]:.6f} > eps"
        if kg > 1:
            assert tau[kg - 2] > eps - CERT_TOL, f"{where}: k={kg} not minimal ({tau[kg - 2]:.6f} <= eps)"
        g = idx[b, qp, h]
        assert np.all(g[kg:] == -1), f"{where}: padding"
        gs = g[:kg]
        assert np.all(gs >= 0) and np.all(gs < vis) and np.all(np.diff(gs) > 0), f"{where}: kept list"
        top = np.sort(order[:kg])
        diff = np.setxor1d(gs, top)
        kth = s[order[kg - 1]]
        assert np.all(np.abs(s[diff] - kth) <= BAND), f"{where}: set differs outside the tie band"
        if kg == rk and np.array_equal(gs, ri[:kg]):
            assert _close(out[b, qp, h], ro, atol, rtol).all(), f"{where}: out"
            assert abs(tail[b, qp, h] - rt) <= TAIL_TOL, f"{where}: tail {tail[b, qp, h]} vs {rt}"
            continue
        n_diff += kg != rk
        vo, vt = _set_eval(w, s, gs, b, h)
        assert _close(out[b, qp, h], vo, atol, rtol).all(), f"{where}: out invalid for its own set"
        assert abs(tail[b, qp, h] - vt) <= TAIL_TOL, f"{where}: tail invalid for its own set"
    return n_diff


def check_hisa(w, block_size, top_blocks, k, out, idx, tail, bidx, ref, scale=0.0):
    """Asserts parity of topk_hisa_attn_decode with oracle.hisa_attn output `ref`.

    Kept blocks equal the oracle's except blocks whose fp64 block score lies
    within BAND of the oracle's top_blocks-th; kept tokens equal the top k of
    the GPU's own candidates except positions within BAND of the k-th
    candidate score; out and tail match the oracle where the sets agree and an
    fp64 evaluation over the GPU's own sets otherwise.  Returns the number of
    rows checked through the band."""
    out = out.detach().cpu().double().numpy()
    idx = idx.detach().cpu().numpy()
    tail = tail.detach().cpu().double().numpy()
    bidx = bidx.detach().cpu().numpy()
    atol, rtol = out_tol(w.dtype)
    bk = None
    n_band = 0
    for b in range(w.B):
        Lb = int(w.seq_lens[b])
        nblk = -(-Lb // block_size)
        nk = min(top_blocks, nblk)
        for h in range(w.Hq):
            where = f"row (b={b}, h={h})"
            gb, ob = bidx[b, 0, h], ref["block_idx"][b, 0, h]
            assert np.all(gb[nk:] == -1) and np.all(np.diff(gb[:nk]) > 0) and gb[0] >= 0, f"{where}: block list"
            s = oracle.row_scores(w, b, 0, h, scale)
            if not np.array_equal(gb[:nk], ob[:nk]):
                n_band += 1
                if bk is None:
                    bk = oracle.block_pool(w, block_size)
                r = oracle_block_scores(w, bk, b, h, scale)[:nblk]
                kth = np.sort(r)[::-1][nk - 1]
                diff = np.setxor1d(gb[:nk], ob[:nk])
                assert np.all(np.abs(r[diff] - kth) <= BAND), f"{where}: blocks differ outside the tie band"
            cand = np.concatenate([np.arange(j * block_size, min((j + 1) * block_size, Lb)) for j in gb[:nk]])
            kk = min(k, len(cand))
            g = idx[b, 0, h]
            assert np.all(g[kk:] == -1), f"{where}: padding"
            gs = g[:kk]
            assert np.all(np.isin(gs, cand)) and np.all(np.diff(gs) > 0), f"{where}: kept tokens"
            order = np.lexsort((cand, -s[cand]))
            top = np.sort(cand[order[:kk]])
            kth_s = s[cand[order[kk - 1]]]
            assert np.all(np.abs(s[np.setxor1d(gs, top)] - kth_s) <= BAND), f"{where}: tokens outside the tie band"
            if np.array_equal(gb[:nk], ob[:nk]) and np.array_equal(gs, ref["idx"][b, 0, h, :kk]):
                assert _close(out[b, 0, h], ref["out"][b, 0, h], atol, rtol).all(), f"{where}: out"
                assert abs(tail[b, 0, h] - ref["tail"][b, 0, h]) <= TAIL_TOL, f"{where}: tail"
                continue
            n_band += 1
            e_all = np.exp(s[cand] - s[cand].max())
            e = np.exp(s[gs] - s[gs].max())
            V = w.v_cache[b, h // w.G].double().numpy()[gs]
            assert _close(out[b, 0, h], (e[:, None] * V).sum(0) / e.sum(), atol, rtol).all(), f"{where}: out invalid"
            kept_mass = np.exp(s[gs] - s[cand].max()).sum() / e_all.sum()
            assert abs(tail[b, 0, h] - (1.0 - kept_mass)) <= TAIL_TOL, f"{where}: tail invalid"
    return n_band


def index_scores_f64(w, q_idx, w_idx, k_idx):
    """sum_j w_j ReLU(<q_idx_j, k_idx_i>) in fp64 [B, Q, L_max] (positions past a sequence's end: -inf)."""
    dots = torch.einsum("bqjc,blc->bqjl", q_idx.double(), torch.nan_to_num(k_idx.float()).double())
    s = (w_idx.double()[..., None] * torch.relu(dots)).sum(2).numpy()
    for b in range(w.B):
        for qp in range(w.Q):
            s[b, qp, _vis(w, b, qp):] = -np.inf
    return s


def check_indexer(w, k, out, idx, ref, I, scale=0.0):
    """Asserts parity of topk_indexer_attn_decode with oracle.indexer_attn output `ref`.

    Kept tokens equal the oracle's except positions whose fp64 indexer score
    lies within BAND (relative to its scale) of the oracle's k-th; out matches
    the oracle where the sets agree, else an fp64 evaluation over the GPU's
    own set.  I: fp64 indexer scores [B, Q, L_max].  Returns the number of
    positions checked through the band."""
    out = out.detach().cpu().double().numpy()
    idx = idx.detach().cpu().numpy()
    atol, rtol = out_tol(w.dtype)
    n_band = 0
    for b in range(w.B):
        for qp in range(w.Q):
            where = f"position (b={b}, q={qp})"
            vis = _vis(w, b, qp)
            kk = min(k, vis)
            g = idx[b, qp]
            assert np.all(g[kk:] == -1), f"{where}: padding"
            gs = g[:kk]
            assert np.all(gs >= 0) and np.all(gs < vis) and np.all(np.diff(gs) > 0), f"{where}: kept list"
            o = ref["idx"][b, qp, :kk]
            same = np.array_equal(gs, o)
            if not same:
                n_band += 1
                kth = ref["kth"][b, qp]
                tol = BAND * max(1.0, abs(kth))
                diff = np.setxor1d(gs, o)
                assert np.all(np.abs(I[b, qp, diff] - kth) <= tol), f"{where}: set differs outside the tie band"
            for h in range(w.Hq):
                if same:
                    ok = _close(out[b, qp, h], ref["out"][b, qp, h], atol, rtol)
                    assert ok.all(), f"{where}, head {h}: out"
                else:
                    s = oracle.row_scores(w, b, qp, h, scale)
                    e = np.exp(s[gs] - s[gs].max())
                    V = w.v_cache[b, h // w.G].double().numpy()[gs]
                    assert _close(out[b, qp, h], (e[:, None] * V).sum(0) / e.sum(), atol, rtol).all(), \
                        f"{where}, head {h}: out invalid for its own set"
    return n_band
