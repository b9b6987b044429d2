"""Pins for the fp64 oracle, each against something other than the oracle.

* Dense special case: with k >= every row's visible length, Top-k attention is
  ordinary softmax attention ("Sparse Attention in LLM Inference: Practical
  Trade-Offs", section "The Bottleneck of Dense Attention"), checked against
  torch's scaled_dot_product_attention in fp64 with explicit GQA head
  expansion and a causal visibility mask.
* Selection: against numpy lexsort on torch-computed scores, and on tiny rows
  with planted ties against an exhaustive search over all k-subsets.
* A closed form with integer weights (scores ln(i+1), one-hot values).
* "A Mathematical Theory of Top-k Sparse Attention via Total Variation
  Distance" (abstract): TV = discarded tail mass = 1 - exp(-KL(P_hat || P)),
  the head-tail output factorisation, and the Gaussian closed form for the
  tail mass.
* Block variant ("Sparse Attention Landscape", MoBA): mean pooling against
  torch.mean, block choice against lexsort, and the all-blocks case against
  dense attention.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import workloads


def _f64(t):
    return t.to(torch.float64)


def _expanded_kv(w):
    """K, V as fp64 [B, Hq, L, d] with head h reading kv-head h // G; rows past
    a sequence's end (NaN poison) zeroed since the mask removes them anyway."""
    K = _f64(w.k_cache).repeat_interleave(w.G, dim=1)
    V = _f64(w.v_cache).repeat_interleave(w.G, dim=1)
    for b in range(w.B):
        K[b, :, int(w.seq_lens[b]):] = 0
        V[b, :, int(w.seq_lens[b]):] = 0
    return K, V


def _visible_mask(w):
    L = torch.arange(w.L_max)
    m = torch.zeros(w.B, 1, w.Q, w.L_max, dtype=torch.bool)
    for b in range(w.B):
        for qp in range(w.Q):
            m[b, 0, qp] = L < int(w.seq_lens[b]) - w.Q + qp + 1
    return m


def dense_sdpa(w, scale=None):
    """Dense softmax attention via torch SDPA, [B, Q, Hq, d] fp64."""
    q = _f64(w.q).transpose(1, 2)  # [B,Hq,Q,d]
    K, V = _expanded_kv(w)
    o = torch.nn.functional.scaled_dot_product_attention(q, K, V, attn_mask=_visible_mask(w),
                                                         scale=scale)
    return o.transpose(1, 2).numpy()


def torch_scores(w, scale=None):
    """Scores [B, Q, Hq, L] in fp64 via torch.matmul (-inf where not visible)."""
    q = _f64(w.q).transpose(1, 2)
    K, _ = _expanded_kv(w)
    sc = (1.0 / math.sqrt(w.d)) if scale is None else scale
    s = torch.matmul(q, K.transpose(-1, -2)) * sc  # [B,Hq,Q,L]
    s = s.masked_fill(~_visible_mask(w).expand_as(s), -math.inf)
    return s.transpose(1, 2).numpy()


def lexsort_topk(s_row, k):
    """Positions of the k best by (score desc, position asc), via numpy lexsort."""
    vis = int(np.isfinite(s_row).sum())
    pos = np.arange(vis)
    order = np.lexsort((pos, -s_row[:vis]))
    return np.sort(order[:min(k, vis)])


# ----------------------------------------------------------------------------- dense case

@pytest.mark.parametrize("dtype,B,Q,Hq,Hkv,L,lens", [
    ("f32", 1, 1, 1, 1, 97, None),
    ("bf16", 2, 1, 8, 2, 130, [130, 77]),
    ("bf16", 2, 5, 8, 4, 64, [64, 9]),      # causal chunk, short second sequence
    ("f32", 3, 3, 6, 3, 40, [40, 3, 17]),   # vis = 1 for the first query of batch 1
])
def test_full_k_equals_dense_attention(dtype, B, Q, Hq, Hkv, L, lens):
    w = workloads.make_workload(B, Q, Hq, Hkv, L, dtype=dtype, seq_lens=lens, seed=11)
    r = oracle.topk_attn(w, k=L)
    ref = dense_sdpa(w)
    np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-12)
    assert np.all(r["tail"] == 0.0)
    for b in range(B):
        for qp in range(Q):
            vis = int(w.seq_lens[b]) - Q + qp + 1
            want = np.concatenate([np.arange(vis), -np.ones(L - vis, np.int64)])
            assert np.array_equal(r["idx"][b, qp, 0], want)


def test_explicit_scale_matches_sdpa_scale():
    w = workloads.make_workload(1, 1, 4, 2, 50, dtype="f32", seed=5)
    r = oracle.topk_attn(w, k=50, scale=0.37)
    np.testing.assert_allclose(r["out"], dense_sdpa(w, scale=0.37), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- selection

@pytest.mark.parametrize("dtype,Q,lens,k", [
    ("bf16", 1, [300, 211], 17),
    ("f32", 4, [128, 100], 31),
    ("bf16", 2, [64, 64], 64),   # k larger than the visible length of query 0
])
def test_selection_matches_lexsort(dtype, Q, lens, k):
    w = workloads.make_workload(2, Q, 8, 2, max(lens), dtype=dtype, seq_lens=lens, seed=21)
    r = oracle.topk_attn(w, k=k)
    s = torch_scores(w)
    for b in range(w.B):
        for qp in range(Q):
            for h in range(w.Hq):
                want = lexsort_topk(s[b, qp, h], k)
                got = r["idx"][b, qp, h]
                assert np.array_equal(got[:len(want)], want)
                assert np.all(got[len(want):] == -1)
                np.testing.assert_allclose(r["kth"][b, qp, h], s[b, qp, h][want].min(), rtol=1e-12)


def _tie_workload(int_scores, dv=None):
    """One row whose scores are exactly the given integers (scale 1, q = e_0)."""
    L = len(int_scores)
    d = 128
    w = workloads.make_workload(1, 1, 1, 1, L, dtype="f32", seed=1)
    w.q.zero_()
    w.q[0, 0, 0, 0] = 1.0
    w.k_cache.zero_()
    w.k_cache[0, 0, :, 0] = torch.tensor(int_scores, dtype=torch.float32)
    if dv is not None:
        w.v_cache.copy_(dv)
    return w


@pytest.mark.parametrize("seed", range(40))
def test_selection_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(1, 11))
    k = int(rng.integers(1, L + 1))
    scores = rng.integers(-2, 3, size=L).astype(float)  # many exact ties
    w = _tie_workload(scores)
    r = oracle.topk_attn(w, k=k, scale=1.0)
    got = tuple(int(i) for i in r["idx"][0, 0, 0][:k])
    # the unique subset in which every kept position precedes every dropped one
    # in the order (score desc, position asc)
    valid = []
    for sub in itertools.combinations(range(L), k):
        rest = [j for j in range(L) if j not in sub]
        if all(scores[a] > scores[c] or (scores[a] == scores[c] and a < c) for a in sub for c in rest):
            valid.append(sub)
    assert valid == [got]


def test_closed_form_integer_weights():
    # s_i = ln(i+1) so e^{s_i} = i+1 exactly up to rounding; V one-hot.
    L, k, d = 100, 13, 128
    perm = np.random.default_rng(3).permutation(L)
    weight = perm + 1.0                         # position j has weight perm[j]+1
    V = torch.zeros(1, 1, L, d, dtype=torch.float32)
    V[0, 0, torch.arange(L), torch.arange(L)] = 1.0
    w = _tie_workload(np.log(weight), dv=V)
    r = oracle.topk_attn(w, k=k, scale=1.0)
    keep = np.sort(np.argsort(-weight)[:k])
    assert np.array_equal(r["idx"][0, 0, 0], keep)
    Z = L * (L + 1) / 2
    Zk = sum(range(L - k + 1, L + 1))
    assert abs(r["tail"][0, 0, 0] - (1 - Zk / Z)) < 1e-7
    want = np.zeros(d)
    want[keep] = weight[keep] / Zk
    np.testing.assert_allclose(r["out"][0, 0, 0], want, atol=1e-7)


def test_k1_returns_value_row_of_argmax():
    w = workloads.make_workload(2, 2, 8, 4, 257, dtype="bf16", seq_lens=[257, 190], seed=8)
    r = oracle.topk_attn(w, k=1)
    s = torch_scores(w)
    for b in range(2):
        for qp in range(2):
            for h in range(8):
                j = int(np.argmax(s[b, qp, h]))
                assert r["idx"][b, qp, h, 0] == j
                np.testing.assert_array_equal(r["out"][b, qp, h], _f64(w.v_cache[b, h // 2, j]).numpy())


# ----------------------------------------------------------------------------- TV identities

@pytest.mark.parametrize("k", [1, 7, 64, 200])
def test_tail_mass_is_tv_and_kl_identity(k):
    w = workloads.make_workload(2, 2, 8, 2, 300, dtype="bf16", seq_lens=[300, 123], k_mean_std=0.5, seed=31)
    r = oracle.topk_attn(w, k=k)
    P = torch.softmax(torch.from_numpy(torch_scores(w)), dim=-1).numpy()
    for b in range(2):
        for qp in range(2):
            for h in range(8):
                sel = r["idx"][b, qp, h]
                sel = sel[sel >= 0]
                p = P[b, qp, h]
                tau = r["tail"][b, qp, h]
                head = p[sel].sum()
                assert abs(tau - (1 - head)) < 1e-12
                # TV(P, P_hat) = 1/2 sum |P - P_hat|
                p_hat = np.zeros_like(p)
                p_hat[sel] = p[sel] / head
                assert abs(tau - 0.5 * np.abs(p - p_hat).sum()) < 1e-12
                kl = np.sum(p_hat[sel] * np.log(p_hat[sel] / p[sel]))
                assert abs(tau - (1 - math.exp(-kl))) < 1e-9


@pytest.mark.parametrize("k", [3, 40, 150])
def test_output_error_factorises_head_tail(k):
    w = workloads.make_workload(1, 3, 4, 2, 200, dtype="f32", seed=41)
    r = oracle.topk_attn(w, k=k)
    dense = dense_sdpa(w)
    P = torch.softmax(torch.from_numpy(torch_scores(w)), dim=-1).numpy()
    _, V = _expanded_kv(w)
    V = V.numpy()
    for qp in range(3):
        for h in range(4):
            sel = r["idx"][0, qp, h]
            sel = sel[sel >= 0]
            p = P[0, qp, h]
            tau = r["tail"][0, qp, h]
            rest = np.setdiff1d(np.arange(len(p)), sel)
            mu_tail = (p[rest, None] * V[0, h, rest]).sum(0) / tau
            mu_head = r["out"][0, qp, h]
            lhs = np.linalg.norm(dense[0, qp, h] - mu_head)
            rhs = tau * np.linalg.norm(mu_tail - mu_head)
            assert abs(lhs - rhs) <= 1e-9 * max(lhs, 1e-300)


def test_gaussian_closed_form_tail_mass():
    # i.i.d. Gaussian scores s ~ N(0, sigma^2), sigma = |q|/sqrt(d): the tail
    # mass of Top-k is Phi(Phi^{-1}(1 - k/n) - sigma) asymptotically.
    from scipy.stats import norm
    errs = []
    for seed in range(64):
        w = workloads.make_workload(1, 1, 1, 1, 4096, dtype="f32", seed=5000 + seed)
        r = oracle.topk_attn(w, k=64)
        sigma = float(torch.linalg.vector_norm(_f64(w.q[0, 0, 0]))) / math.sqrt(128)
        pred = norm.cdf(norm.ppf(1 - 64 / 4096) - sigma)
        errs.append(r["tail"][0, 0, 0] - pred)
    errs = np.array(errs)
    assert abs(errs.mean()) < 3e-3, errs.mean()
    assert np.abs(errs).max() < 0.04, np.abs(errs).max()


# ----------------------------------------------------------------------------- poison / causal

def test_rows_past_sequence_end_are_never_read():
    w = workloads.make_workload(3, 4, 8, 2, 256, dtype="bf16", seq_lens=[256, 100, 4], seed=51)
    assert torch.isnan(w.k_cache[1, :, 100:].float()).all()
    r = oracle.topk_attn(w, k=50)
    assert np.isfinite(r["out"]).all() and np.isfinite(r["tail"]).all()
    for b, Lb in enumerate([256, 100, 4]):
        for qp in range(4):
            vis = Lb - 4 + qp + 1
            sel = r["idx"][b, qp]
            assert (sel < vis).all()
            assert ((sel >= 0).sum(axis=-1) == min(50, vis)).all()


def test_bad_arguments_rejected():
    w = workloads.make_workload(1, 4, 4, 2, 8, dtype="f32", seq_lens=[3], seed=1)
    with pytest.raises(ValueError):
        oracle.topk_attn(w, k=2)    # Q = 4 > seq_len 3
    w = workloads.make_workload(1, 1, 4, 2, 8, dtype="f32", seed=1)
    with pytest.raises(ValueError):
        oracle.topk_attn(w, k=0)


# ----------------------------------------------------------------------------- block variant

@pytest.mark.parametrize("L,lens,bs", [(256, [256, 200], 16), (130, [130, 64], 32), (64, [64, 1], 64)])
def test_block_pool_is_block_mean(L, lens, bs):
    w = workloads.make_workload(2, 1, 4, 2, L, dtype="bf16", seq_lens=lens, seed=61)
    bk = oracle.block_pool(w, bs)
    nblk = -(-L // bs)
    for b, Lb in enumerate(lens):
        for h in range(2):
            for j in range(nblk):
                lo, hi = j * bs, min(j * bs + bs, Lb)
                want = _f64(w.k_cache[b, h, lo:hi]).mean(0).numpy() if hi > lo else np.zeros(128)
                np.testing.assert_allclose(bk[b, h, j], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("lens,bs,top", [([1024, 1000], 64, 4), ([700, 333], 32, 5), ([96, 64], 32, 1)])
def test_block_selection_matches_lexsort(lens, bs, top):
    L = max(lens)
    w = workloads.make_workload(2, 1, 8, 2, L, dtype="bf16", seq_lens=lens, seed=71)
    r = oracle.block_attn(w, bs, top)
    bk = torch.from_numpy(oracle.block_pool(w, bs))  # pinned above
    for b, Lb in enumerate(lens):
        nblk = -(-Lb // bs)
        for h in range(8):
            q = _f64(w.q[b, 0, h])
            rs = (bk[b, h // 4, :nblk - 1] @ q).numpy() / math.sqrt(128)
            order = np.lexsort((np.arange(nblk - 1), -rs))
            want = np.sort(np.concatenate([order[:top], [nblk - 1]]))
            got = r["block_idx"][b, 0, h]
            assert np.array_equal(got[:len(want)], want)
            assert np.all(got[len(want):] == -1)


@pytest.mark.parametrize("lens,bs", [([256, 250], 64), ([100, 37], 16)])
def test_block_all_blocks_is_dense(lens, bs):
    L = max(lens)
    w = workloads.make_workload(2, 1, 8, 4, L, dtype="f32", seq_lens=lens, seed=81)
    r = oracle.block_attn(w, bs, top_blocks=-(-L // bs))
    np.testing.assert_allclose(r["out"], dense_sdpa(w), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["tail"], 0.0, atol=1e-15)


def test_block_attention_over_kept_tokens():
    # dense attention restricted to the kept blocks' tokens, via SDPA with a mask
    w = workloads.make_workload(2, 1, 8, 2, 512, dtype="bf16", seq_lens=[512, 300], seed=91)
    bs, top = 32, 3
    r = oracle.block_attn(w, bs, top)
    K, V = _expanded_kv(w)
    q = _f64(w.q).transpose(1, 2)
    mask = torch.zeros(2, 8, 1, 512, dtype=torch.bool)
    for b in range(2):
        for h in range(8):
            for j in r["block_idx"][b, 0, h]:
                if j >= 0:
                    mask[b, h, 0, j * bs:min(j * bs + bs, int(w.seq_lens[b]))] = True
    ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, attn_mask=mask).transpose(1, 2)
    np.testing.assert_allclose(r["out"], ref.numpy(), rtol=1e-12, atol=1e-12)
    P = torch.softmax(torch.from_numpy(torch_scores(w)), dim=-1).numpy()
    kept_mass = (P * mask.transpose(1, 2).numpy()).sum(-1)
    np.testing.assert_allclose(r["tail"], 1 - kept_mass, atol=1e-12)


# ----------------------------------------------------------------------------- certified adaptive Top-k

def test_certified_large_eps_keeps_only_the_argmax():
    w = workloads.make_workload(2, 2, 8, 4, 300, dtype="bf16", seq_lens=[300, 211], seed=61)
    r = oracle.certified_attn(w, eps=1.0 - 1e-12, k_max=64)
    s = torch_scores(w)
    assert np.all(r["k_used"] == 1)
    for b in range(2):
        for qp in range(2):
            for h in range(8):
                j = int(np.argmax(s[b, qp, h]))
                assert r["idx"][b, qp, h, 0] == j and np.all(r["idx"][b, qp, h, 1:] == -1)
                np.testing.assert_array_equal(r["out"][b, qp, h], _f64(w.v_cache[b, h // 2, j]).numpy())


def test_certified_zero_eps_is_dense_attention():
    w = workloads.make_workload(2, 3, 4, 2, 90, dtype="f32", seq_lens=[90, 41], seed=62)
    r = oracle.certified_attn(w, eps=0.0, k_max=90)
    np.testing.assert_allclose(r["out"], dense_sdpa(w), rtol=1e-12, atol=1e-12)
    for b in range(2):
        for qp in range(3):
            assert np.all(r["k_used"][b, qp] == int(w.seq_lens[b]) - 3 + qp + 1)
    assert np.all(r["tail"] == 0.0)


@pytest.mark.parametrize("eps,k_max", [(0.3, 600), (0.05, 600), (0.5, 40), (0.2, 150)])
def test_certified_k_is_the_smallest_certified_prefix(eps, k_max):
    """Brute force on softmax probabilities from torch: the kept set is the
    lexsort top-k_used, its discarded mass is <= eps, and one key fewer would
    leave more than eps outside (unless k_used is at the cap)."""
    w = workloads.make_workload(2, 2, 4, 2, 600, dtype="bf16", seq_lens=[600, 350], k_mean_std=0.5, seed=63)
    r = oracle.certified_attn(w, eps=eps, k_max=k_max)
    s = torch_scores(w)
    P = torch.softmax(torch.from_numpy(s), dim=-1).numpy()
    for b in range(2):
        for qp in range(2):
            for h in range(4):
                vis = int(w.seq_lens[b]) - 2 + qp + 1
                ku = int(r["k_used"][b, qp, h])
                sel = lexsort_topk(s[b, qp, h], ku)
                got = r["idx"][b, qp, h]
                assert np.array_equal(got[:ku], sel) and np.all(got[ku:] == -1)
                order = np.lexsort((np.arange(vis), -s[b, qp, h, :vis]))
                cum = np.cumsum(P[b, qp, h][order])
                tau = 1.0 - cum[ku - 1]
                assert abs(r["tail"][b, qp, h] - tau) < 1e-12
                cap = min(k_max, vis)
                if ku < cap or tau <= eps:
                    assert tau <= eps + 1e-12
                else:
                    assert ku == cap and tau > eps  # not certifiable within the cap
                if ku > 1:
                    assert 1.0 - cum[ku - 2] > eps - 1e-12


def test_certified_minimal_k_follows_the_gaussian_rule():
    # i.i.d. Gaussian scores N(0, sigma^2), sigma = |q|/sqrt(d): the smallest
    # k with tail mass <= eps satisfies k/n ~ 1 - Phi(sigma + Phi^{-1}(eps)).
    from scipy.stats import norm
    errs = []
    for seed in range(32):
        w = workloads.make_workload(1, 1, 1, 1, 4096, dtype="f32", seed=7000 + seed)
        r = oracle.certified_attn(w, eps=0.2, k_max=4096)
        sigma = float(torch.linalg.vector_norm(_f64(w.q[0, 0, 0]))) / math.sqrt(128)
        pred = norm.sf(sigma + norm.ppf(0.2))
        errs.append(r["k_used"][0, 0, 0] / 4096 - pred)
    errs = np.array(errs)
    assert abs(errs.mean()) < 0.01, errs.mean()
    assert np.abs(errs).max() < 0.05, np.abs(errs).max()


def test_certified_equals_fixed_k_at_the_chosen_k():
    w = workloads.make_workload(1, 2, 4, 1, 500, dtype="bf16", seed=64)
    r = oracle.certified_attn(w, eps=0.25, k_max=500)
    for qp in range(2):
        for h in range(4):
            ku = int(r["k_used"][0, qp, h])
            f = oracle.topk_attn(w, k=ku)
            np.testing.assert_array_equal(r["out"][0, qp, h], f["out"][0, qp, h])
            np.testing.assert_array_equal(r["idx"][0, qp, h, :ku], f["idx"][0, qp, h])
            assert r["tail"][0, qp, h] == f["tail"][0, qp, h]


# ----------------------------------------------------------------------------- hierarchical block -> token

def test_hisa_with_every_block_is_token_topk():
    w = workloads.make_workload(2, 1, 8, 2, 700, dtype="bf16", seq_lens=[700, 260], seed=71)
    h = oracle.hisa_attn(w, block_size=32, top_blocks=64, k=100)
    t = oracle.topk_attn(w, k=100)
    np.testing.assert_array_equal(h["idx"], t["idx"])
    np.testing.assert_array_equal(h["out"], t["out"])
    np.testing.assert_array_equal(h["tail"], t["tail"])


@pytest.mark.parametrize("bs,top,k", [(16, 3, 20), (32, 4, 200), (64, 2, 7)])
def test_hisa_brute_force(bs, top, k):
    """Block means, block ranking, candidate ranking and attention recomputed
    with torch and numpy lexsort."""
    w = workloads.make_workload(2, 1, 4, 2, 400, dtype="bf16", seq_lens=[400, 150], k_mean_std=0.5, seed=72)
    r = oracle.hisa_attn(w, block_size=bs, top_blocks=top, k=k)
    s_all = torch_scores(w)
    for b in range(2):
        Lb = int(w.seq_lens[b])
        nblk = -(-Lb // bs)
        for h in range(4):
            Kh = _f64(w.k_cache[b, h // 2, :Lb])
            means = torch.stack([Kh[j * bs:min((j + 1) * bs, Lb)].mean(0) for j in range(nblk)])
            rb = (means @ _f64(w.q[b, 0, h])).numpy() / math.sqrt(128)
            kept_b = np.sort(np.lexsort((np.arange(nblk), -rb))[:min(top, nblk)])
            got_b = r["block_idx"][b, 0, h]
            assert np.array_equal(got_b[:len(kept_b)], kept_b) and np.all(got_b[len(kept_b):] == -1)
            cand = np.concatenate([np.arange(j * bs, min((j + 1) * bs, Lb)) for j in kept_b])
            sc = s_all[b, 0, h, cand]
            order = np.lexsort((cand, -sc))
            kk = min(k, len(cand))
            sel = np.sort(cand[order[:kk]])
            got = r["idx"][b, 0, h]
            assert np.array_equal(got[:kk], sel) and np.all(got[kk:] == -1)
            p = torch.softmax(torch.from_numpy(s_all[b, 0, h, sel]), dim=0).numpy()
            want = (p[:, None] * _f64(w.v_cache[b, h // 2, sel]).numpy()).sum(0)
            np.testing.assert_allclose(r["out"][b, 0, h], want, rtol=1e-12, atol=1e-12)
            pc = torch.softmax(torch.from_numpy(sc), dim=0).numpy()
            assert abs(r["tail"][b, 0, h] - (1.0 - pc[order[:kk]].sum())) < 1e-12


# ----------------------------------------------------------------------------- lightning indexer

def _torch_index_scores(w, q_idx, w_idx, k_idx):
    """Sum_j w_j ReLU(<q_idx_j, k_idx_i>) in fp64 via torch, [B, Q, L] (-inf where not visible)."""
    dots = torch.einsum("bqjc,blc->bqjl", _f64(q_idx), _f64(torch.nan_to_num(k_idx.float())))
    s = (w_idx.double()[..., None] * torch.relu(dots)).sum(2)
    return s.masked_fill(~_visible_mask(w)[:, 0], -math.inf).numpy()


@pytest.mark.parametrize("Q,H_I,d_I,k", [(1, 4, 64, 40), (3, 8, 32, 100), (2, 1, 128, 7)])
def test_indexer_selection_and_attention_brute_force(Q, H_I, d_I, k):
    w = workloads.make_workload(2, Q, 8, 2, 300, dtype="bf16", seq_lens=[300, 140], seed=81)
    qi, wi, ki = workloads.make_indexer_inputs(w, H_I, d_I)
    r = oracle.indexer_attn(w, qi, wi, ki, k)
    I = _torch_index_scores(w, qi, wi, ki)
    s = torch_scores(w)
    for b in range(2):
        for qp in range(Q):
            vis = int(w.seq_lens[b]) - Q + qp + 1
            sel = lexsort_topk(I[b, qp], k)
            got = r["idx"][b, qp]
            assert np.array_equal(got[:len(sel)], sel) and np.all(got[len(sel):] == -1)
            for h in range(8):
                p = torch.softmax(torch.from_numpy(s[b, qp, h, sel]), dim=0).numpy()
                want = (p[:, None] * _f64(w.v_cache[b, h // 4, sel]).numpy()).sum(0)
                np.testing.assert_allclose(r["out"][b, qp, h], want, rtol=1e-12, atol=1e-12)
            assert vis >= 1


def test_indexer_keeping_every_token_is_dense_attention():
    w = workloads.make_workload(2, 2, 8, 4, 120, dtype="f32", seq_lens=[120, 33], seed=82)
    qi, wi, ki = workloads.make_indexer_inputs(w, 4, 64)
    r = oracle.indexer_attn(w, qi, wi, ki, 120)
    np.testing.assert_allclose(r["out"], dense_sdpa(w), rtol=1e-12, atol=1e-12)
