// Select step (device code, included by the kernels that run it): for one
// query row, the k highest-scoring visible positions
// (ties at the k-th score go to the lower position), in ascending position
// order, together with the softmax statistics the attention step needs.
//
// "Top-K Selection: retaining the K historical positions with the highest
// scores" ("Evolution of Sparse Attention in Long-Context LLMs", section 2);
// the discarded mass is the Top-k tail mass of "A Mathematical Theory of
// Top-k Sparse Attention via Total Variation Distance" (abstract).
//
// One CTA (16 or 32 warps) per row; every warp owns a contiguous segment of
// the row, lane l reading positions l, l + 32, ... of it, so a warp compacts
// 32 consecutive positions at a time with one ballot.  Ranks are taken on
// order-preserving uint32 keys with -0 folded into +0 (canon_key), so key
// order is float order and a key threshold is also a float threshold.  The
// row is read from L2 (the scores were just written) once, after a sample:
//   sample  the maximum and the histogram of the top 11 key bits of every
//           eighth group of 32 positions (every position of a short row);
//           with the next 11 key bits of the sample keys inside the coarse
//           bin, this gives lo_t, the sample key of the k-th key's sample
//           rank pushed down by 5 binomial standard deviations (to 2^10
//           keys): below the k-th score with high probability;
//   pass    the row maximum m, sum_all e^{s - m_s} against the sample maximum
//           m_s (rescaled to m afterwards), and every score >= lo_t appended
//           with its position to a per-warp list in position order (one
//           ballot per 32 positions) -- a little more than k entries;
//   the exact k-th key T among the list entries by radix levels of up to 11
//           bits over the keys between lo_t and m, and how many of the keys
//           equal to T are kept (the lowest positions);
//   emit    from the lists only: every kept entry (s > T, or s = T among the
//           first ties) to its final ascending slot, with Z_k over the kept
//           terms; Z_tail = sum_all - Z_k, the tail mass Z_tail / (Z_k + Z_tail).
// A row the sample holds whole (at most 32 kS positions per warp) skips the
// pass and the lists when the sample histogram settles the k-th score
// (select_short).  If fewer than k scores reach lo_t, a warp's list
// overflows, or the sample maximum lies too far below the row maximum for the
// sum against it, the row falls back to three exact histogram passes and an
// ordered compaction pass over the row.
#pragma once

#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace tka {

namespace {

// A row is taken by one CTA: 1024 threads when there are no more rows than
// SMs (one row per SM), else 512 threads so that two rows share an SM.  Up to
// 32 warps: per-warp words are reduced by one warp, lane w reading warp w's.
constexpr int kU = 8;                // scores per lane per streamed chunk (two chunks in flight)
constexpr int kS = 8;                // sampled groups of 32 positions per warp (held in registers)

constexpr int kBatch = 8;  // float4 loads in flight per thread

// Calls f(i, s[i]) for every i < n, 4 * kBatch elements per thread per round.
template <typename F>
__device__ __forceinline__ void visit_row(const float *s, int n, F &&f) {
    const int n4 = n >> 2;
    const float4 *s4 = reinterpret_cast<const float4 *>(s);
    const int stride = blockDim.x;
    int i = threadIdx.x;
    for (; i + (kBatch - 1) * stride < n4; i += kBatch * stride) {
        float4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; u++) v[u] = __ldcg(s4 + i + u * stride);
#pragma unroll
        for (int u = 0; u < kBatch; u++) {
            const int e = 4 * (i + u * stride);
            f(e, v[u].x);
            f(e + 1, v[u].y);
            f(e + 2, v[u].z);
            f(e + 3, v[u].w);
        }
    }
    for (; i < n4; i += stride) {
        const float4 v = __ldcg(s4 + i);
        f(4 * i, v.x);
        f(4 * i + 1, v.y);
        f(4 * i + 2, v.z);
        f(4 * i + 3, v.w);
    }
    for (int j = 4 * n4 + threadIdx.x; j < n; j += stride) f(j, __ldcg(s + j));
}

// Loads 4 consecutive positions i0..i0+3 (zeros past n).
__device__ __forceinline__ void load4(const float *s, int i0, int n, float (&x)[4]) {
    if (i0 + 3 < n) {
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(s + i0));
        x[0] = v.x;
        x[1] = v.y;
        x[2] = v.z;
        x[3] = v.w;
    } else {
#pragma unroll
        for (int j = 0; j < 4; j++) x[j] = i0 + j < n ? __ldcg(s + i0 + j) : 0.f;
    }
}

struct SelectSmem {
    uint32_t *hist;  // [2048]
    uint32_t *tmp;   // [32]
    float *red;      // [64]
    uint32_t *scal;  // [2]: bin, above
};

// Writes stats, tail and counter of a finished row.
__device__ __forceinline__ void finish_row(const SelectParams &p, int row, float m, float zk, float zt,
                                           uint32_t written, uint32_t kept, const SelectSmem &sm) {
    {
        // both block sums with one pair of barriers
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
        zk = warp_sum(zk);
        zt = warp_sum(zt);
        __syncthreads();
        if (lane == 0) {
            sm.red[2 * warp] = zk;
            sm.red[2 * warp + 1] = zt;
        }
        __syncthreads();
        zk = warp_sum(lane < nw ? sm.red[2 * lane] : 0.f);
        zt = fmaxf(warp_sum(lane < nw ? sm.red[2 * lane + 1] : 0.f), 0.f);  // formed as total - kept: >= 0
    }
    if (threadIdx.x == 0) {
        if (written != kept) raise_status(p.status, TKA_DEV_INTERNAL);
        p.stats[row] = make_float4(m, zk, zt, 0.f);
        if (p.tail) p.tail[row] = zt / (zk + zt);
        p.counters[row] = 0u;
    }
}

// k >= visible keys: every position is kept, in order.
__device__ void select_all(const SelectParams &p, int row, int vis, float m, const SelectSmem &sm) {
    const float *s = p.scores + (size_t)row * p.ld;
    int32_t *idx = p.idx + (size_t)row * p.k;
    float *wv = p.w + (size_t)row * p.k;
    float zk = 0.f;
    visit_row(s, vis, [&](int i, float x) {
        const float e = __expf(x - m);
        idx[i] = i;
        wv[i] = e;
        zk += e;
    });
    for (int j = vis + threadIdx.x; j < p.k; j += blockDim.x) idx[j] = -1;
    finish_row(p, row, m, zk, 0.f, vis, vis, sm);
}

// Three histogram passes and an ordered compaction pass (too many candidates
// in the boundary bin).
__device__ void select_multipass(const SelectParams &p, int row, int vis, const SelectSmem &sm) {
    const float *s = p.scores + (size_t)row * p.ld;
    const int k = p.k;
    uint32_t *hist = sm.hist;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    float m = -INFINITY;
    visit_row(s, vis, [&](int, float x) {
        m = fmaxf(m, x);
        atomicAdd(&hist[canon_key(x) >> 21], 1u);
    });
    m = block_max(m, sm.red);
    __syncthreads();
    __syncthreads();  // the histogram is complete
    block_find_bins<2048>(hist, (uint32_t)k, (uint32_t)k, sm.tmp, sm.scal);
    const uint32_t b1 = sm.scal[0];
    uint32_t above = sm.scal[1];
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    visit_row(s, vis, [&](int, float x) {
        const uint32_t key = canon_key(x);
        if ((key >> 21) == b1) atomicAdd(&hist[(key >> 10) & 0x7ffu], 1u);
    });
    __syncthreads();
    __syncthreads();  // the histogram is complete
    block_find_bins<2048>(hist, (uint32_t)k - above, (uint32_t)k - above, sm.tmp, sm.scal);
    const uint32_t b2 = sm.scal[0];
    above += sm.scal[1];
    const uint32_t pre = (b1 << 11) | b2;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    visit_row(s, vis, [&](int, float x) {
        const uint32_t key = canon_key(x);
        if ((key >> 10) == pre) atomicAdd(&hist[key & 0x3ffu], 1u);
    });
    __syncthreads();
    __syncthreads();  // the histogram is complete
    block_find_bins<1024>(hist, (uint32_t)k - above, (uint32_t)k - above, sm.tmp, sm.scal);
    const uint32_t b3 = sm.scal[0];
    above += sm.scal[1];
    const uint32_t T = (pre << 10) | b3, n_eq = hist[b3], r_eq = (uint32_t)k - above;
    const bool rank_ties = n_eq != r_eq;

    int32_t *idx = p.idx + (size_t)row * k;
    float *wv = p.w + (size_t)row * k;
    uint32_t base_sel = 0u, base_eq = 0u;
    float zk = 0.f, zt = 0.f;
    for (int tile = 0; tile < vis; tile += 4 * blockDim.x) {
        const int i0 = tile + 4 * threadIdx.x;
        float x[4];
        load4(s, i0, vis, x);
        uint32_t key[4], n_eq_t = 0u;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            key[j] = canon_key(x[j]);
            if (i0 + j < vis && key[j] == T) n_eq_t++;
        }
        uint32_t eq_total = 0u, eq_rank = base_eq;
        if (rank_ties) eq_rank += block_excl_scan(n_eq_t, sm.tmp, &eq_total);
        bool sel[4];
        uint32_t n_sel_t = 0u;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            bool v = i0 + j < vis;
            if (v) v = key[j] == T ? (!rank_ties || eq_rank++ < r_eq) : key[j] > T;
            sel[j] = v;
            n_sel_t += v;
        }
        uint32_t sel_total;
        uint32_t pos = base_sel + block_excl_scan(n_sel_t, sm.tmp, &sel_total);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            if (i0 + j >= vis) continue;
            const float e = __expf(x[j] - m);
            if (sel[j]) {
                if (pos < (uint32_t)k) {  // always true unless the search above is wrong
                    idx[pos] = i0 + j;
                    wv[pos] = e;
                }
                pos++;
                zk += e;
            } else {
                zt += e;
            }
        }
        base_sel += sel_total;
        base_eq += eq_total;
    }
    finish_row(p, row, m, zk, zt, base_sel, (uint32_t)k, sm);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Entries of a warp's ordered list (score, position) -- enough for twice the
// kept positions of an evenly spread row, at least 64 -- plus one slot that
// absorbs the writes past a full list.
__host__ __device__ constexpr int list_cap_for(int k, int warps) {
    const int c = (2 * k + 1024 + warps - 1) / warps;
    return ((c < 64 ? 64 : c) + 31) & ~31;
}

__host__ __device__ constexpr size_t smem_words_for(int k, int warps) {
    return 2048 + 104 + (size_t)warps * 8 + 2 * (size_t)warps * (list_cap_for(k, warps) + 1);
}

// A position known to lie inside the streamed range (a compile-time true).
struct InRange {
    __device__ __forceinline__ constexpr operator bool() const { return true; }
};

// Streams positions [lo, hi) of s through f(x, pos, valid) in chunks of
// 32 kU positions (lane l: pos = chunk start + 32 u + l), the next chunk's
// loads in flight while the current one is processed.  valid is the
// compile-time constant InRange{} for every chunk that lies wholly inside the
// range; past the range x is -inf.
// kEvictFirst: the scores of all rows exceed L2, so part of them was pushed
// out by the ones written after; evict-first loads keep the lines still
// resident from being pushed out by the ones this read brings back.
template <bool kEvictFirst>
__device__ __forceinline__ float ld_score(const float *a, uint64_t pol) {
    if constexpr (kEvictFirst)
        return ld_l2_hint(a, pol);
    else
        return __ldcg(a);
}

template <bool kEvictFirst, typename F>
__device__ __forceinline__ void stream_range(const float *s, int lo, int hi, int lane, F &&f) {
    const int nch = (hi - lo + 32 * kU - 1) / (32 * kU);
    float a[kU], b[kU];
    const uint64_t pol = kEvictFirst ? l2_evict_first() : 0ull;
    auto load = [&](float(&x)[kU], int c) {
        const int p0 = lo + c * 32 * kU + lane;
        if (lo + (c + 1) * 32 * kU <= hi) {
#pragma unroll
            for (int u = 0; u < kU; u++) x[u] = ld_score<kEvictFirst>(s + p0 + 32 * u, pol);
        } else {
#pragma unroll
            for (int u = 0; u < kU; u++)
                x[u] = p0 + 32 * u < hi ? ld_score<kEvictFirst>(s + p0 + 32 * u, pol) : -INFINITY;
        }
    };
    auto run = [&](float(&x)[kU], int c) {
        const int p0 = lo + c * 32 * kU + lane;
        if (lo + (c + 1) * 32 * kU <= hi) {
#pragma unroll
            for (int u = 0; u < kU; u++) f(x[u], p0 + 32 * u, InRange{});
        } else {
#pragma unroll
            for (int u = 0; u < kU; u++) f(x[u], p0 + 32 * u, p0 + 32 * u < hi);
        }
    };
    if (nch > 0) load(a, 0);
    for (int c = 0; c < nch; c += 2) {
        if (c + 1 < nch) load(b, c + 1);
        run(a, c);
        if (c + 1 < nch) {
            if (c + 2 < nch) load(a, c + 2);
            run(b, c + 1);
        }
    }
}

// A 64-bit shared-memory store {x, y} made only when p holds.
__device__ __forceinline__ void st_shared_v2_if(bool p, void *a, uint32_t x, uint32_t y) {
    asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %0, 0;\n @q st.shared.v2.u32 [%1], {%2, %3};\n}\n" ::"r"(
                     (uint32_t)p),
                 "r"(static_cast<uint32_t>(__cvta_generic_to_shared(a))), "r"(x), "r"(y)
                 : "memory");
}

// The select step of a row the sample holds whole (lane l of a warp holding
// positions lo + l + 32 j of the warp's segment [lo, hi) in sv[j]): the sample
// histogram's bin b* of the k-th score (scal[0], with scal[1] scores above it)
// bounds it exactly, so the kept scores are those in bins above b* and, in b*,
// either all of it (when that completes k) or, with at most 32 scores there,
// those above the exact k-th key T plus the lowest-positioned ties at T.  They
// are emitted straight from the registers: no second read of the row, no
// lists.  Returns false, having written nothing, when b* holds more than 32
// scores and is not kept whole (the caller takes the general route).
template <int kThreads>
__device__ __forceinline__ bool select_short(const SelectParams &p, int row, int lo, int hi, const float (&sv)[kS],
                                             float min_s, float m_s, float scale_s, uint32_t *wstat,
                                             const SelectSmem &sm) {
    constexpr int kWarps = kThreads / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = lanemask_lt();
    const int k = p.k;
    auto wword = [&](int f) { return lane < kWarps ? wstat[lane * 8 + f] : 0u; };
    // the sample histogram's bin function, expression for expression
    auto binv = [&](float x) { return (uint32_t)min(2047, (int)((x - min_s) * scale_s)); };
    const uint32_t bstar = sm.scal[0], c_star = sm.hist[bstar], r = (uint32_t)k - sm.scal[1];  // 1 <= r <= c_star
    const bool by_bin = r == c_star;
    if (!by_bin && c_star > 32u) {
        __syncthreads();  // every thread has read the histogram before the caller clears it
        return false;
    }
    uint32_t T_key = 0u, r_eq = 0u;
    if (!by_bin) {
        uint32_t *cand = sm.tmp;  // [32]: free after the bin search
        if (threadIdx.x == 0) sm.scal[4] = 0u;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kS; j++)
            if (lo + 32 * j + lane < hi && binv(sv[j]) == bstar) cand[atomicAdd(&sm.scal[4], 1u)] = canon_key(sv[j]);
        __syncthreads();
        if (warp == 0) {
            const uint32_t mine = lane < (int)c_star ? cand[lane] : 0u;
            uint32_t g = 0u, e = 0u;
            for (uint32_t j = 0; j < c_star; j++) {
                const uint32_t o = cand[j];
                g += o > mine;
                e += o == mine;
            }
            const uint32_t hit = __ballot_sync(0xffffffffu, lane < (int)c_star && g < r && r <= g + e);
            const int L = hit ? __ffs(hit) - 1 : 0;
            const uint32_t tk = __shfl_sync(0xffffffffu, mine, L), tg = __shfl_sync(0xffffffffu, g, L);
            if (lane == 0) {
                sm.scal[5] = tk;
                sm.scal[6] = r - tg;
                if (!hit) raise_status(p.status, TKA_DEV_INTERNAL);
            }
        }
        __syncthreads();
        T_key = sm.scal[5];
        r_eq = sm.scal[6];
    }
    auto above = [&](float x) { return by_bin ? binv(x) >= bstar : canon_key(x) > T_key; };
    auto tie = [&](float x) { return !by_bin && canon_key(x) == T_key; };

    // ---- per warp: kept scores above T and ties at T, then output offsets
    {
        uint32_t g = 0u, t = 0u;
#pragma unroll
        for (int j = 0; j < kS; j++) {
            if (lo + 32 * j + lane < hi) {
                g += above(sv[j]);
                t += tie(sv[j]);
            }
        }
        g = warp_sum(g);
        t = warp_sum(t);
        if (lane == 0) {
            wstat[warp * 8 + 5] = g;
            wstat[warp * 8 + 6] = t;
        }
    }
    __syncthreads();
    uint32_t out_run, tie_run, n_eq;
    {
        const uint32_t tie_l = wword(6);
        const uint32_t tie_incl = warp_incl_scan(tie_l), tie_excl = tie_incl - tie_l;
        const uint32_t kept_l = wword(5) + (r_eq > tie_excl ? min(tie_l, r_eq - tie_excl) : 0u);
        const uint32_t out_incl = warp_incl_scan(kept_l);
        out_run = __shfl_sync(0xffffffffu, out_incl - kept_l, warp);
        tie_run = __shfl_sync(0xffffffffu, tie_excl, warp);
        n_eq = __shfl_sync(0xffffffffu, tie_incl, 31);
    }
    const bool rank_ties = r_eq < n_eq;
    const uint32_t out_begin = out_run;

    // ---- emit in position order; Z_k over the kept, Z_tail over the rest
    int32_t *idx = p.idx + (size_t)row * k;
    float *wv = p.w + (size_t)row * k;
    const float m = m_s;  // the sample is the whole row
    const float m_l2e = m * kLog2e;
    float zk = 0.f, zt = 0.f;
#pragma unroll
    for (int j = 0; j < kS; j++) {
        const int pos = lo + 32 * j + lane;
        const bool in = pos < hi;
        const float xv = sv[j];
        bool sel = in && above(xv);
        if (rank_ties) {
            const bool t = in && tie(xv);
            const uint32_t tb = __ballot_sync(0xffffffffu, t);
            sel = sel || (t && tie_run + __popc(tb & lt) < r_eq);
            tie_run += __popc(tb);
        } else {
            sel = sel || (in && tie(xv));
        }
        const uint32_t sb = __ballot_sync(0xffffffffu, sel);
        if (in) {
            const float ew = exp2_approx(fmaf(xv, kLog2e, -m_l2e));
            if (sel) {
                const uint32_t o = out_run + __popc(sb & lt);
                if (o < (uint32_t)k) {  // always true unless the counts above are wrong
                    idx[o] = pos;
                    wv[o] = ew;
                }
                zk += ew;
            } else {
                zt += ew;
            }
        }
        out_run += __popc(sb);
    }
    zk = warp_sum(zk);
    zt = warp_sum(zt);
    if (lane == 0) {  // words 1-3: words 5 and 6 may still be read by a slower warp's scan
        wstat[warp * 8 + 1] = __float_as_uint(zk);
        wstat[warp * 8 + 2] = out_run - out_begin;
        wstat[warp * 8 + 3] = __float_as_uint(zt);
    }
    __syncthreads();
    if (warp == 0) {
        const float zk_row = warp_sum(lane < kWarps ? __uint_as_float(wstat[lane * 8 + 1]) : 0.f);
        const float zt_row = warp_sum(lane < kWarps ? __uint_as_float(wstat[lane * 8 + 3]) : 0.f);
        const uint32_t written = warp_sum(wword(2));
        if (lane == 0) {
            if (written != (uint32_t)k) raise_status(p.status, TKA_DEV_INTERNAL);
            p.stats[row] = make_float4(m, zk_row, zt_row, 0.f);
            if (p.tail) p.tail[row] = zt_row / (zk_row + zt_row);
            p.counters[row] = 0u;
        }
    }
    return true;
}

// The select step of one row by the whole CTA (kThreads threads, the dynamic
// shared memory select_smem_bytes(kThreads, p.k)); kEvictFirst as for
// ld_score.
template <int kThreads, bool kEvictFirst = false>
__device__ void select_row(const SelectParams &p, int row) {
    constexpr int kWarps = kThreads / 32;
    static_assert(kWarps <= 32 && kThreads % 32 == 0, "at most 32 whole warps");
    extern __shared__ __align__(16) uint32_t dyn[];
    SelectSmem sm;
    sm.hist = dyn;                                        // [2048]
    sm.tmp = dyn + 2048;                                  // [32]
    sm.red = reinterpret_cast<float *>(dyn + 2048 + 32);  // [64]
    sm.scal = dyn + 2048 + 96;                            // [8]
    uint32_t *wstat = dyn + 2048 + 104;                   // [kWarps][8]
    const int cap = list_cap_for(p.k, kWarps);
    uint2 *lists = reinterpret_cast<uint2 *>(wstat + kWarps * 8);  // [kWarps][cap + 1] {score bits, position}

    const int b = row / (p.Q * p.Hq), qpos = (row / p.Hq) % p.Q;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) {
        if (threadIdx.x == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    const int vis = p.row_len ? p.row_len[row] : visible_keys(seq_len, p.Q, qpos);
    const int k = p.k;
    const float *s = p.scores + (size_t)row * p.ld;
    if (k >= vis) {  // every visible key is kept
        float m = -INFINITY;
        visit_row(s, vis, [&](int, float x) { m = fmaxf(m, x); });
        m = block_max(m, sm.red);
        select_all(p, row, vis, m, sm);
        return;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = lanemask_lt();
    // this warp's contiguous segment [lo, hi) of the row
    const int seg = (((vis + kWarps - 1) / kWarps) + 31) & ~31;
    const int lo = min(vis, warp * seg), hi = min(vis, lo + seg);
    // word f of the lane-th warp (0 past the last warp), for warp-wide reductions
    auto wword = [&](int f) { return lane < kWarps ? wstat[lane * 8 + f] : 0u; };

    // ---- sample: up to kS groups of 32 positions per warp, evenly spaced over
    // its segment (every group of a segment of at most kS groups), kept in
    // registers; their minimum, maximum and a histogram in 2048 bins of equal
    // width between the two give lo_t, a value at or below the sample's
    // rank-(k * nsample / vis) score pushed down by 5 binomial standard
    // deviations (on an unsampled row, at or below the k-th score itself)
    const int gstep = max(1, ((seg >> 5) + kS - 1) / kS);
    const bool sampled = gstep > 1;
    float sv[kS];
    float smin = INFINITY, smax = -INFINITY;
    uint32_t nsample = 0u;
#pragma unroll
    for (int j = 0; j < kS; j++) {
        const int pos = lo + 32 * j * gstep + lane;
        sv[j] = pos < hi ? ld_score<kEvictFirst>(s + pos, kEvictFirst ? l2_evict_first() : 0ull) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kS; j++) {
        if (lo + 32 * j * gstep + lane < hi) {
            smin = fminf(smin, sv[j]);
            smax = fmaxf(smax, sv[j]);
            nsample++;
        }
    }
    nsample = warp_sum(nsample);
    smin = warp_min(smin);
    smax = warp_max(smax);
    if (lane == 0) {
        wstat[warp * 8 + 0] = nsample;
        wstat[warp * 8 + 1] = __float_as_uint(smin);
        wstat[warp * 8 + 2] = __float_as_uint(smax);
    }
    for (int i = threadIdx.x; i < 2048; i += kThreads) sm.hist[i] = 0u;
    __syncthreads();
    const uint32_t total_sample = warp_sum(wword(0));
    const float min_s = warp_min(lane < kWarps ? __uint_as_float(wstat[lane * 8 + 1]) : INFINITY);
    const float m_s = warp_max(lane < kWarps ? __uint_as_float(wstat[lane * 8 + 2]) : -INFINITY);
    const float scale_s = m_s > min_s ? 2048.f / (m_s - min_s) : 0.f;
#pragma unroll
    for (int j = 0; j < kS; j++)
        if (lo + 32 * j * gstep + lane < hi)
            atomicAdd(&sm.hist[min(2047, (int)((sv[j] - min_s) * scale_s))], 1u);
    __syncthreads();
    float lo_t;
    {
        const float ks = (float)k * (float)total_sample / (float)vis;
        const float margin = sampled ? 5.f * sqrtf(ks) + 4.f : 0.f;
        const uint32_t need = (uint32_t)fminf((float)total_sample, fmaxf(1.f, ceilf(ks + margin)));
        block_find_bins<2048>(sm.hist, need, need, sm.tmp, sm.scal);
        const uint32_t b_lo = sm.scal[0];
        // one bin lower than the bin's bottom edge: below every sample score in it
        lo_t = b_lo > 0u ? min_s + (float)(b_lo - 1u) / scale_s : -INFINITY;
    }
    // a row the sample holds whole: the bin search above bounds the k-th score exactly
    if (!sampled && select_short<kThreads>(p, row, lo, hi, sv, min_s, m_s, scale_s, wstat, sm)) return;
    for (int i = threadIdx.x; i < 2048; i += kThreads) sm.hist[i] = 0u;  // for the list histogram

    // ---- the one pass over the row: its maximum, sum e^{s - m_s} against the
    // sample maximum, and every score >= lo_t appended with its position to
    // this warp's list in position order (one ballot per 32 positions; a full
    // list keeps counting, its extra writes go to the spare slot)
    uint2 *my_list = lists + warp * (cap + 1);
    const float ms_l2e = m_s * kLog2e;
    float m_lane = -INFINITY, zall = 0.f;
    uint32_t nl = 0u;
    stream_range<kEvictFirst>(s, lo, hi, lane, [&](float x, int pos, auto valid) {
        m_lane = fmaxf(m_lane, x);
        zall += exp2_approx(fmaf(x, kLog2e, -ms_l2e));
        const bool sel = valid && x >= lo_t;
        const uint32_t bal = __ballot_sync(0xffffffffu, sel);
        const uint32_t slot = min(nl + __popc(bal & lt), (uint32_t)cap);
        st_shared_v2_if(sel, my_list + slot, __float_as_uint(x), (uint32_t)pos);
        nl += __popc(bal);
    });
    {
        const float mw = warp_max(m_lane);
        const float zw = warp_sum(zall);
        if (lane == 0) {
            wstat[warp * 8 + 3] = nl;
            wstat[warp * 8 + 4] = __float_as_uint(mw);
            wstat[warp * 8 + 5] = __float_as_uint(zw);
        }
    }
    __syncthreads();
    const float m = warp_max(lane < kWarps ? __uint_as_float(wstat[lane * 8 + 4]) : -INFINITY);  // row maximum
    const uint32_t total = warp_sum(wword(3));
    const bool overflow = __any_sync(0xffffffffu, wword(3) > (uint32_t)cap);
    if (overflow || total < (uint32_t)k || (m - m_s) * kLog2e > 96.f) {
        // a warp's list is full, the sample misled, or the sum against the
        // sample maximum could overflow: take the exact multi-pass route
        __syncthreads();
        select_multipass(p, row, vis, sm);
        return;
    }
    // sum_all e^{s - m}
    const float z_all =
        warp_sum(lane < kWarps ? __uint_as_float(wstat[lane * 8 + 5]) : 0.f) * exp2_approx((m_s - m) * kLog2e);

    // ---- which list entries are kept.  Either every entry whose bin (2048
    // bins of equal width between lo_t and m) is at or above the bin b* that
    // holds the k-th score, when b* is kept whole; or the rule s > T, or
    // s == T among the first r_eq ties, with T the exact k-th score.
    bool by_bin = false;
    uint32_t bstar = 0u;
    const float scale1 = m > lo_t && lo_t > -INFINITY ? 2048.f / (m - lo_t) : 0.f;
    auto bin1 = [&](float x) { return min(2047u, (uint32_t)((x - lo_t) * scale1)); };
    uint32_t T_key = 0u, r_eq = 0u;
    bool resolved = false;
    if (scale1 > 0.f) {
        for (uint32_t i = lane; i < nl; i += 32) atomicAdd(&sm.hist[bin1(__uint_as_float(my_list[i].x))], 1u);
        if (threadIdx.x == 0) sm.scal[4] = 0u;  // entries of b* collected below
        __syncthreads();
        block_find_bins<2048>(sm.hist, (uint32_t)k, (uint32_t)k, sm.tmp, sm.scal);
        bstar = sm.scal[0];
        const uint32_t c_star = sm.hist[bstar], r = (uint32_t)k - sm.scal[1];  // 1 <= r <= c_star
        if (r == c_star) {
            by_bin = true;
            resolved = true;
        } else if (c_star <= 32u) {
            uint32_t *cand = sm.tmp;  // [32]: the tmp words are free until the next block search
            for (uint32_t i = lane; i < nl; i += 32) {
                const float xv = __uint_as_float(my_list[i].x);
                if (bin1(xv) == bstar) cand[atomicAdd(&sm.scal[4], 1u)] = canon_key(xv);
            }
            __syncthreads();
            if (warp == 0) {
                const uint32_t mine = lane < (int)c_star ? cand[lane] : 0u;
                uint32_t g = 0u, e = 0u;
                for (uint32_t j = 0; j < c_star; j++) {
                    const uint32_t o = cand[j];
                    g += o > mine;
                    e += o == mine;
                }
                const uint32_t hit = __ballot_sync(0xffffffffu, lane < (int)c_star && g < r && r <= g + e);
                const int L = hit ? __ffs(hit) - 1 : 0;
                const uint32_t tk = __shfl_sync(0xffffffffu, mine, L), tg = __shfl_sync(0xffffffffu, g, L);
                if (lane == 0) {
                    sm.scal[5] = tk;
                    sm.scal[6] = r - tg;
                    if (!hit) raise_status(p.status, TKA_DEV_INTERNAL);
                }
            }
            __syncthreads();
            T_key = sm.scal[5];
            r_eq = sm.scal[6];
            resolved = true;
        }
    }
    if (!resolved) {
        // many scores share b*, or no bins could be formed: radix levels of
        // up to 11 bits over the keys of the list entries, from the smallest
        // possible to that of m
        __syncthreads();  // every thread has read the words of the pass above
        uint32_t base = lo_t > -INFINITY ? canon_key(lo_t) : 0u, gt = 0u;
        const uint32_t span_m1 = canon_key(m) - base;
        int rem = span_m1 ? 32 - __clz(span_m1) : 0;
        while (rem > 0) {
            const int sh = rem > 11 ? rem - 11 : 0;
            __syncthreads();
            for (int i = threadIdx.x; i < 2048; i += kThreads) sm.hist[i] = 0u;
            __syncthreads();
            for (uint32_t i = lane; i < nl; i += 32) {
                const uint32_t d = canon_key(__uint_as_float(my_list[i].x)) - base;
                if ((rem >= 32 || d < (1u << rem)) && (d >> sh) < 2048u) atomicAdd(&sm.hist[d >> sh], 1u);
            }
            __syncthreads();
            block_find_bins<2048>(sm.hist, (uint32_t)k - gt, (uint32_t)k - gt, sm.tmp, sm.scal);
            gt += sm.scal[1];
            base += sm.scal[0] << sh;
            rem = sh;
        }
        T_key = base;
        r_eq = (uint32_t)k - gt;
    }
    const float T_f = key_float(T_key);
    const float m_l2e = m * kLog2e;
    auto above = [&](float x) { return by_bin ? bin1(x) >= bstar : x > T_f; };
    auto tie = [&](float x) { return !by_bin && x == T_f; };

    // ---- per warp: kept entries above T and ties at T, then output offsets
    {
        uint32_t g = 0u, t = 0u;
        for (uint32_t i = lane; i < nl; i += 32) {
            const float xv = __uint_as_float(my_list[i].x);
            g += above(xv);
            t += tie(xv);
        }
        g = warp_sum(g);
        t = warp_sum(t);
        if (lane == 0) {
            wstat[warp * 8 + 5] = g;
            wstat[warp * 8 + 6] = t;
        }
    }
    __syncthreads();
    uint32_t out_run, tie_run, n_eq;
    {
        const uint32_t tie_l = wword(6);
        const uint32_t tie_incl = warp_incl_scan(tie_l), tie_excl = tie_incl - tie_l;
        const uint32_t kept_l = wword(5) + (r_eq > tie_excl ? min(tie_l, r_eq - tie_excl) : 0u);
        const uint32_t out_incl = warp_incl_scan(kept_l);
        out_run = __shfl_sync(0xffffffffu, out_incl - kept_l, warp);
        tie_run = __shfl_sync(0xffffffffu, tie_excl, warp);
        n_eq = __shfl_sync(0xffffffffu, tie_incl, 31);
    }
    const bool rank_ties = r_eq < n_eq;
    const uint32_t out_begin = out_run;

    // ---- emit every kept entry straight to its final ascending slot
    int32_t *idx = p.idx + (size_t)row * k;
    float *wv = p.w + (size_t)row * k;
    float zk = 0.f;
    for (uint32_t i0 = 0; i0 < nl; i0 += 32) {
        const uint32_t i = i0 + lane;
        const uint2 e = i < nl ? my_list[i] : make_uint2(__float_as_uint(-INFINITY), 0u);
        const float xv = __uint_as_float(e.x);
        const bool in = i < nl;
        bool sel = in && above(xv);
        if (rank_ties) {
            const bool t = in && tie(xv);
            const uint32_t tb = __ballot_sync(0xffffffffu, t);
            sel = sel || (t && tie_run + __popc(tb & lt) < r_eq);
            tie_run += __popc(tb);
        } else {
            sel = sel || (in && tie(xv));
        }
        const uint32_t sb = __ballot_sync(0xffffffffu, sel);
        if (sel) {
            const float ew = exp2_approx(fmaf(xv, kLog2e, -m_l2e));
            const uint32_t o = out_run + __popc(sb & lt);
            if (o < (uint32_t)k) {  // always true unless the counts above are wrong
                idx[o] = (int32_t)e.y;
                wv[o] = ew;
            }
            zk += ew;
        }
        out_run += __popc(sb);
    }
    zk = warp_sum(zk);
    if (lane == 0) {
        // words 1 and 2 (the sample's, read long before): words 5 and 6 may
        // still be read by a slower warp's offset scan above
        wstat[warp * 8 + 1] = __float_as_uint(zk);
        wstat[warp * 8 + 2] = out_run - out_begin;
    }
    __syncthreads();
    if (warp == 0) {
        const float zk_row = warp_sum(lane < kWarps ? __uint_as_float(wstat[lane * 8 + 1]) : 0.f);
        const uint32_t written = warp_sum(wword(2));
        if (lane == 0) {
            const float zt = fmaxf(z_all - zk_row, 0.f);  // formed as total - kept: >= 0
            if (written != (uint32_t)k) raise_status(p.status, TKA_DEV_INTERNAL);
            p.stats[row] = make_float4(m, zk_row, zt, 0.f);
            if (p.tail) p.tail[row] = zt / (zk_row + zt);
            p.counters[row] = 0u;
        }
    }
}

}  // namespace
}  // namespace tka
