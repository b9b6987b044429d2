// Select step: for one query row, the k highest-scoring visible positions
// (ties at the k-th score go to the lower position), in ascending position
// order, together with the softmax statistics the attention step needs.
//
// "Top-K Selection: retaining the K historical positions with the highest
// scores" ("Evolution of Sparse Attention in Long-Context LLMs", section 2);
// the discarded mass is the Top-k tail mass of "A Mathematical Theory of
// Top-k Sparse Attention via Total Variation Distance" (abstract).
//
// One CTA (16 or 32 warps) per row; every warp owns a contiguous segment of
// the row, lane l holding positions l, l + 32, ... of it, so a warp compacts 32
// consecutive positions at a time with one ballot.  A segment of up to 32 x 32
// positions is read once and kept in registers for every pass; a longer one
// is streamed in double-buffered steps of 16 scores per lane.  Ranks are taken
// on order-preserving uint32 keys with -0 folded into +0 (canon_key), so key
// order is float order and the per-position tests below are plain float
// comparisons:
//   pass 1  the histogram of the top 11 key bits of a sample (every eighth
//           group of 32 positions) gives a bin range that holds the k-th key
//           with high probability;
//   pass 2  the one pass over the whole row: the row maximum (a running
//           maximum per lane) and sum_all e^{s-m}; scores above the range are
//           counted, keys inside it are collected (unordered) into per-warp
//           candidate lists, and every score at or above the range is
//           appended with its position to a per-warp list in position order;
//   exact radix selection over the candidates' keys, in levels of up to 11
//           bits over the key range the band spans, yields the k-th key T
//           and how many of the keys equal to T are kept (the lowest
//           positions); the bins are searched by the whole block;
//   pass 3  over the ordered lists only: the kept positions are written
//           straight to their ascending slots (ballots plus per-warp offsets)
//           with Z_k = sum_kept e^{s-m}; Z_tail = sum_all - Z_k, and the tail
//           mass is Z_tail / (Z_k + Z_tail).  A warp whose ordered list
//           overflowed tests its whole segment again instead.
// If the sampled range misses the k-th key, or a warp collects more
// candidates than fit, the row falls back to three exact histogram passes and
// an ordered compaction pass over the row.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace tka {

namespace {

// A row is taken by one CTA of kThreads threads: 1024 when the select runs
// alone (one CTA per SM), 512 when it shares the SMs with the scorer of the
// next batch chunk (a 512-thread CTA and a scorer CTA fit one SM's registers
// and shared memory together).  Up to 32 warps: per-warp words are reduced by
// one warp, lane w reading warp w's.
constexpr int kCandWords = 8192;  // candidate keys held in shared memory per row, split evenly over the warps
constexpr int kPlusWords = 6144;  // (score, position) pairs of the scores at or above the band, split likewise
constexpr int kHeld = 32;  // scores per lane held in registers (a resident segment: 32 x 32 positions)
constexpr int kStep = 16;  // scores per lane per step of a streamed segment (half the registers)
constexpr int kSampleMinLen = 16384;            // rows this long histogram a 1/8 sample in pass 1

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

// Two 32-bit shared-memory stores, both made only when p holds.
__device__ __forceinline__ void st_shared_if(bool p, void *a, uint32_t va, void *b, uint32_t vb) {
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.u32 q, %0, 0;\n @q st.shared.u32 [%1], %2;\n @q st.shared.u32 [%3], %4;\n}\n" ::"r"(
            (uint32_t)p),
        "r"(static_cast<uint32_t>(__cvta_generic_to_shared(a))), "r"(va),
        "r"(static_cast<uint32_t>(__cvta_generic_to_shared(b))), "r"(vb)
        : "memory");
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__host__ __device__ constexpr size_t smem_words(int warps) {
    return 2048 + 104 + warps * 8 + kCandWords + 2048 + 2 * kPlusWords;
}

template <int kThreads>
__global__ void __launch_bounds__(kThreads, 1024 / kThreads) select_topk(SelectParams p) {
    constexpr int kWarps = kThreads / 32;
    static_assert(kWarps <= 32 && kThreads % 32 == 0, "at most 32 whole warps");
    constexpr int kWarpCand = kCandWords / kWarps;  // a warp's candidate list
    extern __shared__ __align__(16) uint32_t dyn[];
    SelectSmem sm;
    sm.hist = dyn;                                                   // [2048]
    sm.tmp = dyn + 2048;                                             // [32]
    sm.red = reinterpret_cast<float *>(dyn + 2048 + 32);             // [64]
    sm.scal = dyn + 2048 + 96;                                       // [8]
    uint32_t *wstat = dyn + 2048 + 104;                              // [kWarps][8]
    uint32_t *wc_key = wstat + kWarps * 8;                           // [kWarps][kWarpCand]
    uint32_t *hist2 = wc_key + kWarps * kWarpCand;                   // [2048] second radix histogram
    constexpr int kPlusCap = kPlusWords / kWarps;                    // a warp's list of scores >= the band
    float *plus_x = reinterpret_cast<float *>(hist2 + 2048);         // [kWarps][kPlusCap]
    int32_t *plus_pos = reinterpret_cast<int32_t *>(plus_x + kPlusWords);  // [kWarps][kPlusCap]

    const int row = blockIdx.x;
    pdl_wait();  // the scores come from the kernel before
    pdl_trigger();
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
    // this warp's contiguous segment; lane l holds positions lo + 32 r + l of
    // it, -inf past the segment's end (so the passes below need no bounds
    // tests: -inf is never kept and weighs 0).  A segment of up to 32 kHeld
    // positions is loaded once and kept in registers for every pass; a longer
    // one is streamed in steps of 32 kStep positions through the two halves
    // of the same registers, the loads of the next step in flight while the
    // current one is processed.
    const int seg = (((vis + kWarps - 1) / kWarps) + 31) & ~31;
    const int lo = min(vis, warp * seg), hi = min(vis, lo + seg);
    const bool resident = hi - lo <= 32 * kHeld;
    const int nstep = (hi - lo + 32 * kStep - 1) / (32 * kStep);
    float x[kHeld];
    // positions lo + 32 (n0 + r) + lane into x[off + r], r < cnt
    auto load_into = [&](auto off_c, auto cnt_c, int n0) {
        constexpr int off = decltype(off_c)::value, cnt = decltype(cnt_c)::value;
        const int p0 = lo + 32 * n0 + lane;
        if (lo + 32 * (n0 + cnt) <= hi) {  // the whole part lies in the segment (every part but the last)
#pragma unroll
            for (int r = 0; r < cnt; r++) x[off + r] = __ldcg(s + p0 + 32 * r);
        } else {
#pragma unroll
            for (int r = 0; r < cnt; r++) x[off + r] = p0 + 32 * r < hi ? __ldcg(s + p0 + 32 * r) : -INFINITY;
        }
    };
    using C0 = std::integral_constant<int, 0>;
    using CS = std::integral_constant<int, kStep>;
    using CH = std::integral_constant<int, kHeld>;
    // calls f(off_c, cnt_c, p0) on every part of the segment held in x
    auto for_segment = [&](auto &&f) {
        if (resident) {
            f(C0{}, CH{}, lo + lane);
            return;
        }
        load_into(C0{}, CS{}, 0);
        for (int st = 0; st < nstep; st += 2) {
            if (st + 1 < nstep) load_into(CS{}, CS{}, (st + 1) * kStep);
            f(C0{}, CS{}, lo + 32 * st * kStep + lane);
            if (st + 1 < nstep) {
                if (st + 2 < nstep) load_into(C0{}, CS{}, (st + 2) * kStep);
                f(CS{}, CS{}, lo + 32 * (st + 1) * kStep + lane);
            }
        }
    };
    if (resident) load_into(C0{}, CH{}, 0);

    // pass 1: the histogram of the top 11 key bits of a sample: every eighth
    // group of 32 consecutive positions (every position on short rows) -- the
    // threshold is looked for there.  A streamed segment reads just its
    // sample here.
    for (int i = threadIdx.x; i < 2048; i += kThreads) sm.hist[i] = 0u;
    __syncthreads();
    const bool sampled = vis >= kSampleMinLen;  // always so for a streamed segment
    uint32_t nsample = 0u;
    if (resident) {
        if (sampled) {
#pragma unroll
            for (int r = 0; r < kHeld; r += 8) {
                if (lo + lane + 32 * r < hi) {
                    atomicAdd(&sm.hist[canon_key(x[r]) >> 21], 1u);
                    nsample++;
                }
            }
        } else {
#pragma unroll
            for (int r = 0; r < kHeld; r++) {
                if (lo + lane + 32 * r < hi) {
                    atomicAdd(&sm.hist[canon_key(x[r]) >> 21], 1u);
                    nsample++;
                }
            }
        }
    } else {
        // groups 0, 8, 16, ... of the segment, four loads in flight
        for (int g0 = 0; lo + 32 * g0 < hi; g0 += 32) {
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int pos = lo + 32 * (g0 + 8 * u) + lane;
                v[u] = pos < hi ? __ldcg(s + pos) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 4; u++) {
                if (lo + 32 * (g0 + 8 * u) + lane < hi) {
                    atomicAdd(&sm.hist[canon_key(v[u]) >> 21], 1u);
                    nsample++;
                }
            }
        }
    }
    if (lane == 0) wstat[warp * 8 + 1] = 0u;  // this warp's candidate count, for pass 2
    nsample = warp_sum(nsample);
    if (lane == 0) wstat[warp * 8 + 6] = nsample;
    __syncthreads();  // the histogram and the sample counts are complete
    // word f of the lane-th warp (0 past the last warp), for warp-wide reductions
    auto wword = [&](int f) { return lane < kWarps ? wstat[lane * 8 + f] : 0u; };
    const uint32_t total_sample = warp_sum(wword(6));
    // bins above b_hi are kept; bins [b_lo, b_hi] hold the candidates.  On the
    // sample the k-th key has rank about k * nsample / vis; the range is
    // widened by 4 binomial standard deviations each way and checked exactly
    // below.  As floats: x >= hi_t is above, lo_t <= x < hi_t a candidate.
    float hi_t, lo_t;
    uint32_t b_hi, b_lo;
    {
        const float ks = (float)k * (float)total_sample / (float)vis;
        const float margin = sampled ? 4.f * sqrtf(ks) + 4.f : 0.f;
        const uint32_t need_hi = (uint32_t)fmaxf(1.f, floorf(ks - margin));
        const uint32_t need_lo = (uint32_t)fminf((float)total_sample, ceilf(ks + margin));
        block_find_bins<2048>(sm.hist, need_hi, max(need_lo, need_hi), sm.tmp, sm.scal);
        b_hi = sm.scal[0];
        b_lo = sm.scal[2];
        // a NaN threshold compares false: nothing above bin 2044 (+inf) or below bin 4 (-FLT_MAX)
        hi_t = b_hi >= 2044u ? __uint_as_float(0x7fc00000u) : key_float((b_hi + 1u) << 21);
        lo_t = key_float(b_lo << 21);
    }

    // pass 2: the row maximum; count the positions above the range; collect
    // the keys inside it (in any order: only their values matter) into this
    // warp's candidate list; append every score at or above the range, with
    // its position, to this warp's ordered list (one ballot per round keeps
    // position order); sum e^{s - m_lane} over this lane's positions against
    // a running lane maximum m_lane (rescaled when it grows)
    uint32_t nwin = 0u, nplus = 0u;
    uint32_t *my_key = wc_key + warp * kWarpCand;
    float *my_px = plus_x + warp * kPlusCap;
    int32_t *my_pp = plus_pos + warp * kPlusCap;
    float m_lane = -INFINITY, zall = 0.f;
    for_segment([&](auto off_c, auto cnt_c, int p0) {
        constexpr int off = decltype(off_c)::value, cnt = decltype(cnt_c)::value;
        float bm = x[off];
#pragma unroll
        for (int r = 1; r < cnt; r++) bm = fmaxf(bm, x[off + r]);
        if (bm > m_lane) {  // never true for a part with no position (all -inf)
            zall *= exp2_approx((m_lane - bm) * kLog2e);
            m_lane = bm;
        }
        const float ml = m_lane == -INFINITY ? 0.f : m_lane * kLog2e;
#pragma unroll
        for (int r = 0; r < cnt; r++) {
            const float xv = x[off + r];
            zall += exp2_approx(fmaf(xv, kLog2e, -ml));
            const bool above = xv >= hi_t;
            nwin += above;
            const bool plus = xv >= lo_t;
            const uint32_t pb = __ballot_sync(0xffffffffu, plus);
            // the ordered list's slot for this lane; the two stores are
            // predicated (no branch per round)
            const uint32_t slot = nplus + __popc(pb & lt);
            st_shared_if(plus && slot < (uint32_t)kPlusCap, my_px + slot, __float_as_uint(xv), my_pp + slot,
                         (uint32_t)(p0 + 32 * r));
            if (plus && !above) {
                const uint32_t cs = atomicAdd(&wstat[warp * 8 + 1], 1u);
                if (cs < (uint32_t)kWarpCand) my_key[cs] = __float_as_uint(xv);  // converted when ranked
            }
            nplus += __popc(pb);
        }
    });
    float m = warp_max(m_lane);
    if (lane == 0) wstat[warp * 8 + 5] = __float_as_uint(m);
    nwin = warp_sum(nwin);
    if (lane == 0) wstat[warp * 8 + 0] = nwin;
    __syncthreads();
    m = warp_max(lane < kWarps ? __uint_as_float(wstat[lane * 8 + 5]) : -INFINITY);  // the row maximum
    const float m_l2e = m * kLog2e;
    // this lane's sum against the row maximum
    zall = m_lane == -INFINITY ? 0.f : zall * exp2_approx((m_lane - m) * kLog2e);
    // block totals, every warp reducing the per-warp words (lane w reads warp w's)
    const uint32_t above = warp_sum(wword(0));
    const uint32_t ncand = warp_sum(wword(1));
    const bool overflow = __any_sync(0xffffffffu, wword(1) > (uint32_t)kWarpCand);
    if (overflow || above >= (uint32_t)k || above + ncand < (uint32_t)k) {
        // the sampled range missed the k-th key or a warp's list overflowed:
        // take the exact multi-pass route
        __syncthreads();
        select_multipass(p, row, vis, sm);
        return;
    }

    // exact radix selection over the candidates' keys.  They lie in the
    // band's key range [base, base + 2^rem) (bins b_lo..b_hi of 2^21 keys;
    // with no upper threshold, everything up to the top key), so every level
    // splits the current range into at most 2048 bins and the candidates
    // spread over the bins instead of piling into the few bins of the band
    // (few conflicting atomics); two levels reach a single key unless the
    // band spans more than two bins.
    const uint32_t need = (uint32_t)k - above;
    uint32_t gt = 0u, base = b_lo << 21;
    int rem;
    {
        const uint32_t nb = (b_hi >= 2044u ? 2047u : b_hi) - b_lo + 1u;  // >= 1
        rem = 21 + (nb > 1u ? 32 - __clz(nb - 1u) : 0);                // <= 32
    }
    // two histograms: level L counts into sm.hist (L even) or hist2 (L odd)
    // while the other one is cleared for level L + 1; warp 0 searches between
    // two barriers
    for (int i = threadIdx.x; i < 2048; i += kThreads) {
        sm.hist[i] = 0u;
        hist2[i] = 0u;
    }
    __syncthreads();
    const uint32_t my_cand = wstat[warp * 8 + 1];
    for (int level = 0; rem > 0; level++) {
        const int sh = rem > 11 ? rem - 11 : 0;
        uint32_t *h = (level & 1) ? hist2 : sm.hist;
        const unsigned long long span = 1ull << rem;
        for (uint32_t i = lane; i < my_cand; i += 32) {  // this warp's own list
            const uint32_t key = canon_key(__uint_as_float(my_key[i]));
            if (key >= base && (unsigned long long)(key - base) < span) atomicAdd(&h[(key - base) >> sh], 1u);
        }
        if (level >= 1) {  // the previous level's histogram, for the next level
            uint32_t *hn = (level & 1) ? sm.hist : hist2;
            for (int i = threadIdx.x; i < 2048; i += kThreads) hn[i] = 0u;
        }
        __syncthreads();  // the histogram is complete
        block_find_bins<2048>(h, need - gt, need - gt, sm.tmp, sm.scal);
        gt += sm.scal[1];
        base += sm.scal[0] << sh;
        rem = sh;
    }
    const uint32_t T = base;
    // keys equal to T: the first r_eq of them (by position) are kept
    const uint32_t r_eq = need - gt;

    // per warp: candidates above T and ties at T, then output offsets
    {
        uint32_t g = 0u, t = 0u;
        for (uint32_t i = lane; i < wstat[warp * 8 + 1]; i += 32) {
            const uint32_t key = canon_key(__uint_as_float(my_key[i]));
            g += key > T;
            t += key == T;
        }
        g = warp_sum(g);
        t = warp_sum(t);
        if (lane == 0) {
            wstat[warp * 8 + 2] = g;
            wstat[warp * 8 + 3] = t;
        }
    }
    __syncthreads();
    // output offsets: warp w keeps its scores above the range, its candidates
    // above T and the ties at T that fall among the first r_eq of the row
    uint32_t out_run, tie_run, n_eq;
    {
        const uint32_t tie_l = wword(3);
        const uint32_t tie_incl = warp_incl_scan(tie_l), tie_excl = tie_incl - tie_l;
        const uint32_t kept_l = wword(0) + wword(2) +
                                (r_eq > tie_excl ? min(tie_l, r_eq - tie_excl) : 0u);
        const uint32_t out_incl = warp_incl_scan(kept_l);
        out_run = __shfl_sync(0xffffffffu, out_incl - kept_l, warp);
        tie_run = __shfl_sync(0xffffffffu, tie_excl, warp);
        n_eq = __shfl_sync(0xffffffffu, tie_incl, 31);
    }
    const bool rank_ties = n_eq != r_eq;
    const uint32_t out_begin = out_run;

    // pass 3: the exact rule -- s > T, or s == T among the first r_eq ties
    // (s >= T when every tie is kept) -- written straight to the final
    // ascending positions, with the softmax sums of kept and dropped scores.
    // As float comparisons: canon_key order is float order.  A warp whose
    // ordered list is complete takes its kept positions from the list (every
    // kept score is at or above the range) and its dropped mass as the total
    // less the kept; a warp whose list overflowed streams its segment again.
    const float T_f = key_float(T);
    int32_t *idx = p.idx + (size_t)row * k;
    float *wv = p.w + (size_t)row * k;
    float zk = 0.f, zt = 0.f;
    auto emit = [&](bool sel, float e, int pos) {
        const uint32_t sb = __ballot_sync(0xffffffffu, sel);
        if (sel) {
            const uint32_t o = out_run + __popc(sb & lt);
            if (o < (uint32_t)k) {  // always true unless the counts above are wrong
                idx[o] = pos;
                wv[o] = e;
            }
            zk += e;
        } else {
            zt += e;
        }
        out_run += __popc(sb);
    };
    if (nplus <= (uint32_t)kPlusCap) {
        for (uint32_t i0 = 0; i0 < nplus; i0 += 32) {
            const uint32_t i = i0 + lane;
            const float xv = i < nplus ? my_px[i] : -INFINITY;
            bool sel;
            if (rank_ties) {
                const bool tie = xv == T_f;
                const uint32_t tb = __ballot_sync(0xffffffffu, tie);
                sel = xv > T_f || (tie && tie_run + __popc(tb & lt) < r_eq);
                tie_run += __popc(tb);
            } else {
                sel = xv >= T_f;
            }
            const uint32_t sb = __ballot_sync(0xffffffffu, sel);
            if (sel) {
                const float e = exp2_approx(fmaf(xv, kLog2e, -m_l2e));
                const uint32_t o = out_run + __popc(sb & lt);
                if (o < (uint32_t)k) {  // always true unless the counts above are wrong
                    idx[o] = my_pp[i];
                    wv[o] = e;
                }
                zk += e;
            }
            out_run += __popc(sb);
        }
        // dropped = all - kept, per warp (the warp's lanes sum to its totals)
        zt = zall - zk;
    } else {
        for_segment([&](auto off_c, auto cnt_c, int p0) {
            constexpr int off = decltype(off_c)::value, cnt = decltype(cnt_c)::value;
#pragma unroll
            for (int r = 0; r < cnt; r++) {
                const float xv = x[off + r];
                bool sel = xv >= T_f;
                if (rank_ties) {
                    const bool tie = xv == T_f;
                    const uint32_t tb = __ballot_sync(0xffffffffu, tie);
                    sel = xv > T_f || (tie && tie_run + __popc(tb & lt) < r_eq);
                    tie_run += __popc(tb);
                }
                emit(sel, exp2_approx(fmaf(xv, kLog2e, -m_l2e)), p0 + 32 * r);
            }
        });
    }
    if (lane == 0) wstat[warp * 8 + 4] = out_run - out_begin;
    __syncthreads();
    const uint32_t written = warp_sum(wword(4));
    finish_row(p, row, m, zk, zt, written, (uint32_t)k, sm);
}

}  // namespace

size_t select_smem_bytes(int threads) { return smem_words(threads / 32) * 4; }

namespace {

template <int kThreads>
cudaError_t launch_n(const SelectParams &p, cudaStream_t stream, bool pdl) {
    const int rows = p.B * p.Q * p.Hq;
    const size_t smem = select_smem_bytes(kThreads);
    static bool attr_set[64] = {};  // per device: the shared-memory opt-in is a function attribute
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (smem > 48 * 1024 && (dev < 0 || dev >= 64 || !attr_set[dev])) {
        e = cudaFuncSetAttribute(select_topk<kThreads>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    return launch_k(pdl, select_topk<kThreads>, dim3(rows), dim3(kThreads), smem, stream, p);
}

}  // namespace

cudaError_t launch_select(const SelectParams &p, cudaStream_t stream, int threads, bool pdl) {
    return threads == 512 ? launch_n<512>(p, stream, pdl) : launch_n<1024>(p, stream, pdl);
}

}  // namespace tka
