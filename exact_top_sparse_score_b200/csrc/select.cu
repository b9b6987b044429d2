// Select step: for one query row, the k highest-scoring visible positions
// (ties at the k-th score go to the lower position), in ascending position
// order, together with the softmax statistics the attention step needs.
//
// "Top-K Selection: retaining the K historical positions with the highest
// scores" ("Evolution of Sparse Attention in Long-Context LLMs", section 2);
// the discarded mass is the Top-k tail mass of "A Mathematical Theory of
// Top-k Sparse Attention via Total Variation Distance" (abstract).
//
// One CTA (32 warps) per row; every warp owns a contiguous
// segment of the row, lane l holding positions l, l + 32, ... of it, so a warp
// compacts 32 consecutive positions at a time with one ballot.  A segment is
// streamed in batches of 32 x 32 positions with all loads of a batch in
// flight together (a segment that fits one batch is read once and kept in
// registers for all passes); the rows come from L2.  Scores are compared as
// order-preserving uint32 keys:
//   pass 1  the row maximum and the histogram of the top 11 key bits of a
//           position-uniform 1/8 sample give a bin range that holds the k-th
//           key with high probability;
//   pass 2  keys above the range are counted, keys inside it are collected
//           (in position order) into per-warp candidate lists;
//   exact radix selection over the candidates' full keys (11 + 11 + 10 bits)
//           yields the k-th key T and how many of the keys equal to T are
//           kept (the lowest positions);
//   pass 3  every key is tested against that exact rule and the kept
//           positions are written straight to their ascending slots (warp
//           prefix sums plus per-warp offsets), while Z_k = sum_kept e^{s-m}
//           and Z_tail = sum_dropped e^{s-m} are accumulated; the tail mass
//           Z_tail / (Z_k + Z_tail) is formed from the dropped terms directly.
// If the sampled range misses the k-th key, or a warp collects more
// candidates than fit, the row falls back to three exact histogram passes and
// an ordered compaction pass over the row.
#include "common.cuh"
#include "kernels.h"

namespace tka {

namespace {

constexpr int kSelectThreads = 1024;
constexpr int kWarps = kSelectThreads / 32;
constexpr int kWarpCand = 256;                  // candidates per warp held in shared memory
constexpr int kHeld = 32;                       // scores per lane held in registers per batch
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
    float *red;      // [32]
    uint32_t *scal;  // [2]: bin, above
};

// Writes stats, tail and counter of a finished row.
__device__ __forceinline__ void finish_row(const SelectParams &p, int row, float m, float zk, float zt,
                                           uint32_t written, uint32_t kept, const SelectSmem &sm) {
    zk = block_sum(zk, sm.red);
    __syncthreads();
    zt = block_sum(zt, sm.red);
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
        atomicAdd(&hist[order_key(x) >> 21], 1u);
    });
    m = block_max(m, sm.red);
    __syncthreads();
    find_bin(hist, 2048, (uint32_t)k, sm.tmp, &sm.scal[0], &sm.scal[1]);
    const uint32_t b1 = sm.scal[0];
    uint32_t above = sm.scal[1];
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    visit_row(s, vis, [&](int, float x) {
        const uint32_t key = order_key(x);
        if ((key >> 21) == b1) atomicAdd(&hist[(key >> 10) & 0x7ffu], 1u);
    });
    __syncthreads();
    find_bin(hist, 2048, (uint32_t)k - above, sm.tmp, &sm.scal[0], &sm.scal[1]);
    const uint32_t b2 = sm.scal[0];
    above += sm.scal[1];
    const uint32_t pre = (b1 << 11) | b2;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    visit_row(s, vis, [&](int, float x) {
        const uint32_t key = order_key(x);
        if ((key >> 10) == pre) atomicAdd(&hist[key & 0x3ffu], 1u);
    });
    __syncthreads();
    find_bin(hist, 1024, (uint32_t)k - above, sm.tmp, &sm.scal[0], &sm.scal[1]);
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
            key[j] = order_key(x[j]);
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

__global__ void __launch_bounds__(kSelectThreads, 1) select_topk(SelectParams p) {
    extern __shared__ __align__(16) uint32_t dyn[];
    SelectSmem sm;
    sm.hist = dyn;                                                   // [2048]
    sm.tmp = dyn + 2048;                                             // [32]
    sm.red = reinterpret_cast<float *>(dyn + 2048 + 32);             // [32]
    sm.scal = dyn + 2048 + 64;                                       // [8]
    uint32_t *wstat = dyn + 2048 + 72;                               // [kWarps][8]
    uint32_t *wc_key = wstat + kWarps * 8;                           // [kWarps][kWarpCand]
    int32_t *wc_pos = reinterpret_cast<int32_t *>(wc_key + kWarps * kWarpCand);  // [kWarps][kWarpCand]

    const int row = blockIdx.x;
    const int b = row / (p.Q * p.Hq), qpos = (row / p.Hq) % p.Q;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) {
        if (threadIdx.x == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    const int vis = visible_keys(seq_len, p.Q, qpos);
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
    // each batch of 32 * kHeld positions
    const int seg = (((vis + kWarps - 1) / kWarps) + 31) & ~31;
    const int lo = min(vis, warp * seg), hi = min(vis, lo + seg);
    const int nbatch = (hi - lo + 32 * kHeld - 1) / (32 * kHeld);
    const bool resident = nbatch <= 1;  // the whole segment fits in registers
    float x[kHeld];
    auto load_batch = [&](int bi) {
        const int p0 = lo + bi * 32 * kHeld + lane;
#pragma unroll
        for (int r = 0; r < kHeld; r++) x[r] = p0 + 32 * r < hi ? __ldcg(s + p0 + 32 * r) : 0.f;
    };
    if (resident) load_batch(0);

    // pass 1: the row maximum, and the histogram of the top 11 key bits of a
    // position-uniform sample (positions that are multiples of 8; every
    // position on short rows) -- the threshold is looked for there
    for (int i = threadIdx.x; i < 2048; i += kSelectThreads) sm.hist[i] = 0u;
    __syncthreads();
    const bool sampled = vis >= kSampleMinLen;
    const bool sampler = !sampled || (lane & 7) == 0;  // lo is a multiple of 32
    float m = -INFINITY;
    for (int bi = 0; bi < nbatch; bi++) {
        if (!resident) load_batch(bi);
        const int p0 = lo + bi * 32 * kHeld + lane;
#pragma unroll
        for (int r = 0; r < kHeld; r++) {
            if (p0 + 32 * r < hi) {
                m = fmaxf(m, x[r]);
                if (sampler) atomicAdd(&sm.hist[order_key(x[r]) >> 21], 1u);
            }
        }
    }
    m = block_max(m, sm.red);
    __syncthreads();
    // bins above b_hi are kept; bins [b_lo, b_hi] hold the candidates.  On the
    // sample the k-th key has rank about k/8; the range is widened by 4
    // binomial standard deviations each way and checked exactly below.
    uint32_t b_hi, b_lo;
    {
        const int slog = sampled ? 3 : 0;
        const uint32_t nsample = (uint32_t)((vis + (1 << slog) - 1) >> slog);
        const float ks = (float)k / (float)(1 << slog);
        const float margin = sampled ? 4.f * sqrtf(ks) + 4.f : 0.f;
        const uint32_t need_hi = (uint32_t)fmaxf(1.f, floorf(ks - margin));
        const uint32_t need_lo = (uint32_t)fminf((float)nsample, ceilf(ks + margin));
        find_bin(sm.hist, 2048, need_hi, sm.tmp, &sm.scal[0], &sm.scal[1]);
        b_hi = sm.scal[0];
        find_bin(sm.hist, 2048, max(need_lo, need_hi), sm.tmp, &sm.scal[0], &sm.scal[1]);
        b_lo = sm.scal[0];
    }

    // pass 2: count the keys of bins above b_hi; collect the keys of bins
    // [b_lo, b_hi], in position order, into this warp's candidate list
    uint32_t nwin = 0u, ncw = 0u;
    uint32_t *my_key = wc_key + warp * kWarpCand;
    int32_t *my_pos = wc_pos + warp * kWarpCand;
    for (int bi = 0; bi < nbatch; bi++) {
        if (!resident) load_batch(bi);
        const int p0 = lo + bi * 32 * kHeld + lane;
#pragma unroll
        for (int r = 0; r < kHeld; r++) {
            const bool valid = p0 + 32 * r < hi;
            const uint32_t key = order_key(x[r]);
            const uint32_t bin = key >> 21;
            nwin += __popc(__ballot_sync(0xffffffffu, valid && bin > b_hi));
            const bool cand = valid && bin >= b_lo && bin <= b_hi;
            const uint32_t cb = __ballot_sync(0xffffffffu, cand);
            if (cand) {
                const uint32_t slot = ncw + __popc(cb & lt);
                if (slot < (uint32_t)kWarpCand) {
                    my_key[slot] = key;
                    my_pos[slot] = p0 + 32 * r;
                }
            }
            ncw += __popc(cb);
        }
    }
    if (lane == 0) {
        wstat[warp * 8 + 0] = nwin;
        wstat[warp * 8 + 1] = ncw;
    }
    __syncthreads();
    uint32_t above = 0u, ncand = 0u;
    bool overflow = false;
    for (int w = 0; w < kWarps; w++) {
        above += wstat[w * 8 + 0];
        ncand += wstat[w * 8 + 1];
        overflow |= wstat[w * 8 + 1] > (uint32_t)kWarpCand;
    }
    if (overflow || above >= (uint32_t)k || above + ncand < (uint32_t)k) {
        // the sampled range missed the k-th key or a warp's list overflowed:
        // take the exact multi-pass route
        __syncthreads();
        select_multipass(p, row, vis, sm);
        return;
    }

    // exact radix selection over the candidates' full 32-bit keys (11 + 11 +
    // 10 bits): r of them are kept
    const uint32_t need = (uint32_t)k - above;
    uint32_t pre = 0u, gt = 0u, T = 0u;
    for (int level = 0; level < 3; level++) {
        const int shift = level == 0 ? 21 : (level == 1 ? 10 : 0);
        const int nb = level == 2 ? 1024 : 2048;
        for (int i = threadIdx.x; i < 2048; i += kSelectThreads) sm.hist[i] = 0u;
        __syncthreads();
        for (int e = threadIdx.x; e < kWarps * kWarpCand; e += kSelectThreads) {
            const int w = e / kWarpCand, i = e - w * kWarpCand;
            if ((uint32_t)i >= wstat[w * 8 + 1]) continue;
            const uint32_t key = wc_key[e];
            if (level == 0 || (key >> (shift + (level == 1 ? 11 : 10))) == pre)
                atomicAdd(&sm.hist[(key >> shift) & (uint32_t)(nb - 1)], 1u);
        }
        __syncthreads();
        find_bin(sm.hist, nb, need - gt, sm.tmp, &sm.scal[0], &sm.scal[1]);
        const uint32_t bin = sm.scal[0];
        gt += sm.scal[1];
        if (level < 2)
            pre = (pre << (level == 0 ? 0 : 11)) | bin;
        else
            T = (pre << 10) | bin;
    }
    // keys equal to T: the first r_eq of them (by position) are kept
    const uint32_t r_eq = need - gt;

    // per warp: candidates above T and ties at T, then output offsets
    {
        uint32_t g = 0u, t = 0u;
        for (uint32_t i = lane; i < ncw; i += 32) {
            g += my_key[i] > T;
            t += my_key[i] == T;
        }
        g = warp_sum(g);
        t = warp_sum(t);
        if (lane == 0) {
            wstat[warp * 8 + 2] = g;
            wstat[warp * 8 + 3] = t;
        }
    }
    __syncthreads();
    uint32_t out_run = 0u, tie_run = 0u, n_eq = 0u;
    for (int w = 0; w < kWarps; w++) {
        const uint32_t tie_w = wstat[w * 8 + 3];
        if (w < warp) {
            const uint32_t kept_ties = r_eq > tie_run ? min(tie_w, r_eq - tie_run) : 0u;
            out_run += wstat[w * 8 + 0] + wstat[w * 8 + 2] + kept_ties;
            tie_run += tie_w;
        }
        n_eq += tie_w;
    }
    const bool rank_ties = n_eq != r_eq;
    const uint32_t out_begin = out_run;

    // pass 3: the exact rule -- key > T, or key == T among the first r_eq
    // ties -- written straight to the final ascending positions, with the
    // softmax sums of kept and dropped keys
    int32_t *idx = p.idx + (size_t)row * k;
    float *wv = p.w + (size_t)row * k;
    float zk = 0.f, zt = 0.f;
    for (int bi = 0; bi < nbatch; bi++) {
        if (!resident) load_batch(bi);
        const int p0 = lo + bi * 32 * kHeld + lane;
#pragma unroll
        for (int r = 0; r < kHeld; r++) {
            const bool valid = p0 + 32 * r < hi;
            const uint32_t key = order_key(x[r]);
            bool sel = valid && key > T;
            if (rank_ties) {
                const bool tie = valid && key == T;
                const uint32_t tb = __ballot_sync(0xffffffffu, tie);
                if (tie) sel = tie_run + __popc(tb & lt) < r_eq;
                tie_run += __popc(tb);
            } else {
                sel = sel || (valid && key == T);
            }
            const uint32_t sb = __ballot_sync(0xffffffffu, sel);
            if (valid) {
                const float e = __expf(x[r] - m);
                if (sel) {
                    const uint32_t o = out_run + __popc(sb & lt);
                    if (o < (uint32_t)k) {  // always true unless the counts above are wrong
                        idx[o] = p0 + 32 * r;
                        wv[o] = e;
                    }
                    zk += e;
                } else {
                    zt += e;
                }
            }
            out_run += __popc(sb);
        }
    }
    if (lane == 0) wstat[warp * 8 + 4] = out_run - out_begin;
    __syncthreads();
    uint32_t written = 0u;
    for (int w = 0; w < kWarps; w++) written += wstat[w * 8 + 4];
    finish_row(p, row, m, zk, zt, written, (uint32_t)k, sm);
}

}  // namespace

size_t select_smem_bytes(int) {
    return (size_t)(2048 + 72 + kWarps * 8) * 4 + (size_t)kWarps * kWarpCand * 8;
}

cudaError_t launch_select(const SelectParams &p, cudaStream_t stream) {
    const int rows = p.B * p.Q * p.Hq;
    const size_t smem = select_smem_bytes(p.k);
    static bool attr_set[64] = {};  // per device: the shared-memory opt-in is a function attribute
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (smem > 48 * 1024 && (dev < 0 || dev >= 64 || !attr_set[dev])) {
        e = cudaFuncSetAttribute(select_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    select_topk<<<rows, kSelectThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tka
