// Block-sparse (MoBA) decode attention.
//
// "Sparse Attention Landscape", section "Block Sparse Attention": the cache is
// cut into blocks, each block gets one relevance score, the top blocks are
// kept and attention runs over the tokens inside them; MoBA's block score is
// the dot product of the query with the mean-pooled keys of the block.  The
// last (current) block is always kept.
//
// Kernels:
//   block_pool    block_keys[b,h,j,:] = mean of the block's keys (fp32), built
//                 when blocks change, not per decode step.
//   block_scores  grid (64-block chunk, b*kv-head): each block key is read once
//                 and scored against all G query heads that share it.
//   block_topk    one CTA per query row: a radix selection over the competing
//                 blocks' scores finds the top_blocks best (score desc, block
//                 asc); they and the current block are written ascending.
//   block_attn    grid (kept slot, row): a kept block's K rows and V rows are
//                 each one contiguous range of the cache, so one CTA fetches
//                 both with two bulk asynchronous copies in flight together,
//                 then computes the block's scores, local max m, sum l and
//                 sum p*V from shared memory; the last CTA of the row merges
//                 the slots with the usual max-rescaled softmax merge, in slot
//                 order.
#include <string.h>

#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace tka {

namespace {

template <typename T>
__device__ __forceinline__ float load_f32(const T *p) {
    if constexpr (sizeof(T) == 4)
        return *reinterpret_cast<const float *>(p);
    else
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
}

// 4 consecutive elements as fp32 (8-byte load for bf16, 16-byte for fp32).
template <typename T>
__device__ __forceinline__ float4 load4(const T *p) {
    if constexpr (sizeof(T) == 4) {
        return __ldg(reinterpret_cast<const float4 *>(p));
    } else {
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
        return make_float4(bf16lo_to_f32(w.x), bf16hi_to_f32(w.x), bf16lo_to_f32(w.y), bf16hi_to_f32(w.y));
    }
}

// The same conversions from shared memory.
template <typename T>
__device__ __forceinline__ float4 load4s(const T *p) {
    if constexpr (sizeof(T) == 4) {
        return *reinterpret_cast<const float4 *>(p);
    } else {
        const uint2 w = *reinterpret_cast<const uint2 *>(p);
        return make_float4(bf16lo_to_f32(w.x), bf16hi_to_f32(w.x), bf16lo_to_f32(w.y), bf16hi_to_f32(w.y));
    }
}

template <typename T>
__device__ __forceinline__ float load1s(const T *p) {
    if constexpr (sizeof(T) == 4)
        return *p;
    else
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
}

template <typename T>
__global__ void __launch_bounds__(128) block_pool(BlockPoolParams p) {
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    const int j = blockIdx.x, bh = blockIdx.y, b = bh / p.Hkv;
    const int seq_len = p.seq_lens[b];
    if (seq_len < 1 || seq_len > p.L_max) {
        if (j == 0 && threadIdx.x == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    const int lo = j * p.block_size, hi = min(lo + p.block_size, seq_len);
    const T *kb = reinterpret_cast<const T *>(p.k) + (size_t)bh * p.L_max * kHeadDim + threadIdx.x;
    float acc = 0.f;
    for (int i = lo; i < hi; i++) acc += load_f32(kb + (size_t)i * kHeadDim);
    p.block_keys[((size_t)bh * p.nblk_max + j) * kHeadDim + threadIdx.x] = hi > lo ? acc / (float)(hi - lo) : 0.f;
}

constexpr int kScoreBlocks = 64;  // blocks per CTA of block_scores
constexpr int kSelThreads = 256;
constexpr int kClusterCtas = 8;   // CTAs of block_select_cluster per (b, kv-head)
constexpr size_t kClusterSmem = 96 * 1024;  // shared memory block_select_cluster may take

// bscore[row, j] = scale * <q_row, block_keys[b, kvh, j, :]> for the competing
// blocks j < nblk - 1 of every query row of kv-head kvh.  Eight lanes share a
// block key, lane c of the eight holding float4 columns c, c + 8, c + 16 and
// c + 24 (so each load instruction reads 128 contiguous bytes per block), and
// a thread keeps both of its blocks' loads in flight before any arithmetic.
template <typename T>
__global__ void __launch_bounds__(kSelThreads) block_scores(BlockSelectParams p) {
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    extern __shared__ float4 qs[];  // [G][32]: the group's query rows as fp32
    const int bh = blockIdx.y, b = bh / p.Hkv, kvh = bh - b * p.Hkv;
    const int seq_len = p.seq_lens[b];
    if (seq_len < 1 || seq_len > p.L_max) return;  // block_topk raises the status
    const int ncomp = (seq_len + p.block_size - 1) / p.block_size - p.force_last;
    const int j0 = blockIdx.x * kScoreBlocks;
    if (j0 >= ncomp || ncomp <= p.top_blocks) return;  // nothing to rank here
    const T *q = reinterpret_cast<const T *>(p.q) + ((size_t)b * p.Hq + (size_t)kvh * p.G) * kHeadDim;
    for (int e = threadIdx.x; e < p.G * 32; e += kSelThreads) qs[e] = load4(q + 4 * e);
    const int c = threadIdx.x & 7;
    const float4 *bk = reinterpret_cast<const float4 *>(p.block_keys + (size_t)bh * p.nblk_max * kHeadDim);
    constexpr int kPerThread = kScoreBlocks / (kSelThreads / 8);  // 2
    int jj[kPerThread];
    float4 kv[kPerThread][4];
#pragma unroll
    for (int r = 0; r < kPerThread; r++) {
        jj[r] = j0 + r * (kSelThreads / 8) + (threadIdx.x >> 3);
#pragma unroll
        for (int u = 0; u < 4; u++)
            kv[r][u] = jj[r] < ncomp ? __ldg(bk + (size_t)jj[r] * 32 + c + 8 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    float *out = p.bscore + ((size_t)b * p.Hq + (size_t)kvh * p.G) * p.nblk_max;
    for (int g = 0; g < p.G; g++) {
        float4 qv[4];
#pragma unroll
        for (int u = 0; u < 4; u++) qv[u] = qs[g * 32 + c + 8 * u];
#pragma unroll
        for (int r = 0; r < kPerThread; r++) {
            float s = 0.f;
#pragma unroll
            for (int u = 0; u < 4; u++)
                s += qv[u].x * kv[r][u].x + qv[u].y * kv[r][u].y + qv[u].z * kv[r][u].z + qv[u].w * kv[r][u].w;
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            if (c == 0 && jj[r] < ncomp) out[(size_t)g * p.nblk_max + jj[r]] = s * p.scale;
        }
    }
}

// Keeps the `top` largest of the ncomp keys ukey[0..ncomp) (ties to the lower
// block) and, when force_last is set, the current block nblk - 1; writes them
// ascending to out[0..top + force_last).  Requires 0 < top < ncomp.  The
// threshold key T (the top-th largest) comes from a radix selection over the
// keys, 8 bits at a time; the kept blocks are then compacted in block order,
// the blocks whose key equals T kept from the lowest index up.  Called by the
// whole block (kSelThreads threads).
__device__ void keep_top_blocks(const uint32_t *ukey, int ncomp, int nblk, int top, int force_last, int32_t *out,
                                unsigned *status, uint32_t *hist, uint32_t *tmp, uint32_t *s_bin, uint32_t *s_above) {
    uint32_t prefix = 0u, mask = 0u, need = (uint32_t)top;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += kSelThreads) hist[i] = 0u;
        __syncthreads();
        for (int j = threadIdx.x; j < ncomp; j += kSelThreads) {
            const uint32_t u = ukey[j];
            if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
        }
        __syncthreads();
        find_bin(hist, 256, need, tmp, s_bin, s_above);
        prefix |= *s_bin << shift;
        mask |= 255u << shift;
        need -= *s_above;
    }
    const uint32_t T = prefix;  // keys above T are kept, and the first `need` keys equal to T
    const int per = (ncomp + kSelThreads - 1) / kSelThreads;
    const int lo = threadIdx.x * per, hi = min(lo + per, ncomp);
    uint32_t gt = 0u, eq = 0u;
    for (int j = lo; j < hi; j++) {
        gt += ukey[j] > T;
        eq += ukey[j] == T;
    }
    uint32_t total;
    const uint32_t eq_before = block_excl_scan(eq, tmp, &total);
    const uint32_t take_eq = need > eq_before ? min(eq, need - eq_before) : 0u;
    uint32_t pos = block_excl_scan(gt + take_eq, tmp, &total);
    if (total != (uint32_t)top) {  // never true unless the selection above is wrong
        if (threadIdx.x == 0) raise_status(status, TKA_DEV_INTERNAL);
        return;
    }
    uint32_t eqr = eq_before;
    for (int j = lo; j < hi; j++) {
        const uint32_t u = ukey[j];
        bool keep = u > T;
        if (u == T) keep = eqr++ < need;
        if (keep) out[pos++] = j;
    }
    if (threadIdx.x == 0 && force_last) out[top] = nblk - 1;  // the current block has the highest index
}

// keep_top_blocks with one histogram level instead of radix levels: the
// scores' minimum and maximum, a histogram in 2048 bins of equal width between
// them, the bin b* that holds the top-th score; when b* is kept whole, every
// block whose bin is at or above b* is kept, else the exact top-th key T is
// ranked among the (at most 32) blocks of b* by one warp, ties at T kept from
// the lowest block up.  One block-wide scan then writes the kept blocks in
// ascending order.  Returns false, having written nothing, when more than 32
// blocks share b* or the scores are all equal (the caller takes the radix
// route).  x holds the ncomp competing blocks' scores; ukey receives their
// order keys.
__device__ bool keep_top_blocks_hist(const float *x, uint32_t *ukey, int ncomp, int nblk, int top, int force_last,
                                     int32_t *out, unsigned *status, uint32_t *hist, uint32_t *tmp, uint32_t *scal,
                                     float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kSelThreads / 32;
    float lo = INFINITY, hi = -INFINITY;
    for (int j = threadIdx.x; j < ncomp; j += kSelThreads) {
        const float v = x[j];
        ukey[j] = order_key(v);
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
    for (int i = threadIdx.x; i < 2048; i += kSelThreads) hist[i] = 0u;
    lo = warp_min(lo);
    hi = warp_max(hi);
    if (lane == 0) {
        red[warp] = lo;
        red[kWarps + warp] = hi;
    }
    if (threadIdx.x == 0) scal[4] = 0u;
    __syncthreads();
    lo = warp_min(lane < kWarps ? red[lane] : INFINITY);
    hi = warp_max(lane < kWarps ? red[kWarps + lane] : -INFINITY);
    if (!(hi > lo) || !(hi - lo < INFINITY)) return false;  // all equal (or not finite): radix route
    const float scale = 2048.f / (hi - lo);
    auto bin = [&](float v) { return min(2047u, (uint32_t)((v - lo) * scale)); };
    for (int j = threadIdx.x; j < ncomp; j += kSelThreads) atomicAdd(&hist[bin(x[j])], 1u);
    __syncthreads();
    block_find_bins<2048>(hist, (uint32_t)top, (uint32_t)top, tmp, scal);
    const uint32_t bstar = scal[0];
    const uint32_t c_star = hist[bstar], r = (uint32_t)top - scal[1];  // 1 <= r <= c_star
    if (c_star > 32u) return false;  // uniform: every thread read the same words
    uint32_t T = 0u, r_eq = 0u;
    const bool by_bin = r == c_star;
    if (!by_bin) {
        uint64_t *cand = reinterpret_cast<uint64_t *>(hist);  // [32] (key, block): the bins are no longer read
        __syncthreads();
        for (int j = threadIdx.x; j < ncomp; j += kSelThreads)
            if (bin(x[j]) == bstar) cand[atomicAdd(&scal[4], 1u)] = ((uint64_t)ukey[j] << 32) | (uint32_t)j;
        __syncthreads();
        if (warp == 0) {
            const uint32_t mine = lane < (int)c_star ? (uint32_t)(cand[lane] >> 32) : 0u;
            uint32_t g = 0u, e = 0u;
            for (uint32_t i = 0; i < c_star; i++) {
                const uint32_t o = (uint32_t)(cand[i] >> 32);
                g += o > mine;
                e += o == mine;
            }
            const uint32_t hit = __ballot_sync(0xffffffffu, lane < (int)c_star && g < r && r <= g + e);
            const int L = hit ? __ffs(hit) - 1 : 0;
            const uint32_t tk = __shfl_sync(0xffffffffu, mine, L), tg = __shfl_sync(0xffffffffu, g, L);
            if (lane == 0) {
                scal[5] = tk;
                scal[6] = r - tg;
                if (!hit) raise_status(status, TKA_DEV_INTERNAL);
            }
        }
        __syncthreads();
        T = scal[5];
        r_eq = scal[6];
    }
    // kept: a bin above b*, all of b* when it is kept whole, else a key above
    // T or one of the first r_eq keys equal to T (in block order)
    const int per = (ncomp + kSelThreads - 1) / kSelThreads;
    const int j0 = threadIdx.x * per, j1 = min(j0 + per, ncomp);
    uint32_t kept = 0u, ties = 0u;
    for (int j = j0; j < j1; j++) {
        const uint32_t bj = bin(x[j]);
        if (by_bin) {
            kept += bj >= bstar;
        } else {
            kept += bj > bstar || (bj == bstar && ukey[j] > T);
            ties += bj == bstar && ukey[j] == T;
        }
    }
    uint32_t total;
    const uint32_t before = block_excl_scan(kept | (ties << 16), tmp, &total);  // both counts < 2^16
    uint32_t pos = before & 0xffffu, tie_rank = before >> 16;
    const uint32_t written = (total & 0xffffu) + min(total >> 16, r_eq);
    if (written != (uint32_t)top) {  // never true unless the selection above is wrong
        if (threadIdx.x == 0) raise_status(status, TKA_DEV_INTERNAL);
        return true;
    }
    pos += min(tie_rank, r_eq);  // the ties before this thread's that are kept
    for (int j = j0; j < j1; j++) {
        const uint32_t bj = bin(x[j]);
        bool keep;
        if (by_bin) {
            keep = bj >= bstar;
        } else {
            keep = bj > bstar || (bj == bstar && ukey[j] > T);
            if (bj == bstar && ukey[j] == T) keep = tie_rank++ < r_eq;
        }
        if (keep) out[pos++] = j;
    }
    if (threadIdx.x == 0 && force_last) out[top] = nblk - 1;  // the current block has the highest index
    return true;
}

// The easy cases of a row's block list: every competing block kept, or only
// the current block.  Returns false when the row needs a selection.
__device__ __forceinline__ bool trivial_blocks(int ncomp, int nblk, int top, int width, int32_t *out) {
    if (ncomp <= top) {  // every block is kept: nothing to rank
        for (int i = threadIdx.x; i < width; i += kSelThreads) out[i] = i < nblk ? i : -1;
        return true;
    }
    if (top == 0) {  // only the current block
        if (threadIdx.x == 0) out[0] = nblk - 1;
        return true;
    }
    return false;
}

// One CTA per query row: the row's competing blocks' scores (from
// block_scores), then keep_top_blocks.
__global__ void __launch_bounds__(kSelThreads) block_topk(BlockSelectParams p) {
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    extern __shared__ uint32_t ukey[];  // [ncomp]
    __shared__ __align__(16) uint32_t hist[2048];
    __shared__ uint32_t tmp[32];
    __shared__ uint32_t scal[8];
    __shared__ float red[16];
    const int row = blockIdx.x, b = row / p.Hq;
    const int seq_len = p.seq_lens[b];
    if (seq_len < 1 || seq_len > p.L_max) {
        if (threadIdx.x == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    if (threadIdx.x == 0 && p.counters) p.counters[row] = 0u;
    const int nblk = (seq_len + p.block_size - 1) / p.block_size;
    const int ncomp = nblk - p.force_last;  // blocks competing for the top_blocks slots
    const int top = p.top_blocks, width = top + p.force_last;
    int32_t *out = p.block_idx + (size_t)row * width;
    if (trivial_blocks(ncomp, nblk, top, width, out)) return;
    const float *sc = p.bscore + (size_t)row * p.nblk_max;
    if (keep_top_blocks_hist(sc, ukey, ncomp, nblk, top, p.force_last, out, p.status, hist, tmp, scal, red)) return;
    __syncthreads();
    keep_top_blocks(ukey, ncomp, nblk, top, p.force_last, out, p.status, hist, tmp, &scal[0], &scal[1]);
}

// block_scores and block_topk in one launch, for a kv-head's block scores that
// fit in shared memory: a cluster of kClusterCtas CTAs per (b, kv-head).  CTA
// r of the cluster scores the r-th contiguous chunk of the competing blocks
// against all G query heads of the kv-head (each block key read once) into
// its own shared memory; after a cluster barrier, CTA g mod kClusterCtas
// gathers head g's scores of every chunk from the other CTAs' shared memory
// (distributed shared memory) and keeps its top blocks.  A last cluster
// barrier keeps every CTA's scores in place until all gathers are done.
// (four CTAs per SM: 64 clusters of 8 fit in one wave on 148 SMs)
template <typename T>
__global__ void __launch_bounds__(kSelThreads, 4) block_select_cluster(BlockSelectParams p) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    extern __shared__ float4 dyn4[];
    __shared__ __align__(16) uint32_t hist[2048];
    __shared__ uint32_t tmp[32];
    __shared__ uint32_t scal[8];
    __shared__ float red[16];
    const int G = p.G;
    const int chmax = (p.nblk_max + kClusterCtas - 1) / kClusterCtas;
    float4 *qs = dyn4;                                          // [G][32]
    float *sc = reinterpret_cast<float *>(dyn4 + G * 32);       // [G][chmax]
    uint32_t *ukey = reinterpret_cast<uint32_t *>(sc + (size_t)G * chmax);  // [nblk_max]
    float *xs = reinterpret_cast<float *>(ukey + p.nblk_max);               // [nblk_max] one head's scores
    const int rank = (int)cluster.block_rank();
    const int bh = blockIdx.y, b = bh / p.Hkv, kvh = bh - b * p.Hkv;
    const int seq_len = p.seq_lens[b];
    const bool valid = seq_len >= 1 && seq_len <= p.L_max;
    const int nblk = valid ? (seq_len + p.block_size - 1) / p.block_size : 0;
    const int ncomp = nblk - p.force_last;
    const int top = p.top_blocks, width = top + p.force_last;
    const bool rank_rows = valid && ncomp > top && top > 0;
    const int ch = (max(ncomp, 1) + kClusterCtas - 1) / kClusterCtas;  // <= chmax
    if (rank_rows) {
        const T *q = reinterpret_cast<const T *>(p.q) + ((size_t)b * p.Hq + (size_t)kvh * G) * kHeadDim;
        for (int e = threadIdx.x; e < G * 32; e += kSelThreads) qs[e] = load4(q + 4 * e);
        __syncthreads();
        // eight lanes per block, lane c holding float4 columns c, c + 8, c + 16,
        // c + 24; the loads of kRounds rounds of blocks are issued before any
        // of them is scored (one memory round trip per kRounds rounds)
        constexpr int kRounds = 2;
        const int c = threadIdx.x & 7;
        const float4 *bk = reinterpret_cast<const float4 *>(p.block_keys + (size_t)bh * p.nblk_max * kHeadDim);
        const int j_lo = rank * ch, j_hi = min(ncomp, j_lo + ch);
        for (int j0 = j_lo; j0 < j_hi; j0 += kRounds * (kSelThreads / 8)) {
            float4 kv[kRounds][4];
#pragma unroll
            for (int r = 0; r < kRounds; r++) {
                const int j = j0 + r * (kSelThreads / 8) + (threadIdx.x >> 3);
#pragma unroll
                for (int u = 0; u < 4; u++)
                    kv[r][u] = j < j_hi ? __ldg(bk + (size_t)j * 32 + c + 8 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int r = 0; r < kRounds; r++) {
                const int j = j0 + r * (kSelThreads / 8) + (threadIdx.x >> 3);
                for (int g = 0; g < G; g++) {
                    float s = 0.f;
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const float4 qv = qs[g * 32 + c + 8 * u];
                        s += qv.x * kv[r][u].x + qv.y * kv[r][u].y + qv.z * kv[r][u].z + qv.w * kv[r][u].w;
                    }
                    s += __shfl_xor_sync(0xffffffffu, s, 1);
                    s += __shfl_xor_sync(0xffffffffu, s, 2);
                    s += __shfl_xor_sync(0xffffffffu, s, 4);
                    if (c == 0 && j < j_hi) sc[(size_t)g * chmax + (j - j_lo)] = s * p.scale;
                }
            }
        }
    }
    cluster.sync();  // every chunk's scores are in place
    for (int g = rank; g < G; g += kClusterCtas) {
        const int row = b * p.Hq + kvh * G + g;
        if (!valid) {
            if (threadIdx.x == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
            continue;
        }
        if (threadIdx.x == 0 && p.counters) p.counters[row] = 0u;
        int32_t *out = p.block_idx + (size_t)row * width;
        if (trivial_blocks(ncomp, nblk, top, width, out)) continue;
        for (int j = threadIdx.x; j < ncomp; j += kSelThreads) {
            const int owner = j / ch;
            const float *remote = cluster.map_shared_rank(sc, owner);
            xs[j] = remote[(size_t)g * chmax + (j - owner * ch)];
        }
        __syncthreads();
        if (!keep_top_blocks_hist(xs, ukey, ncomp, nblk, top, p.force_last, out, p.status, hist, tmp, scal, red)) {
            __syncthreads();
            keep_top_blocks(ukey, ncomp, nblk, top, p.force_last, out, p.status, hist, tmp, &scal[0], &scal[1]);
        }
        __syncthreads();  // xs and ukey are rewritten for the next head
    }
    cluster.sync();  // no CTA's scores go away while another CTA still reads them
}

// ---------------------------------------------------------------- hisa_scores
//
// Hierarchical selection ("Sparse Attention Landscape", section "Hierarchical
// Sparse Attention"): token scores only inside the kept blocks.  Grid (slot,
// row): the CTA scores the tokens of the row's slot-th kept block into
// cscore[row, slot * bs + t] (-inf past the sequence end); the kept blocks are
// ascending and only the sequence's last block can be partial, so the valid
// candidates are a prefix of the row, whose length slot 0 records.
template <typename T>
__global__ void __launch_bounds__(128) hisa_scores(HisaScoreParams p) {
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    const int slot = blockIdx.x, row = blockIdx.y, b = row / p.Hq, h = row - b * p.Hq;
    const int seq_len = p.seq_lens[b];
    if (seq_len < 1 || seq_len > p.L_max) return;  // block_topk raised the status
    const int32_t *bi = p.block_idx + (size_t)row * p.top_blocks;
    if (slot == 0 && threadIdx.x == 0) {
        int len = 0;
        for (int s2 = 0; s2 < p.top_blocks && bi[s2] >= 0; s2++)
            len = s2 * p.block_size + min(p.block_size, seq_len - bi[s2] * p.block_size);
        p.row_len[row] = len;
    }
    const int j = bi[slot];
    float *dst = p.cscore + (size_t)row * p.ldc + (size_t)slot * p.block_size;
    if (j < 0) {
        for (int t = threadIdx.x; t < p.block_size; t += 128) dst[t] = -INFINITY;
        return;
    }
    const int lo = j * p.block_size, n = min(p.block_size, seq_len - lo);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float4 qv = load4(reinterpret_cast<const T *>(p.q) + (size_t)row * kHeadDim + 4 * lane);
    const T *K = reinterpret_cast<const T *>(p.k) + (((size_t)b * p.Hkv + h / p.G) * p.L_max + lo) * kHeadDim;
    for (int t = warp; t < p.block_size; t += 4) {
        float s = -INFINITY;
        if (t < n) {
            const float4 kv = load4(K + (size_t)t * kHeadDim + 4 * lane);
            s = warp_sum(qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w) * p.scale;
        }
        if (lane == 0) dst[t] = s;
    }
}

// ---------------------------------------------------------------- block_attn
//
// Persistent: kAttnCtasPerSm CTAs per SM, each walking an equal contiguous
// share of the work items (row, slot) in row-major order.
//   warp 8 (producer) fetches every item's kept block into the next free stage
//     of a ring: for bf16 the K block as two 64-dim boxes of a tensor map with
//     the 128-byte swizzle (so the tensor-core fragment loads below are free
//     of bank conflicts), V rows and the row's query with plain bulk copies,
//     all completing on the stage's mbarrier;
//   warps 0-7 (consumers) take the stages in order: scores q.K^T (bf16: one
//     m16n8k16 tensor-core tile per 8 keys, the query in row 0 of A; fp32:
//     FMA), the block max, e^{s - m} against the row's running max, and
//     P.V with fp32 weights on the FMA pipes, rescaling the running sums
//     (online softmax).  A row whose slots all fall in one CTA is finished in
//     registers and written out;
//   warp 9 (merger) handles the at most two rows this CTA shares with its
//     neighbours: their pieces (m, l, acc) go to the workspace and the CTA
//     that completes a row's last piece (an atomic ticket) merges the pieces
//     in piece order, so the result does not depend on timing.
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kProducerWarp = kConsumerWarps, kMergerWarp = kConsumerWarps + 1;
constexpr int kAttnThreads = kConsumers + 64;
constexpr int kAttnCtasPerSm = 3;
constexpr size_t kStageBudget = 70 * 1024;  // dynamic shared memory per CTA for the ring
constexpr int kMaxStages = 8;
constexpr int kMaxBlockSize = 128;

struct AttnShared {
    uint64_t full[kMaxStages], empty[kMaxStages];
    uint64_t piece_ready[2];  // consumers -> merger: a shared row's piece is in the workspace
    int n[kMaxStages];        // rows of the stage's block (0: an empty slot)
    float sc[kMaxBlockSize];  // the current block's scores
    float pw[kMaxBlockSize];  // e^{s - m} of the current block
    float red[kConsumerWarps][kHeadDim];
    float red_l[kConsumerWarps];
    int abort;
};

// The CTA owning item i when N items are split into `grid` contiguous shares,
// share c being [floor(c N / grid), floor((c + 1) N / grid)).
__device__ __forceinline__ int item_owner(long long i, long long N, int grid) {
    return (int)(((i + 1) * grid + N - 1) / N) - 1;
}

// bar.sync over the consumer warps; returns whether `pred` held in all of them.
__device__ __forceinline__ bool consumers_all(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n"
        ".reg .pred p, q;\n"
        "setp.ne.u32 p, %1, 0;\n"
        "bar.red.and.pred q, 1, %2, p;\n"
        "selp.u32 %0, 1, 0, q;\n"
        "}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "n"(kConsumers)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void consumers_sync() { sm100::named_bar_sync(1, kConsumers); }

// Four 8x8 b16 matrices from shared memory; lane i addresses row i % 8 of matrix i / 8.
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t saddr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr));
}

// D = A (16x16 bf16, row-major) * B (16x8 bf16, column-major) + D, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// kProbe: the pipeline waits are diagnostic probes bounded by p.max_polls
// (the instantiation launched only when a test has lowered the limit)
template <typename T, bool kProbe>
__global__ void __launch_bounds__(kAttnThreads, kAttnCtasPerSm)
    block_attn(const __grid_constant__ CUtensorMap kmap, BlockAttnParams p) {
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    extern __shared__ unsigned char smem_raw[];
    __shared__ AttnShared sh;
    constexpr bool kBf16 = sizeof(T) == 2;
    constexpr uint32_t kRowBytes = kHeadDim * sizeof(T);
    // the swizzled K boxes want 1024-byte aligned stages
    unsigned char *stage_mem = smem_raw + ((1024u - (sm100::smem_addr(smem_raw) & 1023u)) & 1023u);
    const int nslots = p.top_blocks + 1;
    const long long N = (long long)p.B * p.Hq * nslots;
    const long long beg = N * blockIdx.x / gridDim.x, end = N * (blockIdx.x + 1) / gridDim.x;
    const int S = p.stages, bs = p.block_size;
    const uint32_t stage_bytes = p.stage_bytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // rows of this share that other CTAs also hold a piece of: at most the first and the last
    auto row_shared = [&](int row) {
        return item_owner((long long)row * nslots, N, gridDim.x) !=
               item_owner((long long)row * nslots + nslots - 1, N, gridDim.x);
    };
    const int r_first = (int)(beg / nslots), r_last = (int)((end - 1) / nslots);
    const bool first_shared = beg < end && row_shared(r_first);
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            sm100::mbar_init(&sh.full[s], 1);
            sm100::mbar_init(&sh.empty[s], kConsumerWarps);
        }
        sm100::mbar_init(&sh.piece_ready[0], kConsumerWarps);
        sm100::mbar_init(&sh.piece_ready[1], kConsumerWarps);
        sh.abort = 0;
        sm100::fence_barrier_init();
    }
    __syncthreads();
    volatile int *abort = &sh.abort;
    const uint32_t polls = p.max_polls;  // diagnostic probes (kProbe only)

    if (warp == kProducerWarp) {
        // ------------------------------------------------ producer warp
        if (kBf16 && lane == 0) sm100::prefetch_tensormap(&kmap);
        long long issued = 0;
        for (long long i0 = beg; i0 < end; i0 += 32) {
            if (__shfl_sync(0xffffffffu, *abort, 0)) break;
            // the warp looks up 32 items at once: kept block and its row count
            int nj = 0;
            const long long i = i0 + lane;
            if (i < end) {
                const int row = (int)(i / nslots), b = row / p.Hq;
                const int seq_len = p.seq_lens[b];
                if (seq_len >= 1 && seq_len <= p.L_max) {
                    const int j = p.block_idx[i];
                    if (j >= 0 && j * bs < seq_len)
                        nj = min(bs, seq_len - j * bs) | (j << 8);  // block index travels with the count
                    else if (j >= 0)  // never true unless block_topk is wrong
                        raise_status(p.status, TKA_DEV_INTERNAL);
                }
            }
            const int cnt = (int)min((long long)32, end - i0);
            for (int u = 0; u < cnt; u++) {
                const int v = __shfl_sync(0xffffffffu, nj, u);
                if (lane == 0) {
                    const long long k = i0 + u - beg;
                    const int s = (int)(k % S);
                    const bool ok =
                        k < S || sm100::pipe_wait<kProbe>(&sh.empty[s], (uint32_t)((k / S - 1) & 1), abort, polls);
                    if (ok) {
                        const int rows = v & 255;
                        sh.n[s] = rows;
                        if (rows > 0) {
                            const int row = (int)((i0 + u) / nslots), b = row / p.Hq, h = row - b * p.Hq;
                            const size_t krow = ((size_t)b * p.Hkv + h / p.G) * p.L_max + (size_t)(v >> 8) * bs;
                            unsigned char *st = stage_mem + (size_t)s * stage_bytes;
                            uint64_t *bar = &sh.full[s];
                            if constexpr (kBf16) {
                                // K: two 64-dim boxes of bs rows (full boxes even past the sequence end)
                                sm100::mbar_arrive_expect_tx(bar, (uint32_t)bs * kRowBytes + (uint32_t)rows * kRowBytes +
                                                                      kRowBytes);
                                sm100::tma_load_2d(st, &kmap, bar, 0, (int)krow);
                                sm100::tma_load_2d(st + (size_t)bs * 128, &kmap, bar, 64, (int)krow);
                            } else {
                                sm100::mbar_arrive_expect_tx(bar, 2u * rows * kRowBytes + kRowBytes);
                                sm100::bulk_load(st, reinterpret_cast<const T *>(p.k) + krow * kHeadDim,
                                                 (uint32_t)rows * kRowBytes, bar);
                            }
                            sm100::bulk_load(st + (size_t)bs * kRowBytes, reinterpret_cast<const T *>(p.v) + krow * kHeadDim,
                                             (uint32_t)rows * kRowBytes, bar);
                            sm100::bulk_load(st + 2 * (size_t)bs * kRowBytes,
                                             reinterpret_cast<const T *>(p.q) + (size_t)row * kHeadDim, kRowBytes, bar);
                        } else {
                            sm100::mbar_arrive(&sh.full[s]);
                        }
                        issued = k + 1;
                    } else {
                        if (!*abort) raise_status(p.status, TKA_DEV_TIMEOUT);
                        *abort = 1;
                    }
                }
                if (__shfl_sync(0xffffffffu, *abort, 0)) break;
            }
        }
        if (lane == 0 && *abort) {
            // copies still in flight write this CTA's shared memory: wait for
            // them (bounded) before the CTA may exit
            int never = 0;
            for (long long k = issued > S ? issued - S : 0; k < issued; k++)
                sm100::mbar_wait(&sh.full[k % S], (uint32_t)((k / S) & 1), &never);
        }
        return;
    }

    if (warp == kMergerWarp) {
        // ------------------------------------------------ merger warp
        int erow[2], ne = 0;
        if (first_shared) erow[ne++] = r_first;
        if (beg < end && r_last != r_first && row_shared(r_last)) erow[ne++] = r_last;
        for (int e = 0; e < ne; e++) {
            if (!sm100::pipe_wait<kProbe>(&sh.piece_ready[e], 0, abort, polls)) break;
            const int row = erow[e];
            const int seq_len = p.seq_lens[row / p.Hq];
            if (seq_len < 1 || seq_len > p.L_max) continue;  // block_topk raised the status
            const int o_first = item_owner((long long)row * nslots, N, gridDim.x);
            const int npieces = item_owner((long long)row * nslots + nslots - 1, N, gridDim.x) - o_first + 1;
            __threadfence();  // the consumers' piece, seen through piece_ready, before the ticket
            unsigned ticket = 0u;
            if (lane == 0) ticket = atomicAdd(&p.counters[row], 1u);
            ticket = __shfl_sync(0xffffffffu, ticket, 0);
            if (ticket != (unsigned)npieces - 1) continue;
            __threadfence();
            const size_t p0 = (size_t)row * nslots;
            float M = -INFINITY;
            for (int q = 0; q < npieces; q++) M = fmaxf(M, __ldcg(&p.part_ml[p0 + q].x));
            float L = 0.f;
            float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int q = 0; q < npieces; q++) {
                const float4 ml = __ldcg(&p.part_ml[p0 + q]);
                if (ml.y == 0.f) continue;
                const float f = __expf(ml.x - M);
                const float4 a = __ldcg(reinterpret_cast<const float4 *>(p.part_acc + (p0 + q) * kHeadDim) + lane);
                L += ml.y * f;
                A.x += a.x * f;
                A.y += a.y * f;
                A.z += a.z * f;
                A.w += a.w * f;
            }
            const float inv = 1.f / L;
            reinterpret_cast<float4 *>(p.out + (size_t)row * kHeadDim)[lane] =
                make_float4(A.x * inv, A.y * inv, A.z * inv, A.w * inv);
            if (lane == 0) p.counters[row] = 0u;
        }
        return;
    }

    // ---------------------------------------------------- consumer warps
    // P.V mapping: dg = lane & 15 picks 8 output dims, rows rg, rg + 16, ...
    const int dg = lane & 15, rg = threadIdx.x >> 4;
    auto dim_of = [&](int e) {  // output dim of this thread's accumulator e
        return kBf16 ? 8 * dg + e : (e < 4 ? 4 * dg + e : 64 + 4 * dg + e - 4);
    };
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; e++) acc[e] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    int cur_row = -1;
    bool cur_valid = false;

    // finishes this CTA's piece of row `row`
    auto flush = [&](int row) {
#pragma unroll
        for (int e = 0; e < 8; e++) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
        const float lw = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
        if (lane < 16) {
#pragma unroll
            for (int e = 0; e < 8; e++) sh.red[warp][dim_of(e)] = acc[e];
        }
        if (lane == 0) sh.red_l[warp] = lw;
        consumers_sync();
        const bool shared = row_shared(row);
        const int d = threadIdx.x;
        if (cur_valid && d < kHeadDim) {
            float A = 0.f, L = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; w++) {
                A += sh.red[w][d];
                L += sh.red_l[w];
            }
            if (!shared) {
                p.out[(size_t)row * kHeadDim + d] = A / L;
            } else {
                const size_t ps = (size_t)row * nslots + ((int)blockIdx.x - item_owner((long long)row * nslots, N, gridDim.x));
                p.part_acc[ps * kHeadDim + d] = A;
                if (d == 0) p.part_ml[ps] = make_float4(m_run, L, 0.f, 0.f);
            }
        }
        if (shared) {
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&sh.piece_ready[(row == r_first || !first_shared) ? 0 : 1]);
        }
#pragma unroll
        for (int e = 0; e < 8; e++) acc[e] = 0.f;
        m_run = -INFINITY;
        l_run = 0.f;
    };

    for (long long i = beg; i < end; i++) {
        const long long k = i - beg;
        const int s = (int)(k % S);
        const int row = (int)(i / nslots);
        if (row != cur_row) {
            if (cur_row >= 0) flush(cur_row);
            cur_row = row;
            const int sl = p.seq_lens[row / p.Hq];
            cur_valid = sl >= 1 && sl <= p.L_max;
        }
        const bool landed = sm100::pipe_wait<kProbe>(&sh.full[s], (uint32_t)((k / S) & 1), abort, polls);
        if (!consumers_all(landed)) {
            if (threadIdx.x == 0) {
                if (!*abort) raise_status(p.status, TKA_DEV_TIMEOUT);
                *abort = 1;
            }
            cur_row = -1;  // no result for the rows left
            break;
        }
        const int n = sh.n[s];
        if (n > 0) {
            const unsigned char *st = stage_mem + (size_t)s * stage_bytes;
            const unsigned char *Vs = st + (size_t)bs * kRowBytes;
            const unsigned char *Qs = st + 2 * (size_t)bs * kRowBytes;
            if constexpr (kBf16) {
                // scores on the tensor cores: warp w takes keys 8 nt .. 8 nt + 7 for nt = w, w + 8;
                // the query is row 0 of A (lanes 0-3 hold it), the keys are the columns of B
                const uint32_t *qw = reinterpret_cast<const uint32_t *>(Qs) + (lane & 3);
                const bool qrow = lane < 4;
                const uint32_t kbase = sm100::smem_addr(st);
                for (int nt = warp; nt * 8 < n; nt += kConsumerWarps) {
                    float dacc[4] = {0.f, 0.f, 0.f, 0.f};
                    const int key = nt * 8 + (lane & 7);
#pragma unroll
                    for (int kp = 0; kp < 4; kp++) {
                        // k-steps 2kp and 2kp+1: 16-byte chunks c0 .. c0+3 of box kp/2
                        const int chunk = (kp & 1) * 4 + (lane >> 3);
                        const uint32_t addr = kbase + (uint32_t)(kp >> 1) * (uint32_t)bs * 128u + (uint32_t)key * 128u +
                                              (uint32_t)((chunk ^ (key & 7)) << 4);
                        uint32_t b[4];
                        ldmatrix_x4(b, addr);
                        // A row 0: dims 16 ks + 2 (lane & 3) (+1) and 16 ks + 8 + 2 (lane & 3) (+1)
                        const uint32_t a00 = qrow ? qw[16 * kp] : 0u, a02 = qrow ? qw[16 * kp + 4] : 0u;
                        const uint32_t a10 = qrow ? qw[16 * kp + 8] : 0u, a12 = qrow ? qw[16 * kp + 12] : 0u;
                        mma_16816(dacc, a00, 0u, a02, 0u, b[0], b[1]);
                        mma_16816(dacc, a10, 0u, a12, 0u, b[2], b[3]);
                    }
                    if (lane < 4) {
                        const int t = nt * 8 + 2 * lane;
                        if (t < n) sh.sc[t] = dacc[0] * p.scale;
                        if (t + 1 < n) sh.sc[t + 1] = dacc[1] * p.scale;
                    }
                }
            } else {
                // fp32: eight lanes per key, lane c holding float4 columns c, c + 8, c + 16, c + 24
                const int c = lane & 7, sub = lane >> 3;
                float4 qv[4];
#pragma unroll
                for (int u = 0; u < 4; u++) qv[u] = reinterpret_cast<const float4 *>(Qs)[c + 8 * u];
                for (int t0 = warp * 4; t0 < n; t0 += kConsumerWarps * 4) {
                    const int t = t0 + sub;
                    const float4 *kr = reinterpret_cast<const float4 *>(st + (size_t)min(t, n - 1) * kRowBytes);
                    float sd = 0.f;
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const float4 w = kr[c + 8 * u];
                        sd = fmaf(qv[u].x, w.x, sd);
                        sd = fmaf(qv[u].y, w.y, sd);
                        sd = fmaf(qv[u].z, w.z, sd);
                        sd = fmaf(qv[u].w, w.w, sd);
                    }
                    sd += __shfl_xor_sync(0xffffffffu, sd, 1);
                    sd += __shfl_xor_sync(0xffffffffu, sd, 2);
                    sd += __shfl_xor_sync(0xffffffffu, sd, 4);
                    if (c == 0 && t < n) sh.sc[t] = sd * p.scale;
                }
            }
            consumers_sync();
            // block max (every warp computes it), new running max, weights
            float mb = -INFINITY;
            for (int t = lane; t < n; t += 32) mb = fmaxf(mb, sh.sc[t]);
            mb = warp_max(mb);
            const float m_new = fmaxf(m_run, mb);
            const float f = __expf(m_run - m_new);  // 0 for the row's first block
            m_run = m_new;
            if (threadIdx.x < n) sh.pw[threadIdx.x] = __expf(sh.sc[threadIdx.x] - m_new);
            consumers_sync();
#pragma unroll
            for (int e = 0; e < 8; e++) acc[e] *= f;
            l_run *= f;
            for (int t = rg; t < n; t += 16) {
                const float w = sh.pw[t];
                const unsigned char *vr = Vs + (size_t)t * kRowBytes;
                if constexpr (kBf16) {
                    const uint4 v = reinterpret_cast<const uint4 *>(vr)[dg];
                    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        acc[2 * e] = fmaf(w, bf16lo_to_f32(vw[e]), acc[2 * e]);
                        acc[2 * e + 1] = fmaf(w, bf16hi_to_f32(vw[e]), acc[2 * e + 1]);
                    }
                } else {
                    const float4 v0 = reinterpret_cast<const float4 *>(vr)[dg];
                    const float4 v1 = reinterpret_cast<const float4 *>(vr)[16 + dg];
                    acc[0] = fmaf(w, v0.x, acc[0]);
                    acc[1] = fmaf(w, v0.y, acc[1]);
                    acc[2] = fmaf(w, v0.z, acc[2]);
                    acc[3] = fmaf(w, v0.w, acc[3]);
                    acc[4] = fmaf(w, v1.x, acc[4]);
                    acc[5] = fmaf(w, v1.y, acc[5]);
                    acc[6] = fmaf(w, v1.z, acc[6]);
                    acc[7] = fmaf(w, v1.w, acc[7]);
                }
                l_run += w;
            }
        }
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&sh.empty[s]);
    }
    if (cur_row >= 0) flush(cur_row);
}


// Opts a kernel in to `smem` bytes of dynamic shared memory when that, with
// the kernel's static shared memory, passes the 48 KB available without it.
template <typename F>
cudaError_t allow_smem(F *kernel, size_t smem) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    if (smem + fa.sharedSizeBytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

}  // namespace

cudaError_t launch_block_pool(const BlockPoolParams &p, cudaStream_t stream) {
    const dim3 grid(p.nblk_max, p.B * p.Hkv);
    if (p.dtype == TKA_BF16) return launch_k(true, block_pool<__nv_bfloat16>, grid, dim3(128), 0, stream, p);
    return launch_k(true, block_pool<float>, grid, dim3(128), 0, stream, p);
}

cudaError_t launch_block_select(const BlockSelectParams &p, cudaStream_t stream) {
    cudaError_t e;
    // one launch on a cluster per (b, kv-head) when the kv-head's scores fit
    // in shared memory: query rows, G chunks of scores and the gathered keys
    const size_t chmax = (p.nblk_max + kClusterCtas - 1) / kClusterCtas;
    const size_t csmem = (size_t)p.G * 32 * sizeof(float4) + (size_t)p.G * chmax * sizeof(float) +
                         (size_t)p.nblk_max * (sizeof(uint32_t) + sizeof(float));
    if (csmem <= kClusterSmem) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kClusterCtas, p.B * p.Hkv);
        cfg.blockDim = dim3(kSelThreads);
        cfg.dynamicSmemBytes = csmem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kClusterCtas;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        if (p.dtype == TKA_BF16) {
            if ((e = allow_smem(block_select_cluster<__nv_bfloat16>, csmem)) != cudaSuccess) return e;
            return cudaLaunchKernelEx(&cfg, block_select_cluster<__nv_bfloat16>, p);
        }
        if ((e = allow_smem(block_select_cluster<float>, csmem)) != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, block_select_cluster<float>, p);
    }
    // otherwise: scores to the workspace, then one CTA per row
    const dim3 sgrid((p.nblk_max + kScoreBlocks - 1) / kScoreBlocks, p.B * p.Hkv);
    const size_t qsmem = (size_t)p.G * kHeadDim * sizeof(float);
    if (p.dtype == TKA_BF16) {
        if ((e = allow_smem(block_scores<__nv_bfloat16>, qsmem)) != cudaSuccess) return e;
        e = launch_k(true, block_scores<__nv_bfloat16>, sgrid, dim3(kSelThreads), qsmem, stream, p);
    } else {
        if ((e = allow_smem(block_scores<float>, qsmem)) != cudaSuccess) return e;
        e = launch_k(true, block_scores<float>, sgrid, dim3(kSelThreads), qsmem, stream, p);
    }
    if (e != cudaSuccess) return e;
    const size_t ksmem = (size_t)p.nblk_max * sizeof(uint32_t);
    if ((e = allow_smem(block_topk, ksmem)) != cudaSuccess) return e;  // + 8.3 KB of static shared memory
    return launch_k(true, block_topk, dim3(p.B * p.Hq), dim3(kSelThreads), ksmem, stream, p);
}

cudaError_t launch_hisa_scores(const HisaScoreParams &p, cudaStream_t stream) {
    const dim3 grid(p.top_blocks, p.B * p.Hq);
    if (p.dtype == TKA_BF16) return launch_k(true, hisa_scores<__nv_bfloat16>, grid, dim3(128), 0, stream, p);
    return launch_k(true, hisa_scores<float>, grid, dim3(128), 0, stream, p);
}

cudaError_t launch_block_attn(const BlockAttnParams &p0, const void *k_cache, int num_sms, cudaStream_t stream) {
    BlockAttnParams p = p0;
    const bool bf16 = p.dtype == TKA_BF16;
    const size_t row_bytes = kHeadDim * (bf16 ? 2 : 4);
    p.stage_bytes = (uint32_t)(((2 * (size_t)p.block_size + 1) * row_bytes + 1023) / 1024 * 1024);
    p.stages = (int)max((size_t)1, min((size_t)kMaxStages, kStageBudget / p.stage_bytes));
    const size_t smem = 1024 + (size_t)p.stages * p.stage_bytes;  // + slack to align the ring to 1024 bytes
    const long long items = (long long)p.B * p.Hq * (p.top_blocks + 1);
    const int grid = (int)min((long long)num_sms * kAttnCtasPerSm, items);
    CUtensorMap kmap;
    memset(&kmap, 0, sizeof(kmap));
    cudaError_t e;
    if (bf16) {
        // K cache as rows of 128 bf16: [B*Hkv*L_max, 128]; boxes of block_size rows x 64 dims
        EncodeTiledFn enc = encode_fn();
        if (!enc) return cudaErrorNotSupported;
        const cuuint64_t dims[2] = {128, (cuuint64_t)p.B * p.Hkv * p.L_max};
        const cuuint64_t strides[1] = {256};
        const cuuint32_t box[2] = {64, (cuuint32_t)p.block_size};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(k_cache), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        if ((e = allow_smem(block_attn<__nv_bfloat16, false>, smem)) != cudaSuccess) return e;
        if ((e = allow_smem(block_attn<__nv_bfloat16, true>, smem)) != cudaSuccess) return e;
        if (p.max_polls)
            return launch_k(true, block_attn<__nv_bfloat16, true>, dim3(grid), dim3(kAttnThreads), smem, stream, kmap, p);
        return launch_k(true, block_attn<__nv_bfloat16, false>, dim3(grid), dim3(kAttnThreads), smem, stream, kmap, p);
    }
    if ((e = allow_smem(block_attn<float, false>, smem)) != cudaSuccess) return e;
    if ((e = allow_smem(block_attn<float, true>, smem)) != cudaSuccess) return e;
    if (p.max_polls)
        return launch_k(true, block_attn<float, true>, dim3(grid), dim3(kAttnThreads), smem, stream, kmap, p);
    return launch_k(true, block_attn<float, false>, dim3(grid), dim3(kAttnThreads), smem, stream, kmap, p);
}

}  // namespace tka
