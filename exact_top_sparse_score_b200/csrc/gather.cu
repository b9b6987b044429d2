// Attention step over the kept positions: out = sum_{i in S} (e^{s_i - m} / Z_k) V[i].
//
// "Sparse attention layers first read the KV entries corresponding to
// positions selected by the Indexer" ("Sparse Attention in LLM Inference:
// Practical Trade-Offs", section "Changes in Caching Strategy"): only the k
// kept V rows are read, by position index.  The weights e^{s_i - m} and Z_k
// come from the select step, so no K row is read again.
//
// Grid (splits, rows): each CTA gathers a contiguous slice of a row's kept
// positions.  The slice's positions and weights are first staged in shared
// memory (coalesced), so the V loads that follow depend on nothing in
// flight: a V row is 256 bytes in bf16, read by 16 lanes with one 16-byte
// load each, and every lane keeps 4 rows in flight (eight CTAs per SM).
// The slices of a row are summed by whichever CTA of the row finishes last
// (an atomic ticket, no waiting), in slice order, so the result does not
// depend on scheduling.
#include "common.cuh"
#include "kernels.h"

namespace tka {

namespace {

constexpr int kGatherThreads = 256;
constexpr int kChunk = 512;  // positions staged in shared memory at a time
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

template <typename T>
__device__ __forceinline__ void fma_row(float (&acc)[16 / sizeof(T)], float wt, const uint4 &v) {
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int e = 0; e < 4; e++) {
            acc[2 * e] = fmaf(wt, bf16lo_to_f32(wd[e]), acc[2 * e]);
            acc[2 * e + 1] = fmaf(wt, bf16hi_to_f32(wd[e]), acc[2 * e + 1]);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 4; e++) acc[e] = fmaf(wt, __uint_as_float(wd[e]), acc[e]);
    }
}

template <typename T, bool kPaged>
__global__ void __launch_bounds__(kGatherThreads, 8) gather_pv(GatherParams p) {
    constexpr int kPer = 16 / sizeof(T);              // elements per lane
    constexpr int kLanesPerRow = kHeadDim / kPer;     // 16 (bf16) or 32 (fp32)
    constexpr int kRowsPerWarp = 32 / kLanesPerRow;   // 2 or 1
    constexpr int kWarps = kGatherThreads / 32;
    constexpr int kSlots = kWarps * kRowsPerWarp;
    __shared__ int32_t s_idx[kChunk];
    __shared__ float s_w[kChunk];
    __shared__ float red[kWarps][kHeadDim];
    __shared__ unsigned s_ticket;

    const int row = blockIdx.y, split = blockIdx.x;
    pdl_wait();  // the kept positions and weights come from the kernel before
    pdl_trigger();
    const int b = row / (p.Q * p.Hq), qpos = (row / p.Hq) % p.Q, h = row % p.Hq;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) return;  // the select step raised the status
    const int vis = visible_keys(seq_len, p.Q, qpos);
    const int kept = p.kcount ? min(p.kcount[row], min(p.k, vis)) : min(p.k, vis);
    const int lo = split * p.per_split;
    const int hi = min(kept, lo + p.per_split);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slot = warp * kRowsPerWarp + lane / kLanesPerRow;
    const int c = lane % kLanesPerRow;  // this lane's 16-byte piece of a V row
    // rows are counted from the (b, kv-head) block of a contiguous cache, or
    // from the start of a paged one (staged below as physical row numbers)
    const T *vbase = reinterpret_cast<const T *>(p.v) +
                     (kPaged ? 0 : ((size_t)b * p.Hkv + h / p.G) * p.L_max * kHeadDim) + c * kPer;
    const int32_t *gidx = p.idx + (size_t)row * p.k;
    const float *gw = p.w + (size_t)row * p.k;

    float acc[kPer];
#pragma unroll
    for (int e = 0; e < kPer; e++) acc[e] = 0.f;
    bool bad = false;

    for (int c0 = lo; c0 < hi; c0 += kChunk) {
        const int n = min(kChunk, hi - c0);
        __syncthreads();
        for (int j = threadIdx.x; j < n; j += kGatherThreads) {
            int pos = __ldg(gidx + c0 + j);
            float wt = __ldg(gw + c0 + j);
            if (p.cblock) {  // a candidate index: map it to its position, report the position
                if ((unsigned)pos < (unsigned)p.crow_len[row]) {
                    pos = p.cblock[(size_t)row * p.cstride + pos / p.cbs] * p.cbs + pos % p.cbs;
                    p.idx_out[(size_t)row * p.k + c0 + j] = pos;
                } else {
                    pos = -1;
                }
            }
            if ((unsigned)pos >= (unsigned)vis) {  // never taken unless the select step is wrong
                bad = true;
                pos = 0;
                wt = 0.f;
            }
            if constexpr (kPaged) pos = (int32_t)paged_row(p.pages, p.status, p.Hkv, b, h / p.G, pos);
            s_idx[j] = pos;
            s_w[j] = wt;
        }
        __syncthreads();
        int j = slot;
        for (; j + (kUnroll - 1) * kSlots < n; j += kUnroll * kSlots) {
            uint4 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; u++) v[u] = ldg_stream(vbase + (size_t)s_idx[j + u * kSlots] * kHeadDim);
#pragma unroll
            for (int u = 0; u < kUnroll; u++) fma_row<T>(acc, s_w[j + u * kSlots], v[u]);
        }
        for (; j < n; j += kSlots) fma_row<T>(acc, s_w[j], ldg_stream(vbase + (size_t)s_idx[j] * kHeadDim));
    }
    if (bad) raise_status(p.status, TKA_DEV_INTERNAL);
    // sum the rows of a warp, then the warps of the CTA
    if constexpr (kRowsPerWarp == 2) {
#pragma unroll
        for (int e = 0; e < kPer; e++) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    }
    if (lane < kLanesPerRow) {
#pragma unroll
        for (int e = 0; e < kPer; e++) red[warp][c * kPer + e] = acc[e];
    }
    __syncthreads();
    if (threadIdx.x >= kHeadDim) return;
    const int d = threadIdx.x;  // one output dim per thread
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; w++) sum += red[w][d];
    const float inv_zk = 1.f / p.stats[row].y;
    float *out = p.out + (size_t)row * kHeadDim;
    if (p.splits == 1) {
        out[d] = sum * inv_zk;
        return;
    }
    float *part = p.partial + (size_t)row * p.splits * kHeadDim;
    part[(size_t)split * kHeadDim + d] = sum;
    __threadfence();
    asm volatile("bar.sync 1, %0;\n" ::"r"(kHeadDim));  // the 128 threads that wrote a partial
    if (threadIdx.x == 0) s_ticket = atomicAdd(&p.counters[row], 1u);
    asm volatile("bar.sync 1, %0;\n" ::"r"(kHeadDim));
    if (s_ticket != (unsigned)p.splits - 1) return;
    __threadfence();
    float total = 0.f;
    for (int sp = 0; sp < p.splits; sp++) total += __ldcg(part + (size_t)sp * kHeadDim + d);
    out[d] = total * inv_zk;
    if (threadIdx.x == 0) p.counters[row] = 0u;
}

}  // namespace

cudaError_t launch_gather(const GatherParams &p, cudaStream_t stream, bool pdl) {
    const int rows = p.B * p.Q * p.Hq;
    const dim3 grid(p.splits, rows);
    const bool paged = p.pages.table != nullptr;
    if (p.dtype == TKA_BF16) {
        if (paged)
            return launch_k(pdl, gather_pv<__nv_bfloat16, true>, grid, dim3(kGatherThreads), 0, stream, p);
        else
            return launch_k(pdl, gather_pv<__nv_bfloat16, false>, grid, dim3(kGatherThreads), 0, stream, p);
    } else {
        if (paged)
            return launch_k(pdl, gather_pv<float, true>, grid, dim3(kGatherThreads), 0, stream, p);
        else
            return launch_k(pdl, gather_pv<float, false>, grid, dim3(kGatherThreads), 0, stream, p);
    }
}

}  // namespace tka
