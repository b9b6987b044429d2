// Block-sparse (MoBA) decode attention.
//
// "Sparse Attention Landscape", section "Block Sparse Attention": the cache is
// cut into blocks, each block gets one relevance score, the top blocks are
// kept and attention runs over the tokens inside them; MoBA's block score is
// the dot product of the query with the mean-pooled keys of the block.  The
// last (current) block is always kept.
//
// Three kernels:
//   block_pool    block_keys[b,h,j,:] = mean of the block's keys (fp32), built
//                 when blocks change, not per decode step.
//   block_select  one CTA per query row: scores every competing block against
//                 the block keys, sorts (score desc, block asc) with a bitonic
//                 network in shared memory, keeps the best top_blocks plus the
//                 current block, writes them ascending.
//   block_attn    grid (kept slot, row): one CTA per kept block computes the
//                 block's scores, its local max m, sum l and sum p*V; the last
//                 CTA of the row merges the slots with the usual max-rescaled
//                 softmax merge, in slot order.  Kept blocks are contiguous
//                 rows of the cache, so K and V are read as whole 256-byte rows.
#include "common.cuh"
#include "kernels.h"

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

template <typename T>
__global__ void __launch_bounds__(128) block_pool(BlockPoolParams p) {
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

constexpr int kSelThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kSelThreads) block_select(BlockSelectParams p) {
    extern __shared__ unsigned long long keys[];  // [npow2]
    __shared__ float4 qv[kHeadDim / 4];
    __shared__ int32_t kept[256];
    const int row = blockIdx.x, b = row / p.Hq, h = row % p.Hq;
    const int seq_len = p.seq_lens[b];
    if (seq_len < 1 || seq_len > p.L_max) {
        if (threadIdx.x == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    if (threadIdx.x == 0) p.counters[row] = 0u;
    const int nblk = (seq_len + p.block_size - 1) / p.block_size;
    const int ncomp = nblk - 1;  // blocks competing for the top_blocks slots
    int npow2 = 1;
    while (npow2 < ncomp) npow2 <<= 1;
    const T *q = reinterpret_cast<const T *>(p.q) + (size_t)row * kHeadDim;
    if (threadIdx.x < kHeadDim / 4) qv[threadIdx.x] = load4(q + 4 * threadIdx.x);
    __syncthreads();
    // block scores; composite key orders by (score desc, block asc)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float *bk = p.block_keys + ((size_t)b * p.Hkv + h / p.G) * p.nblk_max * kHeadDim;
    const float4 ql = qv[lane];
    for (int j = warp; j < npow2; j += kSelThreads / 32) {
        unsigned long long key = 0ull;  // padding sorts last
        if (j < ncomp) {
            const float4 kv = __ldg(reinterpret_cast<const float4 *>(bk + (size_t)j * kHeadDim) + lane);
            float s = ql.x * kv.x + ql.y * kv.y + ql.z * kv.z + ql.w * kv.w;
            s = warp_sum(s) * p.scale;
            key = ((unsigned long long)order_key(s) << 32) | (0xffffffffu - (unsigned)j);
        }
        if (lane == 0) keys[j] = key;
    }
    __syncthreads();
    // bitonic sort, descending
    for (int size = 2; size <= npow2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < npow2 / 2; i += kSelThreads) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = ((lo & size) == 0);
                const unsigned long long a = keys[lo], c = keys[hi];
                if ((a < c) == desc) {
                    keys[lo] = c;
                    keys[hi] = a;
                }
            }
            __syncthreads();
        }
    }
    const int nk = min(p.top_blocks, ncomp);
    for (int i = threadIdx.x; i < nk; i += kSelThreads) kept[i] = (int32_t)(0xffffffffu - (unsigned)(keys[i] & 0xffffffffull));
    if (threadIdx.x == 0) kept[nk] = nblk - 1;
    __syncthreads();
    // ascending order by rank
    int32_t *out = p.block_idx + (size_t)row * (p.top_blocks + 1);
    for (int i = threadIdx.x; i <= nk; i += kSelThreads) {
        const int v = kept[i];
        int rank = 0;
        for (int e = 0; e <= nk; e++) rank += kept[e] < v;
        out[rank] = v;
    }
    for (int i = nk + 1 + threadIdx.x; i <= p.top_blocks; i += kSelThreads) out[i] = -1;
}

template <typename T>
__global__ void __launch_bounds__(128) block_attn(BlockAttnParams p) {
    __shared__ float sc[128];
    __shared__ float red[32];
    __shared__ unsigned s_ticket;
    const int slot = blockIdx.x, row = blockIdx.y, b = row / p.Hq, h = row % p.Hq;
    const int nslots = p.top_blocks + 1;
    const int seq_len = p.seq_lens[b];
    if (seq_len < 1 || seq_len > p.L_max) return;  // block_select raised the status
    const int j = p.block_idx[(size_t)row * nslots + slot];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const size_t kvoff = ((size_t)b * p.Hkv + h / p.G) * p.L_max * kHeadDim;
    const T *K = reinterpret_cast<const T *>(p.k) + kvoff;
    const T *V = reinterpret_cast<const T *>(p.v) + kvoff;
    float m = -INFINITY, l = 0.f, acc = 0.f;
    if (j >= 0 && j * p.block_size >= seq_len) {  // never true unless block_select is wrong
        if (threadIdx.x == 0) raise_status(p.status, TKA_DEV_INTERNAL);
    } else if (j >= 0) {
        const int lo = j * p.block_size, n = min(p.block_size, seq_len - lo);
        const float4 qv = load4(reinterpret_cast<const T *>(p.q) + (size_t)row * kHeadDim + 4 * lane);
        for (int t = warp; t < n; t += 4) {
            const float4 kv = load4(K + (size_t)(lo + t) * kHeadDim + 4 * lane);
            float s = qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
            s = warp_sum(s) * p.scale;
            if (lane == 0) sc[t] = s;
        }
        __syncthreads();
        float mt = -INFINITY;
        for (int t = threadIdx.x; t < n; t += 128) mt = fmaxf(mt, sc[t]);
        m = block_max(mt, red);
        // each thread owns output dim d = threadIdx.x
        const T *vcol = V + (size_t)lo * kHeadDim + threadIdx.x;
        for (int t = 0; t < n; t++) {
            const float e = __expf(sc[t] - m);
            l += e;
            acc = fmaf(e, load_f32(vcol + (size_t)t * kHeadDim), acc);
        }
    }
    const size_t ps = (size_t)row * nslots + slot;
    if (threadIdx.x == 0) p.part_ml[ps] = make_float4(m, l, 0.f, 0.f);
    p.part_acc[ps * kHeadDim + threadIdx.x] = acc;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(&p.counters[row], 1u);
    __syncthreads();
    if (s_ticket != (unsigned)nslots - 1) return;
    __threadfence();
    float M = -INFINITY;
    for (int s = 0; s < nslots; s++) M = fmaxf(M, __ldcg(&p.part_ml[(size_t)row * nslots + s].x));
    float L = 0.f, A = 0.f;
    for (int s = 0; s < nslots; s++) {
        const float4 ml = __ldcg(&p.part_ml[(size_t)row * nslots + s]);
        if (ml.y == 0.f) continue;
        const float f = __expf(ml.x - M);
        L += ml.y * f;
        A += __ldcg(&p.part_acc[((size_t)row * nslots + s) * kHeadDim + threadIdx.x]) * f;
    }
    p.out[(size_t)row * kHeadDim + threadIdx.x] = A / L;
    if (threadIdx.x == 0) p.counters[row] = 0u;
}

}  // namespace

cudaError_t launch_block_pool(const BlockPoolParams &p, cudaStream_t stream) {
    const dim3 grid(p.nblk_max, p.B * p.Hkv);
    if (p.dtype == TKA_BF16)
        block_pool<__nv_bfloat16><<<grid, 128, 0, stream>>>(p);
    else
        block_pool<float><<<grid, 128, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_block_select(const BlockSelectParams &p, cudaStream_t stream) {
    int npow2 = 1;
    while (npow2 < p.nblk_max) npow2 <<= 1;
    const size_t smem = (size_t)npow2 * sizeof(unsigned long long);
    const int rows = p.B * p.Hq;
    if (p.dtype == TKA_BF16) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(block_select<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        block_select<__nv_bfloat16><<<rows, kSelThreads, smem, stream>>>(p);
    } else {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(block_select<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        block_select<float><<<rows, kSelThreads, smem, stream>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_block_attn(const BlockAttnParams &p, cudaStream_t stream) {
    const dim3 grid(p.top_blocks + 1, p.B * p.Hq);
    if (p.dtype == TKA_BF16)
        block_attn<__nv_bfloat16><<<grid, 128, 0, stream>>>(p);
    else
        block_attn<float><<<grid, 128, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tka
