// Score step: s[row, i] = scale * <q_row, K[b, kvh, i, :]> for every key i
// below the sequence length, for all Q*G query rows that share kv-head kvh.
//
// This is the relevance-scoring pass over the whole cache ("Sparse Attention
// in LLM Inference: Practical Trade-Offs", sections "The Role of the Indexer"
// and "The Overhead of the Indexer": every decode step scans all historical
// positions), with the exact attention logit as the score.  It is the
// bandwidth-dominant step: the whole K cache streams through once, and each
// key row is reused for all Q*G query rows of its GQA group.
//
// Two kernels:
//   score_bf16_mma  bf16 cache.  Each warp loads 16-key x 128-dim tiles of K
//                   straight from HBM into registers with 16-byte coalesced
//                   loads and multiplies them against the group's queries
//                   with bf16 tensor-core MMAs (fp32 accumulate).  The K tile
//                   is the M side (16 keys), the Q*G query rows the N side.
//                   The 128 head dims are walked in a thread-specific order
//                   (the same permutation on both operands), which lets each
//                   thread load whole 16-byte pieces of a key row.
//   score_generic   fp32 (or any) cache on CUDA cores: a quad of lanes per key,
//                   each lane a quarter of the head dims, quad shuffles to sum.
#include "common.cuh"
#include "kernels.h"

namespace tka {

namespace {

constexpr int kChunkKeys = 128;  // keys per CTA iteration: 4 warps x 2 tiles x 16

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Global row index of query row r (0 <= r < Q*G) of kv-head kvh in batch b.
__device__ __forceinline__ size_t global_row(const ScoreParams &p, int b, int kvh, int r) {
    const int qpos = r / p.G, gi = r - qpos * p.G;
    return ((size_t)b * p.Q + qpos) * p.Hq + (size_t)kvh * p.G + gi;
}

// NT = number of 8-wide query tiles (Q*G <= 8*NT).
template <int NT>
__global__ void __launch_bounds__(128) score_bf16_mma(ScoreParams p) {
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    // q fragments, pre-permuted: [nt][step][lane] -> (b0, b1)
    __shared__ uint2 qfrag[NT][8][32];
    const int bh = blockIdx.y, b = bh / p.Hkv, kvh = bh - b * p.Hkv;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) {
        if (blockIdx.x == 0 && threadIdx.x == 0 && kvh == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    const int NQ = p.Q * p.G;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;

    // Step s of the 128-dim reduction uses, for thread quarter t, the pairs of
    // 16-byte piece c = t + 4*(s/2), half (s%2): words 4c+2(s%2) and +1.
    const uint32_t *qw = reinterpret_cast<const uint32_t *>(p.q);
    for (int e = threadIdx.x; e < NT * 8 * 32; e += blockDim.x) {
        const int nt = e / 256, s = (e / 32) % 8, ln = e % 32;
        const int n = nt * 8 + (ln >> 2), tq = ln & 3;
        const int c = tq + 4 * (s >> 1), w0 = 4 * c + 2 * (s & 1);
        uint2 v = make_uint2(0u, 0u);
        if (n < NQ) {
            const uint32_t *row = qw + global_row(p, b, kvh, n) * (kHeadDim / 2);
            v = make_uint2(row[w0], row[w0 + 1]);
        }
        qfrag[nt][s][ln] = v;
    }
    __syncthreads();

    const __nv_bfloat16 *kbase = reinterpret_cast<const __nv_bfloat16 *>(p.k) +
                                 (size_t)bh * p.L_max * kHeadDim;
    const float scale = p.scale;

    for (int chunk = blockIdx.x; chunk * kChunkKeys < seq_len; chunk += gridDim.x) {
        const int kb0 = chunk * kChunkKeys + warp * 32;  // this warp's two 16-key tiles
        uint4 A[2][2][4];                                // [tile][row half][piece]
#pragma unroll
        for (int mt = 0; mt < 2; mt++) {
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
                const int key = kb0 + mt * 16 + hf * 8 + g;
                const bool ok = key < seq_len;
                const __nv_bfloat16 *row = kbase + (size_t)key * kHeadDim;
#pragma unroll
                for (int j = 0; j < 4; j++)
                    A[mt][hf][j] = ok ? ldg_nc_v4(row + 8 * (t + 4 * j)) : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        float acc[2][NT][4];
#pragma unroll
        for (int mt = 0; mt < 2; mt++)
#pragma unroll
            for (int nt = 0; nt < NT; nt++)
#pragma unroll
                for (int i = 0; i < 4; i++) acc[mt][nt][i] = 0.f;
#pragma unroll
        for (int s = 0; s < 8; s++) {
            const int j = s >> 1;
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
                const uint2 bf = qfrag[nt][s][lane];
#pragma unroll
                for (int mt = 0; mt < 2; mt++) {
                    const uint4 &lo = A[mt][0][j], &hi = A[mt][1][j];
                    if (s & 1)
                        mma_bf16_16816(acc[mt][nt], lo.z, hi.z, lo.w, hi.w, bf.x, bf.y);
                    else
                        mma_bf16_16816(acc[mt][nt], lo.x, hi.x, lo.y, hi.y, bf.x, bf.y);
                }
            }
        }
        // C layout: acc[i] -> key g (+8 for i >= 2), query row 2t + (i & 1).
#pragma unroll
        for (int mt = 0; mt < 2; mt++) {
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int key = kb0 + mt * 16 + g + ((i & 2) ? 8 : 0);
                    const int r = nt * 8 + 2 * t + (i & 1);
                    if (r < NQ && key < seq_len)
                        p.scores[global_row(p, b, kvh, r) * p.ld + key] = acc[mt][nt][i] * scale;
                }
            }
        }
    }
}

// CUDA-core scorer for any dtype and any number of query rows per kv-head.
template <typename T>
__global__ void __launch_bounds__(128) score_generic(ScoreParams p) {
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    extern __shared__ float qs[];  // [NQ][128] fp32
    const int bh = blockIdx.y, b = bh / p.Hkv, kvh = bh - b * p.Hkv;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) {
        if (blockIdx.x == 0 && threadIdx.x == 0 && kvh == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    const int NQ = p.Q * p.G;
    for (int e = threadIdx.x; e < NQ * kHeadDim; e += blockDim.x) {
        const int r = e / kHeadDim, c = e - r * kHeadDim;
        const T *qrow = reinterpret_cast<const T *>(p.q) + global_row(p, b, kvh, r) * kHeadDim;
        if constexpr (sizeof(T) == 4)
            qs[e] = reinterpret_cast<const float *>(qrow)[c];
        else
            qs[e] = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(qrow)[c]);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    constexpr int kPer = 16 / sizeof(T);          // elements per 16-byte piece
    constexpr int kPieces = kHeadDim / kPer / 4;  // pieces per lane
    const T *kbase = reinterpret_cast<const T *>(p.k) + (size_t)bh * p.L_max * kHeadDim;
    for (int chunk = blockIdx.x; chunk * kChunkKeys < seq_len; chunk += gridDim.x) {
        for (int kb = chunk * kChunkKeys + warp * 8; kb < (chunk + 1) * kChunkKeys; kb += 32) {
            const int key = kb + g;
            const bool ok = key < seq_len;
            const T *krow = p.pages.table == nullptr || !ok
                                ? kbase + (size_t)key * kHeadDim
                                : reinterpret_cast<const T *>(p.k) +
                                      (size_t)paged_row(p.pages, p.status, p.Hkv, b, kvh, key) * kHeadDim;
            float kv[kPieces][kPer];
#pragma unroll
            for (int j = 0; j < kPieces; j++) {
                const uint4 v = ok ? *reinterpret_cast<const uint4 *>(krow + kPer * (t + 4 * j))
                                   : make_uint4(0u, 0u, 0u, 0u);
                if constexpr (sizeof(T) == 4) {
                    kv[j][0] = __uint_as_float(v.x);
                    kv[j][1] = __uint_as_float(v.y);
                    kv[j][2] = __uint_as_float(v.z);
                    kv[j][3] = __uint_as_float(v.w);
                } else {
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        kv[j][2 * e] = bf16lo_to_f32(w[e]);
                        kv[j][2 * e + 1] = bf16hi_to_f32(w[e]);
                    }
                }
            }
            for (int r = 0; r < NQ; r++) {
                const float *qr = qs + r * kHeadDim;
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < kPieces; j++)
#pragma unroll
                    for (int e = 0; e < kPer; e++) acc = fmaf(qr[kPer * (t + 4 * j) + e], kv[j][e], acc);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                if (t == 0 && ok) p.scores[global_row(p, b, kvh, r) * p.ld + key] = acc * p.scale;
            }
        }
    }
}

}  // namespace

cudaError_t launch_score(const ScoreParams &p, int num_sms, cudaStream_t stream) {
    const int NQ = p.Q * p.G;
    const int chunks = (p.L_max + kChunkKeys - 1) / kChunkKeys;
    const int units = p.B * p.Hkv;
    // enough CTAs for ~8 resident per SM; each walks its chunks grid-stride
    int gx = (num_sms * 8 + units - 1) / units;
    if (gx > chunks) gx = chunks;
    if (gx < 1) gx = 1;
    const dim3 grid(gx, units);
    if (p.dtype == TKA_BF16 && NQ <= 64 && p.pages.table == nullptr) {  // paged caches take score_generic
        if (NQ <= 8) return launch_k(true, score_bf16_mma<1>, grid, dim3(128), 0, stream, p);
        if (NQ <= 16) return launch_k(true, score_bf16_mma<2>, grid, dim3(128), 0, stream, p);
        if (NQ <= 32) return launch_k(true, score_bf16_mma<4>, grid, dim3(128), 0, stream, p);
        return launch_k(true, score_bf16_mma<8>, grid, dim3(128), 0, stream, p);
    }
    const size_t smem = (size_t)NQ * kHeadDim * sizeof(float);
    if (p.dtype == TKA_BF16) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(score_generic<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        return launch_k(true, score_generic<__nv_bfloat16>, grid, dim3(128), smem, stream, p);
    }
    if (smem > 48 * 1024)
        cudaFuncSetAttribute(score_generic<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch_k(true, score_generic<float>, grid, dim3(128), smem, stream, p);
}

}  // namespace tka
