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
// score_generic runs on CUDA cores, for fp32 caches and for bf16 caches the
// tensor-core kernel (score_tc.cu) does not take: a quad of lanes per key,
// each lane a quarter of the head dims, quad shuffles to sum.
#include "common.cuh"
#include "kernels.h"

namespace tka {

namespace {

constexpr int kChunkKeys = 128;  // keys per CTA iteration (4 warps x 32)

// Global row index of query row r (0 <= r < Q*G) of kv-head kvh in batch b.
__device__ __forceinline__ size_t global_row(const ScoreParams &p, int b, int kvh, int r) {
    const int qpos = r / p.G, gi = r - qpos * p.G;
    return ((size_t)b * p.Q + qpos) * p.Hq + (size_t)kvh * p.G + gi;
}

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
