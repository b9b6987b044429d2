// Token selection by a lightning indexer, then exact attention over the kept
// tokens ("Sparse Attention Landscape", section "Token Sparse Attention":
// DeepSeek Sparse Attention's indexer scores every previous token with a few
// small heads, I_i = sum_j w_j ReLU(<q_idx_j, k_idx_i>), keeps the top k and
// runs the full attention over that subset).  The selection belongs to the
// query position and is shared by all its attention heads.
//
// Kernels:
//   indexer_scores  grid (key chunks, b): a quad of lanes per index key, each
//                   lane a quarter of the dims; every (query position, indexer
//                   head) dot is reduced in the quad, ReLU'd, weighted and
//                   summed; one score per (query position, key).  With bf16
//                   128-dim index keys the dots run on the tensor cores instead
//                   (the score kernel with the indexer heads as query rows of
//                   one kv-head) and indexer_combine forms the weighted sum.
//   (the select step keeps the top k per query position)
//   indexer_attn    grid (splits, b * Q * Hkv): a slice of the kept tokens for
//                   the G heads of one kv-head; every K and V row is read once
//                   for all G heads; per head an online softmax in each warp,
//                   warps and then slices merged in order (last CTA, ticket).
#include "common.cuh"
#include "kernels.h"

namespace tka {

namespace {

constexpr int kIdxChunk = 128;  // index keys per CTA iteration

template <typename T, int DI>
__global__ void __launch_bounds__(128) indexer_scores(IndexerScoreParams p) {
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    extern __shared__ float smem[];
    const int NQ = p.Q * p.H_I;
    float *qs = smem;                 // [NQ][DI]
    float *ws = smem + NQ * DI;       // [NQ]
    const int b = blockIdx.y;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    if (blockIdx.x == 0)  // the attention step's tickets for this sequence's units
        for (int u = threadIdx.x; u < p.Q * p.Hkv; u += blockDim.x) p.attn_counters[(size_t)b * p.Q * p.Hkv + u] = 0u;
    const T *qb = reinterpret_cast<const T *>(p.q_idx) + (size_t)b * NQ * DI;
    for (int e = threadIdx.x; e < NQ * DI; e += blockDim.x) {
        if constexpr (sizeof(T) == 4)
            qs[e] = reinterpret_cast<const float *>(qb)[e];
        else
            qs[e] = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(qb)[e]);
    }
    for (int e = threadIdx.x; e < NQ; e += blockDim.x) ws[e] = p.w_idx[(size_t)b * NQ + e];
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    constexpr int kPer = 16 / sizeof(T);         // elements per 16-byte piece
    constexpr int kPieces = DI / kPer / 4;       // pieces per lane
    const T *kbase = reinterpret_cast<const T *>(p.k_idx) + (size_t)b * p.L_max * DI;
    for (int chunk = blockIdx.x; chunk * kIdxChunk < seq_len; chunk += gridDim.x) {
        for (int kb = chunk * kIdxChunk + warp * 8; kb < (chunk + 1) * kIdxChunk; kb += 32) {
            const int key = kb + g;
            const bool ok = key < seq_len;
            float kv[kPieces][kPer];
#pragma unroll
            for (int j = 0; j < kPieces; j++) {
                const uint4 v = ok ? *reinterpret_cast<const uint4 *>(kbase + (size_t)key * DI + kPer * (t + 4 * j))
                                   : make_uint4(0u, 0u, 0u, 0u);
                if constexpr (sizeof(T) == 4) {
                    kv[j][0] = __uint_as_float(v.x);
                    kv[j][1] = __uint_as_float(v.y);
                    kv[j][2] = __uint_as_float(v.z);
                    kv[j][3] = __uint_as_float(v.w);
                } else {
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        kv[j][2 * e] = bf16lo_to_f32(w4[e]);
                        kv[j][2 * e + 1] = bf16hi_to_f32(w4[e]);
                    }
                }
            }
            for (int qp = 0; qp < p.Q; qp++) {
                float I = 0.f;
                for (int j = 0; j < p.H_I; j++) {
                    const float *qr = qs + (qp * p.H_I + j) * DI;
                    float acc = 0.f;
#pragma unroll
                    for (int pc = 0; pc < kPieces; pc++)
#pragma unroll
                        for (int e = 0; e < kPer; e++) acc = fmaf(qr[kPer * (t + 4 * pc) + e], kv[pc][e], acc);
                    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                    I = fmaf(ws[qp * p.H_I + j], fmaxf(acc, 0.f), I);
                }
                if (t == 0 && key < visible_keys(seq_len, p.Q, qp))
                    p.scores[((size_t)b * p.Q + qp) * p.ld + key] = I;
            }
        }
    }
}

// I = sum_j w_j ReLU(raw_j) from the raw per-head dots the tensor-core scorer
// wrote ([B*Q*H_I, ld], head-minor rows): grid (key chunks of 256, b * Q).
__global__ void __launch_bounds__(256) indexer_combine(IndexerScoreParams p, const float *raw) {
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    __shared__ float ws[256];
    const int bq = blockIdx.y, b = bq / p.Q, qpos = bq - b * p.Q;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    if (blockIdx.x == 0 && qpos == 0)  // the attention step's tickets for this sequence's units
        for (int u = threadIdx.x; u < p.Q * p.Hkv; u += blockDim.x) p.attn_counters[(size_t)b * p.Q * p.Hkv + u] = 0u;
    for (int j = threadIdx.x; j < p.H_I; j += blockDim.x) ws[j] = p.w_idx[(size_t)bq * p.H_I + j];
    __syncthreads();
    const int key = blockIdx.x * 256 + threadIdx.x;
    if (key >= visible_keys(seq_len, p.Q, qpos)) return;
    const float *r = raw + (size_t)bq * p.H_I * p.ld + key;
    float I = 0.f;
    for (int j = 0; j < p.H_I; j++) I = fmaf(ws[j], fmaxf(__ldcg(r + (size_t)j * p.ld), 0.f), I);
    p.scores[(size_t)bq * p.ld + key] = I;
}

constexpr int kAttnWarps = 4;
constexpr int kMaxG = 16;  // heads per kv-head held in registers (G <= kMaxG)

template <typename T, int GG>
__global__ void __launch_bounds__(kAttnWarps * 32) indexer_attn(IndexerAttnParams p) {
    pdl_wait();  // inputs may come from the kernel before
    pdl_trigger();
    __shared__ float sm_ml[kAttnWarps][GG][2];
    __shared__ float sm_acc[kAttnWarps][GG][kHeadDim];
    __shared__ unsigned s_ticket;
    const int unit = blockIdx.y;  // (b, qpos, kvh)
    const int kvh = unit % p.Hkv, bq = unit / p.Hkv, qpos = bq % p.Q, b = bq / p.Q;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) return;  // the indexer step raised the status
    const int vis = visible_keys(seq_len, p.Q, qpos);
    const int kept = min(p.k, vis);
    const int lo = blockIdx.x * p.per_split, hi = min(kept, lo + p.per_split);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // this lane's 4 dims of each of the G query rows
    float4 qv[GG];
#pragma unroll
    for (int h = 0; h < GG; h++) {
        const T *qr = reinterpret_cast<const T *>(p.q) + (((size_t)bq * p.Hq) + (size_t)kvh * GG + h) * kHeadDim + 4 * lane;
        if constexpr (sizeof(T) == 4) {
            qv[h] = *reinterpret_cast<const float4 *>(qr);
        } else {
            const uint2 w2 = *reinterpret_cast<const uint2 *>(qr);
            qv[h] = make_float4(bf16lo_to_f32(w2.x), bf16hi_to_f32(w2.x), bf16lo_to_f32(w2.y), bf16hi_to_f32(w2.y));
        }
    }
    float m[GG], l[GG];
    float4 acc[GG];
#pragma unroll
    for (int h = 0; h < GG; h++) {
        m[h] = -INFINITY;
        l[h] = 0.f;
        acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const size_t kvoff = ((size_t)b * p.Hkv + kvh) * p.L_max * kHeadDim + 4 * lane;
    const int32_t *ir = p.idx + (size_t)bq * p.k;
    bool bad = false;
    for (int i = lo + warp; i < hi; i += kAttnWarps) {
        int pos = __ldg(ir + i);
        if ((unsigned)pos >= (unsigned)vis) {  // never true unless the select step is wrong
            bad = true;
            continue;
        }
        float4 kf, vf;
        if constexpr (sizeof(T) == 4) {
            kf = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(p.kc) + kvoff + (size_t)pos * kHeadDim);
            vf = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(p.vc) + kvoff + (size_t)pos * kHeadDim);
        } else {
            const uint2 k2 = *reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(p.kc) + kvoff +
                                                              (size_t)pos * kHeadDim);
            const uint2 v2 = *reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(p.vc) + kvoff +
                                                              (size_t)pos * kHeadDim);
            kf = make_float4(bf16lo_to_f32(k2.x), bf16hi_to_f32(k2.x), bf16lo_to_f32(k2.y), bf16hi_to_f32(k2.y));
            vf = make_float4(bf16lo_to_f32(v2.x), bf16hi_to_f32(v2.x), bf16lo_to_f32(v2.y), bf16hi_to_f32(v2.y));
        }
#pragma unroll
        for (int h = 0; h < GG; h++) {
            float s = qv[h].x * kf.x + qv[h].y * kf.y + qv[h].z * kf.z + qv[h].w * kf.w;
            s = warp_sum(s) * p.scale;
            const float m_new = fmaxf(m[h], s);
            const float f = __expf(m[h] - m_new), e = __expf(s - m_new);
            m[h] = m_new;
            l[h] = l[h] * f + e;
            acc[h].x = fmaf(e, vf.x, acc[h].x * f);
            acc[h].y = fmaf(e, vf.y, acc[h].y * f);
            acc[h].z = fmaf(e, vf.z, acc[h].z * f);
            acc[h].w = fmaf(e, vf.w, acc[h].w * f);
        }
    }
    if (bad) raise_status(p.status, TKA_DEV_INTERNAL);
    // merge the warps (slot order), one head per pass over the shared arrays
#pragma unroll
    for (int h = 0; h < GG; h++) {
        if (lane == 0) {
            sm_ml[warp][h][0] = m[h];
            sm_ml[warp][h][1] = l[h];
        }
        reinterpret_cast<float4 *>(sm_acc[warp][h])[lane] = acc[h];
    }
    __syncthreads();
    const size_t row0 = (size_t)bq * p.Hq + (size_t)kvh * GG;  // first of the G output rows
    for (int e = threadIdx.x; e < GG * kHeadDim; e += blockDim.x) {
        const int h = e / kHeadDim, d = e - h * kHeadDim;
        float M = -INFINITY;
        for (int wv = 0; wv < kAttnWarps; wv++) M = fmaxf(M, sm_ml[wv][h][0]);
        float L = 0.f, A = 0.f;
        for (int wv = 0; wv < kAttnWarps; wv++) {
            if (sm_ml[wv][h][1] == 0.f) continue;
            const float f = __expf(sm_ml[wv][h][0] - M);
            L += sm_ml[wv][h][1] * f;
            A += sm_acc[wv][h][d] * f;
        }
        const size_t ps = (row0 + h) * p.splits + blockIdx.x;
        if (d == 0) p.part_ml[ps] = make_float4(M, L, 0.f, 0.f);
        p.part_acc[ps * kHeadDim + d] = A;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(&p.counters[unit], 1u);
    __syncthreads();
    if (s_ticket != (unsigned)p.splits - 1) return;
    __threadfence();
    for (int e = threadIdx.x; e < GG * kHeadDim; e += blockDim.x) {
        const int h = e / kHeadDim, d = e - h * kHeadDim;
        const size_t pr = (row0 + h) * p.splits;
        float M = -INFINITY;
        for (int sp = 0; sp < p.splits; sp++) M = fmaxf(M, __ldcg(&p.part_ml[pr + sp].x));
        float L = 0.f, A = 0.f;
        for (int sp = 0; sp < p.splits; sp++) {
            const float4 ml = __ldcg(&p.part_ml[pr + sp]);
            if (ml.y == 0.f) continue;
            const float f = __expf(ml.x - M);
            L += ml.y * f;
            A += __ldcg(&p.part_acc[(pr + sp) * kHeadDim + d]) * f;
        }
        p.out[(row0 + h) * kHeadDim + d] = A / L;
    }
    if (threadIdx.x == 0) p.counters[unit] = 0u;
}

template <int DI>
cudaError_t launch_scores_di(const IndexerScoreParams &p, int num_sms, cudaStream_t stream) {
    const size_t smem = (size_t)p.Q * p.H_I * (DI + 1) * sizeof(float);
    const int chunks = (p.L_max + kIdxChunk - 1) / kIdxChunk;
    int gx = (num_sms * 8 + p.B - 1) / p.B;
    gx = max(1, min(gx, chunks));
    const dim3 grid(gx, p.B);
    cudaError_t e;
    if (p.dtype == TKA_BF16) {
        if (smem > 48 * 1024 && (e = cudaFuncSetAttribute(indexer_scores<__nv_bfloat16, DI>,
                                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        return launch_k(true, indexer_scores<__nv_bfloat16, DI>, grid, dim3(128), smem, stream, p);
    } else {
        if (smem > 48 * 1024 && (e = cudaFuncSetAttribute(indexer_scores<float, DI>,
                                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        return launch_k(true, indexer_scores<float, DI>, grid, dim3(128), smem, stream, p);
    }
}

template <int GG>
cudaError_t launch_attn_g(const IndexerAttnParams &p, cudaStream_t stream) {
    const dim3 grid(p.splits, p.B * p.Q * p.Hkv);
    if (p.dtype == TKA_BF16)
        return launch_k(true, indexer_attn<__nv_bfloat16, GG>, grid, dim3(kAttnWarps * 32), 0, stream, p);
    return launch_k(true, indexer_attn<float, GG>, grid, dim3(kAttnWarps * 32), 0, stream, p);
}

}  // namespace

bool indexer_supported(int G, int d_I) { return (d_I == 64 || d_I == 128) && (G == 1 || G == 2 || G == 4 || G == 8 || G == 16); }

cudaError_t launch_indexer_scores(const IndexerScoreParams &p, int num_sms, cudaStream_t stream) {
    return p.d_I == 64 ? launch_scores_di<64>(p, num_sms, stream) : launch_scores_di<128>(p, num_sms, stream);
}

cudaError_t launch_indexer_combine(const IndexerScoreParams &p, const float *raw, cudaStream_t stream) {
    const dim3 grid((p.L_max + 255) / 256, p.B * p.Q);
    return launch_k(true, indexer_combine, grid, dim3(256), 0, stream, p, raw);
}

cudaError_t launch_indexer_attn(const IndexerAttnParams &p, cudaStream_t stream) {
    switch (p.G) {
    case 1: return launch_attn_g<1>(p, stream);
    case 2: return launch_attn_g<2>(p, stream);
    case 4: return launch_attn_g<4>(p, stream);
    case 8: return launch_attn_g<8>(p, stream);
    default: return launch_attn_g<kMaxG>(p, stream);
    }
}

}  // namespace tka
