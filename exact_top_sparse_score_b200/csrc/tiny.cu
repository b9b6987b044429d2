// Small decode problems in one launch.
//
// For a cache of at most a few ten thousand keys the three steps of the
// decode (score, select, attention over the kept keys; "Sparse Attention in
// LLM Inference: Practical Trade-Offs", sections "The Role of the Indexer" and
// "Changes in Caching Strategy") each take a few microseconds of work but a
// kernel launch and a grid-wide wait each.  Here one cooperative grid does all
// three: every CTA scores a share of the keys on the CUDA cores (a quad of
// lanes per key, the kv-head's query rows in shared memory), the grid meets at
// one grid-wide barrier, and then CTA r takes query row r: the select step of
// select_device.cuh on the row's scores, then the softmax-weighted sum of the
// kept V rows (out = sum_S e^{s - m} V / Z_k).  The results are those of the
// three-kernel path up to the scores' fp32 rounding.
#include <cooperative_groups.h>

#include "select_device.cuh"

namespace tka {

namespace {

constexpr int kTinyThreads = 512;
constexpr int kTinyChunk = 128;  // keys per CTA per step of the scoring phase

template <typename T>
__global__ void __launch_bounds__(kTinyThreads, 1) decode_tiny(TinyParams p) {
    namespace cg = cooperative_groups;
    extern __shared__ __align__(16) uint32_t dyn[];
    const SelectParams &sp = p.sel;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kTinyThreads / 32;
    const int NQ = sp.Q * p.G;

    // ---- scores: CTA c < B*Hkv*cpb takes kv-head c / cpb and its chunks
    // c % cpb, c % cpb + cpb, ... of kTinyChunk keys
    const int units = sp.B * p.Hkv;
    if ((int)blockIdx.x < units * p.cpb) {
        const int bh = blockIdx.x / p.cpb, part = blockIdx.x % p.cpb, b = bh / p.Hkv, kvh = bh - b * p.Hkv;
        const int seq_len = sp.seq_lens[b];
        if (seq_len_ok(seq_len, sp.Q, sp.L_max)) {
            float *qs = reinterpret_cast<float *>(dyn);  // [NQ][128]
            for (int e = threadIdx.x; e < NQ * kHeadDim; e += kTinyThreads) {
                const int r = e / kHeadDim, c = e - r * kHeadDim;
                const int qpos = r / p.G, gi = r - qpos * p.G;
                const size_t qrow = ((size_t)b * sp.Q + qpos) * sp.Hq + (size_t)kvh * p.G + gi;
                const T *qr = reinterpret_cast<const T *>(p.q) + qrow * kHeadDim;
                if constexpr (sizeof(T) == 4)
                    qs[e] = reinterpret_cast<const float *>(qr)[c];
                else
                    qs[e] = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(qr)[c]);
            }
            __syncthreads();
            const int g = lane >> 2, t = lane & 3;        // 8 keys per warp, a quad of lanes per key
            constexpr int kPer = 16 / sizeof(T);          // elements per 16-byte piece
            constexpr int kPieces = kHeadDim / kPer / 4;  // pieces per lane
            const T *kbase = reinterpret_cast<const T *>(p.k) + (size_t)bh * sp.L_max * kHeadDim;
            for (int c0 = part * kTinyChunk; c0 < seq_len; c0 += p.cpb * kTinyChunk) {
                for (int kb = c0 + warp * 8; kb < c0 + kTinyChunk; kb += kWarps * 8) {
                    const int key = kb + g;
                    const bool ok = key < seq_len;
                    const T *krow = kbase + (size_t)(ok ? key : 0) * kHeadDim;
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
                        const int qpos = r / p.G, gi = r - qpos * p.G;
                        // keys a causal query position cannot see are not stored
                        if (t == 0 && ok && key < visible_keys(seq_len, sp.Q, qpos)) {
                            const size_t row = ((size_t)b * sp.Q + qpos) * sp.Hq + (size_t)kvh * p.G + gi;
                            p.scores[row * sp.ld + key] = acc * p.scale;
                        }
                    }
                }
            }
        }
    }
    __threadfence();
    cg::this_grid().sync();  // every score is written

    // ---- per row: select, then the weighted sum of the kept V rows
    constexpr int kLanesPerRow = sizeof(T) == 2 ? 16 : 32;  // 16-byte pieces per V row
    constexpr int kElems = 16 / sizeof(T);
    constexpr int kGroups = kTinyThreads / kLanesPerRow;
    const int rows = sp.B * sp.Q * sp.Hq;
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
        __syncthreads();  // the scoring phase's (or the previous row's) shared memory is free
        select_row<kTinyThreads>(sp, row);
        __syncthreads();  // idx, weights and statistics of the row are written
        const int b = row / (sp.Q * sp.Hq), qpos = (row / sp.Hq) % sp.Q, h = row % sp.Hq;
        const int seq_len = sp.seq_lens[b];
        if (!seq_len_ok(seq_len, sp.Q, sp.L_max)) continue;  // the select step raised the status
        const int kept = min(sp.k, visible_keys(seq_len, sp.Q, qpos));
        const int grp = threadIdx.x / kLanesPerRow, c = threadIdx.x % kLanesPerRow;
        const T *vb =
            reinterpret_cast<const T *>(p.v) + ((size_t)b * p.Hkv + h / p.G) * sp.L_max * kHeadDim + c * kElems;
        const int32_t *ix = sp.idx + (size_t)row * sp.k;
        const float *wv = sp.w + (size_t)row * sp.k;
        float acc[kElems];
#pragma unroll
        for (int e = 0; e < kElems; e++) acc[e] = 0.f;
        bool bad = false;
        for (int j = grp; j < kept; j += kGroups) {
            int pos = __ldcg(ix + j);
            float wt = __ldcg(wv + j);
            if ((unsigned)pos >= (unsigned)seq_len) {  // never true unless the select step is wrong
                bad = true;
                pos = 0;
                wt = 0.f;
            }
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(vb + (size_t)pos * kHeadDim));
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
            if constexpr (sizeof(T) == 2) {
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    acc[2 * e] = fmaf(wt, bf16lo_to_f32(vw[e]), acc[2 * e]);
                    acc[2 * e + 1] = fmaf(wt, bf16hi_to_f32(vw[e]), acc[2 * e + 1]);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 4; e++) acc[e] = fmaf(wt, __uint_as_float(vw[e]), acc[e]);
            }
        }
        if (bad) raise_status(sp.status, TKA_DEV_INTERNAL);
        float *red = reinterpret_cast<float *>(dyn);  // [kGroups][128]: the select's shared memory is free now
        __syncthreads();
#pragma unroll
        for (int e = 0; e < kElems; e++) red[grp * kHeadDim + c * kElems + e] = acc[e];
        __syncthreads();
        if (threadIdx.x < kHeadDim) {
            float sum = 0.f;
            for (int gq = 0; gq < kGroups; gq++) sum += red[gq * kHeadDim + threadIdx.x];
            p.out[(size_t)row * kHeadDim + threadIdx.x] = sum / __ldcg(&sp.stats[row].y);
        }
    }
}

}  // namespace

size_t tiny_smem_bytes(int NQ, int k) {
    const size_t sel = select_smem_bytes(kTinyThreads, k);
    const size_t qs = (size_t)NQ * kHeadDim * sizeof(float);
    const size_t red = (size_t)kTinyThreads / 16 * kHeadDim * sizeof(float);
    size_t m = sel > qs ? sel : qs;
    return m > red ? m : red;
}

cudaError_t launch_tiny(const TinyParams &p, int grid, cudaStream_t stream) {
    const size_t smem = tiny_smem_bytes(p.sel.Q * p.G, p.sel.k);
    void (*kernel)(TinyParams) = p.dtype == TKA_BF16 ? decode_tiny<__nv_bfloat16> : decode_tiny<float>;
    // per device and dtype: the largest size any call takes, set once
    static std::atomic<bool> attr_set[64][2] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int di = p.dtype == TKA_BF16 ? 1 : 0;
    if (dev < 0 || dev >= 64 || !attr_set[dev][di].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tiny_smem_bytes(64, kMaxK));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev][di].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kTinyThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

}  // namespace tka
