// Launch interfaces of the Top-k decode-attention kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace tka {

constexpr int kMaxK = 8192;  // largest k (and k_max) the select and certify steps take

struct ScoreParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const void *q;            // [B, Q, Hq, 128]
    const void *k;            // [B, Hkv, L_max, 128], or the paged cache
    const int32_t *seq_lens;  // [B]
    float *scores;            // [B*Q*Hq, ld]
    int B, Q, Hq, Hkv, G, L_max, ld, dtype;
    float scale;
    PageTable pages;
};

struct ScoreTcParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const int32_t *seq_lens;  // [B]
    float *scores;            // [B*Q*Hq, ld]
    int B, Q, Hq, Hkv, G, L_max, ld, NQ;
    float scale;
    PageTable pages;          // paged cache: the K tensor map covers [num_pages*Hkv*page, 128]
    uint32_t max_polls = 0;   // polls before a pipeline wait gives up (0: the default bound)
};

struct SelectParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const float *scores;      // [rows, ld]
    const int32_t *seq_lens;
    int B, Q, Hq, L_max, ld, k;
    int32_t *idx;             // [rows, k] ascending, -1 padded
    float *w;                 // [rows, k] e^{s_i - m} of the kept positions
    float4 *stats;            // [rows] {m, Z_k, Z_tail, 0}
    float *tail;              // [rows] or null
    unsigned *counters;       // [rows], zeroed here for the combine step
    const int32_t *row_len = nullptr;  // [rows] scores per row (compact candidate rows), or null:
                                       // the visible keys of the row
};

struct GatherParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const void *v;            // [B, Hkv, L_max, 128]
    const int32_t *seq_lens;
    int B, Q, Hq, Hkv, G, L_max, k, dtype;
    const int32_t *idx;       // [rows, k]
    const float *w;           // [rows, k]
    const float4 *stats;      // [rows]
    float *partial;           // [rows, splits, 128]
    unsigned *counters;       // [rows]
    float *out;               // [rows, 128]
    int splits, per_split;
    const int32_t *kcount;    // [rows] kept positions per row, or null: min(k, visible keys)
    PageTable pages;          // v is the paged cache when pages.table is set
    // Candidate rows (hierarchical selection): idx holds indices into a row of
    // candidates, slot-major over the kept blocks; position = cblock[row,
    // c / cbs] * cbs + c % cbs.  The gather writes the positions back to idx.
    const int32_t *cblock = nullptr;  // [rows, cstride]
    const int32_t *crow_len = nullptr;  // [rows] valid candidates
    int32_t *idx_out = nullptr;         // [rows, k] the same buffer as idx
    int cbs = 0, cstride = 0;
};

struct HisaScoreParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const void *q, *k;        // q [B, 1, Hq, 128], K [B, Hkv, L_max, 128]
    const int32_t *seq_lens;
    const int32_t *block_idx; // [rows, top_blocks] ascending, -1 padded
    int B, Hq, Hkv, G, L_max, block_size, top_blocks, ldc, dtype;
    float scale;
    float *cscore;            // [rows, ldc] candidate scores, slot-major
    int32_t *row_len;         // [rows] valid candidates (a prefix of the row)
};

struct CertifyParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const float *scores;      // [rows, ld]
    const int32_t *seq_lens;
    int B, Q, Hq, L_max, ld, k_max;
    float eps;
    int32_t *idx;             // [rows, k_max] in: the top k_max ascending; out: the certified prefix
    float *w;                 // [rows, k_max] e^{s - m}, compacted like idx
    float4 *stats;            // [rows] {m, Z_k, Z_tail, 0}, rewritten
    float *tail;              // [rows] or null
    int32_t *k_used;          // [rows]
};

struct IndexerScoreParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const void *q_idx;        // [B, Q, H_I, d_I] indexer queries
    const float *w_idx;       // [B, Q, H_I] indexer head weights
    const void *k_idx;        // [B, L_max, d_I] indexer keys
    const int32_t *seq_lens;
    int B, Q, Hkv, L_max, H_I, d_I, ld, dtype;
    float *scores;            // [B*Q, ld] indexer scores
    unsigned *attn_counters;  // [B*Q*Hkv], zeroed here for the attention step
};

struct IndexerAttnParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const void *q, *kc, *vc;  // q [B, Q, Hq, 128]; caches [B, Hkv, L_max, 128]
    const int32_t *seq_lens;
    const int32_t *idx;       // [B*Q, k] kept positions, ascending
    int B, Q, Hq, Hkv, G, L_max, k, dtype;
    float scale;
    float4 *part_ml;          // [B*Q*Hq, splits] {m, l}
    float *part_acc;          // [B*Q*Hq, splits, 128]
    unsigned *counters;       // [B*Q*Hkv]
    float *out;               // [B*Q*Hq, 128]
    int splits, per_split;
};

struct BlockPoolParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const void *k;
    const int32_t *seq_lens;
    float *block_keys;        // [B, Hkv, nblk_max, 128]
    int B, Hkv, L_max, block_size, nblk_max, dtype;
};

struct BlockSelectParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const void *q;            // [B, 1, Hq, 128]
    const float *block_keys;  // [B, Hkv, nblk_max, 128]
    const int32_t *seq_lens;
    int B, Hq, Hkv, G, L_max, block_size, nblk_max, top_blocks, dtype;
    float scale;
    float *bscore;            // [B*Hq, nblk_max] block scores of the competing blocks
    int32_t *block_idx;       // [B*Hq, top_blocks + force_last] (workspace or caller's)
    unsigned *counters;       // [B*Hq], zeroed here for the attention step (may be null)
    int force_last = 1;       // 1: the current block is always kept and does not compete (MoBA);
                              // 0: every block competes for the top_blocks slots
};

struct BlockAttnParams {
    unsigned *status;         // device status word (TKA_DEV_* bits)
    const void *q, *k, *v;
    const int32_t *seq_lens;
    const int32_t *block_idx; // [rows, top_blocks + 1]
    int B, Hq, Hkv, G, L_max, block_size, top_blocks, dtype;
    float scale;
    float4 *part_ml;          // [rows, top_blocks + 1] {m, l} per piece of a row
    float *part_acc;          // [rows, top_blocks + 1, 128]
    unsigned *counters;       // [rows]
    float *out;               // [rows, 128]
    int stages;               // set by the launcher
    uint32_t stage_bytes;
    uint32_t max_polls = 0;   // polls before a pipeline wait gives up (0: the default bound)
};

// The one-launch decode of a small problem (tiny.cu): the select step's
// parameters (scores, idx, w, stats, tail, counters, shape and k) plus what
// scoring and the attention step need.
struct TinyParams {
    SelectParams sel;
    float *scores;            // the same buffer as sel.scores, written by the scoring phase
    const void *q, *k, *v;    // q [B, Q, Hq, 128]; caches [B, Hkv, L_max, 128]
    int Hkv, G, dtype;
    float scale;
    float *out;               // [B*Q*Hq, 128]
    int cpb;                  // CTAs scoring each kv-head
};

// Launches kernel<<<grid, block, smem, stream>>>(args...), allowed to start
// early behind the previous kernel on the stream when pdl is set (the kernel
// calls pdl_wait() before reading earlier results).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                     Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// cuTensorMapEncodeTiled, fetched from the driver once (null if unavailable).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();

cudaError_t launch_score(const ScoreParams &p, int num_sms, cudaStream_t stream);
bool score_tc_supported(int dtype, int NQ);
// Called right before a kernel launch, after all host-side preparation
// (tensor-map encoding, function attributes); a null fn is skipped.
struct ScoreTcHook {
    cudaError_t (*fn)(void *ctx) = nullptr;
    void *ctx = nullptr;
};
cudaError_t launch_score_tc(const ScoreTcParams &p, const void *q, const void *k_cache, int num_sms,
                            cudaStream_t stream, const ScoreTcHook &hook, bool pdl = false);
// threads: 1024 (one row per SM) or 512 (two rows per SM)
cudaError_t launch_select(const SelectParams &p, cudaStream_t stream, int threads = 1024, bool pdl = false);
size_t select_smem_bytes(int threads, int k);
cudaError_t launch_gather(const GatherParams &p, cudaStream_t stream, bool pdl = false);
cudaError_t launch_certify(const CertifyParams &p, cudaStream_t stream, bool pdl = false);
size_t tiny_smem_bytes(int NQ, int k);
// One cooperative grid of `grid` CTAs (all resident at once)
cudaError_t launch_tiny(const TinyParams &p, int grid, cudaStream_t stream);
bool indexer_supported(int G, int d_I);
cudaError_t launch_indexer_scores(const IndexerScoreParams &p, int num_sms, cudaStream_t stream);
cudaError_t launch_indexer_attn(const IndexerAttnParams &p, cudaStream_t stream);
cudaError_t launch_indexer_combine(const IndexerScoreParams &p, const float *raw, cudaStream_t stream);
cudaError_t launch_block_pool(const BlockPoolParams &p, cudaStream_t stream);
cudaError_t launch_block_select(const BlockSelectParams &p, cudaStream_t stream);
cudaError_t launch_hisa_scores(const HisaScoreParams &p, cudaStream_t stream);
cudaError_t launch_block_attn(const BlockAttnParams &p, const void *k_cache, int num_sms, cudaStream_t stream);

}  // namespace tka
