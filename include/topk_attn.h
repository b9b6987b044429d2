/*
 * topk_attn.h -- C ABI of the B200 exact Top-k sparse decode-attention library.
 *
 * The operation ("A Preliminary Study on the Promises and Challenges of Native
 * Top-k Sparse Attention", abstract: exact Top-k decoding keeps only the keys
 * most similar to the query; "Sparse Attention in LLM Inference: Practical
 * Trade-Offs", section "The Role of the Indexer": score every historical
 * position, keep the Top-K, attend only to those):
 *
 *   for every query row (b, qpos, h), with G = Hq / Hkv and kv-head h / G,
 *     vis   = seq_lens[b] - Q + qpos + 1                   (causal visibility)
 *     s_i   = scale * <q[b,qpos,h,:], K[b,h/G,i,:]>        for i < vis
 *     S     = the min(k, vis) positions with the highest s_i, ties to the lower i
 *     out   = sum_{i in S} softmax_S(s)_i * V[b,h/G,i,:]
 *     tail  = sum_{i not in S} softmax(s)_i                (discarded softmax mass;
 *             "A Mathematical Theory of Top-k Sparse Attention via Total
 *             Variation Distance", abstract: equals TV(P, P_hat))
 *
 * and a block-sparse variant (MoBA, "Sparse Attention Landscape", section
 * "Block Sparse Attention"): blocks of `block_size` keys are scored by
 * <q, mean of the block's keys>, the best `top_blocks` blocks other than the
 * last are kept together with the last (current) block, and dense softmax
 * attention runs over the kept blocks' keys.
 *
 * Conventions shared by every entry point:
 *   - Every data pointer is DEVICE memory owned by the caller.  The library
 *     never allocates, frees or synchronises inside a compute call; it only
 *     enqueues kernels on `stream` (a cudaStream_t; NULL = legacy default).
 *     The kernels are launched with programmatic stream serialization (they
 *     may be scheduled while the kernel before them on the stream finishes)
 *     and wait for all earlier work on the stream before reading anything,
 *     so results are ordered exactly as with plain launches.  A caller that
 *     launches its own next kernel with that attribute must likewise wait
 *     (griddepcontrol.wait) before reading this library's outputs.
 *   - Layouts are row-major and contiguous:
 *       q         [B, Q, Hq, d]        dtype of the cache
 *       k_cache   [B, Hkv, L_max, d]   bf16 or fp32
 *       v_cache   [B, Hkv, L_max, d]   same dtype as k_cache
 *       seq_lens  int32 [B]            valid keys per sequence, Q <= seq_lens[b] <= L_max
 *       out       fp32 [B, Q, Hq, d]
 *       idx       int32 [B, Q, Hq, k]  kept positions, ascending, -1 padded when vis < k
 *       tail_mass fp32 [B, Q, Hq]
 *     q, k_cache, v_cache and out must be 16-byte aligned, the workspace
 *     256-byte aligned.
 *     Cache rows at positions >= seq_lens[b] never affect a result.  V rows
 *     there are never read; K rows are read in tiles of 128 positions, so the
 *     last tile below seq_lens[b] may read up to 127 rows past it (inside
 *     [0, L_max) of the same kv-head, or of the page pool for a paged cache),
 *     and those scores are discarded.
 *   - Arguments are checked on the host before anything is launched; a bad
 *     argument returns an error code and launches nothing.  seq_lens lives on
 *     the device, so its values are checked by the kernels: a sequence whose
 *     length is out of range is skipped (its outputs are left untouched) and
 *     TKA_DEV_BAD_SEQ_LEN is raised in the device status word, readable with
 *     topk_attn_device_status().
 *   - Supported: d = 128, dtype bf16 or fp32, Hq % Hkv == 0, 1 <= k <= 8192,
 *     Q <= 64.  Anything else returns TKA_ERR_UNSUPPORTED.
 */
#ifndef TOPK_ATTN_H
#define TOPK_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TKA_OK = 0,
    TKA_ERR_INVALID_ARG = 1, /* null pointer, misaligned pointer, non-positive size */
    TKA_ERR_UNSUPPORTED = 2, /* valid but outside the supported set above */
    TKA_ERR_WORKSPACE = 3,   /* workspace pointer missing or smaller than required */
    TKA_ERR_CUDA = 4,        /* a launch or CUDA runtime call failed */
    TKA_ERR_TIMEOUT = 5      /* topk_attn_last_device_status only: a bounded wait inside a kernel gave up */
} tka_status;

typedef enum { TKA_F32 = 0, TKA_BF16 = 1 } tka_dtype;

/* Bits of the device status word (OR-ed by kernels, cleared by reading). */
#define TKA_DEV_BAD_SEQ_LEN 0x1u /* a seq_lens value was out of range; that sequence was skipped */
#define TKA_DEV_INTERNAL 0x2u    /* an internal consistency check failed (a library bug) */
#define TKA_DEV_TIMEOUT 0x4u     /* a bounded wait inside a kernel gave up; results are incomplete */
#define TKA_DEV_BAD_PAGE 0x8u    /* a block-table entry names no page of the paged cache */

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st *tka_stream_t;

typedef struct {
    int32_t B;      /* sequences */
    int32_t Q;      /* query positions per sequence (1 for plain decode) */
    int32_t Hq;     /* query heads */
    int32_t Hkv;    /* key/value heads; Hq % Hkv == 0 */
    int32_t d;      /* head dimension (128) */
    int32_t L_max;  /* cache capacity per sequence */
    int32_t dtype;  /* tka_dtype of q, k_cache and v_cache */
    float scale;    /* score scale; 0 means 1/sqrt(d) */
} tka_shape;

/* Bytes of scratch topk_attn_decode needs for this shape and k (0 on a bad
 * shape).  The caller allocates it once and may reuse it for every call with
 * the same or a smaller shape; calls sharing one workspace must not overlap. */
size_t topk_attn_workspace_size(const tka_shape *shape, int32_t k);

/* Exact Top-k decode attention for all B*Q*Hq query rows (see top of file).
 * idx is required; tail_mass may be NULL.  Three kernels (score, select,
 * attention over the kept rows); a small problem -- at most 65536 cache rows
 * in all (B*Hkv*L_max), no more query rows and kv-heads than the GPU has SMs,
 * at most 64 query rows per kv-head -- runs as one cooperative launch with the
 * same results up to the rounding of the fp32 scores. */
tka_status topk_attn_decode(const tka_shape *shape, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *seq_lens, int32_t k, float *out,
                            int32_t *idx, float *tail_mass, void *workspace, size_t workspace_bytes,
                            tka_stream_t stream);

/* Same as topk_attn_decode, and additionally records the caller's CUDA events
 * (cudaEvent_t, created by the caller) on `stream` around the three kernels:
 * events[0] before the score kernel, events[1] between score and select,
 * events[2] between select and gather (idx is final there: a caller may start
 * copying it out while the gather runs), events[3] after gather.  Any entry
 * may be null (not recorded).  Used to time each step, or to overlap the idx
 * read-back with the gather; a kernel that follows a recorded event does not
 * start early behind the kernel before it.  This call always runs the three
 * kernels (a small problem included), with the results topk_attn_decode gives
 * up to the rounding of the fp32 scores. */
typedef struct CUevent_st *tka_event_t;
tka_status topk_attn_decode_staged(const tka_shape *shape, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *seq_lens, int32_t k, float *out,
                                   int32_t *idx, float *tail_mass, void *workspace, size_t workspace_bytes,
                                   tka_stream_t stream, const tka_event_t events[4]);

/* topk_attn_decode over a paged KV cache ("Sparse Attention in LLM Inference:
 * Practical Trade-Offs", section "Changes in Caching Strategy": the selected
 * entries are read by index from the cache wherever they live).  The cache is
 * a pool of pages of page_size positions:
 *   k_pages, v_pages  [num_pages, Hkv, page_size, d] (cache dtype); each page
 *                     holds page_size consecutive positions of every kv-head.
 *   block_table       int32 [B, max_pages] device buffer: logical page j of
 *                     sequence b (positions j*page_size .. (j+1)*page_size - 1)
 *                     is physical page block_table[b * max_pages + j]; only
 *                     the entries below ceil(seq_lens[b] / page_size) are read.
 *   page_size         a power of two >= 16.
 *   shape->L_max      the logical capacity, at most max_pages * page_size.
 * Everything else (q, outputs, workspace = topk_attn_workspace_size(shape, k),
 * results) is as topk_attn_decode, which gives the same out, idx and tail on
 * the equivalent contiguous cache.  A table entry outside [0, num_pages)
 * raises TKA_DEV_BAD_PAGE (page 0 is read instead).  num_pages * Hkv *
 * page_size must stay below 2^31 (TKA_ERR_UNSUPPORTED otherwise). */
tka_status topk_attn_decode_paged(const tka_shape *shape, const void *q, const void *k_pages,
                                  const void *v_pages, const int32_t *block_table, int32_t max_pages,
                                  int32_t num_pages, int32_t page_size, const int32_t *seq_lens, int32_t k,
                                  float *out, int32_t *idx, float *tail_mass, void *workspace,
                                  size_t workspace_bytes, tka_stream_t stream);

/* Certified adaptive Top-k ("A Mathematical Theory of Top-k Sparse Attention
 * via Total Variation Distance", abstract: the Top-k truncation error in total
 * variation is the discarded softmax tail mass).  Per query row, k is the
 * smallest number of keys, taken in (score descending, position ascending)
 * order, whose discarded tail mass 1 - Z_k / Z is at most eps, capped at
 * min(k_max, visible keys); when even k_max keys leave more than eps outside,
 * the row keeps k_max and its tail_mass exceeds eps.  out, idx and tail_mass
 * are then exactly those of topk_attn_decode with that row's k.
 *   eps       in [0, 1); 0 keeps every visible key (when k_max allows).
 *   k_max     1..8192; idx is int32 [B,Q,Hq,k_max], ascending, -1 padded
 *             past the row's k.
 *   k_used    int32 [B,Q,Hq] device buffer: each row's k.
 *   workspace topk_attn_workspace_size(shape, k_max) bytes.
 * Other arguments, layouts and errors as topk_attn_decode; eps outside
 * [0, 1) or a missing k_used is TKA_ERR_INVALID_ARG. */
tka_status topk_attn_decode_certified(const tka_shape *shape, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *seq_lens, float eps, int32_t k_max,
                                      float *out, int32_t *idx, float *tail_mass, int32_t *k_used,
                                      void *workspace, size_t workspace_bytes, tka_stream_t stream);

/* topk_attn_decode without a workspace argument, for callers that cannot
 * allocate device memory (an engine that reserves all device memory for its
 * own pool and forbids other allocations while serving, or a host runtime with
 * no device allocator).  The pages describe no such call; it is a library
 * convenience.  The scratch space is an array compiled into the library,
 * topk_attn_static_workspace_capacity() bytes (48 MiB) on every GPU that loads
 * it, held until the process exits.  The first call on a device (with that
 * device current) looks up the array's device address; make that first call
 * before any stream capture.  Every call on a device shares the array: calls
 * whose work overlaps on the GPU race, so order them (one stream, or events).
 * Arguments are checked first, as topk_attn_decode checks them (an invalid
 * argument returns that error); a valid call whose topk_attn_workspace_size()
 * exceeds the capacity returns TKA_ERR_WORKSPACE.  Allocates nothing. */
size_t topk_attn_static_workspace_capacity(void);
tka_status topk_attn_decode_static(const tka_shape *shape, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *seq_lens, int32_t k, float *out,
                                   int32_t *idx, float *tail_mass, tka_stream_t stream);

/* MoBA block keys: block_keys[b, h, j, :] = mean of K[b, h, i, :] over the keys
 * of block j below seq_lens[b] (a partial last block is averaged over the keys
 * it holds; blocks past the end are written as zero).  block_keys is fp32
 * [B, Hkv, ceil(L_max / block_size), d].  Only shape->B, Hkv, d, L_max and
 * dtype are used.  Called when blocks change, not once per decode step. */
tka_status topk_block_pool_keys(const tka_shape *shape, const void *k_cache, const int32_t *seq_lens,
                                int32_t block_size, float *block_keys, tka_stream_t stream);

/* Bytes of scratch topk_block_attn_decode needs (0 on a bad shape). */
size_t topk_block_attn_workspace_size(const tka_shape *shape, int32_t block_size, int32_t top_blocks);

/* Block-sparse (MoBA) decode attention, one query position per sequence
 * (shape->Q == 1).  With nblk = ceil(seq_lens[b] / block_size), the blocks
 * j < nblk - 1 compete on r_j = scale * <q, block_keys[b, h/G, j, :]>; the
 * best top_blocks of them (ties to the lower j) and block nblk - 1 are kept,
 * and out is dense softmax attention over their keys below seq_lens[b].
 * block_idx (nullable) is int32 [B, 1, Hq, top_blocks + 1], ascending, -1
 * padded.  Supported: block_size in {16, 32, 64, 128}, 0 <= top_blocks <= 255,
 * ceil(L_max / block_size) <= 8192, and for bf16 B * Hkv * L_max < 2^31. */
tka_status topk_block_attn_decode(const tka_shape *shape, const void *q, const void *k_cache,
                                  const void *v_cache, const float *block_keys,
                                  const int32_t *seq_lens, int32_t block_size, int32_t top_blocks,
                                  float *out, int32_t *block_idx, void *workspace,
                                  size_t workspace_bytes, tka_stream_t stream);

/* Lightning-indexer token selection ("Sparse Attention Landscape", section
 * "Token Sparse Attention", DeepSeek Sparse Attention): per query position,
 *   I_i = sum_j w_idx[j] * ReLU(<q_idx[j], k_idx[i]>)   (j < H_I)
 * over its visible tokens; the top k tokens by I (ties to the lower position)
 * are kept for the position, shared by all its Hq heads, and every head
 * attends over them with its exact scores: out = softmax(scale * q.K) V over
 * the kept tokens.  No tail mass: the method scores the tokens with I only.
 *   q_idx   [B, Q, H_I, d_I], k_idx [B, L_max, d_I]: the indexer's projected
 *           queries and keys, in the cache dtype; w_idx fp32 [B, Q, H_I].
 *   idx     int32 [B, Q, k] ascending, -1 padded.
 *   workspace topk_indexer_attn_workspace_size(shape, H_I, d_I, k) bytes.
 * Supported: d_I in {64, 128}, 1 <= H_I <= 64, Q * H_I <= 256,
 * G = Hq / Hkv in {1, 2, 4, 8, 16}, 1 <= k <= 8192. */
size_t topk_indexer_attn_workspace_size(const tka_shape *shape, int32_t H_I, int32_t d_I, int32_t k);
tka_status topk_indexer_attn_decode(const tka_shape *shape, const void *q, const void *k_cache,
                                    const void *v_cache, const void *q_idx, const float *w_idx,
                                    const void *k_idx, int32_t H_I, int32_t d_I, const int32_t *seq_lens,
                                    int32_t k, float *out, int32_t *idx, void *workspace,
                                    size_t workspace_bytes, tka_stream_t stream);

/* Hierarchical block -> token Top-k ("Sparse Attention Landscape", section
 * "Hierarchical Sparse Attention"), one query per sequence (shape->Q == 1).
 * With nblk = ceil(seq_lens[b] / block_size): every block j < nblk scores
 * r_j = scale * <q, block_keys[b, h/G, j, :]> (the mean keys of
 * topk_block_pool_keys); the best top_blocks blocks (ties to the lower j) are
 * kept; exact token scores are computed only for the tokens of the kept
 * blocks (the candidates); the top k candidates (ties to the lower position)
 * are kept and out is softmax attention over them.
 *   idx        int32 [B, 1, Hq, k] ascending positions, -1 padded when fewer
 *              than k candidates exist.
 *   tail_mass  (nullable) the candidates' discarded softmax mass, relative to
 *              all candidates.
 *   block_idx  (nullable) int32 [B, 1, Hq, top_blocks] ascending, -1 padded.
 *   workspace  topk_hisa_attn_workspace_size(shape, block_size, top_blocks, k)
 *              bytes (0 on unsupported arguments).
 * Supported: block_size in {16, 32, 64, 128}, 1 <= top_blocks <= 8192,
 * 1 <= k <= 8192, ceil(L_max / block_size) <= 8192. */
size_t topk_hisa_attn_workspace_size(const tka_shape *shape, int32_t block_size, int32_t top_blocks, int32_t k);
tka_status topk_hisa_attn_decode(const tka_shape *shape, const void *q, const void *k_cache,
                                 const void *v_cache, const float *block_keys, const int32_t *seq_lens,
                                 int32_t block_size, int32_t top_blocks, int32_t k, float *out, int32_t *idx,
                                 float *tail_mass, int32_t *block_idx, void *workspace,
                                 size_t workspace_bytes, tka_stream_t stream);

/* Synchronises `stream`, returns the device status word of the current device
 * (TKA_DEV_* bits raised by kernels since the last read) in *bits and clears it. */
tka_status topk_attn_device_status(tka_stream_t stream, uint32_t *bits);

/* The same read as a status code: synchronises `stream`, reads and clears the
 * device status word of the current device, and returns TKA_ERR_TIMEOUT if a
 * bounded wait inside a kernel gave up (TKA_DEV_TIMEOUT), else
 * TKA_ERR_INVALID_ARG for a bad sequence length or page (TKA_DEV_BAD_SEQ_LEN,
 * TKA_DEV_BAD_PAGE), else TKA_ERR_CUDA for a failed internal check
 * (TKA_DEV_INTERNAL), else TKA_OK.  Errors of the read itself are returned as
 * topk_attn_device_status returns them. */
tka_status topk_attn_last_device_status(tka_stream_t stream);

/* Diagnostics: the number of polls after which a pipeline wait inside the
 * tensor-core score kernel and the block-attention kernel gives up (0, the
 * default, restores the kernels' own bound of about 4 million polls).  A
 * wait that gives up raises TKA_DEV_TIMEOUT; the kernel then stops, lets the
 * copies and tensor-core operations it has issued complete, frees what it
 * holds and returns, leaving that call's results incomplete.  Meant for tests
 * of that path (a limit of a few polls makes the first wait give up); it
 * applies to the calls made after it, process-wide. */
void topk_attn_debug_set_wait_limit(uint32_t polls);

/* Human-readable name of a status code. */
const char *topk_attn_status_string(tka_status status);

#ifdef __cplusplus
}
#endif

#endif /* TOPK_ATTN_H */
