// Score step on the 5th-generation tensor cores (bf16 cache).
//
// s[row, i] = scale * <q_row, K[b, kvh, i, :]> for every key below the
// sequence length, all Q*G query rows of a kv-head at once: a
// [128 keys x 128 dims] x [128 dims x N rows] product per tile of 128 keys,
// i.e. the relevance scan of the whole cache ("Sparse Attention in LLM
// Inference: Practical Trade-Offs", sections "The Role of the Indexer" and
// "The Overhead of the Indexer") with the exact logit as the score.
//
// Persistent kernel, one CTA per SM.  The valid tiles (b, kv-head, 128-key
// block below seq_lens[b]) are numbered in order and each CTA takes one
// contiguous, equal share, so every CTA streams a contiguous run of the cache
// and sees at most a few kv-heads.  Warp roles:
//   warp 0      TMA producer: K tiles (two 64-dim boxes, 128-byte swizzle) into
//               a ring of shared-memory stages; the kv-head's query rows into
//               one of two query buffers whenever the kv-head changes.
//   warp 1      MMA issuer: allocates TMEM, issues 8 tcgen05.mma (K = 16 each)
//               per tile into one of two TMEM accumulators, commits to the
//               stage's "empty" and the accumulator's "full" barriers.
//   warps 2-5   epilogue: TMEM -> registers (one key per thread, N query
//               columns), scale, coalesced score stores (32 consecutive keys
//               per warp per row; row addresses advance incrementally, no
//               division in the loop).
// K is read exactly once, so its TMA loads carry an L2 evict-first policy:
// the scores written here stay in L2 for the select step.
// Every barrier wait is bounded; a wait that gives up raises TKA_DEV_TIMEOUT,
// makes the other roles stop, drains the copies and MMAs in flight, frees
// TMEM and returns.
#include <cuda.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace tka {

namespace {

using namespace sm100;

constexpr int kTileKeys = 128;
constexpr int kKBlockBytes = kTileKeys * 128;  // 64 bf16 dims x 128 keys
constexpr int kTileBytes = 2 * kKBlockBytes;   // 128 dims
constexpr int kThreads = 192;

__host__ __device__ constexpr int stages_for(int N) { return N <= 64 ? 4 : 3; }
__host__ __device__ constexpr int tmem_cols_for(int N) { return 2 * N < 32 ? 32 : 2 * N; }

__device__ __forceinline__ int tiles_of(const ScoreTcParams &p, int b) {
    const int L = p.seq_lens[b];
    if (!seq_len_ok(L, p.Q, p.L_max)) return 0;
    return (L + kTileKeys - 1) / kTileKeys;
}

// Walks this CTA's share of the valid tiles in (bh, tile) order.
struct TileWalk {
    int bh, t, ntb, count;
    __device__ void init(const ScoreTcParams &p) {
        long long total = 0;
        for (int b = 0; b < p.B; b++) total += (long long)p.Hkv * tiles_of(p, b);
        const long long lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
        count = (int)(hi - lo);
        long long cum = 0;
        bh = 0;
        t = 0;
        ntb = 0;
        if (count == 0) return;
        for (int b = 0; b < p.B; b++) {
            const int nt = tiles_of(p, b);
            const long long here = (long long)p.Hkv * nt;
            if (lo < cum + here) {
                const long long off = lo - cum;
                bh = b * p.Hkv + (int)(off / nt);
                t = (int)(off % nt);
                ntb = nt;
                return;
            }
            cum += here;
        }
    }
    __device__ bool seg_first(int i) const { return i == 0 || t == 0; }
    __device__ bool seg_last(int i) const { return i == count - 1 || t + 1 == ntb; }
    __device__ void next(const ScoreTcParams &p) {
        if (++t < ntb) return;
        t = 0;
        do {
            ++bh;
            ntb = bh < p.B * p.Hkv ? tiles_of(p, bh / p.Hkv) : 1;
        } while (ntb == 0);
    }
};

// 32 or 64 query columns: the epilogue stages each tile's scores in shared
// memory (two staging tiles, 64 KB with 64 columns: the 4 K stages, both query
// buffers and both staging tiles take 225 KB of the 227 KB a CTA may have) and
// one TMA store writes them (a 3-D box [Q][G][128 keys] of the scores viewed
// as [B*Q, Hq, ld]); fewer columns store straight from registers
__host__ __device__ constexpr bool tma_store_for(int N) { return N == 32 || N == 64; }

// kProbe: the pipeline waits are diagnostic probes bounded by p.max_polls
// (the instantiation launched only when a test has lowered the limit)
template <int N, bool kProbe>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
             const __grid_constant__ CUtensorMap smap, ScoreTcParams p) {
    constexpr int S = stages_for(N);
    constexpr uint32_t kCols = tmem_cols_for(N);
    constexpr int kQBuf = N * 256;  // two 64-dim blocks of N rows x 128 B
    constexpr int kOutBytes = tma_store_for(N) ? 2 * N * kTileKeys * 4 : 0;  // two tiles of scores, [n][key]
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = base;
    uint8_t *qbuf = stages + S * kTileBytes;
    float *outbuf = reinterpret_cast<float *>(qbuf + 2 * kQBuf);
    uint64_t *bars = reinterpret_cast<uint64_t *>(qbuf + 2 * kQBuf + kOutBytes);
    uint64_t *full = bars, *empty = bars + S, *qfull = bars + 2 * S, *qempty = qfull + 2, *tfull = qempty + 2,
             *tempty = tfull + 2, *drain = tempty + 2;
    uint32_t *misc = reinterpret_cast<uint32_t *>(drain + 1);
    // misc: [0] TMEM base, [1] abort flag, [2] K tiles issued, [3] query loads issued
    volatile int *abort = reinterpret_cast<volatile int *>(&misc[1]);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();  // the queries, the cache and the lengths may come from the kernel before
    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < 2; j++) {
            mbar_init(&qfull[j], 1);
            mbar_init(&qempty[j], 1);
            mbar_init(&tfull[j], 1);
            mbar_init(&tempty[j], 128);
        }
        mbar_init(drain, 1);
        misc[1] = 0;
        misc[2] = 0;
        misc[3] = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&misc[0], kCols);
    if (threadIdx.x == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&qmap);
        if (tma_store_for(N)) prefetch_tensormap(&smap);
        if (blockIdx.x == 0)
            for (int b = 0; b < p.B; b++)
                if (!seq_len_ok(p.seq_lens[b], p.Q, p.L_max)) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    TileWalk w;
    w.init(p);
    bool ok = true;
    const uint32_t polls = p.max_polls;  // diagnostic probes (kProbe only)

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t evict_first = policy_evict_first();
            // paged cache: a tile is box_rows-row pieces of one or more pages;
            // the physical pages of a tile's pieces are read one tile ahead
            // (independent loads, their latency hidden behind the copies of
            // the tile before); a piece past the sequence end rereads its last
            // page (those keys are never stored)
            constexpr int kMaxPieces = kTileKeys / 16;  // pages hold >= 16 positions
            const bool paged = p.pages.table != nullptr;
            const int pshift = p.pages.page_shift;
            const int box_rows = paged ? min(1 << pshift, kTileKeys) : kTileKeys;
            const int npieces = kTileKeys / box_rows;
            int phys_cur[kMaxPieces], phys_nxt[kMaxPieces];
            auto load_pages = [&](const TileWalk &t, int (&ph)[kMaxPieces]) {
                const int b = t.bh / p.Hkv;
                const int lastp = max(p.seq_lens[b] - 1, 0) >> pshift;
                const int32_t *trow = p.pages.table + (size_t)b * p.pages.max_pages;
#pragma unroll
                for (int piece = 0; piece < kMaxPieces; piece++)
                    if (piece < npieces) ph[piece] = __ldg(trow + min((t.t * kTileKeys + piece * box_rows) >> pshift, lastp));
            };
            // pages of a tile or more: one piece, its page read right before its copies
            const bool ahead = paged && npieces > 1;
            if (ahead && w.count > 0) load_pages(w, phys_cur);
            int seg = 0;
            for (int i = 0; i < w.count && ok; i++) {
                const int b = w.bh / p.Hkv, kvh = w.bh - b * p.Hkv;
                if (w.seg_first(i)) {
                    const int qb = seg & 1;
                    if (seg >= 2) ok = pipe_wait<kProbe>(&qempty[qb], ((seg >> 1) - 1) & 1, abort, polls);
                    if (!ok) break;
                    uint8_t *dst = qbuf + qb * kQBuf;
                    mbar_arrive_expect_tx(&qfull[qb], 2u * 128u * p.NQ);
                    tma_load_3d(dst, &qmap, &qfull[qb], 0, kvh * p.G, b * p.Q);
                    tma_load_3d(dst + N * 128, &qmap, &qfull[qb], 64, kvh * p.G, b * p.Q);
                    misc[3] = seg + 1;
                }
                const int s = i % S;
                if (i >= S) ok = pipe_wait<kProbe>(&empty[s], ((i / S) - 1) & 1, abort, polls);
                if (!ok) break;
                mbar_arrive_expect_tx(&full[s], kTileBytes);
                if (p.pages.table == nullptr) {
                    const int row0 = w.bh * p.L_max + w.t * kTileKeys;
                    tma_load_2d_hint(stages + s * kTileBytes, &kmap, &full[s], 0, row0, evict_first);
                    tma_load_2d_hint(stages + s * kTileBytes + kKBlockBytes, &kmap, &full[s], 64, row0, evict_first);
                } else {
                    if (!ahead) load_pages(w, phys_cur);
#pragma unroll
                    for (int piece = 0; piece < kMaxPieces; piece++) {
                        if (piece >= npieces) break;
                        int phys = phys_cur[piece];
                        if ((unsigned)phys >= (unsigned)p.pages.num_pages) {
                            raise_status(p.status, TKA_DEV_BAD_PAGE);  // page 0 is read instead
                            phys = 0;
                        }
                        const int pos = w.t * kTileKeys + piece * box_rows;
                        const int row0 = (int)((((long long)phys * p.Hkv + kvh) << pshift) + (pos & ((1 << pshift) - 1)));
                        uint8_t *dst = stages + s * kTileBytes + piece * box_rows * 128;
                        tma_load_2d_hint(dst, &kmap, &full[s], 0, row0, evict_first);
                        tma_load_2d_hint(dst + kKBlockBytes, &kmap, &full[s], 64, row0, evict_first);
                    }
                    // the next tile's pages, read after this tile's copies are out
                    // (the producer issues in order: a load that waits on another
                    // load must not hold up the copies)
                    if (ahead && i + 1 < w.count) {
                        TileWalk wn = w;
                        wn.next(p);
                        load_pages(wn, phys_nxt);
#pragma unroll
                        for (int piece = 0; piece < kMaxPieces; piece++) phys_cur[piece] = phys_nxt[piece];
                    }
                }
                misc[2] = i + 1;
                if (w.seg_last(i)) seg++;
                w.next(p);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, N);
            int seg = 0;
            for (int i = 0; i < w.count && ok; i++) {
                const int qb = seg & 1;
                if (w.seg_first(i)) ok = pipe_wait<kProbe>(&qfull[qb], (seg >> 1) & 1, abort, polls);
                const int s = i % S, buf = i & 1;
                if (ok) ok = pipe_wait<kProbe>(&full[s], (i / S) & 1, abort, polls);
                if (ok && i >= 2) ok = pipe_wait<kProbe>(&tempty[buf], ((i >> 1) - 1) & 1, abort, polls);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a0 = smem_addr(stages + s * kTileBytes), b0 = smem_addr(qbuf + qb * kQBuf);
#pragma unroll
                for (int k = 0; k < 8; k++) {
                    const uint64_t ad = smem_desc_sw128(a0 + (k >> 2) * kKBlockBytes + (k & 3) * 32);
                    const uint64_t bd = smem_desc_sw128(b0 + (k >> 2) * (N * 128) + (k & 3) * 32);
                    mma_bf16(tmem + buf * N, ad, bd, idesc, k > 0 ? 1u : 0u);
                }
                mma_commit(&empty[s]);
                mma_commit(&tfull[buf]);
                if (w.seg_last(i)) {
                    mma_commit(&qempty[qb]);
                    seg++;
                }
                w.next(p);
            }
            // every MMA issued above has completed once this arrives (waited
            // for even after an abort: TMEM is freed below)
            mma_commit(drain);
            int no_abort = 0;
            if (!mbar_wait(drain, 0, reinterpret_cast<volatile int *>(&no_abort))) ok = false;
        }
    } else if (tma_store_for(N)) {
        // each tile: TMEM -> registers (every column's load issued before
        // one wait) -> one of two shared-memory tiles (column n at [n][key]);
        // the 128 epilogue threads decide together whether to go on (a
        // barrier that ANDs their waits: no thread is left behind at the
        // barriers below), the accumulator is released as soon as it has been
        // read, and one thread stores the tile with TMA.  A staging tile is
        // rewritten two tiles later, once its store has read it.  Scores a
        // causal query position cannot see are stored too: nothing reads them.
        const int quarter = warp & 3;  // TMEM lanes [32*quarter, +32)
        const uint32_t tlane = (uint32_t)(quarter * 32) << 16;
        const int kq = quarter * 32 + lane;
        const bool issuer = warp == 2 && lane == 0;
        const float scale = p.scale;
        for (int i = 0; i < w.count; i++) {
            const int b = w.bh / p.Hkv, kvh = w.bh - b * p.Hkv;
            const int buf = i & 1;
            ok = pipe_wait<kProbe>(&tfull[buf], (i >> 1) & 1, abort, polls);
            ok = named_bar_and(1, 128, ok);
            if (!ok) break;
            tc_fence_after();
            float *stage = outbuf + (i & 1) * (N * kTileKeys);
            uint32_t r[N / 16][16];
#pragma unroll
            for (int c = 0; c < N / 16; c++)
                if (c * 16 < p.NQ) tmem_ld16(tmem + tlane + buf * N + c * 16, r[c]);
            if (issuer) bulk_wait_read_but_one();  // the store of two tiles ago has read this stage
            tmem_wait_ld();
            named_bar_sync(1, 128);  // the stage is free
#pragma unroll
            for (int c = 0; c < N / 16; c++) {
                if (c * 16 >= p.NQ) break;
#pragma unroll
                for (int j = 0; j < 16; j++)
                    if (c * 16 + j < p.NQ) stage[(c * 16 + j) * kTileKeys + kq] = __uint_as_float(r[c][j]) * scale;
            }
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
            fence_proxy_async_shared();
            named_bar_sync(1, 128);  // the tile is complete
            if (issuer) {
                tma_store_3d(&smap, stage, w.t * kTileKeys, kvh * p.G, b * p.Q);
                bulk_commit_group();
            }
            w.next(p);
        }
        if (issuer) bulk_wait_all();  // the shared tile outlives every store reading it
    } else {
        const int quarter = warp & 3;      // TMEM lanes [32*quarter, +32)
        const uint32_t tlane = (uint32_t)(quarter * 32) << 16;
        const float scale = p.scale;
        for (int i = 0; i < w.count && ok; i++) {
            const int b = w.bh / p.Hkv, kvh = w.bh - b * p.Hkv;
            const int seq_len = p.seq_lens[b];
            const int buf = i & 1;
            ok = pipe_wait<kProbe>(&tfull[buf], (i >> 1) & 1, abort, polls);
            if (!ok) break;
            tc_fence_after();
            const int key = w.t * kTileKeys + quarter * 32 + lane;
            // column n = qpos * G + gi is query row (b, qpos, kvh*G + gi); walk it without division
            float *dst = p.scores + (((size_t)b * p.Q) * p.Hq + (size_t)kvh * p.G) * p.ld + key;
            int qpos = 0, gi = 0, vis = seq_len - p.Q + 1;
#pragma unroll
            for (int c = 0; c < N / 16; c++) {
                if (c * 16 >= p.NQ) break;
                uint32_t r[16];
                tmem_ld16(tmem + tlane + buf * N + c * 16, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    if (c * 16 + j >= p.NQ) break;
                    // keys a causal query position cannot see are not stored
                    if (key < vis) *dst = __uint_as_float(r[j]) * scale;
                    dst += p.ld;
                    if (++gi == p.G) {
                        gi = 0;
                        ++qpos;
                        ++vis;
                        dst += (size_t)(p.Hq - p.G) * p.ld;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
            w.next(p);
        }
    }

    if (!ok) {
        *abort = 1;
        raise_status(p.status, TKA_DEV_TIMEOUT);
    }
    __syncthreads();
    if (*abort && threadIdx.x == 0) {
        // let every copy still in flight land before the shared memory goes away
        const int issued = (int)misc[2], qissued = (int)misc[3];
        for (int s = 0; s < S && s < issued; s++) {
            const int last = issued - 1 - ((issued - 1 - s) % S);
            int dummy = 0;
            mbar_wait(&full[s], (last / S) & 1, reinterpret_cast<volatile int *>(&dummy));
        }
        for (int j = 0; j < 2 && j < qissued; j++) {
            const int last = qissued - 1 - ((qissued - 1 - j) % 2);
            int dummy = 0;
            mbar_wait(&qfull[j], (last >> 1) & 1, reinterpret_cast<volatile int *>(&dummy));
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kCols);
    }
}

template <int N>
size_t smem_bytes() {
    constexpr int S = stages_for(N);
    return 1024 + (size_t)S * kTileBytes + 2 * (size_t)N * 256 +
           (tma_store_for(N) ? 2 * (size_t)N * kTileKeys * 4 : 0) +
           (2 * S + 9) * 8 + 64;
}

template <int N>
cudaError_t launch_n(const CUtensorMap &km, const CUtensorMap &qm, const CUtensorMap &sm, const ScoreTcParams &p,
                     int num_sms, cudaStream_t stream, const ScoreTcHook &hook, bool pdl) {
    const size_t smem = smem_bytes<N>();
    static std::atomic<bool> attr_set[64] = {};  // per device: the shared-memory opt-in is a function attribute
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(score_tc<N, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(score_tc<N, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
    }
    if (hook.fn) {
        e = hook.fn(hook.ctx);  // e.g. a timing event, right before the launch
        if (e != cudaSuccess) return e;
    }
    if (p.max_polls)
        return launch_k(pdl, score_tc<N, true>, dim3(num_sms), dim3(kThreads), smem, stream, km, qm, sm, p);
    return launch_k(pdl, score_tc<N, false>, dim3(num_sms), dim3(kThreads), smem, stream, km, qm, sm, p);
}

}  // namespace

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

bool score_tc_supported(int dtype, int NQ) { return dtype == TKA_BF16 && NQ <= 128 && encode_fn() != nullptr; }

cudaError_t launch_score_tc(const ScoreTcParams &p, const void *q, const void *k_cache, int num_sms,
                            cudaStream_t stream, const ScoreTcHook &hook, bool pdl) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap km, qm;
    {
        // K cache as rows of 128 bf16: [B*Hkv*L_max, 128] (paged: [num_pages*Hkv*page, 128]);
        // boxes of 128 rows (paged: min(page, 128) rows) x 64 dims.  (A 3-D map
        // [B*Hkv][L_max][128] with boxes one kv-head deep streamed 5 % slower.)
        const bool paged = p.pages.table != nullptr;
        const cuuint64_t nrows = paged ? (cuuint64_t)p.pages.num_pages * p.Hkv << p.pages.page_shift
                                       : (cuuint64_t)p.B * p.Hkv * p.L_max;
        const cuuint64_t dims[2] = {128, nrows};
        const cuuint64_t strides[1] = {256};
        const cuuint32_t box[2] = {64, paged ? (cuuint32_t)min(1 << p.pages.page_shift, kTileKeys) : (cuuint32_t)kTileKeys};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(k_cache), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        // queries as [B*Q, Hq, 128]; one box = the G heads of a kv-head at all Q positions
        const cuuint64_t dims[3] = {128, (cuuint64_t)p.Hq, (cuuint64_t)p.B * p.Q};
        const cuuint64_t strides[2] = {256, (cuuint64_t)p.Hq * 256};
        const cuuint32_t box[3] = {64, (cuuint32_t)p.G, (cuuint32_t)p.Q};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const int NQ = p.NQ;
    CUtensorMap sm;
    memset(&sm, 0, sizeof(sm));
    if (NQ > 16 && NQ <= 64) {
        // the scores as [B*Q, Hq, ld] fp32; one box = 128 keys of the G heads of a kv-head at all Q positions
        const cuuint64_t dims[3] = {(cuuint64_t)p.ld, (cuuint64_t)p.Hq, (cuuint64_t)p.B * p.Q};
        const cuuint64_t strides[2] = {(cuuint64_t)p.ld * 4, (cuuint64_t)p.Hq * p.ld * 4};
        const cuuint32_t box[3] = {(cuuint32_t)kTileKeys, (cuuint32_t)p.G, (cuuint32_t)p.Q};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&sm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.scores, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    if (NQ <= 16) return launch_n<16>(km, qm, sm, p, num_sms, stream, hook, pdl);
    if (NQ <= 32) return launch_n<32>(km, qm, sm, p, num_sms, stream, hook, pdl);
    if (NQ <= 64) return launch_n<64>(km, qm, sm, p, num_sms, stream, hook, pdl);
    return launch_n<128>(km, qm, sm, p, num_sms, stream, hook, pdl);
}

}  // namespace tka
