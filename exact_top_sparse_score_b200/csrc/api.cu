// C ABI entry points: argument checks, workspace layout and the launch
// sequence of each operation.  Nothing here allocates or synchronises on the
// compute path; every launch goes onto the caller's stream.
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace tka {
namespace {

__device__ unsigned int g_status = 0u;

// Polls before a pipeline wait inside a kernel gives up (0: the kernels'
// default bound); set only through topk_attn_debug_set_wait_limit.
std::atomic<uint32_t> g_wait_polls{0u};

constexpr int kMaxDevices = 64;
constexpr int kMaxQ = 64;
constexpr int kMaxRowsPerKvHead = 256;  // Q * G
constexpr int kMaxLen = 1 << 24;
constexpr int kMinKeysPerSplit = 64;

struct DeviceInfo {
    std::atomic<bool> ready{false};  // published (release) once the fields below are set
    int num_sms = 0;
    unsigned *status = nullptr;  // device address of g_status
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;  // serialises the first lookup on a device

// SM count and status-word address of the current device (looked up once;
// concurrent first calls from several host threads wait for one lookup).
cudaError_t device_info(DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    DeviceInfo &d = g_dev[dev];
    if (!d.ready.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(g_dev_mu);
        if (!d.ready.load(std::memory_order_relaxed)) {
            e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            e = cudaGetSymbolAddress(reinterpret_cast<void **>(&d.status), g_status);
            if (e != cudaSuccess) return e;
            d.ready.store(true, std::memory_order_release);
        }
    }
    *out = &d;
    return cudaSuccess;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

cudaError_t record(const tka_event_t *events, int i, cudaStream_t s) {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[i]), s);
}

bool has_event(const tka_event_t *events, int i) { return events && events[i]; }

struct RecordCtx {
    const tka_event_t *events;
    int i;
    cudaStream_t s;
};
cudaError_t record_hook(void *ctx) {
    const RecordCtx *c = static_cast<const RecordCtx *>(ctx);
    return record(c->events, c->i, c->s);
}

float resolve_scale(const tka_shape *s) { return s->scale > 0.f ? s->scale : 1.f / sqrtf((float)s->d); }

// Shape checks shared by both variants.
tka_status check_shape(const tka_shape *s) {
    if (!s) return TKA_ERR_INVALID_ARG;
    if (s->B < 1 || s->Q < 1 || s->Hq < 1 || s->Hkv < 1 || s->d < 1 || s->L_max < 1) return TKA_ERR_INVALID_ARG;
    if (s->Hq % s->Hkv) return TKA_ERR_INVALID_ARG;
    if (!(s->scale >= 0.f) || isinf(s->scale)) return TKA_ERR_INVALID_ARG;
    if (s->Q > s->L_max) return TKA_ERR_INVALID_ARG;
    if (s->d != kHeadDim) return TKA_ERR_UNSUPPORTED;
    if (s->dtype != TKA_F32 && s->dtype != TKA_BF16) return TKA_ERR_UNSUPPORTED;
    if (s->Q > kMaxQ || s->L_max > kMaxLen) return TKA_ERR_UNSUPPORTED;
    if ((long long)s->Q * (s->Hq / s->Hkv) > kMaxRowsPerKvHead) return TKA_ERR_UNSUPPORTED;
    if ((long long)s->B * s->Hkv > 65535 || (long long)s->B * s->Q * s->Hq > 65535) return TKA_ERR_UNSUPPORTED;
    return TKA_OK;
}

// Workspace of topk_attn_decode, in order, each region 256-byte aligned:
//   scores   fp32 [rows, ld]          ld = L_max rounded up to 64
//   weights  fp32 [rows, k]           e^{s - m} of the kept positions
//   stats    float4 [rows]            {m, Z_k, Z_tail, 0}
//   partial  fp32 [rows, max_splits, 128]
//   counters uint32 [rows]
struct TokenLayout {
    size_t scores, weights, stats, partial, counters, total;
    int ld, max_splits;
};

TokenLayout token_layout(const tka_shape *s, int k) {
    TokenLayout L;
    const size_t rows = (size_t)s->B * s->Q * s->Hq;
    L.ld = (int)align_up((size_t)s->L_max, 64);
    L.max_splits = (k + kMinKeysPerSplit - 1) / kMinKeysPerSplit;
    size_t off = 0;
    L.scores = off;
    off = align_up(off + rows * L.ld * sizeof(float), 256);
    L.weights = off;
    off = align_up(off + rows * (size_t)k * sizeof(float), 256);
    L.stats = off;
    off = align_up(off + rows * sizeof(float4), 256);
    L.partial = off;
    off = align_up(off + rows * (size_t)L.max_splits * kHeadDim * sizeof(float), 256);
    L.counters = off;
    off = align_up(off + rows * sizeof(unsigned), 256);
    L.total = off;
    return L;
}

// Workspace of topk_block_attn_decode:
//   bscore    fp32 [rows, nblk_max]  block scores
//   block_idx int32 [rows, top+1]  (used when the caller passes none)
//   part_ml   float4 [rows, top+1]
//   part_acc  fp32 [rows, top+1, 128]
//   counters  uint32 [rows]
struct BlockLayout {
    size_t bscore, block_idx, part_ml, part_acc, counters, total;
};

BlockLayout block_layout(const tka_shape *s, int block_size, int top_blocks) {
    BlockLayout L;
    const size_t rows = (size_t)s->B * s->Hq, slots = (size_t)top_blocks + 1;
    const size_t nblk_max = ((size_t)s->L_max + block_size - 1) / block_size;
    size_t off = 0;
    L.bscore = off;
    off = align_up(off + rows * nblk_max * sizeof(float), 256);
    L.block_idx = off;
    off = align_up(off + rows * slots * sizeof(int32_t), 256);
    L.part_ml = off;
    off = align_up(off + rows * slots * sizeof(float4), 256);
    L.part_acc = off;
    off = align_up(off + rows * slots * kHeadDim * sizeof(float), 256);
    L.counters = off;
    off = align_up(off + rows * sizeof(unsigned), 256);
    L.total = off;
    return L;
}

tka_status check_block_args(const tka_shape *s, int block_size, int top_blocks) {
    tka_status st = check_shape(s);
    if (st != TKA_OK) return st;
    if (block_size < 1 || top_blocks < 0) return TKA_ERR_INVALID_ARG;
    if (block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128) return TKA_ERR_UNSUPPORTED;
    if (s->Q != 1 || top_blocks > 255) return TKA_ERR_UNSUPPORTED;
    if ((s->L_max + block_size - 1) / block_size > 8192) return TKA_ERR_UNSUPPORTED;
    // bf16 K blocks are fetched through a tensor map whose row coordinate is a 32-bit int
    if (s->dtype == TKA_BF16 && (long long)s->B * s->Hkv * s->L_max >= (1ll << 31)) return TKA_ERR_UNSUPPORTED;
    return TKA_OK;
}

// Workspace of topk_hisa_attn_decode, in order (256-byte aligned regions):
//   bscore    fp32 [rows, nblk_max]   block scores
//   block_idx int32 [rows, top]       (when the caller passes none)
//   cscore    fp32 [rows, ldc]        candidate scores, ldc = top * bs rounded up to 64
//   row_len   int32 [rows]            valid candidates per row
//   weights   fp32 [rows, k], stats float4 [rows], partial fp32 [rows, k/64, d], counters uint32 [rows]
struct HisaLayout {
    size_t bscore, block_idx, cscore, row_len, weights, stats, partial, counters, total;
    int ldc, max_splits;
};

HisaLayout hisa_layout(const tka_shape *s, int block_size, int top_blocks, int k) {
    HisaLayout L;
    const size_t rows = (size_t)s->B * s->Hq;
    const size_t nblk_max = ((size_t)s->L_max + block_size - 1) / block_size;
    L.ldc = (int)align_up((size_t)top_blocks * block_size, 64);
    L.max_splits = (k + kMinKeysPerSplit - 1) / kMinKeysPerSplit;
    size_t off = 0;
    L.bscore = off;
    off = align_up(off + rows * nblk_max * sizeof(float), 256);
    L.block_idx = off;
    off = align_up(off + rows * (size_t)top_blocks * sizeof(int32_t), 256);
    L.cscore = off;
    off = align_up(off + rows * (size_t)L.ldc * sizeof(float), 256);
    L.row_len = off;
    off = align_up(off + rows * sizeof(int32_t), 256);
    L.weights = off;
    off = align_up(off + rows * (size_t)k * sizeof(float), 256);
    L.stats = off;
    off = align_up(off + rows * sizeof(float4), 256);
    L.partial = off;
    off = align_up(off + rows * (size_t)L.max_splits * kHeadDim * sizeof(float), 256);
    L.counters = off;
    off = align_up(off + rows * sizeof(unsigned), 256);
    L.total = off;
    return L;
}

// Workspace of topk_indexer_attn_decode (256-byte aligned regions):
//   iscores fp32 [B*Q, ld], weights fp32 [B*Q, k], stats float4 [B*Q],
//   sel counters uint32 [B*Q], part_ml float4 [B*Q*Hq, k/64],
//   part_acc fp32 [B*Q*Hq, k/64, d], attn counters uint32 [B*Q*Hkv]
struct IndexerLayout {
    size_t iscores, weights, stats, sel_counters, part_ml, part_acc, attn_counters, raw, total;
    int ld, max_splits;
};

// tensor-core indexer dots: bf16 128-dim index keys, all heads of a sequence as query rows of one kv-head
bool indexer_tc(const tka_shape *s, int H_I, int d_I) {
    return d_I == 128 && s->dtype == TKA_BF16 && score_tc_supported(TKA_BF16, s->Q * H_I) &&
           (long long)s->B * s->L_max < (1ll << 31);
}

IndexerLayout indexer_layout(const tka_shape *s, int k, int H_I, int d_I) {
    IndexerLayout L;
    const size_t units = (size_t)s->B * s->Q, rows = units * s->Hq;
    L.ld = (int)align_up((size_t)s->L_max, 64);
    L.max_splits = (k + kMinKeysPerSplit - 1) / kMinKeysPerSplit;
    size_t off = 0;
    L.iscores = off;
    off = align_up(off + units * L.ld * sizeof(float), 256);
    L.weights = off;
    off = align_up(off + units * (size_t)k * sizeof(float), 256);
    L.stats = off;
    off = align_up(off + units * sizeof(float4), 256);
    L.sel_counters = off;
    off = align_up(off + units * sizeof(unsigned), 256);
    L.part_ml = off;
    off = align_up(off + rows * L.max_splits * sizeof(float4), 256);
    L.part_acc = off;
    off = align_up(off + rows * L.max_splits * kHeadDim * sizeof(float), 256);
    L.attn_counters = off;
    off = align_up(off + units * s->Hkv * sizeof(unsigned), 256);
    L.raw = off;  // per-head dots of the tensor-core path: fp32 [B*Q*H_I, ld]
    if (indexer_tc(s, H_I, d_I)) off = align_up(off + units * H_I * (size_t)L.ld * sizeof(float), 256);
    L.total = off;
    return L;
}

tka_status check_indexer_args(const tka_shape *s, int H_I, int d_I, int k) {
    tka_status st = check_shape(s);
    if (st != TKA_OK) return st;
    if (H_I < 1 || d_I < 1 || k < 1) return TKA_ERR_INVALID_ARG;
    if (!indexer_supported(s->Hq / s->Hkv, d_I) || H_I > 64 || s->Q * H_I > 256 || k > kMaxK)
        return TKA_ERR_UNSUPPORTED;
    return TKA_OK;
}

tka_status check_hisa_args(const tka_shape *s, int block_size, int top_blocks, int k) {
    tka_status st = check_shape(s);
    if (st != TKA_OK) return st;
    if (block_size < 1 || top_blocks < 1 || k < 1) return TKA_ERR_INVALID_ARG;
    if (block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128) return TKA_ERR_UNSUPPORTED;
    if (s->Q != 1 || top_blocks > 8192 || k > kMaxK) return TKA_ERR_UNSUPPORTED;
    if ((s->L_max + block_size - 1) / block_size > 8192) return TKA_ERR_UNSUPPORTED;
    return TKA_OK;
}

}  // namespace
}  // namespace tka

using namespace tka;

extern "C" {

size_t topk_attn_workspace_size(const tka_shape *shape, int32_t k) {
    if (check_shape(shape) != TKA_OK || k < 1 || k > kMaxK) return 0;
    return token_layout(shape, k).total;
}

}  // extern "C"

namespace {

// The certified variant's extra arguments (null for a fixed k).
struct CertArgs {
    float eps;
    int32_t *k_used;
};

// Everything decode_impl resolved before the launches.
struct DecodeArgs {
    const tka_shape *shape;
    const void *q, *k_cache, *v_cache;
    const int32_t *seq_lens;
    int k, G;
    float *out, *tail;
    int32_t *idx;
    char *ws;
    TokenLayout L;
    DeviceInfo *dev;
    const CertArgs *cert;
    const PageTable *pages;
    bool tc;
};

// The score kernel of a decode on s.
tka_status launch_score(const DecodeArgs &a, cudaStream_t s, const tka_event_t *events) {
    const tka_shape *sh = a.shape;
    float *scores = reinterpret_cast<float *>(a.ws + a.L.scores);
    if (a.tc) {
        ScoreTcParams tp;
        tp.status = a.dev->status;
        tp.seq_lens = a.seq_lens;
        tp.scores = scores;
        tp.B = sh->B; tp.Q = sh->Q; tp.Hq = sh->Hq; tp.Hkv = sh->Hkv; tp.G = a.G;
        tp.L_max = sh->L_max; tp.ld = a.L.ld; tp.NQ = sh->Q * a.G;
        tp.scale = resolve_scale(sh);
        if (a.pages) tp.pages = *a.pages;
        tp.max_polls = g_wait_polls.load(std::memory_order_relaxed);
        RecordCtx rc{events, 0, s};
        ScoreTcHook hook;
        hook.fn = record_hook;
        hook.ctx = &rc;
        if (launch_score_tc(tp, a.q, a.k_cache, a.dev->num_sms, s, hook, !has_event(events, 0)) != cudaSuccess)
            return TKA_ERR_CUDA;
    } else {
        if (record(events, 0, s) != cudaSuccess) return TKA_ERR_CUDA;
        ScoreParams sp;
        sp.status = a.dev->status;
        sp.q = a.q;
        sp.k = a.k_cache;
        sp.seq_lens = a.seq_lens;
        sp.scores = scores;
        sp.B = sh->B; sp.Q = sh->Q; sp.Hq = sh->Hq; sp.Hkv = sh->Hkv; sp.G = a.G;
        sp.L_max = sh->L_max; sp.ld = a.L.ld; sp.dtype = sh->dtype;
        sp.scale = resolve_scale(sh);
        if (a.pages) sp.pages = *a.pages;
        if (tka::launch_score(sp, a.dev->num_sms, s) != cudaSuccess) return TKA_ERR_CUDA;
    }
    return TKA_OK;
}

// Select (k) -> [certify] -> gather of a decode on s.
tka_status launch_rest(const DecodeArgs &a, cudaStream_t s, int select_threads, const tka_event_t *events) {
    const tka_shape *sh = a.shape;
    const int rows = sh->B * sh->Q * sh->Hq;
    const float *scores = reinterpret_cast<const float *>(a.ws + a.L.scores);
    int32_t *idx = a.idx;
    float *w = reinterpret_cast<float *>(a.ws + a.L.weights);
    float4 *stats = reinterpret_cast<float4 *>(a.ws + a.L.stats);
    unsigned *counters = reinterpret_cast<unsigned *>(a.ws + a.L.counters);
    float *tail = a.tail;
    int32_t *k_used = a.cert ? a.cert->k_used : nullptr;

    SelectParams se;
    se.status = a.dev->status;
    se.scores = scores;
    se.seq_lens = a.seq_lens;
    se.B = sh->B; se.Q = sh->Q; se.Hq = sh->Hq; se.L_max = sh->L_max; se.ld = a.L.ld; se.k = a.k;
    se.idx = idx;
    se.w = w;
    se.stats = stats;
    se.tail = tail;
    se.counters = counters;
    // a kernel with no event recorded just before it may start behind the one before
    if (launch_select(se, s, select_threads, !has_event(events, 1)) != cudaSuccess) return TKA_ERR_CUDA;
    if (a.cert) {
        CertifyParams cp;
        cp.status = a.dev->status;
        cp.scores = scores;
        cp.seq_lens = a.seq_lens;
        cp.B = sh->B; cp.Q = sh->Q; cp.Hq = sh->Hq; cp.L_max = sh->L_max; cp.ld = a.L.ld;
        cp.k_max = a.k;
        cp.eps = a.cert->eps;
        cp.idx = idx;
        cp.w = w;
        cp.stats = stats;
        cp.tail = tail;
        cp.k_used = k_used;
        if (launch_certify(cp, s, true) != cudaSuccess) return TKA_ERR_CUDA;
    }
    if (record(events, 2, s) != cudaSuccess) return TKA_ERR_CUDA;

    GatherParams gp;
    gp.status = a.dev->status;
    gp.v = a.v_cache;
    gp.seq_lens = a.seq_lens;
    gp.B = sh->B; gp.Q = sh->Q; gp.Hq = sh->Hq; gp.Hkv = sh->Hkv; gp.G = a.G;
    gp.L_max = sh->L_max; gp.k = a.k; gp.dtype = sh->dtype;
    gp.idx = idx;
    gp.w = w;
    gp.stats = stats;
    gp.partial = reinterpret_cast<float *>(a.ws + a.L.partial);
    gp.counters = counters;
    gp.out = a.out;
    gp.kcount = k_used;
    if (a.pages) gp.pages = *a.pages;
    // one wave of eight CTAs per SM (splits = floor(8 x SMs / rows), at least 1),
    // never fewer than kMinKeysPerSplit keys per CTA
    int splits = (a.dev->num_sms * 8) / rows;
    if (splits > a.L.max_splits) splits = a.L.max_splits;
    if (splits < 1) splits = 1;
    gp.per_split = (a.k + splits - 1) / splits;
    gp.splits = (a.k + gp.per_split - 1) / gp.per_split;
    if (launch_gather(gp, s, !has_event(events, 2)) != cudaSuccess) return TKA_ERR_CUDA;
    return TKA_OK;
}

// Whether a decode is small enough for the one-launch path: at most kTinyKeys
// cache rows in all, no more query rows and kv-heads than SMs (one CTA per
// query row after the grid barrier, every CTA resident at once), and at most
// 64 query rows per kv-head (their query vectors sit in shared memory).
constexpr long long kTinyKeys = 1 << 16;

bool use_tiny(const tka_shape *sh, int num_sms) {
    const long long rows = (long long)sh->B * sh->Q * sh->Hq, units = (long long)sh->B * sh->Hkv;
    return (long long)sh->B * sh->Hkv * sh->L_max <= kTinyKeys && rows <= num_sms && units <= num_sms &&
           sh->Q * (sh->Hq / sh->Hkv) <= 64;
}

tka_status launch_tiny_decode(const DecodeArgs &a, cudaStream_t s) {
    const tka_shape *sh = a.shape;
    TinyParams tp;
    SelectParams &se = tp.sel;
    se.status = a.dev->status;
    se.scores = reinterpret_cast<const float *>(a.ws + a.L.scores);
    se.seq_lens = a.seq_lens;
    se.B = sh->B; se.Q = sh->Q; se.Hq = sh->Hq; se.L_max = sh->L_max; se.ld = a.L.ld; se.k = a.k;
    se.idx = a.idx;
    se.w = reinterpret_cast<float *>(a.ws + a.L.weights);
    se.stats = reinterpret_cast<float4 *>(a.ws + a.L.stats);
    se.tail = a.tail;
    se.counters = reinterpret_cast<unsigned *>(a.ws + a.L.counters);
    tp.scores = reinterpret_cast<float *>(a.ws + a.L.scores);
    tp.q = a.q; tp.k = a.k_cache; tp.v = a.v_cache;
    tp.Hkv = sh->Hkv; tp.G = a.G; tp.dtype = sh->dtype;
    tp.scale = resolve_scale(sh);
    tp.out = a.out;
    const int units = sh->B * sh->Hkv, rows = sh->B * sh->Q * sh->Hq;
    const int chunks = (sh->L_max + 127) / 128;
    tp.cpb = max(1, min(a.dev->num_sms / units, chunks));
    const int grid = max(units * tp.cpb, rows);
    return launch_tiny(tp, grid, s) == cudaSuccess ? TKA_OK : TKA_ERR_CUDA;
}

// Score -> select (k) -> [certify] -> gather on `stream`.
tka_status decode_impl(const tka_shape *shape, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *seq_lens, int32_t k, float *out, int32_t *idx, float *tail_mass,
                       void *workspace, size_t workspace_bytes, tka_stream_t stream, const tka_event_t events[4],
                       const CertArgs *cert, const PageTable *pages = nullptr) {
    tka_status st = check_shape(shape);
    if (st != TKA_OK) return st;
    if (k < 1) return TKA_ERR_INVALID_ARG;
    if (k > kMaxK) return TKA_ERR_UNSUPPORTED;
    if (!q || !k_cache || !v_cache || !seq_lens || !out || !idx) return TKA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
        !aligned(idx, 4) || !aligned(seq_lens, 4) || (tail_mass && !aligned(tail_mass, 4)))
        return TKA_ERR_INVALID_ARG;
    DecodeArgs a;
    a.shape = shape;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.seq_lens = seq_lens;
    a.k = k;
    a.G = shape->Hq / shape->Hkv;
    a.out = out;
    a.tail = tail_mass;
    a.idx = idx;
    a.L = token_layout(shape, k);
    a.cert = cert;
    a.pages = pages;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < a.L.total) return TKA_ERR_WORKSPACE;
    a.ws = static_cast<char *>(workspace);
    if (device_info(&a.dev) != cudaSuccess) return TKA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the tensor map addresses cache rows with int32 coordinates (a K cache of
    // 2^31 rows, 512 GB, does not fit one GPU; the CUDA-core scorer takes it)
    a.tc = score_tc_supported(shape->dtype, shape->Q * a.G) &&
           (pages || (long long)shape->B * shape->Hkv * shape->L_max < (1LL << 31));

    // a small problem (no events to record between steps): one launch does
    // all three steps
    if (!events && !cert && !pages && use_tiny(shape, a.dev->num_sms)) return launch_tiny_decode(a, s);

    st = launch_score(a, s, events);
    if (st != TKA_OK) return st;
    if (record(events, 1, s) != cudaSuccess) return TKA_ERR_CUDA;
    // more rows than SMs: 512-thread select CTAs, two rows per SM at a time
    // (a 1024-thread CTA takes a whole SM's registers, and the rows would run
    // in waves of one per SM); otherwise 1024 threads per row
    const int rows = shape->B * shape->Q * shape->Hq;
    st = launch_rest(a, s, rows > a.dev->num_sms ? 512 : 1024, events);
    if (st != TKA_OK) return st;
    if (record(events, 3, s) != cudaSuccess) return TKA_ERR_CUDA;
    return TKA_OK;
}

}  // namespace

extern "C" {

tka_status topk_attn_decode_staged(const tka_shape *shape, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *seq_lens, int32_t k, float *out,
                                   int32_t *idx, float *tail_mass, void *workspace, size_t workspace_bytes,
                                   tka_stream_t stream, const tka_event_t events[4]) {
    return decode_impl(shape, q, k_cache, v_cache, seq_lens, k, out, idx, tail_mass, workspace, workspace_bytes,
                       stream, events, nullptr);
}

tka_status topk_attn_decode_paged(const tka_shape *shape, const void *q, const void *k_pages, const void *v_pages,
                                  const int32_t *block_table, int32_t max_pages, int32_t num_pages,
                                  int32_t page_size, const int32_t *seq_lens, int32_t k, float *out, int32_t *idx,
                                  float *tail_mass, void *workspace, size_t workspace_bytes, tka_stream_t stream) {
    if (!block_table || !aligned(block_table, 4)) return TKA_ERR_INVALID_ARG;
    if (page_size < 16 || (page_size & (page_size - 1)) || max_pages < 1 || num_pages < 1)
        return TKA_ERR_INVALID_ARG;
    if (!shape) return TKA_ERR_INVALID_ARG;
    if ((long long)max_pages * page_size < shape->L_max) return TKA_ERR_INVALID_ARG;
    // rows of the paged cache are addressed with 32-bit row numbers
    if ((long long)num_pages * shape->Hkv * page_size >= (1ll << 31)) return TKA_ERR_UNSUPPORTED;
    PageTable pt;
    pt.table = block_table;
    pt.max_pages = max_pages;
    pt.num_pages = num_pages;
    pt.page_shift = __builtin_ctz((unsigned)page_size);
    return decode_impl(shape, q, k_pages, v_pages, seq_lens, k, out, idx, tail_mass, workspace, workspace_bytes,
                       stream, nullptr, nullptr, &pt);
}

tka_status topk_attn_decode_certified(const tka_shape *shape, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *seq_lens, float eps, int32_t k_max,
                                      float *out, int32_t *idx, float *tail_mass, int32_t *k_used,
                                      void *workspace, size_t workspace_bytes, tka_stream_t stream) {
    if (!(eps >= 0.f) || !(eps < 1.f) || !k_used || !aligned(k_used, 4)) return TKA_ERR_INVALID_ARG;
    const CertArgs cert{eps, k_used};
    return decode_impl(shape, q, k_cache, v_cache, seq_lens, k_max, out, idx, tail_mass, workspace,
                       workspace_bytes, stream, nullptr, &cert);
}

tka_status topk_attn_decode(const tka_shape *shape, const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *seq_lens, int32_t k, float *out, int32_t *idx, float *tail_mass,
                            void *workspace, size_t workspace_bytes, tka_stream_t stream) {
    return topk_attn_decode_staged(shape, q, k_cache, v_cache, seq_lens, k, out, idx, tail_mass, workspace,
                                   workspace_bytes, stream, nullptr);
}

tka_status topk_block_pool_keys(const tka_shape *shape, const void *k_cache, const int32_t *seq_lens,
                                int32_t block_size, float *block_keys, tka_stream_t stream) {
    if (!shape) return TKA_ERR_INVALID_ARG;
    if (shape->B < 1 || shape->Hkv < 1 || shape->L_max < 1 || block_size < 1) return TKA_ERR_INVALID_ARG;
    if (shape->d != kHeadDim) return TKA_ERR_UNSUPPORTED;
    if (shape->dtype != TKA_F32 && shape->dtype != TKA_BF16) return TKA_ERR_UNSUPPORTED;
    if (shape->L_max > kMaxLen || (long long)shape->B * shape->Hkv > 65535) return TKA_ERR_UNSUPPORTED;
    if (!k_cache || !seq_lens || !block_keys) return TKA_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(block_keys, 16) || !aligned(seq_lens, 4)) return TKA_ERR_INVALID_ARG;
    const int nblk_max = (shape->L_max + block_size - 1) / block_size;
    if (nblk_max > (1 << 20)) return TKA_ERR_UNSUPPORTED;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return TKA_ERR_CUDA;
    BlockPoolParams p;
    p.status = dev->status;
    p.k = k_cache;
    p.seq_lens = seq_lens;
    p.block_keys = block_keys;
    p.B = shape->B; p.Hkv = shape->Hkv; p.L_max = shape->L_max; p.block_size = block_size;
    p.nblk_max = nblk_max; p.dtype = shape->dtype;
    if (launch_block_pool(p, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return TKA_ERR_CUDA;
    return TKA_OK;
}

size_t topk_block_attn_workspace_size(const tka_shape *shape, int32_t block_size, int32_t top_blocks) {
    if (check_block_args(shape, block_size, top_blocks) != TKA_OK) return 0;
    return block_layout(shape, block_size, top_blocks).total;
}

tka_status topk_block_attn_decode(const tka_shape *shape, const void *q, const void *k_cache, const void *v_cache,
                                  const float *block_keys, const int32_t *seq_lens, int32_t block_size,
                                  int32_t top_blocks, float *out, int32_t *block_idx, void *workspace,
                                  size_t workspace_bytes, tka_stream_t stream) {
    tka_status st = check_block_args(shape, block_size, top_blocks);
    if (st != TKA_OK) return st;
    if (!q || !k_cache || !v_cache || !block_keys || !seq_lens || !out) return TKA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(block_keys, 16) ||
        !aligned(out, 16) || !aligned(seq_lens, 4) || (block_idx && !aligned(block_idx, 4)))
        return TKA_ERR_INVALID_ARG;
    const BlockLayout L = block_layout(shape, block_size, top_blocks);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < L.total) return TKA_ERR_WORKSPACE;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return TKA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    const int G = shape->Hq / shape->Hkv;
    const int nblk_max = (shape->L_max + block_size - 1) / block_size;
    int32_t *bidx = block_idx ? block_idx : reinterpret_cast<int32_t *>(ws + L.block_idx);
    unsigned *counters = reinterpret_cast<unsigned *>(ws + L.counters);

    BlockSelectParams sp;
    sp.status = dev->status;
    sp.q = q;
    sp.block_keys = block_keys;
    sp.seq_lens = seq_lens;
    sp.B = shape->B; sp.Hq = shape->Hq; sp.Hkv = shape->Hkv; sp.G = G; sp.L_max = shape->L_max;
    sp.block_size = block_size; sp.nblk_max = nblk_max; sp.top_blocks = top_blocks; sp.dtype = shape->dtype;
    sp.scale = resolve_scale(shape);
    sp.bscore = reinterpret_cast<float *>(ws + L.bscore);
    sp.block_idx = bidx;
    sp.counters = counters;
    if (launch_block_select(sp, s) != cudaSuccess) return TKA_ERR_CUDA;

    BlockAttnParams ap;
    ap.status = dev->status;
    ap.q = q; ap.k = k_cache; ap.v = v_cache;
    ap.seq_lens = seq_lens;
    ap.block_idx = bidx;
    ap.B = shape->B; ap.Hq = shape->Hq; ap.Hkv = shape->Hkv; ap.G = G; ap.L_max = shape->L_max;
    ap.block_size = block_size; ap.top_blocks = top_blocks; ap.dtype = shape->dtype;
    ap.scale = sp.scale;
    ap.part_ml = reinterpret_cast<float4 *>(ws + L.part_ml);
    ap.part_acc = reinterpret_cast<float *>(ws + L.part_acc);
    ap.counters = counters;
    ap.out = out;
    ap.max_polls = g_wait_polls.load(std::memory_order_relaxed);
    if (launch_block_attn(ap, k_cache, dev->num_sms, s) != cudaSuccess) return TKA_ERR_CUDA;
    return TKA_OK;
}

size_t topk_hisa_attn_workspace_size(const tka_shape *shape, int32_t block_size, int32_t top_blocks, int32_t k) {
    if (check_hisa_args(shape, block_size, top_blocks, k) != TKA_OK) return 0;
    return hisa_layout(shape, block_size, top_blocks, k).total;
}

tka_status topk_hisa_attn_decode(const tka_shape *shape, const void *q, const void *k_cache, const void *v_cache,
                                 const float *block_keys, const int32_t *seq_lens, int32_t block_size,
                                 int32_t top_blocks, int32_t k, float *out, int32_t *idx, float *tail_mass,
                                 int32_t *block_idx, void *workspace, size_t workspace_bytes, tka_stream_t stream) {
    tka_status st = check_hisa_args(shape, block_size, top_blocks, k);
    if (st != TKA_OK) return st;
    if (!q || !k_cache || !v_cache || !block_keys || !seq_lens || !out || !idx) return TKA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(block_keys, 16) ||
        !aligned(out, 16) || !aligned(idx, 4) || !aligned(seq_lens, 4) || (tail_mass && !aligned(tail_mass, 4)) ||
        (block_idx && !aligned(block_idx, 4)))
        return TKA_ERR_INVALID_ARG;
    const HisaLayout L = hisa_layout(shape, block_size, top_blocks, k);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < L.total) return TKA_ERR_WORKSPACE;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return TKA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    const int G = shape->Hq / shape->Hkv;
    const int rows = shape->B * shape->Hq;
    const int nblk_max = (shape->L_max + block_size - 1) / block_size;
    int32_t *bidx = block_idx ? block_idx : reinterpret_cast<int32_t *>(ws + L.block_idx);
    int32_t *row_len = reinterpret_cast<int32_t *>(ws + L.row_len);
    unsigned *counters = reinterpret_cast<unsigned *>(ws + L.counters);
    const float scale = resolve_scale(shape);

    // 1. blocks: every block competes for the top_blocks slots
    BlockSelectParams bp;
    bp.status = dev->status;
    bp.q = q;
    bp.block_keys = block_keys;
    bp.seq_lens = seq_lens;
    bp.B = shape->B; bp.Hq = shape->Hq; bp.Hkv = shape->Hkv; bp.G = G; bp.L_max = shape->L_max;
    bp.block_size = block_size; bp.nblk_max = nblk_max; bp.top_blocks = top_blocks; bp.dtype = shape->dtype;
    bp.scale = scale;
    bp.bscore = reinterpret_cast<float *>(ws + L.bscore);
    bp.block_idx = bidx;
    bp.counters = nullptr;
    bp.force_last = 0;
    if (launch_block_select(bp, s) != cudaSuccess) return TKA_ERR_CUDA;

    // 2. token scores inside the kept blocks
    HisaScoreParams hp;
    hp.status = dev->status;
    hp.q = q; hp.k = k_cache;
    hp.seq_lens = seq_lens;
    hp.block_idx = bidx;
    hp.B = shape->B; hp.Hq = shape->Hq; hp.Hkv = shape->Hkv; hp.G = G; hp.L_max = shape->L_max;
    hp.block_size = block_size; hp.top_blocks = top_blocks; hp.ldc = L.ldc; hp.dtype = shape->dtype;
    hp.scale = scale;
    hp.cscore = reinterpret_cast<float *>(ws + L.cscore);
    hp.row_len = row_len;
    if (launch_hisa_scores(hp, s) != cudaSuccess) return TKA_ERR_CUDA;

    // 3. the top k candidates (candidate order is position order)
    SelectParams se;
    se.status = dev->status;
    se.scores = hp.cscore;
    se.seq_lens = seq_lens;
    se.B = shape->B; se.Q = 1; se.Hq = shape->Hq; se.L_max = shape->L_max; se.ld = L.ldc; se.k = k;
    se.idx = idx;
    se.w = reinterpret_cast<float *>(ws + L.weights);
    se.stats = reinterpret_cast<float4 *>(ws + L.stats);
    se.tail = tail_mass;
    se.counters = counters;
    se.row_len = row_len;
    if (launch_select(se, s) != cudaSuccess) return TKA_ERR_CUDA;

    // 4. softmax over the kept tokens and P.V; candidate indices become positions
    GatherParams gp;
    gp.status = dev->status;
    gp.v = v_cache;
    gp.seq_lens = seq_lens;
    gp.B = shape->B; gp.Q = 1; gp.Hq = shape->Hq; gp.Hkv = shape->Hkv; gp.G = G;
    gp.L_max = shape->L_max; gp.k = k; gp.dtype = shape->dtype;
    gp.idx = idx;
    gp.w = se.w;
    gp.stats = se.stats;
    gp.partial = reinterpret_cast<float *>(ws + L.partial);
    gp.counters = counters;
    gp.out = out;
    gp.kcount = row_len;
    gp.cblock = bidx;
    gp.crow_len = row_len;
    gp.idx_out = idx;
    gp.cbs = block_size;
    gp.cstride = top_blocks;
    int splits = (dev->num_sms * 8) / rows;
    if (splits > L.max_splits) splits = L.max_splits;
    if (splits < 1) splits = 1;
    gp.per_split = (k + splits - 1) / splits;
    gp.splits = (k + gp.per_split - 1) / gp.per_split;
    if (launch_gather(gp, s) != cudaSuccess) return TKA_ERR_CUDA;
    return TKA_OK;
}

size_t topk_indexer_attn_workspace_size(const tka_shape *shape, int32_t H_I, int32_t d_I, int32_t k) {
    if (check_indexer_args(shape, H_I, d_I, k) != TKA_OK) return 0;
    return indexer_layout(shape, k, H_I, d_I).total;
}

tka_status topk_indexer_attn_decode(const tka_shape *shape, const void *q, const void *k_cache, const void *v_cache,
                                    const void *q_idx, const float *w_idx, const void *k_idx, int32_t H_I,
                                    int32_t d_I, const int32_t *seq_lens, int32_t k, float *out, int32_t *idx,
                                    void *workspace, size_t workspace_bytes, tka_stream_t stream) {
    tka_status st = check_indexer_args(shape, H_I, d_I, k);
    if (st != TKA_OK) return st;
    if (!q || !k_cache || !v_cache || !q_idx || !w_idx || !k_idx || !seq_lens || !out || !idx)
        return TKA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q_idx, 16) ||
        !aligned(k_idx, 16) || !aligned(w_idx, 4) || !aligned(out, 16) || !aligned(idx, 4) || !aligned(seq_lens, 4))
        return TKA_ERR_INVALID_ARG;
    const IndexerLayout L = indexer_layout(shape, k, H_I, d_I);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < L.total) return TKA_ERR_WORKSPACE;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return TKA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    const int G = shape->Hq / shape->Hkv;
    const int units = shape->B * shape->Q;

    // 1. indexer scores of every visible token, per query position
    IndexerScoreParams ip;
    ip.status = dev->status;
    ip.q_idx = q_idx; ip.w_idx = w_idx; ip.k_idx = k_idx;
    ip.seq_lens = seq_lens;
    ip.B = shape->B; ip.Q = shape->Q; ip.Hkv = shape->Hkv; ip.L_max = shape->L_max;
    ip.H_I = H_I; ip.d_I = d_I; ip.ld = L.ld; ip.dtype = shape->dtype;
    ip.scores = reinterpret_cast<float *>(ws + L.iscores);
    ip.attn_counters = reinterpret_cast<unsigned *>(ws + L.attn_counters);
    if (indexer_tc(shape, H_I, d_I)) {
        ScoreTcParams tp;
        tp.status = dev->status;
        tp.seq_lens = seq_lens;
        tp.scores = reinterpret_cast<float *>(ws + L.raw);
        tp.B = shape->B; tp.Q = shape->Q; tp.Hq = H_I; tp.Hkv = 1; tp.G = H_I;
        tp.L_max = shape->L_max; tp.ld = L.ld; tp.NQ = shape->Q * H_I;
        tp.scale = 1.f;
        tp.max_polls = g_wait_polls.load(std::memory_order_relaxed);
        if (launch_score_tc(tp, q_idx, k_idx, dev->num_sms, s, ScoreTcHook{}) != cudaSuccess) return TKA_ERR_CUDA;
        if (launch_indexer_combine(ip, tp.scores, s) != cudaSuccess) return TKA_ERR_CUDA;
    } else if (launch_indexer_scores(ip, dev->num_sms, s) != cudaSuccess) {
        return TKA_ERR_CUDA;
    }

    // 2. the top k tokens of each query position (one row per position)
    SelectParams se;
    se.status = dev->status;
    se.scores = ip.scores;
    se.seq_lens = seq_lens;
    se.B = shape->B; se.Q = shape->Q; se.Hq = 1; se.L_max = shape->L_max; se.ld = L.ld; se.k = k;
    se.idx = idx;
    se.w = reinterpret_cast<float *>(ws + L.weights);
    se.stats = reinterpret_cast<float4 *>(ws + L.stats);
    se.tail = nullptr;
    se.counters = reinterpret_cast<unsigned *>(ws + L.sel_counters);
    if (launch_select(se, s) != cudaSuccess) return TKA_ERR_CUDA;

    // 3. every head attends over its position's kept tokens with exact scores
    IndexerAttnParams ap;
    ap.status = dev->status;
    ap.q = q; ap.kc = k_cache; ap.vc = v_cache;
    ap.seq_lens = seq_lens;
    ap.idx = idx;
    ap.B = shape->B; ap.Q = shape->Q; ap.Hq = shape->Hq; ap.Hkv = shape->Hkv; ap.G = G;
    ap.L_max = shape->L_max; ap.k = k; ap.dtype = shape->dtype;
    ap.scale = resolve_scale(shape);
    ap.part_ml = reinterpret_cast<float4 *>(ws + L.part_ml);
    ap.part_acc = reinterpret_cast<float *>(ws + L.part_acc);
    ap.counters = ip.attn_counters;
    ap.out = out;
    int splits = (dev->num_sms * 8) / (units * shape->Hkv);
    if (splits > L.max_splits) splits = L.max_splits;
    if (splits < 1) splits = 1;
    ap.per_split = (k + splits - 1) / splits;
    ap.splits = (k + ap.per_split - 1) / ap.per_split;
    if (launch_indexer_attn(ap, s) != cudaSuccess) return TKA_ERR_CUDA;
    return TKA_OK;
}

tka_status topk_attn_device_status(tka_stream_t stream, uint32_t *bits) {
    if (!bits) return TKA_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return TKA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned v = 0u;
    if (cudaStreamSynchronize(s) != cudaSuccess) return TKA_ERR_CUDA;
    if (cudaMemcpy(&v, dev->status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return TKA_ERR_CUDA;
    if (cudaMemset(dev->status, 0, sizeof v) != cudaSuccess) return TKA_ERR_CUDA;
    *bits = v;
    return TKA_OK;
}

tka_status topk_attn_last_device_status(tka_stream_t stream) {
    uint32_t bits = 0u;
    const tka_status st = topk_attn_device_status(stream, &bits);
    if (st != TKA_OK) return st;
    if (bits & TKA_DEV_TIMEOUT) return TKA_ERR_TIMEOUT;
    if (bits & (TKA_DEV_BAD_SEQ_LEN | TKA_DEV_BAD_PAGE)) return TKA_ERR_INVALID_ARG;
    if (bits & TKA_DEV_INTERNAL) return TKA_ERR_CUDA;
    return TKA_OK;
}

void topk_attn_debug_set_wait_limit(uint32_t polls) { g_wait_polls.store(polls, std::memory_order_relaxed); }

const char *topk_attn_status_string(tka_status status) {
    switch (status) {
        case TKA_OK: return "TKA_OK";
        case TKA_ERR_INVALID_ARG: return "TKA_ERR_INVALID_ARG";
        case TKA_ERR_UNSUPPORTED: return "TKA_ERR_UNSUPPORTED";
        case TKA_ERR_WORKSPACE: return "TKA_ERR_WORKSPACE";
        case TKA_ERR_CUDA: return "TKA_ERR_CUDA";
        case TKA_ERR_TIMEOUT: return "TKA_ERR_TIMEOUT";
    }
    return "unknown tka_status";
}

}  // extern "C"
