// Select step: for one query row, the k highest-scoring visible positions
// (ties at the k-th score go to the lower position), in ascending position
// order, together with the softmax statistics the attention step needs.
//
// "Top-K Selection: retaining the K historical positions with the highest
// scores" ("Evolution of Sparse Attention in Long-Context LLMs", section 2);
// the discarded mass is the Top-k tail mass of "A Mathematical Theory of
// Top-k Sparse Attention via Total Variation Distance" (abstract).
//
// One CTA per row.  Scores are compared as order-preserving uint32 keys, so
// the k-th largest is found exactly by radix selection on the key bits.  Pass
// 1 builds the histogram of the top 11 key bits and the row maximum; the bin
// holding the k-th key is read off the histogram.  Pass 2 compacts, in
// position order, the keys of higher bins (certainly kept) and collects the
// keys of that bin as candidates in shared memory; the candidates are
// resolved exactly there (radix on the low 21 bits, ties to the lower
// position) and the two ascending lists are merged.  The row is read from L2
// (the scorer keeps the K stream out of L2), with 8 float4 loads per thread
// in flight.  A boundary bin with more candidates than fit falls back to
// three histogram passes (11 + 11 + 10 bits) and an ordered compaction pass.
// The pass that writes the output also forms Z_k = sum_kept e^{s-m} and
// Z_tail = sum_dropped e^{s-m}; the tail mass is Z_tail / (Z_k + Z_tail),
// formed from the dropped terms directly.
#include "common.cuh"
#include "kernels.h"

namespace tka {

namespace {

constexpr int kSelectThreads = 512;
constexpr int kCandCap = 4096;

__device__ __forceinline__ float key_to_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Exclusive prefix sum of one value per thread over the block; *total gets
// the block sum.  `tmp` holds >= 32 words of shared memory.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *tmp, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < nw ? tmp[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        tmp[lane] = s;
    }
    __syncthreads();
    *total = tmp[nw - 1];
    return (warp ? tmp[warp - 1] : 0u) + x - v;
}

// Finds the bin holding the need-th largest element of a histogram whose
// bins are ordered by key: writes the bin and the count of elements in higher
// bins to *out_bin / *out_above.  Requires 1 <= need <= total count.
__device__ void find_bin(const uint32_t *hist, int nbins, uint32_t need, uint32_t *tmp, uint32_t *out_bin,
                         uint32_t *out_above) {
    const int per = (nbins + blockDim.x - 1) / blockDim.x;
    const int p0 = threadIdx.x * per;  // descending positions [p0, p0 + per)
    uint32_t local = 0;
    for (int p = p0; p < p0 + per && p < nbins; p++) local += hist[nbins - 1 - p];
    uint32_t total;
    uint32_t cum = block_excl_scan(local, tmp, &total);
    for (int p = p0; p < p0 + per && p < nbins; p++) {
        const uint32_t h = hist[nbins - 1 - p];
        if (cum < need && cum + h >= need) {
            *out_bin = (uint32_t)(nbins - 1 - p);
            *out_above = cum;
        }
        cum += h;
    }
    __syncthreads();
}

constexpr int kBatch = 8;  // float4 loads in flight per thread

// Calls f(i, s[i]) for every i < n, 4 * kBatch elements per thread per round.
template <typename F>
__device__ __forceinline__ void visit_row(const float *s, int n, F &&f) {
    const int n4 = n >> 2;
    const float4 *s4 = reinterpret_cast<const float4 *>(s);
    const int stride = blockDim.x;
    int i = threadIdx.x;
    for (; i + (kBatch - 1) * stride < n4; i += kBatch * stride) {
        float4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; u++) v[u] = __ldcg(s4 + i + u * stride);
#pragma unroll
        for (int u = 0; u < kBatch; u++) {
            const int e = 4 * (i + u * stride);
            f(e, v[u].x);
            f(e + 1, v[u].y);
            f(e + 2, v[u].z);
            f(e + 3, v[u].w);
        }
    }
    for (; i < n4; i += stride) {
        const float4 v = __ldcg(s4 + i);
        f(4 * i, v.x);
        f(4 * i + 1, v.y);
        f(4 * i + 2, v.z);
        f(4 * i + 3, v.w);
    }
    for (int j = 4 * n4 + threadIdx.x; j < n; j += stride) f(j, __ldcg(s + j));
}

// Loads 4 consecutive positions i0..i0+3 (zeros past n).
__device__ __forceinline__ void load4(const float *s, int i0, int n, float (&x)[4]) {
    if (i0 + 3 < n) {
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(s + i0));
        x[0] = v.x;
        x[1] = v.y;
        x[2] = v.z;
        x[3] = v.w;
    } else {
#pragma unroll
        for (int j = 0; j < 4; j++) x[j] = i0 + j < n ? __ldcg(s + i0 + j) : 0.f;
    }
}

struct SelectSmem {
    uint32_t *hist;  // [2048]
    uint32_t *tmp;   // [32]
    float *red;      // [32]
    uint32_t *scal;  // [2]: bin, above
};

// Writes stats, tail and counter of a finished row.
__device__ __forceinline__ void finish_row(const SelectParams &p, int row, float m, float zk, float zt,
                                           uint32_t written, uint32_t kept, const SelectSmem &sm) {
    zk = block_sum(zk, sm.red);
    __syncthreads();
    zt = block_sum(zt, sm.red);
    if (threadIdx.x == 0) {
        if (written != kept) raise_status(p.status, TKA_DEV_INTERNAL);
        p.stats[row] = make_float4(m, zk, zt, 0.f);
        if (p.tail) p.tail[row] = zt / (zk + zt);
        p.counters[row] = 0u;
    }
}

// k >= visible keys: every position is kept, in order.
__device__ void select_all(const SelectParams &p, int row, int vis, float m, const SelectSmem &sm) {
    const float *s = p.scores + (size_t)row * p.ld;
    int32_t *idx = p.idx + (size_t)row * p.k;
    float *wv = p.w + (size_t)row * p.k;
    float zk = 0.f;
    visit_row(s, vis, [&](int i, float x) {
        const float e = __expf(x - m);
        idx[i] = i;
        wv[i] = e;
        zk += e;
    });
    for (int j = vis + threadIdx.x; j < p.k; j += blockDim.x) idx[j] = -1;
    finish_row(p, row, m, zk, 0.f, vis, vis, sm);
}

// Three histogram passes and an ordered compaction pass (too many candidates
// in the boundary bin).
__device__ void select_multipass(const SelectParams &p, int row, int vis, const SelectSmem &sm) {
    const float *s = p.scores + (size_t)row * p.ld;
    const int k = p.k;
    uint32_t *hist = sm.hist;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    float m = -INFINITY;
    visit_row(s, vis, [&](int, float x) {
        m = fmaxf(m, x);
        atomicAdd(&hist[order_key(x) >> 21], 1u);
    });
    m = block_max(m, sm.red);
    __syncthreads();
    find_bin(hist, 2048, (uint32_t)k, sm.tmp, &sm.scal[0], &sm.scal[1]);
    const uint32_t b1 = sm.scal[0];
    uint32_t above = sm.scal[1];
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    visit_row(s, vis, [&](int, float x) {
        const uint32_t key = order_key(x);
        if ((key >> 21) == b1) atomicAdd(&hist[(key >> 10) & 0x7ffu], 1u);
    });
    __syncthreads();
    find_bin(hist, 2048, (uint32_t)k - above, sm.tmp, &sm.scal[0], &sm.scal[1]);
    const uint32_t b2 = sm.scal[0];
    above += sm.scal[1];
    const uint32_t pre = (b1 << 11) | b2;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    visit_row(s, vis, [&](int, float x) {
        const uint32_t key = order_key(x);
        if ((key >> 10) == pre) atomicAdd(&hist[key & 0x3ffu], 1u);
    });
    __syncthreads();
    find_bin(hist, 1024, (uint32_t)k - above, sm.tmp, &sm.scal[0], &sm.scal[1]);
    const uint32_t b3 = sm.scal[0];
    above += sm.scal[1];
    const uint32_t T = (pre << 10) | b3, n_eq = hist[b3], r_eq = (uint32_t)k - above;
    const bool rank_ties = n_eq != r_eq;

    int32_t *idx = p.idx + (size_t)row * k;
    float *wv = p.w + (size_t)row * k;
    uint32_t base_sel = 0u, base_eq = 0u;
    float zk = 0.f, zt = 0.f;
    for (int tile = 0; tile < vis; tile += 4 * blockDim.x) {
        const int i0 = tile + 4 * threadIdx.x;
        float x[4];
        load4(s, i0, vis, x);
        uint32_t key[4], n_eq_t = 0u;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            key[j] = order_key(x[j]);
            if (i0 + j < vis && key[j] == T) n_eq_t++;
        }
        uint32_t eq_total = 0u, eq_rank = base_eq;
        if (rank_ties) eq_rank += block_excl_scan(n_eq_t, sm.tmp, &eq_total);
        bool sel[4];
        uint32_t n_sel_t = 0u;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            bool v = i0 + j < vis;
            if (v) v = key[j] == T ? (!rank_ties || eq_rank++ < r_eq) : key[j] > T;
            sel[j] = v;
            n_sel_t += v;
        }
        uint32_t sel_total;
        uint32_t pos = base_sel + block_excl_scan(n_sel_t, sm.tmp, &sel_total);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            if (i0 + j >= vis) continue;
            const float e = __expf(x[j] - m);
            if (sel[j]) {
                if (pos < (uint32_t)k) {  // always true unless the search above is wrong
                    idx[pos] = i0 + j;
                    wv[pos] = e;
                }
                pos++;
                zk += e;
            } else {
                zt += e;
            }
        }
        base_sel += sel_total;
        base_eq += eq_total;
    }
    finish_row(p, row, m, zk, zt, base_sel, (uint32_t)k, sm);
}

// Number of elements of the ascending array a[0..n) that are < x.
__device__ __forceinline__ int lower_bound(const int32_t *a, int n, int32_t x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] < x)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(kSelectThreads) select_topk(SelectParams p) {
    extern __shared__ uint32_t dyn[];
    SelectSmem sm;
    sm.hist = dyn;
    sm.tmp = dyn + 2048;
    sm.red = reinterpret_cast<float *>(dyn + 2048 + 32);
    sm.scal = dyn + 2048 + 64;
    int32_t *a_idx = reinterpret_cast<int32_t *>(dyn + 2048 + 64 + 8);  // [k]
    float *a_w = reinterpret_cast<float *>(a_idx + p.k);                 // [k]
    uint32_t *c_key = reinterpret_cast<uint32_t *>(a_w + p.k);           // [kCandCap]
    int32_t *c_idx = reinterpret_cast<int32_t *>(c_key + kCandCap);      // [kCandCap]

    const int row = blockIdx.x;
    const int b = row / (p.Q * p.Hq), qpos = (row / p.Hq) % p.Q;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) {
        if (threadIdx.x == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    const int vis = visible_keys(seq_len, p.Q, qpos);
    const int k = p.k;
    const float *s = p.scores + (size_t)row * p.ld;

    // pass 1: histogram of the top 11 key bits and the row maximum
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) sm.hist[i] = 0u;
    __syncthreads();
    const bool count = k < vis;
    float m = -INFINITY;
    visit_row(s, vis, [&](int, float x) {
        m = fmaxf(m, x);
        if (count) atomicAdd(&sm.hist[order_key(x) >> 21], 1u);
    });
    m = block_max(m, sm.red);
    if (!count) {
        select_all(p, row, vis, m, sm);
        return;
    }
    __syncthreads();
    find_bin(sm.hist, 2048, (uint32_t)k, sm.tmp, &sm.scal[0], &sm.scal[1]);
    const uint32_t b1 = sm.scal[0], above = sm.scal[1], ncand = sm.hist[b1];
    if (ncand > (uint32_t)kCandCap) {
        __syncthreads();
        select_multipass(p, row, vis, sm);
        return;
    }

    // pass 2: keys of higher bins go to list A (in position order), keys of
    // bin b1 to the candidates; kBatch tiles of loads are issued before
    // their prefix sums
    uint32_t base_a = 0u, base_c = 0u;
    float zk = 0.f, zt = 0.f;
    const int tile_len = 4 * blockDim.x;
    for (int base = 0; base < vis; base += kBatch * tile_len) {
        float x[kBatch][4];
#pragma unroll
        for (int u = 0; u < kBatch; u++) load4(s, base + u * tile_len + 4 * threadIdx.x, vis, x[u]);
#pragma unroll
        for (int u = 0; u < kBatch; u++) {
            const int i0 = base + u * tile_len + 4 * threadIdx.x;
            if (base + u * tile_len >= vis) break;  // uniform across the block
            uint32_t key[4], cnt = 0u;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                key[j] = order_key(x[u][j]);
                if (i0 + j < vis) cnt += (key[j] >> 21) > b1 ? 1u : ((key[j] >> 21) == b1 ? 0x10000u : 0u);
            }
            uint32_t tot;
            const uint32_t ex = block_excl_scan(cnt, sm.tmp, &tot);
            uint32_t pa = base_a + (ex & 0xffffu), pc = base_c + (ex >> 16);
#pragma unroll
            for (int j = 0; j < 4; j++) {
                if (i0 + j >= vis) continue;
                const uint32_t bin = key[j] >> 21;
                if (bin > b1) {
                    const float e = __expf(x[u][j] - m);
                    if (pa < above) {  // always true unless the histogram is wrong
                        a_idx[pa] = i0 + j;
                        a_w[pa] = e;
                    }
                    pa++;
                    zk += e;
                } else if (bin == b1) {
                    if (pc < ncand) {
                        c_key[pc] = key[j];
                        c_idx[pc] = i0 + j;
                    }
                    pc++;
                } else {
                    zt += __expf(x[u][j] - m);
                }
            }
            base_a += tot & 0xffffu;
            base_c += tot >> 16;
        }
    }
    if (base_a != above || base_c != ncand) {
        // the two passes disagree (a library bug); recompute safely
        if (threadIdx.x == 0) raise_status(p.status, TKA_DEV_INTERNAL);
        __syncthreads();
        select_multipass(p, row, vis, sm);
        return;
    }
    __syncthreads();

    // resolve the boundary bin: r of its ncand keys are kept
    const uint32_t r = (uint32_t)k - above;
    uint32_t *hist = sm.hist;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    for (uint32_t c = threadIdx.x; c < ncand; c += blockDim.x) atomicAdd(&hist[(c_key[c] >> 10) & 0x7ffu], 1u);
    __syncthreads();
    find_bin(hist, 2048, r, sm.tmp, &sm.scal[0], &sm.scal[1]);
    const uint32_t b2 = sm.scal[0];
    uint32_t gt = sm.scal[1];
    const uint32_t pre = (b1 << 11) | b2;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    for (uint32_t c = threadIdx.x; c < ncand; c += blockDim.x)
        if ((c_key[c] >> 10) == pre) atomicAdd(&hist[c_key[c] & 0x3ffu], 1u);
    __syncthreads();
    find_bin(hist, 1024, r - gt, sm.tmp, &sm.scal[0], &sm.scal[1]);
    const uint32_t b3 = sm.scal[0];
    gt += sm.scal[1];
    const uint32_t T = (pre << 10) | b3, n_eq = hist[b3], r_eq = r - gt;
    const bool rank_ties = n_eq != r_eq;

    // compact the chosen candidates in place (candidates are in position order)
    uint32_t base_b = 0u, base_eq = 0u;
    for (uint32_t c0 = 0; c0 < ncand; c0 += blockDim.x) {
        const uint32_t c = c0 + threadIdx.x;
        const bool have = c < ncand;
        const uint32_t key = have ? c_key[c] : 0u;
        const int32_t pos = have ? c_idx[c] : 0;
        uint32_t eq_total = 0u, eq_rank = base_eq;
        if (rank_ties) eq_rank += block_excl_scan(have && key == T ? 1u : 0u, sm.tmp, &eq_total);
        const bool chosen = have && (key == T ? (!rank_ties || eq_rank < r_eq) : key > T);
        uint32_t tot;
        const uint32_t dst = base_b + block_excl_scan(chosen ? 1u : 0u, sm.tmp, &tot);  // ends with a barrier
        if (have) {
            const float e = __expf(key_to_float(key) - m);
            if (chosen) {
                c_idx[dst] = pos;
                reinterpret_cast<float *>(c_key)[dst] = e;
                zk += e;
            } else {
                zt += e;
            }
        }
        __syncthreads();
        base_b += tot;
        base_eq += eq_total;
    }
    // merge the two ascending lists into the output
    int32_t *idx = p.idx + (size_t)row * k;
    float *wv = p.w + (size_t)row * k;
    const float *b_w = reinterpret_cast<const float *>(c_key);
    const int na = (int)above, nb = (int)base_b;
    for (int i = threadIdx.x; i < na; i += blockDim.x) {
        const int pos = i + lower_bound(c_idx, nb, a_idx[i]);
        idx[pos] = a_idx[i];
        wv[pos] = a_w[i];
    }
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
        const int pos = i + lower_bound(a_idx, na, c_idx[i]);
        idx[pos] = c_idx[i];
        wv[pos] = b_w[i];
    }
    finish_row(p, row, m, zk, zt, above + base_b, (uint32_t)k, sm);
}

}  // namespace

size_t select_smem_bytes(int k) {
    return (size_t)(2048 + 64 + 8) * 4 + (size_t)k * 8 + (size_t)kCandCap * 8;
}

cudaError_t launch_select(const SelectParams &p, cudaStream_t stream) {
    const int rows = p.B * p.Q * p.Hq;
    const size_t smem = select_smem_bytes(p.k);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(select_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    select_topk<<<rows, kSelectThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tka
