// Select step: for one query row, the k highest-scoring visible positions
// (ties at the k-th score go to the lower position), in ascending position
// order, together with the softmax statistics the attention step needs.
//
// "Top-K Selection: retaining the K historical positions with the highest
// scores" ("Evolution of Sparse Attention in Long-Context LLMs", section 2);
// the discarded mass is the Top-k tail mass of "A Mathematical Theory of
// Top-k Sparse Attention via Total Variation Distance" (abstract).
//
// One CTA per row.  Scores are mapped to order-preserving uint32 keys and the
// k-th largest key is found exactly by a three-level radix select (11 + 11 +
// 10 bits), each level one histogram pass over the row (the row is read from
// L2: the score workspace of a decode step is small enough to stay resident).
// A final pass walks the row in position order and compacts the kept
// positions with block-wide prefix sums, so the output is ascending and a tie
// at the threshold key is resolved by position.  The same pass computes
// Z_k = sum_kept e^{s-m} and Z_tail = sum_dropped e^{s-m}, so the tail mass
// Z_tail / (Z_k + Z_tail) is formed from the dropped terms directly rather
// than as a difference.
#include "common.cuh"
#include "kernels.h"

namespace tka {

namespace {

constexpr int kSelectThreads = 512;

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

// Calls f(i, s[i]) for every i < n, 16 elements per thread per round.
template <typename F>
__device__ __forceinline__ void visit_row(const float *s, int n, F &&f) {
    const int n4 = n >> 2;
    const float4 *s4 = reinterpret_cast<const float4 *>(s);
    const int stride = blockDim.x;
    int i = threadIdx.x;
    for (; i + 3 * stride < n4; i += 4 * stride) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; u++) v[u] = __ldcg(s4 + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; u++) {
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

__global__ void __launch_bounds__(kSelectThreads) select_topk(SelectParams p) {
    __shared__ uint32_t hist[2048];
    __shared__ uint32_t tmp[32];
    __shared__ float red[32];
    __shared__ uint32_t s_bin, s_above;

    const int row = blockIdx.x;
    const int b = row / (p.Q * p.Hq), qpos = (row / p.Hq) % p.Q;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) {
        if (threadIdx.x == 0) raise_status(p.status, TKA_DEV_BAD_SEQ_LEN);
        return;
    }
    const int vis = visible_keys(seq_len, p.Q, qpos);
    const float *s = p.scores + (size_t)row * p.ld;
    const int k = p.k;
    const bool take_all = k >= vis;

    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
    __syncthreads();

    // pass 1: row max and histogram of the top 11 key bits
    float m = -INFINITY;
    visit_row(s, vis, [&](int, float x) {
        m = fmaxf(m, x);
        if (!take_all) atomicAdd(&hist[order_key(x) >> 21], 1u);
    });
    m = block_max(m, red);

    uint32_t T = 0u, n_eq = 0u, r_eq = 0u;  // threshold key, its multiplicity, how many of those to keep
    if (!take_all) {
        __syncthreads();
        find_bin(hist, 2048, (uint32_t)k, tmp, &s_bin, &s_above);
        const uint32_t b1 = s_bin;
        uint32_t above = s_above;
        for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        // pass 2: next 11 bits among keys in bin b1
        visit_row(s, vis, [&](int, float x) {
            const uint32_t key = order_key(x);
            if ((key >> 21) == b1) atomicAdd(&hist[(key >> 10) & 0x7ffu], 1u);
        });
        __syncthreads();
        find_bin(hist, 2048, (uint32_t)k - above, tmp, &s_bin, &s_above);
        const uint32_t b2 = s_bin;
        above += s_above;
        const uint32_t pre = (b1 << 11) | b2;
        for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        // pass 3: last 10 bits among keys matching the 22-bit prefix
        visit_row(s, vis, [&](int, float x) {
            const uint32_t key = order_key(x);
            if ((key >> 10) == pre) atomicAdd(&hist[key & 0x3ffu], 1u);
        });
        __syncthreads();
        find_bin(hist, 1024, (uint32_t)k - above, tmp, &s_bin, &s_above);
        const uint32_t b3 = s_bin;
        above += s_above;
        T = (pre << 10) | b3;
        n_eq = hist[b3];
        r_eq = (uint32_t)k - above;
    }
    const bool rank_ties = !take_all && n_eq != r_eq;

    // pass 4: ordered compaction, 4 consecutive positions per thread per tile
    int32_t *idx = p.idx + (size_t)row * k;
    float *wv = p.w + (size_t)row * k;
    uint32_t base_sel = 0u, base_eq = 0u;
    float zk = 0.f, zt = 0.f;
    for (int tile = 0; tile < vis; tile += 4 * blockDim.x) {
        const int i0 = tile + 4 * threadIdx.x;
        float x[4];
        if (i0 + 3 < vis) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(s + i0));
            x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
        } else {
#pragma unroll
            for (int j = 0; j < 4; j++) x[j] = i0 + j < vis ? __ldcg(s + i0 + j) : 0.f;
        }
        uint32_t key[4], n_eq_t = 0u;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            key[j] = order_key(x[j]);
            if (i0 + j < vis && key[j] == T) n_eq_t++;
        }
        uint32_t eq_total = 0u, eq_rank = base_eq;
        if (rank_ties) eq_rank += block_excl_scan(n_eq_t, tmp, &eq_total);
        bool sel[4];
        uint32_t n_sel_t = 0u;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            bool v = i0 + j < vis;
            if (v && !take_all) {
                if (key[j] == T)
                    v = !rank_ties || (eq_rank++ < r_eq);
                else
                    v = key[j] > T;
            }
            sel[j] = v;
            n_sel_t += v;
        }
        uint32_t sel_total;
        uint32_t pos = base_sel + block_excl_scan(n_sel_t, tmp, &sel_total);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            if (i0 + j >= vis) continue;
            const float e = __expf(x[j] - m);
            if (sel[j]) {
                if (pos < (uint32_t)k) {  // always true unless the select above is wrong
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
    const int kept = take_all ? vis : k;
    for (int j = kept + threadIdx.x; j < k; j += blockDim.x) idx[j] = -1;
    zk = block_sum(zk, red);
    __syncthreads();
    zt = block_sum(zt, red);
    if (threadIdx.x == 0) {
        if (base_sel != (uint32_t)kept) raise_status(p.status, TKA_DEV_INTERNAL);
        p.stats[row] = make_float4(m, zk, zt, 0.f);
        if (p.tail) p.tail[row] = zt / (zk + zt);
        p.counters[row] = 0u;
    }
}

}  // namespace

cudaError_t launch_select(const SelectParams &p, cudaStream_t stream) {
    const int rows = p.B * p.Q * p.Hq;
    select_topk<<<rows, kSelectThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tka
