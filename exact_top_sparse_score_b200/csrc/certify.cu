// Certified adaptive Top-k: per row, the smallest k whose discarded softmax
// tail mass is at most eps.
//
// "A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance" (abstract): the total-variation error of Top-k truncation is the
// discarded tail mass, and a certified Top-k keeps the fewest keys that bring
// it under a prescribed budget eps.  The row's keys are ranked by (score
// descending, position ascending), as in the fixed-k path.
//
// The step runs after the select step has kept the top k_max positions of
// every row (ascending in idx, with w = e^{s - m} and the row's
// {m, Z_k, Z_tail}).  One CTA per row:
//   - every kept weight becomes an exact fixed-point integer (w * 2^40), so
//     that all sums below are exact and independent of their order;
//   - the target is (1 - eps) Z, Z = Z_k + Z_tail of the row; if the k_max
//     kept keys do not reach it, the row keeps them all (the certificate then
//     fails and the returned tail mass exceeds eps);
//   - otherwise a mass-weighted radix selection over the scores' order keys
//     (levels of at most 2048 bins over the range the kept keys span) finds
//     the key T at which the cumulative mass from the top reaches the target, the mass and count above T, and from the mass of
//     one key equal to T how many such keys (lowest positions first) are needed;
//   - the kept positions are compacted in place, in ascending order, and the
//     row's stats, tail mass and k are rewritten.
#include "common.cuh"
#include "kernels.h"

namespace tka {

namespace {

constexpr int kCertThreads = 1024;                  // most threads per row (k_max = 8192)
constexpr int kCertPer = kMaxK / kCertThreads;      // consecutive kept entries per thread
constexpr int kFixedShift = 40;                 // w in (0, 1] -> integer w * 2^40; 8192 of them fit in 2^53

__device__ __forceinline__ unsigned long long warp_incl_scan64(unsigned long long v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

__device__ __forceinline__ unsigned long long warp_sum64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// On warp 0: the bin b of a mass histogram (bins ordered by key) with
// mass(bins > b) < need <= mass(bins >= b), the mass above it and the count
// above it.  Requires 1 <= need <= total mass.
template <int NB>
__device__ void warp_find_mass(const unsigned long long *hm, const uint32_t *hc, unsigned long long need,
                               uint32_t &bin, unsigned long long &mass_above, uint32_t &cnt_above) {
    constexpr int kPer = NB / 32;
    const int lane = threadIdx.x & 31;
    const int top = NB - 1 - lane * kPer;  // lane l holds bins top, top - 1, ..., top - kPer + 1
    unsigned long long local = 0ull;
#pragma unroll
    for (int i = 0; i < kPer; i++) local += hm[top - i];
    const unsigned long long cum = warp_incl_scan64(local);
    const unsigned long long before = cum - local;
    const uint32_t hit = __ballot_sync(0xffffffffu, before < need && cum >= need);
    bin = 0u;
    mass_above = 0ull;
    cnt_above = 0u;
    if (hit == 0u) return;  // need outside [1, total]: never the case for a valid call
    const int L = __ffs(hit) - 1;
    const int topL = NB - 1 - L * kPer;
    unsigned long long c = __shfl_sync(0xffffffffu, before, L);
    int found = -1;
#pragma unroll
    for (int i0 = 0; i0 < kPer; i0 += 32) {
        const unsigned long long h = i0 + lane < kPer ? hm[topL - i0 - lane] : 0ull;
        const unsigned long long inc = warp_incl_scan64(h);
        const unsigned long long excl = c + inc - h;
        const uint32_t fb = __ballot_sync(0xffffffffu, i0 + lane < kPer && excl < need && excl + h >= need);
        if (fb != 0u) {
            const int f = __ffs(fb) - 1;
            found = topL - i0 - f;
            mass_above = __shfl_sync(0xffffffffu, excl, f);
            break;
        }
        c += __shfl_sync(0xffffffffu, inc, 31);
    }
    bin = (uint32_t)found;
    // keys in bins above the found one
    uint32_t cnt = 0u;
#pragma unroll
    for (int i = 0; i < kPer; i++) cnt += top - i > found ? hc[top - i] : 0u;
    cnt_above = warp_sum(cnt);
}

// blockDim.x = k_max / kCertPer rounded up to whole warps (at least two), so
// that short rows leave room for several CTAs per SM.
template <int kMaxThreads>
__global__ void __launch_bounds__(kMaxThreads) certify_topk(CertifyParams p) {
    __shared__ unsigned long long hmass[2048];
    __shared__ uint32_t hcnt[2048];
    __shared__ uint32_t tmp[32];
    __shared__ unsigned long long red64[32];
    __shared__ float redf[64];
    __shared__ unsigned long long s_mass;
    __shared__ uint32_t s_bin, s_cnt;
    __shared__ uint32_t s_kmin[32], s_kmax[32];
    pdl_wait();  // the selection comes from the kernel before
    pdl_trigger();

    const int row = blockIdx.x;
    const int b = row / (p.Q * p.Hq), qpos = (row / p.Hq) % p.Q;
    const int seq_len = p.seq_lens[b];
    if (!seq_len_ok(seq_len, p.Q, p.L_max)) return;  // the select step raised the status
    const int vis = visible_keys(seq_len, p.Q, qpos);
    const int kk = min(p.k_max, vis);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t *idx = p.idx + (size_t)row * p.k_max;
    float *wv = p.w + (size_t)row * p.k_max;
    const float *srow = p.scores + (size_t)row * p.ld;

    // this thread's kept entries j = kCertPer * tid + u, in ascending position order
    int32_t pos[kCertPer];
    float w[kCertPer];
    uint32_t key[kCertPer];
    unsigned long long fx[kCertPer];
    unsigned long long mine = 0ull;
#pragma unroll
    for (int u = 0; u < kCertPer; u++) {
        const int j = kCertPer * threadIdx.x + u;
        pos[u] = j < kk ? idx[j] : -1;
        w[u] = j < kk ? wv[j] : 0.f;
        if (j < kk && (unsigned)pos[u] >= (unsigned)vis) {  // never true unless the select step is wrong
            raise_status(p.status, TKA_DEV_INTERNAL);
            pos[u] = 0;
        }
        key[u] = j < kk ? canon_key(srow[pos[u]]) : 0u;
        fx[u] = (unsigned long long)((double)w[u] * (double)(1ull << kFixedShift));  // w <= 1: exact below 2^-40
        mine += fx[u];
    }
    // total kept mass
    mine = warp_sum64(mine);
    if (lane == 0) red64[warp] = mine;
    __syncthreads();
    const int nw = blockDim.x >> 5;
    const unsigned long long kept_mass = warp_sum64(lane < nw ? red64[lane] : 0ull);
    const float4 st = p.stats[row];
    const double Z = (double)st.y + (double)st.z;
    const double target_d = ceil((1.0 - (double)p.eps) * Z * (double)(1ull << kFixedShift));
    const unsigned long long target = target_d < 1.0 ? 1ull : (unsigned long long)target_d;

    int k = kk;
    uint32_t T = 0u, need_eq = 0u;
    bool cut = kept_mass >= target;  // otherwise all kk stay (not certifiable within k_max)
    if (cut) {
        // The kept keys lie in [kmin, kmax].  Each level splits the current
        // key range [lo, lo + 2^span) into at most 2048 bins of 2^shift keys,
        // so the bins follow where the keys actually are (few keys share a
        // bin: few conflicting atomics), and at most three levels reach a
        // single key.
        uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
        for (int u = 0; u < kCertPer; u++) {
            if (kCertPer * (int)threadIdx.x + u < kk) {
                kmin = min(kmin, key[u]);
                kmax = max(kmax, key[u]);
            }
        }
        kmin = __reduce_min_sync(0xffffffffu, kmin);
        kmax = __reduce_max_sync(0xffffffffu, kmax);
        if (lane == 0) {
            s_kmin[warp] = kmin;
            s_kmax[warp] = kmax;
        }
        __syncthreads();
        kmin = __reduce_min_sync(0xffffffffu, lane < nw ? s_kmin[lane] : 0xffffffffu);
        kmax = __reduce_max_sync(0xffffffffu, lane < nw ? s_kmax[lane] : 0u);
        uint32_t lo = kmin;
        int span = 32 - __clz((int)(kmax - kmin));  // bits of the range
        unsigned long long mass_above = 0ull;
        uint32_t cnt_above = 0u;
        for (;;) {
            const int shift = span > 11 ? span - 11 : 0;
            for (int i = threadIdx.x; i < 2048; i += blockDim.x) {
                hmass[i] = 0ull;
                hcnt[i] = 0u;
            }
            __syncthreads();
#pragma unroll
            for (int u = 0; u < kCertPer; u++) {
                const uint32_t rel = key[u] - lo;  // wraps for keys below lo
                if (kCertPer * (int)threadIdx.x + u < kk && (span >= 32 || (rel >> span) == 0u)) {
                    const uint32_t bn = rel >> shift;
                    atomicAdd(&hmass[bn], fx[u]);
                    atomicAdd(&hcnt[bn], 1u);
                }
            }
            __syncthreads();
            if (warp == 0) {
                uint32_t bn, ca;
                unsigned long long ma;
                warp_find_mass<2048>(hmass, hcnt, target - mass_above, bn, ma, ca);
                if (lane == 0) {
                    s_bin = bn;
                    s_mass = ma;
                    s_cnt = ca;
                }
            }
            __syncthreads();
            mass_above += s_mass;
            cnt_above += s_cnt;
            lo += s_bin << shift;
            span = shift;
            if (shift == 0) {
                // keys equal to T = lo all carry the same weight
                const unsigned long long m_eq = hmass[s_bin];
                const uint32_t n_eq = hcnt[s_bin];
                const unsigned long long w_eq = n_eq ? m_eq / n_eq : 1ull;
                const unsigned long long rest = target - mass_above;
                need_eq = (uint32_t)min((unsigned long long)n_eq, (rest + w_eq - 1ull) / w_eq);
                break;
            }
            __syncthreads();  // the histograms are cleared again next level
        }
        T = lo;
        k = (int)(cnt_above + need_eq);
    }

    // ordered compaction: keys above T, then the first need_eq keys equal to T
    uint32_t n_eq_t = 0u;
#pragma unroll
    for (int u = 0; u < kCertPer; u++) n_eq_t += (kCertPer * (int)threadIdx.x + u < kk && key[u] == T) ? 1u : 0u;
    uint32_t total;
    uint32_t eq_rank = block_excl_scan(cut ? n_eq_t : 0u, tmp, &total);
    bool keep[kCertPer];
    uint32_t n_keep = 0u;
#pragma unroll
    for (int u = 0; u < kCertPer; u++) {
        const int j = kCertPer * threadIdx.x + u;
        bool kp = j < kk;
        if (kp && cut) {
            if (key[u] > T) {
                kp = true;
            } else if (key[u] == T) {
                kp = eq_rank < need_eq;
                eq_rank++;
            } else {
                kp = false;
            }
        }
        keep[u] = kp;
        n_keep += kp;
    }
    uint32_t o = block_excl_scan(n_keep, tmp, &total);
    if (total != (uint32_t)k && threadIdx.x == 0) raise_status(p.status, TKA_DEV_INTERNAL);
    float zk = 0.f, zdrop = 0.f;
    // every thread has read its entries (block_excl_scan ends with a barrier): rewrite in place
#pragma unroll
    for (int u = 0; u < kCertPer; u++) {
        if (keep[u]) {
            if (o < (uint32_t)p.k_max) {
                idx[o] = pos[u];
                wv[o] = w[u];
            }
            o++;
            zk += w[u];
        } else if (kCertPer * (int)threadIdx.x + u < kk) {
            zdrop += w[u];
        }
    }
    __syncthreads();  // all kept entries placed before the padding is written
    for (int j = k + (int)threadIdx.x; j < kk; j += blockDim.x) idx[j] = -1;
    // both sums with one barrier pair
    zk = warp_sum(zk);
    zdrop = warp_sum(zdrop);
    if (lane == 0) {
        redf[2 * warp] = zk;
        redf[2 * warp + 1] = zdrop;
    }
    __syncthreads();
    zk = warp_sum(lane < nw ? redf[2 * lane] : 0.f);
    zdrop = warp_sum(lane < nw ? redf[2 * lane + 1] : 0.f);
    if (threadIdx.x == 0) {
        const float zt = st.z + zdrop;
        p.stats[row] = make_float4(st.x, zk, zt, 0.f);
        if (p.tail) p.tail[row] = zt / (zk + zt);
        p.k_used[row] = k;
    }
}

}  // namespace

cudaError_t launch_certify(const CertifyParams &p, cudaStream_t stream, bool pdl) {
    if (p.k_max > kMaxK) return cudaErrorInvalidValue;
    const int threads = max(64, min(kCertThreads, (p.k_max + kCertPer * 32 - 1) / (kCertPer * 32) * 32));
    if (threads <= 256)
        return launch_k(pdl, certify_topk<256>, dim3(p.B * p.Q * p.Hq), dim3(threads), 0, stream, p);
    else
        return launch_k(pdl, certify_topk<kCertThreads>, dim3(p.B * p.Q * p.Hq), dim3(threads), 0, stream, p);
}

}  // namespace tka
