// Device helpers shared by the Top-k decode-attention kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/topk_attn.h"

namespace tka {

constexpr int kHeadDim = 128;

// Kernels report problems they can only see on the device (TKA_DEV_* bits) by
// OR-ing them into the library's per-device status word, whose address every
// launch receives.
__device__ __forceinline__ void raise_status(unsigned int *status, unsigned int bits) { atomicOr(status, bits); }

// A paged cache: pages of 2^page_shift positions, [num_pages, Hkv, page, 128];
// logical page j of sequence b is physical page table[b * max_pages + j].
// A null table means the contiguous layout [B, Hkv, L_max, 128].
struct PageTable {
    const int32_t *table = nullptr;
    int max_pages = 0, num_pages = 0, page_shift = 0;
};

// Row (of 128 elements) holding position pos of (b, kvh) in a paged cache.
// A table entry out of range raises TKA_DEV_BAD_PAGE and reads page 0.
__device__ __forceinline__ long long paged_row(const PageTable &pt, unsigned *status, int Hkv, int b, int kvh, int pos) {
    int phys = __ldg(pt.table + (size_t)b * pt.max_pages + (pos >> pt.page_shift));
    if ((unsigned)phys >= (unsigned)pt.num_pages) {
        raise_status(status, TKA_DEV_BAD_PAGE);
        phys = 0;
    }
    return ((long long)phys * Hkv + kvh) * (1ll << pt.page_shift) + (pos & ((1 << pt.page_shift) - 1));
}

// Rows are (b, qpos, h) in that order: row = (b * Q + qpos) * Hq + h.
struct RowGeom {
    int B, Q, Hq, Hkv, G, L_max;
};

// Visible keys of query position qpos in a chunk of Q queries ending at the
// sequence's last position.
__device__ __forceinline__ int visible_keys(int seq_len, int Q, int qpos) { return seq_len - Q + qpos + 1; }

__device__ __forceinline__ bool seq_len_ok(int seq_len, int Q, int L_max) { return seq_len >= Q && seq_len <= L_max; }

// Order-preserving map from fp32 to uint32: a > b (as floats, no NaN) iff
// key(a) > key(b); -0.0 and +0.0 get distinct adjacent keys.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// order_key with -0.0 mapped to +0.0, so that key order is exactly the order
// of float comparisons (for non-NaN values): a > b iff key(a) > key(b), and
// a == b iff key(a) == key(b).
__device__ __forceinline__ uint32_t canon_key(float f) { return order_key(__fadd_rn(f, 0.f)); }

// Programmatic dependent launch.  A kernel launched with launch_pdl may be
// started while the kernel before it on the stream is still running: it must
// call pdl_wait() before it reads anything that kernel (or any earlier work)
// wrote -- the wait returns once the earlier grid has completed and its
// writes are visible, and at once for a kernel launched without the
// attribute.  pdl_trigger() lets the launch of the next kernel begin.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// An L2 policy for data read once: the lines it brings in are evicted first,
// so that streaming it does not push out lines still to be read.
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t pol;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// A 4-byte load that bypasses L1 and allocates in L2 under policy `pol`.
__device__ __forceinline__ float ld_l2_hint(const float *a, uint64_t pol) {
    float v;
    asm("ld.global.L1::no_allocate.L2::cache_hint.f32 %0, [%1], %2;" : "=f"(v) : "l"(a), "l"(pol));
    return v;
}

// 2^t by the hardware approximation (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float exp2_approx(float t) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(t));
    return r;
}

constexpr float kLog2e = 1.4426950408889634f;  // log2(e): e^x = 2^(x log2 e)

// Inverse of order_key.
__device__ __forceinline__ float key_float(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Block-wide max of one value per thread (blockDim.x multiple of 32, <= 1024).
// `red` is >= 32 floats of shared memory; contains two barriers.
__device__ __forceinline__ float block_max(float v, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_max(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = lane < nw ? red[lane] : -INFINITY;
    return warp_max(t);
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

// Inclusive prefix sum of v over the warp.
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

// Finds, on one warp, the bin holding the need-th largest element of a
// histogram of NB bins ordered by key: the bin and the count of elements in
// higher bins, in every lane.  Requires 1 <= need <= total count and NB a
// power of two in [32, 2048].  Lane l sums the NB/32 bins below the top
// l NB/32 (all loads in flight together, starting at a lane-dependent bin so
// that they spread over the banks), a prefix sum over the lanes finds the
// lane holding the bin, and the warp then scans that lane's bins 32 at a time.
template <int NB>
__device__ inline void warp_find_bin(const uint32_t *hist, uint32_t need, uint32_t &bin, uint32_t &above) {
    static_assert(NB >= 32 && NB <= 2048 && (NB & (NB - 1)) == 0, "bins: a power of two in [32, 2048]");
    constexpr int kPer = NB / 32;
    const int lane = threadIdx.x & 31;
    const int top = NB - 1 - lane * kPer;
    uint32_t local = 0u;
#pragma unroll
    for (int i = 0; i < kPer; i++) local += hist[top - ((i + lane) & (kPer - 1))];
    const uint32_t cum = warp_incl_scan(local);
    const uint32_t before = cum - local;
    const uint32_t hit = __ballot_sync(0xffffffffu, before < need && cum >= need);
    bin = 0u;  // need outside [1, total]: never the case for a valid call
    above = 0u;
    if (hit != 0u) {
        const int L = __ffs(hit) - 1;
        const int topL = NB - 1 - L * kPer;
        uint32_t c = __shfl_sync(0xffffffffu, before, L);
#pragma unroll
        for (int i0 = 0; i0 < kPer; i0 += 32) {
            const uint32_t h = i0 + lane < kPer ? hist[topL - i0 - lane] : 0u;
            const uint32_t inc = warp_incl_scan(h);
            const uint32_t excl = c + inc - h;
            const uint32_t fb = __ballot_sync(0xffffffffu, excl < need && excl + h >= need);
            if (fb != 0u) {
                const int f = __ffs(fb) - 1;
                bin = (uint32_t)(topL - i0 - f);
                above = __shfl_sync(0xffffffffu, excl, f);
                break;
            }
            c += __shfl_sync(0xffffffffu, inc, 31);
        }
    }
}

// The same search spread over the whole block, for two targets at once: the
// bins holding the need_a-th and the need_b-th largest element (1 <= need <=
// total count).  Thread t sums the NB / blockDim.x bins below the top
// t NB / blockDim.x, a block-wide prefix sum over the threads (warp scans plus
// one word per warp in `wtot`, >= 32 words) locates the thread holding each
// target, and that thread scans its few bins.  out[0], out[1] = bin and count
// above it for need_a; out[2], out[3] for need_b.  The histogram must be
// complete when the block enters (the first barrier here does not wait for
// it), and every thread reads `out` after the call.
template <int NB>
__device__ inline void block_find_bins(const uint32_t *hist, uint32_t need_a, uint32_t need_b, uint32_t *wtot,
                                       uint32_t *out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int per = NB / (int)blockDim.x;  // >= 1: NB >= blockDim.x, both powers of two
    const int top = NB - 1 - (int)threadIdx.x * per;
    uint32_t local = 0u;
    for (int j = 0; j < per; j++) local += hist[top - j];
    const uint32_t incl = warp_incl_scan(local);
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    const uint32_t wt = lane < nw ? wtot[lane] : 0u;
    const uint32_t winc = warp_incl_scan(wt);
    const uint32_t before = __shfl_sync(0xffffffffu, winc - wt, warp) + incl - local;
#pragma unroll
    for (int t = 0; t < 2; t++) {
        const uint32_t need = t == 0 ? need_a : need_b;
        if (before < need && before + local >= need) {
            uint32_t c = before;
            for (int j = 0; j < per; j++) {
                const uint32_t h = hist[top - j];
                if (c + h >= need) {
                    out[2 * t] = (uint32_t)(top - j);
                    out[2 * t + 1] = c;
                    break;
                }
                c += h;
            }
        }
    }
    __syncthreads();
}

// The same search for the whole block: the block first meets at a barrier
// (so the histogram is complete and the results of a previous call have been
// read), warp 0 searches and writes the results, and the block meets again.
template <int NB>
__device__ inline void find_bin_n(const uint32_t *hist, uint32_t need, uint32_t *out_bin, uint32_t *out_above) {
    __syncthreads();
    if (threadIdx.x < 32) {
        uint32_t bin, above;
        warp_find_bin<NB>(hist, need, bin, above);
        if (threadIdx.x == 0) {
            *out_bin = bin;
            *out_above = above;
        }
    }
    __syncthreads();
}

// find_bin_n for nbins = 256, 1024 or 2048 (the sizes the kernels use).
__device__ inline void find_bin(const uint32_t *hist, int nbins, uint32_t need, uint32_t *, uint32_t *out_bin,
                                uint32_t *out_above) {
    if (nbins == 2048)
        find_bin_n<2048>(hist, need, out_bin, out_above);
    else if (nbins == 1024)
        find_bin_n<1024>(hist, need, out_bin, out_above);
    else
        find_bin_n<256>(hist, need, out_bin, out_above);
}

}  // namespace tka
