// topk_attn_decode_static: the decode call for callers that cannot allocate.
//
// Some callers cannot call cudaMalloc, or any other device allocator, to
// provide the scratch workspace topk_attn_decode needs: for example a serving
// engine that reserves all device memory for its own pool up front and lets
// nothing else allocate while it serves, or host code in a runtime that has no
// binding to a device allocator at all.  This entry point takes the same
// arguments minus the workspace and uses a scratch array compiled into the
// library instead.
//
// The array is a file-scope __device__ variable of kStaticWsBytes bytes: every
// GPU that loads the library holds it until the process exits.  Host code
// cannot use the array's name as a device address, so the first call on each
// device (with that device current) asks the runtime for the address with
// cudaGetSymbolAddress and keeps it.  Every call on a device shares the one
// array and finds the previous call's contents in it; nothing in it has to
// start at zero, because each call writes every part of the workspace it later
// reads.  Two calls whose kernels overlap on the GPU (different streams, or
// different host threads without ordering) race on the array.
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/topk_attn.h"
#include <cuda_runtime.h>

namespace {

constexpr size_t kStaticWsBytes = (size_t)48 << 20;  // 48 MiB

__device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_ws_addr[kMaxDevices] = {};  // device address of g_static_ws, per device
std::mutex g_ws_mu;                                // serialises the first lookup on a device

}  // namespace

extern "C" {

size_t topk_attn_static_workspace_capacity(void) { return kStaticWsBytes; }

tka_status topk_attn_decode_static(const tka_shape *shape, const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *seq_lens, int32_t k, float *out, int32_t *idx, float *tail_mass,
                                   tka_stream_t stream) {
    // every argument but the workspace is checked exactly as topk_attn_decode
    // checks it: without a workspace a valid call stops at TKA_ERR_WORKSPACE,
    // before anything is launched, and any other code is the argument error
    const tka_status args = topk_attn_decode(shape, q, k_cache, v_cache, seq_lens, k, out, idx, tail_mass, nullptr,
                                             0, stream);
    if (args != TKA_ERR_WORKSPACE) return args;
    const size_t need = topk_attn_workspace_size(shape, k);
    if (need == 0 || need > kStaticWsBytes) return TKA_ERR_WORKSPACE;  // larger than the built-in scratch array
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TKA_ERR_CUDA;
    void *ws = g_ws_addr[dev].load(std::memory_order_acquire);
    if (!ws) {
        std::lock_guard<std::mutex> lock(g_ws_mu);
        ws = g_ws_addr[dev].load(std::memory_order_relaxed);
        if (!ws) {
            if (cudaGetSymbolAddress(&ws, g_static_ws) != cudaSuccess || !ws) return TKA_ERR_CUDA;
            g_ws_addr[dev].store(ws, std::memory_order_release);
        }
    }
    return topk_attn_decode(shape, q, k_cache, v_cache, seq_lens, k, out, idx, tail_mass, ws, kStaticWsBytes,
                            stream);
}

}  // extern "C"
