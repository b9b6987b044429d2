// Select step kernel and launcher: one CTA per query row runs select_row
// (select_device.cuh).
#include "select_device.cuh"

namespace tka {

namespace {

template <int kThreads, bool kEvictFirst>
__global__ void __launch_bounds__(kThreads, 1024 / kThreads) select_topk(SelectParams p) {
    pdl_wait();  // the scores come from the kernel before
    pdl_trigger();
    select_row<kThreads, kEvictFirst>(p, blockIdx.x);
}

// Score buffers above this size did not stay in L2 (126 MB): their rows are
// read with evict-first loads (measured: the 268 MB of the 16-position causal
// chunk 101 -> 96 us; the 33.5 MB and 67 MB buffers lose ~1 us with them).
constexpr size_t kEvictFirstScores = 96ull << 20;

}  // namespace

size_t select_smem_bytes(int threads, int k) { return smem_words_for(k, threads / 32) * 4; }

namespace {

template <int kThreads, bool kEvictFirst>
cudaError_t launch_n(const SelectParams &p, cudaStream_t stream, bool pdl) {
    const int rows = p.B * p.Q * p.Hq;
    const size_t smem = select_smem_bytes(kThreads, p.k);
    static std::atomic<bool> attr_set[64] = {};  // per device: the shared-memory opt-in is a function attribute
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
        // the largest size any k takes, so that one setting serves every call
        e = cudaFuncSetAttribute(select_topk<kThreads, kEvictFirst>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)select_smem_bytes(kThreads, kMaxK));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
    }
    return launch_k(pdl, select_topk<kThreads, kEvictFirst>, dim3(rows), dim3(kThreads), smem, stream, p);
}

}  // namespace

cudaError_t launch_select(const SelectParams &p, cudaStream_t stream, int threads, bool pdl) {
    const bool big = (size_t)p.B * p.Q * p.Hq * p.ld * sizeof(float) > kEvictFirstScores;
    if (threads == 512) return big ? launch_n<512, true>(p, stream, pdl) : launch_n<512, false>(p, stream, pdl);
    return big ? launch_n<1024, true>(p, stream, pdl) : launch_n<1024, false>(p, stream, pdl);
}

}  // namespace tka
