// Select step kernel and launcher: one CTA per query row runs select_row
// (select_device.cuh).
#include "select_device.cuh"

namespace tka {

namespace {

template <int kThreads>
__global__ void __launch_bounds__(kThreads, 1024 / kThreads) select_topk(SelectParams p) {
    pdl_wait();  // the scores come from the kernel before
    pdl_trigger();
    select_row<kThreads>(p, blockIdx.x);
}

}  // namespace

size_t select_smem_bytes(int threads, int k) { return smem_words_for(k, threads / 32) * 4; }

namespace {

template <int kThreads>
cudaError_t launch_n(const SelectParams &p, cudaStream_t stream, bool pdl) {
    const int rows = p.B * p.Q * p.Hq;
    const size_t smem = select_smem_bytes(kThreads, p.k);
    static std::atomic<bool> attr_set[64] = {};  // per device: the shared-memory opt-in is a function attribute
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
        // the largest size any k takes, so that one setting serves every call
        e = cudaFuncSetAttribute(select_topk<kThreads>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)select_smem_bytes(kThreads, kMaxK));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
    }
    return launch_k(pdl, select_topk<kThreads>, dim3(rows), dim3(kThreads), smem, stream, p);
}

}  // namespace

cudaError_t launch_select(const SelectParams &p, cudaStream_t stream, int threads, bool pdl) {
    return threads == 512 ? launch_n<512>(p, stream, pdl) : launch_n<1024>(p, stream, pdl);
}

}  // namespace tka
