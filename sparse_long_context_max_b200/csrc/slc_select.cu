// Fixed-budget page selection kernel: one 256-thread CTA per (sequence, kv
// head) unit runs the exact two-level selection of slc_select_impl.cuh
// ("Accelerating Long-Context Decoding in Large-Scale Hybrid LLMs Without
// Retraining", abstract: a fixed budget of the most relevant tokens).
#include "slc_select_impl.cuh"

namespace slc {

namespace {

constexpr int kThreads = 256;
constexpr int kSurvivorCap = 8192;  // survivors held in shared memory
constexpr int kSelectSmem = sel::kLiveBytes + kSurvivorCap * 8;

__global__ void __launch_bounds__(kThreads) select_kernel(SelectParams p) {
    __shared__ sel::Scratch<kThreads> sc;
    extern __shared__ __align__(16) uint8_t buf[];
    grid_dep_wait();  // the scores come from the preceding kernel
    grid_dep_launch();
    sel::select_unit<kThreads>(p, blockIdx.x, buf, kSelectSmem, sc);
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
    if (p.batch * p.hkv == 0) return cudaSuccess;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(
            select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelectSmem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    return launch_pdl(select_kernel, dim3(p.batch * p.hkv), dim3(kThreads), kSelectSmem, stream,
                      p);
}

}  // namespace slc
