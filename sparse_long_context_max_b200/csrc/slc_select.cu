// Fixed-budget page selection kernel: one 1024-thread CTA per (sequence, kv
// head) unit runs the register-resident exact selection of
// slc_select_impl.cuh ("Accelerating Long-Context Decoding in Large-Scale
// Hybrid LLMs Without Retraining", abstract: a fixed budget of the most
// relevant tokens).
#include "slc_select_impl.cuh"

namespace slc {

namespace {

constexpr int kThreads = 1024;
constexpr int kSurvivorCap = 8192;  // survivors held in shared memory

// Dynamic shared memory: the unit's scores (KPT per thread), then the
// survivors (key and index each).
template <int KPT>
constexpr int select_smem() {
    return kThreads * KPT * 4 + kSurvivorCap * 8;
}

template <int KPT>
__global__ void __launch_bounds__(kThreads, 1) select_kernel(SelectParams p) {
    __shared__ sel::Scratch<kThreads> sc;
    __shared__ uint64_t bar;
    extern __shared__ __align__(128) uint32_t smem[];
    float* stage = reinterpret_cast<float*>(smem);
    uint32_t* surv = smem + kThreads * KPT;
    grid_dep_wait();  // the scores come from the preceding kernel
    grid_dep_launch();
    sel::select_unit<kThreads, KPT>(p, blockIdx.x, sc, surv, kSurvivorCap, stage, &bar);
}

template <int KPT>
cudaError_t launch(const SelectParams& p, cudaStream_t stream) {
    return launch_pdl(select_kernel<KPT>, dim3(p.batch * p.hkv), dim3(kThreads),
                      select_smem<KPT>(), stream, 1, p);
}

}  // namespace

cudaError_t setup_select(DeviceCfg&) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel<16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         select_smem<16>());
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(select_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                select_smem<32>());
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
    if (p.batch * p.hkv == 0) return cudaSuccess;
    // candidates per unit are at most max_pages (<= kMaxCandidates)
    if (p.max_pages <= 16 * kThreads) return launch<16>(p, stream);
    return launch<32>(p, stream);
}

}  // namespace slc
