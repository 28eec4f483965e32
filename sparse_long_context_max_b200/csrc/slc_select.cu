// Fixed-budget page selection kernel: one 1024-thread CTA per (sequence, kv
// head) unit runs the register-resident exact selection of
// slc_select_impl.cuh ("Accelerating Long-Context Decoding in Large-Scale
// Hybrid LLMs Without Retraining", abstract: a fixed budget of the most
// relevant tokens).
#include "slc_attend_impl.cuh"
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

// CTA u < units selects unit u; CTA units + u (when m.dst_base >= 0) merges
// unit u's forced-list partials into slot m.dst_base + u.
template <int KPT>
__global__ void __launch_bounds__(kThreads, 1) select_kernel(SelectParams p, PremergeParams m) {
    static_assert(kThreads * KPT * 4 >= kThreads * (16 + 8), "merge scratch fits the stage");
    __shared__ sel::Scratch<kThreads> sc;
    __shared__ uint64_t bar;
    __shared__ long long sh_range[2];
    extern __shared__ __align__(128) uint32_t smem[];
    float* stage = reinterpret_cast<float*>(smem);
    uint32_t* surv = smem + kThreads * KPT;
    grid_dep_wait();  // the scores and partials come from the preceding kernel
    grid_dep_launch();
    const int units = p.batch * p.hkv;
    if ((int)blockIdx.x < units) {
        sel::select_unit<kThreads, KPT>(p, blockIdx.x, sc, surv, kSurvivorCap, stage, &bar);
        return;
    }
    const int u = blockIdx.x - units;
    if (threadIdx.x < 32) {  // the unit's forced-list slots
        const attn::Chunking cf = attn::forced_chunking(m.at, m.forced_chunks);
        const long long s0 = attn::unit_list_start(m.at, u);
        const int len = attn::list_len(m.at, u / m.at.hkv);
        if (threadIdx.x == 0) {
            sh_range[0] = len > 0 ? u + s0 / cf.cpp : 0;
            sh_range[1] = len > 0 ? u + (s0 + len - 1) / cf.cpp : -1;
        }
    }
    __syncthreads();
    if (sh_range[1] < sh_range[0]) return;  // no forced pages
    float4* sh_num = reinterpret_cast<float4*>(smem);
    float* sh_m = reinterpret_cast<float*>(sh_num + kThreads);
    attn::merge_slots<kThreads>(m.at, m.v4, sh_range[0], sh_range[1], m.dst_base + u, sh_num,
                                sh_m, sh_m + kThreads);
}

template <int KPT>
cudaError_t launch(const SelectParams& p, const PremergeParams& m, int ctas,
                   cudaStream_t stream) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel<KPT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             select_smem<KPT>());
        if (e != cudaSuccess) return e;
        configured = true;
    }
    return launch_pdl(select_kernel<KPT>, dim3(ctas), dim3(kThreads), select_smem<KPT>(), stream,
                      p, m);
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream, const PremergeParams* pm) {
    const int units = p.batch * p.hkv;
    if (units == 0) return cudaSuccess;
    PremergeParams m{};
    m.dst_base = -1;
    int ctas = units;
    if (pm) {
        m = *pm;
        ctas = 2 * units;
    }
    // candidates per unit are at most max_pages (<= kMaxCandidates)
    if (p.max_pages <= 16 * kThreads) return launch<16>(p, m, ctas, stream);
    return launch<32>(p, m, ctas, stream);
}

}  // namespace slc
