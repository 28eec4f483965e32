// Candidate-page scoring kernel: the Quest upper bound of q.k over every
// candidate page, summed over the query heads that share the kv head
// ("Hybrid LLM Decoding 2.2x Faster at 256k, No Retraining", section "The
// method: sliding window + prefix + query-aware pages, searched per
// layer"); the per-tile arithmetic is in slc_score_impl.cuh.  The kernel is
// HBM-bound: it streams 4*D bytes of metadata per candidate page.
//
// Work split: tiles (16 consecutive candidate pages of one unit) of all
// units are numbered in (b, h, tile) order and every warp of the
// (persistent) grid takes a contiguous range of them (score_range in
// slc_score_impl.cuh).  Each warp streams its tiles through a private
// shared-memory ring (two 8 KB tiles at D=128) filled by 16-byte
// asynchronous copies, one cp.async group per tile.  Three 4-warp CTAs per
// SM keep 24 tiles (192 KB) in flight.  The streaming kernel
// (slc_stream.cu) runs the same range code after its prefix/window
// attention.
#include "slc_score_impl.cuh"

namespace slc {

namespace {

using namespace scr;

constexpr int kScoreWarps = 4;  // warps per CTA

template <int D>
struct ScoreCfg : TileGeom<D> {
    static constexpr int NT = D == 128 ? 2 : 1;  // tiles in flight per warp
    static constexpr int RING_B = NT * TileGeom<D>::TILE_B;
    static constexpr int SMEM = kScoreWarps * RING_B;  // 64 KB: three CTAs per SM
};

template <int D>
__global__ void __launch_bounds__(kScoreWarps * 32, 3) score_kernel(ScoreParams p) {
    using C = ScoreCfg<D>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    // inputs (q, metadata, lengths) may come from the preceding kernel
    grid_dep_wait();
    grid_dep_launch();
    score_range<D, C::NT>(p, smem + warp * C::RING_B, blockIdx.x * kScoreWarps + warp,
                          gridDim.x * kScoreWarps);
}

}  // namespace

cudaError_t setup_score(DeviceCfg& d) {
    const int smem128 = ScoreCfg<128>::SMEM, smem256 = ScoreCfg<256>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(score_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem128);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_score[0], score_kernel<128>,
                                                          kScoreWarps * 32, smem128);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(score_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem256);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_score[1], score_kernel<256>,
                                                          kScoreWarps * 32, smem256);
    for (int i = 0; i < 2; ++i)
        if (d.occ_score[i] < 1) d.occ_score[i] = 1;
    return e;
}

cudaError_t launch_score(const ScoreParams& p, int head_dim, const DeviceCfg& d,
                         cudaStream_t stream) {
    const bool d128 = head_dim == 128;
    const int smem = d128 ? ScoreCfg<128>::SMEM : ScoreCfg<256>::SMEM;
    const int blocks = d.num_sms * d.occ_score[d128 ? 0 : 1];
    if (d128)
        return launch_pdl(score_kernel<128>, dim3(blocks), dim3(kScoreWarps * 32), smem, stream,
                          1, p);
    return launch_pdl(score_kernel<256>, dim3(blocks), dim3(kScoreWarps * 32), smem, stream, 1,
                      p);
}

}  // namespace slc
