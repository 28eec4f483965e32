// Candidate-page scoring kernel: the Quest upper bound of q.k over every
// candidate page, summed over the query heads that share the kv head
// ("Hybrid LLM Decoding 2.2x Faster at 256k, No Retraining", section "The
// method: sliding window + prefix + query-aware pages, searched per
// layer"); the per-tile arithmetic is in slc_score_impl.cuh.  The kernel is
// HBM-bound: it streams 4*D bytes of metadata per candidate page.
//
// Work split: tiles (16 consecutive candidate pages of one unit) of all
// units are numbered in (b, h, tile) order and every warp of the
// (persistent) grid takes a contiguous range of them.  Each warp streams its
// tiles through a private shared-memory ring (two 8 KB tiles at D=128)
// filled by asynchronous copies (score_run in slc_score_impl.cuh).  Three
// 4-warp CTAs per SM keep 24 tiles (192 KB) in flight.  The streaming kernel
// of the sparse decode (slc_stream.cu) scores with the same code.
#include "slc_score_impl.cuh"

namespace slc {

namespace {

using namespace scr;

constexpr int kScoreWarps = 4;  // warps per CTA

// Ring per warp: two 8 KB tiles at D = 128 (bf16), one 16 KB tile at D =
// 256; E4M3 tiles are half the size, so twice as many fit.
template <int D, bool FP8>
struct ScoreCfg {
    static constexpr int NT = (D == 128 ? 2 : 1) * (FP8 ? 2 : 1);  // tiles in flight per warp
    static constexpr int RING_B = NT * TileGeom<D, FP8>::TILE_B;
    static constexpr int SMEM = kScoreWarps * RING_B;               // 64 KB: three CTAs per SM
};

template <int D, bool FP8>
__global__ void __launch_bounds__(kScoreWarps * 32, 3) score_kernel(ScoreParams p) {
    using C = ScoreCfg<D, FP8>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    // inputs (q, metadata, lengths) may come from the preceding kernel
    grid_dep_wait();
    grid_dep_launch();
    auto tiles_of = [&](int b) {
        const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
        const PageRanges r = page_ranges(L, p.prefix, p.window);
        return (r.ws - r.np + kTilePages - 1) / kTilePages;
    };
    const long long total = total_units(p.batch, p.hkv, tiles_of);
    const long long nw = (long long)gridDim.x * kScoreWarps;
    const long long per = (total + nw - 1) / nw;
    long long g = ((long long)blockIdx.x * kScoreWarps + warp) * per;
    const long long g_end = min(total, g + per);
    if (g >= g_end) return;
    int u;
    long long ustart;
    locate_unit(g, p.batch, p.hkv, tiles_of, &u, &ustart);
    // the units this warp's range crosses, in order
    while (g < g_end && u < p.batch * p.hkv) {
        const int L = checked_len(p.seq_lens, u / p.hkv, p.max_pages, p.status);
        const PageRanges r = page_ranges(L, p.prefix, p.window);
        const long long uend = ustart + (r.ws - r.np + kTilePages - 1) / kTilePages;
        const long long stop = min(g_end, uend);
        if (stop > g) {
            float w[TileGeom<D>::CPL][8];
            load_weights<D>(p, u, w);
            score_run<D, C::NT, FP8>(p, smem + warp * C::RING_B, u, r, (int)(g - ustart),
                                     (int)(stop - ustart), w);
            g = stop;
        }
        ustart = uend;
        ++u;
    }
}

template <int D, bool FP8>
cudaError_t setup_one(int* occ) {
    constexpr int smem = ScoreCfg<D, FP8>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(score_kernel<D, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, score_kernel<D, FP8>,
                                                          kScoreWarps * 32, smem);
    if (*occ < 1) *occ = 1;
    return e;
}

template <int D, bool FP8>
cudaError_t run(const ScoreParams& p, int occ, const DeviceCfg& d, cudaStream_t stream) {
    // the metadata is read once per call: streamed through L2
    return launch_pdl_streaming(score_kernel<D, FP8>, dim3(d.num_sms * occ),
                                dim3(kScoreWarps * 32), ScoreCfg<D, FP8>::SMEM, stream, 1,
                                metadata_range(p.meta, p.num_pages, p.hkv, D, p.meta_format, d),
                                p);
}

}  // namespace

cudaError_t setup_score(DeviceCfg& d) {
    cudaError_t e = setup_one<128, false>(&d.occ_score[0]);
    if (e == cudaSuccess) e = setup_one<256, false>(&d.occ_score[1]);
    int occ;  // the E4M3 forms have the same shared memory: same occupancy
    if (e == cudaSuccess) e = setup_one<128, true>(&occ);
    if (e == cudaSuccess) e = setup_one<256, true>(&occ);
    return e;
}

cudaError_t launch_score(const ScoreParams& p, int head_dim, const DeviceCfg& d,
                         cudaStream_t stream) {
    const bool fp8 = p.meta_format == SLC_META_FP8_E4M3;
    if (head_dim == 128)
        return fp8 ? run<128, true>(p, d.occ_score[0], d, stream)
                   : run<128, false>(p, d.occ_score[0], d, stream);
    return fp8 ? run<256, true>(p, d.occ_score[1], d, stream)
               : run<256, false>(p, d.occ_score[1], d, stream);
}

}  // namespace slc
