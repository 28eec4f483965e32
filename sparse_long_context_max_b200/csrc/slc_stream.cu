// The streaming half of the sparse decode step: everything that does not
// depend on the selection, in one persistent HBM-bound kernel over every SM.
//
//   - attention over each unit's prefix and window pages (the pages every
//     query keeps: "Hybrid LLM Decoding 2.2x Faster at 256k, No
//     Retraining", section "The method: sliding window + prefix +
//     query-aware pages, searched per layer"), as split partials exactly
//     like the dense kernel's (slot = unit + chunk, the forced lists of all
//     units concatenated and cut into one chunk per attending CTA);
//   - the Quest bound of every candidate page (same section), written by
//     candidate into 16-byte aligned rows, as score_kernel does, with the
//     same per-warp copy pipeline (score_run in slc_score_impl.cuh).
//
// The two run side by side: the first CTAs of the grid attend, the others
// score, split in proportion to their bytes (forced_ctas in
// slc_attend_impl.cuh; a K+V page stage and a 16-page metadata tile are
// both 64*D bytes).  The finishing kernel (slc_finish.cu) then selects,
// attends the selected pages and merges everything.
#include "slc_attend_impl.cuh"
#include "slc_score_impl.cuh"

namespace slc {

namespace {

using namespace attn;

template <int D>
struct StreamCfg {
    static constexpr int NW = 4;                   // warps per CTA
    static constexpr int STAGES = D == 128 ? 2 : 3;  // ring stages per warp
    static constexpr int RING = STAGES * 2 * kPage * D * 2;
    // a K+V page stage holds one bf16 metadata tile or two E4M3 tiles
    static constexpr int NBAR = STAGES;
    static constexpr int SMEM = NW * (RING + NBAR * 8 + STAGES * 4);
    static constexpr int MIN_BLOCKS = D == 128 ? 3 : 1;
};

template <int D, bool FP8>
__global__ void __launch_bounds__(StreamCfg<D>::NW * 32, StreamCfg<D>::MIN_BLOCKS)
    stream_kernel(StreamParams p) {
    using C = StreamCfg<D>;
    static_assert(C::RING == C::STAGES * scr::TileGeom<D>::TILE_B, "ring holds STAGES tiles");
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Ring ring;
    ring.tiles = smem + warp * C::RING;
    ring.bars = reinterpret_cast<uint64_t*>(smem + C::NW * C::RING) + warp * C::NBAR;
    ring.nvalid =
        reinterpret_cast<int*>(smem + C::NW * C::RING + C::NW * C::NBAR * 8) + warp * C::STAGES;
    if (lane == 0) {
        for (int s = 0; s < C::NBAR; ++s) mbar_init(ring.bars + s, 1);
        fence_mbar_init();
    }
    __syncwarp();
    // q, the cache, the metadata and the lengths may come from the preceding
    // kernel (kv_append); the finishing kernel waits for this one
    grid_dep_wait();
    grid_dep_launch();

    const AttendParams& a = p.at;
    const int nf = forced_ctas(a, p.sc.scores != nullptr, gridDim.x);
    if ((int)blockIdx.x < nf) {
        // this CTA's chunk of the concatenated prefix/window lists
        auto len_of = [&](int b) { return list_len(a, b); };
        const long long total = total_units(a.batch, a.hkv, len_of);
        const long long cpp = (total + nf - 1) / nf;
        const long long s = (long long)blockIdx.x * cpp;
        const long long e = min(total, s + cpp);
        uint32_t it = 0;
        bool ok = true;
        attend_range<D, C::NW, C::STAGES>(a, smem, ring, it, ok, s, e, blockIdx.x);
    } else if (p.sc.scores != nullptr) {
        // candidate scores: the tiles of all units in (b, h, tile) order, a
        // contiguous range per warp of the remaining CTAs, each unit's
        // segment through the warp's ring (asynchronous 16-byte copies)
        const ScoreParams& sp = p.sc;
        constexpr int NS = C::RING / scr::TileGeom<D, FP8>::TILE_B;
        auto tiles_of = [&](int b) {
            const int L = checked_len(sp.seq_lens, b, sp.max_pages, sp.status);
            const PageRanges r = page_ranges(L, sp.prefix, sp.window);
            return (r.ws - r.np + kSelTile - 1) / kSelTile;
        };
        const long long total = total_units(sp.batch, sp.hkv, tiles_of);
        const long long nw = (long long)(gridDim.x - nf) * C::NW;
        const long long per = (total + nw - 1) / nw;
        long long g = ((long long)(blockIdx.x - nf) * C::NW + warp) * per;
        const long long g_end = min(total, g + per);
        if (g < g_end) {
            int u;
            long long ustart;
            locate_unit(g, sp.batch, sp.hkv, tiles_of, &u, &ustart);
            while (g < g_end && u < sp.batch * sp.hkv) {
                const int L = checked_len(sp.seq_lens, u / sp.hkv, sp.max_pages, sp.status);
                const PageRanges r = page_ranges(L, sp.prefix, sp.window);
                const long long uend = ustart + (r.ws - r.np + kSelTile - 1) / kSelTile;
                const long long stop = min(g_end, uend);
                if (stop > g) {
                    float w[scr::TileGeom<D>::CPL][8];
                    scr::load_weights<D>(sp, u, w);
                    scr::score_run<D, NS, FP8>(sp, ring.tiles, u, r, (int)(g - ustart),
                                               (int)(stop - ustart), w);
                    g = stop;
                }
                ustart = uend;
                ++u;
            }
        }
    }
}

template <int D, bool FP8>
cudaError_t setup_one(int* occ) {
    cudaError_t e = cudaFuncSetAttribute(stream_kernel<D, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         StreamCfg<D>::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, stream_kernel<D, FP8>,
                                                      StreamCfg<D>::NW * 32, StreamCfg<D>::SMEM);
    if (*occ < 1) *occ = 1;
    return e;
}

template <int D, bool FP8>
cudaError_t run(StreamParams& p, int blocks, const DeviceCfg& d, cudaStream_t stream) {
    // the metadata is read once per call: streamed through L2
    const StreamingRange meta =
        p.sc.scores != nullptr ? metadata_range(p.sc.meta, p.sc.num_pages, p.sc.hkv, D,
                                                p.sc.meta_format, d)
                               : StreamingRange{};
    return launch_pdl_streaming(stream_kernel<D, FP8>, dim3(blocks), dim3(StreamCfg<D>::NW * 32),
                                StreamCfg<D>::SMEM, stream, 1, meta, p);
}

}  // namespace

cudaError_t setup_stream(DeviceCfg& d) {
    // one occupancy per head_dim: the E4M3 forms use the same resources
    // (the grid size, hence the chunk count, must not depend on the format)
    cudaError_t e = setup_one<128, false>(&d.occ_stream[0]);
    if (e == cudaSuccess) e = setup_one<256, false>(&d.occ_stream[1]);
    int occ;
    if (e == cudaSuccess) e = setup_one<128, true>(&occ);
    if (e == cudaSuccess && occ < d.occ_stream[0]) d.occ_stream[0] = occ;
    if (e == cudaSuccess) e = setup_one<256, true>(&occ);
    if (e == cudaSuccess && occ < d.occ_stream[1]) d.occ_stream[1] = occ;
    return e;
}

int stream_chunks(int head_dim, const DeviceCfg& d) {
    const int blocks = d.num_sms * d.occ_stream[head_dim == 128 ? 0 : 1];
    return blocks < kMaxAttendChunks ? blocks : kMaxAttendChunks;
}

cudaError_t launch_stream(StreamParams& p, int head_dim, const DeviceCfg& d,
                          cudaStream_t stream) {
    const bool d128 = head_dim == 128;
    const int blocks = stream_chunks(head_dim, d);
    p.at.num_chunks = blocks;
    p.at.list = kListForced;
    const bool fp8 = p.sc.meta_format == SLC_META_FP8_E4M3;
    if (d128)
        return fp8 ? run<128, true>(p, blocks, d, stream) : run<128, false>(p, blocks, d, stream);
    return fp8 ? run<256, true>(p, blocks, d, stream) : run<256, false>(p, blocks, d, stream);
}

}  // namespace slc
