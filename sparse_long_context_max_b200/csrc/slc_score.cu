// Candidate-page scoring kernel: the Quest upper bound of q.k over every
// candidate page, summed over the query heads that share the kv head
// ("Hybrid LLM Decoding 2.2x Faster at 256k, No Retraining", section "The
// method: sliding window + prefix + query-aware pages, searched per
// layer"); the per-tile arithmetic is in slc_score_impl.cuh.  The kernel is
// HBM-bound: it streams 4*D bytes of metadata per candidate page.
//
// Work split: tiles (16 consecutive candidate pages of one unit) of all
// units are numbered in (b, h, tile) order and every warp of the
// (persistent) grid takes a contiguous range of them.  Each warp streams
// its tiles through a private shared-memory ring (two 8 KB tiles at D=128)
// filled by 16-byte asynchronous copies, one cp.async group per tile.
// Three 4-warp CTAs per SM keep 24 tiles (192 KB) in flight.  The kernel
// also writes each tile's maximum score when asked, which the selection
// uses to discard most pages without reading their scores.
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

// Cursor over the tiles of consecutive units.
struct TileCursor {
    int u;
    int ustart;  // global index of the unit's first tile
    int ntiles;  // tiles of unit u
    PageRanges r;
};

__device__ __forceinline__ void cursor_seek(const ScoreParams& p, TileCursor& c, int g) {
    while (true) {
        const int L = checked_len(p.seq_lens, c.u / p.hkv, p.max_pages, p.status);
        c.r = page_ranges(L, p.prefix, p.window);
        c.ntiles = (c.r.ws - c.r.np + kTilePages - 1) / kTilePages;
        if (g - c.ustart < c.ntiles) return;
        c.ustart += c.ntiles;
        ++c.u;
    }
}

template <int D>
__global__ void __launch_bounds__(kScoreWarps * 32, 3) score_kernel(ScoreParams p) {
    using C = ScoreCfg<D>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    uint8_t* ring = smem + warp * C::RING_B;

    // inputs (q, metadata, lengths) may come from the preceding kernel
    grid_dep_wait();
    grid_dep_launch();

    const int gw = blockIdx.x * kScoreWarps + warp;
    const int nw = gridDim.x * kScoreWarps;
    auto tiles_of = [&](int b) {
        const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
        const PageRanges r = page_ranges(L, p.prefix, p.window);
        return (r.ws - r.np + kTilePages - 1) / kTilePages;
    };
    const int total = (int)total_units(p.batch, p.hkv, tiles_of);
    const int per = (total + nw - 1) / nw;
    const int g0 = gw * per;
    const int g_end = min(total, g0 + per);
    if (g0 >= g_end) return;

    TileCursor use, iss;
    {
        long long us;
        locate_unit(g0, p.batch, p.hkv, tiles_of, &use.u, &us);
        use.ustart = (int)us;
    }
    cursor_seek(p, use, g0);
    iss = use;
    // issue side: tile gi is the next to copy; pf holds its page ids, loaded
    // one copy ahead so the lookup overlaps the ring traffic.  Every call
    // commits exactly one group (possibly empty) so that wait_group<NT-1>
    // always means "the oldest tile has landed".
    int gi = g0;
    int pf = tile_phys(p, iss.u, iss.r, gi - iss.ustart);
    auto copy_next = [&](int slot) {
        if (gi < g_end) {
            copy_tile<D>(p, iss.u % p.hkv, pf, ring + slot * C::TILE_B);
            ++gi;
            if (gi < g_end) {
                if (gi - iss.ustart >= iss.ntiles) cursor_seek(p, iss, gi);
                pf = tile_phys(p, iss.u, iss.r, gi - iss.ustart);
            }
        } else {
            cp_async_commit();
        }
    };
#pragma unroll
    for (int k = 0; k < C::NT; ++k) copy_next(k);

    int wu = -1;  // unit whose weights are loaded
    float w[C::CPL][8];
    for (int g = g0; g < g_end; ++g) {
        if (g - use.ustart >= use.ntiles) cursor_seek(p, use, g);
        if (use.u != wu) {
            wu = use.u;
            load_weights<D>(p, use.u, w);
        }
        const int slot = (g - g0) % C::NT;
        cp_async_wait<C::NT - 1>();  // this lane's chunks of the tile have landed
        score_tile<D>(p, use.u, use.r, g - use.ustart, ring + slot * C::TILE_B, w);
        copy_next(slot);  // refill: this lane's reads of the slot are done
    }
    cp_async_wait<0>();
}

}  // namespace

cudaError_t launch_score(const ScoreParams& p, int head_dim, int num_sms, cudaStream_t stream) {
    static int occ128 = 0, occ256 = 0;
    int& occ = head_dim == 128 ? occ128 : occ256;
    const int smem = head_dim == 128 ? ScoreCfg<128>::SMEM : ScoreCfg<256>::SMEM;
    if (occ == 0) {
        cudaError_t e;
        if (head_dim == 128) {
            e = cudaFuncSetAttribute(score_kernel<128>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e == cudaSuccess)
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, score_kernel<128>,
                                                                  kScoreWarps * 32, smem);
        } else {
            e = cudaFuncSetAttribute(score_kernel<256>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e == cudaSuccess)
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, score_kernel<256>,
                                                                  kScoreWarps * 32, smem);
        }
        if (e != cudaSuccess) return e;
        if (occ < 1) occ = 1;
    }
    const int blocks = num_sms * occ;
    if (head_dim == 128)
        return launch_pdl(score_kernel<128>, dim3(blocks), dim3(kScoreWarps * 32), smem, stream, p);
    return launch_pdl(score_kernel<256>, dim3(blocks), dim3(kScoreWarps * 32), smem, stream, p);
}

}  // namespace slc
