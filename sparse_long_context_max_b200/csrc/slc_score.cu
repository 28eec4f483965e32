// Candidate-page scoring: the Quest upper bound of q.k over a page, summed
// over the query heads that share the kv head ("Hybrid LLM Decoding 2.2x
// Faster at 256k, No Retraining", section "The method: sliding window +
// prefix + query-aware pages, searched per layer").
//
// For kmin <= kmax, max(q*kmin, q*kmax) is q*kmax when q >= 0 and q*kmin
// otherwise, so the group score is exactly
//     s = sum_d  Qneg_d * kmin_d + Qpos_d * kmax_d,
//     Qpos_d = sum_h max(q_hd, 0),  Qneg_d = sum_h min(q_hd, 0),
// two FMAs per metadata element whatever the group size.  The kernel is
// HBM-bound: it streams 4*D bytes of metadata per candidate page.
//
// Work split: a tile is 16 consecutive candidate pages of one (sequence,
// kv head) unit.  Tiles of all units are numbered in (b, h, tile) order and
// every warp of the (persistent) grid takes a contiguous range of them.
// Each warp streams its tiles through a private shared-memory ring (two
// 8 KB tiles at D=128) filled by 16-byte asynchronous copies: for every
// page, lane l copies the chunks it later reads itself, so completion is
// tracked per thread by cp.async groups (one per tile) and no register
// holds data in flight.  Three 4-warp CTAs per SM keep 24 tiles (192 KB)
// in flight.  Each lane dots its chunks with its query weights (one unpack
// and one FMA per element) and a transposed butterfly (16 shuffles) leaves
// page i's score in lanes 2i and 2i+1.  The kernel also writes each tile's
// maximum score, which the selection uses to discard most pages without
// reading their scores.
#include "slc_internal.h"

namespace slc {

namespace {

// 8 bf16 of a 16-byte chunk dotted with 8 fp32 weights: one unpack and one
// FMA per element.
__device__ __forceinline__ float dot8(const float (&w)[8], uint4 v) {
    float s = w[0] * bf16_lo(v.x);
    s = fmaf(w[1], bf16_hi(v.x), s);
    s = fmaf(w[2], bf16_lo(v.y), s);
    s = fmaf(w[3], bf16_hi(v.y), s);
    s = fmaf(w[4], bf16_lo(v.z), s);
    s = fmaf(w[5], bf16_hi(v.z), s);
    s = fmaf(w[6], bf16_lo(v.w), s);
    s = fmaf(w[7], bf16_hi(v.w), s);
    return s;
}

constexpr int kTilePages = kSelTile;  // pages per tile (16)
constexpr int kScoreWarps = 4;        // warps per CTA

template <int D>
struct ScoreCfg {
    static constexpr int CPR = D / 8;                   // chunks per metadata row
    static constexpr int CPL = 2 * CPR / 32;            // chunks per lane per page
    static constexpr int PAGE_B = 4 * D;                // metadata bytes per (page, kv head)
    static constexpr int TILE_B = kTilePages * PAGE_B;  // 8 KB / 16 KB
    static constexpr int NT = D == 128 ? 2 : 1;         // tiles in flight per warp
    static constexpr int RING_B = NT * TILE_B;
    static constexpr int SMEM = kScoreWarps * RING_B;   // 64 KB: three CTAs per SM
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

// Physical page of lane i's page (i < 16) of tile g (cursor c), or -1 for
// a page past the candidates or a block-table entry outside the pool.
__device__ __forceinline__ int tile_phys(const ScoreParams& p, const TileCursor& c, int g) {
    const int lane = threadIdx.x & 31;
    const int j = c.r.np + (g - c.ustart) * kTilePages + lane;
    int phys = -1;
    if (lane < kTilePages && j < c.r.ws) {
        phys = p.block_table[(long long)(c.u / p.hkv) * p.max_pages + j];
        if (phys < 0 || phys >= p.num_pages) {
            atomicOr(p.status, SLC_STATUS_BAD_PAGE);
            phys = -1;
        }
    }
    return phys;
}

// Copy a tile of kv head h into ring slot `slot`: for every page, lane l
// copies the 16-byte chunks l, l+32, ... that it later reads itself, so no
// cross-lane hand-off is needed.  One commit group per tile.
template <int D>
__device__ __forceinline__ void copy_tile(const ScoreParams& p, int h, int phys, uint8_t* ring,
                                          int slot) {
    using C = ScoreCfg<D>;
    const int lane = threadIdx.x & 31;
    const uint8_t* src0 =
        static_cast<const uint8_t*>(p.meta) + (long long)h * C::PAGE_B + lane * 16;
    uint8_t* dst0 = ring + slot * C::TILE_B + lane * 16;
#pragma unroll
    for (int pg = 0; pg < kTilePages; ++pg) {
        const int ph = __shfl_sync(0xffffffffu, phys, pg);
        if (ph >= 0) {
            const uint8_t* src = src0 + (long long)ph * p.hkv * C::PAGE_B;
#pragma unroll
            for (int m = 0; m < C::CPL; ++m)
                cp_async16(dst0 + pg * C::PAGE_B + m * 512, src + m * 512);
        }
    }
    cp_async_commit();
}

template <int D>
__global__ void __launch_bounds__(kScoreWarps * 32, 3) score_kernel(ScoreParams p) {
    using C = ScoreCfg<D>;
    constexpr int CPR = C::CPR, CPL = C::CPL;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
    int pf = tile_phys(p, iss, gi);
    auto copy_next = [&](int slot) {
        if (gi < g_end) {
            copy_tile<D>(p, iss.u % p.hkv, pf, ring, slot);
            ++gi;
            if (gi < g_end) {
                if (gi - iss.ustart >= iss.ntiles) cursor_seek(p, iss, gi);
                pf = tile_phys(p, iss, gi);
            }
        } else {
            cp_async_commit();
        }
    };
#pragma unroll
    for (int k = 0; k < C::NT; ++k) copy_next(k);

    int wu = -1;  // unit whose weights are loaded
    float w[CPL][8];
    for (int g = g0; g < g_end; ++g) {
        if (g - use.ustart >= use.ntiles) cursor_seek(p, use, g);
        if (use.u != wu) {
            // group-reduced query weights of this lane's chunks: chunk
            // lane + 32m is kmin dims (chunk < CPR) or kmax dims
            wu = use.u;
            const int b = use.u / p.hkv, h = use.u % p.hkv;
            const __nv_bfloat16* qb =
                static_cast<const __nv_bfloat16*>(p.q) + ((long long)b * p.hq + h * p.group) * D;
#pragma unroll
            for (int m = 0; m < CPL; ++m) {
                const bool is_max = lane + 32 * m >= CPR;
                const int d0 = 8 * ((lane + 32 * m) % CPR);
                uint4 qv[kMaxGroup];
#pragma unroll
                for (int gq = 0; gq < kMaxGroup; ++gq)
                    if (gq < p.group)
                        qv[gq] = __ldg(reinterpret_cast<const uint4*>(qb + gq * D + d0));
#pragma unroll
                for (int e = 0; e < 8; ++e) w[m][e] = 0.f;
#pragma unroll
                for (int gq = 0; gq < kMaxGroup; ++gq) {
                    if (gq < p.group) {
                        const uint4 v = qv[gq];
                        const float qf[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y),
                                             bf16_hi(v.y), bf16_lo(v.z), bf16_hi(v.z),
                                             bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            w[m][e] += is_max ? fmaxf(qf[e], 0.f) : fminf(qf[e], 0.f);
                    }
                }
            }
        }
        const int t = g - g0;
        const int slot = t % C::NT;
        cp_async_wait<C::NT - 1>();  // this lane's chunks of tile t have landed
        const uint8_t* tile = ring + slot * C::TILE_B + lane * 16;
        float acc[kTilePages];
#pragma unroll
        for (int pg = 0; pg < kTilePages; ++pg) {
            float sacc = 0.f;
#pragma unroll
            for (int m = 0; m < CPL; ++m)
                sacc += dot8(w[m], lds128(tile + pg * C::PAGE_B + m * 512));
            acc[pg] = sacc;
        }
        const int jt = g - use.ustart;
        copy_next(slot);  // refill: this lane's reads of the slot are done
        // transposed butterfly over 16 pages: lanes l and l^1 end with the
        // score of page (l >> 1)
#pragma unroll
        for (int lvl = 8; lvl >= 1; lvl >>= 1) {
            const bool upper = (lane & (2 * lvl)) != 0;
#pragma unroll
            for (int i = 0; i < lvl; ++i) {
                const float send = upper ? acc[i] : acc[i + lvl];
                const float keep = upper ? acc[i + lvl] : acc[i];
                acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2 * lvl);
            }
        }
        acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
        const int j = use.r.np + jt * kTilePages + (lane >> 1);
        float sc = -INFINITY;
        if (j < use.r.ws) {
            // a page whose block-table entry failed its check scores -inf
            const int phys = p.block_table[(long long)(use.u / p.hkv) * p.max_pages + j];
            sc = (phys < 0 || phys >= p.num_pages) ? -INFINITY : acc[0];
            if ((lane & 1) == 0) p.scores[(long long)use.u * p.max_pages + j] = sc;
        }
        if (p.tile_max) {
#pragma unroll
            for (int dist = 16; dist >= 2; dist >>= 1)
                sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, dist));
            if (lane == 0) p.tile_max[(long long)use.u * p.tile_stride + jt] = sc;
        }
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
