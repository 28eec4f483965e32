// Candidate-page scoring building blocks of the scoring kernel
// (slc_score.cu): the Quest
// upper bound of q.k over a page, summed over the query heads that share
// the kv head ("Hybrid LLM Decoding 2.2x Faster at 256k, No Retraining",
// section "The method: sliding window + prefix + query-aware pages,
// searched per layer").
//
// For kmin <= kmax, max(q*kmin, q*kmax) is q*kmax when q >= 0 and q*kmin
// otherwise, so the group score is exactly
//     s = sum_d  Qneg_d * kmin_d + Qpos_d * kmax_d,
//     Qpos_d = sum_h max(q_hd, 0),  Qneg_d = sum_h min(q_hd, 0),
// two FMAs per metadata element whatever the group size.
//
// A tile is 16 consecutive candidate pages of one (sequence, kv head)
// unit; one warp scores a tile held in shared memory (16 metadata rows, in
// page order, of 4*D bytes (bf16) or 2*D bytes (E4M3)), brought in by bulk
// copies (TMA engine, one per page, issued by lanes 0..15) completing on
// the ring stage's mbarrier.  Lane l owns chunks l, l+32, ... of every row
// (16 bytes = 8 bf16, or 8 bytes = 8 E4M3: the same 8 dims either way) and
// dots them with its query weights; a transposed butterfly (16 shuffles)
// then leaves page i's score in lanes 2i and 2i+1.
#pragma once

#include "slc_internal.h"

namespace slc {
namespace scr {

constexpr int kTilePages = kSelTile;  // pages per tile (16)

template <int D, bool FP8 = false>
struct TileGeom {
    static constexpr int CPR = D / 8;                   // chunks (8 dims) per metadata row
    static constexpr int CPL = 2 * CPR / 32;            // chunks per lane per page
    static constexpr int CHUNK_B = FP8 ? 8 : 16;        // bytes per chunk
    static constexpr int PAGE_B = 2 * CPR * CHUNK_B;    // metadata bytes per (page, kv head)
    static constexpr int TILE_B = kTilePages * PAGE_B;  // bf16 8 KB / 16 KB, E4M3 half
};

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

// 8 E4M3 codes (8 bytes, low byte first) dotted with 8 fp32 weights.
__device__ __forceinline__ float dot8_e4m3(const float (&w)[8], uint2 v, float oor) {
    const float2 a = e4m3x2_to_float2(v.x, oor), b = e4m3x2_to_float2(v.x >> 16, oor);
    const float2 c = e4m3x2_to_float2(v.y, oor), d = e4m3x2_to_float2(v.y >> 16, oor);
    float s = w[0] * a.x;
    s = fmaf(w[1], a.y, s);
    s = fmaf(w[2], b.x, s);
    s = fmaf(w[3], b.y, s);
    s = fmaf(w[4], c.x, s);
    s = fmaf(w[5], c.y, s);
    s = fmaf(w[6], d.x, s);
    s = fmaf(w[7], d.y, s);
    return s;
}

// Group-reduced query weights of this lane's chunks of unit u: chunk
// lane + 32m holds kmin dims (chunk < CPR, weights Qneg) or kmax dims
// (weights Qpos).
template <int D>
__device__ __forceinline__ void load_weights(const ScoreParams& p, int u,
                                             float (&w)[TileGeom<D>::CPL][8]) {
    using C = TileGeom<D>;
    const int lane = threadIdx.x & 31;
    const int b = u / p.hkv, h = u % p.hkv;
    const __nv_bfloat16* qb =
        static_cast<const __nv_bfloat16*>(p.q) + ((long long)b * p.hq + h * p.group) * D;
#pragma unroll
    for (int m = 0; m < C::CPL; ++m) {
        const bool is_max = lane + 32 * m >= C::CPR;
        const int d0 = 8 * ((lane + 32 * m) % C::CPR);
        uint4 qv[kMaxGroup];
#pragma unroll
        for (int gq = 0; gq < kMaxGroup; ++gq)
            if (gq < p.group) qv[gq] = __ldg(reinterpret_cast<const uint4*>(qb + gq * D + d0));
#pragma unroll
        for (int e = 0; e < 8; ++e) w[m][e] = 0.f;
#pragma unroll
        for (int gq = 0; gq < kMaxGroup; ++gq) {
            if (gq < p.group) {
                const uint4 v = qv[gq];
                const float qf[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                                     bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    w[m][e] += is_max ? fmaxf(qf[e], 0.f) : fminf(qf[e], 0.f);
            }
        }
    }
}

// Physical page of lane i's page (i < 16) of tile jt of unit u, or -1 for
// a page past the candidates or a block-table entry outside the pool.
__device__ __forceinline__ int tile_phys(const ScoreParams& p, int u, const PageRanges& r,
                                         int jt) {
    const int lane = threadIdx.x & 31;
    const int j = r.np + jt * kTilePages + lane;
    int phys = -1;
    if (lane < kTilePages && j < r.ws) {
        phys = p.block_table[(long long)(u / p.hkv) * p.max_pages + j];
        if (phys < 0 || phys >= p.num_pages) {
            atomicOr(p.status, SLC_STATUS_BAD_PAGE);
            phys = -1;
        }
    }
    return phys;
}

// Score the landed tile jt of unit u (rows in `tile`) and write the page
// scores; lane i < 16 holds page i's physical page in tphys (-1: the
// block-table entry failed its check, and the page scores -inf).
template <int D, bool FP8>
__device__ __forceinline__ void score_tile(const ScoreParams& p, int u, const PageRanges& r,
                                           int jt, const uint8_t* tile,
                                           const float (&w)[TileGeom<D>::CPL][8], int tphys) {
    using C = TileGeom<D, FP8>;
    const int lane = threadIdx.x & 31;
    const uint8_t* t = tile + lane * C::CHUNK_B;
    float acc[kTilePages];
#pragma unroll
    for (int pg = 0; pg < kTilePages; ++pg) {
        float sacc = 0.f;
#pragma unroll
        for (int m = 0; m < C::CPL; ++m) {
            const uint8_t* src = t + pg * C::PAGE_B + m * 32 * C::CHUNK_B;
            if (FP8) {
                // kmin chunks (lane + 32m < CPR) read an out-of-range code as
                // -kBf16Max, kmax chunks as +kBf16Max
                const float oor = lane + 32 * m < C::CPR ? -kBf16Max : kBf16Max;
                sacc += dot8_e4m3(w[m], lds64(src), oor);
            } else {
                sacc += dot8(w[m], lds128(src));
            }
        }
        acc[pg] = sacc;
    }
    __syncwarp();  // the caller may refill the tile's buffer after this
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
    const int j = r.np + jt * kTilePages + (lane >> 1);
    const int phys = __shfl_sync(0xffffffffu, tphys, lane >> 1);
    // a page whose block-table entry failed its check scores -inf
    const float sc = phys < 0 ? -INFINITY : acc[0];
    if (j < r.ws && (lane & 1) == 0) {
        if (p.cand_stride)
            p.scores[(long long)u * p.cand_stride + (j - r.np)] = sc;
        else
            p.scores[(long long)u * p.max_pages + j] = sc;
    }
    if (p.tile_max) {  // the tile's largest key, over its candidates
        const uint32_t m = __reduce_max_sync(0xffffffffu, j < r.ws ? order_key(sc) : 0u);
        if (lane == 0) p.tile_max[(long long)u * (p.cand_stride / kTilePages) + jt] = m;
    }
}


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

// Score the tiles of warp gw of nw (tiles of all units numbered in (b, h,
// tile) order, a contiguous range per warp) through this warp's ring of NT
// tiles at `ring` (NT * TILE_B bytes), each filled by bulk copies completing
// on its mbarrier.  bars: NT mbarriers (count 1) whose next phase parity is
// `it` (ring uses so far, advanced here).  A bounded wait that gives up sets
// SLC_STATUS_WAIT_TIMEOUT; the warp then drains its copies and stops.  The
// caller has waited for the kernel that produces q, the metadata or the
// lengths.
template <int D, int NT, bool FP8>
__device__ void score_range_bulk(const ScoreParams& p, uint8_t* ring, uint64_t* bars,
                                 uint32_t& it, int gw, int nw) {
    using C = TileGeom<D, FP8>;
    const int lane = threadIdx.x & 31;
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
    int gi = g0;
    int pf = tile_phys(p, iss.u, iss.r, gi - iss.ustart);
    int sp[NT];  // page ids of the tile in each slot (lane i: page i)
    const uint8_t* meta = static_cast<const uint8_t*>(p.meta);
    // issue tile gi into stage `slot` (page ids in pf), then look one tile ahead
    auto copy_next = [&](int slot) {
        if (gi >= g_end) return;
#pragma unroll
        for (int k = 0; k < NT; ++k)
            if (k == slot) sp[k] = pf;
        const unsigned have = __ballot_sync(0xffffffffu, pf >= 0);
        if (lane == 0) {
            if (have) mbar_arrive_expect_tx(bars + slot, __popc(have) * C::PAGE_B);
            else mbar_arrive(bars + slot);
        }
        __syncwarp();
        if (pf >= 0) {
            const long long src = ((long long)pf * p.hkv + iss.u % p.hkv) * C::PAGE_B;
            bulk_g2s(ring + slot * C::TILE_B + lane * C::PAGE_B, meta + src, C::PAGE_B,
                     bars + slot);
        }
        ++gi;
        if (gi < g_end) {
            if (gi - iss.ustart >= iss.ntiles) cursor_seek(p, iss, gi);
            pf = tile_phys(p, iss.u, iss.r, gi - iss.ustart);
        }
    };
    fence_proxy_async_smem();  // earlier generic accesses of the ring first
#pragma unroll
    for (int k = 0; k < NT; ++k) copy_next((it + k) % NT);

    int wu = -1;  // unit whose weights are loaded
    float w[C::CPL][8];
    for (int g = g0; g < g_end; ++g) {
        if (g - use.ustart >= use.ntiles) cursor_seek(p, use, g);
        if (use.u != wu) {
            wu = use.u;
            load_weights<D>(p, use.u, w);
        }
        const uint32_t u_ = it + (g - g0);
        const int slot = u_ % NT;
        if (!mbar_wait_bounded(bars + slot, (u_ / NT) & 1u, 1u << 22)) {
            if (lane == 0) {
                atomicOr(p.status, SLC_STATUS_WAIT_TIMEOUT);
                for (int k = g + 1; k < g_end && k < g + NT; ++k) {
                    const uint32_t u2 = it + (k - g0);
                    mbar_wait_bounded(bars + u2 % NT, (u2 / NT) & 1u, 1u << 22);
                }
            }
            __syncwarp();
            return;
        }
        int tp = sp[0];
#pragma unroll
        for (int k = 1; k < NT; ++k)
            if (k == slot) tp = sp[k];
        score_tile<D, FP8>(p, use.u, use.r, g - use.ustart, ring + slot * C::TILE_B, w, tp);
        fence_proxy_async_smem();  // this warp's reads of the slot precede its refill
        copy_next(slot);
    }
    it += g_end - g0;
}

}  // namespace scr
}  // namespace slc
