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
// page order, of 4*D bytes (bf16) or 2*D bytes (E4M3)), brought in by
// asynchronous 16- or 8-byte copies (score_run).  Lane l owns chunks l,
// l+32, ... of every row (16 bytes = 8 bf16, or 8 bytes = 8 E4M3: the same
// 8 dims either way) and dots them with its query weights; a transposed
// butterfly (16 shuffles) then leaves page i's score in lanes 2i and 2i+1.
// (Per-page bulk copies through the TMA engine were measured slower here:
// 512-byte copies cap the read rate well below the HBM rate.)
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

// 8 bf16 of a 16-byte chunk dotted with 8 fp32 weights: one unpack per
// element and one packed two-lane FMA per pair.
__device__ __forceinline__ float dot8(const float (&w)[8], uint4 v) {
    float2 s = make_float2(bf16_lo(v.x) * w[0], bf16_hi(v.x) * w[1]);
    s = ffma2(make_float2(bf16_lo(v.y), bf16_hi(v.y)), make_float2(w[2], w[3]), s);
    s = ffma2(make_float2(bf16_lo(v.z), bf16_hi(v.z)), make_float2(w[4], w[5]), s);
    s = ffma2(make_float2(bf16_lo(v.w), bf16_hi(v.w)), make_float2(w[6], w[7]), s);
    return s.x + s.y;
}

// 8 E4M3 codes (8 bytes, low byte first) dotted with 8 fp32 weights.
__device__ __forceinline__ float dot8_e4m3(const float (&w)[8], uint2 v, float oor) {
    const float2 a = e4m3x2_to_float2(v.x, oor), b = e4m3x2_to_float2(v.x >> 16, oor);
    const float2 c = e4m3x2_to_float2(v.y, oor), d = e4m3x2_to_float2(v.y >> 16, oor);
    float2 s = make_float2(a.x * w[0], a.y * w[1]);
    s = ffma2(b, make_float2(w[2], w[3]), s);
    s = ffma2(c, make_float2(w[4], w[5]), s);
    s = ffma2(d, make_float2(w[6], w[7]), s);
    return s.x + s.y;
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


// Score tiles [j0, j1) of unit u (page ranges r) with this warp, through
// its ring of NS tiles at `ring` (NS * TILE_B bytes).  Every lane copies its
// own chunks of each page (asynchronous 16- or 8-byte copies: one warp
// instruction moves one page's row, fully coalesced), one copy group per
// tile, NS tiles in flight; each lane reads back only the chunks it copied.
// (Copies that give each lane a contiguous half row take one shuffle per
// tile instead of sixteen but coalesce worse, and measured slower.)  w: the
// unit's query weights (load_weights).  The caller has waited for the kernel
// that produces q, the metadata or the lengths, and nothing else writes the
// ring meanwhile.
template <int D, int NS, bool FP8>
__device__ void score_run(const ScoreParams& p, uint8_t* ring, int u, const PageRanges& r,
                          int j0, int j1, const float (&w)[TileGeom<D>::CPL][8]) {
    using C = TileGeom<D, FP8>;
    const int lane = threadIdx.x & 31;
    const int n = j1 - j0;
    if (n <= 0) return;
    const uint8_t* meta = static_cast<const uint8_t*>(p.meta) +
                          (long long)(u % p.hkv) * C::PAGE_B + lane * C::CHUNK_B;
    const long long page_stride = (long long)p.hkv * C::PAGE_B;
    int pf = tile_phys(p, u, r, j0);  // lane i < 16: page i of the next tile to copy
    int sp[NS];                       // the same for the tile in each slot
#pragma unroll
    for (int k = 0; k < NS; ++k) sp[k] = -1;
    // copy tile j0 + k into slot k % NS (nothing past the range), then look
    // one tile ahead; always one commit, so group k is tile k
    auto issue = [&](int k) {
        if (k < n) {
            const int slot = k % NS;
#pragma unroll
            for (int s2 = 0; s2 < NS; ++s2)
                if (s2 == slot) sp[s2] = pf;
            uint8_t* dst = ring + slot * C::TILE_B + lane * C::CHUNK_B;
#pragma unroll
            for (int pg = 0; pg < kTilePages; ++pg) {
                const int ph = __shfl_sync(0xffffffffu, pf, pg);
                if (ph >= 0) {
                    const uint8_t* src = meta + ph * page_stride;
#pragma unroll
                    for (int m = 0; m < C::CPL; ++m)
                        cp_async_chunk<C::CHUNK_B>(dst + pg * C::PAGE_B + m * 32 * C::CHUNK_B,
                                                   src + m * 32 * C::CHUNK_B);
                }
            }
            if (k + 1 < n) pf = tile_phys(p, u, r, j0 + k + 1);
        }
        cp_async_commit();
    };
#pragma unroll
    for (int k = 0; k < NS; ++k) issue(k);
    for (int k = 0; k < n; ++k) {
        cp_async_wait<NS - 1>();  // tile k (this lane's chunks) has landed
        const int slot = k % NS;
        int tp = sp[0];
#pragma unroll
        for (int s2 = 1; s2 < NS; ++s2)
            if (s2 == slot) tp = sp[s2];
        score_tile<D, FP8>(p, u, r, j0 + k, ring + slot * C::TILE_B, w, tp);
        issue(k + NS);
    }
    cp_async_wait<0>();
}

}  // namespace scr
}  // namespace slc
