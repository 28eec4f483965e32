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
// unit; one warp scores a tile held in shared memory (16 metadata rows of
// 4*D bytes, in page order).  Lane l owns 16-byte chunks l, l+32, ... of
// every row: it copies them itself (16-byte asynchronous copies, tracked by
// its own cp.async groups) and dots them with its query weights; a
// transposed butterfly (16 shuffles) then leaves page i's score in lanes
// 2i and 2i+1.
#pragma once

#include "slc_internal.h"

namespace slc {
namespace scr {

constexpr int kTilePages = kSelTile;  // pages per tile (16)

template <int D>
struct TileGeom {
    static constexpr int CPR = D / 8;                   // chunks per metadata row
    static constexpr int CPL = 2 * CPR / 32;            // chunks per lane per page
    static constexpr int PAGE_B = 4 * D;                // metadata bytes per (page, kv head)
    static constexpr int TILE_B = kTilePages * PAGE_B;  // 8 KB / 16 KB
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

// Copy the tile of kv head h whose page ids lane i < 16 holds (phys) into
// dst (TILE_B bytes): for every page, lane l copies the 16-byte chunks l,
// l+32, ... that it later reads itself.  Commits one cp.async group.
template <int D>
__device__ __forceinline__ void copy_tile(const ScoreParams& p, int h, int phys, uint8_t* dst) {
    using C = TileGeom<D>;
    const int lane = threadIdx.x & 31;
    const uint8_t* src0 =
        static_cast<const uint8_t*>(p.meta) + (long long)h * C::PAGE_B + lane * 16;
    uint8_t* dst0 = dst + lane * 16;
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

// Score the landed tile jt of unit u (rows in `tile`) and write the page
// scores.
template <int D>
__device__ __forceinline__ void score_tile(const ScoreParams& p, int u, const PageRanges& r,
                                           int jt, const uint8_t* tile,
                                           const float (&w)[TileGeom<D>::CPL][8]) {
    using C = TileGeom<D>;
    const int lane = threadIdx.x & 31;
    const uint8_t* t = tile + lane * 16;
    float acc[kTilePages];
#pragma unroll
    for (int pg = 0; pg < kTilePages; ++pg) {
        float sacc = 0.f;
#pragma unroll
        for (int m = 0; m < C::CPL; ++m)
            sacc += dot8(w[m], lds128(t + pg * C::PAGE_B + m * 512));
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
    if (j < r.ws && (lane & 1) == 0) {
        // a page whose block-table entry failed its check scores -inf
        const int phys = p.block_table[(long long)(u / p.hkv) * p.max_pages + j];
        const float sc = (phys < 0 || phys >= p.num_pages) ? -INFINITY : acc[0];
        if (p.cand_stride)
            p.scores[(long long)u * p.cand_stride + (j - r.np)] = sc;
        else
            p.scores[(long long)u * p.max_pages + j] = sc;
    }
}

}  // namespace scr
}  // namespace slc
