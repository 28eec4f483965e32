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
// Work split: a tile is 32 consecutive candidate pages of one (sequence,
// kv head) unit.  Tiles of all units are numbered in (b, h, tile) order and
// every warp of the (persistent) grid takes a contiguous range of them.
// Within a tile each lane loads 16-byte chunks of every page's metadata
// (all 32 pages in flight), forms 32 partial dot products, and a transposed
// butterfly reduction (31 shuffles) leaves page i's score in lane i.
#include "slc_internal.h"

namespace slc {

namespace {

// 8 bf16 of a 16-byte chunk dotted with 8 fp32 weights.
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

template <int D>
__global__ void __launch_bounds__(256) score_kernel(ScoreParams p) {
    constexpr int CPR = D / 8;         // 16-byte chunks per metadata row (kmin or kmax)
    constexpr int CPL = 2 * CPR / 32;  // chunks per lane per page
    const int lane = threadIdx.x & 31;
    const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    const long long nw = (long long)gridDim.x * (blockDim.x >> 5);

    auto tiles_of = [&](int b) {
        const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
        const PageRanges r = page_ranges(L, p.prefix, p.window);
        return (r.ws - r.np + 31) / 32;
    };
    const long long total = total_units(p.batch, p.hkv, tiles_of);
    const long long per = (total + nw - 1) / nw;
    long long g = gw * per;
    const long long g_end = min(total, g + per);
    if (g >= g_end) return;

    int u;
    long long ustart;
    locate_unit(g, p.batch, p.hkv, tiles_of, &u, &ustart);

    int cur = -1;
    PageRanges r{0, 0, 0};
    int utiles = 0;
    float w[CPL][8];
    for (; g < g_end; ++g) {
        if (cur < 0 || g - ustart >= utiles) {
            if (cur >= 0) {
                ustart += utiles;
                ++u;
            }
            // skip units without candidates
            while (true) {
                const int L = checked_len(p.seq_lens, u / p.hkv, p.max_pages, p.status);
                r = page_ranges(L, p.prefix, p.window);
                utiles = (r.ws - r.np + 31) / 32;
                if (g - ustart < utiles) break;
                ustart += utiles;
                ++u;
            }
            cur = u;
            // group-reduced query weights for this lane's chunks
            const int b = u / p.hkv, h = u % p.hkv;
#pragma unroll
            for (int m = 0; m < CPL; ++m) {
                const int chunk = lane + 32 * m;
                const bool is_max = chunk >= CPR;
                const int d0 = 8 * (chunk % CPR);
#pragma unroll
                for (int e = 0; e < 8; ++e) w[m][e] = 0.f;
                // all group rows are loaded before any is used (one round trip)
                uint4 qv[kMaxGroup];
#pragma unroll
                for (int gq = 0; gq < kMaxGroup; ++gq)
                    if (gq < p.group)
                        qv[gq] = __ldg(reinterpret_cast<const uint4*>(
                            static_cast<const __nv_bfloat16*>(p.q) +
                            ((long long)b * p.hq + h * p.group + gq) * D + d0));
#pragma unroll
                for (int gq = 0; gq < kMaxGroup; ++gq) {
                    if (gq < p.group) {
                        const float qf[8] = {bf16_lo(qv[gq].x), bf16_hi(qv[gq].x), bf16_lo(qv[gq].y),
                                             bf16_hi(qv[gq].y), bf16_lo(qv[gq].z), bf16_hi(qv[gq].z),
                                             bf16_lo(qv[gq].w), bf16_hi(qv[gq].w)};
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            w[m][e] += is_max ? fmaxf(qf[e], 0.f) : fminf(qf[e], 0.f);
                    }
                }
            }
        }
        const int b = u / p.hkv, h = u % p.hkv;
        const int j = r.np + (int)(g - ustart) * 32 + lane;
        const bool valid = j < r.ws;
        int phys = valid ? p.block_table[(long long)b * p.max_pages + j] : 0;
        const bool bad = valid && (phys < 0 || phys >= p.num_pages);
        if (bad) {
            atomicOr(p.status, SLC_STATUS_BAD_PAGE);
        }
        if (!valid || bad) phys = 0;  // load something harmless, discard below

        const uint4* meta = static_cast<const uint4*>(p.meta);
        float acc[32];
        // every load of a phase is issued before the first is used: PH pages
        // x CPL chunks = 32 x 16 bytes in flight per lane
        constexpr int PH = 32 / CPL;
#pragma unroll
        for (int ph0 = 0; ph0 < 32; ph0 += PH) {
            uint4 v[PH][CPL];
#pragma unroll
            for (int i = 0; i < PH; ++i) {
                const int pg = __shfl_sync(0xffffffffu, phys, ph0 + i);
                const uint4* base = meta + ((long long)pg * p.hkv + h) * (2 * CPR);
#pragma unroll
                for (int m = 0; m < CPL; ++m) v[i][m] = __ldg(base + lane + 32 * m);
            }
#pragma unroll
            for (int i = 0; i < PH; ++i) {
                float s = 0.f;
#pragma unroll
                for (int m = 0; m < CPL; ++m) s += dot8(w[m], v[i][m]);
                acc[ph0 + i] = s;
            }
        }
        // transposed butterfly: after level `lvl`, a lane keeps the half of
        // its pages selected by lane bit `lvl`; finally acc[0] = page `lane`
#pragma unroll
        for (int lvl = 16; lvl >= 1; lvl >>= 1) {
            const bool upper = (lane & lvl) != 0;
#pragma unroll
            for (int i = 0; i < lvl; ++i) {
                const float send = upper ? acc[i] : acc[i + lvl];
                const float keep = upper ? acc[i + lvl] : acc[i];
                acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, lvl);
            }
        }
        if (valid) p.scores[(long long)u * p.max_pages + j] = bad ? -INFINITY : acc[0];
    }
}

}  // namespace

cudaError_t launch_score(const ScoreParams& p, int head_dim, int num_sms, cudaStream_t stream) {
    static int occ128 = 0, occ256 = 0;
    int& occ = head_dim == 128 ? occ128 : occ256;
    if (occ == 0) {
        cudaError_t e = head_dim == 128
                            ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, score_kernel<128>, 256, 0)
                            : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, score_kernel<256>, 256, 0);
        if (e != cudaSuccess) return e;
        if (occ < 1) occ = 1;
    }
    const int blocks = num_sms * occ;
    if (head_dim == 128)
        score_kernel<128><<<blocks, 256, 0, stream>>>(p);
    else
        score_kernel<256><<<blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace slc
