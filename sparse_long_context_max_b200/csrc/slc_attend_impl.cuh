// Split-KV flash-decode building blocks of the attention kernels
// (slc_attend.cu, slc_stream.cu, slc_finish.cu): page lists, the per-warp
// streaming attention over a list, and the combine of a CTA's warp partials
// into one partial.  slc_attend.cu describes the data flow and the
// tensor-core fragment layout.
#pragma once

#include "slc_internal.h"

namespace slc {
namespace attn {

constexpr uint32_t kWaitLimit = 1u << 22;  // bounded mbarrier polls

struct Ring {
    uint8_t* tiles;  // STAGES x (K tile, V tile)
    uint64_t* bars;  // STAGES
    int* nvalid;     // STAGES
};

// A unit's list (AttendParams::list):
//   kListDense   pages 0..n-1;
//   kListForced  prefix pages, then window pages.

// Length of the list of each unit of sequence b.
__device__ __forceinline__ int list_len(const AttendParams& p, int b) {
    const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
    const PageRanges r = page_ranges(L, p.prefix, p.window);
    if (p.list == kListDense) return r.n;
    return r.np + (r.n - r.ws);
}

// Logical page of list position i of a unit.
__device__ __forceinline__ int list_page(const AttendParams& p, const PageRanges& r, int i) {
    if (p.list == kListDense || i < r.np) return i;
    return r.ws + (i - r.np);
}

// Physical page and valid-token count of logical page j of sequence b of L
// tokens; (0, 0) for a block-table entry outside the pool (flagged).
__device__ __forceinline__ void resolve_logical(const AttendParams& p, int b, int L, int j,
                                                int* phys, int* nv) {
    const int ph = p.block_table[(long long)b * p.max_pages + j];
    *phys = 0;
    *nv = 0;
    if (ph < 0 || ph >= p.num_pages) {
        atomicOr(p.status, SLC_STATUS_BAD_PAGE);
        return;
    }
    *phys = ph;
    *nv = min(kPage, L - j * kPage);
}

// Lane 0: bulk-copy the K and V tiles of (phys, h) into ring stage `stage`.
template <int D>
__device__ __forceinline__ void issue_kv(const AttendParams& p, const Ring& ring, int stage,
                                         int h, int phys, int nv) {
    constexpr uint32_t TILE = kPage * D * 2;
    ring.nvalid[stage] = nv;
    uint64_t* bar = ring.bars + stage;
    if (nv <= 0) {  // nothing to read: complete the phase without a copy
        mbar_arrive(bar);
        return;
    }
    mbar_arrive_expect_tx(bar, 2 * TILE);
    const long long off = ((long long)phys * p.hkv + h) * (kPage * D);
    uint8_t* dst = ring.tiles + stage * 2 * TILE;
    bulk_g2s(dst, static_cast<const __nv_bfloat16*>(p.k_cache) + off, TILE, bar);
    bulk_g2s(dst + TILE, static_cast<const __nv_bfloat16*>(p.v_cache) + off, TILE, bar);
}

// Per-warp partial state: the running max of head r_ (log2 units), this
// thread's share of the running sum, and the O^T accumulators of heads 2c,
// 2c+1 over dims (D/8)*r_ .. (D/8)*r_ + D/8 - 1.
template <int D>
struct WarpState {
    float m, l;
    float acc[D / 16][4];
};

// Attend list positions i0, i0 + stride, ... < i1 of unit u (sequence b of
// L tokens, kv head h) with this warp's ring; resolve(i, &phys, &nv) gives
// the physical page and valid tokens of position i (nv = 0: skip it).  `it`
// counts the warp's ring uses (stage = it % STAGES).  `ok` turns false if a
// bounded wait gave up; the warp then drains its copies in flight and skips
// all further work (it still reaches every CTA barrier).
template <int D, int STAGES, class Resolve>
__device__ void warp_attend(const AttendParams& p, const Ring& ring, uint32_t& it, bool& ok,
                            int b, int h, int i0, int i1, int stride, WarpState<D>& st,
                            Resolve resolve) {
    constexpr int TILE_W = kPage * D / 2;  // 32-bit words per tile
    constexpr int ROW_W = D / 2;           // words per token row
    constexpr int KS = D / 16;             // k-steps of Q K^T, m-blocks of V^T P^T
    const int lane = threadIdx.x & 31;
    const int r_ = lane >> 2, c_ = lane & 3;
    const int G = p.group;
    st.m = -INFINITY;
    st.l = 0.f;
#pragma unroll
    for (int i = 0; i < KS; ++i) st.acc[i][0] = st.acc[i][1] = st.acc[i][2] = st.acc[i][3] = 0.f;
    const int npg = i1 > i0 ? (i1 - i0 + stride - 1) / stride : 0;
    if (!ok || npg == 0) return;

    // page ids of this warp's pages, 32 at a time: lane t holds page k0 + t
    int id_phys = 0, id_nv = 0;
    auto load_ids = [&](int k0) {
        const int k = k0 + lane;
        if (k < npg) resolve(i0 + k * stride, &id_phys, &id_nv);
    };
    load_ids(0);
    __syncwarp();  // this warp's earlier reads of the ring are done
    fence_proxy_async_smem();
    for (int k = 0; k < STAGES && k < npg; ++k) {
        const int ph = __shfl_sync(0xffffffffu, id_phys, k);
        const int nv = __shfl_sync(0xffffffffu, id_nv, k);
        if (lane == 0) issue_kv<D>(p, ring, (it + k) % STAGES, h, ph, nv);
    }
    __syncwarp();

    // query fragments (rows >= G and rows 8..15 are zero)
    uint32_t qa[KS][2];
    if (r_ < G) {
        const uint4* qrow = reinterpret_cast<const uint4*>(
            static_cast<const __nv_bfloat16*>(p.q) + ((long long)b * p.hq + h * G + r_) * D);
#pragma unroll
        for (int m = 0; m < D / 32; ++m) {
            const uint4 v = __ldg(qrow + c_ + 4 * m);
            qa[2 * m][0] = v.x;
            qa[2 * m][1] = v.y;
            qa[2 * m + 1][0] = v.z;
            qa[2 * m + 1][1] = v.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < KS; ++k) qa[k][0] = qa[k][1] = 0u;
    }

    for (int k = 0; k < npg; ++k) {
        const uint32_t use = it + k;
        const int stage = use % STAGES;
        if (!mbar_wait_bounded(ring.bars + stage, (use / STAGES) & 1u, kWaitLimit)) {
            if (lane == 0) {
                atomicOr(p.status, SLC_STATUS_WAIT_TIMEOUT);
                for (int kk = k; kk < npg && kk < k + STAGES; ++kk) {
                    const uint32_t u2 = it + kk;
                    mbar_wait_bounded(ring.bars + u2 % STAGES, (u2 / STAGES) & 1u, kWaitLimit);
                }
            }
            __syncwarp();
            ok = false;
            return;
        }
        const int nv = ring.nvalid[stage];
        if (nv > 0) {
            const uint32_t* Kw =
                reinterpret_cast<const uint32_t*>(ring.tiles) + stage * 2 * TILE_W;
            const uint32_t* Vw = Kw + TILE_W;

            // S = Q K^T for tokens nb*8 + (0..7): two accumulators per block
            // (even and odd k-steps) halve the dependent chain of mma
            float s[2][4];
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                float s2[4] = {0.f, 0.f, 0.f, 0.f};
                s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
                const uint32_t* krow = Kw + (nb * 8 + r_) * ROW_W;
#pragma unroll
                for (int m = 0; m < D / 32; ++m) {
                    const uint4 kv = lds128(krow + (c_ + 4 * m) * 4);
                    mma_bf16(s[nb], qa[2 * m][0], 0u, qa[2 * m][1], 0u, kv.x, kv.y);
                    mma_bf16(s2, qa[2 * m + 1][0], 0u, qa[2 * m + 1][1], 0u, kv.z, kv.w);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) s[nb][e] += s2[e];
            }
            // this thread: head r_, tokens 2c, 2c+1, 8+2c, 9+2c
            const int t0 = 2 * c_;
            float x[4];
            x[0] = t0 < nv ? s[0][0] * p.scale_log2 : -INFINITY;
            x[1] = t0 + 1 < nv ? s[0][1] * p.scale_log2 : -INFINITY;
            x[2] = t0 + 8 < nv ? s[1][0] * p.scale_log2 : -INFINITY;
            x[3] = t0 + 9 < nv ? s[1][1] * p.scale_log2 : -INFINITY;
            float pmax = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
            pmax = fmaxf(pmax, __shfl_xor_sync(0xffffffffu, pmax, 1));
            pmax = fmaxf(pmax, __shfl_xor_sync(0xffffffffu, pmax, 2));
            const float m_new = fmaxf(st.m, pmax);
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            const float alpha = ex2(st.m - m_use);
            float pr[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) pr[e] = ex2(x[e] - m_use);
            st.l = st.l * alpha + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
            st.m = m_new;
            if (__any_sync(0xffffffffu, alpha != 1.f)) {  // some head's maximum moved
                const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * c_);
                const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * c_ + 4);
#pragma unroll
                for (int i = 0; i < KS; ++i) {
                    st.acc[i][0] *= a0;
                    st.acc[i][1] *= a1;
                    st.acc[i][2] *= a0;
                    st.acc[i][3] *= a1;
                }
            }
            // P^T fragments (tokens 2c,2c+1 / 2c+8,2c+9 of head r_), hi + lo
            const uint32_t bh0 = pack_bf16x2(pr[0], pr[1]);
            const uint32_t bh1 = pack_bf16x2(pr[2], pr[3]);
            const uint32_t bl0 = pack_bf16x2(pr[0] - bf16_lo(bh0), pr[1] - bf16_hi(bh0));
            const uint32_t bl1 = pack_bf16x2(pr[2] - bf16_lo(bh1), pr[3] - bf16_hi(bh1));

            // V rows of tokens 2c, 2c+1, 2c+8, 2c+9, dims (D/8)*r_ .. +D/8
            constexpr int WPT = D / 16;  // words per token per thread
            uint32_t vw[4][WPT];
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
                const int tok = t0 + (tt & 1) + (tt >> 1) * 8;
                const uint32_t* vrow = Vw + tok * ROW_W + WPT * r_;
#pragma unroll
                for (int q4 = 0; q4 < WPT / 4; ++q4) {
                    const uint4 v = lds128(vrow + 4 * q4);
                    vw[tt][4 * q4 + 0] = v.x;
                    vw[tt][4 * q4 + 1] = v.y;
                    vw[tt][4 * q4 + 2] = v.z;
                    vw[tt][4 * q4 + 3] = v.w;
                }
            }
            if (nv < kPage) {  // partial page: zero slots past the length (may hold NaN)
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    const bool live = t0 + (tt & 1) + (tt >> 1) * 8 < nv;
#pragma unroll
                    for (int i = 0; i < WPT; ++i) vw[tt][i] = live ? vw[tt][i] : 0u;
                }
            }
#pragma unroll
            for (int i = 0; i < KS; ++i) {
                const uint32_t a0r = __byte_perm(vw[0][i], vw[1][i], 0x5410);
                const uint32_t a1r = __byte_perm(vw[0][i], vw[1][i], 0x7632);
                const uint32_t a2r = __byte_perm(vw[2][i], vw[3][i], 0x5410);
                const uint32_t a3r = __byte_perm(vw[2][i], vw[3][i], 0x7632);
                mma_bf16(st.acc[i], a0r, a1r, a2r, a3r, bh0, bh1);
                mma_bf16(st.acc[i], a0r, a1r, a2r, a3r, bl0, bl1);
            }
        }
        __syncwarp();
        const int kn = k + STAGES;
        if (kn < npg) {  // refill this stage (warp-uniform branch)
            if ((kn & 31) == 0) load_ids(kn);
            const int ph = __shfl_sync(0xffffffffu, id_phys, kn & 31);
            const int nv2 = __shfl_sync(0xffffffffu, id_nv, kn & 31);
            if (lane == 0) {
                fence_proxy_async_smem();
                issue_kv<D>(p, ring, stage, h, ph, nv2);
            }
        }
    }
    it += npg;
    // full sum of head r_ (the four threads of a quad hold parts of it)
    st.l += __shfl_xor_sync(0xffffffffu, st.l, 1);
    st.l += __shfl_xor_sync(0xffffffffu, st.l, 2);
}

// Combine the NW warp partials of one unit piece (each warp's WarpState,
// staged through its own ring, which must be idle) into one partial and hand
// it to store(g, d4, num, M, den) (num: float4 of dims 4*d4.., unnormalised;
// M: max in log2 units; den: sum).  Called by every thread of the CTA;
// store runs for every (g, d4), g < group, spread over the threads.
template <int D, int NW, int RING, int NT = NW * 32, class Store>
__device__ __forceinline__ void cta_combine(const AttendParams& p, uint8_t* smem,
                                            const WarpState<D>& st, Store store) {
    constexpr int KS = D / 16;
    constexpr int DPT = D / 8;
    static_assert(RING >= (kMaxGroup * D + 2 * kMaxGroup) * 4, "ring holds a warp partial");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r_ = lane >> 2, c_ = lane & 3;
    const int G = p.group;
    __syncthreads();  // every warp is done with its ring
    float* wacc = reinterpret_cast<float*>(smem + warp * RING);     // [G][D]
    float2* wml = reinterpret_cast<float2*>(wacc + kMaxGroup * D);  // [G]
    // warps NW.. (threads beyond the attending warps) hold no partial
    if (warp < NW && c_ == 0 && r_ < G) wml[r_] = make_float2(st.m, st.l);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int head = 2 * c_ + hh;
        if (warp < NW && head < G) {
            float4* dst = reinterpret_cast<float4*>(wacc + head * D + DPT * r_);
#pragma unroll
            for (int i2 = 0; i2 < KS / 2; ++i2)
                dst[i2] = make_float4(st.acc[2 * i2][hh], st.acc[2 * i2][2 + hh],
                                      st.acc[2 * i2 + 1][hh], st.acc[2 * i2 + 1][2 + hh]);
        }
    }
    __syncthreads();
    for (int item = threadIdx.x; item < G * (D / 4); item += NT) {
        const int g = item / (D / 4), d4 = item % (D / 4);
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float2 ml = reinterpret_cast<const float2*>(
                reinterpret_cast<const float*>(smem + w * RING) + kMaxGroup * D)[g];
            M = fmaxf(M, ml.x);
        }
        const float Mu = M == -INFINITY ? 0.f : M;
        float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
        float den = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float* wa = reinterpret_cast<const float*>(smem + w * RING);
            const float2 ml = reinterpret_cast<const float2*>(wa + kMaxGroup * D)[g];
            const float wt = ex2(ml.x - Mu);
            const float4 a = reinterpret_cast<const float4*>(wa + g * D)[d4];
            num.x = fmaf(wt, a.x, num.x);
            num.y = fmaf(wt, a.y, num.y);
            num.z = fmaf(wt, a.z, num.z);
            num.w = fmaf(wt, a.w, num.w);
            den = fmaf(wt, ml.y, den);
        }
        store(g, d4, num, M, den);
    }
    __syncthreads();  // the rings are reused afterwards
}

// Attend positions [s, e) of the concatenated lists of all units with the
// CTA's NW warps (each warp: ring of STAGES stages at smem + warp * RING).
// Every unit piece yields one partial, stored in slot unit + chunk.  The
// caller has waited for the preceding kernel (which may write the cache, or
// read the partial slots).
template <int D, int NW, int STAGES>
__device__ __forceinline__ void attend_range(const AttendParams& p, uint8_t* smem,
                                             const Ring& ring, uint32_t& it, bool& ok,
                                             long long s, long long e, long long chunk) {
    constexpr int RING = STAGES * 2 * kPage * D * 2;
    const int warp = threadIdx.x >> 5;
    if (s >= e) return;
    auto len_of = [&](int b) { return list_len(p, b); };
    int u;
    long long ustart;
    locate_unit(s, p.batch, p.hkv, len_of, &u, &ustart);
    WarpState<D> st;
    while (s < e) {
        const int b = u / p.hkv, h = u % p.hkv;
        const int len = list_len(p, b);
        if (len == 0) {
            ++u;
            continue;
        }
        const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
        const PageRanges r = page_ranges(L, p.prefix, p.window);
        const int i0 = (int)(s - ustart);
        const int i1 = (int)(min(e, ustart + len) - ustart);
        warp_attend<D, STAGES>(p, ring, it, ok, b, h, i0 + warp, i1, NW, st,
                               [&](int i, int* phys, int* nv) {
                                   resolve_logical(p, b, L, list_page(p, r, i), phys, nv);
                               });
        const long long slot = u + chunk;
        cta_combine<D, NW, RING>(p, smem, st, [&](int g, int d4, float4 num, float M, float den) {
            reinterpret_cast<float4*>(p.part_acc + (slot * p.group + g) * D)[d4] = num;
            if (d4 == 0) p.part_ml[slot * p.group + g] = make_float2(M, den);
        });
        s = ustart + len;
        ustart = s;
        ++u;
    }
}

// Start of unit u's list in the concatenation of all units' lists
// (warp-wide; every lane gets the result).
__device__ __forceinline__ long long unit_list_start(const AttendParams& p, int u) {
    const int lane = threadIdx.x & 31;
    const int b = u / p.hkv, h = u % p.hkv;
    long long base = 0;
    for (int b0 = 0; b0 < b; b0 += 32) {
        const int bb = b0 + lane;
        long long c = bb < b ? (long long)list_len(p, bb) * p.hkv : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        base += c;
    }
    return base + (long long)h * list_len(p, b);
}

// The streaming kernel's split of its grid (slc_stream.cu): the first
// forced_ctas(...) CTAs attend the prefix/window lists (one chunk each), the
// others score the candidate tiles, so the two run side by side.  A forced
// page (K + V) and a 16-page bf16 metadata tile are both 64*D bytes; the
// CTAs are split so that both sides end together (a tile costs a CTA about
// 1.5 pages' time), with at least one CTA for a non-empty side and at least
// kMinForcedPages pages per attending CTA.
// Warp-wide (every lane gets the result); the finishing
// kernel recomputes it to find the prefix/window partials.
constexpr int kMinForcedPages = 8;

__device__ __forceinline__ int forced_ctas(const AttendParams& a, bool scoring, int grid) {
    auto forced_of = [&](int b) { return list_len(a, b); };
    auto tiles_of = [&](int b) {
        const int L = checked_len(a.seq_lens, b, a.max_pages, a.status);
        const PageRanges r = page_ranges(L, a.prefix, a.window);
        return (r.ws - r.np + kSelTile - 1) / kSelTile;
    };
    // a CTA attends about 1.5x the bytes per unit time that it scores
    // (measured at 64k and 256k), so a tile weighs 3 and a page 2
    const long long pages = total_units(a.batch, a.hkv, forced_of);
    const long long f = 2 * pages;
    const long long t = scoring ? 3 * total_units(a.batch, a.hkv, tiles_of) : 0;
    if (f == 0) return t == 0 ? grid : 0;
    long long n = t == 0 ? grid : (f * grid + (f + t) / 2) / (f + t);
    // at least kMinForcedPages pages per attending CTA: fewer, fuller chunks
    // (each chunk of a unit's list is one partial for the finishing kernel)
    n = min(n, (pages + kMinForcedPages - 1) / kMinForcedPages);
    if (n < 1) n = 1;
    if (t > 0 && n > grid - 1) n = grid - 1;
    return (int)n;
}

// Fold the split partial of slot `slot` (head g, dims 4*d4..) into an
// online log-sum-exp accumulation (M: running max in log2 units).
__device__ __forceinline__ void fold_partial(float2 ml, float4 a, float& M, float4& num,
                                             float& den) {
    if (ml.x == -INFINITY) return;  // empty partial
    if (ml.x > M) {                 // new maximum: rescale what was summed so far
        const float c = ex2(M - ml.x);
        num.x *= c;
        num.y *= c;
        num.z *= c;
        num.w *= c;
        den *= c;
        M = ml.x;
    }
    const float w = ex2(ml.x - M);
    num.x = fmaf(w, a.x, num.x);
    num.y = fmaf(w, a.y, num.y);
    num.z = fmaf(w, a.z, num.z);
    num.w = fmaf(w, a.w, num.w);
    den = fmaf(w, ml.y, den);
}

}  // namespace attn
}  // namespace slc
