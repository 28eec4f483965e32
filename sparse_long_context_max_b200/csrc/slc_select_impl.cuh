// Fixed-budget page selection of one (sequence, kv head) unit by one CTA,
// shared by the selection kernel (slc_select.cu) and the fused sparse
// decode (slc_fused.cu).  Keeps the budget candidate pages with the highest
// scores, equal scores going to the lower page index, and emits them in
// ascending page order ("Accelerating Long-Context Decoding in Large-Scale
// Hybrid LLMs Without Retraining", abstract: a fixed budget of the most
// relevant tokens).
//
// Scores become order-preserving uint32 keys.  Exact selection in two
// levels, built for latency (few dependent memory round trips, few block
// barriers):
//   1. the maximum key of every 16-candidate tile (written by the scoring
//      code, or computed here from the scores): one round trip;
//   2. tau <= the k-th largest tile maximum (k = budget; 0 when there are
//      fewer tiles than the budget).  The k tiles whose maxima are >= that
//      value hold k distinct pages >= tau, so tau <= T, the k-th largest
//      page key: every selected page is >= tau.  The radix search for tau
//      stops after two digits, at the smallest key with the digits found,
//      which is still such a bound;
//   3. the live tiles (maximum >= tau) are listed in index order and their
//      scores read, two tiles per thread per round trip; the pages >= tau
//      (typically little more than the budget) are compacted in index order
//      into shared memory;
//   4. an exact radix select over those survivors finds T and how many keys
//      equal to T to keep (the lowest-indexed ones), and an index-ordered
//      scan writes the result.
// If ties leave more survivors than shared memory holds, steps 3-4 stream
// over every candidate instead, re-reading the scores (cached in L2).
//
// The radix select works on 8-bit digits from the highest bit where the
// set's smallest and largest keys differ, so equal leading bits cost no
// pass, and stops as soon as the chosen digit's bin holds exactly the keys
// still wanted.  Scores and tile maxima are read through L2
// (ld.global.cg): in the fused decode they are written by other CTAs of the
// same grid.
#pragma once

#include "slc_internal.h"

namespace slc {
namespace sel {

constexpr int kTile = kSelTile;  // candidates per tile
constexpr int kMaxTiles = kMaxCandidates / kTile;
constexpr int kLiveBytes = kMaxTiles * (int)sizeof(int);  // live-tile list
constexpr int kLivePerThread = 2;  // live tiles read per thread per round

__device__ __forceinline__ uint32_t order_key(float f) {
    if (f == 0.f) f = 0.f;  // -0 and +0 tie
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int NTHR>
struct Scratch {
    static constexpr int W = NTHR / 32;
    int hist[2][256];
    uint32_t red_min[W], red_max[W];
    int scan[W];
    int digit, above, count, total;
};

// Block-wide exclusive scan of one int per thread; *total = the sum.
template <int NTHR>
__device__ __forceinline__ int block_excl_scan(int v, Scratch<NTHR>& sc, int* total) {
    constexpr int W = NTHR / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int incl = warp_incl_scan(v);
    if (lane == 31) sc.scan[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < W ? sc.scan[lane] : 0;
        const int wi = warp_incl_scan(w);
        if (lane < W) sc.scan[lane] = wi - w;
        if (lane == W - 1) sc.total = wi;
    }
    __syncthreads();
    const int r = sc.scan[warp] + incl - v;
    *total = sc.total;
    __syncthreads();
    return r;
}

// Result of a k-th largest search: the k largest keys are exactly those
// > T plus the first `ties` keys == T (in index order), and lower <= the
// k-th largest key.  A search cut short by max_passes gives `lower` only.
struct Kth {
    uint32_t T;
    int ties;
    uint32_t lower;
};

// Radix search for the `want`-th largest key held by the block (1 <= want
// <= count): thread t holds keys key_at(0 .. n_t-1) (n_t <= KMAX when
// UNROLL: key_at reads a register array).  Key 0 never occurs.
template <int NTHR, int KMAX, bool UNROLL, class KeyAt>
__device__ Kth radix_kth(int n_t, KeyAt key_at, int want, Scratch<NTHR>& sc, int max_passes) {
    constexpr int W = NTHR / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    if (UNROLL) {
#pragma unroll
        for (int k = 0; k < KMAX; ++k)
            if (k < n_t) {
                kmin = min(kmin, key_at(k));
                kmax = max(kmax, key_at(k));
            }
    } else {
        for (int k = 0; k < n_t; ++k) {
            const uint32_t v = key_at(k);
            kmin = min(kmin, v);
            kmax = max(kmax, v);
        }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
        sc.red_min[warp] = kmin;
        sc.red_max[warp] = kmax;
    }
    __syncthreads();
    kmin = lane < W ? sc.red_min[lane] : 0xffffffffu;
    kmax = lane < W ? sc.red_max[lane] : 0u;
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    Kth r{kmin, want, kmin};  // every key equal: the first `want` of them
    if (kmin == kmax) {
        __syncthreads();  // red_min/red_max are rewritten by the next call
        return r;
    }
    int hb = 31 - __clz(kmin ^ kmax);
    uint32_t mask = hb == 31 ? 0u : ~((2u << hb) - 1u);
    uint32_t prefix = kmin & mask;
    int remaining = want;
    int buf = 0;
    for (int i = tid; i < 256; i += NTHR) sc.hist[0][i] = 0;
    __syncthreads();
    for (int pass = 1;; ++pass) {
        const int shift = max(hb - 7, 0);
        const uint32_t dmask = (1u << (hb - shift + 1)) - 1u;
        int* hist = sc.hist[buf];
        for (int i = tid; i < 256; i += NTHR) sc.hist[buf ^ 1][i] = 0;  // next pass
        // keys crowd into few bins (a narrow bulk plus outliers that set the
        // range), so lanes with the same bin add once, together
        auto add = [&](bool in, uint32_t v) {
            const bool hit = in && (v & mask) == prefix;
            const int bin = hit ? (int)((v >> shift) & dmask) : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, bin);
            if (hit && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
        };
        if (UNROLL) {
#pragma unroll
            for (int k = 0; k < KMAX; ++k) add(k < n_t, key_at(k));
        } else {
            const int n_warp = __reduce_max_sync(0xffffffffu, n_t);  // uniform trip count
            for (int k = 0; k < n_warp; ++k) {
                const bool in = k < n_t;
                add(in, in ? key_at(k) : 0u);
            }
        }
        __syncthreads();
        if (warp == 0) {
            int c[8], local = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c[i] = hist[lane * 8 + i];
                local += c[i];
            }
            int suf = local;  // keys in bins >= 8*lane
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += t;
            }
            const int above = suf - local;
            if (above < remaining && suf >= remaining) {
                int cum = above;
#pragma unroll
                for (int i = 7; i >= 0; --i) {
                    if (cum + c[i] >= remaining) {
                        sc.digit = lane * 8 + i;
                        sc.above = cum;
                        sc.count = c[i];
                        break;
                    }
                    cum += c[i];
                }
            }
        }
        __syncthreads();
        remaining -= sc.above;
        prefix |= (uint32_t)sc.digit << shift;
        mask |= dmask << shift;
        const int count = sc.count;
        if (count == remaining && prefix != 0u) {
            // every key of the bin is wanted: all keys >= prefix, none below
            r = Kth{prefix - 1u, 0, prefix};
            break;
        }
        if (shift == 0) {
            r = Kth{prefix, remaining, prefix};
            break;
        }
        if (pass == max_passes) {
            r = Kth{prefix, 0, prefix};
            break;
        }
        hb = shift - 1;
        buf ^= 1;
        // sc.digit/above/count are rewritten only after the next pass's
        // atomics barrier, which every thread reaches after reading them
    }
    __syncthreads();
    return r;
}

// Write, in index order, every key > T and the first `ties` keys == T.
// Thread t's keys are consecutive in index order and precede thread t+1's.
template <int NTHR, class KeyAt, class PageAt>
__device__ void write_selected(int n_t, KeyAt key_at, PageAt page_at, uint32_t T, int ties,
                               Scratch<NTHR>& sc, int32_t* out) {
    int ngt = 0, neq = 0;
    for (int k = 0; k < n_t; ++k) {
        const uint32_t v = key_at(k);
        ngt += v > T;
        neq += v == T;
    }
    int total;
    const int excl = block_excl_scan<NTHR>((ngt << 16) | neq, sc, &total);
    int gt_before = excl >> 16, eq_before = excl & 0xffff;
    for (int k = 0; k < n_t; ++k) {
        const uint32_t v = key_at(k);
        if (v > T) {
            out[gt_before + min(eq_before, ties)] = page_at(k);
            ++gt_before;
        } else if (v == T) {
            if (eq_before < ties) out[gt_before + eq_before] = page_at(k);
            ++eq_before;
        }
    }
}

// Select the pages of unit u (all threads of the CTA call it).  buf is
// shared memory of buf_bytes (16-byte aligned): the live-tile list, then
// the survivors.
template <int NTHR>
__device__ void select_unit(const SelectParams& p, int u, uint8_t* buf, int buf_bytes,
                            Scratch<NTHR>& sc) {
    constexpr int TPT = kMaxTiles / NTHR;  // tiles per thread
    static_assert(TPT * NTHR == kMaxTiles && TPT % 4 == 0, "tile coverage");
    int* live_tile = reinterpret_cast<int*>(buf);
    const int surv_cap = (buf_bytes - kLiveBytes) / 8;
    uint32_t* surv_key = reinterpret_cast<uint32_t*>(buf + kLiveBytes);
    int32_t* surv_page = reinterpret_cast<int32_t*>(surv_key + surv_cap);

    const int b = u / p.hkv;
    const int tid = threadIdx.x;
    const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
    const PageRanges r = page_ranges(L, p.prefix, p.window);
    const int ncand = r.ws - r.np;
    const int nsel = min(p.budget, ncand);
    int32_t* out = p.selected + (long long)u * p.budget;

    if (nsel >= ncand) {  // every candidate is kept (also covers ncand == 0)
        for (int i = tid; i < p.budget; i += NTHR) out[i] = i < ncand ? r.np + i : -1;
        return;
    }
    for (int i = nsel + tid; i < p.budget; i += NTHR) out[i] = -1;
    if (nsel <= 0) return;

    // candidate c's score: rows by candidate, or by page
    const float* s = p.cand_stride ? p.scores + (long long)u * p.cand_stride
                                   : p.scores + (long long)u * p.max_pages + r.np;
    auto cand_key = [&](int c) { return order_key(__ldcg(s + c)); };
    const int ntiles = (ncand + kTile - 1) / kTile;
    const int t0 = tid * TPT;  // this thread's first tile
    const int nt_own = max(0, min(TPT, ntiles - t0));

    // 1. tile maxima
    uint32_t tk[TPT];
    if (p.tile_max) {
        const float4* tm =
            reinterpret_cast<const float4*>(p.tile_max + (long long)u * p.tile_stride);
#pragma unroll
        for (int q = 0; q < TPT / 4; ++q) {
            const float4 a =
                t0 + 4 * q < ntiles ? __ldcg(tm + t0 / 4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float v[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) tk[4 * q + k] = 4 * q + k < nt_own ? order_key(v[k]) : 0u;
        }
    } else {
#pragma unroll
        for (int k = 0; k < TPT; ++k) tk[k] = 0u;
        for (int k = 0; k < nt_own; ++k) {
            const int c0 = (t0 + k) * kTile;
            uint32_t m = 0u;
            uint32_t v[kTile];  // one tile's loads in flight together
#pragma unroll
            for (int i = 0; i < kTile; ++i) v[i] = c0 + i < ncand ? cand_key(c0 + i) : 0u;
#pragma unroll
            for (int i = 0; i < kTile; ++i) m = max(m, v[i]);
            // registers indexed by a runtime k: select into place
#pragma unroll
            for (int kk = 0; kk < TPT; ++kk)
                if (kk == k) tk[kk] = m;
        }
    }

    // 2. tau: at most the nsel-th largest tile maximum (0 keeps every page)
    uint32_t tau = 0u;
    if (ntiles >= nsel)
        tau = radix_kth<NTHR, TPT, true>(nt_own, [&](int k) { return tk[k]; }, nsel, sc, 2).lower;

    // 3. survivors: pages >= tau, from the live tiles (maximum >= tau)
    int nlive_own = 0;
#pragma unroll
    for (int k = 0; k < TPT; ++k) nlive_own += k < nt_own && tk[k] >= tau;
    int nlive;
    int lpos = block_excl_scan<NTHR>(nlive_own, sc, &nlive);
#pragma unroll
    for (int k = 0; k < TPT; ++k)
        if (k < nt_own && tk[k] >= tau) live_tile[lpos++] = t0 + k;
    __syncthreads();
    int nsurv = 0;
    bool overflow = false;
    for (int r0 = 0; r0 < nlive; r0 += NTHR * kLivePerThread) {  // uniform trip count
        uint32_t v[kLivePerThread][kTile];
        int c0[kLivePerThread];
        int cnt = 0;
#pragma unroll
        for (int m = 0; m < kLivePerThread; ++m) {
            const int li = r0 + tid * kLivePerThread + m;  // consecutive per thread
            c0[m] = li < nlive ? live_tile[li] * kTile : ncand;
#pragma unroll
            for (int i = 0; i < kTile; ++i)
                v[m][i] = c0[m] + i < ncand ? cand_key(c0[m] + i) : 0u;
        }
#pragma unroll
        for (int m = 0; m < kLivePerThread; ++m)
#pragma unroll
            for (int i = 0; i < kTile; ++i) cnt += v[m][i] >= tau && v[m][i] != 0u;
        int total;
        int pos = nsurv + block_excl_scan<NTHR>(cnt, sc, &total);
        if (nsurv + total > surv_cap) overflow = true;
        if (!overflow) {
#pragma unroll
            for (int m = 0; m < kLivePerThread; ++m)
#pragma unroll
                for (int i = 0; i < kTile; ++i)
                    if (v[m][i] >= tau && v[m][i] != 0u) {
                        surv_key[pos] = v[m][i];
                        surv_page[pos] = r.np + c0[m] + i;
                        ++pos;
                    }
        }
        nsurv += total;
    }

    if (!overflow) {
        __syncthreads();
        // 4. exact selection among the survivors (consecutive per thread)
        const int per = (nsurv + NTHR - 1) / NTHR;
        const int base = tid * per;
        const int n_t = max(0, min(per, nsurv - base));
        auto key_at = [&](int k) { return surv_key[base + k]; };
        const Kth t = radix_kth<NTHR, 0, false>(n_t, key_at, nsel, sc, 0);
        write_selected<NTHR>(n_t, key_at, [&](int k) { return surv_page[base + k]; }, t.T,
                             t.ties, sc, out);
    } else {
        // heavy ties: stream over every candidate, thread t owning a
        // contiguous range, re-reading scores for each pass
        const int per = (ncand + NTHR - 1) / NTHR;
        const int base = tid * per;
        const int n_t = max(0, min(per, ncand - base));
        auto key_at = [&](int k) { return cand_key(base + k); };
        const Kth t = radix_kth<NTHR, 0, false>(n_t, key_at, nsel, sc, 0);
        write_selected<NTHR>(n_t, key_at, [&](int k) { return r.np + base + k; }, t.T, t.ties,
                             sc, out);
    }
}

}  // namespace sel
}  // namespace slc
