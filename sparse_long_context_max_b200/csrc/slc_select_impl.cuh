// Fixed-budget page selection of one (sequence, kv head) unit by one CTA
// ("Accelerating Long-Context Decoding in Large-Scale Hybrid LLMs Without
// Retraining", abstract: a fixed budget of the most relevant tokens): keep
// the budget (k) candidate pages with the highest scores, equal scores going
// to the lower page index, and emit them in ascending page order.
//
// Built for latency.  The CTA holds every candidate score of the unit in
// registers (thread t: candidates t*KPT .. t*KPT+KPT-1, brought in by one
// bulk copy) as order-preserving uint32 keys, then:
//   1. tau <= the k-th largest of the threads' maxima (0 when fewer than k
//      threads hold candidates): the k threads with the largest maxima hold
//      k distinct keys >= that value, so tau <= T, the k-th largest key,
//      and every selected key is >= tau.  The radix search for tau works on
//      one key per thread and may stop after two digits, at the smallest key
//      with those digits, which is still such a bound;
//   2. the keys >= tau (typically little more than k) are compacted, in
//      index order, into shared memory;
//   3. an exact radix select over those survivors finds T and how many keys
//      equal to T to keep (the lowest-indexed ones), and an index-ordered
//      block scan writes the pages.
// If ties leave more survivors than shared memory holds, step 3 runs on
// the register-resident keys of every candidate instead.
//
// The radix select works on 8-bit digits from the highest bit where the
// set's smallest and largest keys differ (equal leading bits cost no pass)
// and stops as soon as the chosen digit's bin holds exactly the keys still
// wanted.
#pragma once

#include "slc_internal.h"

namespace slc {
namespace sel {


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
    static_assert(W <= 32, "one warp scans the warp totals");
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
// <= count): thread t holds keys key_at(0 .. n_t-1), n_t <= KMAX (KMAX > 0:
// unrolled, key_at reads registers; KMAX == 0: a loop).  Key 0 never
// occurs.
template <int NTHR, int KMAX, class KeyAt>
__device__ Kth radix_kth(int n_t, KeyAt key_at, int want, Scratch<NTHR>& sc, int max_passes) {
    constexpr int W = NTHR / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    if (KMAX > 0) {
#pragma unroll
        for (int k = 0; k < (KMAX > 0 ? KMAX : 1); ++k)
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
    for (int i = tid; i < 256; i += NTHR) sc.hist[0][i] = 0;
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
    const int n_warp = __reduce_max_sync(0xffffffffu, n_t);  // uniform trip count
    int hb = 31 - __clz(kmin ^ kmax);
    uint32_t mask = hb == 31 ? 0u : ~((2u << hb) - 1u);
    uint32_t prefix = kmin & mask;
    int remaining = want;
    int buf = 0;
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
        if (KMAX > 0) {
#pragma unroll
            for (int k = 0; k < (KMAX > 0 ? KMAX : 1); ++k)
                if (k < n_warp) add(k < n_t, k < n_t ? key_at(k) : 0u);
        } else {
            for (int k = 0; k < n_warp; ++k) add(k < n_t, k < n_t ? key_at(k) : 0u);
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

// Output positions, in index order, of every key > T and the first `ties`
// keys == T: emit(position, k) for thread t's keys k (consecutive in index
// order, preceding thread t+1's).
template <int NTHR, int KMAX, class KeyAt, class Emit>
__device__ void write_selected(int n_t, KeyAt key_at, uint32_t T, int ties, Scratch<NTHR>& sc,
                               Emit emit) {
    int ngt = 0, neq = 0;
    auto count = [&](int k) {
        const uint32_t v = key_at(k);
        ngt += v > T;
        neq += v == T;
    };
    if (KMAX > 0) {
#pragma unroll
        for (int k = 0; k < (KMAX > 0 ? KMAX : 1); ++k)
            if (k < n_t) count(k);
    } else {
        for (int k = 0; k < n_t; ++k) count(k);
    }
    int total;
    const int excl = block_excl_scan<NTHR>((ngt << 16) | neq, sc, &total);
    int gt_before = excl >> 16, eq_before = excl & 0xffff;
    auto place = [&](int k) {
        const uint32_t v = key_at(k);
        if (v > T) {
            emit(gt_before + min(eq_before, ties), k);
            ++gt_before;
        } else if (v == T) {
            if (eq_before < ties) emit(gt_before + eq_before, k);
            ++eq_before;
        }
    };
    if (KMAX > 0) {
#pragma unroll
        for (int k = 0; k < (KMAX > 0 ? KMAX : 1); ++k)
            if (k < n_t) place(k);
    } else {
        for (int k = 0; k < n_t; ++k) place(k);
    }
}

// Select the pages of unit u (all NTHR threads of the CTA call it; the
// unit's candidates must number at most NTHR * KPT, and a candidate-indexed
// row at most NTHR * KPT floats).  surv is shared memory for surv_cap
// survivors (keys, then candidate indices); stage holds the score row and
// bar is an mbarrier in shared memory.
template <int NTHR, int KPT>
__device__ void select_unit(const SelectParams& p, int u, Scratch<NTHR>& sc, uint32_t* surv,
                            int surv_cap, float* stage, uint64_t* bar) {
    static_assert(KPT % 4 == 0, "16-byte loads");
    const int b = u / p.hkv;
    const int tid = threadIdx.x;
    // rows by candidate (16-byte aligned, padded, at most NTHR * KPT floats):
    // one bulk copy (TMA engine) of the whole row into `stage`, issued before
    // the lengths are read -- a single CTA cannot keep that many plain loads
    // in flight
    const bool bulk = p.cand_stride > 0;
    if (bulk && tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        const uint32_t bytes = (uint32_t)p.cand_stride * 4;
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(stage, p.scores + (long long)u * p.cand_stride, bytes, bar);
    }
    // every thread; the copy must land before the CTA exits.  Returns false
    // (for every thread) if any thread's bounded wait gave up: the unit's
    // selection is then written as all -1 instead of from unlanded scores.
    auto landed = [&]() -> bool {
        __syncthreads();  // the barrier is initialised
        const bool timed_out = !mbar_wait_bounded(bar, 0, 1u << 22);
        if (__syncthreads_or(timed_out)) {
            if (tid == 0) atomicOr(p.status, SLC_STATUS_WAIT_TIMEOUT);
            mbar_wait_bounded(bar, 0, 1u << 22);  // drain the copy before leaving
            return false;
        }
        return true;
    };
    const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
    const PageRanges r = page_ranges(L, p.prefix, p.window);
    const int ncand = r.ws - r.np;
    const bool delta_mode = p.topd >= 0;  // nsel is then decided from the scores
    int nsel = min(p.budget, ncand);
    int32_t* out = p.selected + (long long)u * p.budget;

    if ((!delta_mode && nsel >= ncand) || nsel <= 0) {
        // every candidate is kept (or none: no candidate, or budget 0)
        for (int i = tid; i < p.budget; i += NTHR) out[i] = i < nsel ? r.np + i : -1;
        if (bulk) (void)landed();
        return;
    }

    // candidate c's score: rows by candidate (16-byte aligned), or by page
    const int c0 = tid * KPT;
    const int n_t = max(0, min(KPT, ncand - c0));
    float f[KPT];
    if (bulk) {
        if (!landed()) {
            for (int i = tid; i < nsel; i += NTHR) out[i] = -1;
            return;
        }
        const float4* s4 = reinterpret_cast<const float4*>(stage + c0);
#pragma unroll
        for (int q = 0; q < KPT / 4; ++q) {
            const float4 a = 4 * q < n_t ? s4[q] : make_float4(0.f, 0.f, 0.f, 0.f);
            f[4 * q] = a.x;
            f[4 * q + 1] = a.y;
            f[4 * q + 2] = a.z;
            f[4 * q + 3] = a.w;
        }
    } else {
        const float* s = p.scores + (long long)u * p.max_pages + r.np + c0;
#pragma unroll
        for (int k = 0; k < KPT; ++k) f[k] = k < n_t ? __ldcg(s + k) : 0.f;
    }
    uint32_t key[KPT];
    uint32_t kmax = 0u;
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
        key[k] = k < n_t ? order_key(f[k]) : 0u;
        kmax = max(kmax, key[k]);
    }
    if (delta_mode) {
        // top-delta ("Faster Than Flash: Fudan FFD Hits 11.6x Kernel Speedup,
        // Pushes Long-Context Decoding to 256K", section "top-delta: Tearing
        // Down "Global Synchronization" Too"): the topd best candidates and
        // every candidate within delta of the best are both prefixes of the
        // (score desc, page asc) order, so their union is the top
        // max(topd, m), m = #{s >= s_max - delta} (threshold in fp32)
        constexpr int W = NTHR / 32;
        const int lane = tid & 31, warp = tid >> 5;
        uint32_t km = __reduce_max_sync(0xffffffffu, kmax);
        if (lane == 0) sc.red_max[warp] = km;
        __syncthreads();
        km = lane < W ? sc.red_max[lane] : 0u;
        km = __reduce_max_sync(0xffffffffu, km);
        __syncthreads();  // red_max is rewritten by the searches below
        const uint32_t tk = delta_threshold_key(km, p.delta);
        int c = 0;
#pragma unroll
        for (int k = 0; k < KPT; ++k) c += k < n_t && key[k] >= tk;
        int m;
        (void)block_excl_scan<NTHR>(c, sc, &m);
        nsel = min(min(max(p.topd, m), p.budget), ncand);
        if (nsel >= ncand) {
            for (int i = tid; i < p.budget; i += NTHR) out[i] = i < ncand ? r.np + i : -1;
            return;
        }
    }
    for (int i = nsel + tid; i < p.budget; i += NTHR) out[i] = -1;

    // 1. tau from the threads' maxima
    uint32_t tau = 0u;
    if ((ncand + KPT - 1) / KPT >= nsel)
        tau = radix_kth<NTHR, 1>(n_t > 0 ? 1 : 0, [&](int) { return kmax; }, nsel, sc, 2).lower;

    // 2. survivors, compacted in index order
    int cnt = 0;
#pragma unroll
    for (int k = 0; k < KPT; ++k) cnt += k < n_t && key[k] >= tau;
    int nsurv;
    int pos = block_excl_scan<NTHR>(cnt, sc, &nsurv);
    auto emit_page = [&](int o, int page) { out[o] = page; };
    if (nsurv <= surv_cap) {
        uint32_t* skey = surv;
        int32_t* sidx = reinterpret_cast<int32_t*>(surv + surv_cap);
#pragma unroll
        for (int k = 0; k < KPT; ++k)
            if (k < n_t && key[k] >= tau) {
                skey[pos] = key[k];
                sidx[pos] = c0 + k;
                ++pos;
            }
        __syncthreads();
        // 3. exact selection among the survivors (consecutive per thread)
        const int per = (nsurv + NTHR - 1) / NTHR;
        const int base = tid * per;
        const int m = max(0, min(per, nsurv - base));
        auto skey_at = [&](int k) { return skey[base + k]; };
        const Kth t = radix_kth<NTHR, 0>(m, skey_at, nsel, sc, 0);
        write_selected<NTHR, 0>(m, skey_at, t.T, t.ties, sc,
                                [&](int o, int k) { emit_page(o, r.np + sidx[base + k]); });
    } else {
        // heavy ties: exact selection among every candidate
        auto key_at = [&](int k) { return key[k]; };
        const Kth t = radix_kth<NTHR, KPT>(n_t, key_at, nsel, sc, 0);
        write_selected<NTHR, KPT>(n_t, key_at, t.T, t.ties, sc,
                                  [&](int o, int k) { emit_page(o, r.np + c0 + k); });
    }
}

}  // namespace sel
}  // namespace slc
