// Fixed-budget page selection: per (sequence, kv head) keep the budget
// candidate pages with the highest scores, equal scores going to the lower
// page index, and emit them in ascending page order ("Accelerating
// Long-Context Decoding in Large-Scale Hybrid LLMs Without Retraining",
// abstract: a fixed budget of the most relevant tokens).
//
// One 256-thread CTA per unit.  Scores become order-preserving uint32 keys.
// Exact selection in two levels:
//   1. the maximum key of every 16-candidate tile (written by the scoring
//      kernel, or computed here from the scores); thread t owns tiles
//      8t .. 8t+7;
//   2. tau = the k-th largest tile maximum (k = budget; tau = -inf when
//      there are fewer tiles than the budget).  The k tiles whose maxima
//      are >= tau hold k distinct pages >= tau, so tau <= T, the k-th
//      largest page key: every selected page is >= tau;
//   3. the pages >= tau (typically little more than the budget) are
//      compacted in index order into shared memory;
//   4. an exact radix select over those survivors finds T and how many keys
//      equal to T to keep (the lowest-indexed ones), and an index-ordered
//      scan writes the result.
// If ties leave more survivors than shared memory holds, steps 3-4 stream
// over every candidate instead, re-reading the scores (cached in L2).
//
// The radix select works on 8-bit digits from the highest bit where the
// set's smallest and largest keys differ, so equal leading bits cost no pass.
#include "slc_internal.h"

namespace slc {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTile = kSelTile;      // candidates per tile
constexpr int kTilesPerThread = 8;   // tiles <= 2048: candidates <= 32768
constexpr int kSurvivorCap = 8192;   // survivors held in shared memory
static_assert(kThreads * kTilesPerThread * kTile >= kMaxCandidates, "tile coverage");

__device__ __forceinline__ uint32_t order_key(float f) {
    if (f == 0.f) f = 0.f;  // -0 and +0 tie
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Scratch {
    int hist[2][256];
    uint32_t red_min[kWarps], red_max[kWarps];
    int scan[kWarps];
    int digit, above, total;
};

// Block-wide exclusive scan of one int per thread; *total = the sum.
__device__ __forceinline__ int block_excl_scan(int v, Scratch& sc, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int incl = warp_incl_scan(v);
    if (lane == 31) sc.scan[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < kWarps ? sc.scan[lane] : 0;
        const int wi = warp_incl_scan(w);
        if (lane < kWarps) sc.scan[lane] = wi - w;
        if (lane == kWarps - 1) sc.total = wi;
    }
    __syncthreads();
    const int r = sc.scan[warp] + incl - v;
    *total = sc.total;
    __syncthreads();
    return r;
}

// Radix select over the keys held by the block: thread t holds keys
// key_at(0 .. n_t-1) (n_t <= KMAX when UNROLL: key_at reads a register
// array).  Finds T, the `want`-th largest key (1 <= want <= count), and
// `ties`, how many keys equal to T are among the `want` largest.  Key 0
// never occurs.
template <int KMAX, bool UNROLL, class KeyAt>
__device__ void radix_threshold(int n_t, KeyAt key_at, int want, Scratch& sc, uint32_t* T_out,
                                int* ties_out) {
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
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) {
        sc.red_min[warp] = kmin;
        sc.red_max[warp] = kmax;
    }
    __syncthreads();
    kmin = lane < kWarps ? sc.red_min[lane] : 0xffffffffu;
    kmax = lane < kWarps ? sc.red_max[lane] : 0u;
    __syncthreads();  // red_min/red_max are rewritten by the next call
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    uint32_t prefix = kmin;
    int remaining = want;
    if (kmin != kmax) {
        int hb = 31 - __clz(kmin ^ kmax);
        uint32_t mask = hb == 31 ? 0u : ~((2u << hb) - 1u);
        prefix = kmin & mask;
        int buf = 0;
        sc.hist[0][tid] = 0;  // kThreads == 256 bins
        __syncthreads();
        while (true) {
            const int shift = max(hb - 7, 0);
            const uint32_t dmask = (1u << (hb - shift + 1)) - 1u;
            int* hist = sc.hist[buf];
            sc.hist[buf ^ 1][tid] = 0;  // the next pass's histogram
            // keys crowd into few bins (a narrow bulk plus outliers that set
            // the range), so lanes with the same bin add once, together
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
            if (shift == 0) break;
            hb = shift - 1;
            buf ^= 1;
            // sc.digit/sc.above are rewritten only after the next pass's
            // atomics barrier, which every thread reaches after reading them
        }
        __syncthreads();
    }
    *T_out = prefix;
    *ties_out = remaining;
}

// Write, in index order, every key > T and the first `ties` keys == T.
// Thread t's keys are consecutive in index order and precede thread t+1's.
template <int KMAX, bool UNROLL, class KeyAt, class PageAt>
__device__ void write_selected(int n_t, KeyAt key_at, PageAt page_at, uint32_t T, int ties,
                               Scratch& sc, int32_t* out) {
    int ngt = 0, neq = 0;
    if (UNROLL) {
#pragma unroll
        for (int k = 0; k < KMAX; ++k)
            if (k < n_t) {
                ngt += key_at(k) > T;
                neq += key_at(k) == T;
            }
    } else {
        for (int k = 0; k < n_t; ++k) {
            const uint32_t v = key_at(k);
            ngt += v > T;
            neq += v == T;
        }
    }
    int total;
    const int excl = block_excl_scan((ngt << 16) | neq, sc, &total);
    int gt_before = excl >> 16, eq_before = excl & 0xffff;
    auto emit = [&](int k) {
        const uint32_t v = key_at(k);
        if (v > T) {
            out[gt_before + min(eq_before, ties)] = page_at(k);
            ++gt_before;
        } else if (v == T) {
            if (eq_before < ties) out[gt_before + eq_before] = page_at(k);
            ++eq_before;
        }
    };
    if (UNROLL) {
#pragma unroll
        for (int k = 0; k < KMAX; ++k)
            if (k < n_t) emit(k);
    } else {
        for (int k = 0; k < n_t; ++k) emit(k);
    }
}

__global__ void __launch_bounds__(kThreads) select_kernel(SelectParams p) {
    __shared__ Scratch sc;
    extern __shared__ uint32_t surv_smem[];  // survivors: keys, then pages
    uint32_t* surv_key = surv_smem;
    int32_t* surv_page = reinterpret_cast<int32_t*>(surv_smem + kSurvivorCap);

    grid_dep_wait();  // the scores come from the preceding kernel
    grid_dep_launch();

    const int u = blockIdx.x;
    const int b = u / p.hkv;
    const int tid = threadIdx.x;
    const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
    const PageRanges r = page_ranges(L, p.prefix, p.window);
    const int ncand = r.ws - r.np;
    const int nsel = min(p.budget, ncand);
    int32_t* out = p.selected + (long long)u * p.budget;

    if (nsel >= ncand) {  // every candidate is kept (also covers ncand == 0)
        for (int i = tid; i < p.budget; i += kThreads) out[i] = i < ncand ? r.np + i : -1;
        return;
    }
    for (int i = nsel + tid; i < p.budget; i += kThreads) out[i] = -1;
    if (nsel <= 0) return;

    const float* s = p.scores + (long long)u * p.max_pages + r.np;
    auto cand_key = [&](int c) { return order_key(__ldg(s + c)); };
    const int ntiles = (ncand + kTile - 1) / kTile;
    const int t0 = tid * kTilesPerThread;  // this thread's first tile
    const int nt_own = max(0, min(kTilesPerThread, ntiles - t0));

    // 1. tile maxima
    uint32_t tk[kTilesPerThread];
    if (p.tile_max) {
        const float4* tm =
            reinterpret_cast<const float4*>(p.tile_max + (long long)u * p.tile_stride);
        const float4 a = t0 < ntiles ? __ldg(tm + t0 / 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 c =
            t0 + 4 < ntiles ? __ldg(tm + t0 / 4 + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float v[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
        for (int k = 0; k < kTilesPerThread; ++k) tk[k] = k < nt_own ? order_key(v[k]) : 0u;
    } else {
#pragma unroll
        for (int k = 0; k < kTilesPerThread; ++k) tk[k] = 0u;
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
            for (int kk = 0; kk < kTilesPerThread; ++kk)
                if (kk == k) tk[kk] = m;
        }
    }

    // 2. tau: the nsel-th largest tile maximum (0 keeps every page)
    uint32_t tau = 0u;
    if (ntiles >= nsel) {
        int dummy;
        radix_threshold<kTilesPerThread, true>(nt_own, [&](int k) { return tk[k]; }, nsel, sc,
                                               &tau, &dummy);
    }

    // 3. survivors: pages >= tau.  The live tiles (maximum >= tau) are first
    // listed in index order, then dealt one per thread per round, so each
    // thread reads one tile's 16 scores in one round trip.
    __shared__ int live_tile[kThreads * kTilesPerThread];
    int nlive_own = 0;
#pragma unroll
    for (int k = 0; k < kTilesPerThread; ++k) nlive_own += k < nt_own && tk[k] >= tau;
    int nlive;
    int lpos = block_excl_scan(nlive_own, sc, &nlive);
#pragma unroll
    for (int k = 0; k < kTilesPerThread; ++k)
        if (k < nt_own && tk[k] >= tau) live_tile[lpos++] = t0 + k;
    __syncthreads();
    int nsurv = 0;
    bool overflow = false;
    for (int r0 = 0; r0 < nlive; r0 += kThreads) {  // uniform trip count
        const int li = r0 + tid;
        uint32_t v[kTile];
        int cnt = 0, c0 = 0;
        if (li < nlive) {
            c0 = live_tile[li] * kTile;
#pragma unroll
            for (int i = 0; i < kTile; ++i) v[i] = c0 + i < ncand ? cand_key(c0 + i) : 0u;
#pragma unroll
            for (int i = 0; i < kTile; ++i) cnt += v[i] >= tau && v[i] != 0u;
        }
        int total;
        int pos = nsurv + block_excl_scan(cnt, sc, &total);
        if (nsurv + total > kSurvivorCap) overflow = true;
        if (!overflow && li < nlive) {
#pragma unroll
            for (int i = 0; i < kTile; ++i) {
                if (v[i] >= tau && v[i] != 0u) {
                    surv_key[pos] = v[i];
                    surv_page[pos] = r.np + c0 + i;
                    ++pos;
                }
            }
        }
        nsurv += total;
    }

    if (!overflow) {
        __syncthreads();
        // 4. exact selection among the survivors (consecutive per thread)
        const int per = (nsurv + kThreads - 1) / kThreads;
        const int base = tid * per;
        const int n_t = max(0, min(per, nsurv - base));
        auto key_at = [&](int k) { return surv_key[base + k]; };
        uint32_t T;
        int ties;
        radix_threshold<0, false>(n_t, key_at, nsel, sc, &T, &ties);
        write_selected<0, false>(n_t, key_at, [&](int k) { return surv_page[base + k]; }, T, ties,
                                 sc, out);
    } else {
        // heavy ties: stream over every candidate, thread t owning a
        // contiguous range, re-reading scores for each pass
        const int per = (ncand + kThreads - 1) / kThreads;
        const int base = tid * per;
        const int n_t = max(0, min(per, ncand - base));
        auto key_at = [&](int k) { return cand_key(base + k); };
        uint32_t T;
        int ties;
        radix_threshold<0, false>(n_t, key_at, nsel, sc, &T, &ties);
        write_selected<0, false>(n_t, key_at, [&](int k) { return r.np + base + k; }, T, ties,
                                 sc, out);
    }
}

constexpr int kSurvivorSmem = kSurvivorCap * 2 * (int)sizeof(uint32_t);

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
    if (p.batch * p.hkv == 0) return cudaSuccess;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(
            select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSurvivorSmem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    return launch_pdl(select_kernel, dim3(p.batch * p.hkv), dim3(kThreads), kSurvivorSmem, stream,
                      p);
}

}  // namespace slc
