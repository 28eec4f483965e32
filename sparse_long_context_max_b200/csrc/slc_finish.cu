// The finishing half of the sparse decode step, one thread-block cluster per
// (sequence, kv head) unit:
//
//   1. the fixed-budget selection ("Accelerating Long-Context Decoding in
//      Large-Scale Hybrid LLMs Without Retraining", abstract: a fixed budget
//      of the most relevant tokens): the min(budget, #candidates) candidate
//      pages with the highest score, equal scores going to the lower page,
//      written in ascending page order;
//   2. attention over the selected pages;
//   3. the log-sum-exp merge of those partials with the streaming kernel's
//      prefix/window partials (slc_stream.cu) into the fp32 output.
//
// Selection across the cluster.  The unit's candidate scores are cut into C
// contiguous slices, one per CTA, held in shared memory as order-preserving
// uint32 keys.  An exact MSB-first radix select finds T, the budget-th
// largest key, and how many keys equal to T to keep (the lowest-indexed
// ones): every CTA histograms the current 8-bit digit of its own keys, and
// after a cluster barrier every CTA reads all C histograms through
// distributed shared memory and every warp derives the same digit (reads
// spread over the SMs; remote atomics into one CTA serialise).  Digits start
// at the highest bit where the unit's smallest and largest keys differ, and
// the search stops as soon as the chosen bin holds exactly the keys still
// wanted.  One cluster barrier and one CTA barrier per digit.  The CTAs then
// exchange their counts of keys above / equal to T, and each writes its
// selected pages at their global ascending positions (warp ballots keep
// index order), with their physical page ids (looked up while the
// selection ran), and requests their K and V into L2.
//
// Attention.  The selected list is spread over all warps of the cluster;
// each warp streams its pages through its own bulk-copy ring (slc_attend_
// impl.cuh).  The CTA combines its warps in shared memory; after a cluster
// barrier each CTA merges a share of the (head, dims) items over the C CTA
// partials (distributed shared memory) and the unit's streaming partials.
//
// Every CTA of a cluster takes the same path through the cluster barriers:
// all branch conditions around them depend on the unit only.  A cluster
// takes units c, c + clusters, ...; no CTA waits for another cluster.
#include <cooperative_groups.h>

#include "slc_attend_impl.cuh"

namespace slc {

namespace {

namespace cg = cooperative_groups;
using namespace attn;

// Eight warps, all attending, one CTA per SM: a unit's clusters take at
// most one CTA per SM anyway at the usual unit counts, and with two warps
// per scheduler the latency-bound per-page work of the attention and the
// selection's steps overlap (four warps per CTA, two CTAs per SM, left one
// warp per scheduler busy and measured slower).
template <int D>
struct FinishCfg {
    static constexpr int NT = 256;                     // threads per CTA
    static constexpr int NW = NT / 32;                 // warps per CTA
    static constexpr int NW_ATT = NW;                  // warps that attend
    static constexpr int STAGES = D == 128 ? 2 : 1;    // ring stages per attending warp
    static constexpr int RING = STAGES * 2 * kPage * D * 2;
    static constexpr int MIN_BLOCKS = 1;
};

constexpr int kBins = 256;       // 8-bit digits
constexpr int kMaxCluster = 16;  // the largest cluster size launched

// Shared memory: rings | bars | nvalid | keys[cap] | phys[cap] | FinishShared
// | this CTA's partial ([G][D] floats, then [G] (max, sum) pairs).
struct alignas(16) FinishShared {
    int hist[2][kBins];  // this CTA's digit histogram (read remotely), double-buffered
    int whist[8][kBins]; // per-warp histograms of the current digit
    int ghist[kBins];    // the cluster's histogram (local copy)
    uint32_t red_min[32], red_max[32];
    int2 wcnt[32];       // per warp: (keys > T, keys == T)
    uint2 minmax;        // this CTA's key range (read remotely)
    int2 counts;         // this CTA's (keys > T, keys == T) (read remotely)
    int scount;          // this CTA's survivors (read remotely)
    int soff[kMaxCluster + 1];  // survivors of the ranks before each rank
    int dcount;          // this CTA's keys within delta of the best (read remotely)
    long long k0, k1;    // the unit's streaming-partial chunks
    uint64_t bar;        // the score copy
};

// The survivor path's use of the shared memory (see finish_kernel): during
// the selection the ring area holds the unit's tile maxima, then this CTA's
// survivors (read remotely) and the cluster's survivors; the keys + phys
// area then holds the selected list.
constexpr int kOwnSurvivorsBytes = 24 << 10;
constexpr int kOwnSurvivorCap = kOwnSurvivorsBytes / 16;
struct Survivor {  // 16 bytes: the order key, the candidate index, the physical page
    uint32_t key;
    int32_t cand;
    int32_t phys;
    int32_t pad;
};

// Byte offsets of the shared-memory carve-up at cluster size `cluster`.
template <int D>
struct FinishLayout {
    using C = FinishCfg<D>;
    static constexpr size_t bars = (size_t)C::NW_ATT * C::RING;
    static constexpr size_t nvalid = bars + C::NW_ATT * C::STAGES * 8;
    static constexpr size_t keys = (nvalid + C::NW_ATT * C::STAGES * 4 + 127) / 128 * 128;
    // a CTA's slice of the candidates, at most (rounded up to 4 keys, as
    // the kernel rounds its slices)
    static constexpr size_t slice(int cluster) {
        return (size_t)(((kMaxCandidates + cluster - 1) / cluster + 3) / 4 * 4);
    }
    static constexpr size_t phys(int cluster) { return keys + slice(cluster) * 4; }
    static constexpr size_t shared(int cluster) { return phys(cluster) + slice(cluster) * 4; }
    static constexpr size_t part(int cluster) { return shared(cluster) + sizeof(FinishShared); }
    static constexpr size_t total(int cluster) {
        return part(cluster) + (kMaxGroup * D + 2 * kMaxGroup) * 4;
    }
};

template <int D>
constexpr size_t finish_smem(int cluster) {
    return FinishLayout<D>::total(cluster);
}


// Rank r's copy of the shared variable *p, for r < kMaxCluster; ranks past
// the cluster read the last rank's copy, so that an unrolled loop over r
// issues its remote loads without branches (callers discard those values).
template <class T>
__device__ __forceinline__ T remote(cg::cluster_group& cl, T* p, int r, int C) {
    return *cl.map_shared_rank(p, r < C ? r : C - 1);
}

// Every warp finds, from the histogram in sh.ghist, the digit holding the
// remaining-th largest key: its bin, the keys in higher bins, and its count.
__device__ __forceinline__ void scan_digit(const FinishShared& sh, int remaining, int* digit,
                                           int* above, int* count) {
    const int lane = threadIdx.x & 31;
    int c[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        c[i] = sh.ghist[lane * 8 + i];
        local += c[i];
    }
    int suf = local;  // keys in bins >= 8*lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += t;
    }
    const int above_lane = suf - local;
    const bool mine = above_lane < remaining && suf >= remaining;
    int d = 0, ab = 0, ct = 0;
    if (mine) {
        int cum = above_lane;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
            if (cum + c[i] >= remaining) {
                d = lane * 8 + i;
                ab = cum;
                ct = c[i];
                break;
            }
            cum += c[i];
        }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    *digit = __shfl_sync(0xffffffffu, d, src);
    *above = __shfl_sync(0xffffffffu, ab, src);
    *count = __shfl_sync(0xffffffffu, ct, src);
}

// The k-th largest of the keys one warp holds in registers (NK per lane,
// only the first nk used; key 0: none), 1 <= k <= their count, by
// bit-by-bit bisection from the highest bit where the warp's smallest and
// largest keys differ: each bit, every lane counts its keys >= T | bit and
// one warp reduction sums the counts (no barrier).  With max_bits below the
// bits left the result is a lower bound (at least k keys are >= it).
template <int NK>
__device__ __forceinline__ uint32_t warp_kth(const uint32_t (&v)[NK], int nk, int k,
                                             int max_bits) {
    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int c = 0; c < NK; ++c)
        if (c < nk && v[c]) {
            kmin = min(kmin, v[c]);
            kmax = max(kmax, v[c]);
        }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (kmin >= kmax) return kmin;
    const int hb = 31 - __clz(kmin ^ kmax);
    uint32_t T = hb == 31 ? 0u : kmin & ~((2u << hb) - 1u);
    const int lo = max(0, hb + 1 - max_bits);
    for (int bit = hb; bit >= lo; --bit) {
        const uint32_t tr = T | (1u << bit);
        int part[4] = {0, 0, 0, 0};  // four partial sums: a shorter add chain
#pragma unroll
        for (int c = 0; c < NK; ++c)
            if (c < nk) part[c & 3] += v[c] >= tr ? 1 : 0;
        const int cnt = __reduce_add_sync(0xffffffffu, (part[0] + part[1]) + (part[2] + part[3]));
        if (cnt >= k) T = tr;
    }
    return T;
}

// The cluster-wide k-th largest key: the k largest keys of the unit are the
// keys > T plus the first `ties` keys == T in index order.  keys[0..cnt) are
// this CTA's; 1 <= k < the unit's key count.
template <int NT>
__device__ void cluster_kth(cg::cluster_group& cl, const uint32_t* keys, int cnt, int k,
                            FinishShared& sh, uint32_t* T_out, int* ties_out) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = (int)cl.num_blocks();
    // range of the unit's keys
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int i = tid; i < cnt; i += NT) {
        kmin = min(kmin, keys[i]);
        kmax = max(kmax, keys[i]);
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
        sh.red_min[warp] = kmin;
        sh.red_max[warp] = kmax;
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t a = 0xffffffffu, b = 0u;
        for (int w = 0; w < NT / 32; ++w) {
            a = min(a, sh.red_min[w]);
            b = max(b, sh.red_max[w]);
        }
        sh.minmax = make_uint2(a, b);
    }
    cl.sync();
    // lane r reads rank r's range (one remote request per lane; lanes past
    // the cluster repeat the last rank, which changes nothing)
    {
        const uint2 m = remote(cl, &sh.minmax, lane & (kMaxCluster - 1), C);
        kmin = __reduce_min_sync(0xffffffffu, m.x);
        kmax = __reduce_max_sync(0xffffffffu, m.y);
    }
    if (kmin == kmax) {  // every key equal: the first k of them
        *T_out = kmin;
        *ties_out = k;
        return;
    }
    int hb = 31 - __clz(kmin ^ kmax);
    uint32_t mask = hb == 31 ? 0u : ~((2u << hb) - 1u);
    uint32_t prefix = kmin & mask;
    int remaining = k;
    for (int pass = 0;; ++pass) {
        const int buf = pass & 1;
        const int shift = max(hb - 7, 0);
        const uint32_t dmask = (1u << (hb - shift + 1)) - 1u;
        // this CTA's histogram of the digit: each warp counts into its own
        // histogram (zeroed), then the CTA sums them into hist[buf]
        int* wh = sh.whist[warp];
        for (int base = 0; base < cnt; base += NT) {
            const int i = base + tid;
            const uint32_t v = i < cnt ? keys[i] : 0u;
            if (i < cnt && (v & mask) == prefix) atomicAdd(&wh[(v >> shift) & dmask], 1);
        }
        __syncthreads();
        for (int bin = tid; bin < kBins; bin += NT) {
            int c = 0;
#pragma unroll
            for (int w = 0; w < NT / 32; ++w) {
                c += sh.whist[w][bin];
                sh.whist[w][bin] = 0;  // ready for the next digit
            }
            sh.hist[buf][bin] = c;
        }
        cl.sync();  // every CTA's histogram is complete
        // (hist[buf ^ 1], rewritten whole by the next digit, was last read
        // remotely for the previous digit, before every CTA reached this
        // barrier)
        // the cluster's histogram, four bins per 16-byte remote request
        static_assert(kBins / 4 <= NT, "one thread per four bins");
        if (tid < kBins / 4) {
            int4 s = make_int4(0, 0, 0, 0);
#pragma unroll
            for (int r = 0; r < kMaxCluster; ++r) {
                const int4 v = remote(cl, reinterpret_cast<int4*>(&sh.hist[buf][0]) + tid, r, C);
                if (r < C) {
                    s.x += v.x;
                    s.y += v.y;
                    s.z += v.z;
                    s.w += v.w;
                }
            }
            reinterpret_cast<int4*>(sh.ghist)[tid] = s;
        }
        __syncthreads();
        int digit, above, count;
        scan_digit(sh, remaining, &digit, &above, &count);
        remaining -= above;
        prefix |= (uint32_t)digit << shift;
        mask |= dmask << shift;
        if (count == remaining && prefix != 0u) {
            // every key of the bin is wanted: exactly the keys >= prefix
            *T_out = prefix - 1u;
            *ties_out = 0;
            return;
        }
        if (shift == 0) {
            *T_out = prefix;
            *ties_out = remaining;
            return;
        }
        hb = shift - 1;
    }
}

// The k-th largest of n keys held by this CTA (keys[i * stride], i < n), by the
// same MSB-first radix search as cluster_kth but with CTA barriers only:
// the k largest keys are the keys > T plus the first `ties` keys == T in
// index order.  1 <= k <= n.  sh.whist must be zero (it is left zero).
template <int NT>
__device__ __noinline__ void cta_kth(const uint32_t* keys, int stride, int n, int k,
                                     FinishShared& sh, uint32_t* T_out,
                        int* ties_out) {
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int i = tid; i < n; i += NT) {
        const uint32_t v = keys[i * stride];
        kmin = min(kmin, v);
        kmax = max(kmax, v);
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
        sh.red_min[warp] = kmin;
        sh.red_max[warp] = kmax;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        kmin = min(kmin, sh.red_min[w]);
        kmax = max(kmax, sh.red_max[w]);
    }
    if (kmin == kmax) {  // every key equal: the first k of them
        *T_out = kmin;
        *ties_out = k;
        return;
    }
    int hb = 31 - __clz(kmin ^ kmax);
    uint32_t mask = hb == 31 ? 0u : ~((2u << hb) - 1u);
    uint32_t prefix = kmin & mask;
    int remaining = k;
    int* wh = sh.whist[warp];
    while (true) {
        const int shift = max(hb - 7, 0);
        const uint32_t dmask = (1u << (hb - shift + 1)) - 1u;
        for (int i = tid; i < n; i += NT) {
            const uint32_t v = keys[i * stride];
            if ((v & mask) == prefix) atomicAdd(&wh[(v >> shift) & dmask], 1);
        }
        __syncthreads();
        for (int bin = tid; bin < kBins; bin += NT) {
            int c = 0;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                c += sh.whist[w][bin];
                sh.whist[w][bin] = 0;
            }
            sh.ghist[bin] = c;
        }
        __syncthreads();
        int digit, above, count;
        scan_digit(sh, remaining, &digit, &above, &count);
        remaining -= above;
        prefix |= (uint32_t)digit << shift;
        mask |= dmask << shift;
        if (count == remaining && prefix != 0u) {
            *T_out = prefix - 1u;
            *ties_out = 0;
            return;
        }
        if (shift == 0) {
            *T_out = prefix;
            *ties_out = remaining;
            return;
        }
        hb = shift - 1;
    }
}

template <int D>
__global__ void __launch_bounds__(FinishCfg<D>::NT, FinishCfg<D>::MIN_BLOCKS)
    finish_kernel(FinishParams p) {
    using C_ = FinishCfg<D>;
    constexpr int NT = C_::NT, NW = C_::NW, NW_ATT = C_::NW_ATT, STAGES = C_::STAGES;
    constexpr int RING = C_::RING;
    extern __shared__ __align__(128) uint8_t smem[];
    cg::cluster_group cl = cg::this_cluster();
    const int C = (int)cl.num_blocks();
    const int rank = (int)cl.block_rank();
    const int cid = blockIdx.x / C, ncl = gridDim.x / C;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const AttendParams& a = p.at;

    using Lay = FinishLayout<D>;
    Ring ring;  // attending warps only
    ring.tiles = smem + (warp < NW_ATT ? warp : 0) * RING;
    ring.bars = reinterpret_cast<uint64_t*>(smem + Lay::bars) + (warp < NW_ATT ? warp : 0) * STAGES;
    ring.nvalid = reinterpret_cast<int*>(smem + Lay::nvalid) + (warp < NW_ATT ? warp : 0) * STAGES;
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem + Lay::keys);
    int32_t* phys = reinterpret_cast<int32_t*>(smem + Lay::phys(C));
    FinishShared& sh = *reinterpret_cast<FinishShared*>(smem + Lay::shared(C));
    float* cacc = reinterpret_cast<float*>(smem + Lay::part(C));     // this CTA's partial [G][D]
    float2* cml = reinterpret_cast<float2*>(cacc + kMaxGroup * D);  // [G]
    if (lane == 0 && warp < NW_ATT) {
        for (int s = 0; s < STAGES; ++s) mbar_init(ring.bars + s, 1);
        if (tid == 0) mbar_init(&sh.bar, 1);
        fence_mbar_init();
    }
    // the per-warp histograms start at zero; every search leaves them zero
    for (int i = tid; i < NW * kBins; i += NT) (&sh.whist[0][0])[i] = 0;
    __syncthreads();

    const int units = a.batch * a.hkv;
    const int G = a.group;
    uint32_t it = 0, score_phase = 0;
    bool ok = true, waited = false;
    for (int u = cid; u < units; u += ncl) {
        const int b = u / a.hkv, h = u % a.hkv;
        const int L = checked_len(a.seq_lens, b, a.max_pages, a.status);
        const PageRanges r = page_ranges(L, a.prefix, a.window);
        const int ncand = r.ws - r.np;
        int nsel = min(p.budget, ncand);
        int32_t* sel_row = p.selected ? p.selected + (long long)u * p.budget : nullptr;
        int32_t* phys_row = p.sel_phys + (long long)u * p.budget;
        // top-delta: the unit's selection size comes from its scores, unless
        // topd alone settles it (topd >= ncand, or budget <= topd: the top
        // min(budget, ncand)); the tile maxima always come with the scores
        const bool by_delta = p.scores != nullptr && p.topd >= 0 && p.topd < ncand &&
                              p.topd < p.budget;
        bool selecting = p.scores != nullptr && nsel > 0 && (by_delta || nsel < ncand);
        // this CTA's slice of the candidates
        const int pc = ((ncand + C - 1) / C + 3) / 4 * 4;
        const int c0 = min(rank * pc, ncand);
        const int cnt = selecting ? min(ncand, c0 + pc) - c0 : 0;

        // what needs only the inputs, before waiting for the streaming kernel:
        // the physical pages of the slice (in flight while the selection
        // runs) and which of the streaming partials belong to this unit
        if (cnt > 0) {
            const int32_t* bt = a.block_table + (long long)b * a.max_pages + r.np + c0;
            for (int i = tid; i < cnt; i += NT) cp_async4(phys + i, bt + i);
            cp_async_commit();
        }
        long long k0 = 0, k1 = -1;
        if (warp == NW - 1) {  // the unit's streaming partials: chunks k0..k1
            auto len_of = [&](int bb) { return list_len(a, bb); };
            const long long total = total_units(a.batch, a.hkv, len_of);
            const long long start = unit_list_start(a, u);
            const int len = list_len(a, b);
            const int nf = forced_ctas(a, p.stream_scored != 0, a.num_chunks);
            if (len > 0) {
                const long long cpp = (total + nf - 1) / nf;
                k0 = start / cpp;
                k1 = (start + len - 1) / cpp;
            }
            if (lane == 0) {
                sh.k0 = k0;
                sh.k1 = k1;
            }
        }
        if (!waited) {
            // the scores and the prefix/window partials come from the
            // streaming kernel
            grid_dep_wait();
            grid_dep_launch();
            waited = true;
        }
        if (warp == NW - 1) {
            // the unit's prefix/window partials start their way into L2
            for (long long k = k0 + lane; k <= k1; k += 32) {
                const long long slot = u + k;
                prefetch_l2(a.part_acc + slot * G * D, (uint32_t)(G * D * 4));
                // the (max, sum) pairs: 8*G bytes, widened to 16-byte bounds (the
                // workspace region is padded to 256 bytes)
                const uintptr_t lo =
                    reinterpret_cast<uintptr_t>(a.part_ml + slot * G) & ~uintptr_t(15);
                const uintptr_t hi =
                    (reinterpret_cast<uintptr_t>(a.part_ml + (slot + 1) * G) + 15) &
                    ~uintptr_t(15);
                prefetch_l2(reinterpret_cast<const void*>(lo), (uint32_t)(hi - lo));
            }
        }

        // ---- 1. selection
        // Survivor path (when the unit has at least nsel tiles): tau, the
        // nsel-th largest tile maximum, is <= T (the nsel tiles with the
        // largest maxima hold nsel distinct keys >= tau), so every selected
        // key is >= tau.  Each CTA finds tau from all the unit's tile maxima,
        // publishes its keys >= tau (few: about nsel in all), gathers every
        // CTA's, and finds T and the selected list itself: two cluster
        // barriers.  Otherwise (or if the survivors overflow their space) the
        // cluster-wide radix search over all keys.
        bool local_list = false;  // the selected list is in this CTA's shared memory
        int2* list = reinterpret_cast<int2*>(keys);  // (page, physical page)
        const int ntiles = (ncand + kSelTile - 1) / kSelTile;
        uint32_t* tkeys = reinterpret_cast<uint32_t*>(smem);  // the ring area
        if (selecting) {
            // the tile maxima serve the survivor path's bound and top-delta's s_max
            const bool tiles_in = p.tile_max != nullptr &&
                                  (by_delta || (ntiles >= nsel && nsel <= kMaxCandidates / C));
            if (cnt > 0 || tiles_in) {
                if (tid == 0) {
                    const uint32_t kb = cnt > 0 ? (uint32_t)((cnt + 3) / 4 * 4) * 4 : 0u;
                    const uint32_t tb = tiles_in ? (uint32_t)((ntiles + 3) / 4 * 4) * 4 : 0u;
                    fence_proxy_async_smem();  // earlier generic accesses of keys[] first
                    mbar_arrive_expect_tx(&sh.bar, kb + tb);
                    if (kb)
                        bulk_g2s(keys, p.scores + (long long)u * p.cand_stride + c0, kb,
                                 &sh.bar);
                    if (tb)
                        bulk_g2s(tkeys, p.tile_max + (long long)u * (p.cand_stride / kSelTile),
                                 tb, &sh.bar);
                }
                if (!mbar_wait_bounded(&sh.bar, score_phase & 1u, kWaitLimit)) {
                    if (tid == 0) atomicOr(a.status, SLC_STATUS_WAIT_TIMEOUT);
                    mbar_wait_bounded(&sh.bar, score_phase & 1u, kWaitLimit);
                }
                ++score_phase;
                __syncthreads();  // every thread's wait is done before keys are rewritten
                for (int i = tid; i < cnt; i += NT)
                    keys[i] = order_key(__uint_as_float(keys[i]));
            }
            __syncthreads();
            if (by_delta) {
                // top-delta ("Faster Than Flash: Fudan FFD Hits 11.6x Kernel
                // Speedup, Pushes Long-Context Decoding to 256K", section
                // "top-delta: Tearing Down "Global Synchronization" Too"): the
                // top topd and the candidates within delta of the best are both
                // prefixes of the (score desc, page asc) order, so their union
                // is the top max(topd, m), m = #{s >= s_max - delta}.  s_max is
                // the largest tile maximum (every CTA holds them all); m sums
                // the CTAs' counts
                uint32_t km = 0u;
                for (int t = tid; t < ntiles; t += NT) km = max(km, tkeys[t]);
                km = __reduce_max_sync(0xffffffffu, km);
                if (lane == 0) sh.red_max[warp] = km;
                __syncthreads();
#pragma unroll
                for (int w2 = 0; w2 < NW; ++w2) km = max(km, sh.red_max[w2]);
                const uint32_t tk = delta_threshold_key(km, p.delta);
                int c = 0;
                for (int i = tid; i < cnt; i += NT) c += keys[i] >= tk ? 1 : 0;
                c = __reduce_add_sync(0xffffffffu, c);
                if (lane == 0) sh.wcnt[warp] = make_int2(c, 0);
                __syncthreads();
                if (tid == 0) {
                    int s2 = 0;
#pragma unroll
                    for (int w2 = 0; w2 < NW; ++w2) s2 += sh.wcnt[w2].x;
                    sh.dcount = s2;
                }
                cl.sync();  // every CTA's count is published
                const int rr = lane & (kMaxCluster - 1);
                const int cr = remote(cl, &sh.dcount, rr, C);
                const int m =
                    __reduce_add_sync(0xffffffffu, lane < kMaxCluster && rr < C ? cr : 0);
                nsel = min(min(max(p.topd, m), p.budget), ncand);
                if (nsel == 0 || nsel >= ncand) {  // none, or every candidate: no search
                    selecting = false;
                    cp_async_wait<0>();  // this thread's phys[] copies, unused now
                }
            }
        }
        if (selecting) {
            const bool bound = p.tile_max != nullptr && ntiles >= nsel &&
                               nsel <= kMaxCandidates / C;  // the list fits keys + phys
            bool fast = false;
            if (bound) {
                // tau: each warp's ceil(nsel / NW)-th largest tile maximum
                // among its share of the tiles (ballot-free bisection, ten
                // bits: a lower bound), the smallest over the warps; at least
                // nsel tile maxima (distinct keys) are >= it whenever every
                // warp holds that many, else tau = 0 (every key survives)
                uint32_t tau;
                {
                    constexpr int TC = kMaxCandidates / kSelTile / NT;  // tile keys per lane
                    const int kw = (nsel + NW - 1) / NW;
                    const int tspan = (ntiles + NW - 1) / NW;
                    const int t0 = warp * tspan, t1 = min(ntiles, t0 + tspan);
                    uint32_t v[TC];
#pragma unroll
                    for (int c = 0; c < TC; ++c) {
                        const int t = t0 + 32 * c + lane;
                        v[c] = t < t1 ? tkeys[t] : 0u;
                    }
                    const bool enough = t1 - t0 >= kw;
                    const uint32_t vw = enough ? warp_kth<TC>(v, (tspan + 31) / 32, kw, 10) : 0u;
                    if (lane == 0) sh.red_min[warp] = vw;
                    __syncthreads();
                    tau = 0xffffffffu;
#pragma unroll
                    for (int w2 = 0; w2 < NW; ++w2) tau = min(tau, sh.red_min[w2]);
                }
                cp_async_wait<0>();  // this thread's phys[] copies
                __syncthreads();     // every phys[] copy landed; tkeys is no longer read
                // this CTA's survivors, in index order, over the tile maxima
                Survivor* own = reinterpret_cast<Survivor*>(smem);
                const int span = ((cnt + NW - 1) / NW + 31) / 32 * 32;
                const int w0 = min(warp * span, cnt), w1 = min(w0 + span, cnt);
                int nk = 0;
                for (int i = w0 + lane; i - lane < w1; i += 32)
                    nk += __popc(__ballot_sync(0xffffffffu, i < w1 && keys[i] >= tau));
                if (lane == 0) sh.wcnt[warp] = make_int2(nk, 0);
                __syncthreads();
                int before = 0, nown = 0;
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    before += w < warp ? sh.wcnt[w].x : 0;
                    nown += sh.wcnt[w].x;
                }
                const unsigned below = (1u << lane) - 1u;
                for (int i = w0 + lane; i - lane < w1; i += 32) {
                    const bool keep = i < w1 && keys[i] >= tau;
                    const unsigned bk = __ballot_sync(0xffffffffu, keep);
                    const int pos = before + __popc(bk & below);
                    if (keep && pos < kOwnSurvivorCap) own[pos] = Survivor{keys[i], c0 + i, phys[i], 0};
                    before += __popc(bk);
                }
                if (tid == 0) sh.scount = nown;
                cl.sync();  // every CTA's survivors are published
                {   // every warp: the ranks' counts (lane r reads rank r's)
                    const int rr = lane & (kMaxCluster - 1);
                    const int cr = remote(cl, &sh.scount, rr, C);
                    const int cv = lane < kMaxCluster && rr < C ? cr : 0;
                    const int incl = warp_incl_scan(cv);
                    if (warp == 0 && lane <= kMaxCluster) sh.soff[lane] = incl - cv;
                    const int total = __shfl_sync(0xffffffffu, incl, 31);
                    const int biggest = __reduce_max_sync(0xffffffffu, cv);
                    fast = biggest <= kOwnSurvivorCap && total >= nsel &&
                           total <= (NW_ATT * RING - kOwnSurvivorsBytes) / 16;
                    if (fast) {
                        __syncthreads();  // sh.soff is written
                        Survivor* merged = reinterpret_cast<Survivor*>(smem + kOwnSurvivorsBytes);
                        // the cluster's survivors in index order: rank r's run follows
                        // the runs of the ranks before it
                        for (int e = tid; e < total; e += NT) {
                            int r0 = 0;
#pragma unroll
                            for (int q = 1; q < kMaxCluster; ++q)
                                if (q < C && sh.soff[q] <= e) r0 = q;
                            const int4 v = *cl.map_shared_rank(
                                reinterpret_cast<int4*>(own) + (e - sh.soff[r0]), r0);
                            reinterpret_cast<int4*>(merged)[e] = v;
                        }
                        __syncthreads();
                        uint32_t T;
                        int ties;
                        cta_kth<NT>(&merged[0].key, 4, total, nsel, sh, &T, &ties);
                        // the selected list: keys > T and the first `ties` keys == T,
                        // in index order (over the keys + phys area)
                        const int mspan = ((total + NW - 1) / NW + 31) / 32 * 32;
                        const int m0 = min(warp * mspan, total), m1 = min(m0 + mspan, total);
                        int ngt = 0, neq = 0;
                        for (int i = m0 + lane; i - lane < m1; i += 32) {
                            const uint32_t v = i < m1 ? merged[i].key : 0u;
                            ngt += __popc(__ballot_sync(0xffffffffu, i < m1 && v > T));
                            neq += __popc(__ballot_sync(0xffffffffu, i < m1 && v == T));
                        }
                        if (lane == 0) sh.wcnt[warp] = make_int2(ngt, neq);
                        __syncthreads();
                        int gt_before = 0, eq_before = 0;
#pragma unroll
                        for (int w = 0; w < NW; ++w)
                            if (w < warp) {
                                gt_before += sh.wcnt[w].x;
                                eq_before += sh.wcnt[w].y;
                            }
                        for (int i = m0 + lane; i - lane < m1; i += 32) {
                            const uint32_t v = i < m1 ? merged[i].key : 0u;
                            const bool gt = i < m1 && v > T, eq = i < m1 && v == T;
                            const unsigned bgt = __ballot_sync(0xffffffffu, gt);
                            const unsigned beq = __ballot_sync(0xffffffffu, eq);
                            const int g_b = gt_before + __popc(bgt & below);
                            const int e_b = eq_before + __popc(beq & below);
                            int pos = -1;
                            if (gt) pos = g_b + min(e_b, ties);
                            else if (eq && e_b < ties) pos = g_b + e_b;
                            if (pos >= 0 && pos < nsel)
                                list[pos] = make_int2(r.np + merged[i].cand, merged[i].phys);
                            gt_before += __popc(bgt);
                            eq_before += __popc(beq);
                        }
                        __syncthreads();  // the list is complete
                        // this CTA's share of selected_out
                        for (int i = rank + C * tid; i < p.budget; i += C * NT)
                            sel_row[i] = i < nsel ? list[i].x : -1;
                        local_list = true;
                    }
                }
            }
            if (!fast) {
                uint32_t T;
                int ties;
                cluster_kth<NT>(cl, keys, cnt, nsel, sh, &T, &ties);
                // warp w owns the keys [w * span, (w + 1) * span) of the slice; its
                // lanes read them 32 at a time, and ballots keep index order
                const int span = ((cnt + NW - 1) / NW + 31) / 32 * 32;
                const int w0 = min(warp * span, cnt), w1 = min(w0 + span, cnt);
                int ngt = 0, neq = 0;
                for (int i = w0 + lane; i - lane < w1; i += 32) {
                    const uint32_t v = i < w1 ? keys[i] : 0u;
                    ngt += __popc(__ballot_sync(0xffffffffu, i < w1 && v > T));
                    neq += __popc(__ballot_sync(0xffffffffu, i < w1 && v == T));
                }
                if (lane == 0) sh.wcnt[warp] = make_int2(ngt, neq);
                cp_async_wait<0>();  // this thread's phys[] copies; the barrier publishes them
                __syncthreads();
                int gt_before = 0, eq_before = 0, tg = 0, te = 0;
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    const int2 c2 = sh.wcnt[w];
                    if (w < warp) {
                        gt_before += c2.x;
                        eq_before += c2.y;
                    }
                    tg += c2.x;
                    te += c2.y;
                }
                if (tid == 0) sh.counts = make_int2(tg, te);
                cl.sync();
                {   // the lower ranks' counts: lane rr reads rank rr's
                    const int rr = lane & (kMaxCluster - 1);
                    const int2 c2 = remote(cl, &sh.counts, rr, C);
                    const bool lower = lane < kMaxCluster && rr < rank;
                    gt_before += __reduce_add_sync(0xffffffffu, lower ? c2.x : 0);
                    eq_before += __reduce_add_sync(0xffffffffu, lower ? c2.y : 0);
                }
                const unsigned below = (1u << lane) - 1u;
                constexpr uint32_t TILE = kPage * D * 2;
                for (int i = w0 + lane; i - lane < w1; i += 32) {
                    const uint32_t v = i < w1 ? keys[i] : 0u;
                    const bool gt = i < w1 && v > T, eq = i < w1 && v == T;
                    const unsigned bgt = __ballot_sync(0xffffffffu, gt);
                    const unsigned beq = __ballot_sync(0xffffffffu, eq);
                    const int g_b = gt_before + __popc(bgt & below);
                    const int e_b = eq_before + __popc(beq & below);
                    int pos = -1;
                    if (gt) pos = g_b + min(e_b, ties);
                    else if (eq && e_b < ties) pos = g_b + e_b;
                    if (pos >= 0 && pos < nsel) {
                        const int ph = phys[i];
                        sel_row[pos] = r.np + c0 + i;
                        phys_row[pos] = ph;
                        if (ph >= 0 && ph < a.num_pages) {
                            // the page's K and V start their way into L2 now, while
                            // the cluster syncs and the warps set up
                            const long long off = ((long long)ph * a.hkv + h) * TILE;
                            prefetch_l2(static_cast<const uint8_t*>(a.k_cache) + off, TILE);
                            prefetch_l2(static_cast<const uint8_t*>(a.v_cache) + off, TILE);
                        }
                    }
                    gt_before += __popc(bgt);
                    eq_before += __popc(beq);
                }
                if (rank == 0)
                    for (int i = nsel + tid; i < p.budget; i += NT) sel_row[i] = -1;
            }
        } else if (p.scores != nullptr && rank == 0) {
            // every candidate kept (or none): no search
            for (int i = tid; i < p.budget; i += NT) sel_row[i] = i < nsel ? r.np + i : -1;
        }
        // the selection rows are written and visible in the cluster, and no CTA
        // reads another's survivors any more (the attention reuses the rings)
        cl.sync();

        // ---- 2. attention over the selected pages (attending warps)
        const int npos = p.scores != nullptr ? nsel : p.budget;
        WarpState<D> st;
        const int gw = rank * NW_ATT + warp;
        const int32_t* given_row = p.given ? p.given + (long long)u * p.budget : nullptr;
        warp_attend<D, STAGES>(a, ring, it, ok, b, h, warp < NW_ATT ? gw : npos, npos,
                               C * NW_ATT, st, [&](int i, int* ph, int* nv) {
            *ph = 0;
            *nv = 0;
            if (local_list) {
                const int2 e = list[i];
                if (e.x < r.np || e.x >= r.ws || e.y < 0 || e.y >= a.num_pages) {
                    atomicOr(a.status, e.y < 0 || e.y >= a.num_pages ? SLC_STATUS_BAD_PAGE
                                                                     : SLC_STATUS_BAD_SELECTION);
                    return;
                }
                *ph = e.y;
                *nv = min(kPage, L - e.x * kPage);
            } else if (selecting) {
                const int j = __ldcg(sel_row + i);
                const int pp = __ldcg(phys_row + i);
                if (j < r.np || j >= r.ws || pp < 0 || pp >= a.num_pages) {
                    atomicOr(a.status, pp < 0 || pp >= a.num_pages ? SLC_STATUS_BAD_PAGE
                                                                   : SLC_STATUS_BAD_SELECTION);
                    return;
                }
                *ph = pp;
                *nv = min(kPage, L - j * kPage);
            } else if (given_row == nullptr) {  // every candidate
                resolve_logical(a, b, L, r.np + i, ph, nv);
            } else {
                const int j = __ldg(given_row + i);
                const int prev = i > 0 ? __ldg(given_row + i - 1) : -1;
                if (j == -1) return;  // padding
                if (j < 0 || j >= r.n || j <= prev) {
                    atomicOr(a.status, SLC_STATUS_BAD_SELECTION);
                    return;
                }
                if (j < r.np || j >= r.ws) return;  // a prefix or window page: attended
                resolve_logical(a, b, L, j, ph, nv);
            }
        });
        cta_combine<D, NW_ATT, RING, NT>(a, smem, st, [&](int g, int d4, float4 num, float M,
                                                           float den) {
            reinterpret_cast<float4*>(cacc + g * D)[d4] = num;
            if (d4 == 0) cml[g] = make_float2(M, den);
        });
        cl.sync();  // every CTA's partial is complete

        // ---- 3. merge: this CTA's share of the (head, dims) items
        const long long sk0 = sh.k0, sk1 = sh.k1;
        for (int item = rank + C * tid; item < G * (D / 4); item += C * NT) {
            const int g = item / (D / 4), d4 = item % (D / 4);
            float M = -INFINITY, den = 0.f;
            float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
            // the CTAs' partials, eight remote loads at a time
#pragma unroll
            for (int r0 = 0; r0 < kMaxCluster; r0 += 8) {
                if (r0 >= C) break;
                float2 mls[8];
                float4 vs[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    mls[i] = remote(cl, cml + g, r0 + i, C);
                    vs[i] = remote(cl, reinterpret_cast<float4*>(cacc + g * D) + d4, r0 + i, C);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (r0 + i < C) fold_partial(mls[i], vs[i], M, num, den);
            }
            for (long long kb = sk0; kb <= sk1; kb += 4) {  // four slots' loads at a time
                float2 mls[4];
                float4 vs[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const long long slot = u + min(kb + i, sk1);
                    mls[i] = __ldcg(a.part_ml + slot * G + g);
                    vs[i] = __ldcg(reinterpret_cast<const float4*>(
                                       a.part_acc + (slot * G + g) * D) + d4);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (kb + i <= sk1) fold_partial(mls[i], vs[i], M, num, den);
            }
            const float inv = den > 0.f ? 1.f / den : 0.f;
            reinterpret_cast<float4*>(a.out + ((long long)b * a.hq + h * G + g) * D)[d4] =
                make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
        }
        cl.sync();  // remote reads of this unit's shared memory are done
    }
}

template <int D>
cudaError_t setup_one(DeviceCfg& d, int di) {
    for (int ci = 0; ci < kNumFinishClusters; ++ci) {
        const int c = kFinishClusters[ci];
        const size_t smem = finish_smem<D>(c);
        // the smallest cluster needs the most shared memory (the largest
        // slices of the candidates)
        cudaError_t e = cudaFuncSetAttribute(
            finish_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
            (int)finish_smem<D>(kFinishClusters[kNumFinishClusters - 1]));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(finish_kernel<D>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(c);
        cfg.blockDim = dim3(FinishCfg<D>::NT);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = c;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, finish_kernel<D>, &cfg);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            n = 0;  // this cluster size cannot be used here
        }
        d.finish_clusters[di][ci] = n;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t setup_finish(DeviceCfg& d) {
    cudaError_t e = setup_one<128>(d, 0);
    if (e == cudaSuccess) e = setup_one<256>(d, 1);
    return e;
}

cudaError_t launch_finish(FinishParams p, int head_dim, const DeviceCfg& d,
                          cudaStream_t stream) {
    const int units = p.at.batch * p.at.hkv;
    if (units == 0) return cudaSuccess;
    const int di = head_dim == 128 ? 0 : 1;
    // the largest cluster size that still gives every unit its own cluster;
    // else the smaller size, whose clusters take several units each
    int ci = kNumFinishClusters - 1;
    for (int i = 0; i < kNumFinishClusters; ++i)
        if (d.finish_clusters[di][i] >= units) {
            ci = i;
            break;
        }
    const int c = kFinishClusters[ci];
    int ncl = d.finish_clusters[di][ci];
    if (ncl < 1) return cudaErrorInvalidConfiguration;
    if (ncl > units) ncl = units;
    const size_t smem = head_dim == 128 ? finish_smem<128>(c) : finish_smem<256>(c);
    if (head_dim == 128)
        return launch_pdl(finish_kernel<128>, dim3(ncl * c), dim3(FinishCfg<128>::NT), smem,
                          stream, c, p);
    return launch_pdl(finish_kernel<256>, dim3(ncl * c), dim3(FinishCfg<256>::NT), smem, stream,
                      c, p);
}

}  // namespace slc
