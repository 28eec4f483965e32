// Fused sparse decode step of one layer: page scoring, per-unit top-k
// selection, split-KV attention over prefix + window + selected pages
// ("Hybrid LLM Decoding 2.2x Faster at 256k, No Retraining", section "The
// method: sliding window + prefix + query-aware pages, searched per
// layer") in one persistent kernel, then the log-sum-exp merge.
//
// The CTAs of decode_kernel take two roles.
//   Selectors (the first S CTAs): selector s owns units s, s+S, ...; for
//     each it waits until every tile of the unit is scored, selects the
//     unit's pages and raises the unit's selection flag.
//   Streamers (the others) take work from two ticket counters:
//     1. per warp, scoring tiles (16 candidate pages of one unit), numbered
//        unit after unit so that units finish scoring one after another;
//        a warp counts each scored tile for its unit;
//     2. per CTA, attention chunks: first over the forced lists (prefix
//        pages, then window pages) of all units, then over the selected
//        pages of all units, unit after unit.  Before a unit's selected
//        pages the CTA waits for the unit's selection flag.
// Selection is latency-bound and runs beside the streams; by the time
// the streamers reach a unit's selected pages its selection is normally
// done.  Every wait is bounded: on timeout the kernel sets the
// wait-timeout status bit and goes on, so a fault shows as a status error,
// never as a hang.  Waits cannot deadlock: a streamer waits only after all
// scoring tiles have been claimed by running warps that never wait, and the
// selectors are the lowest-numbered CTAs, resident first.
//
// Partials: forced chunk c of unit u goes to slot u + c, selected chunk c
// to slot U + chunks_forced + u + c (U units); a chunk covers consecutive
// list positions, so each slot is written once.  merge_kernel then combines
// the slots of every (unit, query head), one CTA each.
#include "slc_attend_impl.cuh"
#include "slc_score_impl.cuh"
#include "slc_select_impl.cuh"

namespace slc {

namespace {

template <int D>
struct FusedCfg;
// D=128: three 4-warp CTAs per SM; attention rings of two stages, scoring
// rings of two tiles, 64 KB each.
template <>
struct FusedCfg<128> {
    static constexpr int NW = 4, STAGES = 2, NT = 2, MINB = 3;
};
// D=256: the attention registers allow two CTAs per SM; one stage and one
// tile per warp keep the data region at 64 KB.
template <>
struct FusedCfg<256> {
    static constexpr int NW = 4, STAGES = 1, NT = 1, MINB = 2;
};

template <int D>
struct FusedGeom : FusedCfg<D> {
    using B = FusedCfg<D>;
    static constexpr int NTHR = B::NW * 32;
    static constexpr int RING = B::STAGES * 2 * kPage * D * 2;        // attention ring per warp
    static constexpr int SRING = B::NT * scr::TileGeom<D>::TILE_B;  // scoring ring per warp
    static constexpr int DATA_ATT = B::NW * RING;
    static constexpr int DATA_SCORE = B::NW * SRING;
    static constexpr int DATA = DATA_ATT > DATA_SCORE ? DATA_ATT : DATA_SCORE;
    static constexpr int SMEM = DATA + B::NW * B::STAGES * (8 + 4);
    static_assert(DATA >= sel::kLiveBytes + 1024 * 8, "selection needs room for survivors");
};

constexpr int kChunkPages = 16;          // target pages per attention chunk
constexpr uint32_t kFlagWait = 1u << 22;  // bounded polls of a flag (~0.4 s)

// Counters (zeroed before the kernel): [0] scoring ticket, [1] attention
// ticket, [2, 2+U) tiles scored per unit, [2+U, 2+2U) selection flags.
struct Counters {
    int* score_ticket;
    int* attn_ticket;
    int* tiles_done;
    int* sel_done;
};
__device__ __forceinline__ Counters counters_of(const FusedParams& p) {
    const int U = p.sc.batch * p.sc.hkv;
    return Counters{p.counters, p.counters + 1, p.counters + 2, p.counters + 2 + U};
}

// Tiles to score for sequence b: none when the budget keeps every
// candidate (the selection is then the candidate range itself).
__device__ __forceinline__ int unit_tiles(const ScoreParams& p, int budget, int b) {
    const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
    const PageRanges r = page_ranges(L, p.prefix, p.window);
    const int ncand = r.ws - r.np;
    return ncand > budget ? (ncand + scr::kTilePages - 1) / scr::kTilePages : 0;
}

// Chunking of one list kind: total positions, chunk count, positions per
// chunk.  Warp-wide; every kernel computes it identically.
struct Chunking {
    long long total, chunks, cpp;
};
__device__ __forceinline__ Chunking chunking(const AttendParams& at) {
    auto len_of = [&](int b) { return attn::list_len(at, b); };
    Chunking c;
    c.total = total_units(at.batch, at.hkv, len_of);
    long long n = (c.total + kChunkPages - 1) / kChunkPages;
    if (n > kMaxAttendChunks) n = kMaxAttendChunks;
    c.cpp = n > 0 ? (c.total + n - 1) / n : 1;
    c.chunks = n > 0 ? (c.total + c.cpp - 1) / c.cpp : 0;
    return c;
}

__device__ __forceinline__ AttendParams with_list(const AttendParams& at, int list) {
    AttendParams r = at;
    r.list = list;
    return r;
}

// A tile of the scoring phase, as located by the issuing warp.
struct TileRef {
    int u, jt;
    PageRanges r;
    bool valid;
};

template <int D>
__device__ void selector(const FusedParams& p, const Counters& ctr, uint8_t* smem,
                         sel::Scratch<FusedGeom<D>::NTHR>& sc, int first, int stride) {
    using F = FusedGeom<D>;
    const ScoreParams& ps = p.sc;
    const int budget = p.se.budget;
    const int U = ps.batch * ps.hkv;
    for (int u = first; u < U; u += stride) {
        const int b = u / ps.hkv;
        const int nt = unit_tiles(ps, budget, b);
        if (nt == 0) {  // every candidate is kept
            const int L = checked_len(ps.seq_lens, b, ps.max_pages, ps.status);
            const PageRanges r = page_ranges(L, ps.prefix, ps.window);
            const int ncand = r.ws - r.np;
            int32_t* out = p.se.selected + (long long)u * budget;
            for (int i = threadIdx.x; i < budget; i += F::NTHR) out[i] = i < ncand ? r.np + i : -1;
        } else {
            if (threadIdx.x == 0 && !wait_at_least(ctr.tiles_done + u, nt, kFlagWait))
                atomicOr(ps.status, SLC_STATUS_WAIT_TIMEOUT);
            __syncthreads();
            sel::select_unit<F::NTHR>(p.se, u, smem, F::DATA, sc);
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) st_release(ctr.sel_done + u, 1);
    }
}

// Scoring phase of one streamer warp: claim tiles until none is left.
template <int D>
__device__ void score_tiles(const FusedParams& p, const Counters& ctr, uint8_t* sring,
                            int n_tiles) {
    using F = FusedGeom<D>;
    using TG = scr::TileGeom<D>;
    constexpr int NT = F::NT;
    const ScoreParams& ps = p.sc;
    const int budget = p.se.budget;
    const int lane = threadIdx.x & 31;
    // tickets: lane 0 claims one ahead; the value is read a tile later
    auto claim = [&]() { return lane == 0 ? atomicAdd(ctr.score_ticket, 1) : 0; };
    auto bcast = [&](int v) { return __shfl_sync(0xffffffffu, v, 0); };
    int cur = bcast(claim());
    if (cur >= n_tiles) return;
    int nxt = bcast(claim());
    // forward-only cursor over units (a warp's tickets grow)
    int cu = 0, cstart = 0, ccount = unit_tiles(ps, budget, 0);
    PageRanges cr = page_ranges(checked_len(ps.seq_lens, 0, ps.max_pages, ps.status),
                                ps.prefix, ps.window);
    auto locate = [&](int g) {
        TileRef t{};
        t.valid = g < n_tiles;
        if (!t.valid) return t;
        while (g >= cstart + ccount) {
            cstart += ccount;
            ++cu;
            const int b = cu / ps.hkv;
            cr = page_ranges(checked_len(ps.seq_lens, b, ps.max_pages, ps.status), ps.prefix,
                             ps.window);
            ccount = unit_tiles(ps, budget, b);
        }
        t.u = cu;
        t.jt = g - cstart;
        t.r = cr;
        return t;
    };
    int issued = 0, consumed = 0;
    auto issue = [&](const TileRef& t) {
        const int phys = scr::tile_phys(ps, t.u, t.r, t.jt);
        scr::copy_tile<D>(ps, t.u % ps.hkv, phys, sring + (issued % NT) * TG::TILE_B);
        ++issued;
    };
    // A tile is counted for its unit one tile later, after a fence that
    // then finds its score stores long completed (a fence right after them
    // would stall the warp on their acknowledgement).
    auto publish = [&](int u) {
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(ctr.tiles_done + u, 1);
    };
    int wu = -1, done_u = -1;
    float w[TG::CPL][8];
    TileRef tcur = locate(cur);
    issue(tcur);
    while (tcur.valid) {
        const TileRef tnxt = locate(nxt);
        const int after = tnxt.valid ? claim() : 0;
        bool nxt_issued = false;
        if (NT > 1 && tnxt.valid) {
            issue(tnxt);
            nxt_issued = true;
        }
        if (nxt_issued)
            cp_async_wait<1>();
        else
            cp_async_wait<0>();
        if (done_u >= 0) publish(done_u);
        if (tcur.u != wu) {
            wu = tcur.u;
            scr::load_weights<D>(ps, wu, w);
        }
        scr::score_tile<D>(ps, tcur.u, tcur.r, tcur.jt, sring + (consumed % NT) * TG::TILE_B, w);
        ++consumed;
        done_u = tcur.u;
        tcur = tnxt;
        nxt = tnxt.valid ? bcast(after) : n_tiles;
        if (tcur.valid && !nxt_issued) issue(tcur);
    }
    publish(done_u);
    cp_async_wait<0>();
}

template <int D>
__global__ void __launch_bounds__(FusedGeom<D>::NTHR, FusedGeom<D>::MINB)
    decode_kernel(FusedParams p, int selectors) {
    using F = FusedGeom<D>;
    constexpr int NW = F::NW;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ sel::Scratch<F::NTHR> sc;
    __shared__ int sh_ticket;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    attn::Ring ring;
    ring.tiles = smem + warp * F::RING;
    ring.bars = reinterpret_cast<uint64_t*>(smem + F::DATA) + warp * F::STAGES;
    ring.nvalid = reinterpret_cast<int*>(smem + F::DATA + NW * F::STAGES * 8) + warp * F::STAGES;
    if (lane == 0) {
        for (int s = 0; s < F::STAGES; ++s) mbar_init(ring.bars + s, 1);
        fence_mbar_init();
    }
    __syncwarp();

    // q, metadata and the zeroed counters come from preceding work
    grid_dep_wait();
    grid_dep_launch();

    const Counters ctr = counters_of(p);
    if ((int)blockIdx.x < selectors) {
        selector<D>(p, ctr, smem, sc, blockIdx.x, selectors);
        return;
    }

    const ScoreParams& ps = p.sc;
    const int budget = p.se.budget;
    auto tiles_of = [&](int b) { return unit_tiles(ps, budget, b); };
    const int n_tiles = budget > 0 ? (int)total_units(ps.batch, ps.hkv, tiles_of) : 0;
    if (n_tiles > 0) score_tiles<D>(p, ctr, smem + warp * F::SRING, n_tiles);
    __syncthreads();  // the scoring rings are idle: the data region turns to attention rings

    const AttendParams atF = with_list(p.at, kListForced);
    const AttendParams atS = with_list(p.at, kListSelected);
    const Chunking cf = chunking(atF), cs = chunking(atS);
    const long long n_tickets = cf.chunks + cs.chunks;
    const long long base_s = (long long)ps.batch * ps.hkv + cf.chunks;
    uint32_t it = 0;
    bool ok = true;
    auto wait_selection = [&](int u) {
        if (threadIdx.x == 0 && !wait_at_least(ctr.sel_done + u, 1, kFlagWait))
            atomicOr(ps.status, SLC_STATUS_WAIT_TIMEOUT);
        __syncthreads();
    };
    if (threadIdx.x == 0) sh_ticket = atomicAdd(ctr.attn_ticket, 1);
    __syncthreads();
    long long t = sh_ticket;
    while (t < n_tickets) {
        // the next ticket is claimed now and published after the chunk
        const int next = threadIdx.x == 0 ? atomicAdd(ctr.attn_ticket, 1) : 0;
        if (t < cf.chunks) {
            const long long s = t * cf.cpp;
            attn::attend_range<D, NW, F::STAGES>(atF, smem, ring, it, ok, s,
                                                 min(cf.total, s + cf.cpp), t, 0, [](int) {});
        } else {
            const long long c = t - cf.chunks;
            const long long s = c * cs.cpp;
            attn::attend_range<D, NW, F::STAGES>(atS, smem, ring, it, ok, s,
                                                 min(cs.total, s + cs.cpp), c, base_s,
                                                 wait_selection);
        }
        if (threadIdx.x == 0) sh_ticket = next;
        __syncthreads();
        t = sh_ticket;
        __syncthreads();  // every thread has read sh_ticket
    }
}

// Log-sum-exp merge of the split partials of one (unit, query head):
//   out = sum_k 2^(m_k - M) acc_k / sum_k 2^(m_k - M) l_k,  M = max_k m_k.
// The block's threads split into kMergeGroups slot groups x D/4 dimension
// quads; each group folds its slots with online rescaling, then the groups
// combine in shared memory.
constexpr int kMergeGroups = 4;

template <int D>
__global__ void __launch_bounds__(kMergeGroups * D / 4) merge_kernel(FusedParams p) {
    constexpr int V4 = D / 4;
    const int u = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x;
    const int grp = tid / V4, d4 = tid % V4;
    const AttendParams atF = with_list(p.at, kListForced);
    const AttendParams atS = with_list(p.at, kListSelected);
    const int b = u / atF.hkv, h = u % atF.hkv;
    const int G = atF.group;
    __shared__ long long sh_r[4];
    __shared__ float sh_m[kMergeGroups];
    __shared__ float4 sh_num[kMergeGroups][V4];
    __shared__ float sh_den[kMergeGroups];
    if (tid < 32) {
        const Chunking cf = chunking(atF), cs = chunking(atS);
        const long long sA = attn::unit_list_start(atF, u);
        const long long sB = attn::unit_list_start(atS, u);
        const int lenA = attn::list_len(atF, b), lenB = attn::list_len(atS, b);
        const long long base_s = (long long)atF.batch * atF.hkv + cf.chunks;
        if (tid == 0) {
            sh_r[0] = lenA > 0 ? u + sA / cf.cpp : 0;
            sh_r[1] = lenA > 0 ? u + (sA + lenA - 1) / cf.cpp : -1;
            sh_r[2] = lenB > 0 ? base_s + u + sB / cs.cpp : 0;
            sh_r[3] = lenB > 0 ? base_s + u + (sB + lenB - 1) / cs.cpp : -1;
        }
    }
    __syncthreads();
    const long long a0 = sh_r[0], a1 = sh_r[1], b0 = sh_r[2], b1 = sh_r[3];
    const long long na = a1 - a0 + 1, nb = b1 - b0 + 1;
    grid_dep_wait();  // the partials come from the decode kernel
    float M = -INFINITY, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (long long i = grp; i < na + nb; i += kMergeGroups) {
        const long long k = i < na ? a0 + i : b0 + (i - na);
        const float2 ml = __ldg(&p.at.part_ml[k * G + g]);
        const float4 a =
            __ldg(reinterpret_cast<const float4*>(p.at.part_acc + (k * G + g) * D) + d4);
        if (ml.x > M) {  // new maximum: rescale what was summed so far
            const float c = ex2(M - ml.x);
            num.x *= c;
            num.y *= c;
            num.z *= c;
            num.w *= c;
            den *= c;
            M = ml.x;
        }
        const float w = ml.x == -INFINITY ? 0.f : ex2(ml.x - M);  // empty partial
        num.x = fmaf(w, a.x, num.x);
        num.y = fmaf(w, a.y, num.y);
        num.z = fmaf(w, a.z, num.z);
        num.w = fmaf(w, a.w, num.w);
        den = fmaf(w, ml.y, den);
    }
    sh_num[grp][d4] = num;
    if (d4 == 0) {
        sh_den[grp] = den;
        sh_m[grp] = M;
    }
    __syncthreads();
    if (grp == 0) {
        float Mt = -INFINITY;
#pragma unroll
        for (int i = 0; i < kMergeGroups; ++i) Mt = fmaxf(Mt, sh_m[i]);
        const float Mu = Mt == -INFINITY ? 0.f : Mt;
        float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
        float dt = 0.f;
#pragma unroll
        for (int i = 0; i < kMergeGroups; ++i) {
            const float c = ex2(sh_m[i] - Mu);  // 0 for an empty group
            const float4 o = sh_num[i][d4];
            tot.x = fmaf(c, o.x, tot.x);
            tot.y = fmaf(c, o.y, tot.y);
            tot.z = fmaf(c, o.z, tot.z);
            tot.w = fmaf(c, o.w, tot.w);
            dt = fmaf(c, sh_den[i], dt);
        }
        const float inv = dt > 0.f ? 1.f / dt : 0.f;
        float* outp = p.at.out + ((long long)b * p.at.hq + h * G + g) * D;
        reinterpret_cast<float4*>(outp)[d4] =
            make_float4(tot.x * inv, tot.y * inv, tot.z * inv, tot.w * inv);
    }
}

template <int D>
cudaError_t run_fused(const FusedParams& p, int num_sms, cudaStream_t stream) {
    using F = FusedGeom<D>;
    static int occ = 0;
    if (occ == 0) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel<D>, F::NTHR,
                                                              F::SMEM);
        if (e != cudaSuccess) return e;
        if (occ < 1) occ = 1;
    }
    const int U = p.sc.batch * p.sc.hkv;
    const int grid = num_sms * occ;
    // selectors: one per unit up to 16, never more than a quarter of the grid
    int selectors = p.se.budget > 0 ? (U < 16 ? U : 16) : 0;
    if (selectors > grid / 4) selectors = grid / 4;
    cudaError_t e = cudaMemsetAsync(p.counters, 0, (size_t)(2 + 2 * U) * sizeof(int), stream);
    if (e != cudaSuccess) return e;
    e = launch_pdl(decode_kernel<D>, dim3(grid), dim3(F::NTHR), F::SMEM, stream, p, selectors);
    if (e != cudaSuccess) return e;
    return launch_pdl(merge_kernel<D>, dim3(U, p.at.group), dim3(kMergeGroups * D / 4), 0, stream,
                      p);
}

}  // namespace

cudaError_t launch_sparse_fused(const FusedParams& p, int head_dim, int num_sms,
                                cudaStream_t stream) {
    if (p.sc.batch * p.sc.hkv == 0) return cudaSuccess;
    if (head_dim == 128) return run_fused<128>(p, num_sms, stream);
    return run_fused<256>(p, num_sms, stream);
}

}  // namespace slc
