// Sparse decode step of one layer ("Hybrid LLM Decoding 2.2x Faster at
// 256k, No Retraining", section "The method: sliding window + prefix +
// query-aware pages, searched per layer"): four kernels chained by
// programmatic dependent launch, none of whose CTAs ever waits for another.
//
//   1. score_forced_kernel (persistent): every CTA first attends one chunk
//      of the forced lists (prefix pages, then window pages) of all units,
//      cut into about one chunk per CTA; then every warp scores candidate
//      tiles (16 pages of one unit) strided over the grid's warps.  Both
//      halves stream HBM; the forced attention needs no selection, so it
//      rides along with the scoring, and the scores are written last, so
//      the selection finds them in L2.
//   2. select_kernel (slc_select.cu): one CTA per unit, from the scores the
//      first kernel left; one more CTA per unit merges its forced-chunk
//      partials.
//   3. attend_kernel (slc_attend.cu) over the selected pages of all units.
//   4. merge_kernel: log-sum-exp merge of both kernels' partials per (unit,
//      query head).
//
// Partials: forced chunk c of unit u goes to slot u + c, selected chunk c
// to slot U + kMaxAttendChunks + u + c (U units); a chunk covers
// consecutive list positions, so each slot is written once.  Extra CTAs of
// the selection kernel merge each unit's forced-chunk partials into slot
// 2 (U + kMaxAttendChunks) + u while the selection runs, so the final merge
// combines that one slot with the selected-chunk slots.
#include "slc_attend_impl.cuh"
#include "slc_score_impl.cuh"

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
};

// Tiles to score for sequence b: none when the budget keeps every
// candidate (the selection is then the candidate range itself).
__device__ __forceinline__ int unit_tiles(const ScoreParams& p, int budget, int b) {
    const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
    const PageRanges r = page_ranges(L, p.prefix, p.window);
    const int ncand = r.ws - r.np;
    return ncand > budget ? (ncand + scr::kTilePages - 1) / scr::kTilePages : 0;
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

// Scoring by one warp: tiles w, w + nw, w + 2 nw, ... (w this warp's index
// among the grid's nw warps).  Tiles are numbered sequence after sequence
// and, within a sequence, (tile, kv head): at any moment the warps sweep
// consecutive tiles, and the kv heads' metadata rows of a page (adjacent
// in memory) are read together.
template <int D>
__device__ void score_tiles(const FusedParams& p, uint8_t* sring, int n_tiles, int w, int nw) {
    using F = FusedGeom<D>;
    using TG = scr::TileGeom<D>;
    constexpr int NT = F::NT;
    const ScoreParams& ps = p.sc;
    const int budget = p.se.budget;
    if (w >= n_tiles) return;
    // forward-only cursor over sequences (a warp's tiles grow)
    int cb = 0, cstart = 0, ccount = unit_tiles(ps, budget, 0) * ps.hkv;
    PageRanges cr = page_ranges(checked_len(ps.seq_lens, 0, ps.max_pages, ps.status),
                                ps.prefix, ps.window);
    auto locate = [&](int g) {
        TileRef t{};
        t.valid = g < n_tiles;
        if (!t.valid) return t;
        while (g >= cstart + ccount) {
            cstart += ccount;
            ++cb;
            cr = page_ranges(checked_len(ps.seq_lens, cb, ps.max_pages, ps.status), ps.prefix,
                             ps.window);
            ccount = unit_tiles(ps, budget, cb) * ps.hkv;
        }
        const int k = g - cstart;
        t.u = cb * ps.hkv + k % ps.hkv;
        t.jt = k / ps.hkv;
        t.r = cr;
        return t;
    };
    int issued = 0, consumed = 0;
    auto issue = [&](const TileRef& t) {
        const int phys = scr::tile_phys(ps, t.u, t.r, t.jt);
        scr::copy_tile<D>(ps, t.u % ps.hkv, phys, sring + (issued % NT) * TG::TILE_B);
        ++issued;
    };
    int wu = -1;
    float wt[TG::CPL][8];
    TileRef tcur = locate(w);
    issue(tcur);
    for (int g = w; tcur.valid; g += nw) {
        const TileRef tnxt = locate(g + nw);
        bool nxt_issued = false;
        if (NT > 1 && tnxt.valid) {
            issue(tnxt);
            nxt_issued = true;
        }
        if (nxt_issued)
            cp_async_wait<1>();
        else
            cp_async_wait<0>();
        if (tcur.u != wu) {
            wu = tcur.u;
            scr::load_weights<D>(ps, wu, wt);
        }
        scr::score_tile<D>(ps, tcur.u, tcur.r, tcur.jt, sring + (consumed % NT) * TG::TILE_B,
                           wt);
        ++consumed;
        tcur = tnxt;
        if (tcur.valid && !nxt_issued) issue(tcur);
    }
    cp_async_wait<0>();
}

template <int D>
__global__ void __launch_bounds__(FusedGeom<D>::NTHR, FusedGeom<D>::MINB)
    score_forced_kernel(FusedParams p) {
    using F = FusedGeom<D>;
    constexpr int NW = F::NW;
    extern __shared__ __align__(128) uint8_t smem[];
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

    // q and the metadata come from preceding work; partial slots may still
    // be read by a preceding merge
    grid_dep_wait();
    grid_dep_launch();

    const AttendParams atF = with_list(p.at, kListForced);
    const attn::Chunking cf = attn::forced_chunking(atF, p.forced_chunks);
    uint32_t it = 0;
    bool ok = true;
    for (long long c = blockIdx.x; c < cf.chunks; c += gridDim.x) {
        const long long s = c * cf.cpp;
        attn::attend_range<D, NW, F::STAGES>(atF, smem, ring, it, ok, s, min(cf.total, s + cf.cpp),
                                             c, 0, [](int) {});
    }
    __syncthreads();  // the attention rings are idle: the data region turns to scoring rings

    const ScoreParams& ps = p.sc;
    const int budget = p.se.budget;
    auto tiles_of = [&](int b) { return unit_tiles(ps, budget, b); };
    const int n_tiles = budget > 0 ? (int)total_units(ps.batch, ps.hkv, tiles_of) : 0;
    if (n_tiles > 0)
        score_tiles<D>(p, smem + warp * F::SRING, n_tiles, blockIdx.x * NW + warp, gridDim.x * NW);
}

// Log-sum-exp merge of the split partials of one (unit, query head):
//   out = sum_k 2^(m_k - M) acc_k / sum_k 2^(m_k - M) l_k,  M = max_k m_k,
// over the forced-list slots and the selected-list slots of the unit.  The
// block's threads split into kMergeGroups slot groups x D/4 dimension
// quads; each group folds its slots with online rescaling, then the groups
// combine in shared memory.
constexpr int kMergeGroups = 8;

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
        const attn::Chunking cf = attn::forced_chunking(atF, p.forced_chunks);
        auto len_sel = [&](int bb) { return attn::list_len(atS, bb); };
        const long long totalS = total_units(atS.batch, atS.hkv, len_sel);
        const long long cppS = totalS > 0 ? (totalS + p.at.num_chunks - 1) / p.at.num_chunks : 1;
        const long long sA = attn::unit_list_start(atF, u);
        const long long sB = attn::unit_list_start(atS, u);
        const int lenA = attn::list_len(atF, b), lenB = attn::list_len(atS, b);
        if (tid == 0) {
            // the forced-list partials, merged into one slot by the selection
            // kernel when it ran
            const bool pre = p.premerged_base >= 0;
            sh_r[0] = lenA > 0 ? (pre ? p.premerged_base + u : u + sA / cf.cpp) : 0;
            sh_r[1] = lenA > 0 ? (pre ? p.premerged_base + u : u + (sA + lenA - 1) / cf.cpp) : -1;
            sh_r[2] = lenB > 0 ? p.at.slot_base + u + sB / cppS : 0;
            sh_r[3] = lenB > 0 ? p.at.slot_base + u + (sB + lenB - 1) / cppS : -1;
        }
    }
    __syncthreads();
    const long long a0 = sh_r[0], a1 = sh_r[1], b0 = sh_r[2], b1 = sh_r[3];
    const long long na = a1 - a0 + 1, nb = b1 - b0 + 1;
    grid_dep_wait();  // the partials come from the attention kernels
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

// stage 0: the four kernels; 1..4: that kernel alone.
template <int D>
cudaError_t run_sparse(const FusedParams& p, int num_sms, cudaStream_t stream, int stage) {
    using F = FusedGeom<D>;
    static int occ = 0;
    if (occ == 0) {
        cudaError_t e = cudaFuncSetAttribute(score_forced_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, score_forced_kernel<D>,
                                                              F::NTHR, F::SMEM);
        if (e != cudaSuccess) return e;
        if (occ < 1) occ = 1;
    }
    const int U = p.sc.batch * p.sc.hkv;
    const int grid = num_sms * occ;
    FusedParams q = p;
    q.forced_chunks = grid;  // about one chunk per CTA
    cudaError_t e = cudaSuccess;
    if (stage == 0 || stage == 1)
        e = launch_pdl(score_forced_kernel<D>, dim3(grid), dim3(F::NTHR), F::SMEM, stream, q);
    if (e != cudaSuccess) return e;
    q.at.list = kListSelected;
    q.at.slot_base = (long long)U + kMaxAttendChunks;
    q.at.num_chunks = 1;
    q.premerged_base = -1;
    if (p.se.budget > 0) {
        PremergeParams pm;
        pm.at = p.at;
        pm.at.list = kListForced;
        pm.forced_chunks = grid;
        pm.dst_base = 2 * ((long long)U + kMaxAttendChunks);
        pm.v4 = D / 4;
        q.premerged_base = pm.dst_base;
        if (stage == 0 || stage == 2) e = launch_select(p.se, stream, &pm);
        if (e != cudaSuccess) return e;
        // the attention launcher sets num_chunks, which the merge needs
        AttendParams at = q.at;
        if (stage == 0 || stage == 3)
            e = launch_attend_partials(at, D, num_sms, stream);
        else
            at.num_chunks = attend_chunks(D, num_sms);
        if (e != cudaSuccess) return e;
        q.at.num_chunks = at.num_chunks;
    }
    if (stage == 0 || stage == 4)
        e = launch_pdl(merge_kernel<D>, dim3(U, p.at.group), dim3(kMergeGroups * D / 4), 0, stream,
                       q);
    return e;
}

}  // namespace

cudaError_t launch_sparse_fused(const FusedParams& p, int head_dim, int num_sms,
                                cudaStream_t stream, int stage) {
    if (p.sc.batch * p.sc.hkv == 0) return cudaSuccess;
    if (head_dim == 128) return run_sparse<128>(p, num_sms, stream, stage);
    return run_sparse<256>(p, num_sms, stream, stage);
}

}  // namespace slc
