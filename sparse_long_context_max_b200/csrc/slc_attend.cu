// Split-KV flash-decode over a paged bf16 KV cache, and the log-sum-exp
// merge of the split partials.
//
// Each (sequence, kv head) unit attends a list of logical pages:
//   dense   all pages [0, n)                       (every key, each step:
//           "Hybrid LLM Decoding 2.2x Faster at 256k, No Retraining",
//           section "The remaining full-attention layers are the
//           long-context bill")
//   forced  prefix pages, then window pages (the part of the sparse step
//           that needs no selection; same article, section "The method:
//           sliding window + prefix + query-aware pages, searched per
//           layer"), attended by the streaming kernel (slc_stream.cu)
// This file holds the dense kernel and the merge; the per-warp attention is
// in slc_attend_impl.cuh.
// The lists of all units are concatenated and cut into equal chunks, one per
// CTA of a persistent grid, so work is balanced by pages whatever the
// sequence lengths.  A chunk that spans unit boundaries yields one partial
// (running max m, sum l, unnormalised accumulator) per unit piece, stored in
// slot (unit + chunk), which is unique.  The merge kernel combines a unit's
// partials: out = sum_k 2^(m_k - M) acc_k / sum_k 2^(m_k - M) l_k.
//
// Within a CTA the warps take a piece's pages round-robin and combine their
// partials in shared memory.  Per warp, pages stream through a private ring
// of shared-memory stages,
// each filled by two 1-D bulk copies (TMA engine: the K and V tiles of one
// (page, kv head) are contiguous, 32*D bytes each) completing on an
// mbarrier.  The group's query heads (G <= 8) and the 16 tokens of a page
// are contracted on tensor cores with mma.sync m16n8k16 (bf16 in, fp32
// accumulate):
//   S   = Q K^T : A = Q (heads padded to 16 rows), B = K^T, 16 mma per page
//   O^T += V^T P^T : A = V^T (16 dims per m-block), B = P^T (8 heads)
// P is split into bf16 hi + lo parts (two mma per m-block) so the weights
// carry ~16 mantissa bits.  The head_dim contraction index is permuted so
// that each thread reads 16-byte vectors: logical k-step 2m / 2m+1 of thread
// (r, c) covers physical dims 8*(c+4m)..8*(c+4m)+7, identically for Q and K.
// For P V, thread (r, c) owns dims (D/8)*r .. (D/8)*r + D/8 - 1, read as
// 16-byte vectors and paired across tokens with byte permutes.
#include "slc_attend_impl.cuh"

namespace slc {

namespace {

using namespace attn;

// One CTA per chunk of the concatenated page lists.  For every unit piece
// of the chunk, the CTA's warps take its pages round-robin, then combine
// their partials in shared memory (reusing their rings) into one partial,
// stored in slot (unit + chunk).
template <int D, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32, (D == 128 && NW == 4) ? 3 : 1)
    attend_kernel(AttendParams p) {
    constexpr int TILE = kPage * D * 2;
    constexpr int RING = STAGES * 2 * TILE;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Ring ring;
    ring.tiles = smem + warp * RING;
    ring.bars = reinterpret_cast<uint64_t*>(smem + NW * RING) + warp * STAGES;
    ring.nvalid = reinterpret_cast<int*>(smem + NW * RING + NW * STAGES * 8) + warp * STAGES;
    if (lane == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(ring.bars + s, 1);
        fence_mbar_init();
    }
    __syncwarp();
    grid_dep_launch();  // the merge may start; it waits before reading partials

    auto len_of = [&](int b) { return list_len(p, b); };
    const long long total = total_units(p.batch, p.hkv, len_of);
    const long long cpp = (total + gridDim.x - 1) / gridDim.x;
    const long long s = (long long)blockIdx.x * cpp;
    const long long e = min(total, s + cpp);
    // every read of data waits for the preceding kernel (which may be writing
    // the cache, or reading the partial slots)
    grid_dep_wait();
    uint32_t it = 0;
    bool ok = true;
    attend_range<D, NW, STAGES>(p, smem, ring, it, ok, s, e, blockIdx.x);
}

// Merge of the CTA partials of one (unit, query head): slots unit + chunk
// for the chunks that cover the unit.  The block's threads split into
// MERGE_GROUPS slot groups x D/4 dimension quads; groups combine in shared
// memory.
constexpr int kMergeGroups = 4;

template <int D>
__global__ void __launch_bounds__(kMergeGroups * D / 4) merge_kernel(AttendParams p) {
    constexpr int V4 = D / 4;
    const int u = blockIdx.x, g = blockIdx.y;
    const int b = u / p.hkv;
    const int G = p.group;
    const int tid = threadIdx.x;
    const int grp = tid / V4, d4 = tid % V4;
    __shared__ long long sh_off, sh_total;
    __shared__ float sh_m[kMergeGroups];
    __shared__ float4 sh_num[kMergeGroups][V4];
    __shared__ float sh_den[kMergeGroups];
    if (tid < 32) {
        auto len_of = [&](int bb) { return list_len(p, bb); };
        const long long total = total_units(p.batch, p.hkv, len_of);
        const long long base = unit_list_start(p, u);
        if (tid == 0) {
            sh_off = base;
            sh_total = total;
        }
    }
    __syncthreads();
    const int len = list_len(p, b);
    float* outp = p.out + ((long long)b * p.hq + (u % p.hkv) * G + g) * D;
    if (len == 0) {
        grid_dep_wait();
        if (grp == 0) reinterpret_cast<float4*>(outp)[d4] = make_float4(0.f, 0.f, 0.f, 0.f);
        return;
    }
    const long long cpp = (sh_total + p.num_chunks - 1) / p.num_chunks;
    const long long k0 = sh_off / cpp, k1 = (sh_off + len - 1) / cpp;
    grid_dep_wait();  // the partials come from the attention kernel
    // one pass per slot group with online rescaling; slots of a group are
    // independent loads
    float M = -INFINITY, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (long long k = k0 + grp; k <= k1; k += kMergeGroups) {
        const float2 ml = __ldg(&p.part_ml[(u + k) * G + g]);
        const float4 a =
            __ldg(reinterpret_cast<const float4*>(p.part_acc + ((u + k) * G + g) * D) + d4);
        fold_partial(ml, a, M, num, den);
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
        reinterpret_cast<float4*>(outp)[d4] =
            make_float4(tot.x * inv, tot.y * inv, tot.z * inv, tot.w * inv);
    }
}

template <int D, int NW, int STAGES>
constexpr int attend_smem() {
    return NW * STAGES * (2 * kPage * D * 2 + 8 + 4);
}

template <int D, int NW, int STAGES>
cudaError_t setup_one(int* occ) {
    constexpr int smem = attend_smem<D, NW, STAGES>();
    cudaError_t e = cudaFuncSetAttribute(attend_kernel<D, NW, STAGES>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, attend_kernel<D, NW, STAGES>,
                                                      NW * 32, smem);
    if (e != cudaSuccess) return e;
    if (*occ < 1) *occ = 1;
    return cudaSuccess;
}

// One CTA (chunk) per resident slot of the GPU, at most kMaxAttendChunks.
template <int D, int NW, int STAGES>
cudaError_t run(AttendParams p, int occ, int num_sms, cudaStream_t stream) {
    constexpr int smem = attend_smem<D, NW, STAGES>();
    int blocks = num_sms * occ;
    if (blocks > kMaxAttendChunks) blocks = kMaxAttendChunks;
    p.num_chunks = blocks;
    cudaError_t e = launch_pdl(attend_kernel<D, NW, STAGES>, dim3(blocks), dim3(NW * 32), smem,
                               stream, 1, p);
    if (e != cudaSuccess) return e;
    return launch_pdl(merge_kernel<D>, dim3(p.batch * p.hkv, p.group),
                      dim3(kMergeGroups * D / 4), 0, stream, 1, p);
}

}  // namespace

// The dense list streams every page: at d = 128 one 8-warp CTA per SM with
// two ring stages per warp keeps the most bytes in flight.
cudaError_t setup_attend(DeviceCfg& d) {
    cudaError_t e = setup_one<128, 8, 2>(&d.occ_attend[1]);
    if (e == cudaSuccess) e = setup_one<256, 4, 3>(&d.occ_attend[2]);
    d.occ_attend[0] = 0;
    return e;
}

cudaError_t launch_dense(AttendParams p, int head_dim, const DeviceCfg& d, cudaStream_t stream) {
    if (p.batch * p.hkv == 0) return cudaSuccess;
    p.list = kListDense;
    if (head_dim == 128) return run<128, 8, 2>(p, d.occ_attend[1], d.num_sms, stream);
    return run<256, 4, 3>(p, d.occ_attend[2], d.num_sms, stream);
}

}  // namespace slc
