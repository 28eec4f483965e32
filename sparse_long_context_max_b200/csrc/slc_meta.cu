// Page metadata kernels: per-page elementwise key min/max (the bounds behind
// Quest-style paged selection, "Hybrid LLM Decoding 2.2x Faster at 256k, No
// Retraining", section "The method: sliding window + prefix + query-aware
// pages, searched per layer").
//
//   kv_append        writes one token per (sequence, kv head) and folds it
//                    into its page's bounds (slot 0 resets them);
//   build_page_meta  rebuilds the bounds of every page from the keys.
//
// min/max of bf16 values is a bf16 value, so the metadata is exact and the
// incremental and rebuilt forms are bit-identical (up to the sign of zero).
// E4M3 metadata (SLC_META_FP8_E4M3) stores the bounds rounded outward;
// outward rounding is monotone, so min(round_down(a), round_down(b)) =
// round_down(min(a, b)) and the incremental and rebuilt E4M3 bounds are
// identical too.
#include "slc_internal.h"

namespace slc {

namespace {

constexpr uint32_t kPosInf2 = 0x7f807f80u;  // bf16x2 (+inf, +inf)
constexpr uint32_t kNegInf2 = 0xff80ff80u;  // bf16x2 (-inf, -inf)

__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmin2(*reinterpret_cast<__nv_bfloat162*>(&a),
                               *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&a),
                               *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint4 min4(uint4 a, uint4 b) {
    return make_uint4(bmin2(a.x, b.x), bmin2(a.y, b.y), bmin2(a.z, b.z), bmin2(a.w, b.w));
}
__device__ __forceinline__ uint4 max4(uint4 a, uint4 b) {
    return make_uint4(bmax2(a.x, b.x), bmax2(a.y, b.y), bmax2(a.z, b.z), bmax2(a.w, b.w));
}
__device__ __forceinline__ uint4 shfl_xor4(uint4 v, int m) {
    return make_uint4(__shfl_xor_sync(0xffffffffu, v.x, m), __shfl_xor_sync(0xffffffffu, v.y, m),
                      __shfl_xor_sync(0xffffffffu, v.z, m), __shfl_xor_sync(0xffffffffu, v.w, m));
}

// 8 bf16 (one 16-byte chunk) rounded outward to E4M3: 8 codes, low byte first.
__device__ __forceinline__ uint2 round8(uint4 v, bool up) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float f = (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
        c[i >> 2] |= e4m3_round(f, up) << (8 * (i & 3));
    }
    return make_uint2(c[0], c[1]);
}

// Bytewise min (up = false) or max (up = true) of two sets of 8 E4M3 codes,
// by value.
__device__ __forceinline__ uint2 pick8(uint2 a, uint2 b, bool up) {
    const uint32_t wa[2] = {a.x, a.y}, wb[2] = {b.x, b.y};
    uint32_t r[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t ca = (wa[i >> 2] >> (8 * (i & 3))) & 0xFFu;
        const uint32_t cb = (wb[i >> 2] >> (8 * (i & 3))) & 0xFFu;
        const float va = e4m3_value(ca), vb = e4m3_value(cb);
        const uint32_t c = up ? (vb > va ? cb : ca) : (vb < va ? cb : ca);
        r[i >> 2] |= c << (8 * (i & 3));
    }
    return make_uint2(r[0], r[1]);
}

// One warp per (sequence, kv head).  Chunk c < D/8 of the row is a 16-byte
// piece of k, chunk c >= D/8 a piece of v.
template <int D>
__global__ void __launch_bounds__(128) kv_append_kernel(KvAppendParams p) {
    grid_dep_wait();
    grid_dep_launch();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= p.batch * p.hkv) return;
    const int b = warp / p.hkv, h = warp % p.hkv;
    const int pos = p.positions[b];
    if (pos < 0 || pos >= p.max_pages * kPage) {
        if (lane == 0) atomicOr(p.status, SLC_STATUS_BAD_LENGTH);
        return;
    }
    const int j = pos / kPage, slot = pos % kPage;
    const int phys = p.block_table[(long long)b * p.max_pages + j];
    if (phys < 0 || phys >= p.num_pages) {
        if (lane == 0) atomicOr(p.status, SLC_STATUS_BAD_PAGE);
        return;
    }
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    const long long tile = (long long)phys * p.hkv + h;
    const uint4* src_k = reinterpret_cast<const uint4*>(p.k_new) + ((long long)b * p.hkv + h) * CPR;
    const uint4* src_v = reinterpret_cast<const uint4*>(p.v_new) + ((long long)b * p.hkv + h) * CPR;
    uint4* dst_k = reinterpret_cast<uint4*>(p.k_cache) + (tile * kPage + slot) * CPR;
    uint4* dst_v = reinterpret_cast<uint4*>(p.v_cache) + (tile * kPage + slot) * CPR;
    const bool fp8 = p.meta_format == SLC_META_FP8_E4M3;
    uint4* meta = reinterpret_cast<uint4*>(p.meta) + tile * 2 * CPR;
    uint2* meta8 = reinterpret_cast<uint2*>(p.meta) + tile * 2 * CPR;  // [2][D] bytes
#pragma unroll
    for (int c = lane; c < 2 * CPR; c += 32) {
        if (c < CPR) {
            const uint4 k = src_k[c];
            dst_k[c] = k;
            if (fp8) {
                const uint2 dn = round8(k, false), up = round8(k, true);
                meta8[c] = slot == 0 ? dn : pick8(meta8[c], dn, false);
                meta8[CPR + c] = slot == 0 ? up : pick8(meta8[CPR + c], up, true);
            } else if (slot == 0) {
                meta[c] = k;
                meta[CPR + c] = k;
            } else {
                meta[c] = min4(meta[c], k);
                meta[CPR + c] = max4(meta[CPR + c], k);
            }
        } else {
            dst_v[c - CPR] = src_v[c - CPR];
        }
    }
}

// One warp per (sequence, logical page, kv head), grid-stride.  For D=128 a
// row is 16 chunks, so lanes l and l^16 split the 16 rows between them and
// combine with one shuffle; for D=256 each lane owns one chunk column.
template <int D>
__global__ void __launch_bounds__(256) build_meta_kernel(BuildMetaParams p) {
    constexpr int CPR = D / 8;
    static_assert(CPR == 16 || CPR == 32, "head_dim 128 or 256");
    constexpr int RG = 32 / CPR;  // row groups per warp
    const int lane = threadIdx.x & 31;
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    const long long total = (long long)p.batch * p.max_pages * p.hkv;
    for (long long task = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; task < total;
         task += nwarps) {
        const int h = (int)(task % p.hkv);
        const long long bj = task / p.hkv;
        const int j = (int)(bj % p.max_pages);
        const int b = (int)(bj / p.max_pages);
        const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
        const int valid = min(kPage, L - j * kPage);
        if (valid <= 0) continue;
        const int phys = p.block_table[(long long)b * p.max_pages + j];
        if (phys < 0 || phys >= p.num_pages) {
            if (lane == 0) atomicOr(p.status, SLC_STATUS_BAD_PAGE);
            continue;
        }
        const long long tile = (long long)phys * p.hkv + h;
        const uint4* k = reinterpret_cast<const uint4*>(p.k_cache) + tile * kPage * CPR;
        const int col = lane % CPR, rg = lane / CPR;
        uint4 mn = make_uint4(kPosInf2, kPosInf2, kPosInf2, kPosInf2);
        uint4 mx = make_uint4(kNegInf2, kNegInf2, kNegInf2, kNegInf2);
#pragma unroll
        for (int i = 0; i < kPage / RG; ++i) {
            const int row = rg * (kPage / RG) + i;
            if (row < valid) {
                const uint4 v = __ldcs(k + row * CPR + col);
                mn = min4(mn, v);
                mx = max4(mx, v);
            }
        }
        if (RG == 2) {
            mn = min4(mn, shfl_xor4(mn, 16));
            mx = max4(mx, shfl_xor4(mx, 16));
        }
        if (p.meta_format == SLC_META_FP8_E4M3) {  // the bounds rounded outward
            uint2* meta8 = reinterpret_cast<uint2*>(p.meta) + tile * 2 * CPR;
            if (RG == 2) {
                if (rg == 0) meta8[col] = round8(mn, false);
                else meta8[CPR + col] = round8(mx, true);
            } else {
                meta8[col] = round8(mn, false);
                meta8[CPR + col] = round8(mx, true);
            }
            continue;
        }
        uint4* meta = reinterpret_cast<uint4*>(p.meta) + tile * 2 * CPR;
        if (RG == 2) {
            if (rg == 0) meta[col] = mn;
            else meta[CPR + col] = mx;
        } else {
            meta[col] = mn;
            meta[CPR + col] = mx;
        }
    }
}

}  // namespace

cudaError_t launch_kv_append(const KvAppendParams& p, int head_dim, cudaStream_t stream) {
    const int warps = p.batch * p.hkv;
    const int threads = 128;
    const int blocks = (warps * 32 + threads - 1) / threads;
    if (head_dim == 128)
        return launch_pdl(kv_append_kernel<128>, dim3(blocks), dim3(threads), 0, stream, 1, p);
    return launch_pdl(kv_append_kernel<256>, dim3(blocks), dim3(threads), 0, stream, 1, p);
}

cudaError_t launch_build_meta(const BuildMetaParams& p, int head_dim, const DeviceCfg& d,
                              cudaStream_t stream) {
    const int num_sms = d.num_sms;
    const long long tasks = (long long)p.batch * p.max_pages * p.hkv;
    const int threads = 256;
    long long blocks = (tasks * 32 + threads - 1) / threads;
    const long long cap = (long long)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (head_dim == 128)
        build_meta_kernel<128><<<(int)blocks, threads, 0, stream>>>(p);
    else
        build_meta_kernel<256><<<(int)blocks, threads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace slc
