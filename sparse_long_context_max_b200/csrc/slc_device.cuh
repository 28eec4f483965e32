// Device-side helpers shared by the sm_100a kernels of libslc.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/slc.h"

namespace slc {

constexpr int kPage = 16;        // tokens per page
constexpr int kMaxGroup = 8;     // query heads per kv head handled per warp
constexpr int kMaxCandidates = 32768;

// ---------------------------------------------------------------- ranges
// Page ranges of one sequence of L tokens (see include/slc.h):
// n pages, prefix [0, np), candidates [np, ws), window [ws, n).
struct PageRanges {
    int n, np, ws;
};

__device__ __forceinline__ PageRanges page_ranges(int L, int prefix, int window) {
    PageRanges r;
    r.n = L > 0 ? (L + kPage - 1) / kPage : 0;
    r.np = min((prefix + kPage - 1) / kPage, r.n);
    int ws = r.n;
    if (window > 0) ws = max(L - window, 0) / kPage;
    r.ws = min(max(ws, r.np), r.n);
    return r;
}

// Sequence length with the device-side range check applied.
__device__ __forceinline__ int checked_len(const int32_t* seq_lens, int b, int max_pages,
                                           unsigned* status) {
    int L = seq_lens[b];
    if (L < 0 || L > max_pages * kPage) {
        atomicOr(status, SLC_STATUS_BAD_LENGTH);
        L = L < 0 ? 0 : max_pages * kPage;
    }
    return L;
}

// Order-preserving uint32 key of a float score: a < b (as floats, -0 == +0)
// iff key(a) < key(b).  Never 0 for a score that is not NaN.
__device__ __forceinline__ uint32_t order_key(float f) {
    if (f == 0.f) f = 0.f;  // -0 and +0 tie
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-delta threshold ("Faster Than Flash: Fudan FFD Hits 11.6x Kernel
// Speedup, Pushes Long-Context Decoding to 256K", section "top-delta: Tearing
// Down "Global Synchronization" Too"): the order key of s_max - delta, s_max
// the score whose key is kmax, computed in fp32.  A candidate is within delta
// of the best iff its key is >= this one.
__device__ __forceinline__ uint32_t delta_threshold_key(uint32_t kmax, float delta) {
    const float smax = (kmax & 0x80000000u) ? __uint_as_float(kmax & 0x7fffffffu)
                                            : __uint_as_float(~kmax);
    return order_key(smax - delta);
}

// ---------------------------------------------------------------- E4M3
// 8-bit floats E4M3 (OCP "FN": sign, 4 exponent bits with bias 7, 3
// mantissa bits; exponent field 0 is subnormal, m/8 * 2^-6; no infinities;
// 0x7F / 0xFF are NaN; the largest finite value is 448).  Page bounds are
// rounded outward and a bound beyond the range keeps the NaN code of its
// sign, read back as the largest bf16 of that sign.

constexpr float kBf16Max = 3.38953139e38f;  // bf16 0x7F7F

// x rounded to E4M3: up -> the smallest value >= x, else the largest value
// <= x; beyond +-448 the NaN code of the rounding's side; zero (and a NaN
// key, conservatively out of range) as documented above.
__device__ __forceinline__ uint32_t e4m3_round(float x, bool up) {
    if (x != x) return up ? 0x7Fu : 0xFFu;
    if (x == 0.f) return 0u;
    const bool neg = x < 0.f;
    const float a = fabsf(x);
    const bool away = up != neg;  // round the magnitude away from zero?
    if (a > 448.f) return away ? (neg ? 0xFFu : 0x7Fu) : (neg ? 0xFEu : 0x7Eu);
    int e = (int)((__float_as_uint(a) >> 23) & 0xFF) - 127;  // floor(log2 a)
    if (e < -6) e = -6;  // below the normal range the grid step stays 2^-9
    // the magnitude in units of the grid step 2^(e-3): exact (power of two)
    const float q = ldexpf(a, 3 - e);
    int mi = (int)(away ? ceilf(q) : floorf(q));  // 0 .. 16
    if (mi == 0) return 0u;
    if (mi == 16) {  // carried into the next binade
        ++e;
        mi = 8;
    }
    const uint32_t E = mi < 8 ? 0u : (uint32_t)(e + 7);  // mi < 8 only for subnormals
    const uint32_t M = mi < 8 ? (uint32_t)mi : (uint32_t)(mi - 8);
    return (neg ? 0x80u : 0u) | (E << 3) | M;
}

// The value of an E4M3 code (NaN codes: +-kBf16Max).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    const uint32_t E = (c >> 3) & 15u, M = c & 7u;
    float v;
    if (E == 15u && M == 7u)
        v = kBf16Max;
    else if (E == 0u)
        v = ldexpf((float)M, -9);
    else
        v = ldexpf((float)(8u + M), (int)E - 10);
    return (c & 0x80u) ? -v : v;
}

// Two E4M3 codes (low byte first) -> two floats, the NaN codes read as
// `oor` (+-kBf16Max: the out-of-range bound of the row).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two, float oor) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((unsigned short)two));
    const __half2 hv = *reinterpret_cast<const __half2*>(&h);
    float2 f = __half22float2(hv);
    f.x = f.x == f.x ? f.x : oor;
    f.y = f.y == f.y ? f.y : oor;
    return f;
}

// ---------------------------------------------------------------- bf16
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------- warp
__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// Locate global index g among segments whose sizes are count(b) * hkv,
// b = 0..batch-1 (each sequence contributes hkv equal units).  Returns the
// unit u = b * hkv + h containing g and the unit's start offset.  Warp-wide:
// every lane must call it with the same g; count(b) must be warp-uniform
// per b.  If g is past the end, returns u = batch * hkv.
template <class CountFn>
__device__ __forceinline__ void locate_unit(long long g, int batch, int hkv, CountFn count,
                                            int* unit_out, long long* start_out) {
    const int lane = threadIdx.x & 31;
    long long base = 0;
    for (int b0 = 0; b0 < batch; b0 += 32) {
        int b = b0 + lane;
        int c = b < batch ? count(b) : 0;
        long long seg = (long long)c * hkv;
        // inclusive scan of seg (64-bit via two 32-bit halves is overkill:
        // segment sizes stay below 2^31 per chunk of 32 sequences)
        int s32 = warp_incl_scan((int)seg);
        long long incl = base + s32;
        unsigned hit = __ballot_sync(0xffffffffu, b < batch && incl > g);
        if (hit) {
            int l = __ffs(hit) - 1;
            long long excl = __shfl_sync(0xffffffffu, incl - seg, l);
            int cb = __shfl_sync(0xffffffffu, c, l);
            int h = (int)((g - excl) / cb);
            *unit_out = (b0 + l) * hkv + h;
            *start_out = excl + (long long)h * cb;
            return;
        }
        base += __shfl_sync(0xffffffffu, s32, 31);
    }
    *unit_out = batch * hkv;
    *start_out = base;
}

// Total of count(b) * hkv over all sequences (warp-wide).
template <class CountFn>
__device__ __forceinline__ long long total_units(int batch, int hkv, CountFn count) {
    const int lane = threadIdx.x & 31;
    long long tot = 0;
    for (int b0 = 0; b0 < batch; b0 += 32) {
        int b = b0 + lane;
        long long c = b < batch ? (long long)count(b) * hkv : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        tot += c;
    }
    return tot;
}

// ---------------------------------------------------------------- PTX
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: gives up after `limit` polls (each try_wait may suspend the
// thread for a hardware-defined interval) and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// 1-D bulk copy global -> shared (TMA engine), completion counted on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
        "[%3];" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// 4-byte asynchronous global -> shared copy (both 4-byte aligned).
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src)
                 : "memory");
}

// 16- or 8-byte asynchronous global -> shared copy (both aligned to its
// size); 16-byte copies bypass L1.
template <int B>
__device__ __forceinline__ void cp_async_chunk(void* dst, const void* src) {
    static_assert(B == 16 || B == 8, "16- or 8-byte copies");
    if (B == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
                     : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_addr(dst)), "l"(src)
                     : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's committed groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's completion
// (no-op without the launch attribute) / let the next grid start early.
__device__ __forceinline__ void grid_dep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Hint: bring `bytes` (a multiple of 16) at p (16-byte aligned) into L2.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint2 lds64(const void* p) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_addr(p)));
    return v;
}

__device__ __forceinline__ uint4 lds128(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_addr(p)));
    return v;
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = a * b + c on both lanes of a float pair (PTX fma.rn.f32x2).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// 2^x on the SFU (PTX ex2.approx.ftz.f32); ex2(-inf) = +0.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace slc
