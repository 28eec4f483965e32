// Fixed-budget page selection: per (sequence, kv head) keep the budget
// candidate pages with the highest scores, equal scores going to the lower
// page index, and emit them in ascending page order ("Accelerating
// Long-Context Decoding in Large-Scale Hybrid LLMs Without Retraining",
// abstract: a fixed budget of the most relevant tokens).
//
// One 1024-thread CTA per unit.  Scores become order-preserving uint32 keys
// held in registers (KPT consecutive candidates per thread).  A radix select
// over 8-bit digits, starting at the highest bit where the unit's smallest
// and largest keys differ (so equal leading bits cost no pass and the first
// histogram is spread), finds the threshold key T and how many keys equal to
// T to keep.  A block-wide scan then writes every key > T, and the lowest-
// indexed keys == T, in index order.
#include "slc_internal.h"

namespace slc {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
    if (f == 0.f) f = 0.f;  // -0 and +0 tie
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int KPT>
__global__ void __launch_bounds__(kThreads, 1) select_kernel(SelectParams p) {
    extern __shared__ uint32_t keys_smem[];  // [kThreads][KPT + 1]
    __shared__ int hist[256];
    __shared__ uint32_t red_min[kWarps], red_max[kWarps];
    __shared__ int scan[kWarps];
    __shared__ int sh_digit, sh_above;

    const int u = blockIdx.x;
    const int b = u / p.hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = checked_len(p.seq_lens, b, p.max_pages, p.status);
    const PageRanges r = page_ranges(L, p.prefix, p.window);
    const int ncand = r.ws - r.np;
    const int nsel = min(p.budget, ncand);
    int32_t* out = p.selected + (long long)u * p.budget;

    if (nsel >= ncand) {  // every candidate is kept (also covers ncand == 0)
        for (int i = tid; i < p.budget; i += kThreads) out[i] = i < ncand ? r.np + i : -1;
        return;
    }
    if (nsel <= 0) {
        for (int i = tid; i < p.budget; i += kThreads) out[i] = -1;
        return;
    }

    // coalesced load, transposed through padded shared memory
    const float* s = p.scores + (long long)u * p.max_pages + r.np;
    {
        float v[KPT];  // all loads in flight before the first store
#pragma unroll
        for (int k = 0; k < KPT; ++k) {
            const int i = tid + k * kThreads;
            v[k] = i < ncand ? __ldg(s + i) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < KPT; ++k) {
            const int i = tid + k * kThreads;
            keys_smem[(i / KPT) * (KPT + 1) + (i % KPT)] = i < ncand ? order_key(v[k]) : 0u;
        }
    }
    __syncthreads();
    uint32_t key[KPT];
#pragma unroll
    for (int k = 0; k < KPT; ++k) key[k] = keys_smem[tid * (KPT + 1) + k];
    const int nown = max(0, min(KPT, ncand - tid * KPT));

    // key range of the unit
    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int k = 0; k < KPT; ++k)
        if (k < nown) {
            kmin = min(kmin, key[k]);
            kmax = max(kmax, key[k]);
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) {
        red_min[warp] = kmin;
        red_max[warp] = kmax;
    }
    __syncthreads();
    kmin = red_min[lane];
    kmax = red_max[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }

    // radix select of the nsel-th largest key
    uint32_t prefix = kmin, mask = 0xffffffffu;
    int remaining = nsel;  // keys still to take at or below the current prefix
    if (kmin != kmax) {
        int hb = 31 - __clz(kmin ^ kmax);  // highest differing bit
        mask = hb == 31 ? 0u : ~((2u << hb) - 1u);
        prefix = kmin & mask;
        while (true) {
            const int shift = max(hb - 7, 0);
            const int nbits = hb - shift + 1;
            const uint32_t dmask = (1u << nbits) - 1u;
            for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
            __syncthreads();
#pragma unroll
            for (int k = 0; k < KPT; ++k)
                if (k < nown && (key[k] & mask) == prefix)
                    atomicAdd(&hist[(key[k] >> shift) & dmask], 1);
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
                const int above = suf - local;  // keys in bins >= 8*(lane+1)
                if (above < remaining && suf >= remaining) {
                    int cum = above;
#pragma unroll
                    for (int i = 7; i >= 0; --i) {
                        if (cum + c[i] >= remaining) {
                            sh_digit = lane * 8 + i;
                            sh_above = cum;
                            break;
                        }
                        cum += c[i];
                    }
                }
            }
            __syncthreads();
            const uint32_t digit = (uint32_t)sh_digit;
            remaining -= sh_above;
            prefix |= digit << shift;
            mask |= dmask << shift;
            if (shift == 0) break;
            hb = shift - 1;
            __syncthreads();  // hist is cleared again next pass
        }
    }
    const uint32_t T = prefix;
    const int ties = remaining;  // keys == T to keep, lowest index first

    // index-ordered compaction: exclusive scan of packed (gt, eq) counts
    int ngt = 0, neq = 0;
#pragma unroll
    for (int k = 0; k < KPT; ++k)
        if (k < nown) {
            ngt += key[k] > T;
            neq += key[k] == T;
        }
    const int packed = (ngt << 16) | neq;
    const int incl = warp_incl_scan(packed);
    if (lane == 31) scan[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = scan[lane];
        const int wi = warp_incl_scan(v);
        scan[lane] = wi - v;
    }
    __syncthreads();
    const int excl = scan[warp] + incl - packed;
    int gt_before = excl >> 16, eq_before = excl & 0xffff;
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
        if (k < nown) {
            const int page = r.np + tid * KPT + k;
            if (key[k] > T) {
                out[gt_before + min(eq_before, ties)] = page;
                ++gt_before;
            } else if (key[k] == T) {
                if (eq_before < ties) out[gt_before + eq_before] = page;
                ++eq_before;
            }
        }
    }
    for (int i = nsel + tid; i < p.budget; i += kThreads) out[i] = -1;
}

template <int KPT>
cudaError_t launch_kpt(const SelectParams& p, cudaStream_t stream) {
    const int smem = kThreads * (KPT + 1) * (int)sizeof(uint32_t);
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel<KPT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    select_kernel<KPT><<<p.batch * p.hkv, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
    if (p.batch * p.hkv == 0) return cudaSuccess;
    const int cap = p.max_pages;  // candidates never exceed the page count
    if (cap <= kThreads * 4) return launch_kpt<4>(p, stream);
    if (cap <= kThreads * 8) return launch_kpt<8>(p, stream);
    if (cap <= kThreads * 16) return launch_kpt<16>(p, stream);
    return launch_kpt<32>(p, stream);
}

}  // namespace slc
