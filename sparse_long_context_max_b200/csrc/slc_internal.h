// Internal launch interface between the C ABI (slc_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "slc_device.cuh"

namespace slc {

// Launch with programmatic stream serialization: the kernel may start while
// the preceding kernel in the stream is still running; it calls
// grid_dep_wait() before touching anything that kernel produces.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Upper bound on the number of attention CTAs (chunks) of one launch; sizes
// the split-partial workspace (slot = unit + chunk index).
constexpr int kMaxAttendChunks = 1024;

struct KvAppendParams {
    const void* k_new;
    const void* v_new;
    void* k_cache;
    void* v_cache;
    void* meta;
    const int32_t* block_table;
    const int32_t* positions;
    unsigned* status;
    int batch, hkv, max_pages, num_pages;
};

struct BuildMetaParams {
    const void* k_cache;
    void* meta;
    const int32_t* block_table;
    const int32_t* seq_lens;
    unsigned* status;
    int batch, hkv, max_pages, num_pages;
};

struct ScoreParams {
    const void* q;
    const void* meta;
    const int32_t* block_table;
    const int32_t* seq_lens;
    float* scores;  // [B][Hkv][max_pages] by page, or by candidate (cand_stride)
    unsigned* status;
    int batch, hq, hkv, group, max_pages, num_pages, prefix, window;
    int cand_stride;  // 0: scores indexed by page; else rows of cand_stride by candidate
};

struct SelectParams {
    const float* scores;  // as ScoreParams::scores (cand_stride)
    const int32_t* seq_lens;
    int32_t* selected;  // [B][Hkv][budget]
    unsigned* status;
    int batch, hkv, max_pages, prefix, window, budget;
    int cand_stride;
};

// Candidates per scoring tile, and the row stride of candidate-indexed
// scores (a multiple of 64 floats: 16-byte aligned rows and tiles).
constexpr int kSelTile = 16;
inline int cand_stride_of(int max_pages) { return (max_pages + 63) / 64 * 64; }

// Page list attended per unit (see slc_attend_impl.cuh).
enum : int { kListDense = 0, kListSparse = 1, kListForced = 2, kListSelected = 3 };

struct AttendParams {
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const int32_t* selected;  // sparse only: [B][Hkv][budget]
    float* part_acc;          // [slots][group][D]
    float2* part_ml;          // [slots][group]  (running max in log2 units, sum)
    float* out;               // [B][Hq][D]
    unsigned* status;
    int batch, hq, hkv, group, max_pages, num_pages;
    int list;  // kListDense, kListSparse, kListForced or kListSelected
    int prefix, window, budget;
    float scale_log2;  // softmax scale * log2(e)
    int num_chunks;    // chunks of the attention launch (one per CTA)
    long long slot_base;  // this launch's partials: slot slot_base + unit + chunk
};

// Workspace carve-up shared by the API and the size query.
struct WorkspaceLayout {
    size_t scores, selected, part_acc, part_ml, total;
};

// Sparse decode step (slc_fused.cu): scoring with the prefix/window
// attention in one grid, selection, selected-page attention, merge.
struct FusedParams {
    ScoreParams sc;
    SelectParams se;
    AttendParams at;  // list is set per kernel
    int forced_chunks;  // target chunk count of the prefix/window attention
    long long premerged_base;  // >= 0: unit u's forced partials merged into this + u
};
// Merge of every unit's forced-list partials into one slot per unit, done
// by extra CTAs of the selection kernel.
struct PremergeParams {
    AttendParams at;    // the forced lists
    int forced_chunks;  // as FusedParams::forced_chunks
    long long dst_base;
    int v4;  // head_dim / 4
};
// Split-partial slots of the sparse decode: two attention launches of at
// most units + kMaxAttendChunks slots each, then one merged slot per unit.
inline size_t fused_slots(size_t units) { return 2 * (units + kMaxAttendChunks) + units; }
WorkspaceLayout workspace_layout(int batch, int hq, int hkv, int head_dim, int max_pages,
                                 int budget);

cudaError_t launch_kv_append(const KvAppendParams& p, int head_dim, cudaStream_t stream);
cudaError_t launch_build_meta(const BuildMetaParams& p, int head_dim, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_score(const ScoreParams& p, int head_dim, int num_sms, cudaStream_t stream);
// The selection; with pm, extra CTAs also merge each unit's forced-list
// partials (they run beside the selection CTAs).
cudaError_t launch_select(const SelectParams& p, cudaStream_t stream,
                          const PremergeParams* pm = nullptr);
// sparse_decode's path: four kernels chained by programmatic dependent
// launch (score + forced attention, select, selected attention, merge).
cudaError_t launch_sparse_fused(const FusedParams& p, int head_dim, int num_sms,
                                cudaStream_t stream, int stage = 0);
// Attention over the list of each unit (dense: all pages; sparse: prefix,
// selected, window), then the merge of the per-warp partials into out.
cudaError_t launch_attend(AttendParams p, int head_dim, int num_sms, cudaStream_t stream,
                          int* kernels_launched);
// The attention alone: partials in slots p.slot_base + unit + chunk; sets
// p.num_chunks (at most kMaxAttendChunks).
cudaError_t launch_attend_partials(AttendParams& p, int head_dim, int num_sms,
                                   cudaStream_t stream);
// The chunk count launch_attend_partials uses.
int attend_chunks(int head_dim, int num_sms);

}  // namespace slc
