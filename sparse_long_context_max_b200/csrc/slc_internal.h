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
enum : int { kListDense = 0, kListSparse = 1 };

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
    int list;  // kListDense or kListSparse
    int prefix, window, budget;
    float scale_log2;  // softmax scale * log2(e)
    int num_chunks;    // chunks of the attention launch (one per CTA)
    int wait_first;    // the preceding kernel writes the selection: L2-prefetch the forced pages first
};

// Workspace carve-up shared by the API and the size query.
struct WorkspaceLayout {
    size_t scores, selected, part_acc, part_ml, total;
};

// Split-partial slots of an attention launch: unit + chunk, chunks <=
// kMaxAttendChunks.
inline size_t partial_slots(size_t units) { return units + kMaxAttendChunks; }

cudaError_t launch_kv_append(const KvAppendParams& p, int head_dim, cudaStream_t stream);
cudaError_t launch_build_meta(const BuildMetaParams& p, int head_dim, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_score(const ScoreParams& p, int head_dim, int num_sms, cudaStream_t stream);
cudaError_t launch_select(const SelectParams& p, cudaStream_t stream);
// Attention over the list of each unit (dense: all pages; sparse: prefix,
// window, selected), then the merge of the split partials into out.  what:
// kAttendAndMerge, or one of the two kernels alone (for stage timing).
enum : int { kAttendAndMerge = 0, kAttendOnly = 1, kMergeOnly = 2 };
cudaError_t launch_attend(AttendParams p, int head_dim, int num_sms, cudaStream_t stream,
                          int what = kAttendAndMerge);

}  // namespace slc
