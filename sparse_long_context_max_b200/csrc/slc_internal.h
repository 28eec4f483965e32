// Internal launch interface between the C ABI (slc_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "slc_device.cuh"

namespace slc {

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
    float* scores;  // [B][Hkv][max_pages]
    unsigned* status;
    int batch, hq, hkv, group, max_pages, num_pages, prefix, window;
};

struct SelectParams {
    const float* scores;
    const int32_t* seq_lens;
    int32_t* selected;  // [B][Hkv][budget]
    unsigned* status;
    int batch, hkv, max_pages, prefix, window, budget;
};

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
    int sparse, prefix, window, budget;
    float scale_log2;  // softmax scale * log2(e)
    int num_chunks;    // chunks of the attention launch (one per CTA)
};

// Workspace carve-up shared by the API and the size query.
struct WorkspaceLayout {
    size_t scores, selected, part_acc, part_ml, total;
};
WorkspaceLayout workspace_layout(int batch, int hq, int hkv, int head_dim, int max_pages,
                                 int budget);

cudaError_t launch_kv_append(const KvAppendParams& p, int head_dim, cudaStream_t stream);
cudaError_t launch_build_meta(const BuildMetaParams& p, int head_dim, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_score(const ScoreParams& p, int head_dim, int num_sms, cudaStream_t stream);
cudaError_t launch_select(const SelectParams& p, cudaStream_t stream);
// Attention over the list of each unit (dense: all pages; sparse: prefix,
// selected, window), then the merge of the per-warp partials into out.
cudaError_t launch_attend(AttendParams p, int head_dim, int num_sms, cudaStream_t stream,
                          int* kernels_launched);

}  // namespace slc
