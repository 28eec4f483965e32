// Internal launch interface between the C ABI (slc_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "slc_device.cuh"

namespace slc {

// An address range a launch reads once, front to back: its L2 lines are
// marked evict-first (an access-policy window with the streaming property),
// so that the stream does not push out what the next kernels reuse (their
// code, the workspace).  bytes = 0: none.
struct StreamingRange {
    const void* base = nullptr;
    size_t bytes = 0;
};

// Launch with programmatic stream serialization: the kernel may start while
// the preceding kernel in the stream is still running; it calls
// grid_dep_wait() before touching anything that kernel produces.
// cluster > 1 also sets the thread-block cluster size (x).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_streaming(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t stream, int cluster, StreamingRange range,
                                 Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[3];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int n = 1;
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    if (range.bytes > 0) {
        attr[n].id = cudaLaunchAttributeAccessPolicyWindow;
        attr[n].val.accessPolicyWindow.base_ptr = const_cast<void*>(range.base);
        attr[n].val.accessPolicyWindow.num_bytes = range.bytes;
        attr[n].val.accessPolicyWindow.hitRatio = 1.0f;
        attr[n].val.accessPolicyWindow.hitProp = cudaAccessPropertyStreaming;
        attr[n].val.accessPolicyWindow.missProp = cudaAccessPropertyStreaming;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, int cluster, Args&&... args) {
    return launch_pdl_streaming(kernel, grid, block, smem, stream, cluster, StreamingRange{},
                                std::forward<Args>(args)...);
}

// Upper bound on the number of attention CTAs (chunks) of one launch; sizes
// the split-partial workspace (slot = unit + chunk index).
constexpr int kMaxAttendChunks = 1024;

// Cluster sizes the finishing kernel may be launched with.
constexpr int kFinishClusters[] = {16, 12, 10, 9, 8, 7, 6, 5, 4};
constexpr int kNumFinishClusters = 9;

// Per-device launch settings, looked up once per device (with that device
// current) by slc_api.cu and passed to every launch.
struct DeviceCfg {
    int device;
    int num_sms;
    unsigned* status;  // the device status word
    int occ_score[2];       // score_kernel CTAs per SM (D = 128, 256)
    int occ_stream[2];      // stream_kernel CTAs per SM (D = 128, 256)
    int occ_attend[3];      // attend_kernel CTAs per SM (D = 128 sparse shape, D = 128 dense, D = 256)
    int finish_clusters[2][kNumFinishClusters];  // co-resident finish clusters (D, cluster size)
    size_t max_window;      // largest L2 access-policy window, bytes (0: none)
};

// The page metadata as a streaming range for the launches that scan it: the
// whole array, or its first max_window bytes.
inline StreamingRange metadata_range(const void* meta, long long num_pages, int hkv, int head_dim,
                                     int meta_format, const DeviceCfg& d) {
    StreamingRange r;
    if (meta == nullptr || d.max_window == 0) return r;
    const size_t elem = meta_format == SLC_META_FP8_E4M3 ? 1 : 2;
    const size_t bytes = (size_t)num_pages * hkv * 2 * head_dim * elem;
    r.base = meta;
    r.bytes = bytes < d.max_window ? bytes : d.max_window;
    return r;
}

cudaError_t setup_score(DeviceCfg& d);
cudaError_t setup_select(DeviceCfg& d);
cudaError_t setup_attend(DeviceCfg& d);
cudaError_t setup_stream(DeviceCfg& d);
cudaError_t setup_finish(DeviceCfg& d);

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
    int meta_format;  // SLC_META_*
};

struct BuildMetaParams {
    const void* k_cache;
    void* meta;
    const int32_t* block_table;
    const int32_t* seq_lens;
    unsigned* status;
    int batch, hkv, max_pages, num_pages;
    int meta_format;  // SLC_META_*
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
    // (rows by candidate only, nullable) the largest order key (see
    // order_key) of each 16-candidate tile: [units][cand_stride / 16]
    uint32_t* tile_max;
    int meta_format;  // SLC_META_*
};

struct SelectParams {
    const float* scores;  // as ScoreParams::scores (cand_stride)
    const int32_t* seq_lens;
    int32_t* selected;  // [B][Hkv][budget]
    unsigned* status;
    int batch, hkv, max_pages, prefix, window, budget;
    int cand_stride;
    // top-delta when topd >= 0: the topd best candidates plus every candidate
    // within delta of the best, at most budget; else the budget best
    int topd;
    float delta;
};

// Candidates per scoring tile, and the row stride of candidate-indexed
// scores (a multiple of 64 floats: 16-byte aligned rows and tiles).
constexpr int kSelTile = 16;
inline int cand_stride_of(int max_pages) { return (max_pages + 63) / 64 * 64; }

// Page list attended per unit (see slc_attend_impl.cuh).
enum : int { kListDense = 0, kListForced = 1 };

struct AttendParams {
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_table;
    const int32_t* seq_lens;
    float* part_acc;          // [slots][group][D]
    float2* part_ml;          // [slots][group]  (running max in log2 units, sum)
    float* out;               // [B][Hq][D]
    unsigned* status;
    int batch, hq, hkv, group, max_pages, num_pages;
    int list;  // kListDense or kListForced
    int prefix, window;
    float scale_log2;  // softmax scale * log2(e)
    int num_chunks;    // chunks of the attention launch (one per CTA)
};

// The streaming kernel: per unit, attention over the prefix and window pages
// (split partials, as attend_kernel with kListForced) and, unless
// score.scores is null, the scores of the candidate pages (as score_kernel,
// rows by candidate).
struct StreamParams {
    AttendParams at;
    ScoreParams sc;
};

// The finishing kernel: per unit, the selection (from the scores, or given),
// attention over the selected pages, and the merge of those partials with
// the streaming kernel's prefix/window partials into out.
struct FinishParams {
    AttendParams at;        // at.part_acc / at.part_ml: the streaming kernel's partials;
                            // at.num_chunks: the streaming kernel's grid
    int stream_scored;      // the streaming kernel scored (its grid split, forced_ctas)
    const float* scores;    // [units][cand_stride] by candidate, or null (selection given)
    const uint32_t* tile_max;  // [units][cand_stride / 16] tile maxima (order keys)
    const int32_t* given;   // [units][budget] given selection (scores == null)
    int32_t* selected;      // [units][budget] out: ascending, -1 padded (scores != null)
    int32_t* sel_phys;      // [units][budget] workspace: physical page of each selected entry
    int budget, cand_stride;
    // top-delta selection (topd >= 0): per unit the top max(topd, m) candidates,
    // m = #{s >= s_max - delta}, at most budget; topd < 0: the top budget
    int topd;
    float delta;
};

// Workspace carve-up shared by the API and the size query.
struct WorkspaceLayout {
    size_t scores, tile_max, selected, sel_phys, part_acc, part_ml, total;
};

// Split-partial slots of an attention launch: unit + chunk, chunks <=
// kMaxAttendChunks.
inline size_t partial_slots(size_t units) { return units + kMaxAttendChunks; }

cudaError_t launch_kv_append(const KvAppendParams& p, int head_dim, cudaStream_t stream);
cudaError_t launch_build_meta(const BuildMetaParams& p, int head_dim, const DeviceCfg& d,
                              cudaStream_t stream);
cudaError_t launch_score(const ScoreParams& p, int head_dim, const DeviceCfg& d,
                         cudaStream_t stream);
cudaError_t launch_select(const SelectParams& p, cudaStream_t stream);
// Dense attention over every page of every unit, then the merge of the split
// partials into out.
cudaError_t launch_dense(AttendParams p, int head_dim, const DeviceCfg& d, cudaStream_t stream);
// The streaming kernel; sets p.at.num_chunks to its grid size
// (stream_chunks) and p.at.list to kListForced.
cudaError_t launch_stream(StreamParams& p, int head_dim, const DeviceCfg& d, cudaStream_t stream);
int stream_chunks(int head_dim, const DeviceCfg& d);
// The finishing kernel (p.at.num_chunks: the streaming kernel's grid).
cudaError_t launch_finish(FinishParams p, int head_dim, const DeviceCfg& d, cudaStream_t stream);

}  // namespace slc
