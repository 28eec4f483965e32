// C ABI of libslc (declared in include/slc.h): argument validation,
// workspace carving and kernel launches.  Validation happens before any
// CUDA call, so argument errors launch nothing and need no GPU.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "slc_internal.h"

// The device status word (SLC_STATUS_* bits), one per GPU that loads the
// library; kernels receive its address.
__device__ unsigned slc_status_word;

namespace slc {

namespace {

constexpr int kMaxDevices = 64;

struct DeviceSlot {
    bool ready;
    DeviceCfg cfg;
};

DeviceSlot g_devices[kMaxDevices];
std::mutex g_mutex;
thread_local char g_cuda_error[256];

int note_cuda(cudaError_t e, const char* where = "") {
    snprintf(g_cuda_error, sizeof g_cuda_error, "%s%s%s: %s", where, *where ? ": " : "",
             cudaGetErrorName(e), cudaGetErrorString(e));
    return SLC_ERR_CUDA;
}

// Per-device facts and launch settings (shared-memory limits, occupancies,
// co-resident clusters), set up once per device on the first call made with
// that device current.
int device_cfg(const DeviceCfg** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return note_cuda(e);
    if (dev < 0 || dev >= kMaxDevices) return SLC_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceSlot& d = g_devices[dev];
    if (!d.ready) {
        DeviceCfg c{};
        c.device = dev;
        e = cudaDeviceGetAttribute(&c.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return note_cuda(e);
        e = cudaGetSymbolAddress(reinterpret_cast<void**>(&c.status), slc_status_word);
        if (e != cudaSuccess) return note_cuda(e);
        int win = 0;  // no access-policy windows where the attribute is not there
        if (cudaDeviceGetAttribute(&win, cudaDevAttrMaxAccessPolicyWindowSize, dev) != cudaSuccess) {
            (void)cudaGetLastError();
            win = 0;
        }
        c.max_window = win > 0 ? (size_t)win : 0;
        if ((e = setup_score(c)) != cudaSuccess) return note_cuda(e, "setup score");
        if ((e = setup_select(c)) != cudaSuccess) return note_cuda(e, "setup select");
        if ((e = setup_attend(c)) != cudaSuccess) return note_cuda(e, "setup attend");
        if ((e = setup_stream(c)) != cudaSuccess) return note_cuda(e, "setup stream");
        if ((e = setup_finish(c)) != cudaSuccess) return note_cuda(e, "setup finish");
        d.cfg = c;
        d.ready = true;
    }
    *out = &d.cfg;
    return SLC_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int check_cache(const slc_cache_t* c) {
    if (!c) return SLC_ERR_INVALID_ARG;
    if (c->page_size != kPage) return SLC_ERR_UNSUPPORTED;
    if (c->head_dim != 128 && c->head_dim != 256) return SLC_ERR_UNSUPPORTED;
    if (c->num_kv_heads <= 0 || c->num_pages <= 0) return SLC_ERR_INVALID_ARG;
    if (c->meta_format != SLC_META_BF16 && c->meta_format != SLC_META_FP8_E4M3)
        return SLC_ERR_UNSUPPORTED;
    if (!c->k_cache || !c->v_cache || !c->meta) return SLC_ERR_INVALID_ARG;
    if (!aligned16(c->k_cache) || !aligned16(c->v_cache) || !aligned16(c->meta))
        return SLC_ERR_INVALID_ARG;
    return SLC_OK;
}

int check_heads(const slc_cache_t* c, int hq) {
    if (hq <= 0 || hq % c->num_kv_heads != 0) return SLC_ERR_INVALID_ARG;
    const int g = hq / c->num_kv_heads;
    if (g > kMaxGroup) return SLC_ERR_UNSUPPORTED;
    return SLC_OK;
}

}  // namespace

WorkspaceLayout workspace_layout(int batch, int hq, int hkv, int head_dim, int max_pages,
                                 int budget) {
    WorkspaceLayout w{};
    const size_t units = (size_t)batch * hkv;
    const size_t group = (size_t)(hq / hkv);
    const size_t slots = partial_slots(units);
    size_t off = 0;
    w.scores = off;  // by candidate, in rows of cand_stride_of(max_pages)
    off = round_up(off + units * (size_t)cand_stride_of(max_pages) * sizeof(float), 256);
    w.tile_max = off;  // one key per 16 candidates
    off = round_up(off + units * (size_t)(cand_stride_of(max_pages) / kSelTile) * 4, 256);
    w.selected = off;
    off = round_up(off + units * (size_t)(budget > 0 ? budget : 1) * sizeof(int32_t), 256);
    w.sel_phys = off;
    off = round_up(off + units * (size_t)(budget > 0 ? budget : 1) * sizeof(int32_t), 256);
    w.part_acc = off;
    off = round_up(off + slots * group * head_dim * sizeof(float), 256);
    w.part_ml = off;
    off = round_up(off + slots * group * sizeof(float2), 256);
    w.total = off;
    return w;
}

}  // namespace slc

using namespace slc;

extern "C" {

const char* slc_error_string(int code) {
    switch (code) {
        case SLC_OK: return "ok";
        case SLC_ERR_INVALID_ARG: return "invalid argument";
        case SLC_ERR_UNSUPPORTED: return "unsupported shape";
        case SLC_ERR_WORKSPACE: return "workspace too small";
        case SLC_ERR_CUDA: return "CUDA error";
        case SLC_ERR_DEVICE: return "device status fault";
        default: return "unknown error";
    }
}

const char* slc_last_cuda_error(void) { return g_cuda_error; }

size_t slc_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                          int32_t head_dim, int32_t max_pages_per_seq, int32_t budget) {
    if (batch < 0 || num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % num_kv_heads ||
        num_q_heads / num_kv_heads > kMaxGroup || (head_dim != 128 && head_dim != 256) ||
        max_pages_per_seq <= 0 || budget < 0)
        return 0;
    return workspace_layout(batch, num_q_heads, num_kv_heads, head_dim, max_pages_per_seq,
                            budget)
        .total;
}

int slc_kv_append(const slc_cache_t* cache, const void* k_new, const void* v_new,
                  const int32_t* block_table, int32_t max_pages_per_seq,
                  const int32_t* positions, int32_t batch, slc_stream_t stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (batch < 0 || max_pages_per_seq <= 0) return SLC_ERR_INVALID_ARG;
    if (batch == 0) return SLC_OK;
    if (!k_new || !v_new || !block_table || !positions) return SLC_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new)) return SLC_ERR_INVALID_ARG;
    const DeviceCfg* dev;
    if ((rc = device_cfg(&dev))) return rc;
    KvAppendParams p{k_new,     v_new,     cache->k_cache,          cache->v_cache,
                     cache->meta, block_table, positions,            dev->status,
                     batch,     cache->num_kv_heads, max_pages_per_seq, cache->num_pages,
                     cache->meta_format};
    cudaError_t e = launch_kv_append(p, cache->head_dim, stream);
    return e == cudaSuccess ? SLC_OK : note_cuda(e);
}

int slc_build_page_meta(const slc_cache_t* cache, const int32_t* block_table,
                        int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                        slc_stream_t stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (batch < 0 || max_pages_per_seq <= 0) return SLC_ERR_INVALID_ARG;
    if (batch == 0) return SLC_OK;
    if (!block_table || !seq_lens) return SLC_ERR_INVALID_ARG;
    const DeviceCfg* dev;
    if ((rc = device_cfg(&dev))) return rc;
    BuildMetaParams p{cache->k_cache, cache->meta, block_table, seq_lens, dev->status, batch,
                      cache->num_kv_heads, max_pages_per_seq, cache->num_pages,
                      cache->meta_format};
    cudaError_t e = launch_build_meta(p, cache->head_dim, *dev, stream);
    return e == cudaSuccess ? SLC_OK : note_cuda(e);
}

int slc_score_pages(const void* q, const slc_cache_t* cache, const int32_t* block_table,
                    int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                    int32_t num_q_heads, int32_t prefix, int32_t window, float* scores,
                    slc_stream_t stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if ((rc = check_heads(cache, num_q_heads))) return rc;
    if (batch < 0 || max_pages_per_seq <= 0 || prefix < 0 || window < 0)
        return SLC_ERR_INVALID_ARG;
    if (batch == 0) return SLC_OK;
    if (!q || !block_table || !seq_lens || !scores || !aligned16(q)) return SLC_ERR_INVALID_ARG;
    const DeviceCfg* dev;
    if ((rc = device_cfg(&dev))) return rc;
    ScoreParams p{q,           cache->meta, block_table, seq_lens,
                  scores,      dev->status, batch,
                  num_q_heads, cache->num_kv_heads, num_q_heads / cache->num_kv_heads,
                  max_pages_per_seq, cache->num_pages, prefix, window, 0, nullptr,
                  cache->meta_format};
    cudaError_t e = launch_score(p, cache->head_dim, *dev, stream);
    return e == cudaSuccess ? SLC_OK : note_cuda(e);
}

int slc_select_pages(const float* scores, int32_t num_kv_heads, int32_t max_pages_per_seq,
                     const int32_t* seq_lens, int32_t batch, int32_t prefix, int32_t window,
                     int32_t budget, int32_t* selected, slc_stream_t stream) {
    if (batch < 0 || num_kv_heads <= 0 || max_pages_per_seq <= 0 || prefix < 0 ||
        window < 0 || budget < 0)
        return SLC_ERR_INVALID_ARG;
    if (max_pages_per_seq > kMaxCandidates) return SLC_ERR_UNSUPPORTED;
    if (batch == 0 || budget == 0) return SLC_OK;
    if (!scores || !seq_lens || !selected) return SLC_ERR_INVALID_ARG;
    const DeviceCfg* dev;
    int rc;
    if ((rc = device_cfg(&dev))) return rc;
    SelectParams p{scores, seq_lens, selected, dev->status, batch, num_kv_heads,
                   max_pages_per_seq, prefix, window, budget, 0, -1, 0.f};
    cudaError_t e = launch_select(p, stream);
    return e == cudaSuccess ? SLC_OK : note_cuda(e);
}

int slc_select_pages_delta(const float* scores, int32_t num_kv_heads, int32_t max_pages_per_seq,
                           const int32_t* seq_lens, int32_t batch, int32_t prefix,
                           int32_t window, int32_t d, float delta, int32_t cap,
                           int32_t* selected, slc_stream_t stream) {
    if (batch < 0 || num_kv_heads <= 0 || max_pages_per_seq <= 0 || prefix < 0 ||
        window < 0 || d < 0 || cap < 0 || delta != delta)
        return SLC_ERR_INVALID_ARG;
    if (max_pages_per_seq > kMaxCandidates) return SLC_ERR_UNSUPPORTED;
    if (batch == 0 || cap == 0) return SLC_OK;
    if (!scores || !seq_lens || !selected) return SLC_ERR_INVALID_ARG;
    const DeviceCfg* dev;
    int rc;
    if ((rc = device_cfg(&dev))) return rc;
    SelectParams p{scores, seq_lens, selected, dev->status, batch, num_kv_heads,
                   max_pages_per_seq, prefix, window, cap, 0, d, delta};
    cudaError_t e = launch_select(p, stream);
    return e == cudaSuccess ? SLC_OK : note_cuda(e);
}

// mode: 0 dense, 1 sparse (stream: prefix/window attention + scores;
// finish: select, attend the selection, merge), 2 sparse attention over the
// caller's selection in `selected_out`.  stage (mode 1): 0 both kernels, 1
// the streaming kernel alone, 2 the finishing kernel alone.
// Argument checks of decode() apart from the workspace (which the caller
// checks), in the order the codes are documented; nothing touches the GPU.
// *nothing_to_do is set for an empty batch.
static int check_decode(int mode, const void* q, const slc_cache_t* cache,
                        const int32_t* block_table, int32_t max_pages_per_seq,
                        const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                        int32_t prefix, int32_t window, int32_t budget, float scale,
                        const float* out, const int32_t* selected_out, bool* nothing_to_do) {
    *nothing_to_do = false;
    int rc = check_cache(cache);
    if (rc) return rc;
    if ((rc = check_heads(cache, num_q_heads))) return rc;
    if (batch < 0 || max_pages_per_seq <= 0 || prefix < 0 || window < 0 || budget < 0)
        return SLC_ERR_INVALID_ARG;
    if (mode != 0 && max_pages_per_seq > kMaxCandidates) return SLC_ERR_UNSUPPORTED;
    if (!(scale == scale) || isinf(scale)) return SLC_ERR_INVALID_ARG;
    if (batch == 0) {
        *nothing_to_do = true;
        return SLC_OK;
    }
    if (!q || !block_table || !seq_lens || !out) return SLC_ERR_INVALID_ARG;
    if (mode == 2 && budget > 0 && !selected_out) return SLC_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out)) return SLC_ERR_INVALID_ARG;
    return SLC_OK;
}

static int decode(int mode, const void* q, const slc_cache_t* cache,
                  const int32_t* block_table, int32_t max_pages_per_seq,
                  const int32_t* seq_lens, int32_t batch, int32_t num_q_heads, int32_t prefix,
                  int32_t window, int32_t budget, float scale, float* out,
                  int32_t* selected_out, void* workspace, size_t workspace_bytes,
                  cudaStream_t stream, int stage = 0, int topd = -1, float delta = 0.f) {
    const bool sparse = mode != 0;
    bool empty;
    int rc = check_decode(mode, q, cache, block_table, max_pages_per_seq, seq_lens, batch,
                          num_q_heads, prefix, window, budget, scale, out, selected_out, &empty);
    if (rc || empty) return rc;
    if (!workspace || !aligned16(workspace)) return SLC_ERR_INVALID_ARG;
    const int hkv = cache->num_kv_heads, D = cache->head_dim;
    const WorkspaceLayout w =
        workspace_layout(batch, num_q_heads, hkv, D, max_pages_per_seq, sparse ? budget : 0);
    if (workspace_bytes < w.total) return SLC_ERR_WORKSPACE;
    const DeviceCfg* dev;
    if ((rc = device_cfg(&dev))) return rc;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (scale <= 0.f) scale = 1.f / sqrtf((float)D);
    AttendParams ap{};
    ap.q = q;
    ap.k_cache = cache->k_cache;
    ap.v_cache = cache->v_cache;
    ap.block_table = block_table;
    ap.seq_lens = seq_lens;
    ap.part_acc = reinterpret_cast<float*>(ws + w.part_acc);
    ap.part_ml = reinterpret_cast<float2*>(ws + w.part_ml);
    ap.out = out;
    ap.status = dev->status;
    ap.batch = batch;
    ap.hq = num_q_heads;
    ap.hkv = hkv;
    ap.group = num_q_heads / hkv;
    ap.max_pages = max_pages_per_seq;
    ap.num_pages = cache->num_pages;
    ap.prefix = sparse ? prefix : 0;
    ap.window = sparse ? window : 0;
    ap.scale_log2 = scale * 1.4426950408889634f;
    cudaError_t e;
    if (!sparse) {
        e = launch_dense(ap, D, *dev, stream);
        return e == cudaSuccess ? SLC_OK : note_cuda(e, "dense");
    }
    const bool scoring = mode == 1 && budget > 0;
    const int cs = cand_stride_of(max_pages_per_seq);
    float* scores = reinterpret_cast<float*>(ws + w.scores);
    StreamParams sp{};
    sp.at = ap;
    uint32_t* tile_max = reinterpret_cast<uint32_t*>(ws + w.tile_max);
    sp.sc = ScoreParams{q,           cache->meta, block_table, seq_lens,
                        scoring ? scores : nullptr, dev->status, batch,
                        num_q_heads, hkv,         num_q_heads / hkv, max_pages_per_seq,
                        cache->num_pages, prefix, window, cs, tile_max, cache->meta_format};
    if (stage == 0 || stage == 1) {
        e = launch_stream(sp, D, *dev, stream);
        if (e != cudaSuccess) return note_cuda(e, "stream");
        if (stage == 1) return SLC_OK;
    } else {
        // the finishing kernel alone: the streaming kernel's chunk count
        sp.at.num_chunks = stream_chunks(D, *dev);
        sp.at.list = kListForced;
    }
    FinishParams fp{};
    fp.at = sp.at;
    fp.scores = mode == 1 ? scores : nullptr;
    fp.tile_max = tile_max;
    fp.given = mode == 2 ? selected_out : nullptr;
    fp.selected = mode == 1
                      ? (selected_out ? selected_out : reinterpret_cast<int32_t*>(ws + w.selected))
                      : nullptr;
    fp.sel_phys = reinterpret_cast<int32_t*>(ws + w.sel_phys);
    fp.budget = budget;
    fp.cand_stride = cs;
    fp.stream_scored = scoring ? 1 : 0;
    fp.topd = mode == 1 ? topd : -1;
    fp.delta = delta;
    e = launch_finish(fp, D, *dev, stream);
    return e == cudaSuccess ? SLC_OK : note_cuda(e, "finish");
}

int slc_sparse_decode(const void* q, const slc_cache_t* cache, const int32_t* block_table,
                      int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                      int32_t num_q_heads, int32_t prefix, int32_t window, int32_t budget,
                      float scale, float* out, int32_t* selected_out, void* workspace,
                      size_t workspace_bytes, slc_stream_t stream) {
    return decode(1, q, cache, block_table, max_pages_per_seq, seq_lens, batch, num_q_heads,
                  prefix, window, budget, scale, out, selected_out, workspace, workspace_bytes,
                  stream);
}

int slc_sparse_decode_stage(int32_t stage, const void* q, const slc_cache_t* cache,
                            const int32_t* block_table, int32_t max_pages_per_seq,
                            const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                            int32_t prefix, int32_t window, int32_t budget, float scale,
                            float* out, int32_t* selected_out, void* workspace,
                            size_t workspace_bytes, slc_stream_t stream) {
    if (stage < 1 || stage > 2) return SLC_ERR_INVALID_ARG;
    return decode(1, q, cache, block_table, max_pages_per_seq, seq_lens, batch, num_q_heads,
                  prefix, window, budget, scale, out, selected_out, workspace, workspace_bytes,
                  stream, stage);
}

int slc_sparse_attend(const void* q, const slc_cache_t* cache, const int32_t* block_table,
                      int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                      int32_t num_q_heads, int32_t prefix, int32_t window, int32_t budget,
                      const int32_t* selected, float scale, float* out, void* workspace,
                      size_t workspace_bytes, slc_stream_t stream) {
    return decode(2, q, cache, block_table, max_pages_per_seq, seq_lens, batch, num_q_heads,
                  prefix, window, budget, scale, out, const_cast<int32_t*>(selected), workspace,
                  workspace_bytes, stream);
}

int slc_sparse_decode_delta(const void* q, const slc_cache_t* cache, const int32_t* block_table,
                            int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                            int32_t num_q_heads, int32_t prefix, int32_t window, int32_t d,
                            float delta, int32_t cap, float scale, float* out,
                            int32_t* selected_out, void* workspace, size_t workspace_bytes,
                            slc_stream_t stream) {
    bool empty;
    int rc = check_decode(1, q, cache, block_table, max_pages_per_seq, seq_lens, batch,
                          num_q_heads, prefix, window, cap, scale, out, selected_out, &empty);
    if (rc) return rc;
    if (d < 0 || delta != delta) return SLC_ERR_INVALID_ARG;
    if (empty) return SLC_OK;
    // the two kernels of slc_sparse_decode; the finishing kernel sets each
    // unit's selection size from its scores
    return decode(1, q, cache, block_table, max_pages_per_seq, seq_lens, batch, num_q_heads,
                  prefix, window, cap, scale, out, selected_out, workspace, workspace_bytes,
                  stream, 0, d, delta);
}

int slc_dense_decode(const void* q, const slc_cache_t* cache, const int32_t* block_table,
                     int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                     int32_t num_q_heads, float scale, float* out, void* workspace,
                     size_t workspace_bytes, slc_stream_t stream) {
    return decode(0, q, cache, block_table, max_pages_per_seq, seq_lens, batch,
                  num_q_heads, 0, 0, 0, scale, out, nullptr, workspace, workspace_bytes,
                  stream);
}

// ----------------------------------------------------------------------
// Decode without any allocation: the workspace is a fixed device array.
// Host code must not pass `slc_static_scratch` itself to a kernel (in host
// code it names a host-side stand-in); its device address is looked up per
// device below.
static __device__ __align__(256) unsigned char slc_static_scratch[SLC_STATIC_SCRATCH_BYTES];

static void* g_static_scratch[slc::kMaxDevices];
static std::mutex g_static_mutex;

// Device address of the scratch array on the current device (looked up
// once per device, with that device current).
static int static_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return note_cuda(e, "static scratch");
    if (dev < 0 || dev >= slc::kMaxDevices) return SLC_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_static_mutex);
    if (!g_static_scratch[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, slc_static_scratch);
        if (e != cudaSuccess) return note_cuda(e, "static scratch");
        g_static_scratch[dev] = ptr;
    }
    *out = g_static_scratch[dev];
    return SLC_OK;
}

int slc_sparse_decode_static(const void* q, const slc_cache_t* cache, const int32_t* block_table,
                             int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                             int32_t num_q_heads, int32_t prefix, int32_t window, int32_t budget,
                             float scale, float* out, int32_t* selected_out,
                             slc_stream_t stream) {
    bool empty;
    int rc = check_decode(1, q, cache, block_table, max_pages_per_seq, seq_lens, batch,
                          num_q_heads, prefix, window, budget, scale, out, selected_out, &empty);
    if (rc || empty) return rc;
    const size_t need = workspace_layout(batch, num_q_heads, cache->num_kv_heads,
                                         cache->head_dim, max_pages_per_seq, budget)
                            .total;
    if (need > SLC_STATIC_SCRATCH_BYTES) return SLC_ERR_WORKSPACE;
    void* scratch = nullptr;
    if ((rc = static_scratch(&scratch))) return rc;
    return slc_sparse_decode(q, cache, block_table, max_pages_per_seq, seq_lens, batch,
                             num_q_heads, prefix, window, budget, scale, out, selected_out,
                             scratch, SLC_STATIC_SCRATCH_BYTES, stream);
}

int slc_device_status(int32_t* status, slc_stream_t stream) {
    if (!status) return SLC_ERR_INVALID_ARG;
    const DeviceCfg* dev;
    int rc;
    if ((rc = device_cfg(&dev))) return rc;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return note_cuda(e);
    unsigned v = 0;
    e = cudaMemcpy(&v, dev->status, sizeof v, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return note_cuda(e);
    e = cudaMemset(dev->status, 0, sizeof v);
    if (e != cudaSuccess) return note_cuda(e);
    *status = (int32_t)v;
    return SLC_OK;
}

}  // extern "C"
