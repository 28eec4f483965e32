/*
 * slc.h — C ABI of the decode-step combined sparse attention library
 * (libslc.so, CUDA for sm_100a).
 *
 * What it computes.  During decode, each remaining full-attention layer of a
 * hybrid LLM lets the new query attend to three things only: a pinned
 * prefix, a sliding window of recent tokens, and a fixed budget of the most
 * query-relevant tokens of the context ("Accelerating Long-Context Decoding
 * in Large-Scale Hybrid LLMs Without Retraining", abstract).  The relevant
 * tokens are chosen by Quest-style paged selection over the paged KV cache
 * ("Hybrid LLM Decoding 2.2x Faster at 256k, No Retraining", section "The
 * method: sliding window + prefix + query-aware pages, searched per layer").
 * The pages give no formulas; the library fixes them as follows.
 *
 *   pages      16 tokens each; sequence b has n_b = ceil(L_b / 16) pages.
 *   prefix     pages [0, np_b), np_b = min(ceil(P / 16), n_b): every page
 *              that overlaps the first P tokens.
 *   window     pages [ws_b, n_b), ws_b = max(floor(max(0, L_b - W) / 16),
 *              np_b) when W > 0 (every page overlapping the last W tokens,
 *              clamped to the prefix); no window pages when W == 0.
 *   candidates pages [np_b, ws_b).
 *   score      s_j = sum over the query heads h of the kv head's group,
 *              sum over d, of max(q_hd * kmin_jd, q_hd * kmax_jd), with
 *              kmin/kmax the elementwise min/max of the page's keys.
 *   selection  per (sequence, kv head): the min(budget, #candidates)
 *              candidates with the highest score; equal scores go to the
 *              lower page index.  The set is shared by the group's heads.
 *   attention  softmax(scale * q.k) v over the tokens t < L_b of the
 *              prefix, window and selected pages; fp32 output.
 *
 * Memory.  Every buffer is allocated and owned by the caller; all pointers
 * are DEVICE pointers unless stated otherwise.  Cache, metadata and workspace
 * base pointers must be 16-byte aligned.  The library allocates no memory
 * and keeps no state apart from one device status word per GPU (see
 * slc_device_status).
 *
 * Layouts (row-major, innermost last):
 *   K, V cache   bf16 [num_pages][num_kv_heads][16][head_dim]
 *   page meta    [num_pages][num_kv_heads][2][head_dim] (kmin, kmax): bf16,
 *                or 8-bit E4M3 rounded outward (slc_cache_t.meta_format)
 *   q            bf16 [batch][num_q_heads][head_dim]
 *   block_table  int32 [batch][max_pages_per_seq]: logical page -> physical
 *   seq_lens     int32 [batch]: tokens in each sequence (the decode query's
 *                own token included: append first, then decode)
 *   out          fp32 [batch][num_q_heads][head_dim]
 * Query head h belongs to kv head h / (num_q_heads / num_kv_heads).
 *
 * Calls.  Every compute call is asynchronous on `stream` (a cudaStream_t;
 * NULL = the legacy default stream) and launches nothing when it returns an
 * error.  Arguments that live on the device (block-table entries, lengths,
 * positions) are range-checked by the kernels: a bad entry is skipped and
 * flagged in the device status word instead of being dereferenced.  Kernels
 * are launched with programmatic dependent launch (a kernel may start while
 * the previous one on the stream finishes; it waits before reading that
 * kernel's results); the launches that scan the page metadata also carry an
 * L2 access-policy window marking the metadata evict-first for that launch
 * only (no device setting changes).
 *
 * Devices.  Calls run on the device current on the calling thread.  Each
 * kernel's shared-memory limit, occupancy and cluster capacity are looked
 * up once per device, on the first call made with that device current
 * (make that first call before any stream capture).
 *
 * Errors.  0 on success; a negative SLC_ERR_* code otherwise.
 */
#ifndef SLC_H
#define SLC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SLC_API __attribute__((visibility("default")))
#else
#define SLC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *slc_stream_t; /* == cudaStream_t */

enum {
    SLC_OK = 0,
    SLC_ERR_INVALID_ARG = -1,   /* null/misaligned pointer, negative size, ... */
    SLC_ERR_UNSUPPORTED = -2,   /* shape outside what the kernels are built for */
    SLC_ERR_WORKSPACE = -3,     /* workspace smaller than slc_workspace_size() */
    SLC_ERR_CUDA = -4,          /* a CUDA runtime call or launch failed */
    SLC_ERR_DEVICE = -5         /* the device status word reported a fault */
};

/* Device status bits (slc_device_status). */
enum {
    SLC_STATUS_BAD_PAGE = 1,      /* block-table entry outside [0, num_pages) */
    SLC_STATUS_BAD_LENGTH = 2,    /* length/position beyond max_pages_per_seq*16 */
    SLC_STATUS_BAD_SELECTION = 4, /* selected page outside the candidate range */
    SLC_STATUS_WAIT_TIMEOUT = 8   /* a bounded wait on a bulk copy gave up */
};

/* Page metadata formats (slc_cache_t.meta_format). */
enum {
    /* bf16 [num_pages][num_kv_heads][2][head_dim]: kmin, kmax exactly */
    SLC_META_BF16 = 0,
    /* uint8 [num_pages][num_kv_heads][2][head_dim]: kmin and kmax as 8-bit
     * floats E4M3 (OCP "FN": bias 7, 3 mantissa bits, no infinities),
     * rounded OUTWARD -- kmin to the largest E4M3 value <= kmin, kmax to the
     * smallest >= kmax -- so the score stays an upper bound of q.k over the
     * page.  A bound beyond +-448 is stored as the NaN code of its sign
     * (0x7F / 0xFF) and read as the largest bf16 value of that sign; zero is
     * 0x00.  Half the metadata bytes the scoring reads.  (Low-bit scanning:
     * "Faster Than Flash: Fudan FFD Hits 11.6x Kernel Speedup, Pushes
     * Long-Context Decoding to 256K", section "The Hard Constraint on an Old
     * Problem".) */
    SLC_META_FP8_E4M3 = 1
};

/* The paged cache of one layer.  head_dim must be 128 or 256, page_size 16.
 * num_q_heads / num_kv_heads (the GQA group) must be 1..8.  meta_format is
 * one of SLC_META_*; the metadata buffer has the layout of that format. */
typedef struct slc_cache {
    void *k_cache;
    void *v_cache;
    void *meta;
    int32_t num_pages;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t page_size;
    int32_t meta_format;
} slc_cache_t;

/* Append one decode token per sequence.  Writes k_new[b][h] / v_new[b][h]
 * (bf16 [batch][num_kv_heads][head_dim]) into slot positions[b] % 16 of
 * logical page positions[b] / 16, and updates that page's metadata: a page's
 * first token (slot 0) sets kmin = kmax = k; later tokens take the
 * elementwise min / max.  positions: device int32 [batch], usually the old
 * length; the caller then increments its lengths.  The caller maps a new
 * page in block_table before appending its first token.  (Page metadata:
 * Quest-style paged selection, "Hybrid LLM Decoding 2.2x Faster at 256k, No
 * Retraining", section "The method: ...".) */
SLC_API int slc_kv_append(const slc_cache_t *cache, const void *k_new, const void *v_new,
                  const int32_t *block_table, int32_t max_pages_per_seq,
                  const int32_t *positions, int32_t batch, slc_stream_t stream);

/* Rebuild the metadata of every page of every sequence from the keys:
 * kmin/kmax over the page's tokens t < seq_lens[b] (slots past the length
 * are never read).  Run once after prefill.  Same citation as above. */
SLC_API int slc_build_page_meta(const slc_cache_t *cache, const int32_t *block_table,
                        int32_t max_pages_per_seq, const int32_t *seq_lens,
                        int32_t batch, slc_stream_t stream);

/* Bytes of device workspace that slc_sparse_decode / slc_dense_decode need
 * for these shapes (scores, selections, split partials).  Host-only; 0 for
 * unsupported shapes. */
SLC_API size_t slc_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                          int32_t head_dim, int32_t max_pages_per_seq, int32_t budget);

/* Score the candidate pages (the Quest bound above, summed over the GQA
 * group) in fp32.  scores: fp32 [batch][num_kv_heads][max_pages_per_seq];
 * only candidate entries [np_b, ws_b) are written. */
SLC_API int slc_score_pages(const void *q, const slc_cache_t *cache, const int32_t *block_table,
                    int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                    int32_t num_q_heads, int32_t prefix, int32_t window, float *scores,
                    slc_stream_t stream);

/* Fixed-budget selection from scores laid out as slc_score_pages writes
 * them.  selected: int32 [batch][num_kv_heads][budget], ascending page
 * indices, padded with -1.  Candidate counts up to 32768 pages. */
SLC_API int slc_select_pages(const float *scores, int32_t num_kv_heads, int32_t max_pages_per_seq,
                     const int32_t *seq_lens, int32_t batch, int32_t prefix, int32_t window,
                     int32_t budget, int32_t *selected, slc_stream_t stream);

/* Top-delta selection ("Faster Than Flash: Fudan FFD Hits 11.6x Kernel
 * Speedup, Pushes Long-Context Decoding to 256K", section "top-delta: Tearing
 * Down "Global Synchronization" Too"): per (sequence, kv head), the d
 * candidate pages with the highest scores together with every candidate
 * page whose score is within delta of the highest candidate score
 * (s_max - s_j <= delta, the threshold computed in fp32), at most cap pages
 * (the cap best of that union, best = higher score, then lower page).
 * Scores as slc_score_pages writes them.  selected: int32
 * [batch][num_kv_heads][cap], ascending page indices, padded with -1.
 * d >= 0, cap >= 0, delta not NaN (+inf keeps every candidate, a negative
 * delta only the top d); SLC_ERR_INVALID_ARG otherwise.  Candidate counts
 * up to 32768 pages. */
SLC_API int slc_select_pages_delta(const float *scores, int32_t num_kv_heads,
                           int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                           int32_t prefix, int32_t window, int32_t d, float delta, int32_t cap,
                           int32_t *selected, slc_stream_t stream);

/* One decode step of one layer, in two kernels:
 *   1 (streaming)  attention over the prefix and window pages, and the
 *                  scores of the candidate pages (all SMs, HBM-bound);
 *   2 (finishing)  per unit, on one thread-block cluster: the selection,
 *                  attention over the selected pages, and the merge of all
 *                  partials into out.
 * scale <= 0 means 1/sqrt(head_dim).  selected_out (nullable) receives the
 * selection as slc_select_pages writes it.  workspace: device, >=
 * slc_workspace_size().  A nonzero device status word after the call
 * (slc_device_status) means out and selected_out may be invalid. */
SLC_API int slc_sparse_decode(const void *q, const slc_cache_t *cache, const int32_t *block_table,
                      int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                      int32_t num_q_heads, int32_t prefix, int32_t window, int32_t budget,
                      float scale, float *out, int32_t *selected_out, void *workspace,
                      size_t workspace_bytes, slc_stream_t stream);

/* One of the two kernels of slc_sparse_decode alone (same arguments), for
 * timing and inspection:
 *   1  the streaming kernel: prefix/window attention partials and candidate
 *      scores, left in the workspace;
 *   2  the finishing kernel: selection (into selected_out when given),
 *      selected-page attention and the merge into out, from what stage 1
 *      left in the same workspace.
 * Running 1 then 2 equals one slc_sparse_decode call.  Returns
 * SLC_ERR_INVALID_ARG for any other stage. */
SLC_API int slc_sparse_decode_stage(int32_t stage, const void *q, const slc_cache_t *cache,
                            const int32_t *block_table, int32_t max_pages_per_seq,
                            const int32_t *seq_lens, int32_t batch, int32_t num_q_heads,
                            int32_t prefix, int32_t window, int32_t budget, float scale,
                            float *out, int32_t *selected_out, void *workspace,
                            size_t workspace_bytes, slc_stream_t stream);

/* Attention over the prefix pages, the window pages and a caller-given
 * selection (same layout as slc_select_pages writes: [batch][num_kv_heads]
 * [budget] ascending logical pages, -1 padded).  The attended set is the
 * union: every entry j with 0 <= j < n_b is attended once (an entry that is
 * itself a prefix or window page of this call adds nothing), -1 entries are
 * padding, and an entry that is out of range or not above the entry before
 * it is skipped and flagged (SLC_STATUS_BAD_SELECTION).  This lets a layer
 * reuse the selection of another layer of the same sequences -- cross-layer
 * index reuse ("IndexCache: cross-layer reuse speeds 30B prefill 1.82x":
 * Shared layers take the top-k of the nearest Full layer) -- even when the
 * two layers' windows differ. */
SLC_API int slc_sparse_attend(const void *q, const slc_cache_t *cache, const int32_t *block_table,
                      int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                      int32_t num_q_heads, int32_t prefix, int32_t window, int32_t budget,
                      const int32_t *selected, float scale, float *out, void *workspace,
                      size_t workspace_bytes, slc_stream_t stream);

/* One decode step with the top-delta selection in place of the fixed
 * budget: the two kernels of slc_sparse_decode, the finishing kernel setting
 * each unit's selection size from its scores (the top d plus every candidate
 * within delta of the best, at most cap; the same selection as
 * slc_select_pages_delta on the same scores), written to selected_out when
 * given (int32 [batch][num_kv_heads][cap], ascending, -1 padded).
 * workspace >= slc_workspace_size(..., budget = cap).  Other arguments and
 * errors as slc_sparse_decode and slc_select_pages_delta. */
SLC_API int slc_sparse_decode_delta(const void *q, const slc_cache_t *cache,
                            const int32_t *block_table, int32_t max_pages_per_seq,
                            const int32_t *seq_lens, int32_t batch, int32_t num_q_heads,
                            int32_t prefix, int32_t window, int32_t d, float delta,
                            int32_t cap, float scale, float *out, int32_t *selected_out,
                            void *workspace, size_t workspace_bytes, slc_stream_t stream);

/* Full attention over every token of every sequence (the comparison
 * point: a full-attention layer reads every key at each step, "Hybrid LLM
 * Decoding 2.2x Faster at 256k, No Retraining", section "The remaining
 * full-attention layers are the long-context bill"). */
SLC_API int slc_dense_decode(const void *q, const slc_cache_t *cache, const int32_t *block_table,
                     int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                     int32_t num_q_heads, float scale, float *out, void *workspace,
                     size_t workspace_bytes, slc_stream_t stream);

/* Bytes of device scratch that slc_sparse_decode_static owns (16 MiB). */
#define SLC_STATIC_SCRATCH_BYTES ((size_t)16 << 20)

/* slc_sparse_decode for callers that cannot allocate device memory: the
 * same decode step (same arguments and results, minus the workspace), with
 * its scratch taken from a fixed SLC_STATIC_SCRATCH_BYTES array that lives
 * in the library's device code.  This entry point has no counterpart in the
 * paper; it exists because some callers cannot allocate device memory at
 * all -- for instance a plugin running inside a host framework that owns
 * every byte of GPU memory through its own pool and forbids direct
 * cudaMalloc -- so they cannot provide the workspace slc_sparse_decode
 * needs.
 *
 * - Allocates nothing: no cudaMalloc/cudaFree and no allocating library
 *   call.  Every GPU that loads the library holds the array until the
 *   process exits.
 * - Shapes whose workspace (slc_workspace_size) exceeds
 *   SLC_STATIC_SCRATCH_BYTES are rejected with SLC_ERR_WORKSPACE before any
 *   CUDA call.
 * - The first call on a device looks up the array's device address (once
 *   per device, with that device current); make that first call before
 *   any stream capture.
 * - Every call on a device shares the one array, and the array keeps the
 *   last call's contents (nothing in it needs to start at zero).  Calls
 *   whose executions overlap on the GPU -- on different streams, or from
 *   different host threads -- race on it: serialise them. */
SLC_API int slc_sparse_decode_static(const void *q, const slc_cache_t *cache,
                             const int32_t *block_table, int32_t max_pages_per_seq,
                             const int32_t *seq_lens, int32_t batch, int32_t num_q_heads,
                             int32_t prefix, int32_t window, int32_t budget, float scale,
                             float *out, int32_t *selected_out, slc_stream_t stream);

/* Synchronise `stream`, read the current GPU's status word into *status
 * (host pointer; SLC_STATUS_* bits), then clear it.  Returns SLC_OK, or
 * SLC_ERR_CUDA. */
SLC_API int slc_device_status(int32_t *status, slc_stream_t stream);

/* Static description of an SLC_ERR_* code. */
SLC_API const char *slc_error_string(int code);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
SLC_API const char *slc_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SLC_H */
