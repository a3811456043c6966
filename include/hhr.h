/*
 * hhr.h — C ABI of the decode-time coarse-to-fine key retrieval path for top-k
 * sparse attention over a paged KV cache, on NVIDIA B200 (sm_100a).
 *
 * The operations follow two pages:
 *   - "HHR: Hierarchical Hash Retrieval for Efficient LLM Generation", Abstract:
 *     Geometry-Aware Key Routing (a head-wise orthogonal transform R_h and
 *     page-level logit bounds that prune pages), then Learned Hash Projection
 *     (binary codes of a head-wise projection W_h, ranked by Hamming distance),
 *     then attention over the selected keys. Appendix Table 4 fixes 128-bit codes;
 *     64 and 256 bits are supported as code-length variants.
 *   - "HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse Attention",
 *     Abstract: a block-level coarse filter over pooled block representatives,
 *     then the original token indexer inside the kept blocks, then token top-k.
 *
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer unless its comment says "host".
 *     The caller owns every buffer. The library never allocates or frees memory
 *     and never synchronises, except hhr_read_device_status.
 *   - Every device buffer starts on a 16-byte boundary (cudaMalloc gives 256);
 *     a misaligned pointer returns HHR_ERR_INVALID_ARG. Workspaces start on a
 *     256-byte boundary.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).
 *   - Host-side validation runs first and returns an error before any launch:
 *     HHR_ERR_INVALID_ARG (null or misaligned pointer, negative size,
 *     H % G != 0, ...),
 *     HHR_ERR_UNSUPPORTED (head_dim != 128, code_bits not 64/128/256, group > 8, a size
 *     beyond a documented limit), HHR_ERR_WORKSPACE (workspace too small).
 *     A failed launch returns HHR_ERR_CUDA.
 *   - Device-side checks never trap: a page id outside [0, n_phys_pages) or a
 *     token index outside the sequence is skipped and recorded in a device status
 *     word that hhr_read_device_status returns and clears.
 *
 * Layouts (row-major; d = head_dim = 128, W = code_bits / 32 = 2, 4 or 8 words)
 *   k_cache, v_cache : bf16 (uint16 bit patterns) [n_phys_pages][G][P][d]
 *   page_table       : int32 [B][max_pages_per_seq], logical page -> physical page
 *   seq_len          : int32 [B], keys currently in each sequence (after appends)
 *   R                : f32 [G][d][d], orthogonal, applied as x' = R x
 *   W                : f32 [G][code_bits][d], applied to the rotated vector x'
 *   page_minmax      : f32 or f16 (dims.summary_fp16) [n_phys_pages][G][2][d];
 *                      [..][0][:] = per-channel min and [..][1][:] = per-channel max
 *                      of the rotated valid keys
 *   codes            : uint32 [n_phys_pages][G][P][W]; bit j of a code is
 *                      [(W R x)_j > 0], stored in word j/32 at bit j%32
 *   block_mean       : f32 [n_phys_pages][G][d], mean of the page's valid raw keys
 *                      (the HISA pooled block representative; page = block)
 *   q (hash mode)    : bf16 [B][Hq][d]; query head h belongs to KV group h / (Hq/G)
 *   q (indexer mode) : bf16 [B][T][d], one indexer head, T chunk queries
 *   q_pos            : int32 [B][T], absolute position of each chunk query
 * Selections are returned as logical token positions within the sequence.
 */
#ifndef HHR_H
#define HHR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HHR_OK = 0,
  HHR_ERR_INVALID_ARG = -1,
  HHR_ERR_UNSUPPORTED = -2,
  HHR_ERR_CUDA = -3,
  HHR_ERR_WORKSPACE = -4,
  HHR_ERR_DEVICE_STATUS = -6
} hhr_status;

typedef enum { HHR_MODE_HASH = 0, HHR_MODE_INDEXER = 1 } hhr_mode;

/* Problem dimensions. In indexer mode n_q_heads is the chunk length T and
 * n_kv_heads must be 1 (a single indexer head). */
typedef struct {
  int batch;              /* B */
  int n_q_heads;          /* Hq (hash) or T (indexer) */
  int n_kv_heads;         /* G */
  int head_dim;           /* d; must be 128 */
  int page_size;          /* P keys per page (HISA: keys per block), 1..256 */
  int code_bits;          /* 64, 128 (the pages' setting) or 256 */
  int max_pages_per_seq;  /* columns of page_table */
  int n_phys_pages;       /* pages in the pool */
  int summary_fp16;       /* page_minmax element type: 0 = f32; 1 = f16 rounded outward
                             (min toward -inf, max toward +inf), so the page bound stays an
                             upper bound; values beyond the f16 range saturate to -inf/+inf
                             (a channel on which the group's folded query is exactly 0 then
                             contributes 0 to the bound, as it does for every finite key) */
  int select_per_head;    /* hash mode: 0 = one selection per KV group (the default reading:
                             bounds and distances summed over the group's query heads);
                             1 = one per query head (a variant): head h scores the summaries
                             and codes of KV group h / (Hq/G) with its own query alone and
                             attends its own set. Selection rows per sequence ("rows" below)
                             are G, or Hq with 1. Indexer mode: must be 0. */
} hhr_dims;

/* Optional copies of the intermediates of hhr_select, for inspection and layered
 * testing. Any field may be NULL. Hash mode fills all fields; indexer mode fills
 * bounds (block scores, -inf for ineligible blocks), kept and kept_count, with
 * rows indexed by (b, query) instead of (b, group). m_max is the row stride of
 * `kept` (see hhr_kept_max). */
typedef struct {
  float* q_rot;           /* [B][Hq][d]     rotated queries R_g q_h */
  uint32_t* q_code;       /* [B][Hq][W]     query codes */
  float* bounds;          /* [B][G][max_pages_per_seq] page bounds */
  int32_t* kept;          /* [B][G][m_max]  kept logical pages, ascending */
  int32_t* kept_count;    /* [B][G]         kept pages per row */
} hhr_trace;

/* Step a0, key encoding (HHR page, Abstract: keys are encoded into binary codes;
 * GKR rotates them and page-level bounds summarise each page).
 *
 * Sequence b has had keys written to k_cache at logical positions
 * [start[b], start[b] + n_new[b]). For each such key, writes its code; for each
 * page those keys touch, recomputes the page's per-channel min/max over every
 * valid key of the page (positions < start[b] + n_new[b]) and, if block_mean is
 * not NULL, the page's mean raw key. page_minmax and codes may be NULL together
 * (then R and W may be NULL), e.g. for an indexer-only cache.
 *   start, n_new : int32 [B] (device)
 *   max_new      : host int, an upper bound on every n_new[b] (sizes the launch;
 *                  a larger n_new[b] is clipped to it and flagged in the device
 *                  status word)
 * Appends of at least 4096 keys (max_new) with page_size 32, 128-bit codes and no block
 * means run on the tensor-core encoder (tcgen05: one GEMM per 128-key tile against
 * [R; W R], fp32 operands split into three bf16 terms); others on the per-page encoder. Both
 * produce the same layout; their results agree within the code and bound tolerances. */
int hhr_encode_keys(const hhr_dims* dims, const uint16_t* k_cache, const int32_t* page_table,
                    const int32_t* start, const int32_t* n_new, int max_new, const float* R,
                    const float* W, void* page_minmax, uint32_t* codes, float* block_mean,
                    void* stream);

/* Kept pages (or blocks) per row for the given sizes: m_pages > 0 keeps
 * min(m_pages, n) pages, else ceil(n / keep_div). Returns the maximum over any
 * sequence of at most max_pages_per_seq pages (the row stride of trace->kept). */
int hhr_kept_max(const hhr_dims* dims, int m_pages, int keep_div);

/* Optional selection settings of hhr_select / hhr_decode_step (hash mode); a NULL pointer
 * means all zero. Forced sink and local pages are a variant: neither HHR nor HISA forces
 * any page (the HHR page's MagicPIG baseline attends to sink tokens and a local window).
 *   sink_pages  : logical pages [0, sink_pages) of every sequence are always kept, and
 *                 their keys are always selected;
 *   local_pages : likewise the last local_pages pages [n_pages - local_pages, n_pages)
 *                 (the local window, which holds the newest key).
 * Forced pages count toward the page budget: m_b' = max(m_b, #forced pages), the rest
 * chosen by the bound. Forced keys come first in the top-k, in token order (if there are
 * more than top_k of them, the top_k lowest), the others by (delta, t).
 * Both must be >= 0, with sink_pages + local_pages <= hhr_kept_max() (else
 * HHR_ERR_INVALID_ARG); indexer mode accepts only zeros (else HHR_ERR_UNSUPPORTED). */
typedef struct {
  int sink_pages;
  int local_pages;
} hhr_select_opts;

/* Workspace needed by hhr_select (bytes, 256-byte multiple); 0 on invalid input. */
size_t hhr_select_workspace_bytes(const hhr_dims* dims, int mode, int m_pages, int keep_div,
                                  int top_k);

/* Steps a1-a4, selection.
 *
 * HHR_MODE_HASH (HHR page, Abstract; one selection per KV group g, scores summed
 * over the group's query heads):
 *   a1  q'_h = R_g q_h; qcode_h = sign bits of W_g q'_h.
 *   a2  bound_p = sum_{h in g} sum_c max(q'_hc * kmin_pc, q'_hc * kmax_pc) for every
 *       page p < ceil(seq_len[b] / P); keep the m_b largest, ties to the lower page,
 *       where m_b = min(m_pages, n) if m_pages > 0 else ceil(n / keep_div).
 *   a3  delta_t = sum_{h in g} popcount(qcode_h XOR code_t) for every valid key t
 *       of the kept pages.
 *   a4  out_idx[b][g][0..k_eff) = the k_eff = min(top_k, #candidates) keys with the
 *       smallest (delta_t, t), sorted ascending; out_count[b][g] = k_eff; entries
 *       past k_eff are set to -1.
 *   Uses q, seq_len, page_table, R, W, page_minmax, codes; block_mean, k_cache and
 *   q_pos may be NULL.
 *   With dims.select_per_head the rows are the query heads: "h in g" above becomes the
 *   row's single head h, scoring KV group h / (Hq/G)'s summaries and codes.
 *   When m_b covers every page (m_pages >= max_pages_per_seq, or keep_div == 1) no page
 *   bound is needed (a flat hash top-k over every key): the bounds are then computed only
 *   if trace->bounds asks for them.
 * HHR_MODE_INDEXER (HISA page, Abstract; n_kv_heads == 1, n_q_heads = T):
 *   a1' score_blk = q_i . block_mean_blk for blocks with blk*P <= q_pos[b][i];
 *       keep the m_b = min(m_pages, #eligible) best, ties to the lower block.
 *   a3  sigma_t = q_i . k_t in fp32 for t in kept blocks with t <= q_pos[b][i], t < n.
 *   a4  out_idx[b][i][0..k_eff) = the k_eff best by (sigma desc, t asc), ascending.
 *   Uses q, seq_len, q_pos, page_table, block_mean, k_cache; R, W, page_minmax and
 *   codes may be NULL. keep_div must be 0.
 * Limits: ceil(seq_len/P) <= 32768 pages per sequence; m_b * P <= 131072 candidates
 * (hash mode: every page of a 128K-key sequence, a flat hash top-k) or <= 32768
 * (indexer mode).
 * out_idx: int32 [B][rows][top_k]; out_count: int32 [B][rows] (rows = G, Hq with
 * dims.select_per_head, or T in indexer mode; trace->bounds/kept/kept_count likewise).
 * opts: may be NULL (see hhr_select_opts).
 * trace: may be NULL. workspace: at least hhr_select_workspace_bytes(). */
int hhr_select(const hhr_dims* dims, int mode, const uint16_t* q, const int32_t* seq_len,
               const int32_t* q_pos, const int32_t* page_table, const float* R, const float* W,
               const void* page_minmax, const uint32_t* codes, const float* block_mean,
               const uint16_t* k_cache, int m_pages, int keep_div, int top_k,
               const hhr_select_opts* opts, int32_t* out_idx, int32_t* out_count,
               void* workspace, size_t ws_bytes, hhr_trace* trace, void* stream);

/* Workspace needed by hhr_sparse_attn (bytes, 256-byte multiple); 0 on invalid input. */
size_t hhr_attn_workspace_bytes(const hhr_dims* dims, int top_k);

/* Step a4 -> a5, GQA sparse attention over the selected rows (HISA page, Abstract:
 * attention is computed only over the selected subset; GQA layout of HHR appendix
 * Table 3, 32 query heads over 8 KV heads):
 *   out[b][h] = sum_{t in S} softmax_t(scale * q_h . k_t) v_t, with
 *   S = idx[b][g][0..count[b][g]) and g = h / (Hq / G). Every selected K/V row is
 *   read once per group and shared by the group's query heads. An empty set gives
 *   a zero output.
 *   With dims.select_per_head, each query head h attends its own set S = idx[b][h].
 *   idx: int32 [B][rows][top_k] logical tokens; count: int32 [B][rows] (clipped to
 *   top_k); an index outside [0, seq_len[b]) is skipped and flagged.
 *   out: f32 [B][Hq][d]. workspace: at least hhr_attn_workspace_bytes(). */
int hhr_sparse_attn(const hhr_dims* dims, const uint16_t* q, const uint16_t* k_cache,
                    const uint16_t* v_cache, const int32_t* page_table, const int32_t* seq_len,
                    const int32_t* idx, const int32_t* count, int top_k, float scale, float* out,
                    void* workspace, size_t ws_bytes, void* stream);

/* Workspace needed by hhr_decode_step (bytes, 256-byte multiple); 0 on invalid input. */
size_t hhr_decode_step_workspace_bytes(const hhr_dims* dims, int m_pages, int keep_div,
                                       int top_k);

/* One whole HHR decode step (steps a0-a5) in one call, for a decode loop that appends one
 * key/value row per sequence and then attends: the same codes, summaries, selections and
 * counts, bit for bit, as
 *   hhr_encode_keys(start = seq_len - 1, n_new = 1) + hhr_select(HHR_MODE_HASH) +
 *   hhr_sparse_attn,
 * but with the append encoder and the query preparation fused into one kernel (one read
 * of R and W) and the kernels chained with programmatic dependent launch. Steps a2-a5 run
 * in one of two ways:
 *   - small batches (128-bit codes, every selection row's cluster resident at once, at most
 *     16384 pages over all rows: e.g. one sequence of 8 KV groups up to 64K keys): one
 *     kernel, a cluster of 16 CTAs (where all rows' clusters fit) or 8 CTAs per selection row
 *     doing its bounds, top-m, Hamming top-k and attention (at most 16 or 8 attention splits
 *     per row, merged in the cluster);
 *   - otherwise: the page bounds, top-m fused with the Hamming top-k, and the attention, its
 *     splits merged inside a cluster of at most 8 CTAs (or by a combine kernel).
 * The attention output is identical bit for bit to hhr_sparse_attn's wherever the latter's
 * split plan has no more splits than the fused path's cluster (16 or 8 CTAs; every size of
 * the tests); otherwise the fused call merges fewer, larger splits and its outputs can differ in
 * the last bits (both within the attention tolerance). hhr_decode_step_kernels tells how
 * many kernels a call launches. The first call on a device sets kernel attributes and queries
 * how many row clusters fit the device (host-side, once per device): make it before capturing
 * the call into a CUDA graph.
 *   seq_len : lengths after the append; the newest row of sequence b is position
 *             seq_len[b] - 1 (its page must be mapped in page_table).
 *   k_new, v_new : bf16 [B][G][d] newest rows, written into k_cache/v_cache at that
 *             position before encoding; both NULL when the caller already wrote them.
 *   opts, out_idx, out_count, out, scale : as in hhr_select / hhr_sparse_attn.
 * workspace: at least hhr_decode_step_workspace_bytes(). Errors as in the separate calls. */
int hhr_decode_step(const hhr_dims* dims, const uint16_t* q, const uint16_t* k_new,
                    const uint16_t* v_new, uint16_t* k_cache, uint16_t* v_cache,
                    const int32_t* page_table, const int32_t* seq_len, const float* R,
                    const float* W, void* page_minmax, uint32_t* codes, int m_pages,
                    int keep_div, int top_k, const hhr_select_opts* opts, float scale,
                    int32_t* out_idx, int32_t* out_count, float* out, void* workspace,
                    size_t ws_bytes, void* stream);

/* Number of kernels one hhr_decode_step call with these dims and budgets launches on the
 * current device: 2 when steps a2-a5 run as one cluster per selection row (small batches),
 * else 3 to 5 (the bound kernel is skipped when every page is kept, the combine kernel runs
 * when a row's attention splits exceed one cluster). Negative status on invalid input. */
int hhr_decode_step_kernels(const hhr_dims* dims, int m_pages, int keep_div, int top_k);

/* hhr_sparse_attn without a workspace argument, for callers that cannot allocate
 * device memory themselves: runtimes without a device allocator, code running
 * while a memory pool is frozen or being captured, or plugins whose host forbids
 * cudaMalloc. The pages have no counterpart of this call (it is a deployment
 * convenience): it computes the same attention as hhr_sparse_attn, with the
 * split-K partials kept in a fixed 8 MiB device array inside the library instead
 * of a caller workspace.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *     The 8 MiB array is part of the library image, so every GPU that loads the
 *     library holds it until the process exits.
 *   - Limit: hhr_attn_workspace_bytes(dims, top_k) must be at most 8 MiB (8388608
 *     bytes), e.g. batch 8 x 8 KV heads x 4-head groups at top_k 2048 needs about
 *     2.1 MB; a larger problem returns HHR_ERR_WORKSPACE before any CUDA call.
 *   - Every call looks up the array's device address in the current device's
 *     context (cudaGetSymbolAddress), so the address stays right after a device
 *     reset or in another context of the same device. The first call on a device
 *     also loads the library's device code there (the set-up); make that first
 *     call before any stream capture.
 *   - Every call shares the one array and it keeps the last call's contents.
 *     Nothing in it needs to start at zero (each partial is written before it is
 *     read, in stream order), but calls that can overlap on the GPU (different
 *     streams, or different host threads, on one device) race on it: serialise
 *     them.
 * Arguments, outputs and other errors are those of hhr_sparse_attn. */
int hhr_sparse_attn_noalloc(const hhr_dims* dims, const uint16_t* q, const uint16_t* k_cache,
                            const uint16_t* v_cache, const int32_t* page_table,
                            const int32_t* seq_len, const int32_t* idx, const int32_t* count,
                            int top_k, float scale, float* out, void* stream);

/* Kernels that hhr_profile_next can bracket with events. */
typedef enum {
  HHR_KERNEL_ENCODE = 0,     /* hhr_encode_keys; hhr_decode_step's fused prologue */
  HHR_KERNEL_QPREP = 1,      /* hhr_select, hash mode, step a1 */
  HHR_KERNEL_BOUND = 2,      /* hhr_select, hash mode, step a2 bounds */
  HHR_KERNEL_TOPM = 3,       /* hhr_select, indexer mode, top-m blocks */
  HHR_KERNEL_HAMMING = 4,    /* hhr_select, hash mode, top-m pages + steps a3-a4 (fused) */
  HHR_KERNEL_BLOCK = 5,      /* hhr_select, indexer mode, block scores (or the whole
                                selection, when it runs as one cluster per query) */
  HHR_KERNEL_TOKEN = 6,      /* hhr_select, indexer mode, token scores */
  HHR_KERNEL_TOKEN_TOPK = 7, /* hhr_select, indexer mode, token top-k */
  HHR_KERNEL_ATTN = 8,       /* hhr_sparse_attn, split chunks */
  HHR_KERNEL_COMBINE = 9,    /* hhr_sparse_attn, merge of the chunks */
  HHR_KERNEL_ROW = 10,       /* hhr_decode_step, small batches: bounds, top-m, Hamming top-k
                                and attention of each selection row in one cluster */
  HHR_KERNEL_COUNT = 11
} hhr_kernel;

/* Measurement hook (no counterpart on the pages): the next launch of `kernel` by
 * the calling host thread is bracketed by cudaEventRecord(start_event) and
 * cudaEventRecord(stop_event) on that launch's stream (recorded as external events,
 * so inside a stream capture they become event-record nodes of the graph). One-shot:
 * the pair is forgotten after use. Events are cudaEvent_t passed as void*; NULL, NULL clears
 * a pending pair. Returns HHR_ERR_INVALID_ARG for an unknown kernel id. */
int hhr_profile_next(int kernel, void* start_event, void* stop_event);

/* Synchronises `stream`, then returns HHR_OK if no device-side check fired since
 * the last call, else HHR_ERR_DEVICE_STATUS; clears the status word. If `bits` is
 * not NULL (host), receives the raw status bits (1 = bad page id, 2 = bad token
 * index, 4 = n_new clipped to max_new, 8 = a bounded wait in the tensor-core encoder
 * gave up). */
int hhr_read_device_status(void* stream, int* bits);

/* The text of the last CUDA error any hhr_* call met on the calling host thread
 * (the cause behind an HHR_ERR_CUDA), or "no error". Static storage. */
const char* hhr_last_cuda_error(void);

/* A static, human-readable name of a status code. */
const char* hhr_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* HHR_H */
