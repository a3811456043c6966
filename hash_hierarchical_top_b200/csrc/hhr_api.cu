// C ABI of the retrieval path: argument validation, workspace layout and launches.
// Every kernel lives in the headers included below (one translation unit, so the
// device status word is a single symbol).
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>

#include <initializer_list>

#include "../../include/hhr.h"
#include "attn.cuh"
#include "common.cuh"
#include "encode.cuh"
#include "encode_tc.cuh"
#include "indexer.cuh"
#include "row_cluster.cuh"
#include "select.cuh"
#include "step.cuh"

using namespace hhr;

namespace {

constexpr int kMaxPagesPerSeq = 32768;  // top-m keys staged in 128 KB of shared memory
constexpr int kMaxTokCand = 32768;      // indexer token candidates per query
constexpr int kMaxDevices = 64;
constexpr int kTcMinBulk = 4096;  // appends at least this long use the tensor-core encoder
constexpr int kTcSlots = 148;     // persistent encoder CTAs (one per SM of a B200)
constexpr size_t kMaxKernelSmem = 200 * 1024;  // below the 227 KB opt-in of sm_100
// Summaries of the first selection rows, about this many bytes, are prefetched into L2 by
// the fused step's prologue for the page-bound kernel that follows it.
#ifndef HHR_WARM_MB
#define HHR_WARM_MB 44
#endif
constexpr size_t kWarmBytes = (size_t)HHR_WARM_MB << 20;
// Indexer mode runs as one cluster of kIxRanks CTAs per query (indexer_cluster_kernel) when
// there are at most this many queries (B x T) and the sizes fit; else as four kernels.
#ifndef HHR_IX_CLUSTER_MAX_QUERIES
#define HHR_IX_CLUSTER_MAX_QUERIES 8
#endif
// Page bounds: 1 = page_bound_stage_kernel (summaries staged page-major in shared memory by
// bulk copies), 0 = page_bound_kernel (summaries loaded to registers).
// 1: hhr_decode_step runs steps a2-a5 of small batches (at most one wave of row clusters)
// in row_cluster_kernel; 0: always the chain of separate kernels.
#ifndef HHR_ROW_CLUSTER
#define HHR_ROW_CLUSTER 1
#endif
// Largest batch x selection rows x pages per sequence for the row-cluster path. Its bounds
// run on the rows' clusters only (64 SMs for 8 rows of 8 CTAs), at about the per-SM rate of
// the page-bound kernel, so past a few MB of summaries the separate page-bound kernel on every
// SM wins. Measured on B200 (one sequence of 8 KV groups, f16 summaries, L2-cold): 32K context
// (8 x 1024 pages) 34.7 us per step against 36.5 us for the kernel chain; 128K (8 x 4096
// pages) 39.1 against 35.2 us.
#ifndef HHR_ROW_MAX_PAGES
#define HHR_ROW_MAX_PAGES 16384
#endif

#ifndef HHR_BOUND_STAGE
#define HHR_BOUND_STAGE 0
#endif

// Every device buffer is read with 16-byte vector loads somewhere on the path.
bool misaligned16(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs)
    if (((uintptr_t)p & 15) != 0) return true;
  return false;
}

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int check_dims(const hhr_dims* d) {
  if (d == nullptr) return HHR_ERR_INVALID_ARG;
  if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1 || d->page_size < 1 ||
      d->max_pages_per_seq < 1 || d->n_phys_pages < 1)
    return HHR_ERR_INVALID_ARG;
  if (d->n_q_heads % d->n_kv_heads != 0) return HHR_ERR_INVALID_ARG;
  if (d->head_dim != kD) return HHR_ERR_UNSUPPORTED;
  if (d->code_bits != 64 && d->code_bits != 128 && d->code_bits != 256) return HHR_ERR_UNSUPPORTED;
  if (d->page_size > 256 || d->batch > 65535 || d->n_kv_heads > 65535)
    return HHR_ERR_UNSUPPORTED;
  if (d->max_pages_per_seq > kMaxPagesPerSeq) return HHR_ERR_UNSUPPORTED;
  if (d->summary_fp16 != 0 && d->summary_fp16 != 1) return HHR_ERR_INVALID_ARG;
  if (d->select_per_head != 0 && d->select_per_head != 1) return HHR_ERR_INVALID_ARG;
  return HHR_OK;
}

// Selection rows per sequence (KV groups, or query heads with select_per_head) and the
// number of rows that share one KV head.
inline int sel_rows(const hhr_dims* d) { return d->select_per_head ? d->n_q_heads : d->n_kv_heads; }
inline int kv_div(const hhr_dims* d) { return sel_rows(d) / d->n_kv_heads; }

// 32-bit code words per key and its index among the supported lengths (2, 4, 8 words).
inline int code_words(const hhr_dims* d) { return d->code_bits / 32; }
inline int cw_index(int cw) { return cw == 2 ? 0 : cw == 4 ? 1 : 2; }

// Group size, and selection rows per sequence (a grid dimension: at most 65535).
int check_group(const hhr_dims* d) {
  if (d->n_q_heads / d->n_kv_heads > kMaxGroup) return HHR_ERR_UNSUPPORTED;
  return sel_rows(d) > 65535 ? HHR_ERR_UNSUPPORTED : HHR_OK;
}

thread_local cudaError_t g_last_cuda = cudaSuccess;

// SMs of the current device (cached per device; 148 on B200 if the query fails).
int sm_count() {
  static int cached[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// Raise a kernel's dynamic shared-memory limit (opt-in maximum minus the kernel's
// static shared memory) once per device, and check that `bytes` fits under it.
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes, bool* done_per_dev) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return g_last_cuda = e;
  if (dev < 0 || dev >= kMaxDevices) return g_last_cuda = cudaErrorInvalidDevice;
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return g_last_cuda = e;
  int optin = 0;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
      cudaSuccess)
    return g_last_cuda = e;
  const size_t limit = (size_t)optin - fa.sharedSizeBytes;
  if (bytes > limit) return g_last_cuda = cudaErrorInvalidValue;
  if (done_per_dev[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)limit);
  if (e == cudaSuccess) done_per_dev[dev] = true;
  else g_last_cuda = e;
  return e;
}

bool g_smem_ix[kMaxDevices], g_smem_stage[2][kMaxDevices], g_smem_tc[kMaxDevices], g_smem_encode[3][kMaxDevices], g_smem_qprep[3][kMaxDevices],
    g_smem_sel[kMaxDevices], g_smem_ham[3][2][4][kMaxDevices], g_smem_blk[kMaxDevices], g_smem_attn[kMaxDevices],
    g_smem_attn_cl[kMaxDevices], g_smem_row[kRowVariants][kMaxDevices];

struct SelectLayout {
  size_t qpn, q_rot, q_code, bounds, kept, kept_count, tok, total;
};

int kept_max(const hhr_dims* d, int m_pages, int keep_div) {
  return kept_for(d->max_pages_per_seq, m_pages, keep_div);
}

SelectLayout select_layout(const hhr_dims* d, int mode, int m_max) {
  SelectLayout L{};
  const size_t B = d->batch, Gs = sel_rows(d), Hq = d->n_q_heads, maxp = d->max_pages_per_seq;
  size_t off = 0;
  if (mode == HHR_MODE_HASH) {
    L.qpn = off;    off += align256(B * (size_t)d->n_kv_heads * 2 * kD * 4);
    L.q_rot = off;  off += align256(B * Hq * kD * 4);
    L.q_code = off; off += align256(B * Hq * code_words(d) * 4);
    L.bounds = off; off += align256(B * Gs * maxp * 4);
    L.kept = off;   off += align256(B * Gs * (size_t)m_max * 4);
    L.kept_count = off; off += align256(B * Gs * 4);
  } else {
    const size_t T = Hq;
    L.bounds = off; off += align256(B * T * maxp * 4);
    L.kept = off;   off += align256(B * T * (size_t)m_max * 4);
    L.kept_count = off; off += align256(B * T * 4);
    L.tok = off;    off += align256(B * T * (size_t)m_max * d->page_size * 4);
  }
  L.total = off;
  return L;
}

int check_select_params(const hhr_dims* d, int mode, int m_pages, int keep_div, int top_k) {
  int st = check_dims(d);
  if (st != HHR_OK) return st;
  if (top_k < 1 || m_pages < 0 || keep_div < 0) return HHR_ERR_INVALID_ARG;
  if (mode == HHR_MODE_HASH) {
    if ((m_pages > 0) == (keep_div > 0)) return HHR_ERR_INVALID_ARG;
    if (check_group(d) != HHR_OK) return HHR_ERR_UNSUPPORTED;
    // B x rows x ranks CTAs of the top-m + Hamming kernel form one grid dimension.
    if ((long long)d->batch * sel_rows(d) * kHamRanks > 0x7fffffffLL) return HHR_ERR_UNSUPPORTED;
    if ((long long)kept_max(d, m_pages, keep_div) * d->page_size > kMaxCand)
      return HHR_ERR_UNSUPPORTED;
    if (topm_hamming_smem(d->n_q_heads / sel_rows(d), code_words(d),
                          kept_max(d, m_pages, keep_div), d->page_size,
                          d->max_pages_per_seq) > kMaxKernelSmem)
      return HHR_ERR_UNSUPPORTED;
  } else if (mode == HHR_MODE_INDEXER) {
    if (m_pages < 1 || keep_div != 0) return HHR_ERR_INVALID_ARG;
    if (d->select_per_head) return HHR_ERR_INVALID_ARG;  // indexer rows are queries already
    if (d->n_kv_heads != 1) return HHR_ERR_INVALID_ARG;
    if ((long long)kept_max(d, m_pages, 0) * d->page_size > kMaxTokCand)
      return HHR_ERR_UNSUPPORTED;
    if ((long long)d->batch * d->n_q_heads > 0x7fffffffLL) return HHR_ERR_UNSUPPORTED;
  } else {
    return HHR_ERR_INVALID_ARG;
  }
  return HHR_OK;
}

// Forced sink/local pages of the options (zero without options), validated.
int read_opts(const hhr_dims* d, int mode, const hhr_select_opts* o, int m_pages, int keep_div,
              int* sink, int* local) {
  *sink = *local = 0;
  if (o == nullptr) return HHR_OK;
  if (o->sink_pages < 0 || o->local_pages < 0) return HHR_ERR_INVALID_ARG;
  if (o->sink_pages == 0 && o->local_pages == 0) return HHR_OK;
  if (mode != HHR_MODE_HASH) return HHR_ERR_UNSUPPORTED;
  if ((long long)o->sink_pages + o->local_pages > kept_max(d, m_pages, keep_div))
    return HHR_ERR_INVALID_ARG;
  *sink = o->sink_pages;
  *local = o->local_pages;
  return HHR_OK;
}

// One-shot event pairs of hhr_profile_next, per host thread.
struct ProfPair {
  cudaEvent_t start, stop;
};
thread_local ProfPair g_prof[HHR_KERNEL_COUNT];

// Inside a stream capture the records are external, so that they become event-record
// nodes of the graph (timestamps taken at every replay) rather than internal
// dependencies; outside a capture they are plain records.
void prof_record(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) cs = cudaStreamCaptureStatusNone;
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  else
    cudaEventRecord(e, s);
}
void prof_begin(int k, cudaStream_t s) {
  if (g_prof[k].start != nullptr) prof_record(g_prof[k].start, s);
}
void prof_end(int k, cudaStream_t s) {
  if (g_prof[k].stop != nullptr) prof_record(g_prof[k].stop, s);
  g_prof[k].start = nullptr;
  g_prof[k].stop = nullptr;
}

int launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) g_last_cuda = e;
  return e == cudaSuccess ? HHR_OK : HHR_ERR_CUDA;
}

// Launch with programmatic stream serialisation: the kernel may start while the previous
// kernel of the stream finishes; it calls griddepcontrol.wait before touching memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Launches the page bounds of every selection row (step a2), with programmatic stream
// serialisation when `pdl`: page_bound_stage_kernel (summaries staged page-major in shared
// memory by bulk copies; persistent, one CTA per SM), or page_bound_kernel (summaries loaded
// to registers) where its shared-memory prefix does not fit or HHR_BOUND_STAGE is 0.
cudaError_t launch_bounds_kernel(const hhr_dims* d, const BoundArgs& ba, bool pdl,
                                 cudaStream_t s) {
  const bool ph = kv_div(d) > 1, f16 = d->summary_fp16 != 0;
  const int B = d->batch, Gs = sel_rows(d), maxp = d->max_pages_per_seq;
  if (HHR_BOUND_STAGE && B <= kStageMaxBatch && stage_slots(d->n_kv_heads, f16) >= 2) {
    void (*k)(BoundArgs, int) = f16 ? page_bound_stage_kernel<true> : page_bound_stage_kernel<false>;
    const size_t smem = stage_smem(d->n_kv_heads, f16, B);
    cudaError_t e = allow_smem(k, smem, g_smem_stage[f16 ? 1 : 0]);
    if (e != cudaSuccess) return e;
    const int S = stage_slots(d->n_kv_heads, f16);
    const dim3 grid(sm_count());
    if (pdl) return launch_pdl(k, grid, dim3(kStageThreads), smem, s, ba, S);
    k<<<grid, kStageThreads, smem, s>>>(ba, S);
    return cudaGetLastError();
  }
  const int ppc = bound_pages_per_cta(f16);
  const dim3 grid = bound_grid(Gs, (maxp + ppc - 1) / ppc, B);
  void (*k)(BoundArgs) =
      f16 ? (ph ? page_bound_kernel<true, true> : page_bound_kernel<true, false>)
          : (ph ? page_bound_kernel<false, true> : page_bound_kernel<false, false>);
  if (pdl) return launch_pdl(k, grid, dim3(kBoundWarps * 32), 0, s, ba);
  k<<<grid, kBoundWarps * 32, 0, s>>>(ba);
  return cudaGetLastError();
}

// Whether a cluster of kIxRanks CTAs of indexer_cluster_kernel can be resident on this
// device with `smem` bytes of dynamic shared memory (checked once per device; the kernel's
// non-portable cluster size is enabled on the way). 0 unknown, 1 yes, -1 no.
int g_ix_ok[kMaxDevices];
bool indexer_cluster_ready(size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (allow_smem(indexer_cluster_kernel, smem, g_smem_ix) != cudaSuccess) return false;
  if (g_ix_ok[dev] == 0) {
    int ok = -1;
    if (cudaFuncSetAttribute(indexer_cluster_kernel,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(kIxRanks, 1);
      cfg.blockDim = dim3(kIxThreads);
      cfg.dynamicSmemBytes = ix_smem(kIxMaxBlocks, kIxMaxCand / 128, 128);
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = kIxRanks;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, indexer_cluster_kernel, &cfg) == cudaSuccess && n > 0)
        ok = 1;
    }
    cudaGetLastError();  // a refused query leaves no sticky error
    g_ix_ok[dev] = ok;
  }
  return g_ix_ok[dev] == 1;
}

// How many clusters of row_cluster_kernel instantiation `index` (`ranks` CTAs of
// kRowThreads threads) can be resident at once on this device: checked once per device and
// instantiation (a non-portable cluster size is enabled on the way); 0 when it cannot run
// or `smem` bytes of dynamic shared memory do not fit.
int g_row_cap[kMaxDevices][kRowVariants];
int row_cluster_capacity(RowClusterFn fn, int index, int ranks, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  if (allow_smem(fn, smem, g_smem_row[index]) != cudaSuccess) return 0;
  int& cap = g_row_cap[dev][index];
  if (cap == 0) {
    int n = -1;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(ranks);
      cfg.blockDim = dim3(kRowThreads);
      cfg.dynamicSmemBytes = attn_smem();
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = ranks;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n <= 0) n = -1;
    }
    cudaGetLastError();  // a refused query leaves no sticky error
    cap = n;
  }
  return cap > 0 ? cap : 0;
}

// hhr_decode_step's steps a2-a5 as row_cluster_kernel: used when the codes are 128-bit, the
// batch's rows hold at most HHR_ROW_MAX_PAGES pages in all, the row's attention splits fit
// the cluster and every selection row's cluster is resident at once: clusters of 16 CTAs
// where they all fit, else of 8.
struct RowPlan {
  bool use;
  int ranks;
  RowClusterFn fn;
  size_t smem;
  AttnPlan attn;
};
RowPlan row_plan(const hhr_dims* d, int m_max, int top_k) {
  RowPlan p{};
  if (!HHR_ROW_CLUSTER || code_words(d) != 4) return p;
  const int Gs = sel_rows(d), rh = d->n_q_heads / Gs;
  const bool f16 = d->summary_fp16 != 0;
  const long long rows = (long long)d->batch * Gs;
  if (rows * d->max_pages_per_seq > HHR_ROW_MAX_PAGES) return p;
  for (int ranks : {16, 8}) {
    p.ranks = ranks;
    p.attn = attn_plan(d->batch, Gs, top_k, ranks);
    p.fn = row_cluster_for(rh, f16, ranks);
    p.smem = row_cluster_smem(rh, 4, m_max, d->page_size, d->max_pages_per_seq, ranks);
    p.use = p.attn.n_splits <= ranks &&
            rows <= row_cluster_capacity(p.fn, row_cluster_index(rh, f16, ranks), ranks, p.smem);
    if (p.use) break;
  }
  return p;
}

int copy_trace(void* dst, const char* ws, size_t off, size_t bytes, cudaStream_t s) {
  if (dst == nullptr || bytes == 0) return HHR_OK;
  cudaError_t e = cudaMemcpyAsync(dst, ws + off, bytes, cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) g_last_cuda = e;
  return e == cudaSuccess ? HHR_OK : HHR_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* hhr_status_string(int s) {
  switch (s) {
    case HHR_OK: return "HHR_OK";
    case HHR_ERR_INVALID_ARG: return "HHR_ERR_INVALID_ARG";
    case HHR_ERR_UNSUPPORTED: return "HHR_ERR_UNSUPPORTED";
    case HHR_ERR_CUDA: return "HHR_ERR_CUDA";
    case HHR_ERR_WORKSPACE: return "HHR_ERR_WORKSPACE";
    case HHR_ERR_DEVICE_STATUS: return "HHR_ERR_DEVICE_STATUS";
    default: return "HHR_UNKNOWN_STATUS";
  }
}

const char* hhr_last_cuda_error(void) {
  return g_last_cuda == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda);
}

int hhr_profile_next(int kernel, void* start_event, void* stop_event) {
  if (kernel < 0 || kernel >= HHR_KERNEL_COUNT) return HHR_ERR_INVALID_ARG;
  g_prof[kernel].start = (cudaEvent_t)start_event;
  g_prof[kernel].stop = (cudaEvent_t)stop_event;
  return HHR_OK;
}

int hhr_kept_max(const hhr_dims* d, int m_pages, int keep_div) {
  if (check_dims(d) != HHR_OK || m_pages < 0 || keep_div < 0 || (m_pages == 0 && keep_div == 0))
    return -1;
  return kept_max(d, m_pages, keep_div);
}

int hhr_encode_keys(const hhr_dims* d, const uint16_t* k_cache, const int32_t* page_table,
                    const int32_t* start, const int32_t* n_new, int max_new, const float* R,
                    const float* W, void* page_minmax, uint32_t* codes, float* block_mean,
                    void* stream) {
  int st = check_dims(d);
  if (st != HHR_OK) return st;
  if (k_cache == nullptr || page_table == nullptr || start == nullptr || n_new == nullptr)
    return HHR_ERR_INVALID_ARG;
  const bool hashing = page_minmax != nullptr || codes != nullptr;
  if (hashing && (page_minmax == nullptr || codes == nullptr || R == nullptr || W == nullptr))
    return HHR_ERR_INVALID_ARG;
  if (!hashing && block_mean == nullptr) return HHR_ERR_INVALID_ARG;
  if (misaligned16({k_cache, R, W, page_minmax, codes, block_mean})) return HHR_ERR_INVALID_ARG;
  if (max_new < 0) return HHR_ERR_INVALID_ARG;
  if (max_new == 0) return HHR_OK;
  const long long pages = (long long)(max_new + d->page_size - 1) / d->page_size + 1;
  if (pages > 0x7fffffffLL) return HHR_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  const int cw = code_words(d);
  if (hashing && block_mean == nullptr && d->page_size == kTcPage && max_new >= kTcMinBulk &&
      cw == kWords) {
    // Bulk append (e.g. a prefill) of 128-bit codes: the tensor-core encoder.
    if (allow_smem(encode_tc_kernel, kTcSmem, g_smem_tc) != cudaSuccess) return HHR_ERR_CUDA;
    const int G = d->n_kv_heads;
    int cpg = kTcSlots / G;
    if (cpg < 1) cpg = 1;
    EncodeTcArgs ta{k_cache, page_table, start, n_new, R, W, page_minmax, codes, d->batch, G,
                    d->max_pages_per_seq, d->n_phys_pages, max_new, d->summary_fp16, cpg,
                    (d->max_pages_per_seq * kTcPage + kTcTile - 1) / kTcTile};
    prof_begin(HHR_KERNEL_ENCODE, s);
    encode_tc_kernel<<<dim3(cpg, G), kTcThreads, kTcSmem, s>>>(ta);
    prof_end(HHR_KERNEL_ENCODE, s);
    return launch_status();
  }
  EncodeArgs a{k_cache, page_table, start, n_new, hashing ? R : nullptr, hashing ? W : nullptr,
               page_minmax, codes, block_mean, d->n_kv_heads, d->page_size,
               d->max_pages_per_seq, d->n_phys_pages, max_new, d->summary_fp16};
  size_t smem = hashing ? encode_page_smem() : 0;
  void (*enc)(EncodeArgs) =
      cw == 2 ? encode_page_kernel<2> : cw == 8 ? encode_page_kernel<8> : encode_page_kernel<4>;
  if (hashing && allow_smem(enc, smem, g_smem_encode[cw_index(cw)]) != cudaSuccess)
    return HHR_ERR_CUDA;
  dim3 grid((unsigned)pages, d->n_kv_heads, d->batch);
  prof_begin(HHR_KERNEL_ENCODE, s);
  enc<<<grid, kMvThreads, smem, s>>>(a);
  prof_end(HHR_KERNEL_ENCODE, s);
  return launch_status();
}

size_t hhr_select_workspace_bytes(const hhr_dims* d, int mode, int m_pages, int keep_div,
                                  int top_k) {
  if (check_select_params(d, mode, m_pages, keep_div, top_k) != HHR_OK) return 0;
  return select_layout(d, mode, kept_max(d, m_pages, keep_div)).total;
}

int hhr_select(const hhr_dims* d, int mode, const uint16_t* q, const int32_t* seq_len,
               const int32_t* q_pos, const int32_t* page_table, const float* R, const float* W,
               const void* page_minmax, const uint32_t* codes, const float* block_mean,
               const uint16_t* k_cache, int m_pages, int keep_div, int top_k,
               const hhr_select_opts* opts, int32_t* out_idx, int32_t* out_count,
               void* workspace, size_t ws_bytes, hhr_trace* trace, void* stream) {
  int st = check_select_params(d, mode, m_pages, keep_div, top_k);
  if (st != HHR_OK) return st;
  int sink = 0, local = 0;
  if ((st = read_opts(d, mode, opts, m_pages, keep_div, &sink, &local)) != HHR_OK) return st;
  if (q == nullptr || seq_len == nullptr || page_table == nullptr || out_idx == nullptr ||
      out_count == nullptr || workspace == nullptr)
    return HHR_ERR_INVALID_ARG;
  if (mode == HHR_MODE_HASH &&
      (R == nullptr || W == nullptr || page_minmax == nullptr || codes == nullptr))
    return HHR_ERR_INVALID_ARG;
  if (mode == HHR_MODE_INDEXER && (q_pos == nullptr || block_mean == nullptr || k_cache == nullptr))
    return HHR_ERR_INVALID_ARG;
  if (misaligned16({q, R, W, page_minmax, codes, block_mean, k_cache})) return HHR_ERR_INVALID_ARG;
  const int m_max = kept_max(d, m_pages, keep_div);
  const SelectLayout L = select_layout(d, mode, m_max);
  if (ws_bytes < L.total) return HHR_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255) != 0) return HHR_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  char* ws = static_cast<char*>(workspace);
  const int B = d->batch, G = d->n_kv_heads, Hq = d->n_q_heads, P = d->page_size;
  const int maxp = d->max_pages_per_seq;
  float* bounds = reinterpret_cast<float*>(ws + L.bounds);
  int32_t* kept = reinterpret_cast<int32_t*>(ws + L.kept);
  int32_t* kept_count = reinterpret_cast<int32_t*>(ws + L.kept_count);
  if (allow_smem(select_largest_kernel,
                 (size_t)4 * (mode == HHR_MODE_HASH ? maxp : max(maxp, m_max * P)),
                 g_smem_sel) != cudaSuccess)
    return HHR_ERR_CUDA;

  if (mode == HHR_MODE_HASH) {
    float* qpn = reinterpret_cast<float*>(ws + L.qpn);
    float* q_rot = reinterpret_cast<float*>(ws + L.q_rot);
    uint32_t* q_code = reinterpret_cast<uint32_t*>(ws + L.q_code);
    const int cw = code_words(d);
    void (*qp)(QPrepArgs) =
        cw == 2 ? qprep_kernel<2> : cw == 8 ? qprep_kernel<8> : qprep_kernel<4>;
    if (allow_smem(qp, qprep_smem(), g_smem_qprep[cw_index(cw)]) != cudaSuccess) return HHR_ERR_CUDA;
    const int Gs = sel_rows(d), rh = Hq / Gs;  // selection rows and their query heads
    const int nt = topm_hamming_threads(cw, (long long)B * Gs * kHamRanks, sm_count());
    if (allow_smem(topm_hamming_for(rh, cw, nt), topm_hamming_smem(rh, cw, m_max, P, maxp),
                   g_smem_ham[cw_index(cw)][nt == 512][hamming_planes(rh) - 1]) != cudaSuccess)
      return HHR_ERR_CUDA;
    prof_begin(HHR_KERNEL_QPREP, s);
    qp<<<dim3(G, B), kMvThreads, qprep_smem(), s>>>(
        QPrepArgs{q, R, W, q_rot, q_code, qpn, Hq, G});
    prof_end(HHR_KERNEL_QPREP, s);
    if ((st = launch_status()) != HHR_OK) return st;
    // Every page kept (flat hash top-k): the bounds are computed only for a trace.
    const bool flat = m_max >= maxp;
    if (!flat || (trace != nullptr && trace->bounds != nullptr)) {
      const BoundArgs ba{qpn, q_rot, page_minmax, page_table, seq_len, bounds, G, P, maxp,
                         d->n_phys_pages, 0, Gs, kv_div(d), B};
      prof_begin(HHR_KERNEL_BOUND, s);
      const cudaError_t e = launch_bounds_kernel(d, ba, false, s);
      prof_end(HHR_KERNEL_BOUND, s);
      if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
    }
    HammingArgs ha{q_code, codes, page_table, seq_len, kept, kept_count, out_idx, out_count,
                   Hq, G, P, maxp, d->n_phys_pages, m_max, top_k, nullptr, sink, local,
                   Gs, kv_div(d)};
    const size_t fsm = topm_hamming_smem(rh, cw, m_max, P, maxp);
    prof_begin(HHR_KERNEL_HAMMING, s);
    topm_hamming_for(rh, cw, nt)<<<B * Gs * kHamRanks, nt, fsm, s>>>(
        TopmHammingArgs{ha, bounds, m_pages, keep_div, flat ? 1 : 0});
    prof_end(HHR_KERNEL_HAMMING, s);
    if ((st = launch_status()) != HHR_OK) return st;
    if (trace != nullptr) {
      if ((st = copy_trace(trace->q_rot, ws, L.q_rot, (size_t)B * Hq * kD * 4, s))) return st;
      if ((st = copy_trace(trace->q_code, ws, L.q_code, (size_t)B * Hq * cw * 4, s))) return st;
      if ((st = copy_trace(trace->bounds, ws, L.bounds, (size_t)B * Gs * maxp * 4, s))) return st;
      if ((st = copy_trace(trace->kept, ws, L.kept, (size_t)B * Gs * m_max * 4, s))) return st;
      if ((st = copy_trace(trace->kept_count, ws, L.kept_count, (size_t)B * Gs * 4, s))) return st;
    }
    return HHR_OK;
  }

  // Indexer variant (HISA).
  const int T = Hq;
  const size_t ixs = ix_smem(maxp, m_max, P);
  if ((long long)B * T <= HHR_IX_CLUSTER_MAX_QUERIES && maxp <= kIxMaxBlocks &&
      (long long)m_max * P <= kIxMaxCand && indexer_cluster_ready(ixs)) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kIxRanks, B * T);
    cfg.blockDim = dim3(kIxThreads);
    cfg.dynamicSmemBytes = ixs;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kIxRanks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    prof_begin(HHR_KERNEL_BLOCK, s);
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, indexer_cluster_kernel,
        IxArgs{q, block_mean, k_cache, page_table, seq_len, q_pos, bounds, kept, kept_count,
               reinterpret_cast<float*>(ws + L.tok), out_idx, out_count, T, P, maxp,
               d->n_phys_pages, m_pages, m_max, top_k});
    prof_end(HHR_KERNEL_BLOCK, s);
    if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
    if (trace != nullptr) {
      if ((st = copy_trace(trace->bounds, ws, L.bounds, (size_t)B * T * maxp * 4, s))) return st;
      if ((st = copy_trace(trace->kept, ws, L.kept, (size_t)B * T * m_max * 4, s))) return st;
      if ((st = copy_trace(trace->kept_count, ws, L.kept_count, (size_t)B * T * 4, s))) return st;
    }
    return HHR_OK;
  }
  float* tok = reinterpret_cast<float*>(ws + L.tok);
  if (allow_smem(block_score_kernel, block_score_smem(), g_smem_blk) != cudaSuccess)
    return HHR_ERR_CUDA;
  prof_begin(HHR_KERNEL_BLOCK, s);
  block_score_kernel<<<dim3((maxp + kBlkTile - 1) / kBlkTile, (T + kQTile - 1) / kQTile, B),
                       kBlkThreads, block_score_smem(), s>>>(
      BlockScoreArgs{q, block_mean, page_table, seq_len, q_pos, bounds, T, P, maxp,
                     d->n_phys_pages});
  prof_end(HHR_KERNEL_BLOCK, s);
  if ((st = launch_status()) != HHR_OK) return st;
  SelectArgs sb{};
  sb.scores = bounds; sb.stride = maxp; sb.rows_per_b = T; sb.seq_len = seq_len;
  sb.q_pos = q_pos; sb.P = P; sb.mode = 0; sb.m_max = m_max; sb.unit = 0;
  sb.m_pages = m_pages; sb.keep_div = 0; sb.top_k = 0;
  sb.out = kept; sb.out_stride = m_max; sb.out_count = kept_count; sb.pad_out = 0;
  cudaError_t e;
  prof_begin(HHR_KERNEL_TOPM, s);
  e = launch_pdl(select_largest_kernel, dim3(B * T), dim3(kSelThreads), (size_t)maxp * 4, s, sb);
  prof_end(HHR_KERNEL_TOPM, s);
  if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
  const int C = m_max * P;
  prof_begin(HHR_KERNEL_TOKEN, s);
  e = launch_pdl(token_score_kernel, dim3((C + kTokWarps * 32 - 1) / (kTokWarps * 32), B * T),
                 dim3(kTokWarps * 32), 0, s,
                 TokenScoreArgs{q, k_cache, page_table, seq_len, q_pos, kept, kept_count, tok, T,
                                P, maxp, d->n_phys_pages, m_max});
  prof_end(HHR_KERNEL_TOKEN, s);
  if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
  SelectArgs sc{};
  sc.scores = tok; sc.stride = C; sc.rows_per_b = T; sc.seq_len = seq_len; sc.q_pos = q_pos;
  sc.P = P; sc.mode = 1; sc.kept_count = kept_count; sc.kept_units = kept; sc.m_max = m_max;
  sc.unit = P; sc.m_pages = 0; sc.keep_div = 0; sc.top_k = top_k;
  sc.out = out_idx; sc.out_stride = top_k; sc.out_count = out_count; sc.pad_out = 1;
  prof_begin(HHR_KERNEL_TOKEN_TOPK, s);
  e = launch_pdl(select_largest_kernel, dim3(B * T), dim3(kSelThreads), (size_t)C * 4, s, sc);
  prof_end(HHR_KERNEL_TOKEN_TOPK, s);
  if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
  if (trace != nullptr) {
    if ((st = copy_trace(trace->bounds, ws, L.bounds, (size_t)B * T * maxp * 4, s))) return st;
    if ((st = copy_trace(trace->kept, ws, L.kept, (size_t)B * T * m_max * 4, s))) return st;
    if ((st = copy_trace(trace->kept_count, ws, L.kept_count, (size_t)B * T * 4, s))) return st;
  }
  return HHR_OK;
}

size_t hhr_attn_workspace_bytes(const hhr_dims* d, int top_k) {
  if (check_dims(d) != HHR_OK || check_group(d) != HHR_OK || top_k < 1) return 0;
  const AttnPlan plan = attn_plan(d->batch, sel_rows(d), top_k);
  const size_t ns = plan.n_splits;
  const size_t rows = (size_t)d->batch * sel_rows(d);
  const size_t gs = d->n_q_heads / sel_rows(d);
  return align256(rows * ns * gs * kD * 4) + align256(rows * ns * gs * 2 * 4);
}

}  // extern "C"

namespace {

// Host-side validation of the attention arguments (everything but the workspace).
int check_attn_args(const hhr_dims* d, const uint16_t* q, const uint16_t* k_cache,
                    const uint16_t* v_cache, const int32_t* page_table, const int32_t* seq_len,
                    const int32_t* idx, const int32_t* count, int top_k, float scale,
                    const float* out) {
  int st = check_dims(d);
  if (st != HHR_OK) return st;
  if ((st = check_group(d)) != HHR_OK) return st;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || page_table == nullptr ||
      seq_len == nullptr || idx == nullptr || count == nullptr || out == nullptr)
    return HHR_ERR_INVALID_ARG;
  if (top_k < 1 || !(scale == scale) || isinf(scale)) return HHR_ERR_INVALID_ARG;
  if (misaligned16({q, k_cache, v_cache, out})) return HHR_ERR_INVALID_ARG;
  // Cache rows are addressed with 32-bit row indices.
  if ((unsigned long long)d->n_phys_pages * d->n_kv_heads * d->page_size >= 0xffffffffull)
    return HHR_ERR_UNSUPPORTED;
  return HHR_OK;
}

}  // namespace

extern "C" {

int hhr_sparse_attn(const hhr_dims* d, const uint16_t* q, const uint16_t* k_cache,
                    const uint16_t* v_cache, const int32_t* page_table, const int32_t* seq_len,
                    const int32_t* idx, const int32_t* count, int top_k, float scale, float* out,
                    void* workspace, size_t ws_bytes, void* stream) {
  int st = check_attn_args(d, q, k_cache, v_cache, page_table, seq_len, idx, count, top_k,
                           scale, out);
  if (st != HHR_OK) return st;
  if (workspace == nullptr) return HHR_ERR_INVALID_ARG;
  const size_t need = hhr_attn_workspace_bytes(d, top_k);
  if (ws_bytes < need) return HHR_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255) != 0) return HHR_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const int B = d->batch, G = d->n_kv_heads, Hq = d->n_q_heads, Gs = sel_rows(d);
  const AttnPlan plan = attn_plan(B, Gs, top_k);
  const int ns = plan.n_splits;
  const int gs = Hq / Gs;
  char* ws = static_cast<char*>(workspace);
  float* part_o = reinterpret_cast<float*>(ws);
  float* part_ml = reinterpret_cast<float*>(ws + align256((size_t)B * Gs * ns * gs * kD * 4));
  AttnArgs a{q, k_cache, v_cache, page_table, seq_len, idx, count, part_o, part_ml, out,
             scale * 1.4426950408889634f, Hq, G, d->page_size, d->max_pages_per_seq,
             d->n_phys_pages, top_k, ns, plan.split_rows, nullptr, Gs, kv_div(d)};
  prof_begin(HHR_KERNEL_ATTN, s);
  if (allow_smem(sparse_attn_kernel<false>, attn_smem(), g_smem_attn) != cudaSuccess)
    return HHR_ERR_CUDA;
  sparse_attn_kernel<false><<<dim3(ns, Gs, B), kAttnThreads, attn_smem(), s>>>(a);
  prof_end(HHR_KERNEL_ATTN, s);
  if ((st = launch_status()) != HHR_OK) return st;
  if (ns > 1) {
    prof_begin(HHR_KERNEL_COMBINE, s);
    attn_combine_kernel<<<dim3(Hq, B), kD, 0, s>>>(
        CombineArgs{part_o, part_ml, count, out, Hq, Gs, top_k, ns, plan.split_rows});
    prof_end(HHR_KERNEL_COMBINE, s);
  }
  return launch_status();
}

size_t hhr_decode_step_workspace_bytes(const hhr_dims* d, int m_pages, int keep_div,
                                       int top_k) {
  const size_t sel = hhr_select_workspace_bytes(d, HHR_MODE_HASH, m_pages, keep_div, top_k);
  const size_t att = hhr_attn_workspace_bytes(d, top_k);
  if (sel == 0 || att == 0) return 0;
  // + the cache row of every selected key, handed from the selection to the attention.
  return sel + att + align256((size_t)d->batch * sel_rows(d) * top_k * 4);
}

int hhr_decode_step(const hhr_dims* d, const uint16_t* q, const uint16_t* k_new,
                    const uint16_t* v_new, uint16_t* k_cache, uint16_t* v_cache,
                    const int32_t* page_table, const int32_t* seq_len, const float* R,
                    const float* W, void* page_minmax, uint32_t* codes, int m_pages,
                    int keep_div, int top_k, const hhr_select_opts* opts, float scale,
                    int32_t* out_idx, int32_t* out_count, float* out, void* workspace,
                    size_t ws_bytes, void* stream) {
  int st = check_select_params(d, HHR_MODE_HASH, m_pages, keep_div, top_k);
  if (st != HHR_OK) return st;
  int sink = 0, local = 0;
  if ((st = read_opts(d, HHR_MODE_HASH, opts, m_pages, keep_div, &sink, &local)) != HHR_OK)
    return st;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || page_table == nullptr ||
      seq_len == nullptr || R == nullptr || W == nullptr || page_minmax == nullptr ||
      codes == nullptr || out_idx == nullptr || out_count == nullptr || out == nullptr ||
      workspace == nullptr)
    return HHR_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return HHR_ERR_INVALID_ARG;
  if (!(scale == scale) || isinf(scale)) return HHR_ERR_INVALID_ARG;
  if (misaligned16({q, k_new, v_new, k_cache, v_cache, R, W, page_minmax, codes, out}))
    return HHR_ERR_INVALID_ARG;
  if ((unsigned long long)d->n_phys_pages * d->n_kv_heads * d->page_size >= 0xffffffffull)
    return HHR_ERR_UNSUPPORTED;
  const size_t need = hhr_decode_step_workspace_bytes(d, m_pages, keep_div, top_k);
  if (need == 0) return HHR_ERR_INVALID_ARG;
  if (ws_bytes < need) return HHR_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255) != 0) return HHR_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const int B = d->batch, G = d->n_kv_heads, Hq = d->n_q_heads, P = d->page_size;
  const int Gs = sel_rows(d), rh = Hq / Gs;  // selection rows and their query heads
  const int maxp = d->max_pages_per_seq, gs = Hq / G;
  const int m_max = kept_max(d, m_pages, keep_div);
  const SelectLayout L = select_layout(d, HHR_MODE_HASH, m_max);
  char* ws = static_cast<char*>(workspace);
  float* qpn = reinterpret_cast<float*>(ws + L.qpn);
  float* q_rot = reinterpret_cast<float*>(ws + L.q_rot);
  uint32_t* q_code = reinterpret_cast<uint32_t*>(ws + L.q_code);
  float* bounds = reinterpret_cast<float*>(ws + L.bounds);
  int32_t* kept = reinterpret_cast<int32_t*>(ws + L.kept);
  int32_t* kept_count = reinterpret_cast<int32_t*>(ws + L.kept_count);
  char* aws = ws + L.total;
  const AttnPlan plan = attn_plan(B, Gs, top_k);
  const int ns = plan.n_splits;
  float* part_o = reinterpret_cast<float*>(aws);
  float* part_ml = reinterpret_cast<float*>(aws + align256((size_t)B * Gs * ns * rh * kD * 4));
  uint32_t* row_buf = reinterpret_cast<uint32_t*>(aws + hhr_attn_workspace_bytes(d, top_k));
  const int cw = code_words(d);
  const bool flat = m_max >= maxp;
  const size_t fsm = topm_hamming_smem(rh, cw, m_max, P, maxp);
  const int nt = topm_hamming_threads(cw, (long long)B * Gs * kHamRanks, sm_count());
  if (allow_smem(topm_hamming_for(rh, cw, nt), fsm,
                 g_smem_ham[cw_index(cw)][nt == 512][hamming_planes(rh) - 1]) != cudaSuccess)
    return HHR_ERR_CUDA;
  if (allow_smem(sparse_attn_kernel<false>, attn_smem(), g_smem_attn) != cudaSuccess)
    return HHR_ERR_CUDA;
  if (allow_smem(sparse_attn_kernel<true>, attn_smem(), g_smem_attn_cl) != cudaSuccess)
    return HHR_ERR_CUDA;
  cudaError_t e;

  // a0 + a1: append and encode the newest key rows, rotate and encode the queries. The staged
  // bound kernel that follows starts each CTA at the beginning of its chunk range: the
  // prologue prefetches those first units into L2 (about kWarmBytes in all; not when an event
  // brackets the bound kernel, whose duration is then that of a cold L2).
  int warm_units = 0, warm_ctas = 0;
  const bool staged = HHR_BOUND_STAGE && B <= kStageMaxBatch &&
                      stage_slots(G, d->summary_fp16 != 0) >= 2;
  const int ub = stage_unit_bytes(G, d->summary_fp16 != 0);
  if (!flat && staged && B <= 64 && g_prof[HHR_KERNEL_BOUND].start == nullptr) {
    warm_ctas = sm_count();
    warm_units = (int)min((size_t)kStageChunk * 64, kWarmBytes / ((size_t)warm_ctas * ub));
  }
  prof_begin(HHR_KERNEL_ENCODE, s);
  step_prologue_for(gs, cw)<<<dim3(kPrologueRanks, G, B), kPrologueThreads, 0, s>>>(
      PrologueArgs{q, k_new, v_new, k_cache, v_cache, page_table, seq_len, R, W, page_minmax,
                   codes, q_rot, q_code, qpn, Hq, G, P, maxp, d->n_phys_pages,
                   d->summary_fp16, warm_units, warm_ctas, ub, kStageChunk});
  prof_end(HHR_KERNEL_ENCODE, s);
  if ((st = launch_status()) != HHR_OK) return st;
  const BoundArgs ba{qpn, q_rot, page_minmax, page_table, seq_len, bounds, G, P, maxp,
                     d->n_phys_pages, 0, Gs, kv_div(d), B};
  HammingArgs ha{q_code, codes, page_table, seq_len, kept, kept_count, out_idx, out_count,
                 Hq, G, P, maxp, d->n_phys_pages, m_max, top_k, row_buf, sink, local,
                 Gs, kv_div(d)};
  ha.pf_k = k_cache;
  ha.pf_v = v_cache;
  const float scale_log2 = scale * 1.4426950408889634f;
  // a2-a5 of small batches: one cluster per selection row.
  {
    const RowPlan rp = row_plan(d, m_max, top_k);
    if (rp.use) {
      ha.pf_split = rp.attn.split_rows;
      const AttnArgs aa{q, k_cache, v_cache, page_table, seq_len, out_idx, out_count, nullptr,
                        nullptr, out, scale_log2, Hq, G, P, maxp, d->n_phys_pages, top_k,
                        rp.attn.n_splits, rp.attn.split_rows, row_buf, Gs, kv_div(d)};
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(rp.ranks * B * Gs);
      cfg.blockDim = dim3(kRowThreads);
      cfg.dynamicSmemBytes = rp.smem;
      cfg.stream = s;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = rp.ranks;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 2;
      prof_begin(HHR_KERNEL_ROW, s);
      e = cudaLaunchKernelEx(&cfg, rp.fn,
                             RowClusterArgs{ba, TopmHammingArgs{ha, bounds, m_pages, keep_div,
                                                                flat ? 1 : 0},
                                            aa, kv_div(d) > 1 ? 1 : 0});
      prof_end(HHR_KERNEL_ROW, s);
      if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
      return HHR_OK;
    }
  }
  // a2: page bounds (none when every page is kept: a flat hash top-k).
  if (!flat) {
    // Launched behind the prologue. With f32 summaries (page_bound_kernel) its first CTAs
    // warm L2 while the prologue runs, unless an event is recorded between the two
    // (profiling), which leaves no overlap to use.
    BoundArgs bw = ba;
    bw.early = g_prof[HHR_KERNEL_BOUND].start != nullptr ? 0 : 3 * sm_count();
    prof_begin(HHR_KERNEL_BOUND, s);
    e = launch_bounds_kernel(d, bw, true, s);
    prof_end(HHR_KERNEL_BOUND, s);
    if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
  }
  // a2 top-m + a3 + a4: kept pages, Hamming distances, deterministic top-k.
  {
    const AttnPlan cp = attn_plan(B, Gs, top_k, kMaxClusterSplits);
    ha.pf_split = cp.n_splits <= kMaxClusterSplits ? cp.split_rows : plan.split_rows;
    prof_begin(HHR_KERNEL_HAMMING, s);
    e = launch_pdl(topm_hamming_for(rh, cw, nt), dim3(B * Gs * kHamRanks), dim3(nt), fsm, s,
                   TopmHammingArgs{ha, bounds, m_pages, keep_div, flat ? 1 : 0});
    prof_end(HHR_KERNEL_HAMMING, s);
    if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
  }
  // a5: sparse attention over the selected rows. The splits of a group form a cluster
  // merged through distributed shared memory when they fit one (at most 8 splits).
  {
    const AttnPlan cp = attn_plan(B, Gs, top_k, kMaxClusterSplits);
    if (cp.n_splits <= kMaxClusterSplits) {
      AttnArgs aa{q, k_cache, v_cache, page_table, seq_len, out_idx, out_count, nullptr, nullptr,
                  out, scale * 1.4426950408889634f, Hq, G, P, maxp, d->n_phys_pages, top_k,
                  cp.n_splits, cp.split_rows, row_buf, Gs, kv_div(d)};
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(cp.n_splits, Gs, B);
      cfg.blockDim = dim3(kAttnThreads);
      cfg.dynamicSmemBytes = attn_smem();
      cfg.stream = s;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cp.n_splits;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 2;
      prof_begin(HHR_KERNEL_ATTN, s);
      e = cudaLaunchKernelEx(&cfg, sparse_attn_kernel<true>, aa);
      prof_end(HHR_KERNEL_ATTN, s);
      if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
    } else {
      AttnArgs aa{q, k_cache, v_cache, page_table, seq_len, out_idx, out_count, part_o, part_ml,
                  out, scale * 1.4426950408889634f, Hq, G, P, maxp, d->n_phys_pages, top_k, ns,
                  plan.split_rows, row_buf, Gs, kv_div(d)};
      prof_begin(HHR_KERNEL_ATTN, s);
      e = launch_pdl(sparse_attn_kernel<false>, dim3(ns, Gs, B), dim3(kAttnThreads), attn_smem(),
                     s, aa);
      prof_end(HHR_KERNEL_ATTN, s);
      if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
      if (ns > 1) {
        prof_begin(HHR_KERNEL_COMBINE, s);
        e = launch_pdl(attn_combine_kernel, dim3(Hq, B), dim3(kD), 0, s,
                       CombineArgs{part_o, part_ml, out_count, out, Hq, Gs, top_k, ns,
                                   plan.split_rows});
        prof_end(HHR_KERNEL_COMBINE, s);
        if (e != cudaSuccess) { g_last_cuda = e; return HHR_ERR_CUDA; }
      }
    }
  }
  return HHR_OK;
}

int hhr_decode_step_kernels(const hhr_dims* d, int m_pages, int keep_div, int top_k) {
  const int st = check_select_params(d, HHR_MODE_HASH, m_pages, keep_div, top_k);
  if (st != HHR_OK) return st;
  const int m_max = kept_max(d, m_pages, keep_div);
  if (row_plan(d, m_max, top_k).use) return 2;
  const bool flat = m_max >= d->max_pages_per_seq;
  const int ns = attn_plan(d->batch, sel_rows(d), top_k).n_splits;
  const bool cluster = attn_plan(d->batch, sel_rows(d), top_k, kMaxClusterSplits).n_splits <=
                       kMaxClusterSplits;
  return 2 + (flat ? 0 : 1) + (cluster || ns == 1 ? 1 : 2);
}

int hhr_read_device_status(void* stream, int* bits) {
  cudaStream_t s = (cudaStream_t)stream;
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return HHR_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HHR_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return HHR_ERR_CUDA;
  }
  if (bits != nullptr) *bits = v;
  return v == 0 ? HHR_OK : HHR_ERR_DEVICE_STATUS;
}

// ---------------------------------------------------------------------------
// Allocation-free attention: the split-K partials live in a fixed device array.
//
// For callers that cannot allocate device memory at call time (for example an
// allocator-less runtime, code that runs while a memory pool is frozen, or a
// host that is not allowed to call cudaMalloc on its own), this variant takes
// no workspace. Its scratch is the file-scope array below, which every GPU that
// loads the library holds until the process exits. Host code cannot pass the
// array's name to a kernel (in host code it names a host-side shadow, not device
// memory), so every call looks up the array's device address with
// cudaGetSymbolAddress in the current device's context: a host-side lookup once the
// first call on that device has loaded the library's device code there, and right
// after a device reset or in another context too, which a cached address would not be.
}  // extern "C"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

}  // namespace

extern "C" {

int hhr_sparse_attn_noalloc(const hhr_dims* d, const uint16_t* q, const uint16_t* k_cache,
                            const uint16_t* v_cache, const int32_t* page_table,
                            const int32_t* seq_len, const int32_t* idx, const int32_t* count,
                            int top_k, float scale, float* out, void* stream) {
  // Size check first: the partials must fit in the fixed array. Then the other arguments,
  // all before any CUDA call.
  const size_t need = hhr_attn_workspace_bytes(d, top_k);
  if (need == 0) {
    int st = check_dims(d);
    if (st != HHR_OK) return st;
    if ((st = check_group(d)) != HHR_OK) return st;
    return HHR_ERR_INVALID_ARG;
  }
  if (need > kNoAllocScratchBytes) return HHR_ERR_WORKSPACE;
  const int st = check_attn_args(d, q, k_cache, v_cache, page_table, seq_len, idx, count, top_k,
                                 scale, out);
  if (st != HHR_OK) return st;
  void* scratch = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
  if (e != cudaSuccess || scratch == nullptr) {
    g_last_cuda = e != cudaSuccess ? e : cudaErrorInvalidSymbol;
    return HHR_ERR_CUDA;
  }
  // The partials are written by the chunk kernel before the merge kernel reads
  // them (same stream), so nothing in the array has to start at zero.
  return hhr_sparse_attn(d, q, k_cache, v_cache, page_table, seq_len, idx, count, top_k, scale,
                         out, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
