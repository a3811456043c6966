// Steps a1-a4: query preparation, page-level bounds, top-m, Hamming scan and top-k
// (HHR), and the block filter + token refinement of the indexer variant (HISA).
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "encode.cuh"

namespace hhr {

// ---------------------------------------------------------------------------- a1
// HHR page, Abstract (queries are rotated by the same R_h and encoded like keys).
// One CTA of kMvThreads threads per (KV group, sequence). For each query head of the
// group: q' = R_g q, code bits = [W_g q' > 0] (row_dot16: the 16 threads of row r own
// channel and bit r). Also folds the group into the two bound vectors
//   qneg_c = sum_h min(q'_hc, 0),  qpos_c = sum_h max(q'_hc, 0),
// so that sum_h max(q'_hc*kmin_c, q'_hc*kmax_c) = qneg_c*kmin_c + qpos_c*kmax_c
// (kmin <= kmax: a positive q' picks kmax, a negative one kmin). The page bound
// then becomes one 256-long dot product per page.
struct QPrepArgs {
  const uint16_t* q;
  const float* R;
  const float* W;
  float* q_rot;      // [B][Hq][d]
  uint32_t* q_code;  // [B][Hq][CW]
  float* qpn;        // [B][G][2][d]: [0] = qneg, [1] = qpos
  int Hq, G;
};

template <int CW>
__global__ void __launch_bounds__(kMvThreads) qprep_kernel(QPrepArgs a) {
  __shared__ __align__(16) float qx[kMaxGroup][kD];
  __shared__ __align__(16) float qr[kMaxGroup][kD];
  __shared__ uint32_t cword[kMaxGroup][CW];
  const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int lrow = mv_lrow();
  const bool row_lead = mv_part() == 0;
  const int gs = a.Hq / a.G;
  // R_g and W_g rows of this thread are fetched up front (one memory latency for both).
  float4 rrow[kRowBlocks][2], wrow[CW][2];
#pragma unroll
  for (int rb = 0; rb < kRowBlocks; ++rb) load_row16(a.R + (size_t)g * kD * kD, rb * 32 + lrow, rrow[rb]);
#pragma unroll
  for (int wb = 0; wb < CW; ++wb)
    load_row16(a.W + (size_t)g * (32 * CW) * kD, wb * 32 + lrow, wrow[wb]);
  for (int i = tid; i < kMaxGroup * kD; i += kMvThreads) {
    const int h = i / kD, c = i % kD;
    qx[h][c] = h < gs ? bf16_to_f(a.q[((size_t)b * a.Hq + g * gs + h) * kD + c]) : 0.f;
  }
  if (tid < kMaxGroup * CW) cword[tid / CW][tid % CW] = 0u;
  __syncthreads();
  float qneg[kRowBlocks], qpos[kRowBlocks];
#pragma unroll
  for (int rb = 0; rb < kRowBlocks; ++rb) {
    qneg[rb] = 0.f;
    qpos[rb] = 0.f;
    for (int h = 0; h < gs; ++h) {
      const float y = row_dot16(rrow[rb], &qx[h][0]);
      qneg[rb] += fminf(y, 0.f);
      qpos[rb] += fmaxf(y, 0.f);
      if (row_lead) {
        qr[h][rb * 32 + lrow] = y;
        a.q_rot[((size_t)b * a.Hq + g * gs + h) * kD + rb * 32 + lrow] = y;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int wb = 0; wb < CW; ++wb) {
    for (int h = 0; h < gs; ++h) {
      const float p = row_dot16(wrow[wb], &qr[h][0]);
      if (row_lead && p > 0.f) atomicOr(&cword[h][wb], 1u << lrow);
    }
  }
  __syncthreads();
  if (tid < gs * CW) {
    const int h = tid / CW, w = tid % CW;
    a.q_code[((size_t)b * a.Hq + g * gs + h) * CW + w] = cword[h][w];
  }
  if (row_lead) {
    float* o = a.qpn + ((size_t)b * a.G + g) * 2 * kD;
#pragma unroll
    for (int rb = 0; rb < kRowBlocks; ++rb) {
      o[rb * 32 + lrow] = qneg[rb];
      o[kD + rb * 32 + lrow] = qpos[rb];
    }
  }
}

inline size_t qprep_smem() { return 0; }

// ---------------------------------------------------------------------------- a2
// HHR page, Abstract: page-level logit bounds of the rotated keys prune pages.
// bound_p = qneg . kmin_p + qpos . kmax_p over the page summary (1 KB per page and
// group in f32, 512 B in f16). The summaries are the dominant HBM stream of the whole
// path, so this kernel is a pure streaming GEMV.
// Tuned on B200 at 128K context, batch 8 (4096 pages x 8 groups x 8 sequences); the
// macros below exist for such sweeps.

#ifndef HHR_BOUND_WARPS
#define HHR_BOUND_WARPS 4
#endif
#ifndef HHR_BOUND_SETS_F16
#define HHR_BOUND_SETS_F16 2
#endif
#ifndef HHR_BOUND_SETS_F32
#define HHR_BOUND_SETS_F32 2
#endif
constexpr int kBoundWarps = HHR_BOUND_WARPS;

// Grid of the bound kernels: (page chunk, group, sequence), or (group, page chunk,
// sequence) when HHR_BOUND_GROUP_FAST is set.
#ifdef HHR_BOUND_GROUP_FAST
__device__ __forceinline__ int bound_group_of(int x, int y) { return x; }
__device__ __forceinline__ int bound_chunk_of(int x, int y) { return y; }
inline dim3 bound_grid(int G, int chunks, int B) { return dim3(G, chunks, B); }
#else
__device__ __forceinline__ int bound_group_of(int x, int y) { return y; }
__device__ __forceinline__ int bound_chunk_of(int x, int y) { return x; }
inline dim3 bound_grid(int G, int chunks, int B) { return dim3(chunks, G, B); }
#endif
__device__ __forceinline__ int bound_group() { return bound_group_of(blockIdx.x, blockIdx.y); }
__device__ __forceinline__ int bound_chunk() { return bound_chunk_of(blockIdx.x, blockIdx.y); }

// L2 warm-up before the dependency wait: with programmatic launch the first CTAs of the
// bound kernel are resident while the previous kernel (the fused step's prologue) still
// runs and HBM idles. The first E = BoundArgs::early CTAs (by linear index) prefetch the
// summaries of CTAs lin, lin + E, ..., lin + (HHR_BOUND_LOOKAHEAD - 1) E into L2. Measured
// on B200 (128K context, batch 8, f16): E = 3 x 148 SMs and 3 strides (about 44 MB, what
// HBM can move during the prologue) take 2 us off the step; more lookahead is slower.
#ifndef HHR_BOUND_LOOKAHEAD
#define HHR_BOUND_LOOKAHEAD 3
#endif

struct BoundArgs {
  const float* qpn;         // [B][G][2][d] folded group queries (rows are KV groups)
  const float* q_rot;       // [B][Hq][d] rotated queries (rows are query heads: folded here)
  const void* page_minmax;  // f32 or f16 [n_phys][G][2][d]
  const int32_t* page_table;
  const int32_t* seq_len;
  float* bounds;  // [B][Gs][maxp]
  int G, P, maxp, n_phys;
  int early;      // CTAs that warm L2 before the dependency wait (0: none)
  int Gs, kv_div; // selection rows per sequence (G, or Hq per head); row r uses KV head r / kv_div
  int batch;      // B
};

// Sum over the warp of 8 per-lane partials (one per page): a butterfly over lane bits 4
// and 3, then a transposition over bits 2..0; lane l ends with the total of page l & 7.
__device__ __forceinline__ float warp_sum8_transposed(float (&v)[8], int lane) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] += __shfl_xor_sync(kFull, v[i], 16);
    v[i] += __shfl_xor_sync(kFull, v[i], 8);
  }
#pragma unroll
  for (int s = 4; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, s);
    }
  }
  return v[0];
}

// One warp per page and load instruction (coalesced: lane l reads 16-byte piece l of the
// page's summary); each warp loads 16 pages (two sets of 8) before any arithmetic and
// folds each set of 8 page sums with one transposed reduction. f32 pages are 1 KB (two
// pieces per lane: channels 4l..4l+3 of the min and of the max row); f16 pages are 512 B
// (one piece: lanes 0-15 hold 8 channels of the min row, lanes 16-31 of the max row).
// Each piece is paired with the matching channels of the folded query (qneg with min,
// qpos with max). Measured on B200 (128K context, batch 8): 16 pages per warp and 4 warps
// per CTA stream fastest (f32 6.25 TB/s, f16 5.07 TB/s); 8 or 24+ pages per warp are slower.
__device__ __forceinline__ float dot8_h(const uint4 h, const float4 q0, const float4 q1) {
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
  const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&h.z));
  const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&h.w));
  return q0.x * a.x + q0.y * a.y + q0.z * b.x + q0.w * b.y + q1.x * c.x + q1.y * c.y +
         q1.z * d.x + q1.w * d.y;
}

// f16 summaries saturate to -inf (min row) or +inf (max row) beyond the f16 range. A folded
// query component that is exactly 0 (no head of the group on that side) then meets an
// infinite summary and 0 * inf is NaN, while that channel's true contribution is 0 for every
// key of the page. dot8_h is NaN exactly in that case (every other product is finite or
// +inf: qneg <= 0 pairs with kmin, which only saturates to -inf, and qpos >= 0 with kmax,
// which only saturates to +inf), and this slow path recomputes it with those terms at 0.
__device__ __forceinline__ float dot8_h_zero_guarded(const uint4 h, const float4 q0,
                                                  const float4 q1) {
  const float q[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
  const uint32_t w[4] = {h.x, h.y, h.z, h.w};
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 k = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    s += q[2 * i] == 0.f ? 0.f : q[2 * i] * k.x;
    s += q[2 * i + 1] == 0.f ? 0.f : q[2 * i + 1] * k.y;
  }
  return s;
}

// 16-byte summary load; the variant is a build-time choice (streaming by default).
#ifndef HHR_BOUND_LOAD
#define HHR_BOUND_LOAD 0
#endif
__device__ __forceinline__ uint4 load_summary16(const uint4* p) {
#if HHR_BOUND_LOAD == 0
  return __ldcs(p);
#elif HHR_BOUND_LOAD == 1
  return __ldg(p);
#elif HHR_BOUND_LOAD == 2
  return *p;
#else
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
#endif
}

// The folded query of selection row r of sequence b, as the lane's halves of the two bound
// vectors (qneg paired with kmin, qpos with kmax): 8 channels of qneg (lanes 0-15) or qpos
// (lanes 16-31) for f16 summaries, channels 4l..4l+3 of both for f32. per_head: the row is one
// query head, folded here from its rotated query (qneg = min(q', 0), qpos = max(q', 0)).
template <bool F16>
__device__ __forceinline__ void bound_query(const BoundArgs& a, int b, int r, bool per_head,
                                            int lane, float4& q0, float4& q1) {
  if (!per_head) {
    const float* qb = a.qpn + ((size_t)b * a.Gs + r) * 2 * kD;
    if constexpr (F16) {
      const float4* qv = reinterpret_cast<const float4*>(qb + (lane >> 4) * kD + 8 * (lane & 15));
      q0 = qv[0];
      q1 = qv[1];
    } else {
      q0 = reinterpret_cast<const float4*>(qb)[lane];
      q1 = reinterpret_cast<const float4*>(qb + kD)[lane];
    }
  } else {
    const float* qh = a.q_rot + ((size_t)b * a.Gs + r) * kD;
    auto lo = [](float4 v) { return make_float4(fminf(v.x, 0.f), fminf(v.y, 0.f), fminf(v.z, 0.f), fminf(v.w, 0.f)); };
    auto hi = [](float4 v) { return make_float4(fmaxf(v.x, 0.f), fmaxf(v.y, 0.f), fmaxf(v.z, 0.f), fmaxf(v.w, 0.f)); };
    if constexpr (F16) {
      const float4* qv = reinterpret_cast<const float4*>(qh + 8 * (lane & 15));
      q0 = lane < 16 ? lo(qv[0]) : hi(qv[0]);
      q1 = lane < 16 ? lo(qv[1]) : hi(qv[1]);
    } else {
      const float4 v = reinterpret_cast<const float4*>(qh)[lane];
      q0 = lo(v);
      q1 = hi(v);
    }
  }
}

// One warp's share of the page bounds of selection row r (KV head g) of sequence b: pages
// [p0, p0 + kPagesPerWarp) (those below npg), written to a.bounds (-inf and a status bit for a
// page id outside the pool). All page ids are loaded first, then all summary pieces, so that
// the warp keeps kPagesPerWarp page summaries in flight.
template <bool F16>
__device__ __forceinline__ void bound_warp(const BoundArgs& a, int b, int r, int g, int p0,
                                           int npg, int lane, float4 q0, float4 q1) {
  constexpr int kSets = F16 ? HHR_BOUND_SETS_F16 : HHR_BOUND_SETS_F32;
  constexpr int kPagesPerWarp = 8 * kSets;
  constexpr int kPieces = F16 ? 32 : 64;
  const uint4* base4 = reinterpret_cast<const uint4*>(a.page_minmax);
  int my_phys = -1;  // lane i < kPagesPerWarp resolves page p0 + i
  if (lane < kPagesPerWarp && p0 + lane < npg)
    my_phys = a.page_table[(size_t)b * a.maxp + p0 + lane];
  uint4 x[kPagesPerWarp], y[F16 ? 1 : kPagesPerWarp];
#pragma unroll
  for (int i = 0; i < kPagesPerWarp; ++i) {
    const int phys = __shfl_sync(kFull, my_phys, i);
    x[i] = make_uint4(0, 0, 0, 0);
    if constexpr (!F16) y[i] = x[i];
    if (phys >= 0 && phys < a.n_phys) {
      const uint4* src = base4 + ((size_t)phys * a.G + g) * kPieces + lane;
      x[i] = load_summary16(src);
      if constexpr (!F16) y[i] = load_summary16(src + 32);
    }
  }
  float* out = a.bounds + ((size_t)b * a.Gs + r) * a.maxp;
#pragma unroll
  for (int st = 0; st < kSets; ++st) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if constexpr (F16) {
        v[i] = dot8_h(x[st * 8 + i], q0, q1);
      } else {
        const float4 mn = *reinterpret_cast<const float4*>(&x[st * 8 + i]);
        const float4 mx = *reinterpret_cast<const float4*>(&y[st * 8 + i]);
        v[i] = q0.x * mn.x + q0.y * mn.y + q0.z * mn.z + q0.w * mn.w + q1.x * mx.x +
               q1.y * mx.y + q1.z * mx.z + q1.w * mx.w;
      }
    }
    float tot = warp_sum8_transposed(v, lane);
    if constexpr (F16) {
      // Rare: a NaN total (a zero folded query component met a saturated summary). The
      // page's pieces are loaded again and summed with those terms at 0.
      unsigned nan_pages = __ballot_sync(kFull, lane < 8 && tot != tot);
      while (nan_pages != 0u) {
        const int l = __ffs(nan_pages) - 1;
        nan_pages &= nan_pages - 1u;
        const int phys = __shfl_sync(kFull, my_phys, st * 8 + l);
        const uint4 piece = load_summary16(base4 + ((size_t)phys * a.G + g) * kPieces + lane);
        const float s = warp_sum(dot8_h_zero_guarded(piece, q0, q1));
        if (lane == l) tot = s;
      }
    }
    // Lane l (< 8) holds the bound of page p0 + st*8 + l; its page id is on lane st*8 + l.
    const int phys_l = __shfl_sync(kFull, my_phys, (st * 8 + lane) & 31);
    const int lp = p0 + st * 8 + lane;
    if (lane < 8 && lp < npg) {
      const bool ok = phys_l >= 0 && phys_l < a.n_phys;
      if (!ok) flag_status(kStatusBadPage);
      out[lp] = ok ? tot : -INFINITY;
    }
  }
}


// Page bounds from summaries staged page-major in shared memory by bulk copies. A unit is
// one physical page's summaries of every KV group, G x 2 x d values stored contiguously
// (G x 512 B in f16, G x 1 KB in f32), so one 1-D bulk copy (cp.async.bulk, global -> this
// CTA's shared memory, no multicast) moves it. A persistent CTA (one per SM) has one
// producer warp and kStageConsumers consumer warps around a ring of unit slots: the producer
// issues each unit's copy into the next free slot (its "empty" mbarrier) and the copy
// completes on the slot's "full" mbarrier; consumer warp w folds units w, w + kStageConsumers,
// ... of the CTA's stream into the bounds of every selection row of the unit's sequence (a
// row reads its KV group's summary), with the arithmetic of bound_warp on the same 16-byte
// pieces per lane, so the bounds are bit-identical; then it hands the slot back.
// Work: chunks of kStageChunk consecutive pages of a sequence (every sequence's chunks below
// its page count, sequences in order); CTA c takes a contiguous range of chunks.
constexpr int kStageThreads = 512;
constexpr int kStageConsumers = kStageThreads / 32 - 1;
constexpr int kStageChunk = 16;
constexpr int kStageMaxSlots = 256;
constexpr int kStageMaxBatch = 4096;  // sequences whose chunk prefix fits in shared memory
constexpr size_t kStageRingBytes = 192 * 1024;
constexpr long long kStageWaitLimit = 1ll << 24;

__host__ __device__ inline int stage_unit_bytes(int G, bool f16) { return G * 2 * kD * (f16 ? 2 : 4); }
inline int stage_slots(int G, bool f16) {
  const int n = (int)(kStageRingBytes / (size_t)stage_unit_bytes(G, f16));
  return n < kStageMaxSlots ? n : kStageMaxSlots;
}
// Dynamic shared memory: the slots, their full and empty mbarriers, their page ids, and the
// chunk prefix over the sequences.
inline size_t stage_smem(int G, bool f16, int B) {
  const int S = stage_slots(G, f16);
  return (size_t)S * stage_unit_bytes(G, f16) + (size_t)S * 16 + (size_t)S * 4 +
         (size_t)(2 * B + 1) * 4 + 16;
}

template <bool F16>
__global__ void __launch_bounds__(kStageThreads, 1) page_bound_stage_kernel(BoundArgs a, int S) {
  extern __shared__ __align__(16) unsigned char st_smem[];
  constexpr int Q = kStageChunk;
  constexpr int kAhead = 4;  // producer batches whose page ids are loaded ahead
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int B = a.batch, G = a.G;
  const int ub = stage_unit_bytes(G, F16);
  unsigned char* slots = st_smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(st_smem + (size_t)S * ub);
  uint64_t* empty = full + S;
  int* slot_phys = reinterpret_cast<int*>(empty + S);
  int* cpre = slot_phys + S;  // [B + 1] chunks of the sequences before b
  int* npgs = cpre + B + 1;   // [B] pages of sequence b
  for (int i = threadIdx.x; i < S; i += kStageThreads) {
    mbar_init(smem_u32(full + i), 1);
    mbar_init(smem_u32(empty + i), 1);
  }
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  // Page counts and chunk prefix (the lengths are inputs: read before the dependency wait).
  if (warp == 0) {
    int run = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      const int np = b < B ? min(ceil_div(max(a.seq_len[b], 0), a.P), a.maxp) : 0;
      const int nc = ceil_div(np, Q);
      const int incl = warp_incl_scan(nc, lane);
      if (b < B) {
        cpre[b] = run + incl - nc;
        npgs[b] = np;
      }
      run += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) cpre[B] = run;
  }
  __syncthreads();
  const int C = cpre[B];
  const int c0 = (int)((long long)blockIdx.x * C / gridDim.x);
  const int c1 = (int)((long long)(blockIdx.x + 1) * C / gridDim.x);
  const int n_units = (c1 - c0) * Q;
  // Unit j of this CTA: sequence b and page p (a unit at p >= npgs[b] is past the end).
  auto unit = [&](int j, int& b, int& p) {
    const int id = c0 + j / Q;
    int lo = 0, hi = B - 1;  // the last b with cpre[b] <= id
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cpre[mid] <= id) lo = mid; else hi = mid - 1;
    }
    b = lo;
    p = (id - cpre[b]) * Q + j % Q;
  };
  if (warp == 0) {
    // Producer: lane l < PB takes units j0 + l of every batch; -1 marks a unit past its
    // sequence's end, -2 a page id outside the pool (no copy for either). PB <= S keeps the
    // lanes of one batch on distinct slots, so no lane waits for a slot that another lane of
    // its batch must fill. Page ids are loaded kAhead batches ahead (the page table is an
    // input: the first ones before the dependency wait).
    const int PB = S < 32 ? S : 32;
    auto page_id = [&](int j) {
      int phys = -1;
      if (lane < PB && j < n_units) {
        int b, p;
        unit(j, b, p);
        if (p < npgs[b]) {
          phys = a.page_table[(size_t)b * a.maxp + p];
          if (phys < 0 || phys >= a.n_phys) phys = -2;
        }
      }
      return phys;
    };
    int ahead[kAhead];
#pragma unroll
    for (int t = 0; t < kAhead; ++t) ahead[t] = page_id(t * PB + lane);
    pdl_wait();
    pdl_trigger();
    for (int j0 = 0, t = 0; j0 < n_units; j0 += PB, ++t) {
      const int phys = ahead[0];
#pragma unroll
      for (int u = 0; u + 1 < kAhead; ++u) ahead[u] = ahead[u + 1];
      ahead[kAhead - 1] = page_id(j0 + kAhead * PB + lane);
      const int j = j0 + lane;
      if (lane < PB && j < n_units) {
        const int slot = j % S;
        if (!mbar_wait_bounded(smem_u32(empty + slot), ((j / S) & 1) ^ 1, kStageWaitLimit))
          flag_status(kStatusWaitGaveUp);
        slot_phys[slot] = phys;
        mbar_arrive_expect_tx(smem_u32(full + slot), phys >= 0 ? (uint32_t)ub : 0u);
        if (phys >= 0)
          bulk_g2s(smem_u32(slots + (size_t)slot * ub),
                   static_cast<const unsigned char*>(a.page_minmax) + (size_t)phys * ub,
                   (uint32_t)ub, smem_u32(full + slot));
      }
    }
    return;
  }
  pdl_wait();
  pdl_trigger();
  // Consumers. The folded queries of up to 8 rows of the current sequence stay in registers.
  constexpr int kPiece = F16 ? 512 : 1024;  // bytes of one KV group's summary
  const bool per_head = a.kv_div > 1;
  const bool cache_q = a.Gs <= 8;
  float4 qc0[8], qc1[8];
  int qb = -1;
  for (int j = warp - 1; j < n_units; j += kStageConsumers) {
    const int slot = j % S;
    int b, p;
    unit(j, b, p);
    if (cache_q && b != qb) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i < a.Gs) bound_query<F16>(a, b, i, per_head, lane, qc0[i], qc1[i]);
      qb = b;
    }
    if (!mbar_wait_bounded(smem_u32(full + slot), (j / S) & 1, kStageWaitLimit) && lane == 0)
      flag_status(kStatusWaitGaveUp);
    const int phys = slot_phys[slot];
    const unsigned char* u = slots + (size_t)slot * ub;
    if (phys != -1) {
      for (int r0 = 0; r0 < a.Gs; r0 += 8) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = r0 + i;
          v[i] = 0.f;
          if (r < a.Gs && phys >= 0) {
            float4 q0, q1;
            if (cache_q) {
              q0 = qc0[i];
              q1 = qc1[i];
            } else {
              bound_query<F16>(a, b, r, per_head, lane, q0, q1);
            }
            const unsigned char* gp = u + (size_t)(a.kv_div == 1 ? r : r / a.kv_div) * kPiece;
            if constexpr (F16) {
              v[i] = dot8_h(*reinterpret_cast<const uint4*>(gp + lane * 16), q0, q1);
            } else {
              const float4 mn = *reinterpret_cast<const float4*>(gp + lane * 16);
              const float4 mx = *reinterpret_cast<const float4*>(gp + 512 + lane * 16);
              v[i] = q0.x * mn.x + q0.y * mn.y + q0.z * mn.z + q0.w * mn.w + q1.x * mx.x +
                     q1.y * mx.y + q1.z * mx.z + q1.w * mx.w;
            }
          }
        }
        float tot = warp_sum8_transposed(v, lane);
        if constexpr (F16) {
          // Rare: a NaN total (a zero folded query component met a saturated summary): the
          // row is summed again with those terms at 0.
          unsigned nan_rows = __ballot_sync(kFull, lane < 8 && tot != tot);
          while (nan_rows != 0u) {
            const int l = __ffs(nan_rows) - 1;
            nan_rows &= nan_rows - 1u;
            const int r = r0 + l;
            float4 q0, q1;
            bound_query<F16>(a, b, r, per_head, lane, q0, q1);
            const unsigned char* gp = u + (size_t)(a.kv_div == 1 ? r : r / a.kv_div) * kPiece;
            const float sum = warp_sum(
                dot8_h_zero_guarded(*reinterpret_cast<const uint4*>(gp + lane * 16), q0, q1));
            if (lane == l) tot = sum;
          }
        }
        const int r = r0 + lane;
        if (lane < 8 && r < a.Gs) {
          if (phys == -2 && r == 0) flag_status(kStatusBadPage);
          a.bounds[((size_t)b * a.Gs + r) * a.maxp + p] = phys >= 0 ? tot : -INFINITY;
        }
      }
    }
    // The unit's shared-memory reads are complete (their values are folded): hand the slot
    // back for its next bulk copy.
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(empty + slot));
  }
}

// PH: one query head per selection row (per-head selection), folded here from q_rot.
template <bool F16, bool PH = false>
__global__ void __launch_bounds__(kBoundWarps * 32) page_bound_kernel(BoundArgs a) {
  // kSets groups of 8 pages per warp are loaded together (all page ids first, then all
  // summary pieces), so that each warp keeps kSets * 8 page summaries in flight.
  constexpr int kSets = F16 ? HHR_BOUND_SETS_F16 : HHR_BOUND_SETS_F32;
  constexpr int kPagesPerWarp = 8 * kSets;
  // A page's summary in units of 16-byte pieces: 64 (f32) or 32 (f16).
  constexpr int kPieces = F16 ? 32 : 64;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if constexpr (HHR_BOUND_LOOKAHEAD > 0) {
    // Reads only inputs no earlier kernel of the step writes (page table, lengths); a
    // prefetch of a summary that the previous kernel is updating is coherent in L2.
    const int lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    const int total = gridDim.x * gridDim.y * gridDim.z;
    if (lin < a.early && lane < kPagesPerWarp) {
#pragma unroll
      for (int j = 0; j < HHR_BOUND_LOOKAHEAD; ++j) {
        const int t = lin + j * a.early;
        if (t < total) {
          const int tx = t % gridDim.x, ty = (t / gridDim.x) % gridDim.y;
          const int tb = t / (gridDim.x * gridDim.y);
          const int tg = bound_group_of(tx, ty);
          const int p = bound_chunk_of(tx, ty) * kBoundWarps * kPagesPerWarp +
                        warp * kPagesPerWarp + lane;
          if (p < min(ceil_div(a.seq_len[tb], a.P), a.maxp)) {
            const int phys = a.page_table[(size_t)tb * a.maxp + p];
            if (phys >= 0 && phys < a.n_phys)
              prefetch_l2(reinterpret_cast<const uint4*>(a.page_minmax) +
                              ((size_t)phys * a.G + (PH ? tg / a.kv_div : tg)) * kPieces,
                          kPieces * 16);
          }
        }
      }
    }
  }
  pdl_wait();
  pdl_trigger();
  const int r = bound_group(), b = blockIdx.z;  // selection row r reads KV head r / kv_div
  const int npg = min(ceil_div(a.seq_len[b], a.P), a.maxp);
  const int p0 = bound_chunk() * kBoundWarps * kPagesPerWarp + warp * kPagesPerWarp;
  if (p0 >= npg) return;
  float4 q0, q1;
  bound_query<F16>(a, b, r, PH, lane, q0, q1);
  bound_warp<F16>(a, b, r, PH ? r / a.kv_div : r, p0, npg, lane, q0, q1);
}

// Pages covered by one CTA of page_bound_kernel.
inline int bound_pages_per_cta(bool f16) {
  return kBoundWarps * 8 * (f16 ? HHR_BOUND_SETS_F16 : HHR_BOUND_SETS_F32);
}

// ---------------------------------------------------------------------------- top-k
// Deterministic selection of the k largest finite scores of a row (ties to the
// lower index), written in ascending index order. Used for the top-m pages (HHR
// pruning), the top-m blocks and the token top-k of the indexer variant.
// Scores of -inf are ineligible. One CTA of 1024 threads per row:
//   1. 4-pass MSB-first radix select (8-bit digits) on order-preserving keys finds
//      the key T of the k-th largest element;
//   2. an ordered compaction keeps every key > T and the first (k - #greater)
//      elements equal to T in index order.
// `unit` > 0 maps an index i to kept_units[i / unit] * unit + i % unit (a token of
// a kept block); unit == 0 writes i itself.
constexpr int kSelThreads = 1024;

struct SelectArgs {
  const float* scores;    // [rows][stride]
  int stride;
  int rows_per_b;         // rows per sequence (G or T)
  const int32_t* seq_len;
  const int32_t* q_pos;   // indexer: eligibility uses min(seq_len, q_pos + 1); may be null
  int P;                  // keys per page/block (for n computation)
  int mode;               // 0: n = pages of the row; 1: n = kept_count[row] * unit
  const int32_t* kept_count;  // mode 1
  const int32_t* kept_units;  // mode 1: [rows][m_max]
  int m_max;
  int unit;
  int m_pages, keep_div;  // mode 0: k = kept_for(n_eligible, m_pages, keep_div)
  int top_k;              // mode 1: k = min(top_k, #finite)
  int32_t* out;           // [rows][out_stride]
  int out_stride;
  int32_t* out_count;     // [rows]
  int pad_out;            // write -1 into out[k..out_stride)
};

// Block-wide sum of one int and min / max of one uint32 per thread, in one pass of
// barriers (contains __syncthreads). sh: 96 words of shared memory.
template <bool kTailSync = true>
__device__ __forceinline__ void block_count_minmax(int cnt, uint32_t lo, uint32_t hi, uint32_t* sh,
                                                   int* out_cnt, uint32_t* out_lo,
                                                   uint32_t* out_hi) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cnt += __shfl_xor_sync(kFull, cnt, o);
    lo = min(lo, __shfl_xor_sync(kFull, lo, o));
    hi = max(hi, __shfl_xor_sync(kFull, hi, o));
  }
  if (lane == 0) { sh[warp] = (uint32_t)cnt; sh[32 + warp] = lo; sh[64 + warp] = hi; }
  __syncthreads();
  cnt = lane < nw ? (int)sh[lane] : 0;
  lo = lane < nw ? sh[32 + lane] : 0xffffffffu;
  hi = lane < nw ? sh[64 + lane] : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cnt += __shfl_xor_sync(kFull, cnt, o);
    lo = min(lo, __shfl_xor_sync(kFull, lo, o));
    hi = max(hi, __shfl_xor_sync(kFull, hi, o));
  }
  *out_cnt = cnt;
  *out_lo = lo;
  *out_hi = hi;
  if (kTailSync) __syncthreads();  // before sh is reused
}

// HC copies of each radix histogram: lane l adds into copy l % HC, so that lanes of one warp
// whose keys share a digit contend less on one shared-memory address; the scan sums the
// copies. Measured on B200: 4 copies take the standalone selection kernel of the 64-query
// indexer chunk from 72.6 to 65.8 us; the 4096-bound top-m of the Hamming kernel is not faster
// with them (2.32 -> 2.43 us of radix passes), so it keeps one.
template <int HC = 1>
struct SelShared {
  static constexpr int kCopies = HC;
  int hist[2][HC][256];  // double-buffered: a pass zeroes the next pass's histogram
  int scratch[66];
  uint32_t mm[96];
  int res[2][3];     // per pass (alternating): digit, rem, cnt
};

constexpr int kSelLoadUnroll = 4;  // score loads in flight per thread

// Where a block selection cuts (after block_select_cut): a key kk (0 = not finite) is taken
// when above(kk); with !whole_bin, keys equal to prefix (tie(kk)) are taken in index order
// until rem of them are taken. k = the number taken.
struct SelCut {
  int k, rem, sel_shift;
  uint32_t prefix;
  bool whole_bin;
  __device__ __forceinline__ bool above(uint32_t kk) const {
    if (kk == 0u || k == 0) return false;
    if (whole_bin) return (kk >> sel_shift) >= (prefix >> sel_shift);
    return kk > prefix;
  }
  __device__ __forceinline__ bool tie(uint32_t kk) const {
    return k > 0 && !whole_bin && kk != 0u && kk == prefix;
  }
};

// Threshold search of a block-wide selection (NT threads, call uniformly) of the k largest
// finite scores of sc[0..n), ties to the lower index. k = kept_for(#finite, m_pages,
// keep_div) when by_kept, else min(top_k, #finite). Leaves the order-preserving keys of
// the scores in keys[0..n) (shared memory, 16-byte aligned). Forced entries i < sink and
// i >= n - local take the largest key (above every finite score) and, when by_kept, k is at
// least their number.
// LU: score loads in flight per thread.
template <int NT, int LU = kSelLoadUnroll, int HC = 1>
__device__ __forceinline__ SelCut block_select_cut(const float* sc, int n, uint32_t* keys,
                                                   SelShared<HC>& sh, bool by_kept, int m_pages,
                                                   int keep_div, int top_k, int sink = 0,
                                                   int local = 0) {
  const int tid = threadIdx.x;
  int nfin = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int base = 0; base < n; base += LU * NT) {
    float f[LU];
#pragma unroll
    for (int j = 0; j < LU; ++j) {
      const int i = base + j * NT + tid;
      f[j] = i < n ? __ldcg(sc + i) : -INFINITY;  // may come from other CTAs of a kernel
    }
#pragma unroll
    for (int j = 0; j < LU; ++j) {
      const int i = base + j * NT + tid;
      const bool forced = i < n && (i < sink || i >= n - local);
      const bool live = forced || f[j] > -INFINITY;
      const uint32_t kk = forced ? 0xffffffffu : live ? f2key(f[j]) : 0u;
      if (i < n) keys[i] = kk;
      nfin += live;
      if (live) { kmin = min(kmin, kk); kmax = max(kmax, kk); }
    }
  }
  // Also orders the key stores before any read (sh.mm is not reused: no tail barrier).
  block_count_minmax<false>(nfin, kmin, kmax, sh.mm, &nfin, &kmin, &kmax);
  SelCut c;
  c.k = by_kept ? max(kept_for(nfin, m_pages, keep_div), min(n, max(sink + local, 0)))
                : min(top_k, nfin);
  // Selection rule after the search: key >> sel_shift > thr >> sel_shift selects; equal
  // keys at sel_shift == 0 are taken in index order until `rem` of them are taken; at
  // sel_shift > 0 the whole bin is taken (>=).
  c.prefix = 0;
  c.rem = c.k;
  c.sel_shift = 0;
  c.whole_bin = false;
  if (c.k > 0) {
    if (c.k == nfin) {
      c.whole_bin = true;          // everything finite is selected
      c.prefix = kmin;
    } else if (kmin == kmax) {
      c.prefix = kmin;             // all equal: the first k in index order
    } else {
      const int hb = 31 - __clz(kmin ^ kmax);          // highest differing bit
      int shift = max(hb - 7, 0);
      uint32_t mask = (hb >= 31) ? 0u : ~((2u << hb) - 1u);   // common high bits
      uint32_t prefix = kmin & mask;
      int rem = c.k;
      // Two barriers per pass: the histogram and the pass result alternate between two
      // buffers, and a pass zeroes the other histogram while it fills its own.
      int cur = 0;
      for (int i = tid; i < HC * 256; i += NT) (&sh.hist[0][0][0])[i] = 0;
      __syncthreads();
      const int copy = (tid & 31) % HC;
      while (true) {
        for (int i = tid; i < n; i += NT) {
          const uint32_t kk = keys[i];
          if (kk != 0u && (kk & mask) == prefix)
            atomicAdd(&sh.hist[cur][copy][(kk >> shift) & 255], 1);
        }
        for (int i = tid; i < HC * 256; i += NT) (&sh.hist[cur ^ 1][0][0])[i] = 0;
        __syncthreads();
        if (tid < 32) {
          // Lane l covers digits 255-8l .. 248-8l (descending).
          int cq[8], sum = 0;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            int c = 0;
#pragma unroll
            for (int cp = 0; cp < HC; ++cp) c += sh.hist[cur][cp][255 - 8 * tid - q];
            cq[q] = c;
            sum += c;
          }
          const int incl = warp_incl_scan(sum, tid);
          const int excl = incl - sum;
          if (excl < rem && rem <= incl) {
            int run = excl;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              if (run < rem && rem <= run + cq[q]) {
                sh.res[cur][0] = 255 - 8 * tid - q;
                sh.res[cur][1] = rem - run;
                sh.res[cur][2] = cq[q];
              }
              run += cq[q];
            }
          }
        }
        __syncthreads();
        prefix |= (uint32_t)sh.res[cur][0] << shift;
        mask |= 255u << shift;
        rem = sh.res[cur][1];
        const int cnt_bin = sh.res[cur][2];
        if (rem == cnt_bin) {  // the whole bin is needed: no tie-break required
          c.whole_bin = true;
          c.sel_shift = shift;
          break;
        }
        if (shift == 0) break;
        // Next 8 bits; when fewer than 8 remain, the last pass covers bits [0, 8) and
        // its already-fixed upper bits are constant across the candidates.
        shift = max(shift - 8, 0);
        cur ^= 1;
      }
      c.prefix = prefix;
      c.rem = rem;
    }
  }
  return c;
}

// Block-wide selection (NT threads, call uniformly): the k largest finite scores of sc[0..n),
// ties to the lower index, written in ascending index order to out[0..k) (global or shared
// memory); see block_select_cut for k. unit > 0 maps index i to kept_units[i / unit] * unit
// + i % unit. keys: shared scratch of n words (16-byte aligned). Returns k.
template <int NT = kSelThreads, int LU = kSelLoadUnroll, int HC = 1>
__device__ __forceinline__ int block_select_largest(const float* sc, int n, uint32_t* keys,
                                                    SelShared<HC>& sh, bool by_kept,
                                                    int m_pages, int keep_div, int top_k,
                                                    int32_t* out, int out_stride,
                                                    const int32_t* kept_units, int unit) {
  const int tid = threadIdx.x;
  const SelCut c =
      block_select_cut<NT, LU, HC>(sc, n, keys, sh, by_kept, m_pages, keep_div, top_k);
  // Compaction in index order over contiguous per-thread ranges. Before thread t's range
  // are gt_before keys above the cut and eq_before equal to it, of which the first
  // min(eq_before, rem) are taken.
  const int per = ceil_div(n, NT);
  const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
  int eq = 0, gt = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t kk = keys[i];
    if (c.above(kk)) ++gt;
    else if (c.tie(kk)) ++eq;
  }
  int2 tot;
  const int2 before = block_excl_scan2(make_int2(gt, eq), sh.scratch, &tot);
  if (c.k > 0) {
    // Keys are visited in chunks of 32: a take mask (keys above the cut, then the first
    // equal ones while fewer than rem equal keys precede them) is built from shared
    // memory, and only its set bits do the writes, in ascending order.
    int e = before.y;
    int pos = before.x + min(e, c.rem);
    for (int c0 = i0; c0 < i1; c0 += 32) {
      const int c1 = min(i1, c0 + 32);
      uint32_t takem = 0u, eqm = 0u;
      for (int i = c0; i < c1; ++i) {
        const uint32_t kk = keys[i];
        const uint32_t bit = 1u << (i - c0);
        if (c.above(kk)) takem |= bit;
        else if (c.tie(kk)) eqm |= bit;
      }
      for (int want = c.rem - e; eqm != 0u; eqm &= eqm - 1u, ++e, --want)
        if (want > 0) takem |= eqm & (0u - eqm);
      while (takem != 0u) {
        const int i = c0 + __ffs(takem) - 1;
        takem &= takem - 1u;
        if (pos < out_stride) out[pos] = unit > 0 ? kept_units[i / unit] * unit + i % unit : i;
        ++pos;
      }
    }
  }
  return c.k;
}

__global__ void __launch_bounds__(kSelThreads) select_largest_kernel(SelectArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ SelShared<4> sh;
  extern __shared__ uint32_t keys[];  // [n], 16-byte aligned
  const int row = blockIdx.x, tid = threadIdx.x;
  const int b = row / a.rows_per_b;
  int n;
  if (a.mode == 0) {
    int len = a.seq_len[b];
    if (a.q_pos != nullptr) len = min(len, a.q_pos[row] + 1);
    n = min(ceil_div(max(len, 0), a.P), a.stride);
  } else {
    n = min(a.kept_count[row] * a.unit, a.stride);
  }
  int32_t* out = a.out + (size_t)row * a.out_stride;
  const int k = block_select_largest<kSelThreads, kSelLoadUnroll, 4>(
      a.scores + (size_t)row * a.stride, n, keys, sh, a.mode == 0, a.m_pages, a.keep_div,
      a.top_k, out, a.out_stride,
      a.unit > 0 ? a.kept_units + (size_t)row * a.m_max : nullptr, a.unit);
  if (a.pad_out)
    for (int i = k + tid; i < a.out_stride; i += kSelThreads) out[i] = -1;
  if (tid == 0) a.out_count[row] = k;
}

// ---------------------------------------------------------------------------- a3 + a4
// HHR page, Abstract (LHP: Hamming distance between binary codes ranks the keys of
// the pages that survive pruning). Candidates are the valid keys of the kept pages, in
// ascending token order.
//   delta_t = sum over the row's query heads of popcount(qcode_h ^ code_t)  (0..gs*32*CW)
// Selection of the k smallest (delta, t): a histogram of the ranked distance (0 for a key of
// a forced page, else 1 + delta) gives the threshold bucket; an ordered compaction keeps
// every key below it and the first ones inside it in token order. Output ascending; -1 past
// k_eff.
//
// Distance by bit planes: channel j of a candidate contributes z_j = #heads with query
// bit 0 when the key bit is 1, else n_j = #heads with query bit 1. n and z are kept per
// code word as NB bit planes (NB = bit width of gs), so one select per plane and word
// gives the contributions' bits, and a carry-save step over each 4 words leaves 3
// popcounts per plane: 3*NB popcounts per 4 words instead of 4*gs.
constexpr int kHamRanks = 2;   // CTAs (a cluster) per (sequence, group)
constexpr int kMaxCand = 131072;  // a flat top-k over 4096 pages of 32 keys
constexpr int kMaxCodeWords = 8;  // 256-bit codes

// Threads of a top-m + Hamming CTA: 1024 (one CTA per SM, at most 64 registers), or 512 with
// two CTAs per SM, for grids larger than the SM count (a latency-bound chain per CTA, so two
// co-resident CTAs halve the waves). 8-word codes always take 512 threads and one CTA per SM
// (their query bit planes need the larger register budget).
template <int CW, int NT>
constexpr int ham_min_blocks() { return (NT == 512 && CW <= 4) ? 2 : 1; }
// Code loads in flight per thread (fewer when the plane words fill the registers).
template <int NB, int CW>
constexpr int ham_load() { return NB * CW >= 16 ? 2 : 4; }

struct HammingArgs {
  const uint32_t* q_code;    // [B][Hq][CW]
  const uint32_t* codes;     // [n_phys][G][P][CW]
  const int32_t* page_table;
  const int32_t* seq_len;
  const int32_t* kept;       // [B][G][m_max]
  const int32_t* kept_count; // [B][G]
  int32_t* out_idx;          // [B][G][top_k]
  int32_t* out_count;        // [B][G]
  int Hq, G, P, maxp, n_phys, m_max, top_k;
  uint32_t* out_rows;        // [B][G][top_k] cache row (phys*G + g)*P + slot of each selected
                             // key, for the attention of the fused step; or null
  int sink, local;           // forced pages [0, sink) and the last `local` of each sequence
  int Gs, kv_div;            // selection rows per sequence (G, or Hq per head); row r of a
                             // sequence uses the KV head r / kv_div and query heads
                             // [r Hq/Gs, (r + 1) Hq/Gs); bounds, kept lists and outputs are
                             // indexed by (sequence, row)
  // With out_rows: the K/V rows of output positions p with p % pf_split < HHR_ATTN_PREFETCH_ROWS
  // (the first tiles of each attention split) are prefetched into L2 (pf_split 0: none).
  const uint16_t* pf_k = nullptr;
  const uint16_t* pf_v = nullptr;
  int pf_split = 0;
};

// Selected K/V rows prefetched into L2 per attention split by the compaction (0: none).
#ifndef HHR_ATTN_PREFETCH_ROWS
#define HHR_ATTN_PREFETCH_ROWS 0
#endif

inline int hamming_planes(int gs) { return 32 - __builtin_clz((unsigned)gs); }

template <int NB, int CW>
struct QueryPlanes {
  uint32_t n[CW][NB];  // bit planes of #heads with a 1 bit
  uint32_t z[CW][NB];  // bit planes of #heads with a 0 bit
};

// One plane set of the bit-sliced counts: thread (kind, w) adds, with ripple carries, the
// bit vector of word w of every head's query code (q_code_w[h * stride], kind 0) or of its
// complement (kind 1). Result: out[b] for b < NB.
template <int NB>
__device__ __forceinline__ void build_plane_word(const uint32_t* q_code_w, int stride, int gs,
                                                 int kind, uint32_t* out) {
  uint32_t pl[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) pl[b] = 0u;
  for (int h = 0; h < gs; ++h) {
    uint32_t c = q_code_w[h * stride];
    if (kind) c = ~c;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const uint32_t t = pl[b] & c;
      pl[b] ^= c;
      c = t;
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) out[b] = pl[b];
}

// CW code words of a candidate (16-byte loads, 8-byte for two words).
template <int CW>
__device__ __forceinline__ void load_code(const uint32_t* p, uint32_t (&c)[CW]) {
  if constexpr (CW == 2) {
    const uint2 v = __ldcs(reinterpret_cast<const uint2*>(p));
    c[0] = v.x;
    c[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < CW / 4; ++i) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(p) + i);
      c[4 * i] = v.x;
      c[4 * i + 1] = v.y;
      c[4 * i + 2] = v.z;
      c[4 * i + 3] = v.w;
    }
  }
}

// Sum over the group's heads of popcount(qcode_h ^ c), from the bit planes: per plane b the
// selected contribution bits of each word, summed with one carry-save step per 4 words (3
// popcounts per 4 words), weighted by 2^b.
template <int NB, int CW>
__device__ __forceinline__ int hamming_delta(const QueryPlanes<NB, CW>& p, const uint32_t (&cw)[CW]) {
  int d = 0;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    uint32_t x[CW];
#pragma unroll
    for (int w = 0; w < CW; ++w) x[w] = (cw[w] & p.z[w][b]) | (~cw[w] & p.n[w][b]);
    int cnt = 0;
    if constexpr (CW == 2) {
      cnt = __popc(x[0]) + __popc(x[1]);
    } else {
#pragma unroll
      for (int w = 0; w < CW; w += 4) {
        const uint32_t sum = x[w] ^ x[w + 1] ^ x[w + 2];
        const uint32_t carry = (x[w] & x[w + 1]) | (x[w + 2] & (x[w] ^ x[w + 1]));
        cnt += __popc(sum) + __popc(x[w + 3]) + 2 * __popc(carry);
      }
    }
    d += cnt << b;
  }
  return d;
}

struct HamShared {
  int scratch[66];
  int T, need_eq;
  int tot[2];  // lower-ranked CTAs' (#below threshold, #at threshold): this rank's output offsets
};

// Steps a3-a4 for one (sequence, group) row on the cluster's CTA `rank` (of RANKS), given the
// row's kept logical pages klp[0..m) (ascending) and their physical pages kphys (-1 invalid),
// in shared memory; n = the sequence's keys. CTA r scores candidates [r*half, (r+1)*half); the
// histograms and the compaction offsets are combined through distributed shared memory.
// hsm: hamming_smem() bytes of shared memory. Call uniformly by all threads. Ends with the
// cluster's shared memory released (a cluster barrier that does not order the compaction's
// global writes: a caller that reads them in other CTAs synchronises the cluster again).
template <int NB, int CW, int NT, int RANKS = kHamRanks>
__device__ __forceinline__ void hamming_topk_cluster(const HammingArgs& a, int row, int rank, const int32_t* klp,
                                     const int32_t* kphys, int m, const uint32_t* qcs,
                                     uint32_t (*planes)[CW][4], uint32_t* hsm, HamShared& hs,
                                     int n) {
  // Ranked distance: 0 for a key of a forced page, else 1 + delta (bins 0 .. gs*32*CW + 1).
  constexpr int kBins = (kMaxGroup * 32 * CW + 2 + NT - 1) / NT;  // threshold bins per thread
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int r = row % a.Gs;
  const int g = a.kv_div == 1 ? r : r / a.kv_div;  // no division on the grouped path
  const int tid = threadIdx.x;
  const int gs = a.Hq / a.Gs;  // query heads of the row
  const int nbins = gs * 32 * CW + 2;
  m = min(m, a.m_max);
  int* hist = reinterpret_cast<int*>(hsm);                                // [nbins]
  uint16_t* dist = reinterpret_cast<uint16_t*>(hist + ((nbins + 31) & ~31));  // [half], 16B-aligned
  const int npg = min(ceil_div(max(n, 0), a.P), a.maxp);  // pages of the sequence
  const int C = min(m * a.P, kMaxCand);
  const int half = ((ceil_div(C, RANKS) + 7) / 8) * 8;
  const int lo = min(C, rank * half), hi = min(C, lo + half);
  const int Cr = hi - lo;
  for (int i = tid; i < nbins; i += NT) hist[i] = 0;
  if (tid == 0) { hs.T = -1; hs.need_eq = 0; hs.tot[0] = 0; hs.tot[1] = 0; }
  if (tid < 2 * CW) {
    const int kind = tid / CW, w = tid % CW;
    build_plane_word<NB>(qcs + w, CW, gs, kind, &planes[kind][w][0]);
  }
  __syncthreads();  // histogram zeroed, planes built
  QueryPlanes<NB, CW> qp;
#pragma unroll
  for (int w = 0; w < CW; ++w) {
#pragma unroll
    for (int pb = 0; pb < NB; ++pb) {
      qp.n[w][pb] = planes[0][w][pb];
      qp.z[w][pb] = planes[1][w][pb];
    }
  }
  // Candidates c = lo + tid + j*NT: consecutive threads read consecutive codes of a page
  // (coalesced); all ham_load() code loads of a thread are issued before any math.
  // c / P by multiply-high: exact for c < 2^24 with magic = floor(2^32 / P) + 1.
  const uint32_t magic = (uint32_t)(0xffffffffu / (uint32_t)a.P) + 1u;
  constexpr int kHamLoad = ham_load<NB, CW>();
  for (int c0 = lo; c0 < hi; c0 += NT * kHamLoad) {
    uint32_t code[kHamLoad][CW];
    bool ok[kHamLoad], fr[kHamLoad];
#pragma unroll
    for (int j = 0; j < kHamLoad; ++j) {
      const int c = c0 + j * NT + tid;
      ok[j] = false;
      fr[j] = false;
#pragma unroll
      for (int w = 0; w < CW; ++w) code[j][w] = 0u;
      if (c < hi) {
        const int i = (a.P == 1) ? c : (int)__umulhi((uint32_t)c, magic);
        const int slot = c - i * a.P;
        const int phys = kphys[i];
        const int lp = klp[i];
        fr[j] = lp < a.sink || lp >= npg - a.local;
        if (phys >= 0 && lp * a.P + slot < n) {
          ok[j] = true;
          load_code<CW>(a.codes + (((size_t)phys * a.G + g) * a.P + slot) * CW, code[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kHamLoad; ++j) {
      const int c = c0 + j * NT + tid;
      const int d = fr[j] ? 0 : 1 + hamming_delta<NB, CW>(qp, code[j]);
      if (ok[j]) atomicAdd(&hist[d], 1);
      if (c < hi) dist[c - lo] = ok[j] ? (uint16_t)d : (uint16_t)0xffff;
    }
  }
  cluster_sync_all();  // every rank's histogram is complete
  // Threshold bucket: smallest T with #(delta <= T) >= k_eff over the summed histograms.
  // Thread t holds bins [kBins t, kBins (t + 1)) (fewer past nbins). The same scan over the
  // histograms of the lower-ranked CTAs gives this rank's output offsets: how many of their
  // candidates lie below T (tot[0]) and at T (tot[1]).
  {
    int hv[kBins], lv[kBins], sum = 0, lsum = 0;
#pragma unroll
    for (int q = 0; q < kBins; ++q) {
      const int i = kBins * tid + q;
      hv[q] = 0;
      lv[q] = 0;
      if (i < nbins) {
#pragma unroll
        for (int r = 0; r < RANKS; ++r) {
          const int c = cl.map_shared_rank(hist, r)[i];
          hv[q] += c;
          if (r < rank) lv[q] += c;
        }
      }
      sum += hv[q];
      lsum += lv[q];
    }
    cluster_arrive();  // no remote shared-memory access after this point
    int2 nvalid;
    const int2 excl = block_excl_scan2<false>(make_int2(sum, lsum), hs.scratch, &nvalid);
    const int keff = min(a.top_k, nvalid.x);  // scratch's next use: after the barrier below
    if (keff > 0 && excl.x < keff && keff <= excl.x + sum) {
      int run = excl.x, lrun = excl.y;
      bool found = false;
#pragma unroll
      for (int q = 0; q < kBins; ++q) {
        if (!found && keff <= run + hv[q]) {
          hs.T = kBins * tid + q;
          hs.need_eq = keff - run;
          hs.tot[0] = lrun;   // lower ranks' candidates below T
          hs.tot[1] = lv[q];  // and at T
          found = true;
        }
        run += hv[q];
        lrun += lv[q];
      }
    }
    if (tid == 0) a.out_count[row] = keff;  // every rank writes the same value
    __syncthreads();
    for (int i = keff + rank * NT + tid; i < a.top_k; i += RANKS * NT)
      a.out_idx[(size_t)row * a.top_k + i] = -1;
  }
  const int T = hs.T, need_eq = hs.need_eq, lt_off = hs.tot[0], eq_off = hs.tot[1];
  // Ordered compaction of this rank's candidates: thread t owns [t*cpt, (t+1)*cpt), cpt a
  // multiple of 8, read as 16-byte groups of 8 distances.
  const int cpt = ((ceil_div(Cr, NT) + 7) / 8) * 8;
  const int ngrp = cpt / 8;
  auto load8 = [&](int i0, uint16_t (&dv)[8]) {
    uint4 raw = make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
    if (i0 < Cr) raw = *reinterpret_cast<const uint4*>(dist + i0);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      dv[2 * q] = (i0 + 2 * q < Cr) ? (uint16_t)(w[q] & 0xffff) : (uint16_t)0xffff;
      dv[2 * q + 1] = (i0 + 2 * q + 1 < Cr) ? (uint16_t)(w[q] >> 16) : (uint16_t)0xffff;
    }
  };
  int eq = 0, lt = 0;
  for (int gi = 0; gi < ngrp; ++gi) {
    uint16_t dv[8];
    load8(tid * cpt + gi * 8, dv);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      eq += (dv[q] == T);
      lt += (dv[q] < T);
    }
  }
  int2 tot;
  const int2 before = block_excl_scan2<false>(make_int2(lt, eq), hs.scratch, &tot);  // last use
  int32_t* out = a.out_idx + (size_t)row * a.top_k;
  {
    int e = eq_off + before.y;
    int pos = lt_off + before.x + min(e, need_eq);
    for (int gi = 0; gi < ngrp; ++gi) {
      uint16_t dv[8];
      const int i0 = tid * cpt + gi * 8;
      load8(i0, dv);
      uint32_t takem = 0u;  // the group's selected candidates, then visited bit by bit
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        bool take = dv[q] < T;
        if (dv[q] == T) { take = e < need_eq; ++e; }
        if (take) takem |= 1u << q;
      }
      while (takem != 0u) {
        const int q = __ffs(takem) - 1;
        takem &= takem - 1u;
        if (pos < a.top_k) {
          const int i = lo + i0 + q;
          const int pi = (a.P == 1) ? i : (int)__umulhi((uint32_t)i, magic);
          const int slot = i - pi * a.P;
          out[pos] = klp[pi] * a.P + slot;
          if (a.out_rows != nullptr) {
            const uint32_t crow =
                ((uint32_t)kphys[pi] * (uint32_t)a.G + (uint32_t)g) * (uint32_t)a.P + (uint32_t)slot;
            a.out_rows[(size_t)row * a.top_k + pos] = crow;
            if (HHR_ATTN_PREFETCH_ROWS > 0 && a.pf_split > 0 &&
                pos % a.pf_split < HHR_ATTN_PREFETCH_ROWS && kphys[pi] >= 0) {
              prefetch_l2(a.pf_k + (size_t)crow * kD, kD * 2);
              prefetch_l2(a.pf_v + (size_t)crow * kD, kD * 2);
            }
          }
          ++pos;
        }
      }
    }
  }
  cluster_wait();  // keep this CTA's shared memory alive until every rank has read it
}

inline size_t hamming_smem(int gs, int cw, int m_max, int P, int ranks = kHamRanks) {
  const int nbins = gs * 32 * cw + 2;
  const size_t ints = (size_t)((nbins + 31) & ~31);
  // This rank's distances, padded so the 16-byte group reads of the last thread stay inside.
  const size_t c = (size_t)m_max * P < (size_t)kMaxCand ? (size_t)m_max * P : (size_t)kMaxCand;
  const size_t half = ((c + ranks - 1) / ranks + 7) & ~(size_t)7;
  return ints * 4 + (half + 8) * 2 + 16;
}

// Top-m pages and the Hamming top-k fused in one cluster of kHamRanks CTAs per (sequence,
// selection row: a KV group, or a query head): every rank selects the same kept pages
// (deterministic), resolving their physical
// pages during the compaction, so the kept list never leaves shared memory (rank 0 copies
// it to `kept`/`kept_count` for inspection). Shared memory: [kept list: m_max words][their
// physical pages: m_max words][union of: top-m keys (maxp words) | Hamming scratch].
struct TopmHammingArgs {
  HammingArgs h;
  const float* bounds;  // [B][G][maxp]; not read when flat
  int m_pages, keep_div;
  int flat;             // every page is kept (flat hash top-k): no bounds, no top-m
};

// 1: the kept-page pass prefetches each kept page's codes into L2 for the Hamming stage.
// Measured on B200 (128K context, batch 8, clock stamps per phase): the 256 bulk prefetches
// per CTA slow the kept-page pass by 0.4 us and speed the Hamming stage by 0.26 us, so the
// default is 0.
#ifndef HHR_TOPM_CODE_PREFETCH
#define HHR_TOPM_CODE_PREFETCH 0
#endif

// Per-warp ballots of the kept-page pass of topm_hamming_kernel: NT / 32 warps share the
// 32768 pages a sequence may hold, in 32-page chunks.
constexpr int kTopmPages = 32768;
constexpr int kTopmPtPre = 4;     // chunks whose page-table entries are loaded up front
template <int NT>
struct TopmShared {
  static constexpr int kWarps = NT / 32;
  static constexpr int kChunks = kTopmPages / 32 / kWarps;
  uint32_t bal[kWarps][kChunks][2];  // (above, tie) ballots per warp and chunk
  int cnt[kWarps][2];                // per-warp counts, then their exclusive prefix
  static_assert(kWarps <= 32, "the warp-prefix scan covers the warps with one warp");
};

// Static shared memory of one selection (top-m + Hamming top-k of one row).
template <int NT>
struct TopmSmem {
  SelShared<1> sh;
  HamShared hs;
  uint32_t qcs[kMaxGroup * kMaxCodeWords];   // the row's query codes
  uint32_t planes[2][kMaxCodeWords][4];      // their bit planes
  TopmShared<NT> ts;
};

// Top-m pages and the Hamming top-k of selection row `row`, on CTA `rank` of its cluster of
// RANKS CTAs (NT threads each; call uniformly). fsm: topm_hamming_smem() bytes of dynamic
// shared memory. Bounds are read through L2. The row's length and first page-table entries
// (inputs that no earlier kernel writes) are loaded first; with dep_wait the programmatic
// dependency wait comes after them, before anything an earlier kernel writes is read.
template <int NB, int CW, int NT, int RANKS = kHamRanks>
__device__ __forceinline__ void topm_hamming_row(const TopmHammingArgs& a, int row, int rank,
                                                 TopmSmem<NT>& S, uint32_t* fsm, bool dep_wait) {
  static_assert(NT == 512 || (NT == 1024 && CW <= 4), "512 threads, or 1024 up to 4 words");
  constexpr int kTopmWarps = NT / 32;
  SelShared<1>& sh = S.sh;
  HamShared& hs = S.hs;
  uint32_t* qcs = S.qcs;
  uint32_t(*planes)[CW][4] = reinterpret_cast<uint32_t(*)[CW][4]>(&S.planes[0][0][0]);
  TopmShared<NT>& ts = S.ts;
  const HammingArgs& h = a.h;
  const int b = row / h.Gs, r = row % h.Gs;
  const int g = h.kv_div == 1 ? r : r / h.kv_div;  // no division on the grouped path
  const int gs = h.Hq / h.Gs;  // query heads of the row
  const int mw = (h.m_max + 3) & ~3;
  int32_t* kept_s = reinterpret_cast<int32_t*>(fsm);
  int32_t* kphys_s = kept_s + mw;
  uint32_t* work = fsm + 2 * mw;
  const int n_keys = h.seq_len[b];
  const int n = min(ceil_div(max(n_keys, 0), h.P), h.maxp);
  // Kept pages: warp w owns pages [w R, (w + 1) R), R a multiple of 32, visited 32 at a time
  // (page w R + 32 j + lane), so that kept flags come from ballots and kept positions from
  // popcounts; every lane with a kept page then does its writes at once.
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int R = ceil_div(ceil_div(n, kTopmWarps), 32) * 32;
  const int J = R / 32;
  const int wbase = warp * R;
  const int32_t* ptab = h.page_table + (size_t)b * h.maxp;
  int32_t* kept_g = const_cast<int32_t*>(h.kept) + (size_t)row * h.m_max;
  const uint32_t* code_g = h.codes + (size_t)g * h.P * CW;
  const size_t code_page = (size_t)h.G * h.P * CW;
  if (a.flat) {  // flat hash top-k: the kept list is every page of the sequence
    if (dep_wait) pdl_wait();
    if (threadIdx.x < gs * CW)  // visible after the barrier below
      qcs[threadIdx.x] = h.q_code[((size_t)b * h.Hq + r * gs) * CW + threadIdx.x];
    const int m = min(n, h.m_max);
    for (int p = threadIdx.x; p < m; p += NT) {
      int phys = ptab[p];
      if (phys < 0 || phys >= h.n_phys) {
        flag_status(kStatusBadPage);
        phys = -1;
      }
      kept_s[p] = p;
      kphys_s[p] = phys;
      if (rank == 0) kept_g[p] = p;
    }
    if (rank == 0 && threadIdx.x == 0) const_cast<int32_t*>(h.kept_count)[row] = m;
    __syncthreads();
    hamming_topk_cluster<NB, CW, NT, RANKS>(h, row, rank, kept_s, kphys_s, m, qcs, planes,
                                            work, hs, n_keys);
    return;
  }
  int pt[kTopmPtPre];  // page-table entries of the first chunks, loaded with the bounds
#pragma unroll
  for (int j = 0; j < kTopmPtPre; ++j) {
    const int p = wbase + 32 * j + lane;
    pt[j] = (j < J && p < n) ? ptab[p] : -1;
  }
  if (dep_wait) pdl_wait();
  if (threadIdx.x < gs * CW)  // visible after the selection's first barrier
    qcs[threadIdx.x] = h.q_code[((size_t)b * h.Hq + r * gs) * CW + threadIdx.x];
  const SelCut cut = block_select_cut<NT>(a.bounds + (size_t)row * h.maxp, n, work, sh,
                                          true, a.m_pages, a.keep_div, 0, h.sink, h.local);
  int ng = 0, ne = 0;
  for (int j = 0; j < J; ++j) {
    const int p = wbase + 32 * j + lane;
    const uint32_t kk = p < n ? work[p] : 0u;
    const uint32_t bg = __ballot_sync(kFull, cut.above(kk));
    const uint32_t be = __ballot_sync(kFull, cut.tie(kk));
    if (lane == 0) {
      ts.bal[warp][j][0] = bg;
      ts.bal[warp][j][1] = be;
    }
    ng += __popc(bg);
    ne += __popc(be);
  }
  if (lane == 0) {
    ts.cnt[warp][0] = ng;
    ts.cnt[warp][1] = ne;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefix over the warps of (above, tie) counts
    const int xg = lane < kTopmWarps ? ts.cnt[lane][0] : 0;
    const int xe = lane < kTopmWarps ? ts.cnt[lane][1] : 0;
    const int ig = warp_incl_scan(xg, lane), ie = warp_incl_scan(xe, lane);
    if (lane < kTopmWarps) {
      ts.cnt[lane][0] = ig - xg;
      ts.cnt[lane][1] = ie - xe;
    }
  }
  __syncthreads();
  const int m = cut.k;
  int e = ts.cnt[warp][1];                 // ties before this warp's pages
  int pos = ts.cnt[warp][0] + min(e, cut.rem);
  for (int j = 0; j < J; ++j) {
    uint32_t takem = ts.bal[warp][j][0];
    uint32_t be = ts.bal[warp][j][1];
    for (int want = cut.rem - e; be != 0u; be &= be - 1u, ++e, --want)  // ties in index order
      if (want > 0) takem |= be & (0u - be);
    if ((takem >> lane) & 1u) {
      const int kpos = pos + __popc(takem & ((1u << lane) - 1u));
      const int p = wbase + 32 * j + lane;
      int phys = 0;
      bool pre = false;
#pragma unroll
      for (int q = 0; q < kTopmPtPre; ++q)
        if (j == q) { phys = pt[q]; pre = true; }
      if (!pre) phys = ptab[p];
      if (phys < 0 || phys >= h.n_phys) {
        flag_status(kStatusBadPage);
        phys = -1;
      } else if (HHR_TOPM_CODE_PREFETCH) {
        prefetch_l2(code_g + (size_t)phys * code_page, (unsigned)(h.P * CW * 4));
      }
      if (kpos < h.m_max) {
        kept_s[kpos] = p;
        kphys_s[kpos] = phys;
        if (rank == 0) kept_g[kpos] = p;
      }
    }
    pos += __popc(takem);
  }
  if (rank == 0 && threadIdx.x == 0) const_cast<int32_t*>(h.kept_count)[row] = m;
  __syncthreads();
  hamming_topk_cluster<NB, CW, NT, RANKS>(h, row, rank, kept_s, kphys_s, m, qcs, planes, work,
                                          hs, n_keys);
}

template <int NB, int CW, int NT>
__global__ void __cluster_dims__(kHamRanks, 1, 1) __launch_bounds__(NT, ham_min_blocks<CW, NT>())
    topm_hamming_kernel(TopmHammingArgs a) {
  __shared__ TopmSmem<NT> S;
  pdl_trigger();
  extern __shared__ uint32_t fsm[];
  topm_hamming_row<NB, CW, NT>(a, blockIdx.x / kHamRanks, blockIdx.x % kHamRanks, S, fsm, true);
}

inline size_t topm_hamming_smem(int gs, int cw, int m_max, int P, int maxp,
                                int ranks = kHamRanks) {
  const size_t sel = (size_t)maxp * 4;
  const size_t ham = hamming_smem(gs, cw, m_max, P, ranks);
  return (size_t)((m_max + 3) & ~3) * 8 + (sel > ham ? sel : ham);
}

using TopmHammingFn = void (*)(TopmHammingArgs);

template <int CW, int NT>
inline TopmHammingFn topm_hamming_for_cw(int gs) {
  switch (hamming_planes(gs)) {
    case 1: return topm_hamming_kernel<1, CW, NT>;
    case 2: return topm_hamming_kernel<2, CW, NT>;
    case 3: return topm_hamming_kernel<3, CW, NT>;
    default: return topm_hamming_kernel<4, CW, NT>;
  }
}

// Threads per CTA for cw code words and a grid of `ctas` CTAs on `sms` SMs (see
// ham_min_blocks). HHR_HAM_THREADS fixes the choice (512 or 1024) for sweeps.
#ifndef HHR_HAM_THREADS
#define HHR_HAM_THREADS 0
#endif
inline int topm_hamming_threads(int cw, long long ctas, int sms) {
  if (cw == 8) return 512;
  if (HHR_HAM_THREADS == 512 || HHR_HAM_THREADS == 1024) return HHR_HAM_THREADS;
  return ctas > sms ? 512 : 1024;
}

// The instantiation for group size gs (1..kMaxGroup), cw code words (2, 4 or 8) and nt
// threads (topm_hamming_threads).
inline TopmHammingFn topm_hamming_for(int gs, int cw, int nt) {
  if (cw == 8) return topm_hamming_for_cw<8, 512>(gs);
  if (cw == 2) return nt == 512 ? topm_hamming_for_cw<2, 512>(gs) : topm_hamming_for_cw<2, 1024>(gs);
  return nt == 512 ? topm_hamming_for_cw<4, 512>(gs) : topm_hamming_for_cw<4, 1024>(gs);
}

// ---------------------------------------------------------------------------- HISA a1'
// HISA page, Abstract: the block-level coarse filter scores pooled block
// representatives (block_mean) against each query. Blocks whose start lies after
// the query position are ineligible (-inf). One CTA of 128 threads handles 32 blocks for up
// to 16 chunk queries: the 32 page ids are read first, then every thread issues its 8
// block-mean pieces at once (warp w loads whole 512-byte rows, one per instruction), staged
// transposed in shared memory; thread t then scores block t % 32 for queries 4 (t / 32) ..
// 4 (t / 32) + 3.
constexpr int kBlkTile = 32;
constexpr int kQTile = 16;
constexpr int kBlkThreads = 128;

struct BlockScoreArgs {
  const uint16_t* q;        // [B][T][d]
  const float* block_mean;  // [n_phys][1][d]
  const int32_t* page_table;
  const int32_t* seq_len;
  const int32_t* q_pos;     // [B][T]
  float* scores;            // [B][T][maxp]
  int T, P, maxp, n_phys;
};

constexpr int kBlkStride = kBlkTile + 1;  // float4 row stride of the staged tile (padded)

__global__ void __launch_bounds__(kBlkThreads) block_score_kernel(BlockScoreArgs a) {
  __shared__ float4 Ms[kD / 4][kBlkStride];  // block means, channel-major
  __shared__ float4 Qs[kQTile][kD / 4];
  __shared__ int ids[kBlkTile];
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.z, q0 = blockIdx.y * kQTile, blk0 = blockIdx.x * kBlkTile;
  const int tid = threadIdx.x;
  const int nblk = min(ceil_div(a.seq_len[b], a.P), a.maxp);
  if (blk0 >= nblk) return;
  const int nq = min(kQTile, a.T - q0);
  if (tid < kBlkTile) {
    const int blk = blk0 + tid;
    int phys = -1;
    if (blk < nblk) {
      phys = a.page_table[(size_t)b * a.maxp + blk];
      if (phys < 0 || phys >= a.n_phys) {
        flag_status(kStatusBadPage);
        phys = -1;
      }
    }
    ids[tid] = phys;
  }
  for (int idx = tid; idx < kQTile * (kD / 4); idx += kBlkThreads) {
    const int qi = idx / (kD / 4), c4 = idx % (kD / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (qi < nq) {
      const uint2 w = *reinterpret_cast<const uint2*>(a.q + ((size_t)b * a.T + q0 + qi) * kD + 4 * c4);
      v = bf16x4_to_f4(w);
    }
    Qs[qi][c4] = v;
  }
  __syncthreads();
  constexpr int kPer = kBlkTile * (kD / 4) / kBlkThreads;  // 8 pieces per thread
  float4 mv[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int idx = i * kBlkThreads + tid;
    const int r = idx / (kD / 4), c4 = idx % (kD / 4);
    const int phys = ids[r];
    mv[i] = phys >= 0 ? reinterpret_cast<const float4*>(a.block_mean + (size_t)phys * kD)[c4]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int idx = i * kBlkThreads + tid;
    Ms[idx % (kD / 4)][idx / (kD / 4)] = mv[i];
  }
  __syncthreads();
  const int r = tid % kBlkTile, qg = tid / kBlkTile;  // block r, queries 4 qg .. 4 qg + 3
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int c4 = 0; c4 < kD / 4; ++c4) {
    const float4 m = Ms[c4][r];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 qv = Qs[4 * qg + i][c4];
      acc[i] = fmaf(qv.x, m.x, fmaf(qv.y, m.y, fmaf(qv.z, m.z, fmaf(qv.w, m.w, acc[i]))));
    }
  }
  const int blk = blk0 + r;
  if (blk < nblk) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int qi = 4 * qg + i;
      if (qi >= nq) break;
      const int pos = a.q_pos[(size_t)b * a.T + q0 + qi];
      const bool elig = (long long)blk * a.P <= (long long)pos;
      a.scores[((size_t)b * a.T + q0 + qi) * a.maxp + blk] = elig ? acc[i] : -INFINITY;
    }
  }
}

inline size_t block_score_smem() { return 0; }

// ---------------------------------------------------------------------------- HISA a3
// HISA page, Abstract: the original token indexer runs only inside the kept blocks.
// sigma_t = q . k_t in fp32 (bf16 products are exact in fp32). One warp scores 32
// candidates: lane l loads channels 4l..4l+3 of each candidate row (a coalesced
// 256-byte row read per candidate), then a transposed warp reduction leaves the
// score of candidate j on lane j. Ineligible candidates (t > pos or t >= n) get -inf.
constexpr int kTokWarps = 8;

struct TokenScoreArgs {
  const uint16_t* q;        // [B][T][d]
  const uint16_t* k_cache;  // [n_phys][1][P][d]
  const int32_t* page_table;
  const int32_t* seq_len;
  const int32_t* q_pos;
  const int32_t* kept;      // [B][T][m_max]
  const int32_t* kept_count;
  float* tok_scores;        // [B][T][m_max * P]
  int T, P, maxp, n_phys, m_max;
};

__global__ void __launch_bounds__(kTokWarps * 32) token_score_kernel(TokenScoreArgs a) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.y, b = row / a.T;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int C = a.kept_count[row] * a.P;
  const int c0 = (blockIdx.x * kTokWarps + warp) * 32;
  if (c0 >= C) return;
  const int n = a.seq_len[b], pos = a.q_pos[row];
  const float4 qv = bf16x4_to_f4(*reinterpret_cast<const uint2*>(a.q + (size_t)row * kD + 4 * lane));
  // Candidate c is slot c % P of kept block kept[c / P]. With P a multiple of 32 the warp's
  // 32 candidates share one block, resolved once (lane 0) so that the row loads are
  // independent; otherwise each candidate resolves its own block.
  const bool one_block = (a.P & 31) == 0;
  int lp_w = -1, phys_w = -1;
  if (one_block && lane == 0) {
    lp_w = a.kept[(size_t)row * a.m_max + c0 / a.P];
    if (lp_w >= 0 && lp_w < a.maxp) {
      phys_w = a.page_table[(size_t)b * a.maxp + lp_w];
      if (phys_w < 0 || phys_w >= a.n_phys) phys_w = -1;
    }
  }
  lp_w = __shfl_sync(kFull, lp_w, 0);
  phys_w = __shfl_sync(kFull, phys_w, 0);
  auto resolve = [&](int c, int& t, int& phys) {
    int lp = lp_w;
    phys = phys_w;
    if (!one_block) {
      lp = a.kept[(size_t)row * a.m_max + c / a.P];
      phys = -1;
      if (lp >= 0 && lp < a.maxp) {
        phys = a.page_table[(size_t)b * a.maxp + lp];
        if (phys < 0 || phys >= a.n_phys) phys = -1;
      }
    }
    t = lp * a.P + c % a.P;
  };
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int c = c0 + j;
    float sc = 0.f;
    if (c < C) {
      int t, phys;
      resolve(c, t, phys);
      if (t < n && t <= pos && phys >= 0) {
        const uint2 w = *reinterpret_cast<const uint2*>(
            a.k_cache + ((size_t)phys * a.P + c % a.P) * kD + 4 * lane);
        const float4 kv = bf16x4_to_f4(w);
        sc = qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
      }
    }
    v[j] = sc;
  }
  const float scv = warp_transpose_sum32(v, lane);
  const int c = c0 + lane;
  if (c < C) {
    int t, phys;
    resolve(c, t, phys);
    bool ok = t < n && t <= pos;
    if (ok && phys < 0) {
      ok = false;
      flag_status(kStatusBadPage);
    }
    a.tok_scores[(size_t)row * a.m_max * a.P + c] = ok ? scv : -INFINITY;
  }
}

}  // namespace hhr
