// Prologue of the fused decode step: append the newest key/value row of every sequence to
// the paged cache, encode that key (step a0) and prepare the group's queries (step a1),
// all with one read of R_g and W_g.
//
// HHR page, Abstract: GKR rotates keys and queries with the head-wise orthogonal R_h and
// summarises each page for its logit bound; LHP encodes both into binary codes. One CTA
// of kMvThreads threads per (KV group, sequence): the newest key (position seq_len-1) and
// the group's query heads form one batch of up to 9 vectors for the two mat-vecs. The key
// and query arithmetic is the same per-vector code as in encode_page_kernel and
// qprep_kernel, so the results are bit-identical to the separate calls.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "encode.cuh"

namespace hhr {

struct PrologueArgs {
  const uint16_t* q;       // [B][Hq][d]
  const uint16_t* k_new;   // [B][G][d] newest key rows, or null (already in the cache)
  const uint16_t* v_new;   // [B][G][d] newest value rows, or null
  uint16_t* k_cache;       // [n_phys][G][P][d]
  uint16_t* v_cache;
  const int32_t* page_table;
  const int32_t* seq_len;  // after the append: the newest key sits at seq_len - 1
  const float* R;
  const float* W;
  void* page_minmax;
  uint32_t* codes;
  float* q_rot;            // [B][Hq][d]
  uint32_t* q_code;        // [B][Hq][4]
  float* qpn;              // [B][G][2][d]
  int Hq, G, P, maxp, n_phys, summary_fp16;
};

constexpr int kMaxStepVecs = 1 + kMaxGroup;  // newest key + query heads

// Loads the stored summary channels `row` of a page that already held keys.
__device__ __forceinline__ void load_summary_row(const void* page_minmax, int fp16, size_t sbase,
                                                 int row, float& mn, float& mx) {
  if (fp16) {
    const __half* mm = reinterpret_cast<const __half*>(page_minmax) + sbase;
    mn = __half2float(mm[row]);
    mx = __half2float(mm[kD + row]);
  } else {
    const float* mm = reinterpret_cast<const float*>(page_minmax) + sbase;
    mn = mm[row];
    mx = mm[kD + row];
  }
}

// Stores summary channel `row`; f16 summaries round outward, as in encode_page_kernel.
__device__ __forceinline__ void store_summary_row(void* page_minmax, int fp16, size_t sbase, int row,
                                                  float mn, float mx) {
  if (fp16) {
    __half* mm = reinterpret_cast<__half*>(page_minmax) + sbase;
    mm[row] = __float2half_rd(mn);
    mm[kD + row] = __float2half_ru(mx);
  } else {
    float* mm = reinterpret_cast<float*>(page_minmax) + sbase;
    mm[row] = mn;
    mm[kD + row] = mx;
  }
}

// Resolves the newest key's slot; phys < 0 when the sequence is empty or its page is bad.
struct NewestSlot {
  int phys, slot;
  size_t krow, sbase;
};

__device__ __forceinline__ NewestSlot newest_slot(const PrologueArgs& a, int b, int g, bool report) {
  const int t = a.seq_len[b] - 1;
  const int lp = t >= 0 ? t / a.P : -1;
  int phys = -1;
  if (t >= 0 && lp < a.maxp) {
    phys = a.page_table[(size_t)b * a.maxp + lp];
    if (phys < 0 || phys >= a.n_phys) phys = -1;
  }
  if (t >= 0 && phys < 0 && report) flag_status(kStatusBadPage);
  NewestSlot s;
  s.phys = phys;
  s.slot = phys >= 0 ? t - lp * a.P : 0;
  s.krow = phys >= 0 ? (((size_t)phys * a.G + g) * a.P + s.slot) * kD : 0;
  s.sbase = ((size_t)(phys >= 0 ? phys : 0) * a.G + g) * 2 * kD;
  return s;
}

// Fills xs[0] with the newest key (written to the cache first when given; only when
// `writer`) and xs[1..gs] with the group's queries.
__device__ __forceinline__ void load_step_vectors(const PrologueArgs& a, int b, int g, const NewestSlot& s,
                                                  bool writer, float (*xs)[kD], int nthreads) {
  const int gs = a.Hq / a.G;
  for (int i = threadIdx.x; i < (1 + gs) * kD; i += nthreads) {
    const int v = i / kD, c = i % kD;
    float x = 0.f;
    if (v == 0) {
      if (s.phys >= 0) {
        uint16_t kb;
        if (a.k_new != nullptr) {
          kb = a.k_new[((size_t)b * a.G + g) * kD + c];
          if (writer) {
            a.k_cache[s.krow + c] = kb;
            if (a.v_new != nullptr) a.v_cache[s.krow + c] = a.v_new[((size_t)b * a.G + g) * kD + c];
          }
        } else {
          kb = a.k_cache[s.krow + c];
        }
        x = bf16_to_f(kb);
      }
    } else {
      x = bf16_to_f(a.q[((size_t)b * a.Hq + g * gs + (v - 1)) * kD + c]);
    }
    xs[v][c] = x;
  }
}

__global__ void __launch_bounds__(kMvThreads) step_prologue_kernel(PrologueArgs a) {
  __shared__ __align__(16) float xs[kMaxStepVecs][kD];  // raw vectors
  __shared__ __align__(16) float xr[kMaxStepVecs][kD];  // rotated vectors
  __shared__ uint32_t cword[kMaxStepVecs][kWords];
  pdl_wait();
  pdl_trigger();
  const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int lrow = mv_lrow();
  const bool row_lead = (tid & 15) == 0;
  const int gs = a.Hq / a.G;

  float4 rrow[kRowBlocks][2], wrow[kRowBlocks][2];
#pragma unroll
  for (int rb = 0; rb < kRowBlocks; ++rb) {
    load_row16(a.R + (size_t)g * kD * kD, rb * 32 + lrow, rrow[rb]);
    load_row16(a.W + (size_t)g * kD * kD, rb * 32 + lrow, wrow[rb]);
  }
  const NewestSlot s = newest_slot(a, b, g, tid == 0);
  const bool has_key = s.phys >= 0;
  float mn[kRowBlocks], mx[kRowBlocks];
#pragma unroll
  for (int rb = 0; rb < kRowBlocks; ++rb) {
    mn[rb] = INFINITY;
    mx[rb] = -INFINITY;
    if (has_key && s.slot > 0 && row_lead)
      load_summary_row(a.page_minmax, a.summary_fp16, s.sbase, rb * 32 + lrow, mn[rb], mx[rb]);
  }
  load_step_vectors(a, b, g, s, true, xs, kMvThreads);
  if (tid < kMaxStepVecs * kWords) cword[tid / kWords][tid % kWords] = 0u;
  __syncthreads();

  // Vector 0 is the newest key, 1..gs the queries: the per-vector arithmetic is that of
  // encode_page_kernel and qprep_kernel.
  float qneg[kRowBlocks], qpos[kRowBlocks];
#pragma unroll
  for (int rb = 0; rb < kRowBlocks; ++rb) {
    const int row = rb * 32 + lrow;
    const float yk = row_dot16(rrow[rb], &xs[0][0]);
    if (has_key) {
      mn[rb] = fminf(mn[rb], yk);
      mx[rb] = fmaxf(mx[rb], yk);
    }
    if (row_lead) xr[0][row] = has_key ? yk : 0.f;
    qneg[rb] = 0.f;
    qpos[rb] = 0.f;
    for (int h = 0; h < gs; ++h) {
      const float y = row_dot16(rrow[rb], &xs[1 + h][0]);
      qneg[rb] += fminf(y, 0.f);
      qpos[rb] += fmaxf(y, 0.f);
      if (row_lead) {
        xr[1 + h][row] = y;
        a.q_rot[((size_t)b * a.Hq + g * gs + h) * kD + row] = y;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int rb = 0; rb < kRowBlocks; ++rb) {
    for (int v = 0; v <= gs; ++v) {
      const float p = row_dot16(wrow[rb], &xr[v][0]);
      if (row_lead && p > 0.f) atomicOr(&cword[v][rb], 1u << lrow);
    }
  }
  __syncthreads();
  if (tid < (1 + gs) * kWords) {
    const int v = tid / kWords, w = tid % kWords;
    if (v == 0) {
      if (has_key) a.codes[(((size_t)s.phys * a.G + g) * a.P + s.slot) * kWords + w] = cword[0][w];
    } else {
      a.q_code[((size_t)b * a.Hq + g * gs + (v - 1)) * kWords + w] = cword[v][w];
    }
  }
  if (row_lead) {
    float* o = a.qpn + ((size_t)b * a.G + g) * 2 * kD;
#pragma unroll
    for (int rb = 0; rb < kRowBlocks; ++rb) {
      const int row = rb * 32 + lrow;
      if (has_key) store_summary_row(a.page_minmax, a.summary_fp16, s.sbase, row, mn[rb], mx[rb]);
      o[row] = qneg[rb];
      o[kD + row] = qpos[rb];
    }
  }
}

// Cluster form of the prologue: a cluster of kPrologueRanks CTAs per (group, sequence),
// CTA r owning rows 32r..32r+31 of R_g and W_g (one row block of row_dot16 each, so every
// thread does 1/16 of a row's dot product). Each CTA rotates every vector on its 32 rows,
// the rotated vectors are assembled through distributed shared memory, and each CTA
// projects them on its 32 rows of W_g: its 32 sign bits are code word r. CTA r also owns
// summary channels and folded-query channels 32r..32r+31. Same arithmetic per value as
// step_prologue_kernel.
constexpr int kPrologueRanks = kRowBlocks;
constexpr int kPrologueThreads = kMvThreads;  // 32 rows x 16 threads

__global__ void __cluster_dims__(kPrologueRanks, 1, 1) __launch_bounds__(kPrologueThreads)
    step_prologue_cluster_kernel(PrologueArgs a) {
  namespace cg = cooperative_groups;
  __shared__ __align__(16) float xs[kMaxStepVecs][kD];     // raw vectors
  __shared__ __align__(16) float xpart[kMaxStepVecs][32];  // my rows, rotated
  __shared__ __align__(16) float xr[kMaxStepVecs][kD];     // all rows, rotated
  __shared__ uint32_t cword[kMaxStepVecs];
  pdl_wait();
  pdl_trigger();
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int lrow = mv_lrow();
  const int row = rank * 32 + lrow;
  const bool row_lead = (tid & 15) == 0;
  const int gs = a.Hq / a.G;

  float4 rr[2], wr[2];
  load_row16(a.R + (size_t)g * kD * kD, row, rr);
  load_row16(a.W + (size_t)g * kD * kD, row, wr);
  if (tid < kMaxStepVecs) cword[tid] = 0u;
  const NewestSlot s = newest_slot(a, b, g, tid == 0 && rank == 0);
  const bool has_key = s.phys >= 0;
  float mn = INFINITY, mx = -INFINITY;
  if (has_key && s.slot > 0 && row_lead) load_summary_row(a.page_minmax, a.summary_fp16, s.sbase, row, mn, mx);
  load_step_vectors(a, b, g, s, rank == 0, xs, kPrologueThreads);
  __syncthreads();

  const float yk = row_dot16(rr, &xs[0][0]);
  if (has_key) {
    mn = fminf(mn, yk);
    mx = fmaxf(mx, yk);
  }
  if (row_lead) xpart[0][lrow] = has_key ? yk : 0.f;
  float qneg = 0.f, qpos = 0.f;
  for (int h = 0; h < gs; ++h) {
    const float y = row_dot16(rr, &xs[1 + h][0]);
    qneg += fminf(y, 0.f);
    qpos += fmaxf(y, 0.f);
    if (row_lead) {
      xpart[1 + h][lrow] = y;
      a.q_rot[((size_t)b * a.Hq + g * gs + h) * kD + row] = y;
    }
  }
  cl.sync();  // every CTA's rotated rows are ready
  for (int i = tid; i < (1 + gs) * kD; i += kPrologueThreads) {
    const int v = i / kD, c = i % kD;
    xr[v][c] = cl.map_shared_rank(&xpart[0][0], c >> 5)[v * 32 + (c & 31)];
  }
  __syncthreads();
  for (int v = 0; v <= gs; ++v) {
    const float p = row_dot16(wr, &xr[v][0]);
    if (row_lead && p > 0.f) atomicOr(&cword[v], 1u << lrow);
  }
  __syncthreads();
  if (tid <= gs) {
    const uint32_t word = cword[tid];
    if (tid == 0) {
      if (has_key) a.codes[(((size_t)s.phys * a.G + g) * a.P + s.slot) * kWords + rank] = word;
    } else {
      a.q_code[((size_t)b * a.Hq + g * gs + (tid - 1)) * kWords + rank] = word;
    }
  }
  if (row_lead) {
    if (has_key) store_summary_row(a.page_minmax, a.summary_fp16, s.sbase, row, mn, mx);
    float* o = a.qpn + ((size_t)b * a.G + g) * 2 * kD;
    o[row] = qneg;
    o[kD + row] = qpos;
  }
  cl.sync();  // keep xpart alive until every CTA has read it
}

}  // namespace hhr
