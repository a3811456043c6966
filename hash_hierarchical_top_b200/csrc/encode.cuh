// Step a0, per-page key encoder (append path).
//
// HHR page, Abstract: GKR applies a head-wise orthogonal transform R_h to keys and
// summarises each page for its page-level logit bound; LHP encodes keys into binary
// codes (Figure 2 caption: a projection followed by sign). The summary is the
// per-channel min/max of the rotated keys of the page; bit j of a code is
// [(W_g R_g k)_j > 0]. HISA page, Abstract: the pooled block representative, read
// here as the mean of the block's keys.
//
// Summaries are updated incrementally: if the page already held keys before this
// append, the new min/max are merged into the stored ones (min/max are exact, so
// this equals recomputing the whole page).
#pragma once
#include "common.cuh"

namespace hhr {

// Row stride of a transposed 128x128 matrix in shared memory (padded: conflict-free
// for both the transposing stores and the column reads). Used by the bulk SIMT path.
constexpr int kTS = kD + 1;

// Mat-vecs with 128x128 row-major fp32 matrices (R_g, W_g) use one canonical row dot
// product everywhere (append encoder, query prep, fused prologues), so that their results
// are bit-identical: the 16 threads of a row each hold float4s part and part+16 of the row,
// multiply them with the same channels of the vector in a fixed fmaf order, and sum over
// the 16 parts with a 4-step butterfly (part ^ 1, ^ 2, ^ 4, ^ 8). A warp holds two rows,
// interleaved (lane = 2 part + row & 1), so that the two rows' reads of the same vector
// channels fall in the same quarter-warp and are served by one shared-memory broadcast.
// With kMvThreads = 512, a CTA covers 32 rows at a time: warp w holds rows 2w and 2w + 1
// of a 32-row block.
constexpr int kVecChunk = 4;
constexpr int kMvThreads = 512;
constexpr int kRowBlocks = kD / 32;

__device__ __forceinline__ int mv_lrow() {  // 0..31
  return (((int)threadIdx.x >> 5) << 1) | ((int)threadIdx.x & 1);
}
__device__ __forceinline__ int mv_part() { return ((int)threadIdx.x & 31) >> 1; }  // 0..15

// Row `row` of M, this thread's part (float4s part and part + 16). The loads are volatile
// asm so that they are issued here, at kernel start, and not sunk past later barriers to
// their first use (which would add a memory latency to the critical path).
__device__ __forceinline__ float4 ldg_f4_now(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];\n"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void load_row16(const float* __restrict__ M, int row, float4 (&m)[2]) {
  const int part = mv_part();
  const float4* r4 = reinterpret_cast<const float4*>(M + (size_t)row * kD);
  m[0] = ldg_f4_now(r4 + part);
  m[1] = ldg_f4_now(r4 + part + 16);
}

__device__ __forceinline__ float row_dot16(const float4 (&m)[2], const float* x) {
  const int part = mv_part();
  const float4 x0 = reinterpret_cast<const float4*>(x)[part];
  const float4 x1 = reinterpret_cast<const float4*>(x)[part + 16];
  float acc = m[0].x * x0.x;
  acc = fmaf(m[0].y, x0.y, acc);
  acc = fmaf(m[0].z, x0.z, acc);
  acc = fmaf(m[0].w, x0.w, acc);
  acc = fmaf(m[1].x, x1.x, acc);
  acc = fmaf(m[1].y, x1.y, acc);
  acc = fmaf(m[1].z, x1.z, acc);
  acc = fmaf(m[1].w, x1.w, acc);
  acc += __shfl_xor_sync(kFull, acc, 2);   // part ^ 1
  acc += __shfl_xor_sync(kFull, acc, 4);   // part ^ 2
  acc += __shfl_xor_sync(kFull, acc, 8);   // part ^ 4
  acc += __shfl_xor_sync(kFull, acc, 16);  // part ^ 8
  return acc;
}

struct EncodeArgs {
  const uint16_t* k_cache;
  const int32_t* page_table;
  const int32_t* start;
  const int32_t* n_new;
  const float* R;
  const float* W;
  void* page_minmax;   // f32 or f16 [n_phys][G][2][d]
  uint32_t* codes;
  float* block_mean;
  int G, P, maxp, n_phys, max_new;
  int summary_fp16;    // 1: store min rounded down and max rounded up to f16
};

// One CTA of kMvThreads threads per (touched page, KV group, sequence). The new keys of
// the page are processed kVecChunk at a time: k' = R_g k (row_dot16; the 16 threads of
// row r own channel r), min/max folded per channel, then p = W_g k' (32 CW rows) and the
// sign bit of row r is OR-ed into the key's code word r / 32. CW: 32-bit code words.
template <int CW>
__global__ void __launch_bounds__(kMvThreads) encode_page_kernel(EncodeArgs a) {
  __shared__ __align__(16) float kx[kVecChunk][kD];  // raw keys (fp32)
  __shared__ __align__(16) float kr[kVecChunk][kD];  // rotated keys
  __shared__ uint32_t cword[kVecChunk][CW];

  const int b = blockIdx.z, g = blockIdx.y, j = blockIdx.x;
  const int tid = threadIdx.x;
  const int P = a.P, G = a.G;

  int nn = a.n_new[b];
  if (nn > a.max_new) {
    if (tid == 0 && j == 0 && g == 0) flag_status(kStatusClipped);
    nn = a.max_new;
  }
  const int s = a.start[b];
  if (nn <= 0 || s < 0) return;
  const int e = s + nn;
  const int lp = s / P + j;
  if (lp * P >= e) return;
  if (lp >= a.maxp) {
    if (tid == 0) flag_status(kStatusBadPage);
    return;
  }
  const int phys = a.page_table[(size_t)b * a.maxp + lp];
  if (phys < 0 || phys >= a.n_phys) {
    if (tid == 0) flag_status(kStatusBadPage);
    return;
  }
  const int pstart = lp * P;
  const int t0 = max(s, pstart), t1 = min(e, pstart + P);
  const uint16_t* kpage = a.k_cache + ((size_t)phys * G + g) * P * kD;
  const int lrow = mv_lrow();
  const bool row_lead = mv_part() == 0;

  if (a.R != nullptr) {
    // R_g and W_g rows of this thread, and the page's stored summary when the page already
    // held keys, are fetched up front (one memory latency for all of them).
    float4 rrow[kRowBlocks][2], wrow[CW][2];
#pragma unroll
    for (int rb = 0; rb < kRowBlocks; ++rb) load_row16(a.R + (size_t)g * kD * kD, rb * 32 + lrow, rrow[rb]);
#pragma unroll
    for (int wb = 0; wb < CW; ++wb)
      load_row16(a.W + (size_t)g * (32 * CW) * kD, wb * 32 + lrow, wrow[wb]);
    const size_t sbase = ((size_t)phys * G + g) * 2 * kD;
    float mn[kRowBlocks], mx[kRowBlocks];
#pragma unroll
    for (int rb = 0; rb < kRowBlocks; ++rb) {
      mn[rb] = INFINITY;
      mx[rb] = -INFINITY;
      if (t0 > pstart && row_lead) {
        const int row = rb * 32 + lrow;
        if (a.summary_fp16) {
          const __half* mm = reinterpret_cast<const __half*>(a.page_minmax) + sbase;
          mn[rb] = __half2float(mm[row]);
          mx[rb] = __half2float(mm[kD + row]);
        } else {
          const float* mm = reinterpret_cast<const float*>(a.page_minmax) + sbase;
          mn[rb] = mm[row];
          mx[rb] = mm[kD + row];
        }
      }
    }
    for (int t = t0; t < t1; t += kVecChunk) {
      const int nv = min(kVecChunk, t1 - t);
      __syncthreads();
      for (int i = tid; i < kVecChunk * kD; i += kMvThreads) {
        const int v = i / kD, c = i % kD;
        kx[v][c] = v < nv ? bf16_to_f(kpage[(size_t)(t + v - pstart) * kD + c]) : 0.f;
      }
      if (tid < kVecChunk * CW) cword[tid / CW][tid % CW] = 0u;
      __syncthreads();
#pragma unroll
      for (int rb = 0; rb < kRowBlocks; ++rb) {
#pragma unroll
        for (int v = 0; v < kVecChunk; ++v) {
          const float y = row_dot16(rrow[rb], &kx[v][0]);
          if (v < nv) {
            mn[rb] = fminf(mn[rb], y);
            mx[rb] = fmaxf(mx[rb], y);
          }
          if (row_lead) kr[v][rb * 32 + lrow] = v < nv ? y : 0.f;
        }
      }
      __syncthreads();
#pragma unroll
      for (int wb = 0; wb < CW; ++wb) {
#pragma unroll
        for (int v = 0; v < kVecChunk; ++v) {
          const float p = row_dot16(wrow[wb], &kr[v][0]);
          if (row_lead && p > 0.f) atomicOr(&cword[v][wb], 1u << lrow);
        }
      }
      __syncthreads();
      if (tid < kVecChunk * CW) {
        const int v = tid / CW, w = tid % CW;
        if (v < nv) a.codes[(((size_t)phys * G + g) * P + (t + v - pstart)) * CW + w] = cword[v][w];
      }
    }
    if (row_lead) {
      // mn/mx started from the stored summary when the page already held keys (min and
      // max are exact, so merging equals recomputing the whole page).
#pragma unroll
      for (int rb = 0; rb < kRowBlocks; ++rb) {
        const int row = rb * 32 + lrow;
        if (a.summary_fp16) {
          __half* mm = reinterpret_cast<__half*>(a.page_minmax) + sbase;
          // Outward rounding keeps the stored interval around every rotated key.
          mm[row] = __float2half_rd(mn[rb]);
          mm[kD + row] = __float2half_ru(mx[rb]);
        } else {
          float* mm = reinterpret_cast<float*>(a.page_minmax) + sbase;
          mm[row] = mn[rb];
          mm[kD + row] = mx[rb];
        }
      }
    }
  }
  if (a.block_mean != nullptr && tid < kD) {
    // Mean of every valid raw key of the page, summed in ascending position order.
    float sum = 0.f;
    for (int t = pstart; t < t1; ++t) sum += bf16_to_f(kpage[(size_t)(t - pstart) * kD + tid]);
    a.block_mean[((size_t)phys * G + g) * kD + tid] = sum / (float)(t1 - pstart);
  }
}

inline size_t encode_page_smem() { return 0; }

}  // namespace hhr
