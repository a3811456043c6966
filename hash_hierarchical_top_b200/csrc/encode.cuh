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

// y_v = M x_v for up to kVecChunk vectors at once, M a 128x128 row-major fp32 matrix,
// with kMvThreads = 512 threads: 4 threads per row. Thread (row r = 8*warp + lane/4,
// quarter q = lane%4) holds float4s q, q+4, ..., q+28 of row r in registers (the four
// threads of a row read 64 contiguous bytes per load), dots them with the same float4s
// of each vector (shared-memory broadcasts), and two shuffles sum the four quarters.
// Every thread of a row ends up with y_v[r].
constexpr int kVecChunk = 4;
constexpr int kMvThreads = 512;

__device__ __forceinline__ int mv_row() { return (threadIdx.x >> 5) * 8 + ((threadIdx.x & 31) >> 2); }

// This thread's quarter of its row of M (8 float4).
__device__ __forceinline__ void load_rows8(const float* __restrict__ M, float4 (&m)[8]) {
  const int q = threadIdx.x & 3;
  const float4* Mr = reinterpret_cast<const float4*>(M + (size_t)mv_row() * kD);
#pragma unroll
  for (int j = 0; j < 8; ++j) m[j] = __ldg(Mr + 4 * j + q);
}

template <int NV>
__device__ __forceinline__ void matvec8(const float4 (&m)[8], const float* xs, int xs_stride,
                                        float (&y)[NV]) {
  const int q = threadIdx.x & 3;
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const float4* xv = reinterpret_cast<const float4*>(xs + v * xs_stride);
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 x = xv[4 * j + q];
      acc = fmaf(m[j].x, x.x, fmaf(m[j].y, x.y, fmaf(m[j].z, x.z, fmaf(m[j].w, x.w, acc))));
    }
    acc += __shfl_xor_sync(kFull, acc, 1);
    acc += __shfl_xor_sync(kFull, acc, 2);
    y[v] = acc;
  }
}

// The 8 sign bits of this warp's rows (8*warp .. 8*warp+7) from a ballot in which the
// lanes 4i carry row 8*warp + i.
__device__ __forceinline__ uint32_t row_bits8(bool positive) {
  const unsigned b = __ballot_sync(kFull, positive);
  uint32_t byte = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) byte |= ((b >> (4 * i)) & 1u) << i;
  return byte;
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
// the page are processed kVecChunk at a time: k' = R_g k (the 4 threads of row r own
// channel r), min/max folded per channel, then p = W_g k'; each warp contributes the 8
// sign bits of its rows as one byte of the code.
__global__ void __launch_bounds__(kMvThreads) encode_page_kernel(EncodeArgs a) {
  __shared__ __align__(16) float kx[kVecChunk][kD];  // raw keys (fp32)
  __shared__ __align__(16) float kr[kVecChunk][kD];  // rotated keys
  __shared__ __align__(16) uint8_t cbytes[kVecChunk][16];

  const int b = blockIdx.z, g = blockIdx.y, j = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
  const int row = mv_row();  // channel / code bit owned after a matvec
  const bool row_lead = (lane & 3) == 0;

  if (a.R != nullptr) {
    // R_g and W_g rows of this thread, and the page's stored summary when the page already
    // held keys, are fetched up front (one memory latency for all of them).
    float4 rrow[8], wrow[8];
    load_rows8(a.R + (size_t)g * kD * kD, rrow);
    load_rows8(a.W + (size_t)g * kD * kD, wrow);
    const size_t sbase = ((size_t)phys * G + g) * 2 * kD;
    float mn = INFINITY, mx = -INFINITY;
    if (t0 > pstart && row_lead) {
      if (a.summary_fp16) {
        const __half* mm = reinterpret_cast<const __half*>(a.page_minmax) + sbase;
        mn = __half2float(mm[row]);
        mx = __half2float(mm[kD + row]);
      } else {
        const float* mm = reinterpret_cast<const float*>(a.page_minmax) + sbase;
        mn = mm[row];
        mx = mm[kD + row];
      }
    }
    for (int t = t0; t < t1; t += kVecChunk) {
      const int nv = min(kVecChunk, t1 - t);
      __syncthreads();
      for (int i = tid; i < kVecChunk * kD; i += kMvThreads) {
        const int v = i / kD, c = i % kD;
        kx[v][c] = v < nv ? bf16_to_f(kpage[(size_t)(t + v - pstart) * kD + c]) : 0.f;
      }
      __syncthreads();
      float y[kVecChunk];
      matvec8<kVecChunk>(rrow, &kx[0][0], kD, y);
#pragma unroll
      for (int v = 0; v < kVecChunk; ++v) {
        if (v < nv) {
          mn = fminf(mn, y[v]);
          mx = fmaxf(mx, y[v]);
        }
        if (row_lead) kr[v][row] = v < nv ? y[v] : 0.f;
      }
      __syncthreads();
      float p[kVecChunk];
      matvec8<kVecChunk>(wrow, &kr[0][0], kD, p);
#pragma unroll
      for (int v = 0; v < kVecChunk; ++v) {
        const uint32_t bits = row_bits8(p[v] > 0.f);  // rows 8w..8w+7
        if (lane == 0) cbytes[v][warp] = (uint8_t)bits;
      }
      __syncthreads();
      if (tid < kVecChunk * kWords) {
        const int v = tid / kWords, w = tid % kWords;
        if (v < nv)
          a.codes[(((size_t)phys * G + g) * P + (t + v - pstart)) * kWords + w] =
              reinterpret_cast<const uint32_t*>(cbytes[v])[w];
      }
    }
    if (row_lead) {
      // mn/mx started from the stored summary when the page already held keys (min and
      // max are exact, so merging equals recomputing the whole page).
      if (a.summary_fp16) {
        __half* mm = reinterpret_cast<__half*>(a.page_minmax) + sbase;
        // Outward rounding keeps the stored interval around every rotated key.
        mm[row] = __float2half_rd(mn);
        mm[kD + row] = __float2half_ru(mx);
      } else {
        float* mm = reinterpret_cast<float*>(a.page_minmax) + sbase;
        mm[row] = mn;
        mm[kD + row] = mx;
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
