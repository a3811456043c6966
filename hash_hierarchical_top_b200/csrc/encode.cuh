// Step a0, per-page key encoder (append path).
//
// HHR page, Abstract: GKR applies a head-wise orthogonal transform R_h to keys and
// summarises each page for its page-level logit bound; LHP encodes keys into binary
// codes (Figure 2 caption: a projection followed by sign). The summary is the
// per-channel min/max of the rotated keys of the page; bit j of a code is
// [(W_g R_g k)_j > 0]. HISA page, Abstract: the pooled block representative, read
// here as the mean of the block's keys.
//
// One CTA of 128 threads per (touched page, KV group, sequence). Thread i owns
// channel i of the rotated key and bit i of the code. R_g^T and W_g^T are staged
// in shared memory (transposed, so thread i reads column i without bank conflicts).
// Summaries are updated incrementally: if the page already held keys before this
// append, the new min/max are merged into the stored ones (min/max are exact, so
// this equals recomputing the whole page).
#pragma once
#include "common.cuh"

namespace hhr {

// Row stride of a transposed 128x128 matrix in shared memory (padded: conflict-free
// for both the transposing stores and the column reads).
constexpr int kTS = kD + 1;

// T[c][r] = M[r][c] for a 128x128 row-major fp32 matrix M; coalesced global reads.
__device__ __forceinline__ void stage_transposed(const float* __restrict__ M, float* T) {
  for (int idx = threadIdx.x; idx < kD * kD; idx += blockDim.x) {
    int r = idx >> 7, c = idx & 127;
    T[c * kTS + r] = M[idx];
  }
}

struct EncodeArgs {
  const uint16_t* k_cache;
  const int32_t* page_table;
  const int32_t* start;
  const int32_t* n_new;
  const float* R;
  const float* W;
  float* page_minmax;
  uint32_t* codes;
  float* block_mean;
  int G, P, maxp, n_phys, max_new;
};

__global__ void __launch_bounds__(128) encode_page_kernel(EncodeArgs a) {
  extern __shared__ float4 smem_f4[];
  float* RT = reinterpret_cast<float*>(smem_f4);        // [128][kTS], RT[j][i] = R[i][j]
  float* WT = RT + kD * kTS;                             // [128][kTS], WT[i][j] = W[j][i]
  float* kx = WT + kD * kTS;                              // raw key (fp32)
  float* kr = kx + kD;                                    // rotated key

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
  const bool hashing = (a.R != nullptr);
  const uint16_t* kpage = a.k_cache + ((size_t)phys * G + g) * P * kD;

  if (hashing) {
    const float* Rg = a.R + (size_t)g * kD * kD;
    const float* Wg = a.W + (size_t)g * kD * kD;
    stage_transposed(Rg, RT);
    stage_transposed(Wg, WT);
  }
  __syncthreads();

  float mn = INFINITY, mx = -INFINITY;
  if (hashing) {
    for (int t = t0; t < t1; ++t) {
      kx[tid] = bf16_to_f(kpage[(size_t)(t - pstart) * kD + tid]);
      __syncthreads();
      float acc = 0.f;
#pragma unroll 8
      for (int c = 0; c < kD; ++c) acc = fmaf(RT[c * kTS + tid], kx[c], acc);
      kr[tid] = acc;
      mn = fminf(mn, acc);
      mx = fmaxf(mx, acc);
      __syncthreads();
      float p = 0.f;
#pragma unroll 8
      for (int c = 0; c < kD; ++c) p = fmaf(WT[c * kTS + tid], kr[c], p);
      unsigned word = __ballot_sync(kFull, p > 0.f);
      if (lane == 0)
        a.codes[(((size_t)phys * G + g) * P + (t - pstart)) * kWords + warp] = word;
      __syncthreads();
    }
    float* mm = a.page_minmax + ((size_t)phys * G + g) * 2 * kD;
    if (t0 > pstart) {  // the page already held keys: merge with its stored summary
      mn = fminf(mn, mm[tid]);
      mx = fmaxf(mx, mm[kD + tid]);
    }
    mm[tid] = mn;
    mm[kD + tid] = mx;
  }
  if (a.block_mean != nullptr) {
    // Mean of every valid raw key of the page, summed in ascending position order.
    float sum = 0.f;
    for (int t = pstart; t < t1; ++t) sum += bf16_to_f(kpage[(size_t)(t - pstart) * kD + tid]);
    a.block_mean[((size_t)phys * G + g) * kD + tid] = sum / (float)(t1 - pstart);
  }
}

inline size_t encode_page_smem() { return (size_t)(2 * kD * kTS + 2 * kD) * sizeof(float); }

}  // namespace hhr
