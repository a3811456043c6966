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

// y_v = M x_v for up to kVecChunk vectors at once, M a 128x128 row-major fp32 matrix
// in global memory (L1/L2-resident: it is shared by every CTA of a group).
// Warp w computes rows 32w..32w+31: lane l reads float4 l of each row (a coalesced
// 512-byte row read per instruction), multiplies it with channels 4l..4l+3 of every
// vector, and a transposed warp reduction leaves y_v[32w + l] on lane l. Each row of
// M is read once per call for all vectors. Requires blockDim.x == 128.
constexpr int kVecChunk = 4;

template <int NV>
__device__ __forceinline__ void matvec_rows(const float* __restrict__ M, const float* xs,
                                            int xs_stride, float (&y)[NV]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float4 xv[NV];
#pragma unroll
  for (int v = 0; v < NV; ++v) xv[v] = reinterpret_cast<const float4*>(xs + v * xs_stride)[lane];
  float acc[NV][32];
  const float4* Mr = reinterpret_cast<const float4*>(M + (size_t)(warp * 32) * kD) + lane;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float4 m = __ldg(Mr + j * (kD / 4));
#pragma unroll
    for (int v = 0; v < NV; ++v)
      acc[v][j] = m.x * xv[v].x + m.y * xv[v].y + m.z * xv[v].z + m.w * xv[v].w;
  }
#pragma unroll
  for (int v = 0; v < NV; ++v) y[v] = warp_transpose_sum32(acc[v], lane);
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

// One CTA of 128 threads per (touched page, KV group, sequence). The new keys of
// the page are processed kVecChunk at a time: k' = R_g k (thread 32w+l ends up
// owning channel 32w+l), min/max folded per channel, then p = W_g k' and the code
// word of warp w is the ballot of its 32 sign bits.
__global__ void __launch_bounds__(128) encode_page_kernel(EncodeArgs a) {
  __shared__ __align__(16) float kx[kVecChunk][kD];  // raw keys (fp32)
  __shared__ __align__(16) float kr[kVecChunk][kD];  // rotated keys

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

  if (a.R != nullptr) {
    const float* Rg = a.R + (size_t)g * kD * kD;
    const float* Wg = a.W + (size_t)g * kD * kD;
    float mn = INFINITY, mx = -INFINITY;
    for (int t = t0; t < t1; t += kVecChunk) {
      const int nv = min(kVecChunk, t1 - t);
      __syncthreads();
      for (int v = 0; v < kVecChunk; ++v)
        kx[v][tid] = v < nv ? bf16_to_f(kpage[(size_t)(t + v - pstart) * kD + tid]) : 0.f;
      __syncthreads();
      float y[kVecChunk];
      matvec_rows<kVecChunk>(Rg, &kx[0][0], kD, y);
#pragma unroll
      for (int v = 0; v < kVecChunk; ++v) {
        if (v < nv) {
          kr[v][tid] = y[v];
          mn = fminf(mn, y[v]);
          mx = fmaxf(mx, y[v]);
        } else {
          kr[v][tid] = 0.f;
        }
      }
      __syncthreads();
      float p[kVecChunk];
      matvec_rows<kVecChunk>(Wg, &kr[0][0], kD, p);
#pragma unroll
      for (int v = 0; v < kVecChunk; ++v) {
        const unsigned word = __ballot_sync(kFull, p[v] > 0.f);
        if (v < nv && lane == 0)
          a.codes[(((size_t)phys * G + g) * P + (t + v - pstart)) * kWords + warp] = word;
      }
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

inline size_t encode_page_smem() { return 0; }

}  // namespace hhr
