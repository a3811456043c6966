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

constexpr int kMaxStepVecs = 1 + kMaxGroup;                 // newest key + query heads
constexpr int kStepChunks = (kMaxStepVecs + kVecChunk - 1) / kVecChunk;

__global__ void __launch_bounds__(kMvThreads) step_prologue_kernel(PrologueArgs a) {
  __shared__ __align__(16) float xs[kStepChunks * kVecChunk][kD];  // raw vectors
  __shared__ __align__(16) float xr[kStepChunks * kVecChunk][kD];  // rotated vectors
  __shared__ __align__(16) uint8_t cbytes[kStepChunks * kVecChunk][16];
  pdl_wait();
  pdl_trigger();
  const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int row = mv_row();
  const bool row_lead = (lane & 3) == 0;
  const int gs = a.Hq / a.G, G = a.G, P = a.P;
  const int nv = 1 + gs;

  float4 rrow[8], wrow[8];
  load_rows8(a.R + (size_t)g * kD * kD, rrow);
  load_rows8(a.W + (size_t)g * kD * kD, wrow);

  // The newest key's slot in the paged cache.
  const int t = a.seq_len[b] - 1;
  const int lp = t >= 0 ? t / P : -1;
  int phys = -1;
  if (t >= 0 && lp < a.maxp) {
    phys = a.page_table[(size_t)b * a.maxp + lp];
    if (phys < 0 || phys >= a.n_phys) phys = -1;
  }
  if (t >= 0 && phys < 0 && tid == 0) flag_status(kStatusBadPage);
  const bool has_key = phys >= 0;
  const int slot = has_key ? t - lp * P : 0;
  const size_t krow = has_key ? (((size_t)phys * G + g) * P + slot) * kD : 0;
  const size_t sbase = ((size_t)(has_key ? phys : 0) * G + g) * 2 * kD;

  // Stored summary of a page that already held keys (prefetched).
  float mn = INFINITY, mx = -INFINITY;
  if (has_key && slot > 0 && row_lead) {
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

  // Vector 0: the newest key (written to the cache first when given); 1..gs: the queries.
  for (int i = tid; i < kStepChunks * kVecChunk * kD; i += kMvThreads) {
    const int v = i / kD, c = i % kD;
    float x = 0.f;
    if (v == 0) {
      if (has_key) {
        uint16_t kb;
        if (a.k_new != nullptr) {
          kb = a.k_new[((size_t)b * G + g) * kD + c];
          a.k_cache[krow + c] = kb;
          if (a.v_new != nullptr) a.v_cache[krow + c] = a.v_new[((size_t)b * G + g) * kD + c];
        } else {
          kb = a.k_cache[krow + c];
        }
        x = bf16_to_f(kb);
      }
    } else if (v <= gs) {
      x = bf16_to_f(a.q[((size_t)b * a.Hq + g * gs + (v - 1)) * kD + c]);
    }
    xs[v][c] = x;
    xr[v][c] = 0.f;
  }
  __syncthreads();

  float qneg = 0.f, qpos = 0.f;
#pragma unroll
  for (int ch = 0; ch < kStepChunks; ++ch) {
    if (ch * kVecChunk >= nv) break;
    float y[kVecChunk];
    matvec8<kVecChunk>(rrow, &xs[ch * kVecChunk][0], kD, y);
#pragma unroll
    for (int v = 0; v < kVecChunk; ++v) {
      const int vi = ch * kVecChunk + v;
      if (vi == 0) {
        if (has_key) {
          mn = fminf(mn, y[v]);
          mx = fmaxf(mx, y[v]);
        }
      } else if (vi < nv) {
        qneg += fminf(y[v], 0.f);
        qpos += fmaxf(y[v], 0.f);
        if (row_lead) a.q_rot[((size_t)b * a.Hq + g * gs + (vi - 1)) * kD + row] = y[v];
      }
      if (row_lead && vi < nv) xr[vi][row] = y[v];
    }
  }
  __syncthreads();
#pragma unroll
  for (int ch = 0; ch < kStepChunks; ++ch) {
    if (ch * kVecChunk >= nv) break;
    float p[kVecChunk];
    matvec8<kVecChunk>(wrow, &xr[ch * kVecChunk][0], kD, p);
#pragma unroll
    for (int v = 0; v < kVecChunk; ++v) {
      const uint32_t bits = row_bits8(p[v] > 0.f);
      if (lane == 0) cbytes[ch * kVecChunk + v][warp] = (uint8_t)bits;
    }
  }
  __syncthreads();
  if (tid < nv * kWords) {
    const int v = tid / kWords, w = tid % kWords;
    const uint32_t word = reinterpret_cast<const uint32_t*>(cbytes[v])[w];
    if (v == 0) {
      if (has_key) a.codes[(((size_t)phys * G + g) * P + slot) * kWords + w] = word;
    } else {
      a.q_code[((size_t)b * a.Hq + g * gs + (v - 1)) * kWords + w] = word;
    }
  }
  if (row_lead) {
    if (has_key) {
      if (a.summary_fp16) {
        __half* mm = reinterpret_cast<__half*>(a.page_minmax) + sbase;
        mm[row] = __float2half_rd(mn);  // outward rounding, as in encode_page_kernel
        mm[kD + row] = __float2half_ru(mx);
      } else {
        float* mm = reinterpret_cast<float*>(a.page_minmax) + sbase;
        mm[row] = mn;
        mm[kD + row] = mx;
      }
    }
    float* o = a.qpn + ((size_t)b * a.G + g) * 2 * kD;
    o[row] = qneg;
    o[kD + row] = qpos;
  }
}

}  // namespace hhr
