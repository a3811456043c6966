// Step a5: GQA split-K sparse attention over the selected K/V rows.
//
// HISA page, Abstract: attention is computed only over the selected subset. HHR
// appendix Table 3: Llama-3.1-8B has 32 query heads over 8 KV heads, so each
// selected row is gathered once per KV group and shared by the group's query heads.
//
// Grid (split, group, sequence); one CTA of 128 threads handles kChunk selected
// rows of one group:
//   1. gather: the chunk's K and V rows (256 B each) are copied into shared memory
//      with 16-byte cp.async (every warp instruction moves two whole rows, so the
//      random row gather is still fully coalesced); V stays in flight while the
//      logits are computed;
//   2. logits: warp w takes rows 32w..32w+31, lane l channels 4l..4l+3; the 32
//      per-row partial dot products are folded by a transposed warp reduction, so
//      lane j ends up with the logit of row j (scaled by scale*log2(e));
//   3. softmax over the chunk (exp2 of logit - chunk max), then P.V with lanes over
//      channels; the 4 warps' partial outputs are summed in shared memory;
//   4. the chunk writes its partial (max, sum, output) per head; a combine kernel
//      merges the chunks of each head (standard split softmax rescaling).
#pragma once
#include "common.cuh"

namespace hhr {

constexpr int kChunk = 128;
constexpr int kAttnThreads = 128;

struct AttnArgs {
  const uint16_t* q;        // [B][Hq][d]
  const uint16_t* k_cache;  // [n_phys][G][P][d]
  const uint16_t* v_cache;
  const int32_t* page_table;
  const int32_t* seq_len;
  const int32_t* idx;       // [B][G][top_k]
  const int32_t* count;     // [B][G]
  float* part_o;            // [B][G][n_splits][gs][d]
  float* part_ml;           // [B][G][n_splits][gs][2]
  float scale_log2;
  int Hq, G, P, maxp, n_phys, top_k, n_splits;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__global__ void __launch_bounds__(kAttnThreads) sparse_attn_kernel(AttnArgs a) {
  extern __shared__ float4 at_smem[];
  uint16_t* Ks = reinterpret_cast<uint16_t*>(at_smem);          // [kChunk][d]
  uint16_t* Vs = Ks + kChunk * kD;                               // [kChunk][d]
  float* Ls = reinterpret_cast<float*>(Vs + kChunk * kD);        // [gs][kChunk]
  long long* off = reinterpret_cast<long long*>(Ls + kMaxGroup * kChunk);  // [kChunk]
  float* ml = reinterpret_cast<float*>(off + kChunk);            // [gs][2]
  float* Os = reinterpret_cast<float*>(Ks);                      // aliases Ks after logits

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gs = a.Hq / a.G;
  const int row = b * a.G + g;
  const int cnt = min(a.count[row], a.top_k);
  const int base = split * kChunk;
  if (base >= cnt) return;
  const int nrows = min(kChunk, cnt - base);
  const int n = a.seq_len[b];

  // Row offsets (elements) of the selected rows; -1 for rows to skip.
  {
    long long o = -1;
    if (tid < nrows) {
      const int t = a.idx[(size_t)row * a.top_k + base + tid];
      const int lp = t / a.P;
      if (t >= 0 && t < n && lp < a.maxp) {
        const int phys = a.page_table[(size_t)b * a.maxp + lp];
        if (phys >= 0 && phys < a.n_phys)
          o = (((long long)phys * a.G + g) * a.P + (t % a.P)) * kD;
        else
          flag_status(kStatusBadPage);
      } else {
        flag_status(kStatusBadToken);
      }
    }
    off[tid] = o;
  }
  __syncthreads();
  // Gather: 16 pieces of 16 B per row; zero-fill skipped rows.
  for (int c = tid; c < kChunk * 16; c += kAttnThreads) {
    const int r = c >> 4, piece = c & 15;
    const long long o = off[r];
    if (o >= 0) cp_async16(Ks + r * kD + piece * 8, a.k_cache + o + piece * 8);
    else *reinterpret_cast<uint4*>(Ks + r * kD + piece * 8) = make_uint4(0, 0, 0, 0);
  }
  cp_async_commit();
  for (int c = tid; c < kChunk * 16; c += kAttnThreads) {
    const int r = c >> 4, piece = c & 15;
    const long long o = off[r];
    if (o >= 0) cp_async16(Vs + r * kD + piece * 8, a.v_cache + o + piece * 8);
    else *reinterpret_cast<uint4*>(Vs + r * kD + piece * 8) = make_uint4(0, 0, 0, 0);
  }
  cp_async_commit();

  // Query pieces of the group's heads (channels 4*lane..4*lane+3), pre-scaled.
  float4 qv[kMaxGroup];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    if (h < gs) {
      uint2 w = *reinterpret_cast<const uint2*>(a.q + ((size_t)b * a.Hq + g * gs + h) * kD +
                                                4 * lane);
      float4 f = bf16x4_to_f4(w);
      qv[h] = make_float4(f.x * a.scale_log2, f.y * a.scale_log2, f.z * a.scale_log2,
                          f.w * a.scale_log2);
    } else {
      qv[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  cp_async_wait<1>();
  __syncthreads();

  // Logits: warp w, rows 32w..32w+31.
  const int r0 = warp * 32;
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    if (h >= gs) break;
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float4 kf = bf16x4_to_f4(*reinterpret_cast<const uint2*>(Ks + (r0 + j) * kD + 4 * lane));
      v[j] = qv[h].x * kf.x + qv[h].y * kf.y + qv[h].z * kf.z + qv[h].w * kf.w;
    }
    float lg = warp_transpose_sum32(v, lane);
    const int r = r0 + lane;
    Ls[h * kChunk + r] = (r < nrows && off[r] >= 0) ? lg : -INFINITY;
  }
  __syncthreads();

  // Softmax statistics per head: warp w handles heads w, w+4, ...
  for (int h = warp; h < gs; h += kAttnThreads / 32) {
    float x[kChunk / 32];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kChunk / 32; ++i) { x[i] = Ls[h * kChunk + lane + 32 * i]; mx = fmaxf(mx, x[i]); }
    mx = warp_max(mx);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kChunk / 32; ++i) {
      float p = (mx == -INFINITY) ? 0.f : exp2f(x[i] - mx);
      Ls[h * kChunk + lane + 32 * i] = p;
      s += p;
    }
    s = warp_sum(s);
    if (lane == 0) { ml[2 * h] = mx; ml[2 * h + 1] = s; }
  }
  cp_async_wait<0>();
  __syncthreads();

  // P.V: warp w, rows 32w..32w+31; lane l owns channels 4l..4l+3.
  float4 acc[kMaxGroup];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int rend = min(32, nrows - r0);
  for (int j = 0; j < rend; ++j) {
    const int r = r0 + j;
    float4 vf = bf16x4_to_f4(*reinterpret_cast<const uint2*>(Vs + r * kD + 4 * lane));
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      if (h < gs) {
        float p = Ls[h * kChunk + r];
        acc[h].x = fmaf(p, vf.x, acc[h].x);
        acc[h].y = fmaf(p, vf.y, acc[h].y);
        acc[h].z = fmaf(p, vf.z, acc[h].z);
        acc[h].w = fmaf(p, vf.w, acc[h].w);
      }
    }
  }
  // Ks is dead now: reuse it for the per-warp partial outputs [4][gs][d].
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h)
    if (h < gs) reinterpret_cast<float4*>(Os + ((size_t)warp * gs + h) * kD)[lane] = acc[h];
  __syncthreads();
  const size_t pbase = ((size_t)row * a.n_splits + split) * gs;
  for (int i = tid; i < gs * kD; i += kAttnThreads) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnThreads / 32; ++w) s += Os[(size_t)w * gs * kD + i];
    a.part_o[pbase * kD + i] = s;
  }
  if (tid < gs) {
    a.part_ml[(pbase + tid) * 2] = ml[2 * tid];
    a.part_ml[(pbase + tid) * 2 + 1] = ml[2 * tid + 1];
  }
}

inline size_t attn_smem() {
  return (size_t)2 * kChunk * kD * 2 + (size_t)kMaxGroup * kChunk * 4 + (size_t)kChunk * 8 +
         kMaxGroup * 2 * 4;
}

// Merge of the chunk partials of one head: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
struct CombineArgs {
  const float* part_o;
  const float* part_ml;
  const int32_t* count;
  float* out;  // [B][Hq][d]
  int Hq, G, top_k, n_splits;
};

__global__ void __launch_bounds__(kD) attn_combine_kernel(CombineArgs a) {
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int gs = a.Hq / a.G, g = h / gs, hh = h % gs;
  const int row = b * a.G + g;
  const int cnt = min(a.count[row], a.top_k);
  const int ns = ceil_div(max(cnt, 0), kChunk);
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s)
    M = fmaxf(M, a.part_ml[(((size_t)row * a.n_splits + s) * gs + hh) * 2]);
  float L = 0.f, o = 0.f;
  if (M > -INFINITY) {
    for (int s = 0; s < ns; ++s) {
      const size_t p = ((size_t)row * a.n_splits + s) * gs + hh;
      const float m = a.part_ml[p * 2];
      if (m == -INFINITY) continue;
      const float w = exp2f(m - M);
      L = fmaf(w, a.part_ml[p * 2 + 1], L);
      o = fmaf(w, a.part_o[p * kD + tid], o);
    }
  }
  a.out[((size_t)b * a.Hq + h) * kD + tid] = (L > 0.f) ? o / L : 0.f;
}

}  // namespace hhr
