// Step a5: GQA split-K sparse attention over the selected K/V rows.
//
// HISA page, Abstract: attention is computed only over the selected subset. HHR
// appendix Table 3: Llama-3.1-8B has 32 query heads over 8 KV heads, so each
// selected row is gathered once per KV group and shared by the group's query heads.
//
// Grid (split, group, sequence); one CTA of 8 warps streams one split of a group's
// selected rows through a 3-stage cp.async pipeline of 64-row tiles:
//   1. gather: each tile's K and V rows (256 B each) are copied into shared memory
//      with 16-byte cp.async; consecutive threads copy consecutive pieces of a row,
//      so the random row gather stays coalesced; two tiles are in flight while one
//      is computed;
//   2. logits: warp w takes 8 rows of the tile, lane l channels 4l..4l+3; the
//      8 rows x 4 heads partial dot products are folded by one transposed warp
//      reduction, so each lane ends up with one (row, head) logit;
//   3. every warp keeps its own online softmax (running max, sum and output per
//      head) over its rows; P.V runs with lanes over channels;
//   4. the 8 warps are merged in shared memory; a split writes its partial (max,
//      sum, output) per head, or the final output when the group is not split; a
//      combine kernel merges the splits (standard split softmax rescaling).
#pragma once
#include "common.cuh"

namespace hhr {

constexpr int kAttnWarps = 8;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kTile = 64;                        // selected rows per pipeline stage
constexpr int kRowsPerWarp = kTile / kAttnWarps; // 8
constexpr int kStages = 3;
constexpr int kMaxSplitRows = 2048;              // rows of one split (offsets in smem)
constexpr int kTargetCtas = 2 * 148;             // two resident CTAs on each of 148 SMs

struct AttnArgs {
  const uint16_t* q;        // [B][Hq][d]
  const uint16_t* k_cache;  // [n_phys][G][P][d]
  const uint16_t* v_cache;
  const int32_t* page_table;
  const int32_t* seq_len;
  const int32_t* idx;       // [B][G][top_k]
  const int32_t* count;     // [B][G]
  float* part_o;            // [B][G][n_splits][gs][d]   (n_splits > 1)
  float* part_ml;           // [B][G][n_splits][gs][2]
  float* out;               // [B][Hq][d]                 (n_splits == 1)
  float scale_log2;
  int Hq, G, P, maxp, n_phys, top_k, n_splits, split_rows;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Shared memory: kStages x (K tile + V tile) of 64 rows x 256 B, the split's row
// offsets, and per-warp softmax weights. The merge area reuses the stage buffers.
inline size_t attn_smem() {
  return (size_t)kStages * 2 * kTile * kD * 2 + (size_t)kMaxSplitRows * 8 +
         (size_t)kAttnWarps * kRowsPerWarp * kMaxGroup * 4 + 64;
}

// GS: compile-time capacity of query heads per group (4 or 8); gs <= GS is masked.
template <int GS>
__global__ void __launch_bounds__(kAttnThreads, GS <= 4 ? 2 : 1) sparse_attn_kernel(AttnArgs a) {
  extern __shared__ float4 at_smem[];
  uint16_t* stage_base = reinterpret_cast<uint16_t*>(at_smem);             // [kStages][2][kTile][d]
  long long* offs = reinterpret_cast<long long*>(stage_base + (size_t)kStages * 2 * kTile * kD);
  float* pbuf = reinterpret_cast<float*>(offs + kMaxSplitRows);             // [warps][8 rows][8 heads]

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gs = a.Hq / a.G;
  const int row = b * a.G + g;
  const int cnt = min(a.count[row], a.top_k);
  const int base = split * a.split_rows;
  if (base >= cnt) return;
  const int nrows = min(a.split_rows, cnt - base);
  const int ntiles = (nrows + kTile - 1) / kTile;
  const int n = a.seq_len[b];

  // Element offsets of the split's rows (-1: skip the row).
  for (int r = tid; r < ntiles * kTile; r += kAttnThreads) {
    long long o = -1;
    if (r < nrows) {
      const int t = a.idx[(size_t)row * a.top_k + base + r];
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
    offs[r] = o;
  }
  __syncthreads();

  // Issue the K and V rows of tile t into stage slot t % kStages: 64 rows x 32 pieces of
  // 16 B; consecutive threads copy consecutive pieces of a row (coalesced 256-byte rows).
  auto issue = [&](int t) {
    uint16_t* Ks = stage_base + (size_t)(t % kStages) * 2 * kTile * kD;
    uint16_t* Vs = Ks + kTile * kD;
#pragma unroll
    for (int i = 0; i < (kTile * 16) / kAttnThreads; ++i) {
      const int c = tid + i * kAttnThreads;
      const int r = c >> 4, piece = c & 15;
      const long long o = offs[t * kTile + r];
      uint16_t* kd = Ks + r * kD + piece * 8;
      uint16_t* vd = Vs + r * kD + piece * 8;
      if (o >= 0) {
        cp_async16(kd, a.k_cache + o + piece * 8);
        cp_async16(vd, a.v_cache + o + piece * 8);
      } else {
        *reinterpret_cast<uint4*>(kd) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(vd) = make_uint4(0, 0, 0, 0);
      }
    }
  };
#pragma unroll
  for (int t = 0; t < kStages - 1; ++t) {
    if (t < ntiles) issue(t);
    cp_async_commit();
  }

  // Query channels 4*lane..4*lane+3 of the group's heads, pre-scaled by scale*log2(e).
  float4 qv[GS];
#pragma unroll
  for (int h = 0; h < GS; ++h) {
    qv[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (h < gs) {
      const float4 f = bf16x4_to_f4(*reinterpret_cast<const uint2*>(
          a.q + ((size_t)b * a.Hq + g * gs + h) * kD + 4 * lane));
      qv[h] = make_float4(f.x * a.scale_log2, f.y * a.scale_log2, f.z * a.scale_log2,
                          f.w * a.scale_log2);
    }
  }
  // Per-warp running softmax state of every head (lane-replicated m and l).
  float m_run[GS], l_run[GS];
  float4 o_acc[GS];
#pragma unroll
  for (int h = 0; h < GS; ++h) {
    m_run[h] = -INFINITY;
    l_run[h] = 0.f;
    o_acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float* pw = pbuf + warp * kRowsPerWarp * kMaxGroup;  // [8 rows][8 heads]

  for (int t = 0; t < ntiles; ++t) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (t + kStages - 1 < ntiles) issue(t + kStages - 1);
    cp_async_commit();
    const uint16_t* Ks = stage_base + (size_t)(t % kStages) * 2 * kTile * kD;
    const uint16_t* Vs = Ks + kTile * kD;
    const int r0 = warp * kRowsPerWarp;          // this warp's 8 rows of the tile
    const int rbase = t * kTile + r0;            // their index within the split
    float4 kf[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
      kf[r] = bf16x4_to_f4(*reinterpret_cast<const uint2*>(Ks + (r0 + r) * kD + 4 * lane));
    // Heads in passes of 4: value index r*4 + hh -> after the transposed reduction lane l
    // holds the logit of row l/4 and head (pass*4 + l%4).
#pragma unroll
    for (int h0 = 0; h0 < GS; h0 += 4) {
      if (h0 >= gs) break;
      float acc[32];
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const float4 qq = qv[h0 + hh];
          acc[r * 4 + hh] = qq.x * kf[r].x + qq.y * kf[r].y + qq.z * kf[r].z + qq.w * kf[r].w;
        }
      float lg = warp_transpose_sum32(acc, lane);
      const int my_r = lane >> 2, my_h = h0 + (lane & 3);
      const bool valid = (my_h < gs) && (rbase + my_r < nrows) && offs[rbase + my_r] >= 0;
      lg = valid ? lg : -INFINITY;
      // Max over the 8 rows of each head: lanes with equal lane%4 (xor 4, 8, 16).
      float mx = lg;
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
      // Lane l now knows the tile max of head h0 + l%4; fetch each head's onto every lane.
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        const int h = h0 + hh;
        const float tmax = __shfl_sync(kFull, mx, hh);
        const float m_new = fmaxf(m_run[h], tmax);
        const float corr = (m_new == -INFINITY) ? 1.f : exp2f(m_run[h] - m_new);
        m_run[h] = m_new;
        l_run[h] *= corr;
        o_acc[h].x *= corr; o_acc[h].y *= corr; o_acc[h].z *= corr; o_acc[h].w *= corr;
      }
      float m_h = 0.f;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh)
        if ((lane & 3) == hh) m_h = m_run[h0 + hh];
      const float p = (lg == -INFINITY) ? 0.f : exp2f(lg - m_h);
      float ps = p;
      ps += __shfl_xor_sync(kFull, ps, 4);
      ps += __shfl_xor_sync(kFull, ps, 8);
      ps += __shfl_xor_sync(kFull, ps, 16);
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) l_run[h0 + hh] += __shfl_sync(kFull, ps, hh);
      pw[my_r * kMaxGroup + (lane & 3) + h0] = p;
    }
    __syncwarp();
    // P.V over the warp's 8 rows; lane l owns channels 4l..4l+3.
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const float4 vf = bf16x4_to_f4(*reinterpret_cast<const uint2*>(Vs + (r0 + r) * kD + 4 * lane));
#pragma unroll
      for (int h = 0; h < GS; ++h) {
        if (h < gs) {
          const float p = pw[r * kMaxGroup + h];
          o_acc[h].x = fmaf(p, vf.x, o_acc[h].x);
          o_acc[h].y = fmaf(p, vf.y, o_acc[h].y);
          o_acc[h].z = fmaf(p, vf.z, o_acc[h].z);
          o_acc[h].w = fmaf(p, vf.w, o_acc[h].w);
        }
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncthreads();

  // Merge the 8 warps' states: o = sum_w 2^(m_w - M) o_w, l = sum_w 2^(m_w - M) l_w.
  float* mo = reinterpret_cast<float*>(stage_base);             // [warps][8 heads][d]
  float* mml = mo + (size_t)kAttnWarps * kMaxGroup * kD;         // [warps][8 heads][2]
#pragma unroll
  for (int h = 0; h < GS; ++h) {
    if (h < gs) {
      reinterpret_cast<float4*>(mo + ((size_t)warp * kMaxGroup + h) * kD)[lane] = o_acc[h];
      if (lane == 0) {
        mml[(warp * kMaxGroup + h) * 2] = m_run[h];
        mml[(warp * kMaxGroup + h) * 2 + 1] = l_run[h];
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < gs * kD; i += kAttnThreads) {
    const int h = i / kD, c = i % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, mml[(w * kMaxGroup + h) * 2]);
    float L = 0.f, O = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float mw = mml[(w * kMaxGroup + h) * 2];
        const float sc = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        L = fmaf(sc, mml[(w * kMaxGroup + h) * 2 + 1], L);
        O = fmaf(sc, mo[((size_t)w * kMaxGroup + h) * kD + c], O);
      }
    }
    if (a.n_splits == 1) {
      a.out[((size_t)b * a.Hq + g * gs + h) * kD + c] = (L > 0.f) ? O / L : 0.f;
    } else {
      const size_t p = ((size_t)row * a.n_splits + split) * gs + h;
      a.part_o[p * kD + c] = O;
      if (c == 0) {
        a.part_ml[p * 2] = M;
        a.part_ml[p * 2 + 1] = L;
      }
    }
  }
}

// Split plan: about two resident CTAs per SM over the whole batch, at most
// kMaxSplitRows rows per split, splits of whole 64-row tiles.
struct AttnPlan {
  int n_splits, split_rows;
};
inline AttnPlan attn_plan(int B, int G, int top_k) {
  const long long rows = (long long)B * G;
  int s = (int)(kTargetCtas / (rows > 0 ? rows : 1));
  if (s < 1) s = 1;
  const int max_s = (top_k + kTile - 1) / kTile;
  if (s > max_s) s = max_s;
  const int min_s = (top_k + kMaxSplitRows - 1) / kMaxSplitRows;
  if (s < min_s) s = min_s;
  int per = (top_k + s - 1) / s;
  per = ((per + kTile - 1) / kTile) * kTile;
  AttnPlan p;
  p.split_rows = per;
  p.n_splits = (top_k + per - 1) / per;
  return p;
}

// Merge of the split partials of one head: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
struct CombineArgs {
  const float* part_o;
  const float* part_ml;
  const int32_t* count;
  float* out;  // [B][Hq][d]
  int Hq, G, top_k, n_splits, split_rows;
};

__global__ void __launch_bounds__(kD) attn_combine_kernel(CombineArgs a) {
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int gs = a.Hq / a.G, g = h / gs, hh = h % gs;
  const int row = b * a.G + g;
  const int cnt = min(a.count[row], a.top_k);
  const int ns = min(a.n_splits, ceil_div(max(cnt, 0), a.split_rows));
  const float* ml = a.part_ml + ((size_t)row * a.n_splits * gs + hh) * 2;
  const float* po = a.part_o + ((size_t)row * a.n_splits * gs + hh) * kD + tid;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, ml[(size_t)s * gs * 2]);
  float L = 0.f, o = 0.f;
  if (M > -INFINITY) {
    for (int s = 0; s < ns; ++s) {
      const float m = ml[(size_t)s * gs * 2];
      const float w = (m == -INFINITY) ? 0.f : exp2f(m - M);
      L = fmaf(w, ml[(size_t)s * gs * 2 + 1], L);
      o = fmaf(w, po[(size_t)s * gs * kD], o);
    }
  }
  a.out[((size_t)b * a.Hq + h) * kD + tid] = (L > 0.f) ? o / L : 0.f;
}

}  // namespace hhr
