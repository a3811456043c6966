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
//   2. logits: warp w takes 8 rows of the tile; S = Q K^T on bf16 mma.sync
//      (m16n8k16, the group's heads on M, the warp's 8 keys on N), so the
//      accumulator fragment holds one (head, key pair) per lane;
//   3. every warp keeps its own online softmax (running max, sum and output per
//      head) over its rows; O^T += V^T P^T on mma.sync m16n8k8, the logit
//      accumulator being directly the B operand (P split into bf16 hi + lo);
//   4. the 8 warps are merged in shared memory; a split writes its partial (max,
//      sum, output) per head, or the final output when the group is not split.
//      The splits are merged either by a combine kernel, or (cluster variant) by
//      the cluster's CTAs through distributed shared memory, each CTA merging its
//      share of the group's outputs (standard split softmax rescaling).
#pragma once
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace hhr {

constexpr int kAttnWarps = 8;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kTile = 64;                        // selected rows per pipeline stage
constexpr int kStages = 3;
constexpr int kMaxSplitRows = 2048;              // rows of one split (offsets in smem)
#ifndef HHR_ATTN_TARGET_CTAS
#define HHR_ATTN_TARGET_CTAS (2 * 148)             // two resident CTAs on each of 148 SMs
#endif
constexpr int kTargetCtas = HHR_ATTN_TARGET_CTAS;
constexpr uint32_t kNoRow = 0xffffffffu;          // offset table: row to skip

struct AttnArgs {
  const uint16_t* q;        // [B][Hq][d]
  const uint16_t* k_cache;  // [n_phys][G][P][d]
  const uint16_t* v_cache;
  const int32_t* page_table;
  const int32_t* seq_len;
  const int32_t* idx;       // [B][Gs][top_k]
  const int32_t* count;     // [B][Gs]
  float* part_o;            // [B][Gs][n_splits][gs][d]   (n_splits > 1)
  float* part_ml;           // [B][Gs][n_splits][gs][2]
  float* out;               // [B][Hq][d]                 (n_splits == 1)
  float scale_log2;
  int Hq, G, P, maxp, n_phys, top_k, n_splits, split_rows;
  const uint32_t* rows;     // [B][Gs][top_k] cache rows of the selected keys, already
                            // resolved and checked (fused step); null: resolve from idx
  int Gs, kv_div;           // selection rows per sequence (G, or Hq per head): row r holds
                            // query heads [r gs, (r + 1) gs), gs = Hq / Gs, and reads the
                            // K/V of head r / kv_div
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// ---- tensor-core fragments (bf16 mma.sync, fp32 accumulate) ----------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D = A(16x16, row) * B(16x8, col) + D
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// D = A(16x8, row) * B(8x8, col) + D
__device__ __forceinline__ void mma_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
__device__ __forceinline__ uint32_t pack_bf16(float x, float y) {
  const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x));
  const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y));
  return lo | (hi << 16);
}
__device__ __forceinline__ float bf16_round(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

// Shared memory: kStages x (K tile + V tile) of 64 rows x 256 B (16-byte chunks of a row
// XOR-swizzled by row % 8, so ldmatrix reads of 8 rows hit 8 distinct bank groups), the
// split's row offsets, and the merge area (reusing the stage buffers).
inline size_t attn_smem() {
  return (size_t)kStages * 2 * kTile * kD * 2 + (size_t)kMaxSplitRows * 4 + 64;
}

__device__ __forceinline__ int swz(int r, int chunk) { return r * kD + ((chunk ^ (r & 7)) << 3); }

// Per warp and tile: the warp's 8 keys. Logits S = Q K^T with Q rows = heads (padded to
// 16, rows >= gs are zero) on mma.m16n8k16 over 8 channel steps; the accumulator lane
// (g = lane/4, t = lane%4) holds S[head g][keys 2t, 2t+1], which is exactly the B
// fragment of O^T = V^T P^T on mma.m16n8k8 (channels on M, heads on N). P is split into
// bf16 hi + lo parts (two MMAs) so its rounding stays near 2^-16 relative.
// kCluster: the splits of a group form one thread-block cluster; after each CTA has
// merged its warps, every CTA merges its share of the group's outputs from all the
// splits' states through distributed shared memory and writes them (no partials in
// global memory, no combine kernel).
// Barrier of the kAttnThreads threads that run one split: the whole CTA of the split kernel
// (named barrier 0), or one half of a CTA of the fused step kernel (named barriers 1, 2).
__device__ __forceinline__ void attn_sync(int bar_id) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(bar_id), "r"(kAttnThreads) : "memory");
}

// One split of one selection row, run by kAttnThreads threads (tid 0..255) behind barrier
// bar_id: rows [base, base + nrows) of the row's selection are gathered and attended; the
// split's softmax state is merged over its warps, and emit(h, c, M, L, O) is called once
// for every (head h < gs, channel c) of the row, M the split's running max of head h (in
// log2 units), L its sum of exponentials and O its output channel c before the division
// by L. smem: the stage buffers followed by the row-offset table of split_rows entries.
// Selection rows, counts and cache rows are read through L2 (they may have been written by
// other CTAs of the same kernel).
template <typename Emit>
__device__ __forceinline__ void attn_split(const AttnArgs& a, int g, int b, int base, int nrows,
                                           uint16_t* stage_base, int tid, int bar_id, Emit emit) {
  uint32_t* offs = reinterpret_cast<uint32_t*>(stage_base + (size_t)kStages * 2 * kTile * kD);
  const int lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;   // fragment coordinates
  const int gs = a.Hq / a.Gs;
  const int row = b * a.Gs + g;
  const uint32_t gkv = (uint32_t)(a.kv_div == 1 ? g : g / a.kv_div);  // KV head of the row
  const int ntiles = (nrows + kTile - 1) / kTile;
  const int n = a.seq_len[b];

  // Cache row index (phys*G + g)*P + slot of each of the split's rows (kNoRow: skip).
  for (int r = tid; r < ntiles * kTile; r += kAttnThreads) {
    uint32_t o = kNoRow;
    if (r < nrows && a.rows != nullptr) {
      o = __ldcg(a.rows + (size_t)row * a.top_k + base + r);
    } else if (r < nrows) {
      const int t = __ldcg(a.idx + (size_t)row * a.top_k + base + r);
      const int lp = t / a.P;
      if (t >= 0 && t < n && lp < a.maxp) {
        const int phys = a.page_table[(size_t)b * a.maxp + lp];
        if (phys >= 0 && phys < a.n_phys)
          o = ((uint32_t)phys * (uint32_t)a.G + gkv) * (uint32_t)a.P + (uint32_t)(t % a.P);
        else
          flag_status(kStatusBadPage);
      } else {
        flag_status(kStatusBadToken);
      }
    }
    offs[r] = o;
  }
  attn_sync(bar_id);

  auto issue = [&](int t) {
    uint16_t* Ks = stage_base + (size_t)(t % kStages) * 2 * kTile * kD;
    uint16_t* Vs = Ks + kTile * kD;
#pragma unroll
    for (int i = 0; i < (kTile * 16) / kAttnThreads; ++i) {
      const int c = tid + i * kAttnThreads;
      const int r = c >> 4, piece = c & 15;
      const uint32_t o = offs[t * kTile + r];
      uint16_t* kd = Ks + swz(r, piece);
      uint16_t* vd = Vs + swz(r, piece);
      if (o != kNoRow) {
        cp_async16(kd, a.k_cache + (size_t)o * kD + piece * 8);
        cp_async16(vd, a.v_cache + (size_t)o * kD + piece * 8);
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

  // A fragments of Q (row gq = head; rows >= gs and the upper 8 rows are zero).
  uint32_t qa0[8], qa2[8];
  {
    const bool hv = gq < gs;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        a.q + ((size_t)b * a.Hq + g * gs + (hv ? gq : 0)) * kD);
#pragma unroll
    for (int s8 = 0; s8 < 8; ++s8) {
      qa0[s8] = hv ? qrow[(16 * s8 + 2 * tq) >> 1] : 0u;
      qa2[s8] = hv ? qrow[(16 * s8 + 2 * tq + 8) >> 1] : 0u;
    }
  }
  const bool head_ok = gq < gs;
  float m_run = -INFINITY, l_run = 0.f;      // of head gq (replicated over tq)
  float oacc[8][4];                          // O^T[channel 16i + gq (+8)][head 2tq (+1)]
#pragma unroll
  for (int i = 0; i < 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  const uint32_t smem0 = (uint32_t)__cvta_generic_to_shared(stage_base);
  const int kr = warp * 8 + (lane & 7);       // ldmatrix row (key) supplied by this lane
  const int mj = lane >> 3;                   // which of the 4 matrices it addresses

  for (int t = 0; t < ntiles; ++t) {
    cp_async_wait<kStages - 2>();
    attn_sync(bar_id);
    if (t + kStages - 1 < ntiles) issue(t + kStages - 1);
    cp_async_commit();
    const uint32_t ks = smem0 + (uint32_t)((t % kStages) * 2 * kTile * kD) * 2;
    const uint32_t vs = ks + (uint32_t)(kTile * kD) * 2;
    // S = Q K^T for the warp's 8 keys: 8 k-steps, ldmatrix.x4 covers two of them.
    float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(ks + (uint32_t)swz(kr, 4 * q4 + mj) * 2, b0, b1, b2, b3);
      mma_16816(sacc, qa0[2 * q4], 0u, qa2[2 * q4], 0u, b0, b1);
      mma_16816(sacc, qa0[2 * q4 + 1], 0u, qa2[2 * q4 + 1], 0u, b2, b3);
    }
    // Keys 2tq, 2tq+1 of the warp's 8 for head gq; mask padding and skipped rows.
    const int kbase = t * kTile + warp * 8 + 2 * tq;
    const bool v0 = head_ok && kbase < nrows && offs[kbase] != kNoRow;
    const bool v1 = head_ok && kbase + 1 < nrows && offs[kbase + 1] != kNoRow;
    const float s0 = v0 ? sacc[0] * a.scale_log2 : -INFINITY;
    const float s1 = v1 ? sacc[1] * a.scale_log2 : -INFINITY;
    float mx = fmaxf(s0, s1);
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float corr = (m_new == -INFINITY) ? 1.f : exp2f(m_run - m_new);
    const float p0 = v0 ? exp2f(s0 - m_new) : 0.f;
    const float p1 = v1 ? exp2f(s1 - m_new) : 0.f;
    float ps = p0 + p1;
    ps += __shfl_xor_sync(kFull, ps, 1);
    ps += __shfl_xor_sync(kFull, ps, 2);
    l_run = l_run * corr + ps;
    m_run = m_new;
    // Rescale O^T columns (heads 2tq, 2tq+1): their factors live on lanes 8tq and 8tq+4.
    const float ca = __shfl_sync(kFull, corr, 8 * tq);
    const float cb = __shfl_sync(kFull, corr, 8 * tq + 4);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      oacc[i][0] *= ca; oacc[i][2] *= ca;
      oacc[i][1] *= cb; oacc[i][3] *= cb;
    }
    const float h0 = bf16_round(p0), h1 = bf16_round(p1);
    const uint32_t phi = pack_bf16(h0, h1);
    const uint32_t plo = pack_bf16(p0 - h0, p1 - h1);
    // O^T += V^T P^T: 8 channel tiles of 16; ldmatrix.x4.trans covers two of them.
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(vs + (uint32_t)swz(kr, 4 * q4 + mj) * 2, a0, a1, a2, a3);
      mma_1688(oacc[2 * q4], a0, a1, phi);
      mma_1688(oacc[2 * q4], a0, a1, plo);
      mma_1688(oacc[2 * q4 + 1], a2, a3, phi);
      mma_1688(oacc[2 * q4 + 1], a2, a3, plo);
    }
  }
  cp_async_wait<0>();
  attn_sync(bar_id);

  // Merge the 8 warps: o = sum_w 2^(m_w - M) o_w, l = sum_w 2^(m_w - M) l_w.
  float* mo = reinterpret_cast<float*>(stage_base);             // [warps][8 heads][d]
  float* mml = mo + (size_t)kAttnWarps * kMaxGroup * kD;         // [warps][8 heads][2]
  {
    float* mw = mo + (size_t)warp * kMaxGroup * kD;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c0 = 16 * i + gq;
      if (2 * tq < gs) {
        mw[(2 * tq) * kD + c0] = oacc[i][0];
        mw[(2 * tq) * kD + c0 + 8] = oacc[i][2];
      }
      if (2 * tq + 1 < gs) {
        mw[(2 * tq + 1) * kD + c0] = oacc[i][1];
        mw[(2 * tq + 1) * kD + c0 + 8] = oacc[i][3];
      }
    }
    if (tq == 0 && head_ok) {
      mml[(warp * kMaxGroup + gq) * 2] = m_run;
      mml[(warp * kMaxGroup + gq) * 2 + 1] = l_run;
    }
  }
  attn_sync(bar_id);
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
    emit(h, c, M, L, O);
  }
}

// Merge of the split partials of output (head hh, channel c) of selection row `row` over its
// first ns splits: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s (0 for an empty set).
// The same arithmetic, in the same order, wherever splits are merged.
__device__ __forceinline__ float merge_splits(const float* part_o, const float* part_ml, int row,
                                              int n_splits, int ns, int gs, int hh, int c) {
  const float* ml = part_ml + ((size_t)row * n_splits * gs + hh) * 2;
  const float* po = part_o + ((size_t)row * n_splits * gs + hh) * kD + c;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, __ldcg(ml + (size_t)s * gs * 2));
  float L = 0.f, o = 0.f;
  if (M > -INFINITY) {
    for (int s = 0; s < ns; ++s) {
      const float m = __ldcg(ml + (size_t)s * gs * 2);
      const float w = (m == -INFINITY) ? 0.f : exp2f(m - M);
      L = fmaf(w, __ldcg(ml + (size_t)s * gs * 2 + 1), L);
      o = fmaf(w, __ldcg(po + (size_t)s * gs * kD), o);
    }
  }
  return (L > 0.f) ? o / L : 0.f;
}

// kCluster: the splits of a group form one thread-block cluster; after each CTA has
// merged its warps, every CTA merges its share of the group's outputs from all the
// splits' states through distributed shared memory and writes them (no partials in
// global memory, no combine kernel).
template <bool kCluster>
__global__ void __launch_bounds__(kAttnThreads, 2) sparse_attn_kernel(AttnArgs a) {
  extern __shared__ float4 at_smem[];
  pdl_wait();
  pdl_trigger();
  uint16_t* stage_base = reinterpret_cast<uint16_t*>(at_smem);             // [kStages][2][kTile][d]
  uint32_t* offs = reinterpret_cast<uint32_t*>(stage_base + (size_t)kStages * 2 * kTile * kD);
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;  // g: selection row
  const int tid = threadIdx.x;
  const int gs = a.Hq / a.Gs;
  const int row = b * a.Gs + g;
  const int cnt = min(__ldcg(a.count + row), a.top_k);
  const int base = split * a.split_rows;
  // A split past the selection does no work (in a cluster it still joins the merge). An
  // unsplit group with an empty selection writes its zero output here, since no merge follows.
  const int nrows = max(0, min(a.split_rows, cnt - base));
  if (!kCluster && nrows == 0) {
    if (a.n_splits == 1)
      for (int i = tid; i < gs * kD; i += kAttnThreads)
        a.out[((size_t)b * a.Hq + g * gs) * kD + i] = 0.f;
    return;
  }
  attn_split(a, g, b, base, nrows, stage_base, tid, 0, [&](int h, int c, float M, float L, float O) {
    if constexpr (kCluster) {
      // This CTA's merged state, in the (now free) offset table: [gs][d] outputs, [gs][2].
      float* res = reinterpret_cast<float*>(offs);
      res[h * kD + c] = O;
      if (c == 0) {
        res[kMaxGroup * kD + 2 * h] = M;
        res[kMaxGroup * kD + 2 * h + 1] = L;
      }
    } else if (a.n_splits == 1) {
      a.out[((size_t)b * a.Hq + g * gs + h) * kD + c] = (L > 0.f) ? O / L : 0.f;
    } else {
      const size_t p = ((size_t)row * a.n_splits + split) * gs + h;
      a.part_o[p * kD + c] = O;
      if (c == 0) {
        a.part_ml[p * 2] = M;
        a.part_ml[p * 2 + 1] = L;
      }
    }
  });
  if constexpr (kCluster) {
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();  // every split's state is in its shared memory
    {
      // Rank r merges outputs [r n/ns, (r + 1) n/ns) of the group's n = gs * d (the same
      // arithmetic per output as merge_splits, split over the cluster's CTAs).
      const int ns = (int)cl.num_blocks(), rk = (int)cl.block_rank();
      const int per = (gs * kD + ns - 1) / ns;
      const int lo = rk * per, hi = min(gs * kD, lo + per);
      float* res_local = reinterpret_cast<float*>(offs);
      for (int i = lo + tid; i < hi; i += kAttnThreads) {
        const int h = i / kD, c = i % kD;
        float M = -INFINITY;
        for (int r = 0; r < ns; ++r)
          M = fmaxf(M, cl.map_shared_rank(res_local, r)[kMaxGroup * kD + 2 * h]);
        float L = 0.f, O = 0.f;
        if (M > -INFINITY) {
          for (int r = 0; r < ns; ++r) {
            const float* rr = cl.map_shared_rank(res_local, r);
            const float mr = rr[kMaxGroup * kD + 2 * h];
            const float sc = (mr == -INFINITY) ? 0.f : exp2f(mr - M);
            L = fmaf(sc, rr[kMaxGroup * kD + 2 * h + 1], L);
            O = fmaf(sc, rr[h * kD + c], O);
          }
        }
        a.out[((size_t)b * a.Hq + g * gs + h) * kD + c] = (L > 0.f) ? O / L : 0.f;
      }
    }
    cl.sync();  // keep every CTA's shared memory alive until every rank has read it
  }
}

// Split plan: about two resident CTAs per SM over the whole batch, at most
// kMaxSplitRows rows per split, splits of whole 64-row tiles.
struct AttnPlan {
  int n_splits, split_rows;
};
// Cluster variant (fused decode step): at most kMaxClusterSplits splits per group.
constexpr int kMaxClusterSplits = 8;
inline AttnPlan attn_plan(int B, int G, int top_k, int max_splits = 1 << 30) {
  const long long rows = (long long)B * G;
  int s = (int)(kTargetCtas / (rows > 0 ? rows : 1));
  if (s < 1) s = 1;
  int max_s = (top_k + kTile - 1) / kTile;
  if (max_s > max_splits) max_s = max_splits;
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
  int Hq, G, top_k, n_splits, split_rows;  // G: selection rows per sequence (Gs)
};

__global__ void __launch_bounds__(kD) attn_combine_kernel(CombineArgs a) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int gs = a.Hq / a.G, g = h / gs, hh = h % gs;
  const int row = b * a.G + g;
  const int cnt = min(a.count[row], a.top_k);
  const int ns = min(a.n_splits, ceil_div(max(cnt, 0), a.split_rows));
  a.out[((size_t)b * a.Hq + h) * kD + tid] =
      merge_splits(a.part_o, a.part_ml, row, a.n_splits, ns, gs, hh, tid);
}

}  // namespace hhr
