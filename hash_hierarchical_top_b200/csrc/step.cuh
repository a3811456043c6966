// Prologue of the fused decode step: append the newest key/value row of every sequence to
// the paged cache, encode that key (step a0) and prepare the group's queries (step a1),
// all with one read of R_g and W_g.
//
// HHR page, Abstract: GKR rotates keys and queries with the head-wise orthogonal R_h and
// summarises each page for its logit bound; LHP encodes both into binary codes. The newest
// key (position seq_len-1) and the group's query heads form one batch of 1 + gs vectors
// for the two mat-vecs. Every rotated channel and projection is row_dot16 on the same
// inputs as in encode_page_kernel and qprep_kernel, and the folds run in the same order, so
// the results are bit-identical to the separate calls.
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
  uint32_t* q_code;        // [B][Hq][CW]
  float* qpn;              // [B][G][2][d]
  int Hq, G, P, maxp, n_phys, summary_fp16;
  // L2 warm-up for page_bound_stage_kernel: the first warm_units units (pages, all groups'
  // summaries, unit_bytes each) of each of its warm_ctas CTAs' chunk ranges; 0 = none.
  int warm_units, warm_ctas, unit_bytes, chunk;
};


// Loads the stored summary channel `row` of a page that already held keys.
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

// The newest key's slot; phys < 0 when the sequence is empty or its page is out of range.
struct NewestSlot {
  int phys, slot;
  size_t krow, sbase;
};

__device__ __forceinline__ NewestSlot newest_slot(const PrologueArgs& a, int len, int b, int g,
                                                  bool report) {
  const int t = len - 1;
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

// Eight bf16 values (one 16-byte piece) to fp32, stored at dst[0..8).
__device__ __forceinline__ void store_bf16x8(const uint4 raw, float* dst) {
  float4* d4 = reinterpret_cast<float4*>(dst);
  d4[0] = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                      __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
  d4[1] = make_float4(__uint_as_float(raw.z << 16), __uint_as_float(raw.z & 0xffff0000u),
                      __uint_as_float(raw.w << 16), __uint_as_float(raw.w & 0xffff0000u));
}

// A cluster of kPrologueRanks CTAs per (group, sequence). CTA r owns rows 32r..32r+31 of R_g
// and W_g (one row block of row_dot16, 16 threads per row). It rotates all 1 + GS vectors on
// its rows and sends the results, as 16-byte pieces, into every CTA's copy of the rotated
// vectors (distributed shared memory); after one cluster barrier it projects them on the
// rows of W_g of code words r, r + 4, ... (below CW), whose 32 sign bits are those words.
// CTA r also owns summary channels and folded-query channels 32r..32r+31. Every input load is issued at the start; only the key's cache slot (and the
// key itself when k_new is null) waits for the page table.
constexpr int kPrologueRanks = kRowBlocks;
constexpr int kPrologueThreads = kMvThreads;  // 32 rows x 16 threads

template <int GS, int CW>
__global__ void __cluster_dims__(kPrologueRanks, 1, 1) __launch_bounds__(kPrologueThreads)
    step_prologue_cluster_kernel(PrologueArgs a) {
  namespace cg = cooperative_groups;
  constexpr int NV = 1 + GS;  // vector 0: the newest key; 1..GS: the query heads
  constexpr int kWpr = (CW + kPrologueRanks - 1) / kPrologueRanks;  // code words per rank
  static_assert(16 * (NV + 1) <= kPrologueThreads, "one 16-byte piece per thread");
  __shared__ __align__(16) float xs[NV][kD];  // raw vectors
  __shared__ __align__(16) float xpart[NV][32];  // rotated vectors, this CTA's rows
  __shared__ __align__(16) float xr[NV][kD];     // rotated vectors, every row
  __shared__ uint32_t cpart[kWpr][NV][kPrologueThreads / 32];  // sign bits of each warp's rows
  pdl_wait();
  pdl_trigger();
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int lrow = mv_lrow(), part = mv_part();
  const int row = rank * 32 + lrow;
  const bool row_lead = part == 0;

  float4 rr[2], wr[kWpr][2];
  load_row16(a.R + (size_t)g * kD * kD, row, rr);
#pragma unroll
  for (int i = 0; i < kWpr; ++i) {
    const int w = rank + kPrologueRanks * i;
    if (w < CW) load_row16(a.W + (size_t)g * (32 * CW) * kD, w * 32 + lrow, wr[i]);
  }
  const int len = a.seq_len[b];
  // L2 warm-up for the page-bound kernel that follows, while HBM is otherwise idle here:
  // thread t of the grid takes unit t % warm_units of that kernel's CTA t / warm_units, whose
  // range of chunks starts at chunk cta * C / warm_ctas (C chunks of `chunk` pages over the
  // sequences in order, as that kernel cuts them). It reads only inputs (lengths, page table);
  // a summary this kernel updates is prefetched coherently (L2 holds the update).
  const int t_lin = ((blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) *
                        kPrologueThreads + tid;
  const void* warm = nullptr;
  if (a.warm_units > 0 && t_lin < a.warm_units * a.warm_ctas) {
    const int B = gridDim.z;
    auto chunks_of = [&](int bb) {
      return ceil_div(min(ceil_div(max(a.seq_len[bb], 0), a.P), a.maxp), a.chunk);
    };
    int C = 0;
    for (int bb = 0; bb < B; ++bb) C += chunks_of(bb);
    const int cta = t_lin / a.warm_units, u = t_lin - cta * a.warm_units;
    int id = (int)((long long)cta * C / a.warm_ctas) + u / a.chunk;
    const int id_end = (int)((long long)(cta + 1) * C / a.warm_ctas);
    if (id < id_end) {
      int wb = 0;
      for (; wb < B; ++wb) {
        const int nc = chunks_of(wb);
        if (id < nc) break;
        id -= nc;
      }
      const int wp = id * a.chunk + u % a.chunk;
      if (wb < B && wp < min(ceil_div(max(a.seq_len[wb], 0), a.P), a.maxp)) {
        const int ph = a.page_table[(size_t)wb * a.maxp + wp];
        if (ph >= 0 && ph < a.n_phys)
          warm = static_cast<const char*>(a.page_minmax) + (size_t)ph * a.unit_bytes;
      }
    }
  }
  // Threads [16v, 16v + 16) load vector v (k_new, then the queries) as 16-byte pieces of
  // 8 channels; threads [16 NV, 16 NV + 16) load v_new.
  const int pv = tid >> 4, c8 = (tid & 15) * 8;
  const bool append = a.k_new != nullptr;
  uint4 raw = make_uint4(0, 0, 0, 0);
  if (pv == 0) {
    if (append) raw = *reinterpret_cast<const uint4*>(a.k_new + ((size_t)b * a.G + g) * kD + c8);
  } else if (pv < NV) {
    raw = *reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.Hq + g * GS + pv - 1) * kD + c8);
  } else if (pv == NV && append && a.v_new != nullptr) {
    raw = *reinterpret_cast<const uint4*>(a.v_new + ((size_t)b * a.G + g) * kD + c8);
  }
  const NewestSlot s = newest_slot(a, len, b, g, tid == 0 && rank == 0);
  const bool has_key = s.phys >= 0;
  if (pv == 0) {
    if (!has_key) {
      raw = make_uint4(0, 0, 0, 0);
    } else if (!append) {
      raw = *reinterpret_cast<const uint4*>(a.k_cache + s.krow + c8);
    } else if (rank == 0) {  // one writer of the new rows
      *reinterpret_cast<uint4*>(a.k_cache + s.krow + c8) = raw;
    }
  } else if (pv == NV && has_key && append && a.v_new != nullptr && rank == 0) {
    *reinterpret_cast<uint4*>(a.v_cache + s.krow + c8) = raw;
  }
  if (pv < NV) store_bf16x8(raw, &xs[pv][c8]);
  float mn = INFINITY, mx = -INFINITY;
  if (has_key && s.slot > 0 && row_lead) load_summary_row(a.page_minmax, a.summary_fp16, s.sbase, row, mn, mx);
  __syncthreads();
  if (warm != nullptr) prefetch_l2(warm, (unsigned)a.unit_bytes);

  // Rotation (steps a0 and a1) of every vector on this thread's row.
  float y[NV];
#pragma unroll
  for (int v = 0; v < NV; ++v) y[v] = row_dot16(rr, &xs[v][0]);
  if (has_key) {
    mn = fminf(mn, y[0]);
    mx = fmaxf(mx, y[0]);
  }
  float qneg = 0.f, qpos = 0.f;
#pragma unroll
  for (int h = 0; h < GS; ++h) {
    qneg += fminf(y[1 + h], 0.f);
    qpos += fmaxf(y[1 + h], 0.f);
  }
  if (row_lead) {
#pragma unroll
    for (int v = 0; v < NV; ++v) xpart[v][lrow] = v == 0 && !has_key ? 0.f : y[v];
  }
#pragma unroll
  for (int h = 0; h < GS; ++h)
    if (h == part) a.q_rot[((size_t)b * a.Hq + g * GS + h) * kD + row] = y[1 + h];
  __syncthreads();
  // Every rank's copy of the rotated vectors receives this CTA's rows: thread i sends
  // 16-byte piece j of vector v to rank r.
  if (tid < NV * 8 * kPrologueRanks) {
    const int v = tid / (8 * kPrologueRanks), r = (tid / 8) % kPrologueRanks, j = tid % 8;
    const float4 val = reinterpret_cast<const float4*>(&xpart[v][0])[j];
    reinterpret_cast<float4*>(cl.map_shared_rank(&xr[v][0], r))[rank * 8 + j] = val;
  }
  cluster_sync_all();  // every rank's rows of every rotated vector have landed

  // LHP codes: the sign of W_g x' on this thread's row of word w is bit lrow of code word
  // w. Warp w holds rows 2w and 2w + 1: an OR-reduction collects the warp's two bits, and
  // warp 0 merges the warps' pieces.
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int i = 0; i < kWpr; ++i) {
    if (rank + kPrologueRanks * i >= CW) continue;  // uniform over the CTA
    float pj[NV];
#pragma unroll
    for (int v = 0; v < NV; ++v) pj[v] = row_dot16(wr[i], &xr[v][0]);
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const uint32_t bits = __reduce_or_sync(kFull, row_lead && pj[v] > 0.f ? 1u << lrow : 0u);
      if (lane == 0) cpart[i][v][warp] = bits;
    }
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int i = 0; i < kWpr; ++i) {
      const int w = rank + kPrologueRanks * i;
      if (w >= CW) continue;
      uint32_t mine = 0u;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const uint32_t word =
            __reduce_or_sync(kFull, lane < kPrologueThreads / 32 ? cpart[i][v][lane] : 0u);
        if (lane == v) mine = word;
      }
      if (lane == 0) {
        if (has_key) a.codes[(((size_t)s.phys * a.G + g) * a.P + s.slot) * CW + w] = mine;
      } else if (lane < NV) {
        a.q_code[((size_t)b * a.Hq + g * GS + (lane - 1)) * CW + w] = mine;
      }
    }
  }
  if (row_lead) {
    if (has_key) store_summary_row(a.page_minmax, a.summary_fp16, s.sbase, row, mn, mx);
    float* o = a.qpn + ((size_t)b * a.G + g) * 2 * kD;
    o[row] = qneg;
    o[kD + row] = qpos;
  }
}

using PrologueFn = void (*)(PrologueArgs);

template <int CW>
inline PrologueFn step_prologue_for_cw(int gs) {
  switch (gs) {
    case 1: return step_prologue_cluster_kernel<1, CW>;
    case 2: return step_prologue_cluster_kernel<2, CW>;
    case 3: return step_prologue_cluster_kernel<3, CW>;
    case 4: return step_prologue_cluster_kernel<4, CW>;
    case 5: return step_prologue_cluster_kernel<5, CW>;
    case 6: return step_prologue_cluster_kernel<6, CW>;
    case 7: return step_prologue_cluster_kernel<7, CW>;
    default: return step_prologue_cluster_kernel<8, CW>;
  }
}

// The instantiation for group size gs (1..kMaxGroup) and cw code words (2, 4 or 8).
inline PrologueFn step_prologue_for(int gs, int cw) {
  return cw == 2 ? step_prologue_for_cw<2>(gs)
                 : cw == 8 ? step_prologue_for_cw<8>(gs) : step_prologue_for_cw<4>(gs);
}

}  // namespace hhr
