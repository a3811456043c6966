// Steps a2-a5 of the fused decode step for small batches: one thread-block cluster of RANKS
// CTAs (16, a non-portable cluster size, or 8; the launch's cluster dimension) per selection
// row does the row's page bounds, top-m pages, Hamming top-k and sparse attention, with
// cluster barriers instead of kernel boundaries between them.
//
// HHR page, Abstract: page-level logit bounds prune the pages, Hamming distances of the keys'
// hash codes rank the keys of the pages that survive, and attention runs over the selected
// keys. With few rows (a batch of one or two sequences) each of the separate kernels runs on a
// few SMs as a latency chain, and the chain of four launches costs their start-up and
// drain times on top. Here each row's steps run across its cluster, with no kernel boundary
// (the bounds then use only the clusters' SMs, so the host takes this path only for a few MB
// of summaries):
//   1. rank r computes the bounds of its slice of the row's pages (bound_warp, one warp per
//      16 pages at a time) and writes them;
//   2. after a cluster barrier every rank selects the same top-m pages from all the bounds
//      (read back through L2) and scores its 1/RANKS share of the kept pages' keys; the
//      distance histograms are summed and the top-k compacted in token order across the
//      cluster (topm_hamming_row / hamming_topk_cluster with RANKS ranks);
//   3. after a cluster barrier rank s < n_splits attends split s of the row's selection
//      (attn_split, 8 of its warps), and the splits are merged through distributed shared
//      memory, each rank writing its share of the row's outputs.
// Every step runs the arithmetic of the separate kernels (bound_warp, the same selection
// functions, attn_split and the split merge in the same order), so codes, bounds, kept pages,
// selections and counts are bit-identical to theirs, and so is the output wherever the
// separate attention's split plan equals this one (at most RANKS splits).
#pragma once
#include <cooperative_groups.h>

#include "attn.cuh"
#include "common.cuh"
#include "select.cuh"

namespace hhr {

constexpr int kRowThreads = 512;   // 16 warps: bound warps, then the selection, then attention
constexpr int kRowWarps = kRowThreads / 32;
static_assert(kRowThreads >= kAttnThreads, "one attention split per CTA");

struct RowClusterArgs {
  BoundArgs bound;       // a2 bounds (early = 0)
  TopmHammingArgs sel;   // a2 top-m, a3, a4; sel.h.out_rows: cache rows of the selection
  AttnArgs attn;         // a5: rows = sel.h.out_rows, n_splits <= the cluster's CTAs
  int per_head;          // selection rows are query heads (bound_query folds the query)
};

// Dynamic shared memory: the selection's (kept lists, bound keys or Hamming scratch) and then
// the attention's stage buffers, one after the other in the same space.
inline size_t row_cluster_smem(int gs, int cw, int m_max, int P, int maxp, int ranks) {
  const size_t sel = topm_hamming_smem(gs, cw, m_max, P, maxp, ranks);
  const size_t att = attn_smem();
  return sel > att ? sel : att;
}

template <int NB, int CW, bool F16, int RANKS>
__global__ void __launch_bounds__(kRowThreads, 1) row_cluster_kernel(RowClusterArgs a) {
  namespace cg = cooperative_groups;
  __shared__ TopmSmem<kRowThreads> S;
  extern __shared__ __align__(16) uint32_t rc_dyn[];
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int row = blockIdx.x / RANKS;
  const BoundArgs& ba = a.bound;
  const int b = row / ba.Gs, r = row % ba.Gs;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_trigger();

  // 1. Bounds of this rank's pages: slices of whole 16-page warp units.
  if (!a.sel.flat) {
    constexpr int kWarpPages = 8 * (F16 ? HHR_BOUND_SETS_F16 : HHR_BOUND_SETS_F32);
    const int npg = min(ceil_div(ba.seq_len[b], ba.P), ba.maxp);
    const int per = ceil_div(ceil_div(npg, RANKS), kWarpPages) * kWarpPages;
    const int lo = rank * per, hi = min(npg, lo + per);
    if (lo + warp * kWarpPages < hi) {
      float4 q0, q1;
      bound_query<F16>(ba, b, r, a.per_head != 0, lane, q0, q1);
      for (int p0 = lo + warp * kWarpPages; p0 < hi; p0 += kRowWarps * kWarpPages)
        bound_warp<F16>(ba, b, r, a.per_head ? r / ba.kv_div : r, p0, hi, lane, q0, q1);
    }
    cluster_sync_all();  // every rank's bounds are written (visible cluster-wide)
  }

  // 2. Top-m pages and the Hamming top-k across the cluster.
  topm_hamming_row<NB, CW, kRowThreads, RANKS>(a.sel, row, rank, S, rc_dyn, false);
  cluster_sync_all();  // every rank's selected keys and cache rows are written

  // 3. Split `rank` of the row's attention, then the cluster-wide merge of the splits.
  const AttnArgs& at = a.attn;
  const int ns = at.n_splits;
  const int gs = at.Hq / at.Gs;
  uint16_t* stage_base = reinterpret_cast<uint16_t*>(rc_dyn);
  float* res = reinterpret_cast<float*>(stage_base + (size_t)kStages * 2 * kTile * kD);
  if (rank < ns && tid < kAttnThreads) {
    const int cnt = min(__ldcg(at.count + row), at.top_k);
    const int base = rank * at.split_rows;
    const int nrows = max(0, min(at.split_rows, cnt - base));
    attn_split(at, r, b, base, nrows, stage_base, tid, 1, [&](int h, int c, float M, float L, float O) {
      res[h * kD + c] = O;
      if (c == 0) {
        res[kMaxGroup * kD + 2 * h] = M;
        res[kMaxGroup * kD + 2 * h + 1] = L;
      }
    });
  }
  cluster_sync_all();  // every split's state is in its CTA's shared memory
  {
    // Rank q writes outputs [q n/R, (q + 1) n/R) of the row's n = gs * d: the merge of
    // merge_splits over the ns splits' states, read through distributed shared memory.
    const int per = ceil_div(gs * kD, RANKS);
    const int lo = rank * per, hi = min(gs * kD, lo + per);
    for (int i = lo + tid; i < hi; i += kRowThreads) {
      const int h = i / kD, c = i % kD;
      float M = -INFINITY;
      for (int s = 0; s < ns; ++s)
        M = fmaxf(M, cl.map_shared_rank(res, s)[kMaxGroup * kD + 2 * h]);
      float L = 0.f, O = 0.f;
      if (M > -INFINITY) {
        for (int s = 0; s < ns; ++s) {
          const float* rs = cl.map_shared_rank(res, s);
          const float ms = rs[kMaxGroup * kD + 2 * h];
          const float sc = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
          L = fmaf(sc, rs[kMaxGroup * kD + 2 * h + 1], L);
          O = fmaf(sc, rs[h * kD + c], O);
        }
      }
      at.out[((size_t)b * at.Hq + r * gs + h) * kD + c] = (L > 0.f) ? O / L : 0.f;
    }
  }
  cluster_sync_all();  // keep every CTA's shared memory alive until every rank has read it
}

using RowClusterFn = void (*)(RowClusterArgs);

template <bool F16, int RANKS>
inline RowClusterFn row_cluster_for_f16(int gs) {
  switch (hamming_planes(gs)) {
    case 1: return row_cluster_kernel<1, 4, F16, RANKS>;
    case 2: return row_cluster_kernel<2, 4, F16, RANKS>;
    case 3: return row_cluster_kernel<3, 4, F16, RANKS>;
    default: return row_cluster_kernel<4, 4, F16, RANKS>;
  }
}

// The instantiation for gs query heads per selection row (128-bit codes) and clusters of
// `ranks` CTAs (16 or 8), and its index among the 16 instantiations.
constexpr int kRowVariants = 16;
inline RowClusterFn row_cluster_for(int gs, bool f16, int ranks) {
  if (ranks == 16)
    return f16 ? row_cluster_for_f16<true, 16>(gs) : row_cluster_for_f16<false, 16>(gs);
  return f16 ? row_cluster_for_f16<true, 8>(gs) : row_cluster_for_f16<false, 8>(gs);
}
inline int row_cluster_index(int gs, bool f16, int ranks) {
  return (ranks == 16 ? 8 : 0) + (f16 ? 4 : 0) + min(hamming_planes(gs), 4) - 1;
}

}  // namespace hhr
