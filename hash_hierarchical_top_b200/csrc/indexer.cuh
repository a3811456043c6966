// HISA indexer selection (steps a1', a3, a4 of the indexer variant) as one thread-block cluster
// per query.
//
// HISA page, Abstract: a block-level coarse filter scores the pooled block representatives
// (the mean key of each block) against the query and keeps the best blocks; the original token
// indexer then scores the keys of the kept blocks only, and the top-k tokens are selected.
// Run as four kernels (block scores, top-m blocks, token scores, token top-k), a decode query
// (T = 1) is a chain of four launches with two single-CTA selections. Here one cluster of
// kIxRanks CTAs does the whole chain for one query:
//   1. rank r scores its contiguous slice of the blocks (a warp per 8 blocks, one coalesced
//      16-byte piece of each block mean per lane) and writes the scores (-inf for a block that
//      starts after the query's position);
//   2. after a cluster barrier every rank reads all block scores back through L2 and selects
//      the same top-m blocks (block_select_largest: deterministic, ties to the lower block);
//   3. rank r scores the tokens of its share of the kept blocks (exact fp32 q . k; tokens after
//      the query's position or past the sequence are ineligible) into the workspace;
//   4. after a second cluster barrier rank 0 selects the top-k tokens from all the token
//      scores (block_select_largest: deterministic, ties to the lower token, output in token
//      order).
// The selection rules and outputs are those of hhr_select's indexer mode.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "select.cuh"

namespace hhr {

constexpr int kIxRanks = 16;          // CTAs per query (a non-portable cluster size)
constexpr int kIxThreads = 512;
constexpr int kIxWarps = kIxThreads / 32;
constexpr int kIxMaxBlocks = 4096;    // blocks per sequence (their keys staged in shared memory)
constexpr int kIxMaxCand = 16384;     // token candidates per query (their keys, on rank 0)
// Copies of the selections' radix histograms (see SelShared). Measured on B200 (128K, one
// query, L2-warm, back-to-back selections): 1 copy 24.6 us, 2 copies 24.0 us, 4 copies 24.4 us.
#ifndef HHR_IX_HC
#define HHR_IX_HC 2
#endif
constexpr int kIxHC = HHR_IX_HC;

struct IxArgs {
  const uint16_t* q;        // [B][T][d]
  const float* block_mean;  // [n_phys][1][d]
  const uint16_t* k_cache;  // [n_phys][1][P][d]
  const int32_t* page_table;
  const int32_t* seq_len;
  const int32_t* q_pos;     // [B][T]
  float* scores;            // [B][T][maxp] block scores
  int32_t* kept;            // [B][T][m_max] kept blocks, ascending
  int32_t* kept_count;      // [B][T]
  float* tok;               // [B][T][m_max * P] token scores of the kept blocks (workspace)
  int32_t* out_idx;         // [B][T][top_k]
  int32_t* out_count;       // [B][T]
  int T, P, maxp, n_phys, m_pages, m_max, top_k;
};

struct IxShared {
  SelShared<kIxHC> sel;  // the block selection (every rank) and the token selection (rank 0)
};

// Dynamic shared memory: block keys [maxp], the sequence's page-table row [maxp], kept blocks
// [m_max], their page ids [m_max], the token keys of the token selection [m_max * P].
inline size_t ix_smem(int maxp, int m_max, int P) {
  return (2 * (size_t)maxp + 2 * (size_t)((m_max + 3) & ~3) + (size_t)m_max * P) * 4;
}

__global__ void __launch_bounds__(kIxThreads, 1) indexer_cluster_kernel(IxArgs a) {
  namespace cg = cooperative_groups;
  __shared__ IxShared sh;
  __shared__ __align__(16) float4 qs[kD / 4];
  extern __shared__ __align__(16) uint32_t ix_dyn[];
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int row = blockIdx.y, b = row / a.T;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mw = (a.m_max + 3) & ~3;
  uint32_t* bkeys = ix_dyn;
  int32_t* pt_s = reinterpret_cast<int32_t*>(bkeys + a.maxp);
  int32_t* kept_s = pt_s + a.maxp;
  int32_t* kphys_s = kept_s + mw;
  uint32_t* tkeys = reinterpret_cast<uint32_t*>(kphys_s + mw);
  // The length, position and page-table row are inputs no earlier kernel writes: staged before
  // the dependency wait.
  const int n = a.seq_len[b], pos = a.q_pos[row];
  const int nblk = min(ceil_div(max(n, 0), a.P), a.maxp);
  for (int i = tid; i < nblk; i += kIxThreads) pt_s[i] = a.page_table[(size_t)b * a.maxp + i];
  pdl_wait();
  pdl_trigger();
  if (tid < kD / 4)
    qs[tid] = bf16x4_to_f4(*reinterpret_cast<const uint2*>(a.q + (size_t)row * kD + 4 * tid));
  __syncthreads();
  const float4 qv = qs[lane];
  float* scores = a.scores + (size_t)row * a.maxp;

  // 1. Block scores of this rank's slice: warp w scores blocks base + 0..7.
  {
    const int per = ceil_div(nblk, kIxRanks);
    const int lo = rank * per, hi = min(nblk, lo + per);
    for (int base = lo + warp * 8; base < hi; base += kIxWarps * 8) {
      int my_phys = -1;
      if (lane < 8 && base + lane < hi) {
        my_phys = pt_s[base + lane];
        if (my_phys < 0 || my_phys >= a.n_phys) my_phys = -2;
      }
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int phys = __shfl_sync(kFull, my_phys, i);
        v[i] = 0.f;
        if (phys >= 0) {
          const float4 m = reinterpret_cast<const float4*>(a.block_mean + (size_t)phys * kD)[lane];
          v[i] = qv.x * m.x + qv.y * m.y + qv.z * m.z + qv.w * m.w;
        }
      }
      const float s = warp_sum8_transposed(v, lane);
      const int blk = base + lane;
      if (lane < 8 && blk < hi) {
        if (my_phys == -2) flag_status(kStatusBadPage);
        const bool elig = my_phys >= 0 && (long long)blk * a.P <= (long long)pos;
        scores[blk] = elig ? s : -INFINITY;
      }
    }
  }
  cluster_sync_all();  // every rank's scores are written (visible cluster-wide)

  // 2. The same top-m blocks in every rank (scores read back through L2).
  const int n_el = min(ceil_div(max(min(n, pos + 1), 0), a.P), a.maxp);
  const int m = block_select_largest<kIxThreads, kSelLoadUnroll, kIxHC>(
      scores, n_el, bkeys, sh.sel, true, a.m_pages, 0, 0, kept_s, a.m_max, nullptr, 0);
  __syncthreads();
  for (int i = tid; i < m; i += kIxThreads) {
    const int blk = kept_s[i];
    int phys = pt_s[blk];
    if (phys < 0 || phys >= a.n_phys) phys = -1;
    kphys_s[i] = phys;
    if (rank == 0) a.kept[(size_t)row * a.m_max + i] = blk;
  }
  if (rank == 0 && tid == 0) a.kept_count[row] = m;
  __syncthreads();

  // 3. Token scores of this rank's kept blocks [bl0, bl1): candidate c is slot c % P of kept
  //    block bl0 + c / P, written at index bl0 * P + c of the query's score row (-inf for an
  //    ineligible token). Each lane resolves its candidate's cache row once; the warp then
  //    reads the 32 rows (lane l: channels 4l..4l+3).
  const int kpr = ceil_div(m, kIxRanks);
  const int bl0 = min(m, rank * kpr), bl1 = min(m, bl0 + kpr);
  const int C = (bl1 - bl0) * a.P;
  float* tok = a.tok + (size_t)row * a.m_max * a.P + (size_t)bl0 * a.P;
  for (int c0 = warp * 32; c0 < C; c0 += kIxWarps * 32) {
    const int c = c0 + lane;
    long long krow = -1;  // cache row of the candidate, or -1
    if (c < C) {
      const int i = bl0 + c / a.P, slot = c - (c / a.P) * a.P;
      const int t = kept_s[i] * a.P + slot;
      const int phys = kphys_s[i];
      if (t < n && t <= pos) {
        if (phys >= 0) krow = (long long)phys * a.P + slot;
        else flag_status(kStatusBadPage);
      }
    }
    // All 32 row loads first (a zero piece for a skipped candidate), then the products.
    uint2 kw[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const long long rj = __shfl_sync(kFull, krow, j);
      kw[j] = rj >= 0 ? *reinterpret_cast<const uint2*>(a.k_cache + rj * kD + 4 * lane)
                      : make_uint2(0u, 0u);
    }
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float4 kv = bf16x4_to_f4(kw[j]);
      v[j] = qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
    }
    const float sc = warp_transpose_sum32(v, lane);
    if (c < C) tok[c] = krow >= 0 ? sc : -INFINITY;
  }
  cluster_sync_all();  // every rank's token scores are written (visible cluster-wide)
  if (rank != 0) return;

  // 4. Token top-k on rank 0: the k_eff = min(top_k, #eligible) best (score desc, token asc)
  //    of the m * P candidates, written in token order (candidate order is token order).
  const int k = block_select_largest<kIxThreads, 16, kIxHC>(
      a.tok + (size_t)row * a.m_max * a.P, m * a.P, tkeys, sh.sel, false, 0, 0, a.top_k,
      a.out_idx + (size_t)row * a.top_k, a.top_k, kept_s, a.P);
  int32_t* out = a.out_idx + (size_t)row * a.top_k;
  for (int i = k + tid; i < a.top_k; i += kIxThreads) out[i] = -1;
  if (tid == 0) a.out_count[row] = k;
}

}  // namespace hhr
