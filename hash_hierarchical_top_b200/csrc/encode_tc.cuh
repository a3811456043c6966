// Step a0 in bulk (a prefill) on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// HHR page, Abstract: keys are rotated by the head-wise orthogonal R_h (GKR) and encoded
// into binary codes of a head-wise projection (LHP). For a block of keys K (rows) both
// are one dense product: [K R_g^T | K (W_g R_g)^T], i.e. D = K B^T with
// B = [R_g ; W_g R_g] (256 x 128). D's first 128 columns are the rotated keys (reduced to
// per-page channel min/max), its last 128 columns the projections (packed sign bits).
//
// Precision: K is bf16 and exact on the tensor cores; B is fp32 and is split into three
// bf16 terms (hi + mid + lo, about 2^-24 relative), each multiplied by K and accumulated
// in fp32 in TMEM — enough for the 1e-4 ||k|| code tolerance, which plain bf16 or tf32
// operands are not.
//
// One persistent CTA of 512 threads per (slot, KV group): it builds B_g once in shared
// memory (M = W_g R_g computed in fp32, then split), then loops over 128-key tiles of its
// group (4 pages of 32 keys) in a two-deep software pipeline. For tile k: the rows, already
// in registers, are stored into the 128-byte-swizzled K-major A buffer; one thread issues 8
// k-steps x 3 splits of tcgen05.mma (M=128, N=256, K=16) into one of two 256-column TMEM
// accumulators and commits to that accumulator's mbarrier; while those MMAs run, the threads
// load tile k+1's rows (through the page table) into registers and run the epilogue of tile
// k-1 from the other accumulator: warp w reads TMEM lanes 32(w % 4)..32(w % 4)+31 (= the keys
// of page w % 4 of the tile), columns of group c = w / 4: rotated channels 32c..32c+31, whose
// min/max over the page a transposed warp reduction gives, and projections of code word c,
// whose 32 sign bits each lane packs for its key. Then the CTA waits for tile k's MMAs (the A
// buffer is free again). A shared-memory double buffer for A does not fit next to the 192 KB
// of B; registers hold the next tile instead (4 x 16 B per thread).
// Measured on B200 (prefill of 128K x 8 sequences x 8 groups): with 4 warps the epilogue was
// instruction-bound (ncu: 6% of warp slots, tensor pipe 23.7% active) and the overlap alone
// gained 3% (3.12 -> 3.04 ms); 16 warps: 1.89 ms, tensor pipe 40.5%; 32 warps (16 columns
// each): 2.23 ms, tensor pipe 34%. All mbarrier waits are bounded.
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"
#include "encode.cuh"

namespace hhr {

constexpr int kTcTile = 128;               // keys per tile (MMA M)
constexpr int kTcN = 256;                  // 128 rotated channels + 128 projections (MMA N)
constexpr int kTcThreads = 512;             // 16 warps: 4 per TMEM lane quarter
constexpr int kTcSplits = 3;
constexpr int kTcPage = 32;                // page size served by this kernel
constexpr uint32_t kTcBHalf = kTcN * 128;  // bytes of one 64-channel half of one split of B
constexpr uint32_t kTcBSplit = 2 * kTcBHalf;
constexpr uint32_t kTcBBytes = kTcSplits * kTcBSplit;  // 192 KB
constexpr uint32_t kTcAHalf = kTcTile * 128;
constexpr uint32_t kTcABytes = 2 * kTcAHalf;           // 32 KB
constexpr size_t kTcSmem = kTcBBytes + kTcABytes + 1024 /*alignment*/ + 64 /*barriers, tmem*/;
constexpr uint32_t kTcTmemCols = 2 * kTcN;             // two accumulators
constexpr int kTcChunks = kTcTile * 16 / kTcThreads;   // 16-byte row chunks per thread
constexpr int kStatusTimeout = 8;
constexpr long long kTcWaitLimit = 1ll << 22;  // try_wait polls before giving up

// Byte offset of element (row, k) of a [rows][128] bf16 operand in the K-major
// 128-byte-swizzle layout: two 64-channel halves, 128 B per row, 16-byte chunk c of row r
// stored at chunk c ^ (r % 8) (atoms of 8 rows x 128 B, 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t half_bytes, int row, int k) {
  const int h = k >> 6, c = (k & 63) >> 3;
  return (uint32_t)h * half_bytes + (uint32_t)row * 128u + (uint32_t)((c ^ (row & 7)) << 4) +
         (uint32_t)((k & 7) << 1);
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);  // start address (16-byte units)
  d |= (uint64_t)1u << 16;                       // leading byte offset (unused for swizzle)
  d |= (uint64_t)(1024u >> 4) << 32;             // stride byte offset: next 8-row atom
  d |= (uint64_t)1u << 46;                       // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                       // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A and B, f32 accumulator, both K-major,
// M = 128, N = 256.
__device__ __forceinline__ uint32_t tc_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTcN >> 3) << 17) |
         ((uint32_t)(kTcTile >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Bounded wait for the mbarrier phase with the given parity. False on time-out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  return mbar_wait_bounded(bar, parity, kTcWaitLimit);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Transposed warp reduction with min (or max): lane l ends with the min (max) over all
// lanes of v[l].
template <bool kMax>
__device__ __forceinline__ float warp_transpose_minmax32(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      const float other = __shfl_xor_sync(kFull, send, s);
      v[i] = kMax ? fmaxf(keep, other) : fminf(keep, other);
    }
  }
  return v[0];
}

struct EncodeTcArgs {
  const uint16_t* k_cache;
  const int32_t* page_table;
  const int32_t* start;
  const int32_t* n_new;
  const float* R;
  const float* W;
  void* page_minmax;
  uint32_t* codes;
  int B, G, maxp, n_phys, max_new, summary_fp16;
  int ctas_per_group, tiles_per_seq;
};

__global__ void __launch_bounds__(kTcThreads, 1) encode_tc_kernel(EncodeTcArgs a) {
  extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slot_cta = blockIdx.x, g = blockIdx.y;
  const uint32_t raw = (uint32_t)__cvta_generic_to_shared(tc_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;          // 1024-aligned swizzle atoms
  uint8_t* gbase = tc_smem_raw + (base - raw);
  const uint32_t sB = base, sA = base + kTcBBytes;
  uint8_t* gB = gbase;
  uint8_t* gA = gbase + kTcBBytes;
  uint32_t* taddr_p = reinterpret_cast<uint32_t*>(gbase + kTcBBytes + kTcABytes + 16);
  const uint32_t bar0 = sA + kTcABytes;  // MMA completion of accumulator 0 (bar0 + 8: 1)

  // ---- B = [R_g ; W_g R_g] as three bf16 splits, in the swizzled K-major layout -------
  const float* Rg = a.R + (size_t)g * kD * kD;
  const float* Wg = a.W + (size_t)g * kD * kD;
  auto put_split = [&](int n, int k, float x) {
    const float hi = __bfloat162float(__float2bfloat16_rn(x));
    const float r1 = x - hi;
    const float mid = __bfloat162float(__float2bfloat16_rn(r1));
    const float lo = r1 - mid;
    const uint32_t off = sw128_offset(kTcBHalf, n, k);
    *reinterpret_cast<__nv_bfloat16*>(gB + off) = __float2bfloat16_rn(hi);
    *reinterpret_cast<__nv_bfloat16*>(gB + kTcBSplit + off) = __float2bfloat16_rn(mid);
    *reinterpret_cast<__nv_bfloat16*>(gB + 2 * kTcBSplit + off) = __float2bfloat16_rn(lo);
  };
  for (int i = tid; i < kD * kD; i += kTcThreads) put_split(i >> 7, i & 127, Rg[i]);
  // M = W_g R_g: warp w computes rows kRowsW w .. kRowsW (w + 1) - 1, 8 rows at a time, lane l
  // columns 4l..4l+3.
  constexpr int kRowsW = kD / (kTcThreads / 32);
  constexpr int kStepR = kRowsW < 8 ? kRowsW : 8;
  static_assert(kRowsW % kStepR == 0, "whole steps of rows");
  for (int r0 = warp * kRowsW; r0 < (warp + 1) * kRowsW; r0 += kStepR) {
    float4 acc[kStepR];
#pragma unroll
    for (int j = 0; j < kStepR; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int l = 0; l < kD; ++l) {
      const float4 rv = __ldg(reinterpret_cast<const float4*>(Rg + (size_t)l * kD) + lane);
#pragma unroll
      for (int j = 0; j < kStepR; ++j) {
        const float w = __ldg(Wg + (size_t)(r0 + j) * kD + l);
        acc[j].x = fmaf(w, rv.x, acc[j].x);
        acc[j].y = fmaf(w, rv.y, acc[j].y);
        acc[j].z = fmaf(w, rv.z, acc[j].z);
        acc[j].w = fmaf(w, rv.w, acc[j].w);
      }
    }
#pragma unroll
    for (int j = 0; j < kStepR; ++j) {
      put_split(kD + r0 + j, 4 * lane + 0, acc[j].x);
      put_split(kD + r0 + j, 4 * lane + 1, acc[j].y);
      put_split(kD + r0 + j, 4 * lane + 2, acc[j].z);
      put_split(kD + r0 + j, 4 * lane + 3, acc[j].w);
    }
  }
  // Tensor-core reads of shared memory go through the async proxy.
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");

  if (tid == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(taddr_p)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = *taddr_p;
  const uint32_t idesc = tc_idesc();
  uint32_t parity = 0u;  // bit i: the phase parity the next wait on accumulator i expects
  bool failed = false;

  // This CTA's tiles: j = slot_cta, slot_cta + ctas_per_group, ... that hold appended keys.
  const int total_tiles = a.B * a.tiles_per_seq;
  auto tile_live = [&](int j) {
    const int b = j / a.tiles_per_seq, ti = j % a.tiles_per_seq;
    int nn = a.n_new[b];
    if (nn > a.max_new) nn = a.max_new;
    const int s0 = a.start[b];
    if (nn <= 0 || s0 < 0) return false;
    const int T0 = ti * kTcTile;
    return T0 < s0 + nn && T0 + kTcTile > s0;
  };
  auto next_tile = [&](int j) {
    for (j += a.ctas_per_group; j < total_tiles; j += a.ctas_per_group)
      if (tile_live(j)) return j;
    return total_tiles;
  };
  // Rows of tile j into registers: thread tid takes chunks q = tid + i * kTcThreads (row q/16,
  // 16-byte chunk q%16); rows outside the appended range (or of a bad page) are zero.
  uint4 rows[kTcChunks];
  auto load_rows = [&](int j) {
    const int b = j / a.tiles_per_seq, T0 = (j % a.tiles_per_seq) * kTcTile;
    int nn = a.n_new[b];
    if (nn > a.max_new) nn = a.max_new;
    const int s0 = a.start[b], e0 = s0 + nn;
#pragma unroll
    for (int i = 0; i < kTcChunks; ++i) {
      const int q = tid + i * kTcThreads;
      const int r = q >> 4, ch = q & 15;
      const int t = T0 + r;
      const int lp = t / kTcPage;
      int phys = -1;
      if (t >= s0 && t < e0 && lp < a.maxp) {
        phys = a.page_table[(size_t)b * a.maxp + lp];
        if (phys >= a.n_phys) phys = -1;
      }
      rows[i] = make_uint4(0, 0, 0, 0);
      if (phys >= 0)
        rows[i] = __ldcs(reinterpret_cast<const uint4*>(
            a.k_cache + (((size_t)phys * a.G + g) * kTcPage + (t % kTcPage)) * kD + ch * 8));
    }
  };
  auto store_rows = [&]() {
#pragma unroll
    for (int i = 0; i < kTcChunks; ++i) {
      const int q = tid + i * kTcThreads;
      *reinterpret_cast<uint4*>(gA + sw128_offset(kTcAHalf, q >> 4, (q & 15) * 8)) = rows[i];
    }
  };
  // Epilogue of tile j from accumulator acc (its MMAs complete).
  auto epilogue = [&](int j, int acc) {
    const int b = j / a.tiles_per_seq, T0 = (j % a.tiles_per_seq) * kTcTile;
    int nn = a.n_new[b];
    if (nn > a.max_new) nn = a.max_new;
    const int s0 = a.start[b], e0 = s0 + nn;
    // Warp w holds the keys of page w % 4 of the tile (positions T0 + 32 (w % 4) + lane) and
    // column group cb = w / 4 (rotated channels 32cb.., code word cb).
    const int quarter = warp & 3, cb = warp >> 2;
    const int t = T0 + quarter * 32 + lane;
    const int lp = t / kTcPage;
    const bool valid = t >= s0 && t < e0;
    int phys = -1;
    if (lp < a.maxp) phys = a.page_table[(size_t)b * a.maxp + lp];
    if (phys >= a.n_phys) phys = -1;
    const bool page_ok = __shfl_sync(kFull, phys, 0) >= 0;
    const int pstart = lp * kTcPage;
    const bool any_valid = __any_sync(kFull, valid);
    const uint32_t trow = tmem + (uint32_t)(acc * kTcN) + ((uint32_t)(quarter * 32) << 16);
    // Rotated channels: per-page min/max (page-uniform phys: all lanes of the warp share lp).
    if (any_valid && page_ok) {
      const size_t sbase = ((size_t)phys * a.G + g) * 2 * kD;
      const bool merge = s0 > pstart;  // the page already held keys before this call
      {
        float v[32], w[32];
        tmem_ld32(trow + (uint32_t)(cb * 32), v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          w[i] = valid ? v[i] : -INFINITY;
          v[i] = valid ? v[i] : INFINITY;
        }
        float mn = warp_transpose_minmax32<false>(v, lane);
        float mx = warp_transpose_minmax32<true>(w, lane);
        const int ch = cb * 32 + lane;
        if (a.summary_fp16) {
          __half* mm = reinterpret_cast<__half*>(a.page_minmax) + sbase;
          if (merge) {
            mn = fminf(mn, __half2float(mm[ch]));
            mx = fmaxf(mx, __half2float(mm[kD + ch]));
          }
          mm[ch] = __float2half_rd(mn);
          mm[kD + ch] = __float2half_ru(mx);
        } else {
          float* mm = reinterpret_cast<float*>(a.page_minmax) + sbase;
          if (merge) {
            mn = fminf(mn, mm[ch]);
            mx = fmaxf(mx, mm[kD + ch]);
          }
          mm[ch] = mn;
          mm[kD + ch] = mx;
        }
      }
      // Projections: code word cb of this lane's key (32 sign bits).
      {
        float v[32];
        tmem_ld32(trow + (uint32_t)(kD + cb * 32), v);
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) word |= (v[i] > 0.f ? 1u : 0u) << i;
        if (valid)
          a.codes[(((size_t)phys * a.G + g) * kTcPage + (t % kTcPage)) * kWords + cb] = word;
      }
    } else if (any_valid && lane == 0) {
      flag_status(kStatusBadPage);
    }
  };

  int cur = tile_live(slot_cta) ? slot_cta : next_tile(slot_cta);
  int prev = -1, acc = 0;
  if (cur < total_tiles) load_rows(cur);
  while (cur < total_tiles) {
    // The A buffer is free (the previous tile's MMAs completed): tile cur's rows go in.
    store_rows();
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t bar = bar0 + 8u * (uint32_t)acc;
    if (tid == 0) {
      const uint32_t d = tmem + (uint32_t)(acc * kTcN);
#pragma unroll 1
      for (int s = 0; s < 8; ++s) {  // k-steps of 16 channels
        const uint32_t koff = (uint32_t)(s & 3) * 32u;  // 16 channels = 32 B into the half
        const uint64_t da = sw128_desc(sA + (uint32_t)(s >> 2) * kTcAHalf + koff);
#pragma unroll
        for (int sp = 0; sp < kTcSplits; ++sp) {
          const uint64_t db =
              sw128_desc(sB + (uint32_t)sp * kTcBSplit + (uint32_t)(s >> 2) * kTcBHalf + koff);
          tc_mma(d, da, db, idesc, (s > 0 || sp > 0) ? 1u : 0u);
        }
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                       bar)
                   : "memory");
    }
    // While tile cur's MMAs run: the next tile's rows into registers, the previous tile's
    // epilogue from the other accumulator.
    const int nxt = next_tile(cur);
    if (nxt < total_tiles) load_rows(nxt);
    if (prev >= 0) epilogue(prev, acc ^ 1);
    const bool ok = mbar_wait(bar, (parity >> acc) & 1u);
    if (__syncthreads_or(!ok)) {  // one decision for the whole CTA
      failed = true;
      if (tid == 0) flag_status(kStatusTimeout);
      break;
    }
    parity ^= 1u << acc;
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    prev = cur;
    cur = nxt;
    acc ^= 1;
  }
  if (!failed && prev >= 0) epilogue(prev, acc ^ 1);
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();

  // On a time-out, give the outstanding MMAs a bounded chance to finish before freeing TMEM.
  if (failed) mbar_wait(bar0 + 8u * (uint32_t)acc, (parity >> acc) & 1u);
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                 "r"(kTcTmemCols)
                 : "memory");
}

}  // namespace hhr
