// Shared device helpers of the retrieval kernels: bf16 widening, warp/block
// reductions and scans, order-preserving float keys and the device status word.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hhr {

constexpr int kD = 128;         // head_dim supported by every kernel
constexpr int kWords = 4;       // 128-bit codes as 4 x uint32 (the tensor-core encoder)
constexpr int kMaxGroup = 8;    // query heads per KV group
constexpr unsigned kFull = 0xffffffffu;

// Device-side status bits (never a trap): bad page id, bad token index, clipped append.
constexpr int kStatusBadPage = 1;
constexpr int kStatusBadToken = 2;
constexpr int kStatusClipped = 4;
constexpr int kStatusWaitGaveUp = 16;  // a bounded wait on staged page summaries gave up

__device__ int g_status;

__device__ __forceinline__ void flag_status(int bit) {
  if ((*(volatile int*)&g_status & bit) == 0) atomicOr(&g_status, bit);
}

// bf16 bit pattern -> float (exact).
__device__ __forceinline__ float bf16_lo(uint32_t two) { return __uint_as_float(two << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t two) { return __uint_as_float(two & 0xffff0000u); }
__device__ __forceinline__ float bf16_to_f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Unpack 4 bf16 (two 32-bit words) to 4 floats.
__device__ __forceinline__ float4 bf16x4_to_f4(uint2 w) {
  return make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

// Transposed warp reduction: on entry every lane holds v[0..31]; on exit lane l
// holds in v[0] the sum over all lanes of v[l]. 31 shuffles instead of 32 x 5.
__device__ __forceinline__ float warp_transpose_sum32(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      float send = upper ? v[i] : v[i + s];
      float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, s);
    }
  }
  return v[0];
}

// Inclusive warp scan of an int.
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Exclusive block scan of one int per thread; blockDim.x a multiple of 32, <= 1024.
// `scratch` holds >= 33 ints of shared memory. Returns the exclusive prefix and
// writes the block total to *total. Contains __syncthreads(): call uniformly. Without the
// tail barrier (kTailSync false) the caller must pass a barrier before scratch is reused.
template <bool kTailSync = true>
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int incl = warp_incl_scan(v, lane);
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? scratch[lane] : 0;
    int wi = warp_incl_scan(w, lane);
    if (lane < nwarps) scratch[lane] = wi - w;
    if (lane == 31) scratch[32] = wi;
  }
  __syncthreads();
  int res = scratch[warp] + incl - v;
  *total = scratch[32];
  if (kTailSync) __syncthreads();  // before scratch is reused
  return res;
}

// Exclusive block scan of two ints per thread in one pass of barriers (same contract as
// block_excl_scan; `scratch` holds >= 66 ints). Returns both prefixes; *total the totals.
template <bool kTailSync = true>
__device__ __forceinline__ int2 block_excl_scan2(int2 v, int* scratch, int2* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int a = v.x, b = v.y;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int na = __shfl_up_sync(kFull, a, o), nb = __shfl_up_sync(kFull, b, o);
    if (lane >= o) { a += na; b += nb; }
  }
  if (lane == 31) { scratch[warp] = a; scratch[33 + warp] = b; }
  __syncthreads();
  if (warp == 0) {
    const int wa = lane < nwarps ? scratch[lane] : 0, wb = lane < nwarps ? scratch[33 + lane] : 0;
    int ia = wa, ib = wb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int na = __shfl_up_sync(kFull, ia, o), nb = __shfl_up_sync(kFull, ib, o);
      if (lane >= o) { ia += na; ib += nb; }
    }
    if (lane < nwarps) { scratch[lane] = ia - wa; scratch[33 + lane] = ib - wb; }
    if (lane == 31) { scratch[32] = ia; scratch[65] = ib; }
  }
  __syncthreads();
  const int2 res = make_int2(scratch[warp] + a - v.x, scratch[33 + warp] + b - v.y);
  *total = make_int2(scratch[32], scratch[65]);
  if (kTailSync) __syncthreads();  // before scratch is reused
  return res;
}

// Cluster barrier in two halves: every thread of every CTA of the cluster arrives (release:
// its earlier shared-memory writes become visible cluster-wide) and later waits (acquire).
// arrive + wait together act as cluster.sync(), which also covers __syncthreads().
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  cluster_arrive();
  cluster_wait();
}

// Bulk prefetch of `bytes` (a multiple of 16, 16-byte aligned) into L2.
__device__ __forceinline__ void prefetch_l2(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
}

// ---- mbarriers and 1-D bulk copies (shared-memory addresses as 32-bit shared::cta) ----
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
// One arrival that also expects `bytes` of bulk-copy completions in the current phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
// One plain arrival.
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
// Bounded wait for the mbarrier phase with the given parity (at most `limit` polls). False
// on time-out.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, long long limit) {
  for (long long i = 0; i < limit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t"
        "}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}
// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from this GPU's
// global memory into this CTA's shared memory, completing on mbarrier `bar`. No multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// Orders this thread's earlier generic-proxy shared-memory accesses before later async-proxy
// (bulk copy) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// Programmatic dependent launch: wait until the preceding kernel in the stream has
// completed and its writes are visible (a no-op when the launch did not ask for
// programmatic serialisation), and let the next kernel start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// Histogram increment aggregated over the warp's lanes that hit the same bin: one
// shared-memory atomic per distinct bin instead of one per lane (similar scores
// crowd into few bins). `active` = lanes that want to add (the call itself must be
// made by every lane of the warp).
__device__ __forceinline__ void hist_add_aggregated(int* hist, int bin, bool active) {
  const unsigned want = __ballot_sync(kFull, active);
  if (!active) return;
  const unsigned peers = __match_any_sync(want, bin);
  const int leader = __ffs(peers) - 1;
  if ((threadIdx.x & 31) == leader) atomicAdd(&hist[bin], __popc(peers));
}

// Order-preserving map of a float to uint32 (larger float -> larger key; -0 < +0).
__device__ __forceinline__ uint32_t f2key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Kept pages (or blocks) for a row of n units: m_pages > 0 -> min(m_pages, n),
// else ceil(n / keep_div), never more than n.
__device__ __host__ __forceinline__ int kept_for(int n, int m_pages, int keep_div) {
  if (n <= 0) return 0;
  if (m_pages > 0) return m_pages < n ? m_pages : n;
  int m = (n + keep_div - 1) / keep_div;
  return m < n ? m : n;
}

}  // namespace hhr
