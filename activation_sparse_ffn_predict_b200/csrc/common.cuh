// Device helpers shared by the asffn kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace asf {

constexpr int kWarp = 32;

// Bits of the device error word (workspace offset 0).
constexpr int kErrIndex = 1;    // idx outside [0, n) or count outside [0, n]
constexpr int kErrTimeout = 2;  // a bounded wait gave up

// Workspace header: error word, compaction ticket, per-column-tile tickets.
constexpr size_t kHeaderBytes = 4096;
constexpr int kMaxTiles = 960;  // ticket slots for the down-projection reduction
struct Header {
  int32_t err;
  uint32_t done;
  uint32_t pad[14];
  uint32_t tile_done[kMaxTiles];
};
static_assert(sizeof(Header) <= kHeaderBytes, "header too large");

// ---------------------------------------------------------------- PTX --
// L2 policy for weight streams: their lines are the first evicted, so the
// streams do not push out what every kernel re-reads -- its code, and the
// small per-step data (x, h, the union mask, index lists, partial sums).
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Streaming 16-byte load of read-only weights: skip L1, evict first from L2.
__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p), "l"(l2_evict_first()));
  return v;
}

// The same, as a volatile asm: it stays where it is written, so weights loaded
// ahead of griddepcontrol.wait are in flight while the kernel waits.
__device__ __forceinline__ uint4 ld_stream_early(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(l2_evict_first()));
  return v;
}

// Load of data another kernel (or CTA) produced: served from L2, never L1.
__device__ __forceinline__ int ld_cg_i32(const int32_t *p) { return __ldcg(p); }
__device__ __forceinline__ float ld_cg_f32(const float *p) { return __ldcg(p); }
__device__ __forceinline__ uint32_t ld_cg_u32(const uint32_t *p) { return __ldcg(p); }

// Programmatic dependent launch: wait for the preceding grid's memory, and
// allow the next grid in the stream to start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Bulk prefetch of a contiguous range into L2 (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ------------------------------------------------ mbarrier + bulk copy --
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t tx) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(tx) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the given phase parity, giving up after limit_ns of wall time.
// Returns false on timeout; the caller records the error and stops using the
// data the barrier guards.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// Bulk asynchronous copy global -> this CTA's shared memory, completing bytes
// on the mbarrier (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// The same for weight streams, with the L2 evict-first policy (pol from
// l2_evict_first()).
__device__ __forceinline__ void bulk_g2s_stream(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                                uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// Named barrier over the first `threads` threads of the CTA.
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Producer side of a named barrier: marks arrival without waiting; the
// threads that bar.sync on the same id (count includes the arrivers) see this
// thread's earlier memory accesses once they pass it.
__device__ __forceinline__ void named_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Ticket for "last CTA to finish" patterns: callers __syncthreads() first so
// the whole CTA's writes precede thread 0's release; the acquire half lets the
// last arriver read every other CTA's writes after a following __syncthreads().
__device__ __forceinline__ uint32_t ticket_acq_rel(uint32_t *p) {
  uint32_t old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

__device__ __forceinline__ void flag_error(int32_t *err, int bit) {
  if (err) atomicOr(err, bit);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------- element types --
// Vec<T>: one 16-byte chunk of weights holds N elements of T.
template <typename T> struct Vec;

template <> struct Vec<float> {
  static constexpr int N = 4;
  // acc + sum_i w_i * x_i, x in the same 16-byte layout
  __device__ __forceinline__ static float dot(uint4 w, uint4 x, float acc) {
    acc = fmaf(__uint_as_float(w.x), __uint_as_float(x.x), acc);
    acc = fmaf(__uint_as_float(w.y), __uint_as_float(x.y), acc);
    acc = fmaf(__uint_as_float(w.z), __uint_as_float(x.z), acc);
    acc = fmaf(__uint_as_float(w.w), __uint_as_float(x.w), acc);
    return acc;
  }
  // acc + sum_i w_i * x_i with x as N floats
  __device__ __forceinline__ static float dotf(uint4 w, const float *x, float acc) {
    const float4 a = *reinterpret_cast<const float4 *>(x);
    acc = fmaf(__uint_as_float(w.x), a.x, acc);
    acc = fmaf(__uint_as_float(w.y), a.y, acc);
    acc = fmaf(__uint_as_float(w.z), a.z, acc);
    acc = fmaf(__uint_as_float(w.w), a.w, acc);
    return acc;
  }
  __device__ __forceinline__ static float dotr(uint4 w, const float (&x)[4], float acc) {
    acc = fmaf(__uint_as_float(w.x), x[0], acc);
    acc = fmaf(__uint_as_float(w.y), x[1], acc);
    acc = fmaf(__uint_as_float(w.z), x[2], acc);
    acc = fmaf(__uint_as_float(w.w), x[3], acc);
    return acc;
  }
  __device__ __forceinline__ static void to_float(uint4 w, float (&f)[4]) {
    f[0] = __uint_as_float(w.x);
    f[1] = __uint_as_float(w.y);
    f[2] = __uint_as_float(w.z);
    f[3] = __uint_as_float(w.w);
  }
};

template <> struct Vec<__half> {
  static constexpr int N = 8;
  __device__ __forceinline__ static float2 h2f(uint32_t u) {
    __half2 h = *reinterpret_cast<__half2 *>(&u);
    return __half22float2(h);
  }
  __device__ __forceinline__ static float dot(uint4 w, uint4 x, float acc) {
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
    const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 a = h2f(wv[i]);
      const float2 b = h2f(xv[i]);
      acc = fmaf(a.x, b.x, acc);
      acc = fmaf(a.y, b.y, acc);
    }
    return acc;
  }
  // x: 8 floats split in two 4-float planes at x0 and x1
  __device__ __forceinline__ static float dotf2(uint4 w, const float *x0, const float *x1,
                                                float acc) {
    const float4 a = *reinterpret_cast<const float4 *>(x0);
    const float4 b = *reinterpret_cast<const float4 *>(x1);
    float2 p;
    p = h2f(w.x); acc = fmaf(p.x, a.x, acc); acc = fmaf(p.y, a.y, acc);
    p = h2f(w.y); acc = fmaf(p.x, a.z, acc); acc = fmaf(p.y, a.w, acc);
    p = h2f(w.z); acc = fmaf(p.x, b.x, acc); acc = fmaf(p.y, b.y, acc);
    p = h2f(w.w); acc = fmaf(p.x, b.z, acc); acc = fmaf(p.y, b.w, acc);
    return acc;
  }
  // acc + sum_i w_i * x_i with x as 8 floats held in registers
  __device__ __forceinline__ static float dotr(uint4 w, const float (&x)[8], float acc) {
    float2 p;
    p = h2f(w.x); acc = fmaf(p.x, x[0], acc); acc = fmaf(p.y, x[1], acc);
    p = h2f(w.y); acc = fmaf(p.x, x[2], acc); acc = fmaf(p.y, x[3], acc);
    p = h2f(w.z); acc = fmaf(p.x, x[4], acc); acc = fmaf(p.y, x[5], acc);
    p = h2f(w.w); acc = fmaf(p.x, x[6], acc); acc = fmaf(p.y, x[7], acc);
    return acc;
  }
  __device__ __forceinline__ static void to_float(uint4 w, float (&f)[8]) {
    float2 p;
    p = h2f(w.x); f[0] = p.x; f[1] = p.y;
    p = h2f(w.y); f[2] = p.x; f[3] = p.y;
    p = h2f(w.z); f[4] = p.x; f[5] = p.y;
    p = h2f(w.w); f[6] = p.x; f[7] = p.y;
  }
};

}  // namespace asf
