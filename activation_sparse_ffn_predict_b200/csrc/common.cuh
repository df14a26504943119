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

// System-scope release store / acquire load of a flag word that other GPUs
// read or write over peer memory, and a relaxed system-scope load of data the
// flag guards.
__device__ __forceinline__ void st_release_sys(uint32_t *p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ float ld_relaxed_sys(const float *p) {
  float v;
  asm volatile("ld.relaxed.sys.global.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void flag_error(int32_t *err, int bit) {
  if (err) atomicOr(err, bit);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------ cp.async --
// 16-byte asynchronous copy global -> shared (L1 bypassed); src_bytes < 16
// zero-fills the rest of the 16 bytes (0 reads nothing).  Weight streams pass
// the L2 evict-first policy.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Order this thread's completed generic-proxy shared-memory writes (cp.async,
// st.shared) before later async-proxy reads (tensor-core operands).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------ tensor-map (TMA) loads --
// A tensor map is a kernel parameter (const __grid_constant__ CUtensorMap);
// these take its generic address.  No multicast.
//
// 2-D tile load of the box at (x, y) into shared memory, completing its bytes
// on bar.  x * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
// Four rows (y0..y3, any order) of a map whose box is one row high, columns
// x.. of the box width, written as four consecutive box rows at dst (the
// swizzle follows the shared-memory address).
__device__ __forceinline__ void tma_gather4(void *dst, const void *tmap, int x, int y0, int y1, int y2, int y3,
                                            uint64_t *bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// ----------------------------------------------------- tcgen05 (sm_100a) --
// Tensor memory: allocated by one whole warp, address written to shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor of a tcgen05 operand: start address,
// leading / stride byte offsets (16-byte units), descriptor version 1 and the
// swizzle mode (kSwz128 / kSwz64 / kSwz32 / kSwzNone).
constexpr uint32_t kSwzNone = 0, kSwz128 = 2, kSwz64 = 4, kSwz32 = 6;
__device__ __forceinline__ uint64_t umma_desc(const void *smem, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t swz) {
  const uint32_t a = smem_u32(smem);
  uint64_t d = (uint64_t)((a >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(swz & 7u) << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: fp16 A and B, fp32 D,
// M x N tile, A / B K-major (0) or MN-major (1).
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4)                                   // D format: f32
         | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16)
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D (tensor memory) += A (smem) * B (smem)^T, or D = ... when accum == 0.
// Issued by one thread.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
// Arrive (once) on an mbarrier when every tcgen05.mma this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 16 consecutive 32-bit columns of this thread's tensor-memory lane (the warp
// reads lanes 32*(warp%4) .. +31), then the wait that makes them usable.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
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
