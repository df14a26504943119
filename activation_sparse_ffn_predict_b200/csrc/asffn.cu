// libasffn: activation-sparse FFN decode path for B200 (sm_100a).
//
// Operations (see include/asffn.h for the ABI contract) and their kernels:
//   predictor layer 1   h = ReLU(W1 x + b1)                        k_pred_l1
//   predictor layer 2   z = W2 h + b2, z > logit(tau), OR of the   k_pred2_ring (B <= 8),
//                       per-token bits into the union mask          k_pred_l2 (B > 8, compacts
//                                                                   in its last CTA)
//   compaction          mask -> ascending idx, count               k_compact (asf_predict),
//                                                                   or inside k_sparse_ffn
//   sparse FFN          a_k = ReLU(Wg[k].x + b_k) * Wu[k].x        k_sparse_ffn + k_reduce_partials
//                       (or ReLU(Wu[k].x + b_k)) for k in idx,      (B <= 4), k_ffn_gu + k_ffn_down
//                       y = sum_k a_k WdT[k]                        (larger batches)
//   profiler            counts[k] += #(ReLU input > 0)             k_act_counts
//   row gather          dst[i] = src[perm[i]]                      k_permute_rows
//
// Method: "PowerInfer Guide: Exploiting Activation Sparsity for LLM AI" (FFN
// equation in "The Hidden Inefficiency"; predictor equation in section 3
// "Adaptive Online Neuron Predictors"; section 4 "Neuron-Aware Sparse GPU
// Operators"; Step 1 profiler) and the 2-layer MLP predictor of the
// "PowerInfer_x64" page.  The kernels are this library's own B200 design:
// weight rows reach shared memory by cp.async.bulk into mbarrier-completed
// rings (or registers, for the register-streaming kernels) with an L2
// evict-first policy, and each weight byte is read once; accumulation is
// fp32; every cross-CTA reduction is a fixed-order sum (no float atomics).
// Consecutive kernels overlap through programmatic dependent launch: each
// kernel touches only weights before griddepcontrol.wait and triggers its
// successor at entry.  Every wait on an mbarrier gives up after 200 ms and
// records ASF_ERR_TIMEOUT in the workspace error word instead of hanging.

#include <cuda.h>            // CUtensorMap and its encoder's types (the encoder comes from the runtime)
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "asffn.h"
#include "common.cuh"

using namespace asf;

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / kWarp;
constexpr int kMaxSplits = 64;        // max CTAs summing into one column tile
constexpr int kTargetCtas = 296;      // 2 CTAs on each of the 148 SMs
constexpr size_t kSmemBudget = 96 * 1024;
constexpr int kFusedWarps = 8;        // consumer warps of the fused sparse FFN
constexpr int kMaxGrid = 256;         // upper bound of one-CTA-per-SM grids (partials, counts)
// Shared memory of the sparse FFN's ring: deep enough to keep ~8 neurons'
// rows in flight per SM, while the layer-1 predictor kernel (one token group
// of x) still fits beside it, so the next layer can start under its tail.
constexpr size_t kFusedSmemDefault = 200 * 1024;
constexpr uint64_t kWaitNs = 200ull * 1000 * 1000;  // bound on any mbarrier wait
constexpr int kInjectWithholdFfn = ASF_INJECT_WITHHOLD_FFN_COPIES;

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ======================================================================== //
// shared building blocks                                                   //
// ======================================================================== //

// Dot products of one weight row with NB activation vectors held in shared
// memory in the weight's own 16-byte chunk layout.  Lane l handles chunks
// l, l+32, ...; U chunks per lane are loaded before any is used (predicated
// at the row end), so a warp keeps U x 512 bytes in flight.
template <typename T, int NB, int U>
__device__ __forceinline__ void row_dot(const T *__restrict__ w, const T *xs, int xs_stride,
                                        int nvec, int lane, float (&acc)[NB]) {
  constexpr int V = Vec<T>::N;
  for (int c0 = lane; c0 < nvec; c0 += U * kWarp) {
    uint4 wv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kWarp;
      wv[u] = c < nvec ? ld_stream(w + (size_t)c * V) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kWarp;
      if (c < nvec) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const uint4 xv = *reinterpret_cast<const uint4 *>(xs + (size_t)b * xs_stride + (size_t)c * V);
          acc[b] = Vec<T>::dot(wv[u], xv, acc[b]);
        }
      }
    }
  }
}

// Same for two rows sharing the activation loads (gate and up of one neuron).
template <typename T, int NB, int U>
__device__ __forceinline__ void row_dot2(const T *__restrict__ w0, const T *__restrict__ w1,
                                         const T *xs, int xs_stride, int nvec, int lane,
                                         float (&acc0)[NB], float (&acc1)[NB]) {
  constexpr int V = Vec<T>::N;
  for (int c0 = lane; c0 < nvec; c0 += U * kWarp) {
    uint4 wa[U], wb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kWarp;
      const bool in = c < nvec;
      wa[u] = in ? ld_stream(w0 + (size_t)c * V) : make_uint4(0u, 0u, 0u, 0u);
      wb[u] = in ? ld_stream(w1 + (size_t)c * V) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kWarp;
      if (c < nvec) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const uint4 xv = *reinterpret_cast<const uint4 *>(xs + (size_t)b * xs_stride + (size_t)c * V);
          acc0[b] = Vec<T>::dot(wa[u], xv, acc0[b]);
          acc1[b] = Vec<T>::dot(wb[u], xv, acc1[b]);
        }
      }
    }
  }
}

// Copy tokens [g0, g0+nb) of x ([B][d], dtype T) into shared memory [NB][d],
// zero-filling the unused token slots.  x may come from the previous kernel,
// so it is read through L2.
template <typename T, int NB>
__device__ __forceinline__ void stage_tokens(T *xs, const T *__restrict__ x, int d, int g0, int nb) {
  constexpr int V = Vec<T>::N;
  const int nvec = d / V;
  constexpr int MAXU = 4;    // loads issued before the first store
  for (int i0 = threadIdx.x; i0 < NB * nvec; i0 += MAXU * blockDim.x) {
    uint4 v[MAXU];
#pragma unroll
    for (int u = 0; u < MAXU; ++u) {
      const int i = i0 + u * blockDim.x;
      const int b = i / nvec;
      v[u] = (i < NB * nvec && b < nb)
                 ? __ldcg(reinterpret_cast<const uint4 *>(x + (size_t)(g0 + b) * d) + (i - b * nvec))
                 : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < MAXU; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < NB * nvec) reinterpret_cast<uint4 *>(xs)[i] = v[u];
    }
  }
}

// Spread an L2 prefetch of [p, p + bytes) over the CTA's threads in 16 KB
// pieces (bytes is a multiple of 16, p 16-byte aligned).
__device__ __forceinline__ void prefetch_range(const void *p, size_t bytes) {
  constexpr size_t kPiece = 16384;
  const unsigned char *c = static_cast<const unsigned char *>(p);
  for (size_t o = (size_t)threadIdx.x * kPiece; o < bytes; o += (size_t)blockDim.x * kPiece)
    prefetch_l2(c + o, (uint32_t)min(kPiece, bytes - o));
}

// Up to two device ranges to pull into L2 for whatever runs next (the
// asf_ffn.l2_next hint).  Sizes are multiples of 16 bytes.
struct L2Next {
  const unsigned char *p[2];
  long long bytes[2];
};

// Lanes of one warp issue this CTA's share (part of parts) of the ranges in
// 32 KB pieces, piece q going to part q mod parts.
__device__ __forceinline__ void prefetch_next(const L2Next &nx, int part, int parts) {
  constexpr long long kPiece = 32768;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (!nx.p[i]) continue;
    const long long np = (nx.bytes[i] + kPiece - 1) / kPiece;
    for (long long q = part + (long long)parts * lane; q < np; q += (long long)parts * kWarp)
      prefetch_l2(nx.p[i] + q * kPiece, (uint32_t)min(kPiece, nx.bytes[i] - q * kPiece));
  }
}

// The FFN rows of a layer's hot block (the leading rows of the hot-first
// storage order): up to three contiguous ranges (one in the packed layout,
// gate / up / down rows otherwise), sizes multiples of 16 bytes.
struct HotBlock {
  const unsigned char *p[3];
  long long bytes[3];
};

// This CTA's share (part of parts) of an L2 prefetch of the hot block, in
// 32 KB pieces issued by the lanes of one warp.
__device__ __forceinline__ void prefetch_hot(const HotBlock &hb, int part, int parts) {
  constexpr long long kPiece = 32768;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    if (!hb.p[i]) continue;
    const long long np = (hb.bytes[i] + kPiece - 1) / kPiece;
    for (long long q = part + (long long)parts * lane; q < np; q += (long long)parts * kWarp)
      prefetch_l2(hb.p[i] + q * kPiece, (uint32_t)min(kPiece, hb.bytes[i] - q * kPiece));
  }
}

// Copy n16 16-byte units from global (data written by the previous kernel,
// read through L2) into shared memory using the first `nthreads` threads.  All
// of a thread's loads are issued before its first store, so the copy costs one
// memory round trip instead of one per unit.
template <int MAXU>
__device__ __forceinline__ void stage16(uint4 *dst, const uint4 *__restrict__ src, int n16, int nthreads) {
  if ((int)threadIdx.x >= nthreads) return;
  uint4 v[MAXU];
#pragma unroll
  for (int u = 0; u < MAXU; ++u) {
    const int i = threadIdx.x + u * nthreads;
    v[u] = i < n16 ? __ldcg(src + i) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u = 0; u < MAXU; ++u) {
    const int i = threadIdx.x + u * nthreads;
    if (i < n16) dst[i] = v[u];
  }
  for (int i = threadIdx.x + MAXU * nthreads; i < n16; i += nthreads) dst[i] = __ldcg(src + i);
}

// ======================================================================== //
// predictor                                                                //
// ======================================================================== //

// Layer 1: h[b][i] = max(W1[i] . x[b] + b1[i], 0).  CTA c owns rows
// [c*rpc, (c+1)*rpc); warps take rows round-robin.  Also clears the union mask
// that layer 2 fills.
template <typename T, int NB, int U>
__global__ void __launch_bounds__(kThreads)
    k_pred_l1(const T *__restrict__ W1, const float *__restrict__ b1, const T *__restrict__ x, int d,
              int r, int B, int rpc, float *__restrict__ h, uint32_t *__restrict__ mask_words,
              int n_words) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T *xs = reinterpret_cast<T *>(smem_raw);
  constexpr int V = Vec<T>::N;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row0 = blockIdx.x * rpc;
  const int row1 = min(r, row0 + rpc);
  const int nvec = d / V;
  // One row per warp and one token group: the warp's W1 row goes into
  // registers before the wait.  This grid becomes resident as the previous
  // layer's sparse FFN starts, while that kernel ranks its list and HBM is
  // idle; a row (8 KB at d = 4096) fits that window.  (Prefetching more --
  // this layer's W2 as well, or half of a longer row -- delayed the FFN's row
  // stream and measured slower.)  The next kernel reads only weights before
  // it waits on this one.
  const bool early = U * kWarp >= nvec && row1 - row0 <= kWarps && B <= NB;
  const int erow = row0 + warp;
  uint4 wpre[U];
  float bias_pre = 0.f;
  if (early) {
    if (erow < row1) bias_pre = __ldg(b1 + erow);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = lane + u * kWarp;
      wpre[u] = (erow < row1 && c < nvec) ? ld_stream_early(W1 + (size_t)erow * d + (size_t)c * V)
                                          : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  pdl_trigger();
  pdl_wait();
  for (int w = blockIdx.x * kThreads + threadIdx.x; w < n_words; w += gridDim.x * kThreads)
    mask_words[w] = 0u;
  if (early) {
    stage_tokens<T, NB>(xs, x, d, 0, B);
    __syncthreads();
    if (erow < row1) {
      float acc[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] = 0.f;
      const float bias = bias_pre;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = lane + u * kWarp;
        if (c < nvec) {
#pragma unroll
          for (int b = 0; b < NB; ++b)
            acc[b] = Vec<T>::dot(wpre[u], *reinterpret_cast<const uint4 *>(xs + (size_t)b * d + (size_t)c * V),
                                 acc[b]);
        }
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float sum = warp_sum(acc[b]);
        if (lane == b && b < B) h[(size_t)b * r + erow] = fmaxf(sum + bias, 0.f);
      }
    }
    return;
  }
  for (int g0 = 0; g0 < B; g0 += NB) {
    const int nb = min(NB, B - g0);
    __syncthreads();
    stage_tokens<T, NB>(xs, x, d, g0, nb);
    __syncthreads();
    for (int row = row0 + warp; row < row1; row += kWarps) {
      float acc[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] = 0.f;
      const float bias = __ldg(b1 + row);     // in flight with the row's loads
      row_dot<T, NB, U>(W1 + (size_t)row * d, xs, d, nvec, lane, acc);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float s = warp_sum(acc[b]);
        if (lane == b && b < nb) h[(size_t)(g0 + b) * r + row] = fmaxf(s + bias, 0.f);
      }
    }
  }
}

// Layer 1 for rows too long to load into registers ahead of the wait (16 KB
// and more at d >= 8192, fp16): the CTA's whole W1 slice goes to shared memory
// in one bulk copy per row, issued at entry, before griddepcontrol.wait.  The
// kernel then needs as much shared memory as the previous layer's sparse FFN
// leaves free only once that kernel's CTAs exit, so its copies overlap the
// FFN's tail and the reduction of its partials instead of following them.
// After the wait it stages x one token group of NB at a time (the slice stays
// in shared memory: W1 is read from HBM once for any batch) and waits for
// each row's copy (bounded).  Two warps share a row, one half of d each (one
// warp per row left the dot products latency-bound at 7 warps per SM); the
// halves are added in order, then the bias.
constexpr int kPred1SmemRows = 16;    // most W1 rows one CTA stages
constexpr int kPred1Warps = 16;       // 2 per row, 8 rows at a time
template <typename T, int NB>
__global__ void __launch_bounds__(kPred1Warps * kWarp)
    k_pred_l1_smem(const T *__restrict__ W1, const float *__restrict__ b1, const T *__restrict__ x, int d,
                   int r, int B, int rpc, float *__restrict__ h, uint32_t *__restrict__ mask_words, int n_words,
                   int32_t *__restrict__ err) {
  extern __shared__ __align__(128) unsigned char smem_p1[];
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem_p1);
  T *ws = reinterpret_cast<T *>(smem_p1 + kPred1SmemRows * 8);
  T *xs = ws + (size_t)rpc * d;
  __shared__ int s_fail;
  __shared__ float sbias[kPred1SmemRows];
  __shared__ float shalf[kPred1SmemRows][2][NB];
  constexpr int V = Vec<T>::N;
  constexpr int NT = kPred1Warps * kWarp;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = warp & 1;
  const int row0 = blockIdx.x * rpc;
  const int nrows = max(0, min(r, row0 + rpc) - row0);
  const int nvec = d / V;
  const int hv = (nvec + 1) / 2;               // 16-byte chunks of the first half
  const int c_lo = half ? hv : 0, c_hi = half ? nvec : hv;
  const uint32_t row_bytes = (uint32_t)((size_t)d * sizeof(T));
  // the next kernel reads only weights before it waits on this one: let it
  // become resident at once (its launch waits for every CTA's trigger)
  pdl_trigger();
  if (threadIdx.x == 0) {
    s_fail = 0;
    for (int i = 0; i < nrows; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
    const uint64_t pol = l2_evict_first();
    for (int i = 0; i < nrows; ++i) {
      mbar_arrive_expect_tx(&bar[i], row_bytes);
      bulk_g2s_stream(ws + (size_t)i * d, W1 + (size_t)(row0 + i) * d, row_bytes, &bar[i], pol);
    }
  }
  // the biases are weights too: loaded before the wait, stored after it
  const float bias = threadIdx.x < nrows ? __ldg(b1 + row0 + threadIdx.x) : 0.f;
  pdl_wait();
  if (threadIdx.x < nrows) sbias[threadIdx.x] = bias;
  for (int w = blockIdx.x * NT + threadIdx.x; w < n_words; w += gridDim.x * NT) mask_words[w] = 0u;
  bool ok = true;
  for (int g0 = 0; g0 < B; g0 += NB) {
    const int nb = min(NB, B - g0);
    __syncthreads();      // also publishes the barrier initialisation and biases (first group)
    stage_tokens<T, NB>(xs, x, d, g0, nb);
    __syncthreads();
    for (int i = warp >> 1; i < nrows; i += kPred1Warps / 2) {
      if (g0 == 0 && ok && !mbar_wait(&bar[i], 0u, kWaitNs)) {
        if (lane == 0) flag_error(err, kErrTimeout);
        ok = false;
        s_fail = 1;
      }
      // two accumulators per token: alternate chunks' products in separate chains
      float acc[2][NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[0][b] = acc[1][b] = 0.f;
      if (ok) {
        const T *wr = ws + (size_t)i * d;
        for (int c0 = c_lo + lane; c0 < c_hi; c0 += 2 * kWarp) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = c0 + e * kWarp;
            if (c < c_hi) {
              const uint4 wv = *reinterpret_cast<const uint4 *>(wr + (size_t)c * V);
#pragma unroll
              for (int b = 0; b < NB; ++b)
                acc[e][b] = Vec<T>::dot(wv, *reinterpret_cast<const uint4 *>(xs + (size_t)b * d + (size_t)c * V),
                                        acc[e][b]);
            }
          }
        }
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float sum = warp_sum(acc[0][b] + acc[1][b]);
        if (lane == b) shalf[i][half][b] = sum;
      }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < nrows * nb; t += NT) {
      const int i = t / nb, b = t - i * nb;
      h[(size_t)(g0 + b) * r + row0 + i] = fmaxf(shalf[i][0][b] + shalf[i][1][b] + sbias[i], 0.f);
    }
  }
  // a copy whose wait gave up may still be in flight: let it land (bounded)
  // before the CTA's shared memory is released
  __syncthreads();
  if (s_fail && threadIdx.x == 0)
    for (int i = 0; i < nrows; ++i) mbar_wait(&bar[i], 0u, kWaitNs);
}

// Stage h[g0..g0+nb) ([B][r] fp32) for dot products with rows of T.  For fp16
// rows (8 elements per 16-byte chunk) the 8 floats of chunk c are split into
// two planes of 4 so that a warp's shared-memory reads are conflict-free.
template <typename T, int NB>
__device__ __forceinline__ void stage_hidden(float *hs, const float *__restrict__ h, int r, int g0, int nb) {
  for (int i = threadIdx.x; i < NB * r; i += blockDim.x) {
    const int b = i / r;
    const int e = i - b * r;
    const float v = (b < nb) ? __ldcg(h + (size_t)(g0 + b) * r + e) : 0.f;
    int pos = e;
    if (sizeof(T) == 2) {
      const int c = e >> 3, q = e & 7;
      pos = (q < 4) ? (c * 4 + q) : (r / 2 + c * 4 + (q - 4));
    }
    hs[(size_t)b * r + pos] = v;
  }
}

template <typename T>
__device__ __forceinline__ float dot_hidden(uint4 w, const float *hsb, int r, int c) {
  if constexpr (sizeof(T) == 2) {
    return Vec<__half>::dotf2(w, hsb + c * 4, hsb + r / 2 + c * 4, 0.f);
  } else {
    return Vec<float>::dotf(w, hsb + c * 4, 0.f);
  }
}

// Layer 2 + threshold + union + compaction.  CTA c owns rows [c*rpc, ...);
// each warp computes R rows at a time.  Bits of rows predicted active for any
// token are OR-ed into the global union mask; the last CTA to finish (atomic
// ticket, no waiting) turns the mask into the ascending index list.
template <typename T, int NB, int R, int UC>
__global__ void __launch_bounds__(kThreads)
    k_pred_l2(const T *__restrict__ W2, const float *__restrict__ b2, const float *__restrict__ h,
              int r, int n, int B, float thr, int rpc, uint32_t *__restrict__ mask_words, int n_words,
              int32_t *__restrict__ idx, int32_t *__restrict__ count, Header *__restrict__ hdr,
              int prefetch) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float *hs = reinterpret_cast<float *>(smem_raw);
  uint32_t *smask = reinterpret_cast<uint32_t *>(hs + (size_t)NB * r);
  __shared__ int s_last;
  __shared__ int s_wsum[kWarps];
  constexpr int V = Vec<T>::N;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row0 = blockIdx.x * rpc;
  const int row1 = min(n, row0 + rpc);
  if (prefetch && row0 < row1) prefetch_range(W2 + (size_t)row0 * r, (size_t)(row1 - row0) * r * sizeof(T));
  const int wfirst = row0 >> 5;
  const int nwl = (row0 < row1) ? (((row1 - 1) >> 5) - wfirst + 1) : 0;
  for (int i = threadIdx.x; i < nwl; i += kThreads) smask[i] = 0u;
  pdl_trigger();
  pdl_wait();
  const int nvec = r / V;
  for (int g0 = 0; g0 < B; g0 += NB) {
    const int nb = min(NB, B - g0);
    __syncthreads();
    stage_hidden<T, NB>(hs, h, r, g0, nb);
    __syncthreads();
    for (int rb = row0 + warp * R; rb < row1; rb += kWarps * R) {
      float acc[R][NB];
      float bq[R];     // in flight with the rows' loads
#pragma unroll
      for (int q = 0; q < R; ++q) {
        bq[q] = (rb + q < row1) ? __ldg(b2 + rb + q) : 0.f;
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[q][b] = 0.f;
      }
      for (int c0 = lane; c0 < nvec; c0 += UC * kWarp) {
        uint4 wv[R][UC];
#pragma unroll
        for (int q = 0; q < R; ++q) {
          const int row = min(rb + q, row1 - 1);
#pragma unroll
          for (int u = 0; u < UC; ++u) {
            const int c = c0 + u * kWarp;
            wv[q][u] = c < nvec ? ld_stream(W2 + (size_t)row * r + (size_t)c * V) : make_uint4(0u, 0u, 0u, 0u);
          }
        }
#pragma unroll
        for (int u = 0; u < UC; ++u) {
          const int c = c0 + u * kWarp;
          if (c < nvec) {
#pragma unroll
            for (int q = 0; q < R; ++q)
#pragma unroll
              for (int b = 0; b < NB; ++b) acc[q][b] += dot_hidden<T>(wv[q][u], hs + (size_t)b * r, r, c);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < R; ++q) {
        const int row = rb + q;
        bool on = false;
        const float bias = bq[q];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float z = warp_sum(acc[q][b]) + bias;
          on |= (b < nb) && (z > thr);
        }
        if (lane == 0 && on && row < row1) atomicOr(&smask[(row >> 5) - wfirst], 1u << (row & 31));
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nwl; i += kThreads)
    if (smask[i]) atomicOr(&mask_words[wfirst + i], smask[i]);
  __syncthreads();
  if (threadIdx.x == 0) s_last = (ticket_acq_rel(&hdr->done) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  // ---- compaction by the last CTA: block-wide exclusive scan of popcounts ----
  const int wpt = (n_words + kThreads - 1) / kThreads;
  const int wbeg = min(n_words, threadIdx.x * wpt);
  const int wend = min(n_words, wbeg + wpt);
  int local = 0;
  for (int w = wbeg; w < wend; ++w) local += __popc(ld_cg_u32(mask_words + w));
  int incl = local;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == kWarp - 1) s_wsum[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += s_wsum[w];
  int off = before + incl - local;
  for (int w = wbeg; w < wend; ++w) {
    uint32_t m = ld_cg_u32(mask_words + w);
    while (m) {
      const int bit = __ffs(m) - 1;
      idx[off++] = w * 32 + bit;
      m &= m - 1u;
    }
  }
  if (threadIdx.x == kThreads - 1) {
    *count = off;
    hdr->done = 0u;
  }
}

// ======================================================================== //
// predictor GEMVs fed by a bulk-copy ring                                  //
// ======================================================================== //

// Shared-memory layout of the ring GEMVs: NSL slots of CR rows of K elements,
// plus the staged activation vector(s).
struct RingLayout {
  size_t full, empty, vec, ring, total;
};
__host__ __device__ inline RingLayout ring_layout(int NSL, int CR, int K, int esz, size_t vec_bytes) {
  RingLayout L;
  size_t o = 0;
  L.full = o;  o += (size_t)NSL * 8;
  L.empty = o; o += (size_t)NSL * 8;
  o = align_up(o, 128);
  L.vec = o;   o += vec_bytes;
  o = align_up(o, 128);
  L.ring = o;  o += (size_t)NSL * CR * K * esz;
  L.total = o;
  return L;
}

constexpr int kRingWarps = 8;   // consumer warps; warp 8 is the producer

// Issue the bulk copy of chunk i of this CTA's contiguous row slice.
template <typename T>
__device__ __forceinline__ void ring_issue(const T *W, int K, int row0, int row1, int CR, int NSL, int i,
                                           T *ring, uint64_t *full) {
  const int s = i % NSL;
  const int ra = row0 + i * CR;
  const int rb = min(row1, ra + CR);
  const uint32_t bytes = (uint32_t)((size_t)(rb - ra) * K * sizeof(T));
  mbar_arrive_expect_tx(&full[s], bytes);
  bulk_g2s_stream(ring + (size_t)s * CR * K, W + (size_t)ra * K, bytes, &full[s], l2_evict_first());
}

// Producer loop for chunks [first, nch): waits for slot release, then issues.
template <typename T>
__device__ __forceinline__ bool ring_produce(const T *W, int K, int row0, int row1, int CR, int NSL, int first,
                                             int nch, T *ring, uint64_t *full, uint64_t *empty) {
  for (int i = first; i < nch; ++i) {
    const int s = i % NSL;
    if (i >= NSL && !mbar_wait(&empty[s], (uint32_t)((i / NSL) - 1) & 1u, kWaitNs)) return false;
    ring_issue(W, K, row0, row1, CR, NSL, i, ring, full);
  }
  return true;
}

// Shared bytes of k_pred2_ring besides the ring: staged h [NB][r], the CTA's
// mask words, and its b2 values.
__host__ __device__ inline size_t pred2_vec_bytes(int NB, int r, int rpc) {
  return (size_t)NB * r * 4 + (size_t)(rpc / 32 + 2) * 4 + (size_t)rpc * 4;
}

// Layer 2 + threshold + union over tokens, B <= NB tokens, with W2 rows fed by
// the bulk-copy ring (its first chunk issued before the wait).  Each CTA ORs the
// bits of its rows into the union mask; the next kernel compacts it.
template <typename T, int NB>
__global__ void __launch_bounds__((kRingWarps + 1) * kWarp, 1)
    k_pred2_ring(const T *__restrict__ W2, const float *__restrict__ b2, const float *__restrict__ h, int r, int n,
                 int B, float thr, int rpc, int CR, int NSL, uint32_t *__restrict__ mask_words,
                 Header *__restrict__ hdr, HotBlock hot) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int V = Vec<T>::N;
  constexpr int NT = (kRingWarps + 1) * kWarp;
  const int nwl_max = rpc / 32 + 2;
  const RingLayout L = ring_layout(NSL, CR, r, (int)sizeof(T), pred2_vec_bytes(NB, r, rpc));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.full);
  uint64_t *empty = reinterpret_cast<uint64_t *>(smem + L.empty);
  float *hs = reinterpret_cast<float *>(smem + L.vec);
  uint32_t *smask = reinterpret_cast<uint32_t *>(smem + L.vec + (size_t)NB * r * 4);
  float *sb = reinterpret_cast<float *>(smask + nwl_max);     // b2 of this CTA's rows
  T *ring = reinterpret_cast<T *>(smem + L.ring);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * rpc, row1 = min(n, row0 + rpc);
  const int nch = row0 < row1 ? (row1 - row0 + CR - 1) / CR : 0;
  const int wfirst = row0 >> 5;
  const int nwl = (row0 < row1) ? (((row1 - 1) >> 5) - wfirst + 1) : 0;
  if (threadIdx.x == 0) {
    for (int q = 0; q < NSL; ++q) {
      mbar_init(&full[q], 1);
      mbar_init(&empty[q], kRingWarps);
    }
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < nwl; i += NT) smask[i] = 0u;
  __syncthreads();
  // One chunk is copied before the wait, so that the first rows are resident
  // when h arrives; the others are issued after it.  Copies issued here share
  // HBM with the previous kernels' tails and layer 1's weights, which are on
  // the critical path: filling the whole ring before the wait measured 1.9%
  // slower at the Llama2-7B shape (layer 1 loading its rows into registers)
  // and the same elsewhere.
  const int pre = min(nch, 1);
  if (warp == kRingWarps && lane == 0) {
    for (int i = 0; i < pre; ++i) ring_issue(W2, r, row0, row1, CR, NSL, i, ring, full);
  }

  // biases are weights too: fetched before the wait, read from shared memory
  // (the consumers' named barrier below orders these stores)
  if (warp < kRingWarps)
    for (int i = threadIdx.x; i < row1 - row0; i += kRingWarps * kWarp) sb[i] = __ldg(b2 + row0 + i);
  pdl_trigger();
  pdl_wait();
  if (warp == kRingWarps) {
    if (lane == 0 && !ring_produce(W2, r, row0, row1, CR, NSL, pre, nch, ring, full, empty))
      flag_error(&hdr->err, kErrTimeout);
    // Every W2 copy of this CTA is queued: the FFN rows of the hot block
    // (active for most tokens) now go to L2, in the window where HBM idles
    // between this kernel's last copies and the sparse FFN's first, which
    // then gathers its active hot rows from L2.  (Issued at this kernel's
    // start instead, the prefetch competed with the W2 stream and measured
    // slower.)
    __syncwarp();
    prefetch_hot(hot, blockIdx.x, gridDim.x);
  } else {
    {
      // 4 consecutive floats of h land together in one plane (r % 8 == 0 for
      // fp16, r % 4 == 0 for fp32), so the copy is 16-byte vectors; every
      // thread issues all its loads before storing
      constexpr int MAXU = 8;
      const int n4 = NB * r / 4;
      const int nt = kRingWarps * kWarp;
      float4 v[MAXU];
#pragma unroll
      for (int u = 0; u < MAXU; ++u) {
        const int i = threadIdx.x + u * nt;
        const int b = (i * 4) / r;
        v[u] = (i < n4 && b < B) ? __ldcg(reinterpret_cast<const float4 *>(h) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      auto place = [&](int i, float4 val) {
        const int b = (i * 4) / r, e = i * 4 - b * r;
        int pos = e;
        if (sizeof(T) == 2) {
          const int c = e >> 3, q = e & 7;
          pos = (q < 4) ? (c * 4) : (r / 2 + c * 4);
        }
        *reinterpret_cast<float4 *>(hs + (size_t)b * r + pos) = val;
      };
#pragma unroll
      for (int u = 0; u < MAXU; ++u) {
        const int i = threadIdx.x + u * nt;
        if (i < n4) place(i, v[u]);
      }
      for (int i = threadIdx.x + MAXU * nt; i < n4; i += nt) {
        const int b = (i * 4) / r;
        place(i, b < B ? __ldcg(reinterpret_cast<const float4 *>(h) + i) : make_float4(0.f, 0.f, 0.f, 0.f));
      }
    }
    named_sync(1, kRingWarps * kWarp);
    const int nvec = r / V;
    // A lane meets the same chunks of h in every row: keep them in registers
    // when they fit (up to HQ chunks per lane, at most 2 tokens).
    constexpr int HQ = 4;
    constexpr bool kRegH = NB <= 2;
    const bool reg_h = kRegH && nvec <= HQ * kWarp;
    float hreg[kRegH ? NB : 1][HQ][V];
    if (reg_h) {
#pragma unroll
      for (int b = 0; b < (kRegH ? NB : 1); ++b)
#pragma unroll
        for (int u = 0; u < HQ; ++u) {
          const int c = lane + u * kWarp;
#pragma unroll
          for (int e = 0; e < V; ++e) {
            float v = 0.f;
            if (c < nvec) {
              if constexpr (sizeof(T) == 2)
                v = hs[(size_t)b * r + (e < 4 ? c * 4 + e : r / 2 + c * 4 + (e - 4))];
              else
                v = hs[(size_t)b * r + c * 4 + e];
            }
            hreg[b][u][e] = v;
          }
        }
    }
    bool ok = true;
    for (int i = 0; i < nch; ++i) {
      const int sl = i % NSL;
      if (ok && !mbar_wait(&full[sl], (uint32_t)(i / NSL) & 1u, kWaitNs)) {
        if (lane == 0) flag_error(&hdr->err, kErrTimeout);
        ok = false;
      }
      const int ra = row0 + i * CR, rb = min(row1, ra + CR);
      // two rows per pass (row and row + kRingWarps): their dot products and
      // warp reductions are independent chains that overlap
      for (int row = ra + warp; row < rb && ok; row += 2 * kRingWarps) {
        const bool two = row + kRingWarps < rb;
        const T *wr = ring + ((size_t)sl * CR + (row - ra)) * r;
        const T *wr2 = wr + (size_t)kRingWarps * r;
        float acc[2][NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[0][b] = acc[1][b] = 0.f;
        if (reg_h) {
#pragma unroll
          for (int u = 0; u < HQ; ++u) {
            const int c = lane + u * kWarp;
            if (c < nvec) {
              const uint4 wv = *reinterpret_cast<const uint4 *>(wr + (size_t)c * V);
              const uint4 wv2 = two ? *reinterpret_cast<const uint4 *>(wr2 + (size_t)c * V) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
              for (int b = 0; b < (kRegH ? NB : 1); ++b) {
                acc[0][b] = Vec<T>::dotr(wv, hreg[b][u], acc[0][b]);
                acc[1][b] = Vec<T>::dotr(wv2, hreg[b][u], acc[1][b]);
              }
            }
          }
        } else {
          for (int c = lane; c < nvec; c += kWarp) {
            const uint4 wv = *reinterpret_cast<const uint4 *>(wr + (size_t)c * V);
            const uint4 wv2 = two ? *reinterpret_cast<const uint4 *>(wr2 + (size_t)c * V) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              acc[0][b] += dot_hidden<T>(wv, hs + (size_t)b * r, r, c);
              acc[1][b] += dot_hidden<T>(wv2, hs + (size_t)b * r, r, c);
            }
          }
        }
        bool on = false, on2 = false;
        const float bias = sb[row - row0];
        const float bias2 = two ? sb[row + kRingWarps - row0] : 0.f;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float z = warp_sum(acc[0][b]) + bias;
          const float z2 = warp_sum(acc[1][b]) + bias2;
          on |= (b < B) && (z > thr);
          on2 |= two && (b < B) && (z2 > thr);
        }
        if (lane == 0 && on) atomicOr(&smask[(row >> 5) - wfirst], 1u << (row & 31));
        if (lane == 0 && on2) {
          const int row2 = row + kRingWarps;
          atomicOr(&smask[(row2 >> 5) - wfirst], 1u << (row2 & 31));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[sl]);
    }
  }
  // publish this CTA's union bits (words at the slice edges are shared with
  // the neighbouring CTAs, hence the atomic OR); k_compact builds the list
  __syncthreads();
  for (int i = threadIdx.x; i < nwl; i += NT)
    if (smask[i]) atomicOr(&mask_words[wfirst + i], smask[i]);
}

// Ascending compaction of the union mask: one CTA reads every mask word,
// scans the popcounts and writes the index list and its length.  A kernel
// boundary is the cheapest grid-wide handoff on B200, so the scan runs as its
// own small kernel right after the mask is complete.
constexpr int kCompactThreads = 1024;
constexpr int kCompactWords = 8;    // words per thread: n <= 1024 * 8 * 32
__global__ void __launch_bounds__(kCompactThreads)
    k_compact(const uint32_t *__restrict__ mask_words, int n_words, int32_t *__restrict__ idx,
              int32_t *__restrict__ count) {
  __shared__ int s_wsum[kCompactThreads / kWarp];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wpt = (n_words + kCompactThreads - 1) / kCompactThreads;
  const int wbeg = min(n_words, (int)threadIdx.x * wpt);
  const int wend = min(n_words, wbeg + wpt);
  uint32_t wv[kCompactWords];
  int local = 0;
#pragma unroll
  for (int q = 0; q < kCompactWords; ++q) {
    wv[q] = (wbeg + q < wend) ? ld_cg_u32(mask_words + wbeg + q) : 0u;
    local += __popc(wv[q]);
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == kWarp - 1) s_wsum[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += s_wsum[w];
  int off = before + incl - local;
#pragma unroll
  for (int q = 0; q < kCompactWords; ++q) {
    uint32_t m = wv[q];
    while (m) {
      const int bit = __ffs(m) - 1;
      idx[off++] = (wbeg + q) * 32 + bit;
      m &= m - 1u;
    }
  }
  if (threadIdx.x == kCompactThreads - 1) *count = off;
}

// ======================================================================== //
// sparse FFN                                                               //
// ======================================================================== //

// Gate/up gather-GEMV and activation.  Warp w of the grid handles list
// positions j = w, w + W, ...; for neuron k = idx[j] it streams the whole
// gate and up rows once and writes a[j][b] for every token b.
template <typename T, int NB, int U, bool REGLU>
__global__ void __launch_bounds__(kThreads)
    k_ffn_gu(const T *__restrict__ Wg, const T *__restrict__ Wu, const float *__restrict__ bias,
             const T *__restrict__ x, int d, long long rs, int n, int B, const int32_t *__restrict__ idx,
             const int32_t *__restrict__ count, float *__restrict__ a, int32_t *__restrict__ err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T *xs = reinterpret_cast<T *>(smem_raw);
  constexpr int V = Vec<T>::N;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  int cnt = n;
  if (idx) {
    const int c = ld_cg_i32(count);
    if (c < 0 || c > n) {
      if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, kErrIndex);
      cnt = max(0, min(c, n));
    } else {
      cnt = c;
    }
  }
  const int nvec = d / V;
  const int wtot = gridDim.x * kWarps;
  const int gw = blockIdx.x * kWarps + warp;
  for (int g0 = 0; g0 < B; g0 += NB) {
    const int nb = min(NB, B - g0);
    __syncthreads();
    stage_tokens<T, NB>(xs, x, d, g0, nb);
    __syncthreads();
    for (int j = gw; j < cnt; j += wtot) {
      const int k = idx ? ld_cg_i32(idx + j) : j;
      float out[NB];
      if ((unsigned)k >= (unsigned)n) {
        if (lane == 0 && g0 == 0) flag_error(err, kErrIndex);
#pragma unroll
        for (int b = 0; b < NB; ++b) out[b] = 0.f;
      } else {
        const float bk = __ldg(bias + k);
        if constexpr (REGLU) {
          float ag[NB], au[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b) ag[b] = au[b] = 0.f;
          row_dot2<T, NB, U>(Wg + (size_t)k * rs, Wu + (size_t)k * rs, xs, d, nvec, lane, ag, au);
#pragma unroll
          for (int b = 0; b < NB; ++b) out[b] = fmaxf(warp_sum(ag[b]) + bk, 0.f) * warp_sum(au[b]);
        } else {
          float au[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b) au[b] = 0.f;
          row_dot<T, NB, 2 * U>(Wu + (size_t)k * rs, xs, d, nvec, lane, au);
#pragma unroll
          for (int b = 0; b < NB; ++b) out[b] = fmaxf(warp_sum(au[b]) + bk, 0.f);
        }
      }
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (lane == b && b < nb) a[(size_t)j * B + g0 + b] = out[b];
    }
  }
}

// Down projection as a gather-accumulate over rows of W_down^T.  CTA (t, s)
// owns column tile t (TW = 32 lanes x one 16-byte chunk) and the s-th slice of
// the index list; warps split the slice, lanes own columns, so each weight row
// chunk is one coalesced 512-byte read.  Warp partials are summed in shared
// memory in warp order; split partials are summed in split order by the last
// CTA of the tile (atomic ticket) -- deterministic, no float atomics.
template <typename T, int NB, int UJ>
__global__ void __launch_bounds__(kThreads)
    k_ffn_down(const T *__restrict__ WdT, const float *__restrict__ a, const int32_t *__restrict__ idx,
               const int32_t *__restrict__ count, int d, long long rs, int n, int B, int S,
               float *__restrict__ part, float *__restrict__ y, Header *__restrict__ hdr,
               int prefetch, L2Next nx) {
  constexpr int V = Vec<T>::N;
  constexpr int TW = kWarp * V;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float *red = reinterpret_cast<float *>(smem_raw);  // [kWarps][NB][TW]
  __shared__ int s_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tile = blockIdx.x, split = blockIdx.y;
  const int col0 = tile * TW;
  const int col = col0 + lane * V;
  const bool col_ok = col < d;
  // The index list was completed two kernels earlier (the gate/up kernel
  // waited for it before letting this grid start), so it can be read before
  // waiting for the activations.
  int cnt = n;
  if (idx) cnt = max(0, min(ld_cg_i32(count), n));
  const int js = (int)(((long long)cnt * split) / S);
  const int je = (int)(((long long)cnt * (split + 1)) / S);
  if (prefetch) {
    const uint32_t bytes = (uint32_t)(min(TW, d - col0) * sizeof(T));
    for (int j = js + threadIdx.x; j < je; j += kThreads) {
      const int k = idx ? ld_cg_i32(idx + j) : j;
      if ((unsigned)k < (unsigned)n) prefetch_l2(WdT + (size_t)k * rs + col0, bytes);
    }
  }
  if (warp == kWarps - 1) prefetch_next(nx, blockIdx.y * gridDim.x + blockIdx.x, gridDim.x * gridDim.y);
  pdl_wait();
  pdl_trigger();
  for (int g0 = 0; g0 < B; g0 += NB) {
    const int nb = min(NB, B - g0);
    float acc[V][NB];
#pragma unroll
    for (int e = 0; e < V; ++e)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[e][b] = 0.f;
    for (int j = js + warp * UJ; j < je; j += kWarps * UJ) {
      uint4 wv[UJ];
      float av[UJ][NB];
#pragma unroll
      for (int u = 0; u < UJ; ++u) {
        const int jj = j + u;
        int k = -1;
        if (jj < je) k = idx ? ld_cg_i32(idx + jj) : jj;
        const bool ok = (unsigned)k < (unsigned)n;
        wv[u] = (ok && col_ok) ? ld_stream(WdT + (size_t)k * rs + col) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int b = 0; b < NB; ++b)
          av[u][b] = (ok && b < nb) ? ld_cg_f32(a + (size_t)jj * B + g0 + b) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < UJ; ++u) {
        float f[V];
        Vec<T>::to_float(wv[u], f);
#pragma unroll
        for (int e = 0; e < V; ++e)
#pragma unroll
          for (int b = 0; b < NB; ++b) acc[e][b] = fmaf(av[u][b], f[e], acc[e][b]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < V; ++e) red[((size_t)warp * NB + b) * TW + lane * V + e] = acc[e][b];
    __syncthreads();
    for (int i = threadIdx.x; i < NB * TW; i += kThreads) {
      const int b = i / TW, c = i - b * TW;
      if (b < nb && col0 + c < d) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[((size_t)w * NB + b) * TW + c];
        if (S == 1)
          y[(size_t)(g0 + b) * d + col0 + c] = s;
        else
          part[((size_t)split * B + g0 + b) * d + col0 + c] = s;
      }
    }
  }
  if (S == 1) return;
  __syncthreads();
  if (threadIdx.x == 0) s_last = (ticket_acq_rel(&hdr->tile_done[tile]) == (unsigned)S - 1u);
  __syncthreads();
  if (!s_last) return;
  const int tw = min(TW, d - col0);
  for (int i = threadIdx.x; i < B * tw; i += kThreads) {
    const int b = i / tw, c = i - b * tw;
    float s = 0.f;
    for (int q0 = 0; q0 < S; q0 += 16) {   // 16 loads in flight, summed in split order
      float v[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        v[q] = q0 + q < S ? ld_cg_f32(part + ((size_t)(q0 + q) * B + b) * d + col0 + c) : 0.f;
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (q0 + q < S) s += v[q];
    }
    y[(size_t)b * d + col0 + c] = s;
  }
  if (threadIdx.x == 0) hdr->tile_done[tile] = 0u;
}

// ======================================================================== //
// many tokens on the tensor cores (tcgen05)                                //
// ======================================================================== //

// For a batch of B > 4 tokens over the union list, gate/up is a small dense
// GEMM over gathered rows: [count x d] . [d x B].  On CUDA cores every weight
// byte then carries B fp32 FMAs, and past a few tokens the FP32 pipe, not
// HBM, bounds it (the CUDA-core kernel also re-streams the rows once per group
// of 8 tokens).  This kernel runs it on the 5th-generation tensor cores:
// producer warps gather the listed rows into shared memory with cp.async (16
// bytes per thread, any row order) directly in the 128-byte-swizzled layout
// tcgen05.mma reads, one thread issues the MMAs, and the fp32 accumulators
// live in tensor memory.  x and the weights are fp16 already, so the products
// are exact and accumulate in fp32, as on the CUDA cores.  The activations go
// to the down projection (k_ffn_down) as fp32.
constexpr int kTcRows = 128;   // neurons per gate/up MMA tile (M)
constexpr int kTcK = 64;       // fp16 elements of d per stage: one 128-byte swizzle row
constexpr int kTcChunk = 32;   // list positions per share unit (one epilogue warp's rows)
constexpr int kTcN = 16;       // tokens per MMA (N); larger batches run as several launches

__device__ __forceinline__ unsigned char *align1024(unsigned char *p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

// Stage = the gate and up tiles [128 rows][64] (16 KB each, 128-byte swizzle,
// K-major) and the x tile [NT][64] of the NT = 16 tokens this launch handles.
template <int NT, bool REGLU>
struct GuTc {
  static constexpr int W = kTcRows * kTcK * 2;
  static constexpr int X = NT * kTcK * 2;
  static constexpr int STAGE = (REGLU ? 2 : 1) * W + X;
  static constexpr int NS = REGLU ? 5 : 8;
  static constexpr int BAR = 1024;
  static constexpr size_t SMEM = 1024 + BAR + (size_t)NS * STAGE;
  static constexpr uint32_t COLS = (REGLU ? 4 : 2) * NT;   // gate and up accumulators, double-buffered
  static_assert(STAGE % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
};

// a[j][g0 + b] (fp32, rows of Btot) for list position j and token b < B of
// this launch's x (tokens g0.. of the batch).
//
// CTA c owns whole chunks [c*nch/G, (c+1)*nch/G) of the list.  Warps 4-7 gather
// (one row per thread per tile), warp 8 issues the MMAs (lane 0) and owns the
// tensor memory, warps 0-3 read the accumulators of a finished tile (lane =
// row), apply ReLU(g + b) * u (or ReLU(u + b)) and write a; two accumulator
// buffers let the epilogue of one tile overlap the MMAs of the next.
template <int NT, bool REGLU>
__global__ void __launch_bounds__(9 * kWarp, 1)
    k_gu_tc(const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_u,
            const __grid_constant__ CUtensorMap tm_x, int use_tma, const __half *__restrict__ Wg,
            const __half *__restrict__ Wu, const float *__restrict__ bias, const __half *__restrict__ x, int d,
            long long rs, int n, int B, const int32_t *__restrict__ idx, const int32_t *__restrict__ count,
            float *__restrict__ a, __half *__restrict__ a2, int Btot, int g0, Header *__restrict__ hdr) {
  using Lg = GuTc<NT, REGLU>;
  constexpr int NS = Lg::NS;
  constexpr int MATS = REGLU ? 2 : 1;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = align1024(smem_raw);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + NS;
  uint64_t *tfull = empty + NS;
  uint64_t *tempty = tfull + 2;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(tempty + 2);
  unsigned char *stages = smem + Lg::BAR;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t *err = &hdr->err;

  __shared__ int srow[REGLU ? kTcRows : 1];    // the current tile's rows (TMA producers)
  if (threadIdx.x == 0) {
    for (int q = 0; q < NS; ++q) {
      mbar_init(&full[q], (REGLU && use_tma) ? 4 : 4 * kWarp);   // one arrival per producer warp / thread
      mbar_init(&empty[q], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4 * kWarp);
    }
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tslot, Lg::COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  // the list comes from the previous kernel; only then may the down kernel start
  pdl_wait();
  pdl_trigger();

  int cnt = n;
  if (idx) {
    const int c = ld_cg_i32(count);
    if ((c < 0 || c > n) && blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, kErrIndex);
    cnt = max(0, min(c, n));
  }
  const int nch = (cnt + kTcChunk - 1) / kTcChunk;
  const int own0 = kTcChunk * (int)((long long)nch * blockIdx.x / gridDim.x);
  const int own1 = kTcChunk * (int)((long long)nch * (blockIdx.x + 1) / gridDim.x);
  const int ntiles = (own1 - own0 + kTcRows - 1) / kTcRows;
  const int nK = (d + kTcK - 1) / kTcK;
  const int total = ntiles * nK;

  if (warp >= 4 && warp < 8 && REGLU && use_tma) {
    // ------------------------------------------------ producers (gate + up) --
    // TMA: warp 4 + p takes the four-row groups p, p + 4, ... of the tile,
    // fetches their rows' indices, and its lane 0 issues, per stage, their
    // gate and up rows as tile::gather4 loads
    // (four rows of 64 columns per instruction; the maps' box is 64 columns x
    // 1 row in the 128-byte swizzle, so the rows land in the layout the MMA
    // reads), with warp 4 also loading x (a 2-D tile of 64 columns x 16
    // tokens); each warp arrives on the stage once with its own bytes.
    // Columns past d and tokens past B are outside the maps and read as
    // zeros; groups of four rows wholly past the list are skipped, and other
    // padding positions load row 0 (the epilogue writes zeros for them).
    // Four issuing warps measured 19% faster (70B shape, B = 16) than the
    // 16-byte cp.async gathers below, and one issuing thread 40% slower.
    const int p = warp - 4;
    const uint64_t pol = l2_evict_first();
    bool ok = true;
    int issued = 0;
    int ng = 0;                      // this warp's four-row groups that hold listed positions
    for (int it = 0; it < total && ok; ++it) {
      const int T = it / nK, kc = it - T * nK, sl = it % NS;
      if (kc == 0) {
        // groups wholly past the list are not loaded: their accumulator rows
        // are discarded by the epilogue, whatever the stage holds there
        const int nvalid = min(kTcRows, max(0, min(own1, cnt) - (own0 + T * kTcRows)));
        ng = min(8, max(0, ((nvalid + 3) / 4 - p + 3) / 4));    // groups p, p + 4, ... below nvalid
        __syncwarp();
        const int r = 4 * (p + 4 * (lane >> 2)) + (lane & 3);      // row 4g + e of group g = p + 4 (lane / 4)
        const int j = own0 + T * kTcRows + r;
        int k = 0;
        if (j < own1 && j < cnt) {
          const int kk = idx ? ld_cg_i32(idx + j) : j;
          if ((unsigned)kk < (unsigned)n) k = kk;
        }
        srow[r] = k;
        __syncwarp();
      }
      if (lane == 0) {
        if (it >= NS && !mbar_wait(&empty[sl], (uint32_t)((it / NS) - 1) & 1u, kWaitNs)) {
          flag_error(err, kErrTimeout);
          ok = false;
        } else {
          unsigned char *st = stages + (size_t)sl * Lg::STAGE;
          const int col0 = kc * kTcK;
          mbar_arrive_expect_tx(&full[sl], (uint32_t)(ng * 2 * 512 + (p == 0 ? NT * kTcK * 2 : 0)));
          for (int i = 0; i < ng; ++i) {
            const int g = p + 4 * i;
            tma_gather4(st + (size_t)g * 512, &tm_g, col0, srow[4 * g], srow[4 * g + 1], srow[4 * g + 2],
                        srow[4 * g + 3], &full[sl], pol);
            tma_gather4(st + (size_t)Lg::W + (size_t)g * 512, &tm_u, col0, srow[4 * g], srow[4 * g + 1],
                        srow[4 * g + 2], srow[4 * g + 3], &full[sl], pol);
          }
          if (p == 0) tma_load_2d(st + (size_t)2 * Lg::W, &tm_x, col0, 0, &full[sl]);
          issued = it + 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    // after a wait gave up, let each slot's last load land (bounded) before
    // the shared memory is released
    if (!ok && lane == 0)
      for (int e = max(0, issued - NS); e < issued; ++e) mbar_wait(&full[e % NS], (uint32_t)(e / NS) & 1u, kWaitNs);
  } else if (warp >= 4 && warp < 8) {
    // ---------------------------------------------------- producers (cp.async) --
    // 16 bytes per thread, one tile row per thread.  Used for ReLU (one matrix
    // per stage: the TMA gathers above measured 2% slower there) and for rows
    // of up to 8 KB (d = 4096: a CTA's tile holds fewer listed rows there, and
    // the TMA gathers measured 2-14% slower).
    const int t = threadIdx.x - 4 * kWarp;        // tile row of this thread
    const uint64_t pol = l2_evict_first();
    const __half *mats[2] = {REGLU ? Wg : Wu, Wu};
    int krow = -1;
    bool ok = true;
    for (int it = 0; it < total && ok; ++it) {
      const int T = it / nK, kc = it - T * nK, sl = it % NS;
      if (kc == 0) {
        const int j = own0 + T * kTcRows + t;
        krow = -1;
        if (j < own1 && j < cnt) {
          const int k = idx ? ld_cg_i32(idx + j) : j;
          if ((unsigned)k < (unsigned)n) krow = k;
        }
      }
      if (it >= NS && !mbar_wait(&empty[sl], (uint32_t)((it / NS) - 1) & 1u, kWaitNs)) {
        flag_error(err, kErrTimeout);
        ok = false;
        break;
      }
      unsigned char *st = stages + (size_t)sl * Lg::STAGE;
      const int col0 = kc * kTcK;
#pragma unroll
      for (int m = 0; m < MATS; ++m) {
        const __half *rowp = mats[m] + (size_t)max(krow, 0) * rs + col0;
        unsigned char *dt = st + (size_t)m * Lg::W + (size_t)t * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const bool in = krow >= 0 && col0 + c * 8 < d;
          cp_async16(dt + ((c ^ (t & 7)) << 4), in ? (const void *)(rowp + c * 8) : (const void *)mats[m],
                     in ? 16u : 0u, pol);
        }
      }
      unsigned char *xt = st + (size_t)MATS * Lg::W;
      for (int q = t; q < NT * 8; q += 4 * kWarp) {
        const int b = q >> 3, c = q & 7;
        const bool in = b < B && col0 + c * 8 < d;
        cp_async16(xt + b * 128 + ((c ^ (b & 7)) << 4),
                   in ? (const void *)(x + (size_t)b * d + col0 + c * 8) : (const void *)x, in ? 16u : 0u);
      }
      cp_async_commit();
      if (it >= NS - 1) {
        cp_async_wait<NS - 1>();
        fence_proxy_async_smem();
        mbar_arrive(&full[(it - (NS - 1)) % NS]);
      }
    }
    // every copy lands before the stages are released or the CTA exits
    cp_async_wait<0>();
    fence_proxy_async_smem();
    if (ok)
      for (int it = max(0, total - (NS - 1)); it < total; ++it) mbar_arrive(&full[it % NS]);
  } else if (warp == 8) {
    // ------------------------------------------------------------------ MMA --
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_f16(kTcRows, NT, 0, 0);
      bool ok = true;
      for (int T = 0; T < ntiles && ok; ++T) {
        const int buf = T & 1;
        if (T >= 2 && !mbar_wait(&tempty[buf], (uint32_t)((T >> 1) - 1) & 1u, kWaitNs)) {
          flag_error(err, kErrTimeout);
          break;
        }
        tc_fence_after();
        const uint32_t du = tbase + (uint32_t)(buf * MATS * NT);
        const uint32_t dg = du + (REGLU ? NT : 0);
        for (int kc = 0; kc < nK; ++kc) {
          const int it = T * nK + kc, sl = it % NS;
          if (!mbar_wait(&full[sl], (uint32_t)(it / NS) & 1u, kWaitNs)) {
            flag_error(err, kErrTimeout);
            ok = false;
            break;
          }
          tc_fence_after();
          unsigned char *st = stages + (size_t)sl * Lg::STAGE;
          const uint64_t dx = umma_desc(st + (size_t)MATS * Lg::W, 16, 1024, kSwz128);
          const uint64_t dwa = umma_desc(st, 16, 1024, kSwz128);
          const uint64_t dwb = umma_desc(st + (REGLU ? Lg::W : 0), 16, 1024, kSwz128);
#pragma unroll
          for (int k4 = 0; k4 < kTcK / 16; ++k4) {
            const uint32_t acc = (kc | k4) != 0;
            if (REGLU) umma_f16(dg, dwa + 2 * k4, dx + 2 * k4, idesc, acc);
            umma_f16(du, dwb + 2 * k4, dx + 2 * k4, idesc, acc);
          }
          umma_commit(&empty[sl]);
        }
        if (ok) umma_commit(&tfull[buf]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue --
    const int r = threadIdx.x;                    // tile row = tensor-memory lane
    const uint32_t lane_addr = tbase + ((uint32_t)(kWarp * warp) << 16);
    for (int T = 0; T < ntiles; ++T) {
      const int buf = T & 1;
      const int j = own0 + T * kTcRows + r;
      const bool owned = j < own1;                // uniform over the warp: 32 rows = one chunk
      int k = -1;
      float bk = 0.f;
      if (owned && j < cnt) {
        k = idx ? ld_cg_i32(idx + j) : j;
        if ((unsigned)k >= (unsigned)n) {
          flag_error(err, kErrIndex);
          k = -1;
        } else {
          bk = __ldg(bias + k);
        }
      }
      const bool got = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], (uint32_t)(T >> 1) & 1u, kWaitNs));
      if (!got && lane == 0) flag_error(err, kErrTimeout);
      tc_fence_after();
      __syncwarp();          // tensor-memory loads below are warp-synchronous
      float u[NT], g[NT];
      if (got) {
        const uint32_t cu = lane_addr + (uint32_t)(buf * MATS * NT);
#pragma unroll
        for (int h = 0; h < NT / 16; ++h) {
          float v[16];
          tmem_ld16(cu + 16 * h, v);
#pragma unroll
          for (int e = 0; e < 16; ++e) u[16 * h + e] = v[e];
          if (REGLU) {
            tmem_ld16(cu + NT + 16 * h, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) g[16 * h + e] = v[e];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
      if (!owned) continue;
      if (a2) {
        // the down kernel's operand: for chunk q of 32 positions and token
        // group gg of 8, rows 0-7 hold fp16(a) of the group's tokens and rows
        // 8-15 fp16(a - fp16(a)); positions past the list and padding tokens
        // are zero (the down kernel reads whole chunks and groups)
        const int q = j / kTcChunk, ngt = (Btot + 7) / 8;
#pragma unroll
        for (int b = 0; b < NT; ++b) {
          const int t = g0 + b;
          if (t >= 8 * ngt) break;
          float v = 0.f;
          if (got && k >= 0 && j < cnt && b < B) v = REGLU ? fmaxf(g[b] + bk, 0.f) * u[b] : fmaxf(u[b] + bk, 0.f);
          const __half hi = __float2half_rn(v);
          const __half lo = __float2half_rn(v - __half2float(hi));
          __half *dst = a2 + (((size_t)q * ngt + (t >> 3)) * 16 + (t & 7)) * kTcChunk + lane;
          dst[0] = hi;
          dst[8 * kTcChunk] = lo;
        }
        continue;
      }
      if (j >= cnt) continue;
#pragma unroll
      for (int b = 0; b < NT; ++b) {
        if (b >= B) break;
        float v = 0.f;
        if (got && k >= 0) v = REGLU ? fmaxf(g[b] + bk, 0.f) * u[b] : fmaxf(u[b] + bk, 0.f);
        a[(size_t)j * Btot + g0 + b] = v;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tbase, Lg::COLS);
  }
}

// Down projection of a batch on the tensor cores: y = sum_k a_k WdT[k] over
// the list, as D[col][n] = sum_k WdT[k][col] a2[n][k] with the activations
// carried as fp16 hi/lo pairs (hi = fp16(a), lo = fp16(a - hi): together a to
// about 2^-22 relative, so the sum stays as close to fp32 as on the CUDA
// cores).  Work item w = (column range r of 128, list split s) of an R x S
// grid of items; CTA c takes items c, c + G, ... .  Per item, the stages are
// the split's chunks of 32 positions: the W_down^T tile [32 neurons][128
// columns] (MN-major, 128-byte swizzle: the 8-neuron group kg and 64-column
// atom at (2 kg + atom) * 1024) and, per group of 8 tokens, the a2 tile [16
// rows][32] (K-major, 64-byte swizzle, 1 KB).  One thread issues, per stage,
// 2 K-steps x NG groups of M 128 x N 16 x K 16 MMAs into the 16-column
// accumulator of each group (64 tensor-memory columns in all); warps 0-3 read
// an item's accumulators (lane = column), add hi and lo and write the item's
// partial y[s][b][col]; k_reduce_partials sums the S splits in order.
template <int NG>
struct DnTc {
  static constexpr int W = kTcChunk * kTcRows * 2;     // 8 KB
  static constexpr int A = NG * 16 * kTcChunk * 2;     // NG KB
  static constexpr int STAGE = W + A;
  static constexpr int NS = 8;
  static constexpr int BAR = 1024;
  static constexpr size_t SMEM = 1024 + BAR + (size_t)NS * STAGE;
  static constexpr uint32_t COLS = 64;
  static_assert(STAGE % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
  static_assert(NG * 16 <= (int)COLS, "one 16-column accumulator per token group");
};

template <int NG>
__global__ void __launch_bounds__(9 * kWarp)
    k_down_tc(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_a,
              const int32_t *__restrict__ idx, const int32_t *__restrict__ count, int d, int n, int B, int R, int S,
              float *__restrict__ part, Header *__restrict__ hdr) {
  using Ld = DnTc<NG>;
  constexpr int NS = Ld::NS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = align1024(smem_raw);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + NS;
  uint64_t *tfull = empty + NS;
  uint64_t *tempty = tfull + 1;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(tempty + 1);
  unsigned char *stages = smem + Ld::BAR;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t *err = &hdr->err;

  if (threadIdx.x == 0) {
    for (int q = 0; q < NS; ++q) {
      mbar_init(&full[q], 4);
      mbar_init(&empty[q], 1);
    }
    mbar_init(&tfull[0], 1);
    mbar_init(&tempty[0], 4 * kWarp);
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tslot, Ld::COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  pdl_wait();
  pdl_trigger();

  int cnt = n;
  if (idx) cnt = max(0, min(ld_cg_i32(count), n));
  const int nch = (cnt + kTcChunk - 1) / kTcChunk;
  const int items = R * S;
  // chunks of item w: the s-th of S equal shares of the list
  auto item_chunks = [&](int w, int &q0) {
    const int sp = w / R;
    q0 = (int)((long long)nch * sp / S);
    return (int)((long long)nch * (sp + 1) / S) - q0;
  };

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ producers --
    // Warp 4 + p issues neurons 8p .. 8p + 7 of every stage; its lanes 0-7
    // keep each its neuron's index four stages ahead (a ring of registers).
    const int p = warp - 4;
    const int kn = 8 * p + (lane & 7);
    const uint64_t pol = l2_evict_first();
    int pw = blockIdx.x, pqi = 0, pq0 = 0, pnq = pw < items ? item_chunks(pw, pq0) : 0;
    while (pw < items && pnq == 0) {
      pw += gridDim.x;
      pnq = pw < items ? item_chunks(pw, pq0) : 0;
    }
    auto next_index = [&]() {
      int raw = -1;
      if (pw < items) {
        const int j = (pq0 + pqi) * kTcChunk + kn;
        if (j < cnt) raw = idx ? ld_cg_i32(idx + j) : j;
        ++pqi;
        while (pw < items && pqi >= pnq) {
          pw += gridDim.x;
          pqi = 0;
          pnq = pw < items ? item_chunks(pw, pq0) : 0;
        }
      }
      return raw;
    };
    int kr0 = next_index(), kr1 = next_index(), kr2 = next_index(), kr3 = next_index();
    const uint32_t tx = (uint32_t)(4 * 512 + (p == 0 ? NG * 1024 : 0));
    bool ok = true;
    int it = 0, issued = 0;
    for (int w = blockIdx.x; w < items && ok; w += gridDim.x) {
      const int col0 = (w % R) * kTcRows;
      int q0;
      const int nq = item_chunks(w, q0);
      for (int qi = 0; qi < nq && ok; ++qi, ++it) {
        const int sl = it % NS;
        const int q = q0 + qi;
        const int raw = kr0;
        kr0 = kr1;
        kr1 = kr2;
        kr2 = kr3;
        kr3 = next_index();
        const int k = (unsigned)raw < (unsigned)n ? raw : 0;   // padding / out of range: row 0, its a is zero
        int rows[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) rows[e] = __shfl_sync(0xffffffffu, k, e);
        if (lane == 0) {
          if (it >= NS && !mbar_wait(&empty[sl], (uint32_t)((it / NS) - 1) & 1u, kWaitNs)) {
            flag_error(err, kErrTimeout);
            ok = false;
          } else {
            unsigned char *st = stages + (size_t)sl * Ld::STAGE;
            mbar_arrive_expect_tx(&full[sl], tx);
            // neurons 8p + 4h .. + 3: 8-neuron group p, rows 4h.. of its two 64-column atoms
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int atom = 0; atom < 2; ++atom)
                tma_gather4(st + (size_t)p * 2048 + (size_t)atom * 1024 + (size_t)h * 512, &tm_w, col0 + atom * 64,
                            rows[4 * h], rows[4 * h + 1], rows[4 * h + 2], rows[4 * h + 3], &full[sl], pol);
            if (p == 0)
#pragma unroll
              for (int g = 0; g < NG; ++g)
                tma_load_2d(st + Ld::W + (size_t)g * 1024, &tm_a, 0, (q * NG + g) * 16, &full[sl]);
            issued = it + 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    // after a wait gave up, let each slot's last load land (bounded) before
    // the shared memory is released
    if (!ok && lane == 0)
      for (int e = max(0, issued - NS); e < issued; ++e) mbar_wait(&full[e % NS], (uint32_t)(e / NS) & 1u, kWaitNs);
  } else if (warp == 8) {
    // ------------------------------------------------------------------ MMA --
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_f16(kTcRows, kTcN, 1, 0);
      bool ok = true;
      int it = 0, done = 0;                          // stages consumed, items with accumulators
      for (int w = blockIdx.x; w < items && ok; w += gridDim.x) {
        int q0;
        const int nq = item_chunks(w, q0);
        if (nq == 0) continue;
        if (done >= 1 && !mbar_wait(&tempty[0], (uint32_t)(done - 1) & 1u, kWaitNs)) {
          flag_error(err, kErrTimeout);
          break;
        }
        tc_fence_after();
        for (int qi = 0; qi < nq; ++qi, ++it) {
          const int sl = it % NS;
          if (!mbar_wait(&full[sl], (uint32_t)(it / NS) & 1u, kWaitNs)) {
            flag_error(err, kErrTimeout);
            ok = false;
            break;
          }
          tc_fence_after();
          unsigned char *st = stages + (size_t)sl * Ld::STAGE;
#pragma unroll
          for (int kk = 0; kk < kTcChunk / 16; ++kk) {
            // neurons 16 kk .. 16 kk + 15: 8-neuron groups 2 kk, 2 kk + 1 (SBO 2048); columns: atoms 0, 1 (LBO 1024)
            const uint64_t ad = umma_desc(st + (size_t)(2 * kk) * 2048, 1024, 2048, kSwz128);
#pragma unroll
            for (int g = 0; g < NG; ++g) {
              const uint64_t bd = umma_desc(st + Ld::W + g * 1024 + kk * 32, 16, 512, kSwz64);
              umma_f16(tbase + (uint32_t)(kTcN * g), ad, bd, idesc, (qi | kk) != 0);
            }
          }
          umma_commit(&empty[sl]);
        }
        if (ok) umma_commit(&tfull[0]);
        ++done;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue --
    const uint32_t lane_addr = tbase + ((uint32_t)(kWarp * warp) << 16);
    int done = 0;
    for (int w = blockIdx.x; w < items; w += gridDim.x) {
      int q0;
      const int nq = item_chunks(w, q0);
      const int col = (w % R) * kTcRows + kWarp * warp + lane;
      const int sp = w / R;
      bool got = false;
      if (nq > 0) {
        got = __all_sync(0xffffffffu, mbar_wait(&tfull[0], (uint32_t)done & 1u, kWaitNs));
        if (!got && lane == 0) flag_error(err, kErrTimeout);
        tc_fence_after();
      }
      float v[NG][16];
      __syncwarp();          // tensor-memory loads below are warp-synchronous
      if (got) {
#pragma unroll
        for (int g = 0; g < NG; ++g) tmem_ld16(lane_addr + (uint32_t)(kTcN * g), v[g]);
      }
      if (nq > 0) {
        tc_fence_before();
        mbar_arrive(&tempty[0]);
        ++done;
      }
      if (col < d) {
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int b = 8 * g + e;
            if (b < B) part[((size_t)sp * B + b) * d + col] = got ? v[g][e] + v[g][8 + e] : 0.f;
          }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tbase, Ld::COLS);
  }
}

// ======================================================================== //
// fused sparse FFN: bulk-copy ring + grid-barrier reduction                //
// ======================================================================== //

// Shared-memory layout of k_sparse_ffn for NS ring slots of M rows of d elements.
struct FusedLayout {
  int NS, grp;
  size_t full, empty, kslot, list, bias, words, pd, x, stage, red, total;
};

// nl_max: most list positions one CTA takes (ceil(n / grid)); mask_words:
// words of the union mask the kernel ranks itself (0 when it gets a list).
__host__ __device__ inline FusedLayout fused_layout(int NS, int d, int M, int esz, int NB, int nl_max,
                                                    int mask_words) {
  FusedLayout L;
  L.NS = NS;
  L.grp = NS / 2 > 0 ? NS / 2 : 1;
  size_t o = 0;
  L.full = o;  o += (size_t)NS * 8;
  L.empty = o; o += (size_t)NS * 8;
  L.kslot = o; o += (size_t)NS * 4;
  L.list = o;  o += (size_t)nl_max * 4;
  L.bias = o;  o += (size_t)nl_max * 4;
  o = align_up(o, 16);
  L.words = o; o += (size_t)(mask_words + 3) / 4 * 16 * 2;    // the words, then their prefix counts
  o = align_up(o, 16);
  L.pd = o;    o += (size_t)2 * kFusedWarps * L.grp * 2 * NB * 4;   // two buffers, alternate groups
  o = align_up(o, 128);
  L.x = o;     o += (size_t)NB * d * esz;
  o = align_up(o, 128);
  L.stage = o; o += (size_t)NS * M * d * esz;
  L.red = 0;
  L.total = o;
  return L;
}

// Ranking the set bits of a union mask (n bits in n_words words) into the
// list positions one CTA of G takes: slist[i] = the bit at position c + i*G.
// NT threads (the consumer warps), each owning a contiguous run of at most
// MAXW words.  First the words' loads are issued (mask_words_load), so that
// they are in flight while x is staged; then rank_mask_block keeps the words
// in shared memory (sw, n_words rounded up to 4), scans the runs' popcounts
// across the block, writes every word's inclusive prefix count (spre), and
// finds each position's word by binary search over spre and the bit within
// it.  Leaves the list length in *s_nl and the number of set bits in *s_cnt.
template <int NT, int MAXW>
__device__ __forceinline__ void mask_words_load(const uint32_t *__restrict__ mask, int n_words,
                                                uint32_t (&w)[MAXW]) {
  const int wpt = (n_words + NT - 1) / NT;
  const int wb = min(n_words, (int)threadIdx.x * wpt), we = min(n_words, wb + wpt);
#pragma unroll
  for (int u = 0; u < MAXW; ++u) w[u] = wb + u < we ? __ldcg(mask + wb + u) : 0u;
}

template <int NT, int MAXW>
__device__ __forceinline__ void rank_mask_block(uint32_t (&w)[MAXW], int n_words, int n, int c, int G, int *slist,
                                                uint32_t *sw, int *spre, int *s_wsum, int *s_nl, int *s_cnt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wpt = (n_words + NT - 1) / NT;
  const int wb = min(n_words, tid * wpt), we = min(n_words, wb + wpt);
  const uint32_t tail = (n & 31) ? ((1u << (n & 31)) - 1u) : 0xffffffffu;
  int tot = 0;
#pragma unroll
  for (int u = 0; u < MAXW; ++u) {
    const int i = wb + u;
    if (i < we) {
      if (i == n_words - 1) w[u] &= tail;
      sw[i] = w[u];
      tot += __popc(w[u]);
    }
  }
  int incl = tot;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == kWarp - 1) s_wsum[warp] = incl;
  named_sync(3, NT);
  int before = 0, all = 0;
#pragma unroll
  for (int q = 0; q < NT / kWarp; ++q) {
    const int v = s_wsum[q];
    all += v;
    if (q < warp) before += v;
  }
  int run = before + incl - tot;
#pragma unroll
  for (int u = 0; u < MAXW; ++u) {
    const int i = wb + u;
    if (i < we) {
      run += __popc(w[u]);
      spre[i] = run;
    }
  }
  named_sync(3, NT);
  const int nl = all > c ? (all - 1 - c) / G + 1 : 0;
  for (int i = tid; i < nl; i += NT) {
    const int p = c + G * i;
    int lo = 0, hi = n_words - 1;          // first word whose inclusive count exceeds p
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (spre[mid] > p) hi = mid; else lo = mid + 1;
    }
    uint32_t m = sw[lo];
    for (int q = p - (lo ? spre[lo - 1] : 0); q > 0; --q) m &= m - 1u;   // drop the lower set bits
    slist[i] = lo * 32 + __ffs(m) - 1;
  }
  if (tid == 0) {
    *s_nl = nl;
    *s_cnt = all;
  }
  named_sync(3, NT);
}

// Most mask words per consumer thread when the sparse FFN ranks the mask.
constexpr int kRankWords = 8;

// One kernel for the whole neuron-sparse FFN of B <= NB tokens.
//
// CTA c of a grid of G takes list positions c, c + G, c + 2G, ...: its first
// index loads need not wait for the count.  The list comes from idx/count, or
// (idx == NULL) is every neuron, or (mask != NULL) is built here from the
// predictor's union mask: the consumer warps rank its set bits (block-wide
// scan) and the producer's idle lanes write this CTA's positions out as
// idx_out/count_out (no separate compaction kernel).  Warp
// kFusedWarps is the producer: one lane streams, for each of its neurons k,
// the rows Wg[k], Wu[k], WdT[k] into a ring of NS shared-memory slots with
// cp.async.bulk, completing on the slot's "full" mbarrier.  The 8 consumer
// warps split d: each owns chunks (q*8 + warp)*32 + lane, so every warp reads
// every slot.  Neurons are consumed in groups of NS/2 (the other half of the
// ring is being refilled): partial gate/up dots over the warp's d-slice go to
// shared memory, one named barrier, every warp sums the 8 partials in warp
// order, applies ReLU(g + b) * u (or ReLU(u + b)), and accumulates
// a * WdT[k] into its registers; then it releases the slot ("empty").
// At the end every CTA stores its y partial; k_reduce_partials, the next
// kernel, sums them in a fixed order (deterministic, no float atomics).
// Once the producer has queued its last copy it issues this CTA's share of the
// asf_ffn.l2_next L2 prefetch.
template <typename T, int NB, int MAXQ, bool REGLU>
__global__ void __launch_bounds__((kFusedWarps + 1) * kWarp)
    k_sparse_ffn(const T *__restrict__ Wg, const T *__restrict__ Wu, const T *__restrict__ WdT,
                 const float *__restrict__ bias, const T *__restrict__ x, int d, int n, int B,
                 const int32_t *__restrict__ idx, const int32_t *__restrict__ count,
                 const uint32_t *__restrict__ mask, int n_words, int32_t *__restrict__ idx_out,
                 int32_t *__restrict__ count_out, int NS, int hot_rows,
                 long long rs, int packed, float *__restrict__ part, float *__restrict__ y,
                 Header *__restrict__ hdr, L2Next nx, int inject) {
  constexpr int V = Vec<T>::N;
  constexpr int M = REGLU ? 3 : 2;
  constexpr int NW = kFusedWarps;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_fail, s_nl, s_cnt;
  __shared__ int s_wsum[kFusedWarps];
  const FusedLayout L = fused_layout(NS, d, M, (int)sizeof(T), NB, (n + (int)gridDim.x - 1) / (int)gridDim.x,
                                     mask ? n_words : 0);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.full);
  uint64_t *empty = reinterpret_cast<uint64_t *>(smem + L.empty);
  int *kslot = reinterpret_cast<int *>(smem + L.kslot);
  int *slist = reinterpret_cast<int *>(smem + L.list);        // neuron at list position c + i*G
  float *sbias = reinterpret_cast<float *>(smem + L.bias);    // its bias
  float *pd = reinterpret_cast<float *>(smem + L.pd);
  T *xs = reinterpret_cast<T *>(smem + L.x);
  T *stage = reinterpret_cast<T *>(smem + L.stage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = d / V;
  const int grp = L.grp;
  int32_t *err = &hdr->err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
      kslot[s] = -1;
    }
    fence_mbar_init();
    s_fail = 0;
  }
  __syncthreads();
  // Speculative warm-up: the leading hot_rows rows (hot neurons stored first)
  // are active for most tokens, so their gate/up/down rows go to L2 while the
  // predictor is still deciding; the bulk copies below then mostly hit L2.
  if (hot_rows > 0 && warp == NW) {
    // packed layout: the hot rows of all matrices are one contiguous block
    const size_t rows = (size_t)min(hot_rows, n);
    const size_t bytes = packed ? rows * (size_t)rs * sizeof(T) : rows * (size_t)d * sizeof(T);
    const size_t per = (bytes / gridDim.x + 15) & ~(size_t)15;
    const size_t o0 = min(bytes, per * blockIdx.x), o1 = min(bytes, o0 + per);
    const T *mats[3] = {REGLU ? Wg : Wu, Wu, WdT};
    for (int m = (REGLU || packed) ? 0 : 1; m < (packed ? 1 : 3); ++m) {
      const unsigned char *base = reinterpret_cast<const unsigned char *>(mats[m]);
      for (size_t o = o0 + (size_t)lane * 16384; o < o1; o += 32 * 16384)
        prefetch_l2(base + o, (uint32_t)min((size_t)16384, o1 - o));
    }
  }
  // The next kernel only prefetches weights before it waits on this one.
  pdl_trigger();
  pdl_wait();

  const int G = gridDim.x, cta = blockIdx.x;
  float acc[MAXQ][V][NB];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q)
#pragma unroll
    for (int e = 0; e < V; ++e)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[q][e][b] = 0.f;

  if (mask) {
    // ------------------------------- the list from the mask (combined call) --
    if (warp < NW) {
      // consumer warps rank the mask; its words load while x is staged
      uint32_t mw[kRankWords];
      mask_words_load<NW * kWarp, kRankWords>(mask, n_words, mw);
      stage16<8>(reinterpret_cast<uint4 *>(xs), reinterpret_cast<const uint4 *>(x), B * nvec, NW * kWarp);
      for (int i = B * nvec + threadIdx.x; i < NB * nvec; i += NW * kWarp)
        reinterpret_cast<uint4 *>(xs)[i] = make_uint4(0u, 0u, 0u, 0u);
      uint32_t *sw = reinterpret_cast<uint32_t *>(smem + L.words);
      rank_mask_block<NW * kWarp, kRankWords>(mw, n_words, n, cta, G, slist, sw,
                                              reinterpret_cast<int *>(sw) + (n_words + 3) / 4 * 4, s_wsum, &s_nl,
                                              &s_cnt);
      named_arrive(2, (NW + 1) * kWarp);     // the list is ready for the producer
    } else {
      named_sync(2, (NW + 1) * kWarp);
      if (lane > 0) {
        // this CTA's positions of the list, written out by the lanes that do
        // not issue copies (all CTAs together write idx_out[0..count))
        const int nlp = s_nl;
        for (int i = lane - 1; i < nlp; i += kWarp - 1) idx_out[cta + (size_t)G * i] = slist[i];
        if (cta == 0 && lane == 1) *count_out = s_cnt;
      }
    }
  } else if (warp == NW) {
    // -------------------------------------------------- this CTA's list --
    int cnt;
    if (idx) {
      // the count and the first 32 positions are fetched together
      const int p0 = cta + G * lane;
      const int c_raw = ld_cg_i32(count);
      const int k0 = p0 < n ? ld_cg_i32(idx + p0) : -1;
      if ((c_raw < 0 || c_raw > n) && cta == 0 && lane == 0) flag_error(err, kErrIndex);
      cnt = max(0, min(c_raw, n));
      const int nl0 = cnt > cta ? (cnt - 1 - cta) / G + 1 : 0;
      if (lane < nl0) slist[lane] = k0;
      for (int i = kWarp + lane; i < nl0; i += kWarp) slist[i] = ld_cg_i32(idx + cta + (size_t)G * i);
    } else {
      cnt = n;
      const int nl0 = n > cta ? (n - 1 - cta) / G + 1 : 0;
      for (int i = lane; i < nl0; i += kWarp) slist[i] = cta + G * i;
    }
    if (lane == 0) s_nl = cnt > cta ? (cnt - 1 - cta) / G + 1 : 0;
    // hand the list to the consumers without waiting for them
    __syncwarp();
    named_arrive(2, (NW + 1) * kWarp);
  } else {
    // consumers: x into shared memory while the list is being fetched
    stage16<8>(reinterpret_cast<uint4 *>(xs), reinterpret_cast<const uint4 *>(x), B * nvec, NW * kWarp);
    for (int i = B * nvec + threadIdx.x; i < NB * nvec; i += NW * kWarp)
      reinterpret_cast<uint4 *>(xs)[i] = make_uint4(0u, 0u, 0u, 0u);
    named_sync(2, (NW + 1) * kWarp);
  }
  const int nl = s_nl;
  int issued = 0;     // ring slots the producer has filled (its lane 0)

  if (warp == NW) {
    // ------------------------------------------------------------ producer --
    // lane 0 issues one neuron's copies per ring slot.  The test hook
    // kInjectWithholdFfn makes CTA 0 issue none, so its consumers' first
    // bounded wait runs out.
    const uint32_t row_bytes = (uint32_t)((size_t)d * sizeof(T));
    const uint64_t pol = l2_evict_first();
    const bool withhold = inject == kInjectWithholdFfn && cta == 0;
    for (int i = 0; i < nl && lane == 0 && !withhold; ++i) {
      const int k = slist[i];
      {
        const int s = i % NS;
        if (i >= NS && !mbar_wait(&empty[s], (uint32_t)((i / NS) - 1) & 1u, kWaitNs)) {
          flag_error(err, kErrTimeout);
          s_fail = 1;
          break;
        } else if (*reinterpret_cast<volatile int *>(&s_fail)) {
          break;     // a consumer gave up: issue nothing more into the ring
        } else if ((unsigned)k >= (unsigned)n) {
          flag_error(err, kErrIndex);
          kslot[s] = -1;
          mbar_arrive(&full[s]);
        } else {
          kslot[s] = k;
          mbar_arrive_expect_tx(&full[s], (uint32_t)M * row_bytes);
          T *dst = stage + (size_t)s * M * d;
          if (packed) {          // the neuron's rows are one contiguous block
            bulk_g2s_stream(dst, (REGLU ? Wg : Wu) + (size_t)k * rs, (uint32_t)M * row_bytes, &full[s], pol);
          } else if constexpr (REGLU) {
            bulk_g2s_stream(dst, Wg + (size_t)k * rs, row_bytes, &full[s], pol);
            bulk_g2s_stream(dst + d, Wu + (size_t)k * rs, row_bytes, &full[s], pol);
            bulk_g2s_stream(dst + 2 * (size_t)d, WdT + (size_t)k * rs, row_bytes, &full[s], pol);
          } else {
            bulk_g2s_stream(dst, Wu + (size_t)k * rs, row_bytes, &full[s], pol);
            bulk_g2s_stream(dst + d, WdT + (size_t)k * rs, row_bytes, &full[s], pol);
          }
        }
        issued = i + 1;
      }
    }
    __syncwarp();
    // Every row copy of this CTA is queued: only now pull the hinted ranges
    // into L2, so that they take bandwidth the row stream leaves idle instead
    // of delaying its first rows.
    prefetch_next(nx, blockIdx.x, gridDim.x);
  } else {
    // ----------------------------------------------------------- consumers --
    // the biases of this CTA's neurons, while the first rows are in flight
    for (int i = threadIdx.x; i < nl; i += NW * kWarp) {
      const int k = slist[i];
      sbias[i] = (unsigned)k < (unsigned)n ? __ldg(bias + k) : 0.f;
    }
    named_sync(1, NW * kWarp);
    // each lane meets the same chunks of x for every neuron: keep them in registers
    uint4 xr[MAXQ][NB];
#pragma unroll
    for (int qq = 0; qq < MAXQ; ++qq) {
      const int ch = (qq * NW + warp) * kWarp + lane;
#pragma unroll
      for (int b = 0; b < NB; ++b)
        xr[qq][b] = ch < nvec ? *reinterpret_cast<const uint4 *>(xs + (size_t)b * d + (size_t)ch * V)
                              : make_uint4(0u, 0u, 0u, 0u);
    }
    bool ok = true;
    for (int g0 = 0; g0 < nl; g0 += grp) {
      const int gn = min(grp, nl - g0);
      // consecutive groups use alternate partial buffers: a warp writing the
      // next group's partials has passed that group's barrier only after
      // every warp has read this group's, so one barrier per group suffices
      float *pdg = pd + (size_t)((g0 / grp) & 1) * (NW * grp * 2 * NB);
      for (int q = 0; q < gn; ++q) {
        const int i = g0 + q, s = i % NS;
        if (ok && !mbar_wait(&full[s], (uint32_t)(i / NS) & 1u, kWaitNs)) {
          if (lane == 0) flag_error(err, kErrTimeout);
          ok = false;
          s_fail = 1;
        }
        float pg[NB], pu[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) pg[b] = pu[b] = 0.f;
        if (ok && kslot[s] >= 0) {
          const T *ru = stage + (size_t)s * M * d + (REGLU ? d : 0);
          const T *rg = stage + (size_t)s * M * d;
#pragma unroll
          for (int qq = 0; qq < MAXQ; ++qq) {
            const int ch = (qq * NW + warp) * kWarp + lane;
            if (ch < nvec) {
              const uint4 wu = *reinterpret_cast<const uint4 *>(ru + (size_t)ch * V);
              uint4 wg = wu;
              if constexpr (REGLU) wg = *reinterpret_cast<const uint4 *>(rg + (size_t)ch * V);
#pragma unroll
              for (int b = 0; b < NB; ++b) {
                pu[b] = Vec<T>::dot(wu, xr[qq][b], pu[b]);
                if constexpr (REGLU) pg[b] = Vec<T>::dot(wg, xr[qq][b], pg[b]);
              }
            }
          }
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          pu[b] = warp_sum(pu[b]);
          if constexpr (REGLU) pg[b] = warp_sum(pg[b]);
        }
        if (lane == 0) {
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            pdg[(((size_t)warp * grp + q) * 2 + 0) * NB + b] = pg[b];
            pdg[(((size_t)warp * grp + q) * 2 + 1) * NB + b] = pu[b];
          }
        }
      }
      named_sync(1, NW * kWarp);
      for (int q = 0; q < gn; ++q) {
        const int i = g0 + q, s = i % NS;
        const int k = kslot[s];
        float a[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float g = 0.f, u = 0.f;
#pragma unroll
          for (int w = 0; w < NW; ++w) {
            g += pdg[(((size_t)w * grp + q) * 2 + 0) * NB + b];
            u += pdg[(((size_t)w * grp + q) * 2 + 1) * NB + b];
          }
          float v = 0.f;
          if (k >= 0 && b < B) {
            const float bk = sbias[i];
            v = REGLU ? fmaxf(g + bk, 0.f) * u : fmaxf(u + bk, 0.f);
          }
          a[b] = v;
        }
        if (ok && k >= 0) {
          const T *rd = stage + (size_t)s * M * d + (size_t)(M - 1) * d;
#pragma unroll
          for (int qq = 0; qq < MAXQ; ++qq) {
            const int ch = (qq * NW + warp) * kWarp + lane;
            if (ch < nvec) {
              float f[V];
              Vec<T>::to_float(*reinterpret_cast<const uint4 *>(rd + (size_t)ch * V), f);
#pragma unroll
              for (int e = 0; e < V; ++e)
#pragma unroll
                for (int b = 0; b < NB; ++b) acc[qq][e][b] = fmaf(a[b], f[e], acc[qq][e][b]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
    if (!ok) s_fail = 1;
  }
  // -------------------------------------------------------- reductions --
  // this CTA's partial y, straight from registers (each lane owns its chunks)
  if (warp < NW) {
#pragma unroll
    for (int qq = 0; qq < MAXQ; ++qq) {
      const int ch = (qq * NW + warp) * kWarp + lane;
      if (ch < nvec) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b < B) {
            float *dst = part + ((size_t)blockIdx.x * B + b) * d + (size_t)ch * V;
#pragma unroll
            for (int e = 0; e < V; e += 4)
              *reinterpret_cast<float4 *>(dst + e) =
                  make_float4(acc[qq][e][b], acc[qq][e + 1][b], acc[qq][e + 2][b], acc[qq][e + 3][b]);
          }
        }
      }
    }
  }
  // After a wait gave up, copies the consumers no longer wait for may still be
  // in flight: let each slot's last one land (bounded) before shared memory is
  // released.
  __syncthreads();
  if (s_fail && warp == NW && lane == 0)
    for (int i = max(0, issued - NS); i < issued; ++i) mbar_wait(&full[i % NS], (uint32_t)(i / NS) & 1u, kWaitNs);
}

// y[b][col] = sum over the G per-CTA partials, in a fixed order: a CTA owns
// 32 * VEC consecutive columns (each lane VEC of them, loaded as one vector),
// the 8 warps split the partials into runs of ceil(G / 8) and every warp sums
// its run in order; warp sums are then combined in warp order (the same order
// for every VEC).  The grid stays resident beside the sparse FFN from that
// kernel's start, and the kernel stays small in registers, since at d = 4096
// the next layer's layer-1 kernel must fit beside both: VEC 1 where that grid
// fits one CTA per SM (128 CTAs at d = 4096), VEC 4 otherwise (64 CTAs at d =
// 8192, 96 at 12288; 256 CTAs of VEC 1 there measured 3% slower end to end,
// 128 of VEC 2 as slow).  part and y are 16-byte aligned and d % 4 == 0
// (every caller's workspace and checked output).
constexpr int kReduceWarps = 8;
constexpr int kReduceMaxPerWarp = 32;      // G <= 256
constexpr int kReduceBatch = 20;           // loads in flight per lane (G <= 160: one batch)

template <int VEC> struct FVec;
template <> struct FVec<1> { using type = float; };
template <> struct FVec<4> { using type = float4; };
__device__ __forceinline__ void fv_zero(float &a) { a = 0.f; }
__device__ __forceinline__ void fv_zero(float4 &a) { a = make_float4(0.f, 0.f, 0.f, 0.f); }
__device__ __forceinline__ void fv_add(float &a, float b) { a += b; }
__device__ __forceinline__ void fv_add(float4 &a, float4 b) { a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w; }

template <int VEC>
__global__ void __launch_bounds__(kReduceWarps * kWarp)
    k_reduce_partials(const float *__restrict__ part, int G, int B, int d, float *__restrict__ y) {
  using F = typename FVec<VEC>::type;
  __shared__ F red[kReduceWarps][kWarp];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int col = (blockIdx.x * kWarp + lane) * VEC;
  const int b = blockIdx.y;
  const int per = (G + kReduceWarps - 1) / kReduceWarps;
  const int q0 = warp * per;
  F s;
  fv_zero(s);
  for (int u0 = 0; u0 < per; u0 += kReduceBatch) {
    F v[kReduceBatch];
#pragma unroll
    for (int u = 0; u < kReduceBatch; ++u) {
      const int q = q0 + u0 + u;
      if (u0 + u < per && q < G && col < d)
        v[u] = __ldcg(reinterpret_cast<const F *>(part + ((size_t)q * B + b) * d + col));
      else
        fv_zero(v[u]);
    }
#pragma unroll
    for (int u = 0; u < kReduceBatch; ++u) fv_add(s, v[u]);
  }
  red[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && col < d) {
    F t;
    fv_zero(t);
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w) fv_add(t, red[w][lane]);
    *reinterpret_cast<F *>(y + (size_t)b * d + col) = t;
  }
}

// ======================================================================== //
// neuron-sharded layer: the final reduction exchanged over peer memory     //
// ======================================================================== //

// Pointers of every rank's publication buffer and flag words, valid on this
// GPU (its own, and the peers' mapped over NVLink).
struct PeerPtrs {
  float *pub[ASF_MAX_PEERS];
  uint32_t *flag[ASF_MAX_PEERS];
};

// y = sum over ranks r = 0..world-1, in rank order, of rank r's sum of its G
// partials (in order).  CTA (column block, token) first sums this rank's
// partials as k_reduce_partials does, then warp 0 publishes the 32 sums in
// this rank's buffer (half e & 1 for call e of the block, so a slow peer still
// reads the previous call's half undisturbed), releases the block's flag
// = e at system scope, waits (bounded) until every peer's flag for the block
// reaches e, and adds all ranks' sums in rank order -- each rank computes the
// same y bit for bit.  The exchange costs (world - 1) x 128 bytes of peer
// reads per block, and no separate collective launch.
//
// blockIdx.z selects one of the ranks a process holds (1 normally; all of them
// in the one-GPU emulation, launched cooperatively so that every block is
// resident while it waits): rank rank0 + z, partials at part + z * part_rs,
// output at y + z * y_rs, call counters at epoch + z * nblk.
__global__ void __launch_bounds__(kReduceWarps * kWarp)
    k_reduce_exchange(const float *__restrict__ part, long long part_rs, int G, int B, int d, int maxB,
                      const __grid_constant__ PeerPtrs pp, uint32_t *__restrict__ epoch, float *__restrict__ y, long long y_rs, int world,
                      int rank0, int32_t *__restrict__ err) {
  __shared__ float red[kReduceWarps][kWarp];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int col = blockIdx.x * kWarp + lane;
  const int b = blockIdx.y;
  const int z = blockIdx.z;
  const int rank = rank0 + z;
  const float *pr = part + (size_t)z * part_rs;
  const int per = (G + kReduceWarps - 1) / kReduceWarps;
  const int q0 = warp * per;
  float v[kReduceMaxPerWarp];
#pragma unroll
  for (int u = 0; u < kReduceMaxPerWarp; ++u) {
    const int q = q0 + u;
    v[u] = (u < per && q < G && col < d) ? ld_cg_f32(pr + ((size_t)q * B + b) * d + col) : 0.f;
  }
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < kReduceMaxPerWarp; ++u) s += v[u];
  red[warp][lane] = s;
  __syncthreads();
  if (warp != 0) return;
  float mine = 0.f;
#pragma unroll
  for (int w = 0; w < kReduceWarps; ++w) mine += red[w][lane];
  const int nbx = (d + kWarp - 1) / kWarp;
  const int blk = b * nbx + blockIdx.x;
  uint32_t *ep = epoch + (size_t)z * nbx * maxB + blk;
  uint32_t e = 0;
  if (lane == 0) {
    e = *ep + 1u;
    *ep = e;
  }
  e = __shfl_sync(0xffffffffu, e, 0);
  const size_t half = ((size_t)(e & 1u) * maxB + b) * d;
  if (col < d) pp.pub[rank][half + col] = mine;
  __threadfence_system();
  __syncwarp();
  if (lane == 0) st_release_sys(pp.flag[rank] + blk, e);
  // every peer's sums for this call
  bool ok = true;
  if (lane < world && lane != rank) {
    const uint32_t *f = pp.flag[lane] + blk;
    if ((int)(ld_acquire_sys(f) - e) < 0) {
      const uint64_t t0 = global_ns();
      while ((int)(ld_acquire_sys(f) - e) < 0) {
        if (global_ns() - t0 > kWaitNs) {
          ok = false;
          break;
        }
      }
    }
  }
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && lane == 0) flag_error(err, kErrTimeout);
  float acc = 0.f;
  for (int h = 0; h < world; ++h) {
    if (h == rank) {
      acc += mine;
    } else if (ok) {
      (void)ld_acquire_sys(pp.flag[h] + blk);      // this lane's own acquire of the peer's release
      acc += col < d ? ld_relaxed_sys(pp.pub[h] + half + col) : 0.f;
    }
  }
  if (col < d) y[(size_t)z * y_rs + (size_t)b * d + col] = acc;
}

// ======================================================================== //
// offline: activation counts and row permutation                           //
// ======================================================================== //

// counts[k] += #{t : W[k] . x_t + bias_k > 0}.  Warps own rows; the row is
// re-read from L1/L2 for every group of NB tokens.
template <typename T, int NB, int U>
__global__ void __launch_bounds__(kThreads)
    k_act_counts(const T *__restrict__ W, const float *__restrict__ bias, const T *__restrict__ x, int d,
                 long long rs, int n, int Ttok, int rpc, int64_t *__restrict__ counts) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T *xs = reinterpret_cast<T *>(smem_raw);
  constexpr int V = Vec<T>::N;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  const int row0 = blockIdx.x * rpc;
  const int row1 = min(n, row0 + rpc);
  const int nvec = d / V;
  for (int rb = row0; rb < row1; rb += kWarps) {
    const int row = rb + warp;
    const bool ok = row < row1;
    long long c = 0;
    const float bk = ok ? __ldg(bias + row) : 0.f;
    for (int g0 = 0; g0 < Ttok; g0 += NB) {
      const int nb = min(NB, Ttok - g0);
      __syncthreads();
      stage_tokens<T, NB>(xs, x, d, g0, nb);
      __syncthreads();
      if (ok) {
        float acc[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = 0.f;
        row_dot<T, NB, U>(W + (size_t)row * rs, xs, d, nvec, lane, acc);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float s = warp_sum(acc[b]) + bk;
          c += (b < nb && s > 0.f) ? 1 : 0;
        }
      }
    }
    if (ok && lane == 0) counts[row] += c;
  }
}

// dst row i (at dst + i*dst_stride) = src row perm[i] (at src + perm[i]*src_stride),
// row_bytes each; identity when perm is null.  One CTA per row (grid-stride),
// widest copy unit the alignment allows.
__global__ void __launch_bounds__(kThreads)
    k_permute_rows(const unsigned char *__restrict__ src, long long src_stride, unsigned char *__restrict__ dst,
                   long long dst_stride, int n_rows, int src_rows, long long row_bytes,
                   const int32_t *__restrict__ perm, int unit) {
  for (int i = blockIdx.x; i < n_rows; i += gridDim.x) {
    const int p = perm ? __ldg(perm + i) : i;
    if ((unsigned)p >= (unsigned)src_rows) continue;
    const unsigned char *s = src + (size_t)p * src_stride;
    unsigned char *t = dst + (size_t)i * dst_stride;
    if (unit == 16) {
      for (long long o = threadIdx.x; o < row_bytes / 16; o += blockDim.x)
        reinterpret_cast<uint4 *>(t)[o] = __ldg(reinterpret_cast<const uint4 *>(s) + o);
    } else if (unit == 4) {
      for (long long o = threadIdx.x; o < row_bytes / 4; o += blockDim.x)
        reinterpret_cast<uint32_t *>(t)[o] = __ldg(reinterpret_cast<const uint32_t *>(s) + o);
    } else {
      for (long long o = threadIdx.x; o < row_bytes; o += blockDim.x) t[o] = s[o];
    }
  }
}

// ======================================================================== //
// host side                                                                //
// ======================================================================== //

struct DevCache {
  int sms = 0;
};
std::mutex g_mu;
DevCache g_dev[64];

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_dev[dev].sms == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    g_dev[dev].sms = v;
  }
  return g_dev[dev].sms;
}

// Process-wide test hook (asf_set_fault_injection): 0 = off.
std::atomic<int> g_inject{0};
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args... args) {
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute((const void *)kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  // Every kernel prefers the largest shared-memory carveout: an SM then never
  // has to be reconfigured between the chained kernels, and a kernel can start
  // beside one that uses less than all of it (the layer-2 predictor beside the
  // layer-1 slice kernel: +1.7% tokens/s at the 70B shape).
  cudaFuncSetAttribute((const void *)kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                       (int)cudaSharedmemCarveoutMaxShared);
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

inline bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool al4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline size_t r256(size_t v) { return (v + 255) & ~size_t(255); }
inline int vec_of(asf_dtype t) { return t == ASF_F16 ? 8 : 4; }
inline int esize(asf_dtype t) { return t == ASF_F16 ? 2 : 4; }

int n_words_of(int n) { return (n + 31) / 32; }

// column tiles and index-list splits of the down projection
int down_tiles(const asf_ffn *f) { return (f->d + kWarp * vec_of(f->wdtype) - 1) / (kWarp * vec_of(f->wdtype)); }
int down_splits(const asf_ffn *f) {
  const int ct = down_tiles(f);
  return std::max(1, std::min(kMaxSplits, (kTargetCtas + ct - 1) / ct));
}

size_t mask_region(const asf_predictor *p) {
  return r256((size_t)std::max(n_words_of(p->n), kMaxGrid) * 4);
}
// Row stride of the FFN matrices in elements (0 in the descriptor = d).
long long ffn_rs(const asf_ffn *f) { return f->row_stride > 0 ? (long long)f->row_stride : (long long)f->d; }

// Neuron-major packed layout: a neuron's gate/up/down rows are one contiguous
// block of M*d elements, so one bulk copy fetches all of them.
bool ffn_packed(const asf_ffn *f) {
  const int M = f->act == ASF_ACT_REGLU ? 3 : 2;
  const size_t rb = (size_t)f->d * esize(f->wdtype);
  if (ffn_rs(f) != (long long)M * f->d) return false;
  const char *first = static_cast<const char *>(f->act == ASF_ACT_REGLU ? f->Wg : f->Wu);
  if (f->act == ASF_ACT_REGLU && static_cast<const char *>(f->Wu) != first + rb) return false;
  return static_cast<const char *>(f->WdT) == first + (size_t)(M - 1) * rb;
}

size_t pred_scratch(const asf_predictor *p, int B) { return mask_region(p) + r256((size_t)B * p->r * 4); }

// Tensor-core down projection: column ranges of 128 and list splits chosen so
// that the R x S work items fill whole waves of CTAs (at least 95% busy when
// some S <= 32 allows it).
int tc_ranges(const asf_ffn *f) { return (f->d + kTcRows - 1) / kTcRows; }
// List splits S of the tensor-core down projection: the fewest whose R x S
// equal work items fill whole waves of one CTA per SM to at least 95% (R = 64
// column ranges at d = 8192 alone would leave 84 of 148 SMs idle).
int tc_splits(const asf_ffn *f) {
  const int R = tc_ranges(f), G = std::min(sm_count(), kMaxGrid);
  int best = 1;
  double best_eff = -1.0;
  for (int S = 1; S <= 32; ++S) {
    const int items = R * S;
    const double eff = (double)items / ((double)((items + G - 1) / G) * G);
    if (eff >= 0.95) return S;
    if (eff > best_eff) {
      best_eff = eff;
      best = S;
    }
  }
  return best;
}
int tc_groups(int B) { return (B + 7) / 8; }
size_t tc_a2_bytes(const asf_ffn *f, int B) {
  return r256((size_t)((f->n + kTcChunk - 1) / kTcChunk) * tc_groups(B) * 16 * kTcChunk * 2);
}

bool tc_ok(const asf_ffn *f, int B);

size_t ffn_scratch(const asf_ffn *f, int B) {
  const size_t two_kernel = r256((size_t)f->n * B * 4) + r256((size_t)down_splits(f) * B * f->d * 4);
  const size_t fused = r256((size_t)std::min(sm_count(), kMaxGrid) * B * f->d * 4);
  const size_t tc = tc_ok(f, B) ? tc_a2_bytes(f, B) + r256((size_t)tc_splits(f) * B * f->d * 4) : 0;
  return std::max({two_kernel, fused, tc});
}

asf_status check_pred(const asf_predictor *p) {
  if (!p || !p->W1 || !p->b1 || !p->W2 || !p->b2) return ASF_ERR_INVALID_ARG;
  if (p->wdtype != ASF_F16 && p->wdtype != ASF_F32) return ASF_ERR_UNSUPPORTED;
  if (p->d <= 0 || p->r <= 0 || p->n <= 0) return ASF_ERR_INVALID_ARG;
  const int v = vec_of(p->wdtype);
  if (p->d % v || p->r % v) return ASF_ERR_MISALIGNED;
  if (!al16(p->W1) || !al16(p->W2) || !al4(p->b1) || !al4(p->b2)) return ASF_ERR_MISALIGNED;
  if ((size_t)p->d * esize(p->wdtype) > kSmemBudget || (size_t)p->r * 4 > kSmemBudget)
    return ASF_ERR_UNSUPPORTED;
  return ASF_OK;
}

L2Next l2_next_of(const asf_ffn *f) {
  L2Next nx{};
  for (int i = 0; i < 2; ++i) {
    const long long b = f->l2_next[i] ? (f->l2_next_bytes[i] & ~15ll) : 0;
    nx.p[i] = b > 0 ? static_cast<const unsigned char *>(f->l2_next[i]) : nullptr;
    nx.bytes[i] = b > 0 ? b : 0;
  }
  return nx;
}

asf_status check_ffn(const asf_ffn *f) {
  if (!f || !f->Wu || !f->WdT || !f->bias) return ASF_ERR_INVALID_ARG;
  if (f->wdtype != ASF_F16 && f->wdtype != ASF_F32) return ASF_ERR_UNSUPPORTED;
  if (f->act != ASF_ACT_RELU && f->act != ASF_ACT_REGLU) return ASF_ERR_UNSUPPORTED;
  if (f->act == ASF_ACT_REGLU && !f->Wg) return ASF_ERR_INVALID_ARG;
  if (f->d <= 0 || f->n <= 0) return ASF_ERR_INVALID_ARG;
  if (f->d % vec_of(f->wdtype)) return ASF_ERR_MISALIGNED;
  if (f->row_stride < 0 || (f->row_stride > 0 && f->row_stride < f->d)) return ASF_ERR_INVALID_ARG;
  if (f->row_stride % vec_of(f->wdtype)) return ASF_ERR_MISALIGNED;
  if (f->hot_rows < 0) return ASF_ERR_INVALID_ARG;
  for (int i = 0; i < 2; ++i) {
    if (f->l2_next_bytes[i] < 0) return ASF_ERR_INVALID_ARG;
    if (f->l2_next[i] && !al16(f->l2_next[i])) return ASF_ERR_MISALIGNED;
  }
  if ((size_t)f->d * esize(f->wdtype) > kSmemBudget) return ASF_ERR_UNSUPPORTED;
  if (down_tiles(f) > kMaxTiles) return ASF_ERR_UNSUPPORTED;
  if (!al16(f->Wu) || !al16(f->WdT) || (f->Wg && !al16(f->Wg)) || !al4(f->bias)) return ASF_ERR_MISALIGNED;
  return ASF_OK;
}

asf_status check_ws(void *ws, size_t ws_bytes, size_t need) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return ASF_ERR_WORKSPACE;
  if (ws_bytes < need) return ASF_ERR_WORKSPACE;
  return ASF_OK;
}

inline asf_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ASF_OK : ASF_ERR_CUDA; }

// largest token group in {1, 2, 4, 8} not above B whose staging fits
int pick_nb(int B, size_t bytes_per_token) {
  int nb = 8;
  while (nb > 1 && (nb > B || (size_t)nb * bytes_per_token > kSmemBudget)) nb >>= 1;
  return nb;
}

// ---------------------------------------------------------------- predict --
template <typename T, int NB>
cudaError_t run_pred_l1(const asf_predictor *p, const void *x, int B, float *h, uint32_t *mask, cudaStream_t st) {
  const int sms = sm_count();
  const int rpc = (p->r + sms - 1) / sms;
  const int grid = (p->r + rpc - 1) / rpc;
  const size_t smem = (size_t)NB * p->d * sizeof(T);
  return launch(k_pred_l1<T, NB, (NB <= 2 ? 16 : 8)>, dim3(grid), dim3(kThreads), smem, st, (const T *)p->W1, p->b1,
                (const T *)x, p->d, p->r, B, rpc, h, mask, n_words_of(p->n));
}

template <typename T, int NB>
cudaError_t run_pred_l2(const asf_predictor *p, int B, float thr, const float *h, uint32_t *mask, int32_t *idx,
                        int32_t *count, Header *hdr, cudaStream_t st) {
  const int sms = sm_count();
  const int rpc = (p->n + sms - 1) / sms;
  const int grid = (p->n + rpc - 1) / rpc;
  const size_t smem = (size_t)NB * p->r * 4 + ((size_t)rpc / 32 + 2) * 4;
  return launch(k_pred_l2<T, NB, (NB <= 2 ? 4 : 2), (NB <= 2 ? 4 : 2)>, dim3(grid), dim3(kThreads), smem, st, (const T *)p->W2, p->b2, h, p->r,
                p->n, B, thr, rpc, mask, n_words_of(p->n), idx, count, hdr, 1);
}

constexpr size_t kRingChunk = 32 * 1024;    // bytes per bulk copy of a ring slot
// Shared memory of the layer-2 ring: with the register-streaming layer-1
// kernel (one token group of x) it fits beside the previous layer's sparse
// FFN tail, and it holds most of a CTA's W2 slice.  (A 200 KB ring, holding
// more of the slice before the wait, measured 1.5-4% slower end to end.)
constexpr size_t kRing2Budget = 136 * 1024;

// rows per chunk and slots for a ring over rows of row_bytes within budget
bool ring_shape(size_t row_bytes, size_t vec_bytes, size_t budget, int rpc, int &CR, int &NSL) {
  CR = (int)std::max<size_t>(1, kRingChunk / row_bytes);
  CR = std::min(CR, std::max(1, rpc));
  const int chunks = (rpc + CR - 1) / CR;        // slots that would hold the whole slice
  for (NSL = std::min(8, std::max(chunks, 2)); NSL >= 2; --NSL)
    if (ring_layout(NSL, CR, 1, (int)row_bytes, vec_bytes).total <= budget) return true;
  return false;
}

// Ring of the layer-2 kernel.  Given the shared memory the layer-1 kernel
// leaves free on an SM (beside > 0: layer 1 holds its W1 slice in shared
// memory), three or more slots of at least 16 KB within it, so that the
// layer-2 CTAs are resident, and their first W2 pieces in flight, while layer
// 1 still runs; otherwise the 136 KB ring of 32 KB pieces, which becomes
// resident as layer 1's CTAs exit.
bool pred2_ring_shape(size_t row_bytes, size_t vec_bytes, size_t beside, int rpc, int &CR, int &NSL) {
  const size_t fixed = ring_layout(8, 0, 1, 1, vec_bytes).total + 128;
  if (beside > fixed) {
    int cr = (int)std::min<size_t>(kRingChunk / row_bytes, (beside - fixed) / (3 * row_bytes));
    cr = std::min(cr, std::max(1, rpc));
    if (cr >= 1 && (size_t)cr * row_bytes >= 16 * 1024) {
      const int chunks = (rpc + cr - 1) / cr;
      for (int nsl = std::min(8, std::max(chunks, 2)); nsl >= 3; --nsl)
        if (ring_layout(nsl, cr, 1, (int)row_bytes, vec_bytes).total <= beside) {
          CR = cr;
          NSL = nsl;
          return true;
        }
    }
  }
  return ring_shape(row_bytes, vec_bytes, kRing2Budget, rpc, CR, NSL);
}

template <typename T, int NB>
cudaError_t run_pred2_ring(const asf_predictor *p, int B, float thr, const float *h, uint32_t *mask, int32_t *idx,
                           int32_t *count, Header *hdr, cudaStream_t st, bool &used, const HotBlock &hot,
                           size_t beside) {
  const int sms = sm_count();
  const int rpc = (p->n + sms - 1) / sms;
  const int grid = (p->n + rpc - 1) / rpc;
  const size_t vec = pred2_vec_bytes(NB, p->r, rpc);
  int CR, NSL;
  used = pred2_ring_shape((size_t)p->r * sizeof(T), vec, beside, rpc, CR, NSL);
  if (!used) return cudaSuccess;
  const size_t smem = ring_layout(NSL, CR, p->r, (int)sizeof(T), vec).total;
  (void)idx;
  (void)count;
  return launch(k_pred2_ring<T, NB>, dim3(grid), dim3((kRingWarps + 1) * kWarp), smem, st, (const T *)p->W2,
                p->b2, h, p->r, p->n, B, thr, rpc, CR, NSL, mask, hdr, hot);
}

// largest token group in {1, 2, 4, 8} covering B (B <= 8)
inline int nb_cover(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : 8; }

template <typename T>
cudaError_t pred2_ring_any(const asf_predictor *p, int B, float thr, const float *h, uint32_t *mask, int32_t *idx,
                           int32_t *count, Header *hdr, cudaStream_t st, bool &used, const HotBlock &hot,
                           size_t beside) {
  switch (nb_cover(B)) {
    case 1: return run_pred2_ring<T, 1>(p, B, thr, h, mask, idx, count, hdr, st, used, hot, beside);
    case 2: return run_pred2_ring<T, 2>(p, B, thr, h, mask, idx, count, hdr, st, used, hot, beside);
    case 4: return run_pred2_ring<T, 4>(p, B, thr, h, mask, idx, count, hdr, st, used, hot, beside);
    default: return run_pred2_ring<T, 8>(p, B, thr, h, mask, idx, count, hdr, st, used, hot, beside);
  }
}

// Shared memory of k_pred_l1_smem: the row barriers, the W1 slice of rpc
// rows and NB tokens of x.
constexpr size_t kPred1SmemMax = 226 * 1024;
size_t pred1_smem_bytes(const asf_predictor *p, int rpc, int NB) {
  return (size_t)kPred1SmemRows * 8 + ((size_t)rpc + NB) * p->d * esize(p->wdtype);
}

// Token group of layer 1 on the shared-memory slice kernel, or 0 when layer 1
// stays on the register-streaming kernel: rows of at most 8 KB load into
// registers before the wait there (a 16 x 16-byte chunk per lane), and that
// kernel, 16 KB of shared memory at one token, sits beside the previous
// layer's sparse FFN.
int pred1_smem_nb(const asf_predictor *p, int B) {
  const int sms = sm_count();
  const int rpc = (p->r + sms - 1) / sms;
  if (rpc > kPred1SmemRows || (size_t)p->d * esize(p->wdtype) <= 8192) return 0;
  int nb = 8;
  while (nb > 1 && (nb > B || pred1_smem_bytes(p, rpc, nb) > kPred1SmemMax)) nb >>= 1;
  return pred1_smem_bytes(p, rpc, nb) <= kPred1SmemMax ? nb : 0;
}

template <typename T, int NB>
cudaError_t run_pred_l1_smem(const asf_predictor *p, const void *x, int B, float *h, uint32_t *mask, int32_t *err,
                             cudaStream_t st) {
  const int sms = sm_count();
  const int rpc = (p->r + sms - 1) / sms;
  const int grid = (p->r + rpc - 1) / rpc;
  return launch(k_pred_l1_smem<T, NB>, dim3(grid), dim3(kPred1Warps * kWarp), pred1_smem_bytes(p, rpc, NB), st,
                (const T *)p->W1, p->b1, (const T *)x, p->d, p->r, B, rpc, h, mask, n_words_of(p->n), err);
}

template <typename T>
cudaError_t pred1_reg_any(const asf_predictor *p, const void *x, int B, float *h, uint32_t *mask, int32_t *err,
                          cudaStream_t st) {
  switch (pred1_smem_nb(p, B)) {
    case 1: return run_pred_l1_smem<T, 1>(p, x, B, h, mask, err, st);
    case 2: return run_pred_l1_smem<T, 2>(p, x, B, h, mask, err, st);
    case 4: return run_pred_l1_smem<T, 4>(p, x, B, h, mask, err, st);
    case 8: return run_pred_l1_smem<T, 8>(p, x, B, h, mask, err, st);
    default: break;
  }
  switch (pick_nb(B, (size_t)p->d * sizeof(T))) {
    case 1: return run_pred_l1<T, 1>(p, x, B, h, mask, st);
    case 2: return run_pred_l1<T, 2>(p, x, B, h, mask, st);
    case 4: return run_pred_l1<T, 4>(p, x, B, h, mask, st);
    default: return run_pred_l1<T, 8>(p, x, B, h, mask, st);
  }
}

template <typename T>
cudaError_t pred2_reg_any(const asf_predictor *p, int B, float thr, const float *h, uint32_t *mask, int32_t *idx,
                          int32_t *count, Header *hdr, cudaStream_t st) {
  switch (pick_nb(B, (size_t)p->r * 4)) {
    case 1: return run_pred_l2<T, 1>(p, B, thr, h, mask, idx, count, hdr, st);
    case 2: return run_pred_l2<T, 2>(p, B, thr, h, mask, idx, count, hdr, st);
    case 4: return run_pred_l2<T, 4>(p, B, thr, h, mask, idx, count, hdr, st);
    default: return run_pred_l2<T, 8>(p, B, thr, h, mask, idx, count, hdr, st);
  }
}

// Whether layer 2 of B tokens runs the bulk-copy ring kernel, which leaves the
// union mask for a compaction step (batches of up to 8 tokens whose W2 slice
// fits the ring); otherwise the register-streaming kernel compacts itself.
template <typename T>
bool pred_leaves_mask(const asf_predictor *p, int B) {
  if (n_words_of(p->n) > kCompactThreads * kCompactWords) return false;
  const int sms = sm_count();
  const int rpc = (p->n + sms - 1) / sms;
  int CR, NSL;
  return ring_shape((size_t)p->r * sizeof(T), pred2_vec_bytes(nb_cover(std::min(B, 8)), p->r, rpc), kRing2Budget,
                    rpc, CR, NSL);
}

constexpr size_t kSmSmem = 228 * 1024;        // shared memory of one SM
constexpr size_t kCtaSmemReserve = 1024;      // the driver's share per resident CTA

// Shared memory the layer-1 slice kernel of a batch of B leaves free on its SM
// for the layer-2 ring (0 when layer 1 runs the register-streaming kernel).
size_t pred2_beside_budget(const asf_predictor *p, int B) {
  const int nb = pred1_smem_nb(p, B);
  if (!nb) return 0;
  const int sms = sm_count();
  const int rpc1 = (p->r + sms - 1) / sms;
  const size_t used = pred1_smem_bytes(p, rpc1, nb) + 1536 + 2 * kCtaSmemReserve;   // + static, reserves
  return used < kSmSmem ? kSmSmem - used : 0;
}

// Layer 1 (register-streaming kernel, token groups of up to 8), then layer 2:
// the bulk-copy ring kernel, once per group of up to 8 tokens -- the union is
// an OR over tokens, so every group ORs into the same mask -- followed by the
// compaction kernel, when the slice fits the ring; otherwise the
// register-streaming layer-2 kernel, which compacts in its last CTA.
template <typename T>
cudaError_t predict_layers(const asf_predictor *p, const void *x, int B, float thr, int32_t *idx, int32_t *count,
                           Header *hdr, uint32_t *mask, float *h, cudaStream_t st, bool &mask_only,
                           const HotBlock &hot = HotBlock()) {
  mask_only = pred_leaves_mask<T>(p, B);
  cudaError_t e = pred1_reg_any<T>(p, x, B, h, mask, &hdr->err, st);
  if (e != cudaSuccess) return e;
  if (mask_only) {
    const size_t beside = pred2_beside_budget(p, B);
    for (int g0 = 0; g0 < B && e == cudaSuccess; g0 += 8) {
      bool used = false;
      e = pred2_ring_any<T>(p, std::min(8, B - g0), thr, h + (size_t)g0 * p->r, mask, idx, count, hdr, st, used,
                            g0 == 0 ? hot : HotBlock(), beside);
      if (e == cudaSuccess && !used) e = cudaErrorInvalidConfiguration;   // pred_leaves_mask said it fits
    }
    return e;
  }
  return pred2_reg_any<T>(p, B, thr, h, mask, idx, count, hdr, st);
}

cudaError_t launch_compact(const asf_predictor *p, const uint32_t *mask, int32_t *idx, int32_t *count,
                           cudaStream_t st) {
  return launch(k_compact, dim3(1), dim3(kCompactThreads), 0, st, mask, n_words_of(p->n), idx, count);
}

template <typename T>
asf_status predict_t(const asf_predictor *p, const void *x, int B, float thr, int32_t *idx, int32_t *count,
                     void *ws, cudaStream_t st) {
  unsigned char *base = static_cast<unsigned char *>(ws);
  Header *hdr = reinterpret_cast<Header *>(base);
  uint32_t *mask = reinterpret_cast<uint32_t *>(base + kHeaderBytes);
  float *h = reinterpret_cast<float *>(base + kHeaderBytes + mask_region(p));
  bool mask_only = false;
  cudaError_t e = predict_layers<T>(p, x, B, thr, idx, count, hdr, mask, h, st, mask_only);
  if (e == cudaSuccess && mask_only) e = launch_compact(p, mask, idx, count, st);
  return cuda_status(e);
}

// ------------------------------------------------------------------- ffn --
template <typename T, int NB>
cudaError_t run_gu(const asf_ffn *f, const void *x, int B, const int32_t *idx, const int32_t *count, float *a,
                   int32_t *err, cudaStream_t st) {
  const int grid = 2 * sm_count();
  const size_t smem = (size_t)NB * f->d * sizeof(T);
  if (f->act == ASF_ACT_REGLU)
    return launch(k_ffn_gu<T, NB, (NB <= 2 ? 8 : 4), true>, dim3(grid), dim3(kThreads), smem, st, (const T *)f->Wg,
                  (const T *)f->Wu, f->bias, (const T *)x, f->d, ffn_rs(f), f->n, B, idx, count, a, err);
  return launch(k_ffn_gu<T, NB, (NB <= 2 ? 8 : 4), false>, dim3(grid), dim3(kThreads), smem, st, (const T *)f->Wg,
                (const T *)f->Wu, f->bias, (const T *)x, f->d, ffn_rs(f), f->n, B, idx, count, a, err);
}

template <typename T, int NB>
cudaError_t run_down(const asf_ffn *f, int B, const int32_t *idx, const int32_t *count, const float *a, float *part,
                     float *y, Header *hdr, cudaStream_t st) {
  constexpr int TW = kWarp * Vec<T>::N;
  const int ct = down_tiles(f);
  const int S = down_splits(f);
  const size_t smem = (size_t)kWarps * NB * TW * 4;
  return launch(k_ffn_down<T, NB, 4>, dim3(ct, S), dim3(kThreads), smem, st, (const T *)f->WdT, a, idx, count,
                f->d, ffn_rs(f), f->n, B, S, part, y, hdr, 1, l2_next_of(f));
}

// ------------------------------------------------------- final reduce --
// The FFN's last kernel sums its partials into y; in a neuron-sharded layer
// (grp != nullptr) it also exchanges the ranks' sums over peer memory.
struct Exchange {
  const asf_peer_group *grp = nullptr;
  int32_t *err = nullptr;
};

PeerPtrs peer_ptrs(const asf_peer_group *g) {
  PeerPtrs pp{};
  for (int r = 0; r < g->world; ++r) {
    pp.pub[r] = g->pub[r];
    pp.flag[r] = g->flag[r];
  }
  return pp;
}

cudaError_t launch_final_reduce(const float *part, int G, int B, int d, float *y, const Exchange &ex,
                                cudaStream_t st) {
  if (!ex.grp) {
    const int sms = sm_count();
    const int vec = (long long)((d + kWarp - 1) / kWarp) * B <= sms ? 1 : 4;
    const dim3 grid((d + kWarp * vec - 1) / (kWarp * vec), B);
    if (vec == 1) return launch(k_reduce_partials<1>, grid, dim3(kReduceWarps * kWarp), 0, st, part, G, B, d, y);
    return launch(k_reduce_partials<4>, grid, dim3(kReduceWarps * kWarp), 0, st, part, G, B, d, y);
  }
  const asf_peer_group *g = ex.grp;
  return launch(k_reduce_exchange, dim3((d + kWarp - 1) / kWarp, B, 1), dim3(kReduceWarps * kWarp), 0, st, part,
                0ll, G, B, d, (int)g->max_batch, peer_ptrs(g), g->epoch, y, 0ll, (int)g->world, (int)g->rank, ex.err);
}

// ------------------------------------------------------ tensor-core ffn --
// fp16 batches of 5..32 tokens: gate/up on tcgen05 in launches of 16 tokens
// (one pass over the rows for B <= 16, two for B <= 32) writing the
// activations as fp16 hi/lo pairs, then the down projection on tcgen05 over
// the same list, and the fixed-order sum of its list splits.  Batches of up
// to 4 the one-kernel FFN cannot hold (B >= 3 at d = 8192) stay on the CUDA
// cores: a 16-token MMA tile would be at most a quarter used, and the
// CUDA-core pair measured about twice as fast there.
bool tc_ok(const asf_ffn *f, int B) { return f->wdtype == ASF_F16 && B > 4 && B <= ASF_MAX_BATCH; }

// cuTensorMapEncodeTiled, from the driver through the runtime (no link to the
// driver library).
using TmapEncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
TmapEncodeFn tmap_encoder() {
  static TmapEncodeFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (TmapEncodeFn) nullptr;
    return reinterpret_cast<TmapEncodeFn>(p);
  }();
  return fn;
}

// Map of `rows` fp16 rows of d elements, `stride` elements apart, read in boxes
// of box_cols columns x box_rows rows (box_cols * 2 bytes = the swizzle span:
// the 128-byte swizzle for 64 columns, the 64-byte one for 32); out-of-range
// rows and columns read as zeros, L2 filled from DRAM in 256-byte pieces.
bool fp16_rows_map(CUtensorMap *tm, const void *base, int d, long long rows, long long stride, int box_rows,
                   int box_cols = kTcK) {
  TmapEncodeFn enc = tmap_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)stride * sizeof(__half)};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz = box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool REGLU>
cudaError_t launch_gu_tc(const asf_ffn *f, const __half *x, int Bh, int Btot, int g0, const int32_t *idx,
                         const int32_t *count, float *a, __half *a2, Header *hdr, cudaStream_t st) {
  // TMA gathers for ReGLU rows longer than 8 KB (measured: +16-19% at d = 8192,
  // 2-14% slower at d = 4096); the cp.async gathers otherwise
  const int use_tma = REGLU && (size_t)f->d * sizeof(__half) > 8192;
  CUtensorMap tmg, tmu, tmx;
  std::memset(&tmg, 0, sizeof(tmg));
  std::memset(&tmu, 0, sizeof(tmu));
  std::memset(&tmx, 0, sizeof(tmx));
  if (use_tma && (!fp16_rows_map(&tmg, f->Wg, f->d, f->n, ffn_rs(f), 1) ||
                  !fp16_rows_map(&tmu, f->Wu, f->d, f->n, ffn_rs(f), 1) ||
                  !fp16_rows_map(&tmx, x, f->d, Bh, f->d, kTcN)))
    return cudaErrorInvalidValue;
  return launch(k_gu_tc<kTcN, REGLU>, dim3(std::min(sm_count(), kMaxGrid)), dim3(9 * kWarp),
                GuTc<kTcN, REGLU>::SMEM, st, tmg, tmu, tmx, use_tma, (const __half *)f->Wg, (const __half *)f->Wu,
                f->bias, x, f->d, ffn_rs(f), f->n, Bh, idx, count, a, a2, Btot, g0, hdr);
}

template <int NG>
cudaError_t launch_down_tc(const asf_ffn *f, int B, const int32_t *idx, const int32_t *count, const __half *a2,
                           float *part, Header *hdr, cudaStream_t st) {
  const int R = tc_ranges(f), S = tc_splits(f);
  const int grid = std::min(std::min(sm_count(), kMaxGrid), R * S);
  // a2 as rows of 32 fp16 (64 bytes, 64-byte swizzle): chunk q, token group g at rows (q * NG + g) * 16
  CUtensorMap tmw, tma;
  const long long a2_rows = (long long)((f->n + kTcChunk - 1) / kTcChunk) * NG * 16;
  if (!fp16_rows_map(&tmw, f->WdT, f->d, f->n, ffn_rs(f), 1) ||
      !fp16_rows_map(&tma, a2, kTcChunk, a2_rows, kTcChunk, 16, kTcChunk))
    return cudaErrorInvalidValue;
  return launch(k_down_tc<NG>, dim3(grid), dim3(9 * kWarp), DnTc<NG>::SMEM, st, tmw, tma, idx, count, f->d, f->n, B,
                R, S, part, hdr);
}

cudaError_t run_tc(const asf_ffn *f, const void *x, int B, const int32_t *idx, const int32_t *count, float *y,
                   Header *hdr, unsigned char *scratch, cudaStream_t st, const Exchange &ex) {
  __half *a2 = reinterpret_cast<__half *>(scratch);
  float *part = reinterpret_cast<float *>(scratch + tc_a2_bytes(f, B));
  const bool reglu = f->act == ASF_ACT_REGLU;
  cudaError_t e = cudaSuccess;
  for (int g0 = 0; g0 < B && e == cudaSuccess; g0 += kTcN) {
    const int Bh = std::min(kTcN, B - g0);
    const __half *xg = static_cast<const __half *>(x) + (size_t)g0 * f->d;
    e = reglu ? launch_gu_tc<true>(f, xg, Bh, B, g0, idx, count, nullptr, a2, hdr, st)
              : launch_gu_tc<false>(f, xg, Bh, B, g0, idx, count, nullptr, a2, hdr, st);
  }
  if (e != cudaSuccess) return e;
  switch (tc_groups(B)) {
    case 1: e = launch_down_tc<1>(f, B, idx, count, a2, part, hdr, st); break;
    case 2: e = launch_down_tc<2>(f, B, idx, count, a2, part, hdr, st); break;
    case 3: e = launch_down_tc<3>(f, B, idx, count, a2, part, hdr, st); break;
    default: e = launch_down_tc<4>(f, B, idx, count, a2, part, hdr, st); break;
  }
  if (e != cudaSuccess) return e;
  return launch_final_reduce(part, tc_splits(f), B, f->d, y, ex, st);
}

// ------------------------------------------------------------- fused ffn --
int fused_maxq(const asf_ffn *f) {
  const int nvec = f->d / vec_of(f->wdtype);
  const int q = (nvec + kFusedWarps * kWarp - 1) / (kFusedWarps * kWarp);
  return q <= 1 ? 1 : q <= 2 ? 2 : q <= 4 ? 4 : q <= 6 ? 6 : 0;
}
int fused_nb(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : 0; }

// One CTA per SM (the ring's shared memory keeps a second one off each SM).
int fused_grid() { return std::min(sm_count(), kMaxGrid); }

// Most list positions one CTA of the grid takes.
int fused_nl_max(const asf_ffn *f) { return (f->n + fused_grid() - 1) / fused_grid(); }

// Ring slots that fit the shared-memory budget (0 if fewer than two).
int fused_slots(const asf_ffn *f, int NB, int mask_words) {
  const int M = f->act == ASF_ACT_REGLU ? 3 : 2;
  for (int ns = 16; ns >= 2; --ns)
    if (fused_layout(ns, f->d, M, esize(f->wdtype), NB, fused_nl_max(f), mask_words).total <= kFusedSmemDefault)
      return ns;
  return 0;
}

bool fused_ok(const asf_ffn *f, int B) {
  const int nb = fused_nb(B), q = fused_maxq(f);
  if (!nb || !q) return false;
  if (q * vec_of(f->wdtype) * nb > 64) return false;   // y accumulators per lane
  return fused_slots(f, nb, 0) >= 2;
}

// The union mask the fused kernel ranks itself (combined predict + FFN call);
// mask == nullptr: the list comes from idx/count.
struct MaskList {
  const uint32_t *mask = nullptr;
  int n_words = 0;
  int32_t *idx_out = nullptr;
  int32_t *count_out = nullptr;
};

template <typename T, int NB, int MAXQ, bool REGLU>
cudaError_t run_fused_k(const asf_ffn *f, const void *x, int B, const int32_t *idx, const int32_t *count, float *part,
                        float *y, Header *hdr, cudaStream_t st, const MaskList &ml, const Exchange &ex) {
  if constexpr (MAXQ * Vec<T>::N * NB > 64) {
    return cudaErrorInvalidConfiguration;
  } else {
    const int M = REGLU ? 3 : 2;
    const int mw = ml.mask ? ml.n_words : 0;
    const int NS = fused_slots(f, NB, mw);
    const FusedLayout L = fused_layout(NS, f->d, M, (int)sizeof(T), NB, fused_nl_max(f), mw);
    const int threads = (kFusedWarps + 1) * kWarp;
    auto kern = k_sparse_ffn<T, NB, MAXQ, REGLU>;
    const int G = fused_grid();
    cudaError_t e = launch(kern, dim3(G), dim3(threads), L.total, st, (const T *)f->Wg, (const T *)f->Wu,
                           (const T *)f->WdT, f->bias, (const T *)x, f->d, f->n, B, idx, count, ml.mask,
                           ml.n_words, ml.idx_out, ml.count_out, NS,
                           idx ? std::max(0, f->hot_rows) : 0, ffn_rs(f), ffn_packed(f) ? 1 : 0, part,
                           y, hdr, l2_next_of(f), g_inject.load(std::memory_order_relaxed));
    if (e != cudaSuccess) return e;
    return launch_final_reduce(part, G, B, f->d, y, ex, st);
  }
}

template <typename T, int NB, int MAXQ>
cudaError_t run_fused_a(const asf_ffn *f, const void *x, int B, const int32_t *idx, const int32_t *count, float *part,
                        float *y, Header *hdr, cudaStream_t st, const MaskList &ml, const Exchange &ex) {
  if (f->act == ASF_ACT_REGLU) return run_fused_k<T, NB, MAXQ, true>(f, x, B, idx, count, part, y, hdr, st, ml, ex);
  return run_fused_k<T, NB, MAXQ, false>(f, x, B, idx, count, part, y, hdr, st, ml, ex);
}

template <typename T, int NB>
cudaError_t run_fused_q(const asf_ffn *f, const void *x, int B, const int32_t *idx, const int32_t *count, float *part,
                        float *y, Header *hdr, cudaStream_t st, const MaskList &ml, const Exchange &ex) {
  switch (fused_maxq(f)) {
    case 1: return run_fused_a<T, NB, 1>(f, x, B, idx, count, part, y, hdr, st, ml, ex);
    case 2: return run_fused_a<T, NB, 2>(f, x, B, idx, count, part, y, hdr, st, ml, ex);
    case 4: return run_fused_a<T, NB, 4>(f, x, B, idx, count, part, y, hdr, st, ml, ex);
    default: return run_fused_a<T, NB, 6>(f, x, B, idx, count, part, y, hdr, st, ml, ex);
  }
}

template <typename T>
cudaError_t run_fused(const asf_ffn *f, const void *x, int B, const int32_t *idx, const int32_t *count, float *part,
                      float *y, Header *hdr, cudaStream_t st, const MaskList &ml, const Exchange &ex) {
  switch (fused_nb(B)) {
    case 1: return run_fused_q<T, 1>(f, x, B, idx, count, part, y, hdr, st, ml, ex);
    case 2: return run_fused_q<T, 2>(f, x, B, idx, count, part, y, hdr, st, ml, ex);
    default: return run_fused_q<T, 4>(f, x, B, idx, count, part, y, hdr, st, ml, ex);
  }
}

// The fused kernel can rank the predictor's mask itself: the mask's words
// still leave at least two ring slots.
bool fused_mask_ok(const asf_ffn *f, int B) {
  if (!fused_ok(f, B)) return false;
  if (n_words_of(f->n) > kRankWords * kFusedWarps * kWarp) return false;   // words per ranking thread
  return fused_slots(f, fused_nb(B), n_words_of(f->n)) >= 2;
}

// Sparse (idx != NULL), dense (idx == NULL) or mask-ranked (ml.mask) FFN.
// hdr: the workspace header; scratch: this call's part of the workspace.
template <typename T>
asf_status ffn_t(const asf_ffn *f, const void *x, int B, const int32_t *idx, const int32_t *count, float *y,
                 Header *hdr, unsigned char *scratch, cudaStream_t st, const MaskList &ml = MaskList(),
                 const Exchange &ex = Exchange()) {
  float *a = reinterpret_cast<float *>(scratch);
  float *part = reinterpret_cast<float *>(scratch + r256((size_t)f->n * B * 4));
  if (fused_ok(f, B)) {
    float *cpart = reinterpret_cast<float *>(scratch);
    return cuda_status(run_fused<T>(f, x, B, idx, count, cpart, y, hdr, st, ml, ex));
  }
  if (ml.mask) return ASF_ERR_UNSUPPORTED;   // callers check fused_mask_ok first
  if (tc_ok(f, B)) return cuda_status(run_tc(f, x, B, idx, count, y, hdr, scratch, st, ex));
  const int nbg = pick_nb(B, (size_t)f->d * sizeof(T));
  cudaError_t e;
  switch (nbg) {
    case 1: e = run_gu<T, 1>(f, x, B, idx, count, a, &hdr->err, st); break;
    case 2: e = run_gu<T, 2>(f, x, B, idx, count, a, &hdr->err, st); break;
    case 4: e = run_gu<T, 4>(f, x, B, idx, count, a, &hdr->err, st); break;
    default: e = run_gu<T, 8>(f, x, B, idx, count, a, &hdr->err, st); break;
  }
  if (e != cudaSuccess) return ASF_ERR_CUDA;
  const int nbd = std::min(B >= 8 ? 8 : (B >= 4 ? 4 : (B >= 2 ? 2 : 1)), 8);
  switch (nbd) {
    case 1: e = run_down<T, 1>(f, B, idx, count, a, part, y, hdr, st); break;
    case 2: e = run_down<T, 2>(f, B, idx, count, a, part, y, hdr, st); break;
    case 4: e = run_down<T, 4>(f, B, idx, count, a, part, y, hdr, st); break;
    default: e = run_down<T, 8>(f, B, idx, count, a, part, y, hdr, st); break;
  }
  // this path writes y itself: the exchange reads it back as a single partial
  if (e == cudaSuccess && ex.grp) e = launch_final_reduce(y, 1, B, f->d, y, ex, st);
  return cuda_status(e);
}

// The FFN rows of the descriptor's hot_rows leading neurons.
HotBlock hot_block_of(const asf_ffn *f) {
  HotBlock hb{};
  const int rows = std::min(std::max(0, f->hot_rows), f->n);
  if (rows == 0) return hb;
  const size_t es = esize(f->wdtype);
  if (ffn_packed(f)) {
    hb.p[0] = static_cast<const unsigned char *>(f->act == ASF_ACT_REGLU ? f->Wg : f->Wu);
    hb.bytes[0] = (long long)((size_t)rows * (size_t)ffn_rs(f) * es) & ~15ll;
    return hb;
  }
  const void *mats[3] = {f->act == ASF_ACT_REGLU ? f->Wg : nullptr, f->Wu, f->WdT};
  for (int i = 0; i < 3; ++i) {
    if (!mats[i]) continue;
    hb.p[i] = static_cast<const unsigned char *>(mats[i]);
    hb.bytes[i] = (long long)(((size_t)(rows - 1) * (size_t)ffn_rs(f) + (size_t)f->d) * es) & ~15ll;
  }
  return hb;
}

// One layer, predictor then sparse FFN.  Workspace: header | predictor
// scratch (mask, h) | FFN scratch.  When layer 2 leaves the union mask and the
// fused FFN can rank it, no compaction kernel runs: the FFN kernel builds its
// own part of the list from the mask and writes idx/count on the way.
// parts: kPartPredict enqueues the predictor's kernels, kPartFfn the rest
// (compaction if needed, the FFN); both together are the whole layer.
constexpr int kPartPredict = 1, kPartFfn = 2;
template <typename T>
asf_status predict_ffn_t(const asf_predictor *p, const asf_ffn *f, const void *x, int B, float thr, int32_t *idx,
                         int32_t *count, float *y, void *ws, cudaStream_t st, int parts,
                         const asf_peer_group *grp = nullptr) {
  unsigned char *base = static_cast<unsigned char *>(ws);
  Header *hdr = reinterpret_cast<Header *>(base);
  uint32_t *mask = reinterpret_cast<uint32_t *>(base + kHeaderBytes);
  float *h = reinterpret_cast<float *>(base + kHeaderBytes + mask_region(p));
  unsigned char *fs = base + kHeaderBytes + pred_scratch(p, B);
  bool mask_only = pred_leaves_mask<T>(p, B);
  if (parts & kPartPredict) {
    if (predict_layers<T>(p, x, B, thr, idx, count, hdr, mask, h, st, mask_only, hot_block_of(f)) != cudaSuccess)
      return ASF_ERR_CUDA;
  }
  if (!(parts & kPartFfn)) return ASF_OK;
  Exchange ex;
  ex.grp = grp;
  ex.err = &hdr->err;
  if (mask_only && fused_mask_ok(f, B)) {
    MaskList ml;
    ml.mask = mask;
    ml.n_words = n_words_of(p->n);
    ml.idx_out = idx;
    ml.count_out = count;
    return ffn_t<T>(f, x, B, nullptr, nullptr, y, hdr, fs, st, ml, ex);
  }
  if (mask_only && launch_compact(p, mask, idx, count, st) != cudaSuccess) return ASF_ERR_CUDA;
  return ffn_t<T>(f, x, B, idx, count, y, hdr, fs, st, MaskList(), ex);
}

template <typename T>
asf_status counts_t(const asf_ffn *f, const void *x, int Ttok, int64_t *counts, cudaStream_t st) {
  const int sms = sm_count();
  const int rpc = (f->n + sms - 1) / sms;
  const int grid = (f->n + rpc - 1) / rpc;
  const void *W = f->act == ASF_ACT_REGLU ? f->Wg : f->Wu;
  const int nb = pick_nb(8, (size_t)f->d * sizeof(T));
  const size_t smem = (size_t)nb * f->d * sizeof(T);
  cudaError_t e;
  switch (nb) {
    case 1: e = launch(k_act_counts<T, 1, 4>, dim3(grid), dim3(kThreads), smem, st, (const T *)W, f->bias, (const T *)x, f->d, ffn_rs(f), f->n, Ttok, rpc, counts); break;
    case 2: e = launch(k_act_counts<T, 2, 4>, dim3(grid), dim3(kThreads), smem, st, (const T *)W, f->bias, (const T *)x, f->d, ffn_rs(f), f->n, Ttok, rpc, counts); break;
    case 4: e = launch(k_act_counts<T, 4, 4>, dim3(grid), dim3(kThreads), smem, st, (const T *)W, f->bias, (const T *)x, f->d, ffn_rs(f), f->n, Ttok, rpc, counts); break;
    default: e = launch(k_act_counts<T, 8, 4>, dim3(grid), dim3(kThreads), smem, st, (const T *)W, f->bias, (const T *)x, f->d, ffn_rs(f), f->n, Ttok, rpc, counts); break;
  }
  return cuda_status(e);
}

}  // namespace

// ======================================================================== //
// scratch for asf_sparse_ffn_noalloc                                       //
// ======================================================================== //
// File-scope device scratch used instead of a caller workspace.  In host code
// the name is only a host-side stand-in; the device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ASF_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64] = {};

asf_status noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ASF_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ASF_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return ASF_OK;
}
}  // namespace

// ======================================================================== //
// C ABI                                                                    //
// ======================================================================== //
extern "C" {

int32_t asf_version(void) { return 106; }

const char *asf_status_string(asf_status s) {
  switch (s) {
    case ASF_OK: return "ok";
    case ASF_ERR_INVALID_ARG: return "invalid argument";
    case ASF_ERR_MISALIGNED: return "misaligned pointer or size";
    case ASF_ERR_UNSUPPORTED: return "unsupported configuration";
    case ASF_ERR_CUDA: return "CUDA error";
    case ASF_ERR_DEVICE_INDEX: return "device saw an index out of range";
    case ASF_ERR_TIMEOUT: return "bounded device wait timed out";
    case ASF_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

size_t asf_workspace_bytes(const asf_predictor *pred, const asf_ffn *ffn, int32_t max_batch) {
  if (max_batch < 1 || max_batch > ASF_MAX_BATCH) return 0;
  if (!pred && !ffn) return 0;
  size_t need = 0;
  if (pred && check_pred(pred) != ASF_OK) return 0;
  if (ffn && check_ffn(ffn) != ASF_OK) return 0;
  // both: room for the combined call, whose FFN scratch follows the predictor's
  if (pred) need += pred_scratch(pred, max_batch);
  if (ffn) need += ffn_scratch(ffn, max_batch);
  return kHeaderBytes + need;
}

asf_status asf_workspace_init(void *ws, size_t ws_bytes, asf_stream_t stream) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < kHeaderBytes) return ASF_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
}

asf_status asf_predict(const asf_predictor *pred, const void *x, int32_t B, float tau, int32_t *idx,
                       int32_t *count, void *ws, size_t ws_bytes, asf_stream_t stream) {
  asf_status s = check_pred(pred);
  if (s != ASF_OK) return s;
  if (!x || !idx || !count) return ASF_ERR_INVALID_ARG;
  if (B < 1 || B > ASF_MAX_BATCH) return ASF_ERR_INVALID_ARG;
  if (!(tau > 0.f && tau < 1.f)) return ASF_ERR_INVALID_ARG;
  if (!al16(x) || !al4(idx) || !al4(count)) return ASF_ERR_MISALIGNED;
  s = check_ws(ws, ws_bytes, kHeaderBytes + pred_scratch(pred, B));
  if (s != ASF_OK) return s;
  // sigmoid(z) > tau  <=>  z > log(tau / (1 - tau)), evaluated once in double
  const float thr = (float)std::log((double)tau / (1.0 - (double)tau));
  if (pred->wdtype == ASF_F16)
    return predict_t<__half>(pred, x, B, thr, idx, count, ws, (cudaStream_t)stream);
  return predict_t<float>(pred, x, B, thr, idx, count, ws, (cudaStream_t)stream);
}

asf_status asf_sparse_ffn(const asf_ffn *ffn, const void *x, int32_t B, const int32_t *idx, const int32_t *count,
                          float *y, void *ws, size_t ws_bytes, asf_stream_t stream) {
  asf_status s = check_ffn(ffn);
  if (s != ASF_OK) return s;
  if (!x || !idx || !count || !y) return ASF_ERR_INVALID_ARG;
  if (B < 1 || B > ASF_MAX_BATCH) return ASF_ERR_INVALID_ARG;
  if (!al16(x) || !al16(y) || !al4(idx) || !al4(count)) return ASF_ERR_MISALIGNED;
  s = check_ws(ws, ws_bytes, kHeaderBytes + ffn_scratch(ffn, B));
  if (s != ASF_OK) return s;
  Header *hdr = static_cast<Header *>(ws);
  unsigned char *scratch = static_cast<unsigned char *>(ws) + kHeaderBytes;
  if (ffn->wdtype == ASF_F16) return ffn_t<__half>(ffn, x, B, idx, count, y, hdr, scratch, (cudaStream_t)stream);
  return ffn_t<float>(ffn, x, B, idx, count, y, hdr, scratch, (cudaStream_t)stream);
}

}  // extern "C"

namespace {
asf_status check_group(const asf_peer_group *g, int d, int B) {
  if (!g) return ASF_ERR_INVALID_ARG;
  if (g->world < 1 || g->world > ASF_MAX_PEERS || g->rank < 0 || g->rank >= g->world) return ASF_ERR_INVALID_ARG;
  if (g->d != d || B < 1 || B > g->max_batch || g->max_batch > ASF_MAX_BATCH) return ASF_ERR_INVALID_ARG;
  if (!g->epoch || !al4(g->epoch)) return ASF_ERR_INVALID_ARG;
  for (int r = 0; r < g->world; ++r) {
    if (!g->pub[r] || !g->flag[r]) return ASF_ERR_INVALID_ARG;
    if (!al4(g->pub[r]) || !al4(g->flag[r])) return ASF_ERR_MISALIGNED;
  }
  return ASF_OK;
}

asf_status predict_sparse_ffn_parts(const asf_predictor *pred, const asf_ffn *ffn, const void *x, int32_t B,
                                    float tau, int32_t *idx, int32_t *count, float *y, void *ws, size_t ws_bytes,
                                    asf_stream_t stream, int parts, const asf_peer_group *grp = nullptr) {
  asf_status s = check_pred(pred);
  if (s != ASF_OK) return s;
  s = check_ffn(ffn);
  if (s != ASF_OK) return s;
  if (pred->d != ffn->d || pred->n != ffn->n || pred->wdtype != ffn->wdtype) return ASF_ERR_INVALID_ARG;
  if (!x || !idx || !count || !y) return ASF_ERR_INVALID_ARG;
  if (B < 1 || B > ASF_MAX_BATCH) return ASF_ERR_INVALID_ARG;
  if (!(tau > 0.f && tau < 1.f)) return ASF_ERR_INVALID_ARG;
  if (!al16(x) || !al16(y) || !al4(idx) || !al4(count)) return ASF_ERR_MISALIGNED;
  s = check_ws(ws, ws_bytes, kHeaderBytes + pred_scratch(pred, B) + ffn_scratch(ffn, B));
  if (s != ASF_OK) return s;
  if (grp) {
    s = check_group(grp, ffn->d, B);
    if (s != ASF_OK) return s;
  }
  const float thr = (float)std::log((double)tau / (1.0 - (double)tau));
  if (pred->wdtype == ASF_F16)
    return predict_ffn_t<__half>(pred, ffn, x, B, thr, idx, count, y, ws, (cudaStream_t)stream, parts, grp);
  return predict_ffn_t<float>(pred, ffn, x, B, thr, idx, count, y, ws, (cudaStream_t)stream, parts, grp);
}
}  // namespace

extern "C" {

asf_status asf_predict_sparse_ffn(const asf_predictor *pred, const asf_ffn *ffn, const void *x, int32_t B,
                                  float tau, int32_t *idx, int32_t *count, float *y, void *ws, size_t ws_bytes,
                                  asf_stream_t stream) {
  return predict_sparse_ffn_parts(pred, ffn, x, B, tau, idx, count, y, ws, ws_bytes, stream,
                                  kPartPredict | kPartFfn);
}

asf_status asf_predict_sparse_ffn_begin(const asf_predictor *pred, const asf_ffn *ffn, const void *x, int32_t B,
                                        float tau, int32_t *idx, int32_t *count, float *y, void *ws,
                                        size_t ws_bytes, asf_stream_t stream) {
  return predict_sparse_ffn_parts(pred, ffn, x, B, tau, idx, count, y, ws, ws_bytes, stream, kPartPredict);
}

asf_status asf_predict_sparse_ffn_end(const asf_predictor *pred, const asf_ffn *ffn, const void *x, int32_t B,
                                      float tau, int32_t *idx, int32_t *count, float *y, void *ws, size_t ws_bytes,
                                      asf_stream_t stream) {
  return predict_sparse_ffn_parts(pred, ffn, x, B, tau, idx, count, y, ws, ws_bytes, stream, kPartFfn);
}

asf_status asf_predict_sparse_ffn_exchange(const asf_predictor *pred, const asf_ffn *ffn, const void *x, int32_t B,
                                           float tau, int32_t *idx, int32_t *count, float *y, void *ws,
                                           size_t ws_bytes, const asf_peer_group *grp, asf_stream_t stream) {
  if (!grp) return ASF_ERR_INVALID_ARG;
  return predict_sparse_ffn_parts(pred, ffn, x, B, tau, idx, count, y, ws, ws_bytes, stream,
                                  kPartPredict | kPartFfn, grp);
}

asf_status asf_reduce_exchange(const float *part, int64_t part_rank_stride, int32_t G, int32_t B, int32_t d,
                               const asf_peer_group *grp, int32_t local_ranks, float *y, int64_t y_rank_stride,
                               void *ws, size_t ws_bytes, asf_stream_t stream) {
  if (!part || !y || G < 1 || G > kMaxGrid || d <= 0) return ASF_ERR_INVALID_ARG;
  asf_status s = check_group(grp, d, B);
  if (s != ASF_OK) return s;
  if (local_ranks != 1 && local_ranks != grp->world) return ASF_ERR_INVALID_ARG;
  if (local_ranks > 1 && grp->rank != 0) return ASF_ERR_INVALID_ARG;
  if (local_ranks > 1 && (part_rank_stride < (int64_t)G * B * d || y_rank_stride < (int64_t)B * d))
    return ASF_ERR_INVALID_ARG;
  if (!al4(part) || !al4(y)) return ASF_ERR_MISALIGNED;
  s = check_ws(ws, ws_bytes, kHeaderBytes);
  if (s != ASF_OK) return s;
  Header *hdr = static_cast<Header *>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  const dim3 grid((d + kWarp - 1) / kWarp, B, local_ranks);
  if (local_ranks == 1)
    return cuda_status(launch(k_reduce_exchange, grid, dim3(kReduceWarps * kWarp), 0, st, part, 0ll, (int)G, (int)B,
                              (int)d, (int)grp->max_batch, peer_ptrs(grp), grp->epoch, y, 0ll, (int)grp->world,
                              (int)grp->rank, &hdr->err));
  // every rank in this process: one cooperative launch, so that all blocks
  // are resident while they wait on one another
  int dev = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_reduce_exchange, kReduceWarps * kWarp, 0) !=
          cudaSuccess)
    return ASF_ERR_CUDA;
  if ((long long)grid.x * grid.y * grid.z > (long long)per_sm * sm_count()) return ASF_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kReduceWarps * kWarp);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, k_reduce_exchange, part, (long long)part_rank_stride, (int)G, (int)B,
                                        (int)d, (int)grp->max_batch, peer_ptrs(grp), grp->epoch, y,
                                        (long long)y_rank_stride, (int)grp->world, 0, &hdr->err));
}

asf_status asf_set_fault_injection(int32_t mode) {
  if (mode != ASF_INJECT_NONE && mode != ASF_INJECT_WITHHOLD_FFN_COPIES) return ASF_ERR_INVALID_ARG;
  g_inject.store(mode, std::memory_order_relaxed);
  return ASF_OK;
}

asf_status asf_dense_ffn(const asf_ffn *ffn, const void *x, int32_t B, float *y, void *ws, size_t ws_bytes,
                         asf_stream_t stream) {
  asf_status s = check_ffn(ffn);
  if (s != ASF_OK) return s;
  if (!x || !y) return ASF_ERR_INVALID_ARG;
  if (B < 1 || B > ASF_MAX_BATCH) return ASF_ERR_INVALID_ARG;
  if (!al16(x) || !al16(y)) return ASF_ERR_MISALIGNED;
  s = check_ws(ws, ws_bytes, kHeaderBytes + ffn_scratch(ffn, B));
  if (s != ASF_OK) return s;
  Header *hdr = static_cast<Header *>(ws);
  unsigned char *scratch = static_cast<unsigned char *>(ws) + kHeaderBytes;
  if (ffn->wdtype == ASF_F16) return ffn_t<__half>(ffn, x, B, nullptr, nullptr, y, hdr, scratch, (cudaStream_t)stream);
  return ffn_t<float>(ffn, x, B, nullptr, nullptr, y, hdr, scratch, (cudaStream_t)stream);
}

asf_status asf_activation_counts(const asf_ffn *ffn, const void *x, int32_t T, int64_t *counts, void *ws,
                                 size_t ws_bytes, asf_stream_t stream) {
  asf_status s = check_ffn(ffn);
  if (s != ASF_OK) return s;
  if (!x || !counts || T < 0) return ASF_ERR_INVALID_ARG;
  if (!al16(x) || (reinterpret_cast<uintptr_t>(counts) & 7u)) return ASF_ERR_MISALIGNED;
  s = check_ws(ws, ws_bytes, kHeaderBytes);
  if (s != ASF_OK) return s;
  if (T == 0) return ASF_OK;
  if (ffn->wdtype == ASF_F16) return counts_t<__half>(ffn, x, T, counts, (cudaStream_t)stream);
  return counts_t<float>(ffn, x, T, counts, (cudaStream_t)stream);
}

asf_status asf_hot_permutation(const int64_t *counts, int32_t n, int32_t *perm_out) {
  if (!counts || !perm_out || n < 0) return ASF_ERR_INVALID_ARG;
  std::vector<int32_t> order((size_t)n);
  for (int32_t i = 0; i < n; ++i) order[(size_t)i] = i;
  std::stable_sort(order.begin(), order.end(),
                   [counts](int32_t a, int32_t b) { return counts[a] > counts[b]; });
  std::memcpy(perm_out, order.data(), (size_t)n * sizeof(int32_t));
  return ASF_OK;
}

asf_status asf_permute_rows(const void *src, void *dst, int32_t n_rows, int64_t row_bytes, const int32_t *perm,
                            asf_stream_t stream) {
  if (!src || !dst || !perm || n_rows < 0 || row_bytes <= 0) return ASF_ERR_INVALID_ARG;
  if (src == dst) return ASF_ERR_INVALID_ARG;
  if (!al4(perm)) return ASF_ERR_MISALIGNED;
  if (n_rows == 0) return ASF_OK;
  int unit = 1;
  if (row_bytes % 16 == 0 && al16(src) && al16(dst))
    unit = 16;
  else if (row_bytes % 4 == 0 && al4(src) && al4(dst))
    unit = 4;
  const int grid = std::min(n_rows, 8 * sm_count());
  return cuda_status(launch(k_permute_rows, dim3(grid), dim3(kThreads), 0, (cudaStream_t)stream,
                            (const unsigned char *)src, (long long)row_bytes, (unsigned char *)dst,
                            (long long)row_bytes, (int)n_rows, (int)n_rows, (long long)row_bytes, perm, unit));
}

asf_status asf_gather_rows(const void *src, int64_t src_stride, int32_t src_rows, void *dst, int64_t dst_stride,
                           int32_t n_rows, int64_t row_bytes, const int32_t *perm, asf_stream_t stream) {
  if (!src || !dst || n_rows < 0 || src_rows < 0 || row_bytes <= 0) return ASF_ERR_INVALID_ARG;
  if (src_stride < row_bytes || dst_stride < row_bytes) return ASF_ERR_INVALID_ARG;
  if (!perm && n_rows > src_rows) return ASF_ERR_INVALID_ARG;
  if (perm && !al4(perm)) return ASF_ERR_MISALIGNED;
  // the source and destination row ranges must not overlap
  const char *s0 = static_cast<const char *>(src), *d0 = static_cast<const char *>(dst);
  const char *s1 = s0 + (size_t)(src_rows > 0 ? src_rows - 1 : 0) * src_stride + row_bytes;
  const char *d1 = d0 + (size_t)(n_rows > 0 ? n_rows - 1 : 0) * dst_stride + row_bytes;
  if (n_rows > 0 && src_rows > 0 && s0 < d1 && d0 < s1) return ASF_ERR_INVALID_ARG;
  if (n_rows == 0) return ASF_OK;
  int unit = 1;
  const auto a16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  const auto a4 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
  if (row_bytes % 16 == 0 && src_stride % 16 == 0 && dst_stride % 16 == 0 && a16(src) && a16(dst))
    unit = 16;
  else if (row_bytes % 4 == 0 && src_stride % 4 == 0 && dst_stride % 4 == 0 && a4(src) && a4(dst))
    unit = 4;
  const int grid = std::min(n_rows, 8 * sm_count());
  return cuda_status(launch(k_permute_rows, dim3(grid), dim3(kThreads), 0, (cudaStream_t)stream,
                            (const unsigned char *)src, (long long)src_stride, (unsigned char *)dst,
                            (long long)dst_stride, (int)n_rows, (int)src_rows, (long long)row_bytes, perm, unit));
}

asf_status asf_sparse_ffn_noalloc(const asf_ffn *ffn, const void *x, int32_t B, const int32_t *idx,
                                  const int32_t *count, float *y, int32_t *fault, asf_stream_t stream) {
  asf_status s = check_ffn(ffn);
  if (s != ASF_OK) return s;
  if (!x || !idx || !count || !y) return ASF_ERR_INVALID_ARG;
  if (B < 1 || B > ASF_MAX_BATCH) return ASF_ERR_INVALID_ARG;
  if (!al16(x) || !al16(y) || !al4(idx) || !al4(count) || (fault && !al4(fault))) return ASF_ERR_MISALIGNED;
  const size_t need = kHeaderBytes + ffn_scratch(ffn, B);
  if (need > (size_t)ASF_NOALLOC_SCRATCH_BYTES) return ASF_ERR_UNSUPPORTED;
  void *ws = nullptr;
  s = noalloc_scratch(&ws);
  if (s != ASF_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  // counters and the fault word must start at zero; the rest is overwritten
  if (cudaMemsetAsync(ws, 0, kHeaderBytes, st) != cudaSuccess) return ASF_ERR_CUDA;
  Header *hdr = static_cast<Header *>(ws);
  unsigned char *scratch = static_cast<unsigned char *>(ws) + kHeaderBytes;
  s = ffn->wdtype == ASF_F16 ? ffn_t<__half>(ffn, x, B, idx, count, y, hdr, scratch, st)
                             : ffn_t<float>(ffn, x, B, idx, count, y, hdr, scratch, st);
  if (s != ASF_OK) return s;
  if (fault && cudaMemcpyAsync(fault, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return ASF_ERR_CUDA;
  return ASF_OK;
}

asf_status asf_read_error(void *ws, int32_t *host_out, asf_stream_t stream) {
  if (!ws || !host_out) return ASF_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return ASF_ERR_WORKSPACE;
  int32_t v = 0;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return ASF_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(int32_t), st) != cudaSuccess) return ASF_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return ASF_ERR_CUDA;
  int32_t out = ASF_OK;
  if (v & kErrIndex)
    out = ASF_ERR_DEVICE_INDEX;
  else if (v & kErrTimeout)
    out = ASF_ERR_TIMEOUT;
  *host_out = out;
  return ASF_OK;
}

}  // extern "C"
