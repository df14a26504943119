/*
 * asffn.h -- C ABI of libasffn.so: activation-sparse FFN decode on B200 (sm_100a).
 *
 * The operations follow the problem statement of the pages on PowerInfer-style
 * neuron-level sparse inference:
 *   - predict(x) -> active index list: the online neuron predictor
 *     ("PowerInfer Guide: Exploiting Activation Sparsity for LLM AI", section 3
 *     "Adaptive Online Neuron Predictors", predictor equation and the Step 2
 *     predictor module), read as the 2-layer MLP of the "PowerInfer_x64" page
 *     ("Prediction and Caching"): h = ReLU(W1 x + b1), z = W2 h + b2,
 *     neuron k active iff sigmoid(z_k) > tau (strict), i.e. z_k > logit(tau).
 *   - sparse_ffn(x, idx) -> y: the neuron-aware sparse operator (PowerInfer
 *     Guide, section 4 "Neuron-Aware Sparse GPU Operators", and the FFN
 *     equation of "The Hidden Inefficiency") evaluated only for listed neurons.
 *   - activation counts + hot permutation: the offline profiler and hot/cold
 *     split (PowerInfer Guide, Step 1), used to store hot rows first.
 *
 * Conventions shared by every call:
 *   - All pointers named "device" are CUDA device pointers owned by the caller;
 *     the library never allocates or frees device memory and never keeps a
 *     pointer after a call returns (the descriptor structs are read at call
 *     time only).
 *   - Calls that take a stream enqueue work on it and return without
 *     synchronising (except asf_read_error).  Launch failures return
 *     ASF_ERR_CUDA; no call terminates the process.
 *   - Arguments are validated on the host before any launch; a call that
 *     returns an error has enqueued nothing.
 *   - Checks that need device data (an index outside [0, n), count > n) cannot
 *     be done on the host: the kernel skips the offending item and records the
 *     fault in the workspace error word, read with asf_read_error.
 *   - Weights, x and y must be 16-byte aligned; d and r must be multiples of 8
 *     (fp16) or 4 (fp32).  x has the weight dtype; y is always fp32.
 *   - Accumulation is fp32 throughout.
 */
#ifndef ASFFN_H
#define ASFFN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ASF_API __attribute__((visibility("default")))
#else
#define ASF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *asf_stream_t;

typedef enum {
  ASF_OK = 0,
  ASF_ERR_INVALID_ARG = 1,  /* null pointer, bad size, tau outside (0,1), ... */
  ASF_ERR_MISALIGNED = 2,   /* a pointer or row length breaks the alignment rule */
  ASF_ERR_UNSUPPORTED = 3,  /* dtype/activation/batch combination not built */
  ASF_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  ASF_ERR_DEVICE_INDEX = 5, /* device saw idx outside [0, n) or count > n */
  ASF_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up */
  ASF_ERR_WORKSPACE = 7     /* workspace missing, misaligned or too small */
} asf_status;

typedef enum { ASF_F32 = 0, ASF_F16 = 1 } asf_dtype;

/* ASF_ACT_RELU : y = W_down ReLU(W_up x + b)                  (up + down)
 * ASF_ACT_REGLU: y = W_down (ReLU(W_gate x + b) * (W_up x))   (gate, up, down) */
typedef enum { ASF_ACT_RELU = 0, ASF_ACT_REGLU = 1 } asf_act;

#define ASF_MAX_BATCH 32

/* Two-layer predictor, borrowed device pointers.  Row-major. */
typedef struct {
  int32_t d;          /* input width (hidden size) */
  int32_t r;          /* predictor hidden width */
  int32_t n;          /* number of FFN neurons (d_ffn) */
  asf_dtype wdtype;   /* dtype of W1, W2 and of x */
  const void *W1;     /* [r][d] */
  const float *b1;    /* [r] */
  const void *W2;     /* [n][r] */
  const float *b2;    /* [n] */
} asf_predictor;

/* One FFN layer, borrowed device pointers.  Row k of every matrix belongs to
 * neuron k in storage order (after any hot permutation). */
typedef struct {
  int32_t d;          /* hidden size */
  int32_t n;          /* number of neurons */
  asf_dtype wdtype;   /* dtype of Wg, Wu, WdT and of x */
  asf_act act;
  const void *Wg;     /* [n][d] gate rows (REGLU), NULL for RELU */
  const void *Wu;     /* [n][d] up rows */
  const void *WdT;    /* [n][d] W_down transposed: row k = column k of W_down */
  const float *bias;  /* [n] bias of the ReLU input: gate (REGLU) or up (RELU) */
  int32_t hot_rows;   /* rows 0..hot_rows-1 are active for most tokens (hot neurons stored
                         first by the offline permutation); asf_sparse_ffn prefetches them
                         into L2 while the list is still being predicted.  0 = no hint.
                         Affects speed only, never results. */
  int32_t row_stride; /* elements between consecutive rows of Wg/Wu/WdT; 0 means d.  With
                         row_stride = m*d and Wu = Wg + d, WdT = Wu + d (REGLU; for RELU
                         WdT = Wu + d) the layer is in the neuron-major packed layout
                         (gate|up|down of a neuron contiguous, see asf_gather_rows), and the
                         sparse FFN fetches each neuron with one bulk copy. */
  const void *l2_next[2];      /* optional L2 prefetch hint: up to two device ranges that are
                                  read soon after this call (for example the next layer's
                                  predictor W1 and W2).  The call's last kernel pulls them into
                                  L2 while it waits for the sparse FFN, whose row stream does
                                  not keep HBM busy on its own.  Each non-NULL range must be
                                  16-byte aligned and mapped for l2_next_bytes[i] bytes (the
                                  tail below a multiple of 16 is skipped).  NULL / 0 = none.
                                  Affects speed only, never results. */
  int64_t l2_next_bytes[2];
} asf_ffn;

/* Bytes of device workspace needed by asf_predict / asf_sparse_ffn /
 * asf_dense_ffn / asf_activation_counts for batches up to max_batch.  Either
 * descriptor may be NULL; with both, the size also serves
 * asf_predict_sparse_ffn (the two scratch areas side by side).  Returns 0 on
 * invalid arguments. */
ASF_API size_t asf_workspace_bytes(const asf_predictor *pred, const asf_ffn *ffn, int32_t max_batch);

/* Zero a freshly allocated workspace (256-byte aligned device buffer).  Must be
 * called once before first use; afterwards every call leaves the workspace's
 * counters at zero again.  One workspace serves one stream at a time. */
ASF_API asf_status asf_workspace_init(void *ws, size_t ws_bytes, asf_stream_t stream);

/* Online predictor for B tokens (1 <= B <= ASF_MAX_BATCH).
 *   x     device [B][d], wdtype
 *   tau   threshold on sigmoid(z), 0 < tau < 1
 *   idx   device int32 [n]: on completion idx[0..count) holds the ascending
 *         storage indices of the neurons predicted active for at least one of
 *         the B tokens (the union); entries past count are left untouched
 *   count device int32 [1]
 * Stays on the device: no host synchronisation. */
ASF_API asf_status asf_predict(const asf_predictor *pred, const void *x, int32_t B, float tau,
                       int32_t *idx, int32_t *count, void *ws, size_t ws_bytes,
                       asf_stream_t stream);

/* Sparse FFN over an index list, every token over the same list.
 *   x     device [B][d], wdtype
 *   idx   device int32 [n]; the first *count entries are used (any order,
 *         duplicates are summed twice); entries outside [0, n) are skipped and
 *         flagged
 *   count device int32 [1], 0 <= *count <= n (larger is clamped and flagged)
 *   y     device fp32 [B][d], overwritten: y_b = sum_j a_{idx_j, b} WdT[idx_j]
 *         with a = ReLU(gate + bias) * up  (REGLU)  or  ReLU(up + bias)  (RELU) */
ASF_API asf_status asf_sparse_ffn(const asf_ffn *ffn, const void *x, int32_t B, const int32_t *idx,
                          const int32_t *count, float *y, void *ws, size_t ws_bytes,
                          asf_stream_t stream);

/* One layer of the decode path in one call: asf_predict followed by
 * asf_sparse_ffn over the predicted list (the predictor-then-sparse-operator
 * flow of the PowerInfer Guide, Step 2 predictor module feeding the Step 3
 * sparse FFN, and the PowerInfer_x64 page's "Prediction and Caching"), with
 * the same results (idx, count and y bit for bit).  For B <= 4 the sparse FFN kernel ranks the predictor's
 * union mask itself, so no separate compaction kernel or index-list round
 * trip sits between the two; larger batches run the two calls' kernels.
 *   pred, ffn   descriptors of the same layer: equal d, n and wdtype
 *   x, B, tau   as for asf_predict
 *   idx, count  outputs as for asf_predict (the list the FFN used)
 *   y           output as for asf_sparse_ffn
 *   ws          at least asf_workspace_bytes(pred, ffn, B) bytes */
ASF_API asf_status asf_predict_sparse_ffn(const asf_predictor *pred, const asf_ffn *ffn, const void *x,
                                          int32_t B, float tau, int32_t *idx, int32_t *count, float *y,
                                          void *ws, size_t ws_bytes, asf_stream_t stream);

/* The same layer in two halves, for callers that put other work or timing
 * events between the predictor and the sparse FFN.  Called in this order on
 * one stream with identical arguments, _begin then _end enqueue exactly the
 * kernels of asf_predict_sparse_ffn and give the same idx, count and y bit for
 * bit.  _begin runs the predictor and leaves its result (the union mask, or
 * for B > 8 the list itself) in the workspace; _end compacts the mask when
 * needed and runs the sparse FFN.  Nothing else may use the workspace between
 * the two.  Arguments, validation and errors as for asf_predict_sparse_ffn. */
ASF_API asf_status asf_predict_sparse_ffn_begin(const asf_predictor *pred, const asf_ffn *ffn, const void *x,
                                                int32_t B, float tau, int32_t *idx, int32_t *count, float *y,
                                                void *ws, size_t ws_bytes, asf_stream_t stream);
ASF_API asf_status asf_predict_sparse_ffn_end(const asf_predictor *pred, const asf_ffn *ffn, const void *x,
                                              int32_t B, float tau, int32_t *idx, int32_t *count, float *y,
                                              void *ws, size_t ws_bytes, asf_stream_t stream);

/* Dense FFN over all n neurons (the unsparsified reference, same kernels with an
 * implicit identity index list).  Arguments as asf_sparse_ffn. */
ASF_API asf_status asf_dense_ffn(const asf_ffn *ffn, const void *x, int32_t B, float *y, void *ws,
                         size_t ws_bytes, asf_stream_t stream);

/* Offline profiler: counts[k] += number of the T tokens of x (device [T][d])
 * whose ReLU input (gate + bias for REGLU, up + bias for RELU) is > 0.
 * counts: device int64 [n], accumulated so calibration can be chunked. */
ASF_API asf_status asf_activation_counts(const asf_ffn *ffn, const void *x, int32_t T, int64_t *counts,
                                 void *ws, size_t ws_bytes, asf_stream_t stream);

/* Strided row gather on the device: dst row i (at dst + i*dst_stride bytes) =
 * src row p (at src + p*src_stride bytes) with p = perm[i] (p = i when perm is
 * NULL), row_bytes each, for i < n_rows; rows with p outside [0, src_rows) are
 * skipped.  With dst_stride = m*d*s and dst offsets 0, d*s, 2*d*s it builds the
 * neuron-major packed layout of asf_ffn (and applies a hot permutation in the
 * same pass).  Source and destination ranges must not overlap. */
ASF_API asf_status asf_gather_rows(const void *src, int64_t src_stride, int32_t src_rows, void *dst,
                                   int64_t dst_stride, int32_t n_rows, int64_t row_bytes,
                                   const int32_t *perm, asf_stream_t stream);

/* Host-side, synchronous: perm = neuron ids in descending count order, equal
 * counts in ascending id order.  counts: host int64 [n]; perm_out: host int32 [n]. */
ASF_API asf_status asf_hot_permutation(const int64_t *counts, int32_t n, int32_t *perm_out);

/* Row gather on the device: dst row i = src row perm[i], for i < n_rows.
 * src, dst: device [n_rows][row_bytes], distinct buffers; perm: device int32
 * [n_rows] with values in [0, n_rows) (out-of-range rows are skipped). */
ASF_API asf_status asf_permute_rows(const void *src, void *dst, int32_t n_rows, int64_t row_bytes,
                            const int32_t *perm, asf_stream_t stream);

/* Sparse FFN that allocates nothing and needs no workspace.
 *
 * No counterpart in the paper: this is a deployment convenience.  Some
 * callers cannot allocate device memory where they run the FFN -- for example
 * a plugin inside a host framework that owns every device allocation through
 * its own pool, or a latency-critical path that cannot afford the implicit
 * device synchronisation of cudaMalloc.  This call computes exactly what
 * asf_sparse_ffn computes (same kernels, same summation order, so the same y
 * bit for bit), but takes its scratch from a file-scope device array of
 * ASF_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits.
 *
 *   ffn, x, B, idx, count, y   as for asf_sparse_ffn
 *   fault   optional device int32: if not NULL, it receives the raw fault bits
 *           of this call (0 = none; bit 0 = index out of range, bit 1 = timeout)
 *
 * Size limit.  The call needs 4096 bytes of counters plus the scratch of
 * asf_sparse_ffn: for B <= 4, G * B * d * 4 bytes of per-CTA partial sums with
 * G = min(SM count, 256) (148 on B200); for larger B, n * B * 4 bytes of
 * activations plus the down projection's S * B * d * 4 bytes of split sums
 * (S <= 64 splits of the index list).  Shapes that need more than
 * ASF_NOALLOC_SCRATCH_BYTES return ASF_ERR_UNSUPPORTED without enqueuing
 * anything.  On B200 the 32 MiB array covers every layer with d <= 12288 and
 * n <= 49152 at every batch up to ASF_MAX_BATCH; the largest need among them,
 * d = 12288 at B = 4, is 29.1 MB.
 *
 * The first call on each device looks up the array's device address for the
 * current device (cudaGetSymbolAddress) and keeps it for the life of the
 * process; make that first call before any stream capture.  The kept address
 * is not valid across cudaDeviceReset (the library's module is reloaded in the
 * new context): do not use this call after resetting a device.  Each call
 * clears the array's counters and fault word on `stream` before its kernels
 * run.  All calls share the one array: calls that can overlap on the GPU
 * (other streams, other threads) race and must be serialised by the caller.
 * No device memory is allocated or freed, directly or by a library routine. */
#define ASF_NOALLOC_SCRATCH_BYTES (32u << 20)
ASF_API asf_status asf_sparse_ffn_noalloc(const asf_ffn *ffn, const void *x, int32_t B, const int32_t *idx,
                                          const int32_t *count, float *y, int32_t *fault, asf_stream_t stream);

/* ---------------------------------------------------------------------------
 * Neuron-sharded layer across GPUs (the layer + neuron partitioning of the
 * "PowerInfer_x64" page's multi-GPU coordination): rank r holds the predictor
 * rows and FFN rows of its own neurons, and the ranks' partial outputs are
 * summed.  Here the sum is part of the layer's last kernel: each rank reduces
 * its own per-CTA partials, publishes the result in its own buffer, and reads
 * the other ranks' published results directly over peer memory (NVLink /
 * NVSwitch), adding all ranks in rank order -- so every rank gets the same y,
 * bit for bit, with no separate collective launch.
 *
 * Every pointer below is a device pointer valid on the calling rank's GPU:
 * its own buffers, and the other ranks' buffers mapped into this process
 * (CUDA IPC handles opened with peer access).  The buffers are owned by the
 * caller and reused by every call; a rank must make the same sequence of
 * calls (same B each time) as every other rank of the group.
 */
#define ASF_MAX_PEERS 8
typedef struct {
  int32_t world;                   /* ranks in the group, 1..ASF_MAX_PEERS */
  int32_t rank;                    /* this rank (0 when one process emulates all ranks) */
  int32_t max_batch;               /* B the buffers were sized for, <= ASF_MAX_BATCH */
  int32_t d;                       /* hidden size */
  float *pub[ASF_MAX_PEERS];       /* rank r's publication buffer: 2 * max_batch * d fp32 */
  uint32_t *flag[ASF_MAX_PEERS];   /* rank r's flag words: ceil(d/32) * max_batch uint32 */
  uint32_t *epoch;                 /* this rank's call counters: ceil(d/32) * max_batch uint32
                                      (times world when one process emulates all ranks);
                                      zero them, and every flag word, once before the first call */
} asf_peer_group;

/* One layer of a neuron-sharded model on this rank: as asf_predict_sparse_ffn
 * over this rank's predictor and FFN rows (idx and count are local storage
 * indices), except that y receives the sum over all ranks of their partial
 * outputs, exchanged through grp.  A peer that does not publish within 200 ms
 * makes the call record ASF_ERR_TIMEOUT in the workspace error word; its share
 * is then missing from y. */
ASF_API asf_status asf_predict_sparse_ffn_exchange(const asf_predictor *pred, const asf_ffn *ffn, const void *x,
                                                   int32_t B, float tau, int32_t *idx, int32_t *count, float *y,
                                                   void *ws, size_t ws_bytes, const asf_peer_group *grp,
                                                   asf_stream_t stream);

/* The exchange on its own: y = sum over ranks r (in rank order) of the sum
 * over g < G (in order) of rank r's part[g][B][d] (fp32).  With
 * local_ranks == 1 the call is this rank's part of the exchange; with
 * local_ranks == grp->world one process holds every rank's partials (rank r
 * at part + r * part_rank_stride, its y at y + r * y_rank_stride, its
 * counters at grp->epoch + r * ceil(d/32) * max_batch) and runs all ranks in
 * one cooperative launch on its GPU (testing the exchange without several
 * GPUs; ASF_ERR_UNSUPPORTED if the ranks' blocks cannot all be resident).
 * 1 <= G <= 256.  ws: a workspace (at least 4096 bytes) for the error word. */
ASF_API asf_status asf_reduce_exchange(const float *part, int64_t part_rank_stride, int32_t G, int32_t B, int32_t d,
                                       const asf_peer_group *grp, int32_t local_ranks, float *y,
                                       int64_t y_rank_stride, void *ws, size_t ws_bytes, asf_stream_t stream);

/* Test hook for the failure path of the bounded device waits (no counterpart
 * in the pages).  Process-wide; read when a call enqueues its kernels.
 *   ASF_INJECT_NONE                 normal operation (the default)
 *   ASF_INJECT_WITHHOLD_FFN_COPIES  in the one-kernel sparse FFN (B <= 4),
 *       CTA 0's producer issues none of its row copies, so that CTA's bounded
 *       wait for its first row runs out (after 200 ms): the kernel records
 *       ASF_ERR_TIMEOUT in the workspace error word, skips that CTA's rows and
 *       returns.  y is then incomplete.  No memory is touched out of bounds,
 *       nothing hangs and the CUDA context stays usable; the next call on the
 *       same workspace (after asf_read_error) runs normally.
 * Returns ASF_ERR_INVALID_ARG for any other mode. */
#define ASF_INJECT_NONE 0
#define ASF_INJECT_WITHHOLD_FFN_COPIES 1
ASF_API asf_status asf_set_fault_injection(int32_t mode);

/* Wait for the stream, then return (in *host_out) and clear the device error
 * word: 0, or the asf_status of the first device-side fault recorded. */
ASF_API asf_status asf_read_error(void *ws, int32_t *host_out, asf_stream_t stream);

/* Static description of a status code. */
ASF_API const char *asf_status_string(asf_status s);

/* ABI version: major * 100 + minor (1.02: asf_ffn.hot_rows, asf_ffn.row_stride, asf_gather_rows;
 * 1.03: asf_ffn.l2_next; 1.04: asf_predict_sparse_ffn; 1.05: asf_sparse_ffn_noalloc;
 * 1.06: asf_predict_sparse_ffn_begin / _end, asf_set_fault_injection, asf_peer_group,
 * asf_predict_sparse_ffn_exchange, asf_reduce_exchange). */
ASF_API int32_t asf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ASFFN_H */
