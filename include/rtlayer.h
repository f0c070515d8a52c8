/*
 * rtlayer.h -- C ABI of librtlayer.so: the forward pass (prefill / training
 * forward) of one Recurrent Transformer (RT) layer on an NVIDIA B200 (sm_100a),
 * computed with the exact dyadic ("lowbit") blocked schedule.
 *
 * Source of the operation: "Recurrent Transformer" paper page
 * (www.lshu.cn/news/403416):
 *   - paper §2.2 (Recurrent Transformer layer): a layer maps x_1..x_N to
 *     z_1..z_N; position i forms its query and a temporary (k, v) from its
 *     input x_i, and a persistent (k_i, v_i) from its output z_i, which is
 *     stored and used by every later position;
 *   - notes §2.2 (temporary vs persistent key/value pairs);
 *   - notes §4.2 / paper §5 (exact blocked schedule): queries are computed up
 *     front; when (k_t, v_t) is revealed, keys (t - lowbit(t), t] are folded
 *     into the online-softmax statistics (m, l, o) of queries
 *     (t, t + lowbit(t)]; exact up to floating-point reordering;
 *   - paper §6.3 (position-major KV cache).
 *
 * Layer (per sequence b, t = 1..N; rms(v) = v / sqrt(mean(v^2) + 1e-6)):
 *   r = rms(x_t); q = W_q r; k~ = W_k r; v~ = W_v r
 *   a_t = per head h (columns h*d_h .. h*d_h + d_h - 1, d_h = d/H):
 *         softmax over {(k_i, v_i) : i < t} + {(k~, v~)} of <k, q_h>/sqrt(d_h)
 *   u = x_t + W_o a_t ; z_t = u + W_2 GELU(W_1 rms(u))   (exact erf GELU)
 *   k_t = W_k rms(z_t) ; v_t = W_v rms(z_t)               (persistent pair)
 *
 * Conventions for every entry point below
 *   - Pointers named *_dev are device memory owned by the caller; the library
 *     allocates no device memory on these paths. Pointers named *_host are
 *     host memory owned by the caller (page-locked for asynchronous copies).
 *   - Storage type: RT_F32 (all tensors fp32, SIMT fp32 arithmetic) or
 *     RT_BF16 (tensors bf16, fp32 accumulation and fp32 softmax statistics).
 *   - Weights use nn.Linear orientation [out][in] (row-major), y = W r:
 *       W_q, W_k, W_v, W_o : [d][d]; W_1 : [d_ff][d]; W_2 : [d][d_ff].
 *   - x and z are [B][N][d] row-major (sequence-major).
 *   - K and V (the persistent pairs) are POSITION-MAJOR [N][B][d], i.e.
 *     [N][B][H][d_h]: the pairs of one position for all sequences are
 *     contiguous, so a block (t - lb, t] is one contiguous slice.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *     Calls are asynchronous on it. Host-detectable errors (null pointers,
 *     unsupported shapes, workspace too small) are returned before anything is
 *     enqueued. Device-side errors (a bounded wait that ran out) are recorded
 *     in an error word inside the workspace and reported by
 *     rt_layer_sync_status.
 *   - Concurrent calls sharing one workspace race; use one workspace per
 *     in-flight call.
 *   - Supported shapes: RT_F32: d_h in {32, 64, 128}. RT_BF16: d_h = 64,
 *     d and d_ff multiples of 64. B, N >= 1. Others: RT_ERR_UNSUPPORTED.
 */
#ifndef RTLAYER_H
#define RTLAYER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RT_OK = 0,
  RT_ERR_INVALID_ARG = -1,  /* null pointer, non-positive size, d % H != 0 */
  RT_ERR_UNSUPPORTED = -2,  /* shape/dtype combination not implemented     */
  RT_ERR_WORKSPACE = -3,    /* workspace pointer null or too small          */
  RT_ERR_CUDA = -4,         /* a CUDA runtime call failed                   */
  RT_ERR_TIMEOUT = -5,      /* a device-side bounded wait ran out           */
  RT_ERR_DEVICE = -6        /* no usable sm_100 device                      */
} rt_status;

typedef enum { RT_F32 = 0, RT_BF16 = 1 } rt_dtype;

/* RT_SCHED_BLOCKED: the exact lowbit schedule (the product path).
 * RT_SCHED_NAIVE: query t attends to all persistent pairs i < t at step t,
 * Theta(N^2) traffic (the ablation of notes §4.1). Same result up to rounding. */
typedef enum { RT_SCHED_BLOCKED = 0, RT_SCHED_NAIVE = 1 } rt_schedule;

/* RT_DRIVER_GRAPH: the whole N-step loop (one kernel per phase of a step:
 * W_o, W_1, W_2, W_kv GEMMs and the block fold) is recorded once into a
 * CUDA graph (cached per argument set, consecutive kernels overlapped by
 * programmatic dependent launch) and replayed with a single launch per call.
 * RT_DRIVER_STREAM: the same kernels, each launched from the host loop.
 * RT_DRIVER_PERSISTENT: bf16, blocked schedule only: the step loop as one
 * persistent kernel per run of steps whose folds have at most 8 keys (every
 * phase of every step inside it, ordered by flags in global memory), the
 * folds of >= 16 keys between them; recorded into a cached graph like
 * RT_DRIVER_GRAPH. RT_ERR_UNSUPPORTED for other dtypes, schedules or shapes
 * whose per-phase flags exceed its flag table. Same results up to rounding
 * order in all three. */
typedef enum { RT_DRIVER_GRAPH = 0, RT_DRIVER_STREAM = 1, RT_DRIVER_PERSISTENT = 2 } rt_driver;

/* Library version (major*10000 + minor*100 + patch). */
int rt_version(void);

/* Text for a status code. Never NULL. */
const char* rt_status_string(int status);

/* The CUDA runtime error (a cudaError_t value) behind the calling thread's
 * most recent RT_ERR_CUDA status; 0 if there was none. */
int rt_last_cuda_error(void);

/* CUDA's text for a cudaError_t value. Never NULL. */
const char* rt_cuda_error_string(int code);

/* Bytes of device workspace rt_layer_forward needs for this shape.
 * Returns 0 for invalid or unsupported arguments. */
size_t rt_layer_workspace_bytes(int B, int N, int d, int H, int d_ff, int dtype,
                                int schedule);

/* The layer forward (paper §2.2 with the schedule of notes §4.2).
 * Inputs : x_dev [B][N][d]; weights as in the conventions.
 * Outputs: z_dev [B][N][d]; K_dev, V_dev position-major [N][B][d].
 * workspace_dev: >= rt_layer_workspace_bytes(...) bytes, 256-byte aligned.
 * Returns RT_OK once the work is enqueued on `stream`. */
int rt_layer_forward(const void* x_dev,
                     const void* W_q_dev, const void* W_k_dev, const void* W_v_dev,
                     const void* W_o_dev, const void* W_1_dev, const void* W_2_dev,
                     int B, int N, int d, int H, int d_ff,
                     int dtype, int schedule, int driver,
                     void* z_dev, void* K_dev, void* V_dev,
                     void* workspace_dev, size_t workspace_bytes, void* stream);

/* The layer in the paper's own parameterisation (paper §2 notation, §2.1 and
 * §2.2, rather than the single-layer configuration above), bf16, blocked
 * schedule, driver as in rt_layer_forward:
 *   RMS(v) = sqrt(D) v / ||v|| (no eps, unit gain); RMS_h = the same over
 *   each head's 64 entries;
 *   r = RMS(x_t); q = RMS_h(W_q r); k~ = RMS_h(W_k r); v~ = W_v r
 *   a_t: per head softmax of <k, q_h> with no scale
 *   u = x_t + W_o a_t / sqrt(L); z_t = u + W_2 GELU(W_1 RMS(u)) / sqrt(L)
 *   k_t = RMS_h(W_k RMS(z_t)); v_t = W_v RMS(z_t)
 * L >= 1 is the depth of the stack the layer belongs to. Arguments, layouts
 * and workspace (rt_layer_workspace_bytes with RT_BF16, RT_SCHED_BLOCKED) as
 * in rt_layer_forward. */
int rt_layer_forward_pages(const void* x_dev,
                           const void* W_q_dev, const void* W_k_dev, const void* W_v_dev,
                           const void* W_o_dev, const void* W_1_dev, const void* W_2_dev,
                           int B, int N, int d, int H, int d_ff, int L,
                           void* z_dev, void* K_dev, void* V_dev,
                           void* workspace_dev, size_t workspace_bytes, void* stream,
                           int driver);

/* Device bytes rt_layer_forward_chunked needs for chunks of C positions;
 * 0 if unsupported. */
size_t rt_layer_chunked_workspace_bytes(int B, int N, int d, int H, int d_ff, int C);

/* The layer with its recurrence executed block-wise, in chunks of C >= 1
 * positions (paper §9 and notes §8 name this depth-for-speed trade-off
 * without defining it; this is our reading): the positions are cut into
 * consecutive chunks of C; a position's persistent pair is visible only to
 * the positions of later chunks, and inside its own chunk a position attends
 * to the temporary pairs of the chunk's positions up to itself. C = 1 is the
 * layer of rt_layer_forward; C >= N the standard causal Transformer layer
 * (paper §2.1), whose K, V outputs are then W_{k,v} rms(z).
 * bf16, the exact blocked schedule at chunk granularity, graph driver: per
 * chunk one attention launch, the four GEMMs with B * C rows, and one block
 * fold (chunks (c - lowbit(c), c] into chunks (c, c + lowbit(c)]).
 * Arguments and layouts as in rt_layer_forward; workspace_dev >=
 * rt_layer_chunked_workspace_bytes(...) bytes, 256-byte aligned. */
int rt_layer_forward_chunked(const void* x_dev,
                             const void* W_q_dev, const void* W_k_dev, const void* W_v_dev,
                             const void* W_o_dev, const void* W_1_dev, const void* W_2_dev,
                             int B, int N, int d, int H, int d_ff, int C,
                             void* z_dev, void* K_dev, void* V_dev,
                             void* workspace_dev, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the device error word of a
 * workspace used by rt_layer_forward. RT_OK, RT_ERR_TIMEOUT or RT_ERR_CUDA. */
int rt_layer_sync_status(void* workspace_dev, void* stream);

/* Device bytes rt_layer_forward_host needs: the workspace of
 * rt_layer_forward plus device copies of x, the weights, z, K and V. */
size_t rt_layer_host_workspace_bytes(int B, int N, int d, int H, int d_ff,
                                     int dtype, int schedule);

/* End-to-end form of rt_layer_forward with HOST buffers: copies x and the
 * weights host->device, runs the layer, copies z, K, V device->host, all
 * enqueued on `stream` (returns once enqueued; synchronise the stream before
 * reading the outputs). All host pointers must stay valid until then.
 * Layouts as in rt_layer_forward; results are bitwise those of
 * rt_layer_forward.
 * bf16 with x, z, K and V page-locked (cudaHostAlloc / cudaHostRegister):
 * the copies overlap the compute -- x goes up in chunks of sequences on a
 * library-owned transfer stream, each chunk projected as soon as it lands,
 * and z, K, V come down in ranges of positions as soon as the step loop has
 * finished them; the transfer streams fork from and join back into `stream`
 * (and into the cached graph). Otherwise the copies run in sequence with the
 * compute on `stream`. */
int rt_layer_forward_host(const void* x_host,
                          const void* W_q_host, const void* W_k_host, const void* W_v_host,
                          const void* W_o_host, const void* W_1_host, const void* W_2_host,
                          int B, int N, int d, int H, int d_ff,
                          int dtype, int schedule, int driver,
                          void* z_host, void* K_host, void* V_host,
                          void* workspace_dev, size_t workspace_bytes, void* stream);

/* Device bytes rt_layer_decode_step needs (bf16); 0 if unsupported. */
size_t rt_layer_decode_workspace_bytes(int B, int d, int H, int d_ff);

/* One autoregressive decode step of the layer (paper §7.3: a new token costs
 * one query against the cached persistent pairs), bf16.
 * Position t (1-based) of B sequences whose persistent pairs of positions
 * 1..t-1 are rows 0..t-2 of K_cache_dev / V_cache_dev, position-major
 * [capacity][B][d] as returned by rt_layer_forward.
 * Inputs : x_t_dev [B][d]; weights as in rt_layer_forward.
 * Outputs: z_t_dev [B][d]; the new persistent pair (k_t, v_t) is written to
 *          row t-1 of the caches (rows >= t are not touched).
 * 1 <= t <= capacity, else RT_ERR_INVALID_ARG. workspace_dev: >=
 * rt_layer_decode_workspace_bytes(...) bytes, 256-byte aligned; its error
 * word is read by rt_layer_sync_status. Enqueued on `stream`; the result is
 * that of rt_layer_forward's position t up to floating-point order. */
int rt_layer_decode_step(const void* x_t_dev,
                         const void* W_q_dev, const void* W_k_dev, const void* W_v_dev,
                         const void* W_o_dev, const void* W_1_dev, const void* W_2_dev,
                         int B, int t, int capacity, int d, int H, int d_ff,
                         void* z_t_dev, void* K_cache_dev, void* V_cache_dev,
                         void* workspace_dev, size_t workspace_bytes, void* stream);

/* Device bytes rt_layer_recompute_kv needs (bf16); 0 if unsupported. */
size_t rt_layer_recompute_workspace_bytes(int B, int N, int d);

/* Activation-checkpoint recompute of the persistent pairs (paper §6.1: with
 * the layer's inputs and outputs stored, the persistent pairs of every
 * position are rebuilt from the outputs in one parallel step):
 *   K[n][b] = W_k rms(z[b][n]),  V[n][b] = W_v rms(z[b][n])
 * for all B*N positions at once, bf16 storage, fp32 accumulation (one
 * tensor-core GEMM of [B*N][d] x [2d][d]^T with the 1/rms(z) row scale in its
 * epilogue). z_dev [B][N][d]; K_dev, V_dev position-major [N][B][d], as
 * rt_layer_forward returns them. d % 64 == 0, B*N <= 2^30.
 * workspace_dev: >= rt_layer_recompute_workspace_bytes(B, N, d) bytes,
 * 256-byte aligned; its first word is the error word (rt_layer_sync_status).
 * Enqueued on `stream`. The forward forms each pair from the bf16 copy of
 * z_t with the fp32 sum of squares of z_t; from the stored bf16 z the result
 * agrees up to that rounding. */
int rt_layer_recompute_kv(const void* z_dev, const void* W_k_dev, const void* W_v_dev,
                          int B, int N, int d, void* K_dev, void* V_dev,
                          void* workspace_dev, size_t workspace_bytes, void* stream);

/* Device bytes rt_layer_backward needs; 0 if unsupported (d_h <= 128). */
size_t rt_layer_backward_workspace_bytes(int B, int N, int d, int H, int d_ff, int dtype);

/* Backward pass of the layer (paper §6.4, whose body is missing from the
 * extracted text: these are the exact derivatives of the forward of paper
 * §2.2), fp32 arithmetic; storage RT_F32, or RT_BF16 (every input and
 * output bf16; the inputs are widened to fp32 working copies inside the
 * workspace and the gradients rounded to bf16 at the end). Gradients of the
 * scalar
 *   sum(z * dz) + sum(K * dK) + sum(V * dV)
 * with respect to x and the six weights, given the forward's inputs and its
 * stored outputs:
 *   x_dev, z_dev, dz_dev : [B][N][d];  K_dev, V_dev, dK_dev, dV_dev :
 *   position-major [N][B][d] (as rt_layer_forward returns K and V);
 *   weights as in rt_layer_forward.
 * Outputs: dx_dev [B][N][d]; dW_*_dev with the shapes of the weights
 * (overwritten, not accumulated).
 * Method: every intermediate of the forward is rebuilt from (x, z, K, V) in
 * parallel (paper §6.1, activation checkpointing); a reverse loop over
 * positions carries the gradient of each persistent pair back through z_t,
 * the MLP, W_o and the attention of query t (whose contributions to the
 * pairs of earlier positions are added in place); dx and the weight
 * gradients are then formed for all positions at once (the backward batched
 * outside the loop, notes §5.3).
 * workspace_dev: >= rt_layer_backward_workspace_bytes(...) bytes, 256-byte
 * aligned. Enqueued on `stream`. */
int rt_layer_backward(const void* x_dev,
                      const void* W_q_dev, const void* W_k_dev, const void* W_v_dev,
                      const void* W_o_dev, const void* W_1_dev, const void* W_2_dev,
                      const void* z_dev, const void* K_dev, const void* V_dev,
                      const void* dz_dev, const void* dK_dev, const void* dV_dev,
                      int B, int N, int d, int H, int d_ff, int dtype,
                      void* dx_dev, void* dW_q_dev, void* dW_k_dev, void* dW_v_dev,
                      void* dW_o_dev, void* dW_1_dev, void* dW_2_dev,
                      void* workspace_dev, size_t workspace_bytes, void* stream);

/* Token-embedding front end of a layer stack: x[b][n][:] = E[ids[b][n]][:].
 * Paper §6.1 stacks layers by feeding each layer's outputs z to the next
 * layer as its inputs; the first layer's inputs are the embedded tokens, so a
 * stack is this call followed by one rt_layer_forward per layer.
 * ids_dev int32 [B][N], each in [0, vocab) (out-of-range ids produce a zero
 * row and set the error word of `workspace_dev` if it is not NULL);
 * E_dev [vocab][d]; x_dev [B][N][d]; storage type `dtype`. */
int rt_embed_forward(const int32_t* ids_dev, const void* E_dev, int B, int N,
                     int vocab, int d, int dtype, void* x_dev,
                     void* workspace_dev, void* stream);

/* ---------------------------------------------------------------------------
 * Component entry points (the same kernels rt_layer_forward runs, exposed for
 * unit parity tests and measurement).
 * ------------------------------------------------------------------------ */

/* One block fold of notes §4.2 on caller-provided state, position-major:
 *   Q_dev  [n_pos][B][q_stride] (query of head h at column h*d_h),
 *   K_dev, V_dev [n_pos][B][kv_stride],
 *   m_dev, l_dev [n_pos][B][H] fp32, o_dev [n_pos][B][H*d_h] fp32.
 * Folds keys [k0, k0 + nk) into queries [q0, q0 + nq) (0-based positions),
 * updating (m, l, o) in place. m is stored in log2 units scaled by
 * log2(e)/sqrt(d_h) (m = -inf marks an empty accumulator).
 * RT_BF16 needs d_h = 64. The kernel is the one rt_layer_forward runs for a
 * block of nk keys: <= 8 the small-block kernel; multiples of 128 from 1024
 * on the tcgen05 kernels; other multiples of 16 the mma.sync kernel; anything
 * else the warp kernel.
 * err_dev: error word of the tcgen05 kernels' bounded waits, as in
 * rt_project_qkv (read with rt_layer_sync_status). */
int rt_block_fold(const void* Q_dev, int q_stride, const void* K_dev,
                  const void* V_dev, int kv_stride, float* m_dev, float* l_dev,
                  float* o_dev, int B, int H, int d_h, int q0, int nq, int k0,
                  int nk, int dtype, void* err_dev, void* stream);

/* Batched projection of all B*N positions (queries depend only on x):
 *   QKV_dev[n][b][0:d] = W_q rms(x[b][n]), [d:2d] = W_k rms(..), [2d:3d] = W_v rms(..)
 * position-major [N][B][3d]. W_qkv_dev is [3d][d] (W_q; W_k; W_v stacked).
 * scratch_dev: >= B*N*4 bytes (RT_BF16) or B*N*d*4 bytes (RT_F32).
 * err_dev: 16 bytes of device memory, 4-byte aligned (e.g. the first bytes
 * of a layer workspace), whose first word is the error word into which the
 * tensor-core kernel's bounded waits record a timeout; it is only ever OR-ed
 * into, so it accumulates over calls until rt_layer_sync_status(err_dev,
 * stream) reads and clears it (the debug library, librtlayer_check.so, also
 * writes a record of the first failure into the next three words). NULL is
 * RT_ERR_INVALID_ARG. */
int rt_project_qkv(const void* x_dev, const void* W_qkv_dev, int B, int N, int d,
                   int dtype, void* QKV_dev, void* scratch_dev, void* err_dev,
                   void* stream);

/* Dense product C[M][Nout] = A[M][Kd] * W[Nout][Kd]^T in bf16 with fp32
 * accumulation on the tcgen05 tensor-core kernel; C is fp32. Kd % 64 == 0.
 * err_dev: error word as in rt_project_qkv (read with rt_layer_sync_status). */
int rt_gemm_bf16(const void* A_dev, const void* W_dev, float* C_dev, int M,
                 int Nout, int Kd, void* err_dev, void* stream);

/* rt_project_qkv for RT_BF16 storage without caller scratch: the per-row
 * 1/rms values live in a fixed array inside the library, so the call needs no
 * device memory beyond x_dev, W_qkv_dev and QKV_dev (same layouts as
 * rt_project_qkv). The paper has no counterpart; this exists for callers that
 * cannot allocate device memory where they call it (runtimes that plan all
 * device memory at start-up, code running while another framework's caching
 * allocator holds the free memory, latency-critical loops).
 *   - Limit: B*N <= 1048576 rows (a 4 MiB array that every GPU loading the
 *     library keeps until exit); larger sizes return RT_ERR_WORKSPACE before
 *     anything is enqueued. d % 64 == 0.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address with cudaGetSymbolAddress; make that first call
 *     before any stream capture.
 *   - All calls share the array and overwrite the rows they use before
 *     reading them; calls that overlap on the GPU race on it.
 *   - A bounded wait of the tensor-core kernel that runs out is recorded in a
 *     device word that also lives inside the library (one per GPU, shared by
 *     every call); rt_project_qkv_noalloc_status reads and clears it.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
int rt_project_qkv_noalloc(const void* x_dev, const void* W_qkv_dev, int B, int N,
                           int d, void* QKV_dev, void* stream);

/* Status of the rt_project_qkv_noalloc calls enqueued so far on the current
 * device: synchronises `stream`, then reads and clears the library's error
 * word. RT_OK, RT_ERR_TIMEOUT (a bounded wait ran out; that call's QKV_dev
 * is incomplete), RT_ERR_CUDA, or RT_ERR_DEVICE if no call has set up the
 * device yet. Allocates nothing. */
int rt_project_qkv_noalloc_status(void* stream);

/* ---------------------------------------------------------------------------
 * Measurement
 * ------------------------------------------------------------------------ */

/* Number of kernels one rt_layer_forward launches for this shape with this
 * driver (RT_DRIVER_GRAPH and RT_DRIVER_STREAM launch the same kernels); -1
 * for invalid arguments or a shape the driver does not take. */
long rt_layer_launch_count(int B, int N, int d, int H, int d_ff, int dtype, int schedule, int driver);

/* Kernel classes reported by rt_layer_forward_timed. */
enum {
  RT_KC_INV_RMS = 0, /* 1/rms of every input row                          */
  RT_KC_PROJ = 1,    /* batched Q / temporary-pair projection             */
  RT_KC_ATTEND = 2,  /* finalise a_t (blocked) or full attention (naive)  */
  RT_KC_WO = 3,      /* a W_o^T + residual                                */
  RT_KC_W1 = 4,      /* GELU(rms(u) W_1^T)                                */
  RT_KC_W2 = 5,      /* h W_2^T + residual = z_t                          */
  RT_KC_WKV = 6,     /* persistent pair rms(z_t) [W_k; W_v]^T             */
  RT_KC_FOLD_WARP = 7, /* block fold, small-block / warp kernels          */
  RT_KC_FOLD_TENSOR = 8, /* block fold on tensor cores (block >= 16: mma.sync
                           below 256 keys, tcgen05 from 256)             */
  RT_KC_STEPS = 9,     /* persistent step kernel: a segment's W_o, W_1,
                          W_2, W_kv GEMMs and its folds of <= 8 keys       */
  RT_KC_FOLD_LEVEL0 = 16, /* + log2(block size): the same folds by level  */
  RT_KC_COUNT = 32
};

/* rt_layer_forward with the host-loop driver and a CUDA event pair recorded
 * on `stream` around every kernel; synchronises `stream`, then writes the
 * summed device time (ms) and the launch count of each kernel class into
 * class_ms[0..n_classes) and class_launches[0..n_classes). For measurement;
 * not for use inside stream capture. */
int rt_layer_forward_timed(const void* x_dev,
                           const void* W_q_dev, const void* W_k_dev, const void* W_v_dev,
                           const void* W_o_dev, const void* W_1_dev, const void* W_2_dev,
                           int B, int N, int d, int H, int d_ff, int dtype, int schedule,
                           void* z_dev, void* K_dev, void* V_dev,
                           void* workspace_dev, size_t workspace_bytes, void* stream,
                           float* class_ms, int* class_launches, int n_classes);

/* Failure-detection self-test: enqueues one kernel whose single thread waits
 * on a shared-memory barrier that nothing ever arrives on, through the same
 * bounded wait every kernel of this library uses, with a limit of limit_ns
 * nanoseconds (1 .. 1e10). The wait gives up, records the timeout in the
 * error word at workspace_dev (as rt_layer_forward's kernels do) and the
 * kernel exits; rt_layer_sync_status(workspace_dev, stream) then returns
 * RT_ERR_TIMEOUT. Nothing traps or hangs. */
int rt_selftest_wait_timeout(unsigned long long limit_ns, void* workspace_dev, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RTLAYER_H */
