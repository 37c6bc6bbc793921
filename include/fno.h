/*
 * fno.h -- C ABI of the B200 (sm_100a) FNO spectral-convolution library.
 *
 * The operation.  A Fourier Neural Operator block maps x[B, Ci, N_0..N_{d-1}]
 * to y[B, Co, N_0..N_{d-1}]:
 *
 *   s      = tanh(x) under FNO_TANH_PREACT, else x
 *   xhat_k = sum_n s[n] exp(-i theta(k, n)),              k in K   (truncated DFT)
 *   yhat   = sum_i xhat[b, i, k] R[i, o, k]                         (per-mode mixing)
 *   yspec  = (1/N) sum_{k in K} c_k Re(yhat_k exp(+i theta(k, n)))  (truncated inverse)
 *   pre    = yspec + W x + b ;  y = GELU(pre)  (exact erf GELU; none under FNO_NO_ACT)
 *
 * theta(k, n) = 2 pi sum_j k_j n_j / N_j, N = prod_j N_j.  The last axis is the
 * real-FFT axis.  The kept set K holds on every non-last axis j the wavenumbers
 * 0..m_j-1 then N_j-m_j..N_j-1, and on the last axis 0..m_{d-1}-1; |K| =
 * m_{d-1} prod_{j<d-1} 2 m_j, flattened row-major in that order.  c_k is 1 on
 * the last axis' DC column (and its Nyquist column, N_{d-1} even) and 2
 * elsewhere, so a DC/Nyquist column contributes only its real part.
 *
 * Sources (web pages, cited by title and section):
 *   [MPFNO]  "Model-Parallel Fourier Neural Operators as Learned Surrogates for
 *            Large-Scale Parametric PDEs" (review), "Proposed method": the
 *            original FNO -- lifting, 4 spectral blocks, width 20, projection --
 *            whose spectral convolution is FNO's linear-algebra form;
 *            gradients by automatic differentiation.
 *   [MPTRAIN] "Guaranteed approximation bounds and efficient mixed-precision
 *            training for neural operators" (summary), "key insights": half
 *            precision Fourier transform and spectral contraction, tanh
 *            pre-activation before the Fourier transform.
 * The pages give no equations; the block above is the standard FNO block and
 * the conventions (mode set, 1/N on the inverse, c_k, exact GELU) are the
 * library's stated readings.
 *
 * Layouts (all row-major, contiguous, no strides):
 *   activations   [B][C][N_0]..[N_{d-1}] in the storage dtype
 *   R             [Ci][Co][|K|][2]  (re, im) in the storage dtype
 *   W             [Co][Ci], b [Co]  in the storage dtype
 *   xhat_save     [B][Ci][|K|][2]   float32 (re, im)
 *   dR            [Ci][Co][|K|][2]  float32;  dW [Co][Ci], db [Co] float32
 *
 * Ownership: the caller owns every buffer (device memory unless stated) and
 * the stream.  The library never allocates or frees; all work is enqueued on
 * `stream` (NULL = legacy default stream) with no host synchronisation.  The
 * workspace is scratch device memory of at least fno_*workspace_size() bytes;
 * its contents on entry do not matter.  Gradient outputs are overwritten, not
 * accumulated.  Device pointers must be 16-byte aligned.  Because nothing is
 * allocated and nothing synchronises, a sequence of calls on a capturing stream
 * records into a CUDA graph (stream capture, relaxed mode) whose replays give
 * the same results as the calls; the graph holds the pointers, so the buffers
 * must stay in place.
 *
 * Errors: every call returns FNO_OK (0) or a negative FNO_ERR_* code and
 * leaves a message for fno_last_error() (thread-local).  Invalid descriptors,
 * NULL or misaligned required pointers and too-small workspaces are rejected
 * before anything is enqueued.  FNO_ERR_CUDA reports a launch failure; an
 * asynchronous device fault surfaces at the caller's next synchronisation.
 */
#ifndef FNO_H
#define FNO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *fno_stream_t; /* identical to cudaStream_t */
typedef struct CUevent_st *fno_event_t;   /* identical to cudaEvent_t */

enum fno_status {
  FNO_OK = 0,
  FNO_ERR_INVALID_ARG = -1, /* bad descriptor, NULL or misaligned pointer */
  FNO_ERR_UNSUPPORTED = -2, /* valid but outside what the kernels handle */
  FNO_ERR_WORKSPACE = -3,   /* workspace smaller than fno_*workspace_size() */
  FNO_ERR_CUDA = -4,        /* CUDA launch / runtime error */
  FNO_ERR_TIMEOUT = -5      /* a bounded device-side wait gave up */
};

enum fno_dtype { FNO_F32 = 0, FNO_F16 = 1, FNO_BF16 = 2 };

enum fno_flags {
  FNO_TANH_PREACT = 1u, /* tanh on the spectral branch's input ([MPTRAIN]) */
  FNO_NO_ACT = 2u       /* block output is pre (no GELU) */
};

enum fno_op {
  FNO_OP_SPECTRAL_FWD = 0,
  FNO_OP_SPECTRAL_BWD = 1,
  FNO_OP_BLOCK_FWD = 2,
  FNO_OP_BLOCK_BWD = 3,
  FNO_OP_NET_FWD = 4,
  FNO_OP_NET_BWD = 5,
  FNO_OP_SPECTRAL_BWD_CP = 6, /* fno_spectral_conv_bwd_cp */
  FNO_OP_BLOCK_BWD_CP = 7     /* fno_block_bwd_cp */
};

#define FNO_MAX_DIMS 3
#define FNO_MAX_LAYERS 16

/* One spectral block.  ndim in 1..3; grid[j], modes[j] for j < ndim (the rest
 * ignored); 1 <= 2 modes[j] <= grid[j] for j < ndim-1 and
 * 1 <= modes[ndim-1] <= grid[ndim-1]/2 + 1. */
typedef struct fno_block_desc {
  int ndim;
  int dtype;      /* enum fno_dtype: storage dtype of activations and params */
  unsigned flags; /* enum fno_flags */
  int cin;
  int cout;
  int64_t batch;
  int64_t grid[FNO_MAX_DIMS];
  int modes[FNO_MAX_DIMS];
} fno_block_desc;

/* The network: v0 = P a + p (lift); v_{l+1} = block_l(v_l), l < n_layers,
 * every block width->width with the same modes and flags;
 * u = Q2 GELU(Q1 v_L + q1) + q2 (projection).  [MPFNO] "Proposed method". */
typedef struct fno_net_desc {
  int ndim;
  int dtype;
  unsigned flags;
  int in_channels;  /* channels of a (field + coordinates) */
  int width;        /* block width */
  int hidden;       /* projection hidden width */
  int out_channels; /* channels of u */
  int n_layers;     /* 1..FNO_MAX_LAYERS */
  int64_t batch;
  int64_t grid[FNO_MAX_DIMS];
  int modes[FNO_MAX_DIMS];
} fno_net_desc;

/* Network parameters (device, storage dtype).  P [width][in], p [width],
 * R[l] [width][width][|K|][2], W[l] [width][width], b[l] [width],
 * Q1 [hidden][width], q1 [hidden], Q2 [out][hidden], q2 [out]. */
typedef struct fno_params {
  const void *P, *p;
  const void *R[FNO_MAX_LAYERS];
  const void *W[FNO_MAX_LAYERS];
  const void *b[FNO_MAX_LAYERS];
  const void *Q1, *q1, *Q2, *q2;
} fno_params;

/* Parameter gradients (device, float32), same shapes as fno_params. */
typedef struct fno_grads {
  float *P, *p;
  float *R[FNO_MAX_LAYERS];
  float *W[FNO_MAX_LAYERS];
  float *b[FNO_MAX_LAYERS];
  float *Q1, *q1, *Q2, *q2;
} fno_grads;

/* Thread-local message of the last failing call on this thread ("" if none). */
const char *fno_last_error(void);

/* Library version string. */
const char *fno_version(void);

/* Number of kernel launches the last successful call on this thread enqueued. */
int fno_last_launch_count(void);

/* Kernel selection.  1 (default): per shape the design measured faster: the
 * truncated transform as a streaming pruned radix-16 FFT on the CUDA cores
 * (2D grids) or a dense DFT-matrix contraction on the tensor cores (3D grids,
 * and shapes the streaming kernel does not take), the mixing on the CUDA
 * cores (on the tensor cores for bfloat16 weights with 64 output channels),
 * a pruned slab-axis inverse on the CUDA cores, the warp-specialised tcgen05
 * TMA pipelines for the epilogue and the projection; 4: as 1 with the
 * transform as a clustered pruned FFT; 3: the tcgen05 TMA pipelines
 * throughout with the dense DFT-matrix transform; 2: the tensor-core kernels
 * without the TMA pipelines (mixing on the CUDA cores); 0: the CUDA-core
 * kernels everywhere.  All are complete
 * implementations; the switch exists to compare them.  Process-wide; any
 * other nonzero value means 1; returns the previous setting. */
int fno_set_tensor_cores(int enable);

/* Synchronises the current device and reads the library's device error word,
 * which a kernel sets when one of its bounded waits on the tensor-core
 * pipeline expires (its results are then invalid).  Returns FNO_OK or
 * FNO_ERR_TIMEOUT; clear != 0 resets the word. */
int fno_device_error(int clear);

/* Bound of every wait of the tensor-core pipelines on the current device, in
 * suspended polls of at most about 16 us (default 131072, about two seconds);
 * returns the previous bound, or a negative error.  A test hook: with 0 each
 * wait gives up after one probe, so a kernel whose roles are not already in
 * step records FNO_ERR_TIMEOUT (fno_device_error) and leaves invalid results;
 * its waits before leaving the GPU (for copies and MMAs already in flight)
 * keep the default bound.  Synchronises the device; restore the default
 * before normal work. */
int fno_set_wait_limit(int spins);

/* Per-kernel timing.  fno_profile_enable(1) starts a recording: from then on
 * every kernel the library launches (on any thread) is bracketed by a pair of
 * CUDA events recorded on its launch stream; fno_profile_enable(0) stops
 * recording.  fno_profile_read() waits for the recorded events and writes, per
 * kernel tag, the number of launches and their summed device time (ms);
 * it returns the number of tags written (at most max) or a negative error.
 * Intended for benchmarking: the extra event records add a little time
 * between kernels.  Not thread-safe against concurrent enable/read calls. */
typedef struct fno_kernel_stat {
  char name[48];
  int launches;
  double total_ms;
} fno_kernel_stat;

int fno_profile_enable(int on);
int fno_profile_read(fno_kernel_stat *out, int max);

/* Workspace bytes needed by a block op (FNO_OP_SPECTRAL_* / FNO_OP_BLOCK_*);
 * 0 for an invalid descriptor (see fno_last_error). */
size_t fno_workspace_size(const fno_block_desc *desc, int op);

/* Workspace bytes for FNO_OP_NET_FWD / FNO_OP_NET_BWD, and bytes of the
 * forward's saved activations that fno_backward reads. */
size_t fno_net_workspace_size(const fno_net_desc *desc, int op);
size_t fno_net_saves_size(const fno_net_desc *desc);

/* Spectral branch only: y = yspec (storage dtype, [B][Co][grid]).
 * xhat_save (optional, may be NULL) receives xhat [B][Ci][|K|][2] float32. */
int fno_spectral_conv_fwd(const fno_block_desc *desc, const void *x, const void *R,
                          void *y, float *xhat_save, void *ws, size_t ws_bytes,
                          fno_stream_t stream);

/* Bytes of the scratch array built into the library for
 * fno_spectral_conv_fwd_noalloc (per GPU that loads the library). */
#define FNO_NOALLOC_SCRATCH_BYTES (32u << 20)

/* fno_spectral_conv_fwd for callers that cannot allocate device memory.
 * The pages have no counterpart; this is a deployment convenience.  Some
 * callers own no allocator at all: a plugin inside a host application that
 * keeps every device byte in its own pool, or code that runs where a
 * cudaMalloc would stall the stream or is simply not permitted.  Such a caller
 * passes only inputs and outputs; the scratch lives in a fixed device array of
 * FNO_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU that
 * loads the library holds until the process exits.  This call allocates and
 * frees nothing, on the host or the device.
 *   - Problems whose fno_workspace_size(desc, FNO_OP_SPECTRAL_FWD) exceeds the
 *     array are rejected with FNO_ERR_WORKSPACE and a message naming both sizes.
 *   - The first call on each device looks up the array's device address (a
 *     host-side lookup that requires that device to be current).  Make that first
 *     call before any stream capture.  The address is kept for the life of the
 *     process, so cudaDeviceReset on that device after the first call is not
 *     supported (the kept address would then be stale).
 *   - All calls share the one array, which keeps whatever the last call left in
 *     it; every scratch byte this operation reads it has first written, so
 *     nothing needs clearing.  Calls whose work overlaps on the GPU (concurrent
 *     streams, or several host threads on one device) race on the array:
 *     serialise them.
 * Arguments, layouts and results are those of fno_spectral_conv_fwd. */
int fno_spectral_conv_fwd_noalloc(const fno_block_desc *desc, const void *x, const void *R,
                                  void *y, float *xhat_save, fno_stream_t stream);

/* Factorised spectral weights (TFNO of [MPTRAIN], summary): the weight is the
 * rank-`rank` CP tensor R[i,o,k] = sum_r lam[r] A[i,r] B[o,r] C[k,r] and is
 * never formed; the mixing contracts xhat with A over i, multiplies by C and
 * contracts with lam B over r (the order the greedy planner picks at low
 * rank).  Factors are complex, (re, im) interleaved in the storage dtype:
 * lam [rank][2], A [Ci][rank][2], B [Co][rank][2], C [|K|][rank][2], K in the
 * order of R.  1 <= rank <= FNO_MAX_CP_RANK.  Workspace, other arguments,
 * results and errors are those of fno_spectral_conv_fwd / fno_block_fwd. */
#define FNO_MAX_CP_RANK 32
int fno_spectral_conv_fwd_cp(const fno_block_desc *desc, int rank, const void *x, const void *lam,
                             const void *A, const void *B, const void *C, void *y,
                             float *xhat_save, void *ws, size_t ws_bytes, fno_stream_t stream);
int fno_block_fwd_cp(const fno_block_desc *desc, int rank, const void *x, const void *lam,
                     const void *A, const void *B, const void *C, const void *W, const void *b,
                     void *y, void *pre_save, float *xhat_save, void *ws, size_t ws_bytes,
                     fno_stream_t stream);

/* Adjoints of the factorised forwards.  The gradient of the dense weight,
 * dR = sum_b conj(xhat) (c_k/N) DFT_K(dz), is formed as in the dense backward
 * (on the weight rebuilt from the factors in the storage dtype), then projected
 * onto the factors by the chain rule (the weight is holomorphic in each factor,
 * so dz = sum dR conj(dR/dz) under the convention dz = dL/dRe z + i dL/dIm z):
 *   dlam[r] = sum_{i,o,k} dR conj(A[i,r] B[o,r] C[k,r]),
 *   dA[i,r] = sum_{o,k} dR conj(lam[r] B[o,r] C[k,r]),  likewise dB, dC.
 * Outputs (float32, (re, im), overwritten): dlam [rank][2], dA [Ci][rank][2],
 * dB [Co][rank][2], dC [|K|][rank][2]; dx (storage dtype), and for the block
 * dW, db as fno_block_bwd.  Workspace: fno_workspace_size(desc,
 * FNO_OP_SPECTRAL_BWD_CP or FNO_OP_BLOCK_BWD_CP). */
int fno_spectral_conv_bwd_cp(const fno_block_desc *desc, int rank, const void *x,
                             const void *lam, const void *A, const void *B, const void *C,
                             const float *xhat_save, const void *dy, void *dx, float *dlam,
                             float *dA, float *dB, float *dC, void *ws, size_t ws_bytes,
                             fno_stream_t stream);
int fno_block_bwd_cp(const fno_block_desc *desc, int rank, const void *x, const void *lam,
                     const void *A, const void *B, const void *C, const void *W,
                     const void *pre_save, const float *xhat_save, const void *dy, void *dx,
                     float *dlam, float *dA, float *dB, float *dC, float *dW, float *db, void *ws,
                     size_t ws_bytes, fno_stream_t stream);

/* Adjoint of fno_spectral_conv_fwd.  Inputs: x (needed for tanh'), xhat_save
 * from the forward (may be NULL: then it is recomputed from x), R, dy
 * [B][Co][grid].  Outputs: dx [B][Ci][grid] (storage dtype),
 * dR = sum_b conj(xhat) (c_k/N) DFT_K(dy) (float32). */
int fno_spectral_conv_bwd(const fno_block_desc *desc, const void *x, const float *xhat_save,
                          const void *R, const void *dy, void *dx, float *dR, void *ws,
                          size_t ws_bytes, fno_stream_t stream);

/* Full block: y = GELU(yspec + W x + b).  pre_save (optional) receives pre in
 * the storage dtype; xhat_save (optional) receives xhat (float32). */
int fno_block_fwd(const fno_block_desc *desc, const void *x, const void *R, const void *W,
                  const void *b, void *y, void *pre_save, float *xhat_save, void *ws,
                  size_t ws_bytes, fno_stream_t stream);

/* Adjoint of fno_block_fwd.  pre_save is required (ignored under FNO_NO_ACT);
 * xhat_save may be NULL (recomputed).  Outputs dx (storage dtype), dR, dW, db
 * (float32, overwritten). */
int fno_block_bwd(const fno_block_desc *desc, const void *x, const void *R, const void *W,
                  const void *pre_save, const float *xhat_save, const void *dy, void *dx,
                  float *dR, float *dW, float *db, void *ws, size_t ws_bytes,
                  fno_stream_t stream);

/* Network forward u = projection(blocks(lift(a))).  a [B][in][grid],
 * u [B][out][grid] (storage dtype).  saves (optional, fno_net_saves_size bytes)
 * receives what fno_backward needs. */
int fno_forward(const fno_net_desc *desc, const void *a, const fno_params *params, void *u,
                void *saves, void *ws, size_t ws_bytes, fno_stream_t stream);

/* Network backward from du [B][out][grid] (storage dtype) and the forward's
 * saves: every parameter gradient (float32, overwritten). */
int fno_backward(const fno_net_desc *desc, const void *a, const fno_params *params,
                 const void *saves, const void *du, fno_grads *grads, void *ws,
                 size_t ws_bytes, fno_stream_t stream);

/* fno_backward that also reports when each group of gradients is final, for
 * data parallelism whose gradient all-reduce overlaps the rest of the backward
 * ("Efficient multi-GPU distributed training strategies for neural operator
 * networks", key methods: all-reduce data parallelism).  The backward finishes
 * the groups in this order and records ready[j] (cudaEventRecord on `stream`)
 * right after group j's last kernel:
 *   ready[0]                 dQ1, dq1, dQ2, dq2 (projection)
 *   ready[1 + j], j < L      dR, dW, db of layer L - 1 - j (L = n_layers)
 *   ready[L + 1]             dP, dp (lift)
 * The events belong to the caller (created by it, any flags); n_ready must be
 * n_layers + 2.  A caller that makes a second stream wait on ready[j] can start
 * group j's all-reduce there while the backward of the earlier layers runs.
 * Arguments, results and errors are otherwise those of fno_backward. */
int fno_backward_ready(const fno_net_desc *desc, const void *a, const fno_params *params,
                       const void *saves, const void *du, fno_grads *grads, void *ws,
                       size_t ws_bytes, fno_stream_t stream, fno_event_t *ready, int n_ready);

/* Mean-squared error over n elements: *loss = mean((u - t)^2) (float32,
 * device), du = 2 (u - t) / n (storage dtype).  du may be NULL. */
int fno_mse(int64_t n, int dtype, const void *u, const void *target, float *loss, void *du,
            fno_stream_t stream);

/* One optimiser step of the training loop over n float32 master weights, fused
 * with the copy the next forward reads.  Adam (Kingma and Ba, "Adam: A Method
 * for Stochastic Optimization", Algorithm 1) with decoupled weight decay
 * (Loshchilov and Hutter, "Decoupled Weight Decay Regularization"); the copy's
 * dtype carries the precision schedule of [MPTRAIN] (mixed, then full
 * precision):
 *   g = grad * grad_scale;  m = beta1 m + (1 - beta1) g;  v = beta2 v + (1 - beta2) g^2
 *   theta -= lr (m / (1 - beta1^step)) / (sqrt(v / (1 - beta2^step)) + eps)
 *            + lr weight_decay theta
 *   param_out = theta rounded to out_dtype (round to nearest even)
 * theta, m, v [n] float32 device, updated in place; grad [n] float32 device;
 * param_out [n] device in out_dtype (enum fno_dtype), may be NULL.  grad NULL
 * copies theta to param_out without an update (m, v, step and the
 * hyper-parameters are then ignored).  step >= 1 is the 1-based step number;
 * 0 <= beta < 1, eps > 0, lr >= 0, weight_decay >= 0.  Pointers 16-byte
 * aligned; param_out overlaps none of theta, m, v, grad.  A flat buffer
 * holding all of fno_params (each parameter at a 16-byte aligned offset) is
 * updated in one call. */
int fno_adam_step(int64_t n, float *theta, float *m, float *v, const float *grad,
                  void *param_out, int out_dtype, int step, float lr, float beta1, float beta2,
                  float eps, float weight_decay, float grad_scale, fno_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FNO_H */
