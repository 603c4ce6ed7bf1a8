/*
 * ttt.h — C ABI of the B200 (sm_100a) VGG-T^3 test-time-training layer.
 *
 * The layer (VGG-T$^3$: Offline Feed-Forward 3D Reconstruction at Scale,
 * Sec. 3.4, Eq. 3 and Eq. 4) replaces global softmax attention by
 *   1. V' = ShortConv2D(V): a depthwise 3x3 convolution of each view's patch
 *      grid of values ("Non-Linear Spatial Mixing via ShortConv2D"; camera and
 *      register tokens pass through, Appendix A);
 *   2. `steps` plain gradient steps theta <- theta - lr * grad L(theta) that fit
 *      a per-head SwiGLU fast-weight MLP T_theta(x) = (silu(x W1) * (x W3)) W2
 *      from K to V' under L = (1/n) sum_i ||T_theta(k_i) - v'_i||^2 (Eq. 3,
 *      "TTT MLP Architecture and Inner Optimization");
 *   3. the read o_i = T_theta*(q_i) (Eq. 4).
 *
 * Layouts (row-major, n = n_views * (n_special + grid_h * grid_w)):
 *   Q, K, V, O     bfloat16 bit patterns, [n][heads][d] (token-major; each
 *                  view's n_special special tokens first, then its patch grid
 *                  row by row).
 *   conv_w         float32 [heads*d][3][3], cross-correlation taps (row, col).
 *   theta          float32, packed [W1: heads*d*h | W3: heads*d*h | W2: heads*h*d],
 *                  W1/W3 per head [d][h], W2 per head [h][d].
 *
 * Ownership and streams: the caller owns every buffer; the library allocates
 * no memory.  Scratch lives in a caller-provided device workspace of at least
 * ttt_workspace_bytes(dims, op) bytes, 256-byte aligned.  All device pointers
 * must be 16-byte aligned.  Work is enqueued on `stream` (a cudaStream_t, or
 * NULL for the legacy default stream) and returns without synchronising;
 * inputs are never modified.  theta_out may alias theta0 (in-place update); no
 * other buffers may overlap.  Calls sharing one workspace must not run
 * concurrently.
 *
 * Errors: host-side validation happens before anything is enqueued and
 * returns a negative ttt_status; nothing throws across the ABI.  A failed
 * launch returns TTT_ECUDA.  Faults detected on the device (a bounded wait that
 * ran out) are recorded in the workspace status word, which every call taking
 * a workspace clears when it starts, and are reported by ttt_check_status as
 * TTT_EDEVICE.
 *
 * Supported shapes: heads >= 1; grid_h, grid_w >= 1; 0 <= n_special; n >= 1;
 * and either
 *   d in {16, 32, 64} and 1 <= h <= 256 (padded internally to a multiple of
 *   128 with zero weights, which is exact): the fused tensor-core kernels; or
 *   d and h multiples of 64 (d <= 8192, h <= 32768), e.g. d = 1024, h = 2048:
 *   the wide-head path, which runs the products as the library's own bf16
 *   tensor-core GEMMs (FP32 accumulation, the gate, residual and chain rule
 *   fused into their epilogues) over chunks of 262144 tokens, the weight
 *   gradients summed over the chunks in a fixed order.
 * Other shapes return TTT_EUNSUPPORTED.
 */
#ifndef TTT_H_
#define TTT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ttt_dims {
  int32_t n_views;    /* views (images) in the collection                     */
  int32_t grid_h;     /* patch-grid rows per view (H/p)                       */
  int32_t grid_w;     /* patch-grid columns per view (W/p)                    */
  int32_t n_special;  /* special tokens per view, stored first, not convolved */
  int32_t heads;      /* fast-weight MLPs, one per head                       */
  int32_t d;          /* head width (MLP input and output)                    */
  int32_t h;          /* SwiGLU hidden width                                  */
} ttt_dims;

typedef enum ttt_status {
  TTT_OK = 0,
  TTT_EINVAL = -1,        /* null pointer, negative size, bad op or steps      */
  TTT_EALIGN = -2,        /* a pointer is not 16-byte (workspace: 256-byte) aligned */
  TTT_EUNSUPPORTED = -3,  /* shape outside the supported set                   */
  TTT_EWORKSPACE = -4,    /* workspace smaller than ttt_workspace_bytes        */
  TTT_ECUDA = -5,         /* a CUDA runtime/driver call or launch failed       */
  TTT_EDEVICE = -6        /* a kernel recorded a device-side fault             */
} ttt_status;

typedef enum ttt_op {
  TTT_OP_WRITE = 0,       /* ttt_write                                         */
  TTT_OP_READ = 1,        /* ttt_read                                          */
  TTT_OP_LAYER = 2,       /* ttt_layer                                         */
  TTT_OP_LAYER_HOST = 3,  /* ttt_layer_host: also holds device copies of Q,K,V,conv_w,theta,O */
  TTT_OP_ATTENTION = 4    /* ttt_attention: the layer plus q, k, v and O of the surround */
} ttt_op;

typedef enum ttt_inner {
  TTT_INNER_SGD = 0,      /* mean-squared loss, SGD steps (ttt_layer)              */
  TTT_INNER_MUON = 1      /* dot-product loss, Muon steps (ttt_layer_muon)         */
} ttt_inner;

/* Bytes of device workspace an op needs for these dims; 0 if dims are invalid
 * or unsupported. */
size_t ttt_workspace_bytes(const ttt_dims* dims, int op);

/* Step 1 alone: V_out = ShortConv2D(V) (VGG-T^3 summary, "Non-Linear Spatial
 * Mixing via ShortConv2D", Appendix A).  V, V_out: bf16 [n][heads*d];
 * conv_w: f32 [heads*d][3][3].  FP32 accumulation, bf16 round-to-nearest-even
 * store.  Special tokens are copied.  Needs no workspace. */
int ttt_shortconv2d(const ttt_dims* dims, const uint16_t* V, const float* conv_w,
                    uint16_t* V_out, void* stream);

/* Write (Eq. 3): V' = ShortConv2D(V), then `steps` (>= 0) full-batch SGD steps
 * from theta0 with learning rate lr; theta_out receives theta*.  Operands are
 * bf16 with FP32 accumulation; theta is kept in FP32 and rounded to bf16 for
 * the tensor cores each step. */
int ttt_write(const ttt_dims* dims, const uint16_t* K, const uint16_t* V,
              const float* conv_w, const float* theta0, float lr, int steps,
              float* theta_out, void* workspace, size_t workspace_bytes, void* stream);

/* The write sharded over processes (one collection's views split between
 * ranks).  The loss gradient is a sum of per-token terms (VGG-T^3: Offline
 * Feed-Forward 3D Reconstruction at Scale, Sec. 3.4, Eq. 5), so a rank
 * evaluates it on its own views, the ranks exchange these sums, and every
 * rank applies the same step.  Per rank: V' = ttt_shortconv2d(V) of its views
 * once, then per step
 *   ttt_grad on (K, V') of its views -> its gradient sum,
 *   an all-gather of the ranks' sums (by the caller, e.g. NCCL),
 *   ttt_sgd_update with all of them and scale = lr * 2 / n_total.
 * With one rank this is ttt_write. */

/* grad = d/dtheta of (1/2) sum_i ||T_theta(k_i) - vp_i||^2 over the n tokens
 * that dims describe (the gradient of Eq. 3's loss is (2/n_total) times the
 * sum of the ranks' grads).  K, Vp: bf16 [n][heads][d], Vp = ShortConv2D(V)
 * of the same views; theta, grad: f32, theta's packed layout.  FP32
 * accumulation over bf16 operands, summed in a fixed order (deterministic).
 * Workspace: ttt_workspace_bytes(dims, TTT_OP_WRITE). */
int ttt_grad(const ttt_dims* dims, const uint16_t* K, const uint16_t* Vp, const float* theta,
             float* grad, void* workspace, size_t workspace_bytes, void* stream);

/* theta_out = theta_in - scale * (grads[0] + ... + grads[n_grads - 1]) for
 * every element, the sum taken in index order, so every rank that applies
 * the same inputs gets the same bits.  grads: n_grads >= 1 contiguous f32
 * buffers of theta's size (for example an all-gather of the ranks' ttt_grad
 * outputs in rank order).  Only heads, d and h of dims are used.  theta_out
 * may alias theta_in.  Needs no workspace. */
int ttt_sgd_update(const ttt_dims* dims, const float* theta_in, const float* grads, int n_grads,
                   float scale, float* theta_out, void* stream);

/* The pages' own inner loop (VGG-T^3, Sec. 3.4, "The dot product loss" and
 * "TTT MLP Architecture and Inner Optimization"): the dot-product loss
 * L = -(1/n) sum_i <T_theta(k_i), v'_i> and Muon steps
 *   theta <- theta - lr * NS5(grad L)   per weight matrix of each head,
 * NS5 = five cubic Newton-Schulz iterations X <- 1.5 X - 0.5 X X^T X from
 * X_0 = G / ||G||_F (the pages give 5 iterations and lr 0.1, no polynomial;
 * the cubic iteration for the orthogonal polar factor is the reading taken,
 * with no momentum and no shape factor).  The step is scale-free, so the 1/n
 * of the loss does not matter.  The loss is linear in T's output, so no
 * forward pass is needed for the gradient.  Both head families are
 * supported.  On the fused path NS5 runs in FP32 FMAs, one CTA per matrix; on
 * the wide-head path (e.g. d = 1024, h = 2048) its products run on the
 * tensor-core GEMM with each FP32 operand split into a pair of bf16 values
 * (about 2^-16 relative per product) and FP32 accumulation.  Everything else
 * is as in ttt_write.  Workspace: as for ttt_write / ttt_layer. */
int ttt_write_muon(const ttt_dims* dims, const uint16_t* K, const uint16_t* V,
                   const float* conv_w, const float* theta0, float lr, int steps,
                   float* theta_out, void* workspace, size_t workspace_bytes, void* stream);
int ttt_layer_muon(const ttt_dims* dims, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                   const float* conv_w, const float* theta0, float lr, int steps,
                   float* theta_out, uint16_t* O, void* workspace, size_t workspace_bytes,
                   void* stream);

/* The Muon write sharded over processes, as ttt_grad / ttt_sgd_update are for
 * the mean-squared loss.  ttt_grad_dot: grad = d/dtheta of
 * -sum_i <T_theta(k_i), vp_i> over the tokens dims describes (workspace of
 * TTT_OP_WRITE; both head families).  ttt_muon_update: theta_out =
 * theta_in - lr * NS5(grads[0] + ... + grads[n_grads - 1]) per weight matrix
 * of each head, the sum in index order; theta_out may alias theta_in; no
 * workspace, so fused shapes only (the wide-head Newton-Schulz needs scratch
 * for its GEMM operands; wide shapes return TTT_EUNSUPPORTED). */
int ttt_grad_dot(const ttt_dims* dims, const uint16_t* K, const uint16_t* Vp, const float* theta,
                 float* grad, void* workspace, size_t workspace_bytes, void* stream);
int ttt_muon_update(const ttt_dims* dims, const float* theta_in, const float* grads, int n_grads,
                    float lr, float* theta_out, void* stream);

/* Read (Eq. 4): O = T_theta(Q) with frozen theta (query mode).  dims describe
 * Q's token count through n_views/grid/n_special; only n, heads, d, h are used. */
int ttt_read(const ttt_dims* dims, const uint16_t* Q, const float* theta, uint16_t* O,
             void* workspace, size_t workspace_bytes, void* stream);

/* The whole layer: ttt_write on (K, V) then ttt_read of Q with theta*. */
int ttt_layer(const ttt_dims* dims, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
              const float* conv_w, const float* theta0, float lr, int steps,
              float* theta_out, uint16_t* O, void* workspace, size_t workspace_bytes,
              void* stream);

/* The global attention layer with the TTT layer in place of softmax
 * attention (VGG-T^3 summary, Sec. 3 "QKV projection with normalization",
 * Eq. 1, with LN_q and LN_k replaced by L2 normalisation as in "The LayerNorm
 * removal"; then the output projection):
 *   q = L2(X Wq), k = L2(X Wk)  each (token, head) row of d scaled to unit
 *                               norm (a zero row stays zero),
 *   v = X Wv                    one tensor-core GEMM launch for all three, the
 *                               normalisation in its epilogue, q, k, v rounded
 *                               to bf16 once;
 *   the layer on (q, k, v)      inner = TTT_INNER_SGD: as ttt_layer;
 *                               TTT_INNER_MUON: as ttt_layer_muon;
 *   out = O Wo                  a tensor-core GEMM, bf16 output.
 * X, out: bf16 [n][C] with C = heads * d; Wq, Wk, Wv, Wo: bf16 [C][C] in the
 * row-vector form x W (no biases); conv_w, theta0, theta_out as for
 * ttt_layer.  Requires d = 64 and h <= 256 (the fused layer kernels); other
 * shapes return TTT_EUNSUPPORTED.  Workspace:
 * ttt_workspace_bytes(dims, TTT_OP_ATTENTION). */
int ttt_attention(const ttt_dims* dims, const uint16_t* X, const uint16_t* Wq, const uint16_t* Wk,
                  const uint16_t* Wv, const uint16_t* Wo, const float* conv_w, const float* theta0,
                  float lr, int steps, int inner, float* theta_out, uint16_t* out,
                  void* workspace, size_t workspace_bytes, void* stream);

/* C = A B on the library's tensor-core GEMM (the kernel of the projections
 * and of the wide-head path): bf16 operands, FP32 accumulation, bf16 output
 * rounded to nearest even.  A is M x K, stored row-major as [M][lda]
 * (a_layout 0) or as its transpose [K][lda] (a_layout 1); B is K x N, stored
 * as [K][ldb] (b_layout 0) or as its transpose [N][ldb] (b_layout 1, a linear
 * layer's [out][in] weight); C is [M][ldc].  M, N, K >= 1; N and the three
 * leading dimensions multiples of 8 elements; pointers 16-byte aligned (else
 * TTT_EALIGN).  Needs no workspace. */
int ttt_gemm_bf16(int M, int N, int K, const uint16_t* A, int64_t lda, int a_layout,
                  const uint16_t* B, int64_t ldb, int b_layout, uint16_t* C, int64_t ldc,
                  void* stream);

/* ttt_layer on HOST buffers: copies Q, K, V, conv_w, theta0 to device copies
 * inside the workspace, runs the layer, and copies theta* and O back to the
 * host buffers.  On the fused path the copies are pipelined: conv_w, theta0,
 * V and K go up first; Q then follows in up to 8 chunks of whole 128-token
 * tiles while the write runs; each chunk is read as soon as it has landed, and
 * its O goes back while the next chunk is read.  The call creates two helper
 * streams and their events, and destroys them before returning (CUDA
 * releases them once their work has completed).  They start after the work
 * enqueued earlier on `stream`, and `stream` waits for all of them, so the
 * call behaves as if everything ran on `stream`.  The wide-head path copies in
 * order on `stream`.  Returns once the work is enqueued; the host outputs are
 * valid after the stream synchronises.  Pinned host memory makes the copies
 * asynchronous and lets them overlap.
 * Workspace: ttt_workspace_bytes(dims, TTT_OP_LAYER_HOST). */
int ttt_layer_host(const ttt_dims* dims, const uint16_t* Q_host, const uint16_t* K_host,
                   const uint16_t* V_host, const float* conv_w_host,
                   const float* theta0_host, float lr, int steps, float* theta_out_host,
                   uint16_t* O_host, void* workspace, size_t workspace_bytes, void* stream);

/* ttt_read for callers that cannot allocate device memory — for example code
 * running under an allocator that forbids new device allocations, or a host
 * that has already handed all device memory to a pool it does not control.
 * The paper has no counterpart of this entry point; it is a packaging
 * convenience.  It takes no workspace: its scratch (the status word and the
 * fast-weight operand images, bf16 W1/W3 and f16 W2) lives in a fixed array of
 * TTT_NOALLOC_SCRATCH_BYTES
 * bytes that is part of the library, which every GPU that loads the library
 * holds until the process exits.  Shapes whose scratch would exceed it
 * (ttt_workspace_bytes(dims, TTT_OP_READ) > TTT_NOALLOC_SCRATCH_BYTES) return
 * TTT_EWORKSPACE.  The first call on each device looks up the array's device
 * address with that device current; make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's
 * contents: calls that may overlap on the GPU (other streams, other threads)
 * race and must be serialised by the caller.  Allocates nothing: no
 * cudaMalloc, no cudaFree, no allocating library routine. */
#define TTT_NOALLOC_SCRATCH_BYTES (4u << 20)
int ttt_read_noalloc(const ttt_dims* dims, const uint16_t* Q, const float* theta, uint16_t* O,
                     void* stream);

/* The device status of ttt_read_noalloc, which has no workspace to pass to
 * ttt_check_status: synchronises `stream`, then reads the status word that
 * the read's kernels keep at the start of the fixed scratch array of the
 * current device.  Returns TTT_OK, TTT_EDEVICE if a kernel recorded a fault
 * (a bounded wait that ran out; the word is then cleared and the read's O
 * must not be used), or TTT_ECUDA.  Each ttt_read_noalloc clears the word
 * when it starts, so call this after the read and before the next one on the
 * device.  Allocates nothing.  The array's device address is looked up once
 * per device; after cudaDeviceReset neither this call nor ttt_read_noalloc
 * may be used again in the process. */
int ttt_read_noalloc_status(void* stream);

/* Sets the limit, in SM clocks, of every bounded wait in the tensor-core
 * kernels launched after the call (process-wide); 0 (the default) selects the
 * built-in limit of 4e9 clocks (about two seconds).  A wait that runs out
 * makes its kernel record TTT_EDEVICE in the status word, stop every role,
 * let its copies and MMAs in flight finish, release its tensor memory and
 * return, so the context stays usable.  For tests of that path: a limit of a
 * few hundred clocks makes waits run out on any workload.  Returns TTT_OK, or
 * TTT_EINVAL for a negative limit. */
int ttt_set_wait_limit(long long clocks);

/* Synchronises `stream`, then reads the device status word of `workspace`:
 * TTT_OK, TTT_EDEVICE if a kernel recorded a fault (the word is cleared), or
 * TTT_ECUDA. */
int ttt_check_status(const void* workspace, void* stream);

/* Static description of a status code. */
const char* ttt_status_str(int status);

/* Per-kernel timing, for measurement only.  Between ttt_profile_start and
 * ttt_profile_stop the library records a CUDA event before and after every
 * kernel it launches (on the launch stream; calling threads must not overlap).
 * ttt_profile_stop synchronises those events and fills, per kernel kind k
 * (0 <= k < TTT_KERNEL_KINDS, named by ttt_kernel_name), the number of
 * launches and their summed device time in milliseconds.  At most 65536
 * launches are recorded per session; later ones are counted in `dropped`.
 * The "reduce_sgd" kind covers every theta-sized step kernel: the split-K
 * reduction with its SGD step, the fixed-order update of ttt_sgd_update and
 * the Newton-Schulz step of the Muon entry points. */
#define TTT_KERNEL_KINDS 12
typedef struct ttt_kernel_times {
  int32_t launches[TTT_KERNEL_KINDS];
  float total_ms[TTT_KERNEL_KINDS];
  int32_t dropped;
} ttt_kernel_times;
int ttt_profile_start(void);
int ttt_profile_stop(ttt_kernel_times* out);
const char* ttt_kernel_name(int kind);

#ifdef __cplusplus
}
#endif

#endif /* TTT_H_ */
