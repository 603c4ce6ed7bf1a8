// wide.cuh — the small kernels of the wide-head path.
//
// For head widths above 64 (the single 1024-wide head with h = 2048 of the
// 2000-view workload) the weights of one head no longer fit on chip, and every
// product of the layer is a plain dense GEMM over a token chunk:
//   Z1 = K W1, Z3 = K W3, Y = A W2, dA = E W2^T, dW1 = K^T dZ1, dW3 = K^T dZ3,
//   dW2 = A^T E
// (VGG-T$^3$: Offline Feed-Forward 3D Reconstruction at Scale, Sec. 3.4,
// Eq. 3-5, "TTT MLP Architecture and Inner Optimization").  They run on the
// tensor-core GEMM of gemm.cuh with the gate, the residual and the chain rule
// fused into its epilogues; these kernels do the rest:
//   wide_pack_kernel  bf16 operand images of theta, per head W13 [d][2 hidp]
//                     (hidden block j of 128 units: the W1 columns, then the
//                     W3 columns; units past h are zero) and W2 [h][d]
//   wide_sgd_kernel   theta_out = theta_in - scale * (sum of the split-K
//                     partials of dW, in split order) for one head
//   wide_grad_kernel  the same sum written into a gradient in theta's layout
//   ns_*_kernel       the elementwise steps of Newton-Schulz (Muon) on wide heads
#pragma once
#include "sm100.cuh"

namespace ttt {

__global__ void wide_pack_kernel(const float* __restrict__ theta, __nv_bfloat16* __restrict__ img13,
                                 __nv_bfloat16* __restrict__ img2, int heads, int d, int h, int hidp) {
  const long long n13 = static_cast<long long>(heads) * d * 2 * hidp;
  const long long n2 = static_cast<long long>(heads) * h * d;
  const long long hdh = static_cast<long long>(heads) * d * h;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n13 + n2;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    if (i < n13) {
      const int col = static_cast<int>(i % (2 * hidp));
      const long long r = i / (2 * hidp);          // head * d + row
      const int head = static_cast<int>(r / d), row = static_cast<int>(r % d);
      const int blk = col / 256, w = col % 256;
      const int hid = blk * 128 + (w & 127);
      float v = 0.f;
      if (hid < h) v = theta[(w < 128 ? 0 : hdh) + (static_cast<long long>(head) * d + row) * h + hid];
      img13[i] = __float2bfloat16_rn(v);
    } else {
      const long long k = i - n13;   // W2 in theta's own per-head [h][d] layout
      img2[k] = __float2bfloat16_rn(theta[2 * hdh + k]);
    }
  }
}

// theta_out = theta_in - scale * sum_{s < splits} dw[s] for head `head`; dw[s]
// = [dW1 d*h | dW3 d*h | dW2 h*d] in the per-head layout of theta.  theta_out
// may alias theta_in.
__global__ void wide_sgd_kernel(const float* theta_in, float* theta_out, const float* __restrict__ dw, int splits,
                                int heads, int d, int h, int head, float scale) {
  const long long per = static_cast<long long>(d) * h;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < 3 * per;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    float g = dw[e];
    for (int s = 1; s < splits; ++s) g += dw[s * 3 * per + e];
    const long long m = e / per, r = e % per;
    const long long off = m * heads * per + static_cast<long long>(head) * per + r;
    theta_out[off] = theta_in[off] - scale * g;
  }
}

// grad = sign * sum_{s < splits} dw[s] of head `head`, scattered into theta's per-head layout.
__global__ void wide_grad_kernel(float* grad, const float* __restrict__ dw, int splits, int heads, int d, int h,
                                 int head, float sign) {
  const long long per = static_cast<long long>(d) * h;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < 3 * per;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    float g = dw[e];
    for (int s = 1; s < splits; ++s) g += dw[s * 3 * per + e];
    const long long m = e / per, r = e % per;
    grad[m * heads * per + static_cast<long long>(head) * per + r] = sign * g;
  }
}

// ------------------------------------------------------------------ Muon on wide heads
// The pages' inner optimiser (Sec. 3.4, "TTT MLP Architecture and Inner
// Optimization": Muon, 5 Newton-Schulz iterations) for heads whose matrices
// no longer fit one CTA: per weight matrix, X_0 = G / ||G||_F, then
// X <- 1.5 X - 0.5 (X X^T) X five times, theta <- theta - lr X_5, with W2's
// h x d gradient transposed to d x h (the iteration commutes with
// transposition).  The products run on the tensor-core GEMM with FP32
// operands split into bf16 pairs, hi = bf16(x), lo = bf16(x - hi), and
// x y = hi_x hi_y + hi_x lo_y + lo_x hi_y (the lo_x lo_y term, ~2^-16 of the
// product, is dropped), accumulated in FP32: the splitting scheme of Henry,
// Tang and Heinecke (using bfloat16 for higher-precision computation, ARITH
// 2019), about 2^-16 relative per product instead of bf16's 2^-8.  Sums of
// squares are reduced in a fixed order, so the step is deterministic.
constexpr int kNsParts = 256;   // blocks of the norm reduction

__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16* hi, __nv_bfloat16* lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  *hi = h;
  *lo = __float2bfloat16_rn(x - __bfloat162float(h));
}

// X [d][h] = sum_r grads[r] of matrix m of head `head` (W2 transposed), and
// per-block partial sums of squares.  Launched with kNsParts blocks.
__global__ void ns_load_kernel(const float* __restrict__ grads, int n_grads, int heads, int d, int h, int head,
                               int m, float* __restrict__ X, float* __restrict__ partial) {
  const long long per = static_cast<long long>(d) * h;
  const long long count = 3LL * heads * per;
  const long long base = m * heads * per + static_cast<long long>(head) * per;
  float ss = 0.f;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < per;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long i = e / h, c = e % h;   // X[i][c]
    const long long o = base + (m < 2 ? i * h + c : c * d + i);
    float g = grads[o];
    for (int r = 1; r < n_grads; ++r) g += grads[static_cast<long long>(r) * count + o];
    X[e] = g;
    ss = fmaf(g, g, ss);
  }
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += red[w];
    partial[blockIdx.x] = t;
  }
}

// X *= 1 / ||X||_F (the partial sums added in block order; a zero matrix stays
// zero), then the bf16 pair of X.
__global__ void ns_normalise_kernel(float* __restrict__ X, const float* __restrict__ partial, long long count,
                                    __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo) {
  __shared__ float inv;
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int b = 0; b < kNsParts; ++b) t += partial[b];
    inv = t > 0.f ? 1.f / sqrtf(t) : 0.f;
  }
  __syncthreads();
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < count;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float x = X[e] * inv;
    X[e] = x;
    split_bf16(x, hi + e, lo + e);
  }
}

// The bf16 pair of an FP32 matrix.
__global__ void ns_split_kernel(const float* __restrict__ G, long long count, __nv_bfloat16* __restrict__ hi,
                                __nv_bfloat16* __restrict__ lo) {
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < count;
       e += static_cast<long long>(gridDim.x) * blockDim.x)
    split_bf16(G[e], hi + e, lo + e);
}

// X <- 1.5 X - 0.5 Y, Y = (X X^T) X; then the bf16 pair of X.
__global__ void ns_combine_kernel(float* __restrict__ X, const float* __restrict__ Y, long long count,
                                  __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo) {
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < count;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float x = 1.5f * X[e] - 0.5f * Y[e];
    X[e] = x;
    split_bf16(x, hi + e, lo + e);
  }
}

// theta_out = theta_in - lr X for matrix m of head `head` (W2 transposed back).
// theta_out may alias theta_in.
__global__ void ns_apply_kernel(const float* theta_in, float* theta_out, const float* __restrict__ X, int heads,
                                int d, int h, int head, int m, float lr) {
  const long long per = static_cast<long long>(d) * h;
  const long long base = m * heads * per + static_cast<long long>(head) * per;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < per;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long i = e / h, c = e % h;
    const long long o = base + (m < 2 ? i * h + c : c * d + i);
    theta_out[o] = theta_in[o] - lr * X[e];
  }
}

}  // namespace ttt
