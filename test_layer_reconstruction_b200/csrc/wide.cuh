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

// grad = sum_{s < splits} dw[s] of head `head`, scattered into theta's per-head layout.
__global__ void wide_grad_kernel(float* grad, const float* __restrict__ dw, int splits, int heads, int d, int h,
                                 int head) {
  const long long per = static_cast<long long>(d) * h;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < 3 * per;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    float g = dw[e];
    for (int s = 1; s < splits; ++s) g += dw[s * 3 * per + e];
    const long long m = e / per, r = e % per;
    grad[m * heads * per + static_cast<long long>(head) * per + r] = g;
  }
}

}  // namespace ttt
