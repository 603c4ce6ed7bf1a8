// wide.cuh — the elementwise steps of the wide-head path.
//
// For head widths above 64 (the single 1024-wide head with h = 2048 of the
// 2000-view workload) the weights of one head no longer fit on chip, and every
// product of the layer is a plain dense GEMM over a token chunk:
//   Z1 = K W1, Z3 = K W3, Y = A W2, dA = E W2^T, dW1 = K^T dZ1, dW3 = K^T dZ3,
//   dW2 = A^T E
// (VGG-T$^3$: Offline Feed-Forward 3D Reconstruction at Scale, Sec. 3.4,
// Eq. 3-5, "TTT MLP Architecture and Inner Optimization").  The host runs
// them as bf16 library GEMMs with FP32 accumulation (dW accumulated in FP32
// over the chunks, Eq. 5); these kernels do everything between them:
//   wide_gate_kernel  A = silu(Z1) * Z3
//   wide_dz_kernel    dZ1 = dA Z3 s (1 + Z1 (1 - s)), dZ3 = dA Z1 s, s = sigmoid(Z1)
//   wide_cast_kernel  bf16 copy of theta (same layout) for the GEMM operands
//   wide_sgd_kernel   theta_out = theta_in - scale * dW of one head
//   wide_grad_kernel  dW of one head into a gradient in theta's layout
// All elementwise math is FP32 on bf16 storage, 8 elements (16 bytes) per
// thread and iteration; these steps are HBM-bound.
#pragma once
#include "sm100.cuh"

namespace ttt {

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16lo(w[i]);
    f[2 * i + 1] = bf16hi(w[i]);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  u.x = pack_bf16x2(f[0], f[1]);
  u.y = pack_bf16x2(f[2], f[3]);
  u.z = pack_bf16x2(f[4], f[5]);
  u.w = pack_bf16x2(f[6], f[7]);
  return u;
}

__device__ __forceinline__ float wide_sigmoid(float z) { return 1.f / (1.f + __expf(-z)); }

// A = silu(Z1) * Z3 over n8 groups of 8 bf16.
__global__ void wide_gate_kernel(const uint4* __restrict__ z1, const uint4* __restrict__ z3, uint4* __restrict__ a,
                                 long long n8) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float x1[8], x3[8], o[8];
    unpack8(z1[i], x1);
    unpack8(z3[i], x3);
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = x1[k] * wide_sigmoid(x1[k]) * x3[k];
    a[i] = pack8(o);
  }
}

// In place: Z1 <- dZ1 = dA Z3 s (1 + Z1 (1 - s)), Z3 <- dZ3 = dA Z1 s.
__global__ void wide_dz_kernel(uint4* __restrict__ z1, uint4* __restrict__ z3, const uint4* __restrict__ da,
                               long long n8) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float x1[8], x3[8], g[8], d1[8], d3[8];
    unpack8(z1[i], x1);
    unpack8(z3[i], x3);
    unpack8(da[i], g);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float s = wide_sigmoid(x1[k]);
      d1[k] = g[k] * x3[k] * s * (1.f + x1[k] * (1.f - s));
      d3[k] = g[k] * x1[k] * s;
    }
    z1[i] = pack8(d1);
    z3[i] = pack8(d3);
  }
}

// bf16 (round-to-nearest-even) copy of `count` floats.
__global__ void wide_cast_kernel(const float* __restrict__ theta, __nv_bfloat16* __restrict__ img, long long count) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    img[i] = __float2bfloat16_rn(theta[i]);
}

// theta_out = theta_in - scale * dW for head `head`; dW = [dW1 d*h | dW3 d*h |
// dW2 h*d] in the per-head layout of theta.  theta_out may alias theta_in.
__global__ void wide_sgd_kernel(const float* theta_in, float* theta_out, const float* __restrict__ dw, int heads,
                                int d, int h, int head, float scale) {
  const long long per = static_cast<long long>(d) * h;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < 3 * per;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long m = e / per, r = e % per;
    const long long off = m * heads * per + static_cast<long long>(head) * per + r;
    theta_out[off] = theta_in[off] - scale * dw[e];
  }
}

// grad = dW of head `head`, scattered into theta's per-head layout.
__global__ void wide_grad_kernel(float* grad, const float* __restrict__ dw, int heads, int d, int h, int head) {
  const long long per = static_cast<long long>(d) * h;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < 3 * per;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long m = e / per, r = e % per;
    grad[m * heads * per + static_cast<long long>(head) * per + r] = dw[e];
  }
}

}  // namespace ttt
