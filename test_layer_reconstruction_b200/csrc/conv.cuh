// conv.cuh — ShortConv2D: depthwise 3x3 convolution of each view's patch grid
// of values (VGG-T$^3$: Offline Feed-Forward 3D Reconstruction at Scale,
// Sec. 3.4 "Non-Linear Spatial Mixing via ShortConv2D": reshape the value
// sequence to (N, H/p, W/p, d), convolve with a 3x3 filter, flatten; the
// convolution stays inside one image; camera and register tokens pass through
// unmixed, Appendix A).  Cross-correlation with zero padding, no bias,
// FP32 accumulation, bf16 round-to-nearest-even store.
//
// HBM-bound: every value is read once from DRAM and V' written once.  A
// thread owns 8 channels (one 16-byte vector) of one grid row of one view and
// sweeps the row left to right with a 3x3 window of vectors in registers, so
// each input vector is fetched by three threads (rows y-1, y, y+1) through
// L1/L2 and only once from DRAM.  A warp covers 32 consecutive vectors of a
// token (512 contiguous bytes); the next column is prefetched one step ahead.
#pragma once
#include "sm100.cuh"

namespace ttt {

struct ConvParams {
  const uint4* V;      // [n][C/8] vectors of 8 bf16
  const float* w;      // [C][3][3]
  uint4* out;          // [n][C/8]
  int n_views, gh, gw, n_special, C;
};

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
  f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
}

// grid: (ceil(C/8 / blockDim.x), grid_h + 1, n_views); blockIdx.y == grid_h copies special tokens.
__global__ void __launch_bounds__(128) shortconv_kernel(const ConvParams p) {
  const int G8 = p.C / 8;
  const int cg = blockIdx.x * blockDim.x + threadIdx.x;
  if (cg >= G8) return;
  const int y = blockIdx.y;
  const long long T = static_cast<long long>(p.n_special) + static_cast<long long>(p.gh) * p.gw;
  const long long vbase = static_cast<long long>(blockIdx.z) * T;
  if (y == p.gh) {
    for (int s = 0; s < p.n_special; ++s) {
      const long long t = vbase + s;
      p.out[t * G8 + cg] = __ldg(p.V + t * G8 + cg);
    }
    return;
  }
  float w[8][9];
#pragma unroll
  for (int c = 0; c < 8; ++c)
#pragma unroll
    for (int k = 0; k < 9; ++k) w[c][k] = __ldg(p.w + static_cast<size_t>(cg * 8 + c) * 9 + k);

  const long long gbase = vbase + p.n_special;  // first patch token of the view
  const uint4 zero = make_uint4(0, 0, 0, 0);
  auto ld = [&](int yy, int xx) -> uint4 {
    if (yy < 0 || yy >= p.gh || xx < 0 || xx >= p.gw) return zero;
    return __ldg(p.V + (gbase + static_cast<long long>(yy) * p.gw + xx) * G8 + cg);
  };
  // columns x-1, x, x+1 (and the prefetched x+2) of rows y-1, y, y+1
  uint4 c0[3], c1[3], c2[3], c3[3];
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    c0[a] = zero;
    c1[a] = ld(y - 1 + a, 0);
    c2[a] = ld(y - 1 + a, 1);
  }
  for (int x = 0; x < p.gw; ++x) {
#pragma unroll
    for (int a = 0; a < 3; ++a) c3[a] = ld(y - 1 + a, x + 2);
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      float f0[8], f1[8], f2[8];
      unpack8(c0[a], f0);
      unpack8(c1[a], f1);
      unpack8(c2[a], f2);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        acc[c] = fmaf(w[c][3 * a + 0], f0[c], acc[c]);
        acc[c] = fmaf(w[c][3 * a + 1], f1[c], acc[c]);
        acc[c] = fmaf(w[c][3 * a + 2], f2[c], acc[c]);
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    p.out[(gbase + static_cast<long long>(y) * p.gw + x) * G8 + cg] = o;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      c0[a] = c1[a];
      c1[a] = c2[a];
      c2[a] = c3[a];
    }
  }
}

}  // namespace ttt
