// conv.cuh — ShortConv2D: depthwise 3x3 convolution of each view's patch grid
// of values (VGG-T$^3$: Offline Feed-Forward 3D Reconstruction at Scale,
// Sec. 3.4 "Non-Linear Spatial Mixing via ShortConv2D": reshape the value
// sequence to (N, H/p, W/p, d), convolve with a 3x3 filter, flatten; the
// convolution stays inside one image; camera and register tokens pass through
// unmixed, Appendix A).  Cross-correlation with zero padding, no bias,
// FP32 accumulation, bf16 round-to-nearest-even store.
//
// HBM-bound: every value is read once from DRAM and V' written once.  A
// thread owns 4 channels (one 8-byte vector) of one grid row of one view and
// sweeps the row left to right with a 3x3 window of vectors in registers, so
// each input vector is fetched by three threads (rows y-1, y, y+1) through
// L1/L2 and only once from DRAM.  A warp covers 32 consecutive vectors of a
// token (256 contiguous bytes).  Columns x+1 and x+2 are in flight while
// column x is computed; 4 channels per thread keep the weights to 36
// registers so three 256-thread blocks fit per SM.
#pragma once
#include "sm100.cuh"

namespace ttt {

constexpr int kConvThreads = 256;

struct ConvParams {
  const uint2* V;      // [n][C/4] vectors of 4 bf16
  const float* w;      // [C][3][3]
  uint2* out;          // [n][C/4]
  int n_views, gh, gw, n_special, C;
};

__device__ __forceinline__ void unpack4(const uint2& u, float (&f)[4]) {
  f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
}

// Persistent blocks: grid = (blocks, ceil(C/4 / blockDim.x)).  Block b walks
// the items b, b + gridDim.x, ... of the (view, grid row) space, item row ==
// grid_h meaning the view's special tokens.  A thread's 36 weights are loaded
// once per block instead of once per row.
__global__ void __launch_bounds__(kConvThreads, 3) shortconv_kernel(const ConvParams p) {
  const int G4 = p.C / 4;
  const int cg = blockIdx.y * blockDim.x + threadIdx.x;
  if (cg >= G4) return;
  const long long T = static_cast<long long>(p.n_special) + static_cast<long long>(p.gh) * p.gw;
  const long long items = static_cast<long long>(p.n_views) * (p.gh + 1);
  float w[4][9];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int k = 0; k < 9; ++k) w[c][k] = __ldg(p.w + static_cast<size_t>(cg * 4 + c) * 9 + k);
  const uint2 zero = make_uint2(0, 0);

  for (long long item = blockIdx.x; item < items; item += gridDim.x) {
    const int view = static_cast<int>(item / (p.gh + 1));
    const int y = static_cast<int>(item % (p.gh + 1));
    const long long vbase = static_cast<long long>(view) * T;
    if (y == p.gh) {
      for (int s = 0; s < p.n_special; ++s) {
        const long long t = vbase + s;
        p.out[t * G4 + cg] = __ldg(p.V + t * G4 + cg);
      }
      continue;
    }
    const long long gbase = vbase + p.n_special;  // first patch token of the view
    const bool row_ok[3] = {y >= 1, true, y + 1 < p.gh};
    auto ld = [&](int a, int xx) -> uint2 {
      if (!row_ok[a] || xx >= p.gw) return zero;
      return __ldg(p.V + (gbase + static_cast<long long>(y - 1 + a) * p.gw + xx) * G4 + cg);
    };
    // columns x-1, x, x+1 of rows y-1, y, y+1, and x+2 in flight
    uint2 c0[3], c1[3], c2[3], c3[3];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      c0[a] = zero;
      c1[a] = ld(a, 0);
      c2[a] = ld(a, 1);
      c3[a] = ld(a, 2);
    }
    for (int x = 0; x < p.gw; ++x) {
      uint2 c4[3];
#pragma unroll
      for (int a = 0; a < 3; ++a) c4[a] = ld(a, x + 3);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int a = 0; a < 3; ++a) {
        float f0[4], f1[4], f2[4];
        unpack4(c0[a], f0);
        unpack4(c1[a], f1);
        unpack4(c2[a], f2);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[c] = fmaf(w[c][3 * a + 0], f0[c], acc[c]);
          acc[c] = fmaf(w[c][3 * a + 1], f1[c], acc[c]);
          acc[c] = fmaf(w[c][3 * a + 2], f2[c], acc[c]);
        }
      }
      uint2 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      p.out[(gbase + static_cast<long long>(y) * p.gw + x) * G4 + cg] = o;
#pragma unroll
      for (int a = 0; a < 3; ++a) {
        c0[a] = c1[a];
        c1[a] = c2[a];
        c2[a] = c3[a];
        c3[a] = c4[a];
      }
    }
  }
}

}  // namespace ttt
