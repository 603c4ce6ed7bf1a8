// conv.cuh — ShortConv2D: depthwise 3x3 convolution of each view's patch grid
// of values (VGG-T$^3$: Offline Feed-Forward 3D Reconstruction at Scale,
// Sec. 3.4 "Non-Linear Spatial Mixing via ShortConv2D": reshape the value
// sequence to (N, H/p, W/p, d), convolve with a 3x3 filter, flatten; the
// convolution stays inside one image; camera and register tokens pass through
// unmixed, Appendix A).  Cross-correlation with zero padding, no bias,
// FP32 accumulation, bf16 round-to-nearest-even store (widened exactly to
// f16, the backward kernel's operand type, in the dot-product-loss path).
//
// HBM-bound: every value is read once from DRAM and V' written once.  A
// thread owns 4 channels (one 8-byte vector) of a band of kConvBand grid rows
// of one view and sweeps the band left to right, reading the kConvBand + 2
// input rows around it.  A warp covers 32 consecutive vectors of a token (256
// contiguous bytes).
//
// What limits such a sweep is the number of bytes in flight per SM, not the
// arithmetic: the threads of neighbouring bands request a shared row from L2
// at about the same moment, so only part of the requests are new DRAM bytes.
// Bands of 2 rows cut the requests per row from three to two, and each thread
// streams its input columns through a private ring of kConvRing columns in
// shared memory with cp.async (no registers held while a copy is in flight;
// the thread reads back only what it copied itself, so cp.async.wait_group is
// the only synchronisation).  The window lives in registers as FP32: columns
// x-1, x, x+1 of the band's input rows; only the column that enters it is read
// and unpacked, and the sweep is unrolled by three so the window's roles
// rotate without register moves.
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

// Two FP32 lanes in one 64-bit register pair, for the packed f32x2 FMA of
// sm_100 (two independent fma.rn.f32 per instruction, bitwise equal to them).
__device__ __forceinline__ uint64_t f32x2_from_bf16x2(uint32_t v) {
  uint64_t r;
  asm("{ .reg .b32 l, h; shl.b32 l, %1, 16; and.b32 h, %1, 0xffff0000; mov.b64 %0, {l, h}; }" : "=l"(r) : "r"(v));
  return r;
}
__device__ __forceinline__ uint64_t f32x2_make(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f32x2_fma(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ uint32_t bf16x2_from_f32x2(uint64_t v) {
  uint32_t r;
  asm("{ .reg .b32 l, h; mov.b64 {l, h}, %1; cvt.rn.bf16x2.f32 %0, h, l; }" : "=r"(r) : "l"(v));
  return r;
}
// Two bf16 values -> two f16 values (rounded to nearest; exact in f16's normal range).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_exact(uint32_t v) {
  return pack_f16x2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

constexpr int kConvRing = 8;   // columns in the per-thread shared-memory ring
constexpr int kConvBand = 3;   // output rows per thread
static_assert((kConvRing & (kConvRing - 1)) == 0, "ring slots are masked");

__host__ __device__ constexpr size_t conv_smem_bytes(int threads) {
  return static_cast<size_t>(kConvRing) * (kConvBand + 2) * threads * sizeof(uint2);
}

// 8-byte asynchronous copy global -> shared; src_bytes == 0 writes zeros and
// reads nothing.
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Persistent blocks: grid = (blocks, ceil(C/4 / blockDim.x)).  A thread
// computes a band of R output rows (y0 .. y0+R-1) from the R+2 input rows
// around it, so a row is requested from L2 (R+2)/R times instead of three.
// Block b walks the items b, b + gridDim.x, ... of the (view, band) space,
// band == bands meaning the view's special tokens.  A thread's 36 weights are
// loaded once per block instead of once per band.
template <int R, bool F16OUT>
__global__ void __launch_bounds__(kConvThreads, 2) shortconv_kernel(const ConvParams p) {
  constexpr int NR = R + 2;   // input rows of a band
  extern __shared__ __align__(16) uint8_t conv_smem[];
  const int G4 = p.C / 4;
  const int cg = blockIdx.y * blockDim.x + threadIdx.x;
  if (cg >= G4) return;
  const long long T = static_cast<long long>(p.n_special) + static_cast<long long>(p.gh) * p.gw;
  const int bands = (p.gh + R - 1) / R;
  const long long items = static_cast<long long>(p.n_views) * (bands + 1);
  // weights of channel pairs (4cg, 4cg+1) and (4cg+2, 4cg+3), per tap
  uint64_t wp[2][9];
#pragma unroll
  for (int q = 0; q < 2; ++q)
#pragma unroll
    for (int k = 0; k < 9; ++k)
      wp[q][k] = f32x2_make(__ldg(p.w + static_cast<size_t>(cg * 4 + 2 * q) * 9 + k),
                            __ldg(p.w + static_cast<size_t>(cg * 4 + 2 * q + 1) * 9 + k));
  // ring slot s, band row i of this thread: consecutive threads, consecutive 8 bytes
  const uint32_t ring = smem_u32(conv_smem) + threadIdx.x * 8u;
  const uint32_t row_stride = blockDim.x * 8u, slot_stride = NR * row_stride;

  for (long long item = blockIdx.x; item < items; item += gridDim.x) {
    const int view = static_cast<int>(item / (bands + 1));
    const int band = static_cast<int>(item % (bands + 1));
    const long long vbase = static_cast<long long>(view) * T;
    if (band == bands) {
      for (int s = 0; s < p.n_special; ++s) {
        const long long t = vbase + s;
        const uint2 v = __ldg(p.V + t * G4 + cg);
        p.out[t * G4 + cg] = F16OUT ? make_uint2(bf16x2_to_f16x2_exact(v.x), bf16x2_to_f16x2_exact(v.y)) : v;
      }
      continue;
    }
    const int y0 = band * R;
    const long long gbase = vbase + p.n_special;  // first patch token of the view
    // rows outside the grid are fetched as zeros (source size 0) from row y0
    uint32_t row_bytes[NR];
    const uint2* rowp[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int yy = y0 - 1 + i;
      const bool ok = yy >= 0 && yy < p.gh;
      row_bytes[i] = ok ? 8u : 0u;
      rowp[i] = p.V + (gbase + static_cast<long long>(ok ? yy : y0) * p.gw) * G4 + cg;
    }
    bool out_ok[R];
#pragma unroll
    for (int r = 0; r < R; ++r) out_ok[r] = y0 + r < p.gh;
    uint2* outp = p.out + (gbase + static_cast<long long>(y0) * p.gw) * G4 + cg;
    const long long out_row = static_cast<long long>(p.gw) * G4;
    auto slot_of = [&](int xx) { return ring + (static_cast<uint32_t>(xx) & (kConvRing - 1)) * slot_stride; };
    // column xx into its ring slot, one commit group per column (empty past the grid)
    auto fetch = [&](int xx) {
      if (xx < p.gw) {
        const uint32_t slot = slot_of(xx);
        const long long off = static_cast<long long>(xx) * G4;
#pragma unroll
        for (int i = 0; i < NR; ++i) cp_async8(slot + i * row_stride, rowp[i] + off, row_bytes[i]);
      }
      cp_async_commit();
    };
    // column xx from its ring slot as FP32 pairs (the caller waited for its group)
    auto take = [&](int xx, uint64_t (&dst)[NR][2]) {
      if (xx < p.gw) {
        const uint32_t slot = slot_of(xx);
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          uint32_t lo, hi;
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(lo), "=r"(hi) : "r"(slot + i * row_stride));
          dst[i][0] = f32x2_from_bf16x2(lo);
          dst[i][1] = f32x2_from_bf16x2(hi);
        }
      } else {
#pragma unroll
        for (int i = 0; i < NR; ++i) dst[i][0] = dst[i][1] = 0ull;
      }
    };
    // One output column x of the band from the window (L, M, R) = columns
    // (x-1, x, x+1).  First the slot of column x-1 (read at least one step
    // earlier) is refilled with column x+kConvRing-1; after the outputs,
    // column x+2 replaces L (it becomes the right column of x+1's window).
    // Pending then are columns x+2 .. x+kConvRing-1, so column x+2 is
    // complete once at most kConvRing-3 groups remain.  Per channel the taps
    // are summed row by row, left to right.
    auto step = [&](uint64_t (&L)[NR][2], uint64_t (&M)[NR][2], uint64_t (&Rt)[NR][2], int x) {
      fetch(x + kConvRing - 1);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            f32x2_fma(acc[q], wp[q][3 * a + 0], L[r + a][q]);
            f32x2_fma(acc[q], wp[q][3 * a + 1], M[r + a][q]);
            f32x2_fma(acc[q], wp[q][3 * a + 2], Rt[r + a][q]);
          }
        // f16 output: V' is rounded to bf16 first, as every path stores it, then
        // widened exactly, so it equals the bf16 output converted to f16.
        if (out_ok[r]) {
          const uint2 b = make_uint2(bf16x2_from_f32x2(acc[0]), bf16x2_from_f32x2(acc[1]));
          outp[r * out_row + static_cast<long long>(x) * G4] =
              F16OUT ? make_uint2(bf16x2_to_f16x2_exact(b.x), bf16x2_to_f16x2_exact(b.y)) : b;
        }
      }
      cp_async_wait<kConvRing - 3>();
      take(x + 2, L);
    };
    uint64_t fa[NR][2], fb[NR][2], fc[NR][2];
    for (int xx = 0; xx < kConvRing - 1; ++xx) fetch(xx);   // columns 0 .. kConvRing-2
#pragma unroll
    for (int i = 0; i < NR; ++i) fa[i][0] = fa[i][1] = 0ull;   // column -1: zero padding
    cp_async_wait<kConvRing - 3>();                              // columns 0 and 1 complete
    take(0, fb);
    take(1, fc);
    for (int x = 0; x < p.gw; x += 3) {
      step(fa, fb, fc, x);
      if (x + 1 >= p.gw) break;
      step(fb, fc, fa, x + 1);
      if (x + 2 >= p.gw) break;
      step(fc, fa, fb, x + 2);
    }
    cp_async_wait<0>();   // no copy of this band may land in the next band's ring
  }
}

}  // namespace ttt
