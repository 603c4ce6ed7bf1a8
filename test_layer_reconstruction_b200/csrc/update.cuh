// update.cuh — the SGD step on the fast weights and the bf16 operand images.
//
// reduce_sgd: g = sum of the backward kernel's partials of a (head, hidden
// slice) in CTA-group order (a fixed order, so the step is deterministic; Eq. 5 of
// VGG-T$^3$: Offline Feed-Forward 3D Reconstruction at Scale says the full
// gradient is exactly the sum of the chunk gradients), then
//   theta_out = theta_in - lr * (2/n) * g
// (plain SGD on the mean-squared loss; the 2/n of its gradient is applied
// here).  theta_out may alias theta_in: each element is read and written by
// one thread.  With theta_in null the kernel writes scale * g into theta_out
// instead: with scale 1 and E = T(K) - V' that is the gradient of
// (1/2) sum_i ||T(k_i) - v'_i||^2 over the call's tokens; with scale -1 and
// E = V' it is the gradient of the dot-product loss sum -sum_i <T(k_i), v'_i>.
//
// sgd_sum: theta_out = theta_in - scale * (g_0 + g_1 + ... + g_{r-1}) over r
// gathered gradients, summed in index order for every element, so every
// process that applies it gets the same bits.
//
// pack_images: theta (f32) -> round-to-nearest-even operand images, hidden
// units padded with zeros up to HIDP:
//   W13 image (bf16), per head, laid out as the forward kernel's shared-memory
//     tile (rows of D elements, swizzled by 8-row atoms): for every 32-unit
//     sub-chunk s, 32 rows of W1^T / 2 (hidden s*32+r; halving is exact) then
//     32 rows of W3^T.
//   W2 image (f16, same tiling), per head: row j = W2[j][:]; the forward
//     kernel's gate operand is f16.
//   WT image (f16, plain rows; write path only), per head and hidden unit r:
//     [W1^T row r / 2 | W3^T row r | W2 row r], the backward kernel's weight
//     rows (halving is exact).
#pragma once
#include "bwd.cuh"

namespace ttt {

struct UpdateParams {
  const float* partials;
  const float* theta_in;   // null: write scale * g
  float* theta_out;
  int heads, d, h, slices, units, max_contrib;
  long long n_items;   // heads * units
  int grid;            // CTA groups of the backward kernel
  float scale;         // lr * 2 / n
};

__global__ void reduce_sgd_kernel(const UpdateParams p) {
  const int D = p.d;
  const long long per_pair = 3LL * 128 * D;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long pairs = static_cast<long long>(p.heads) * p.slices;
  if (idx >= pairs * per_pair) return;
  const long long pair = idx / per_pair;
  const int e = static_cast<int>(idx % per_pair);
  const int m = e / (128 * D);
  const int hr = (e / D) % 128;
  const int i = e % D;
  const int head = static_cast<int>(pair / p.slices);
  const int hid = static_cast<int>(pair % p.slices) * 128 + hr;
  if (hid >= p.h) return;                                   // zero padding
  const long long first = static_cast<long long>(head) * p.units;
  const long long c_lo = owner_cta(first, p.n_items, p.grid);
  const long long c_hi = owner_cta(first + p.units - 1, p.n_items, p.grid);
  const float* src = p.partials + static_cast<size_t>(pair) * p.max_contrib * per_pair + e;
  float g = 0.f;
  for (long long c = 0; c <= c_hi - c_lo; ++c) g += src[c * per_pair];
  const size_t hdh = static_cast<size_t>(p.heads) * D * p.h;
  size_t off;
  if (m == 0) off = static_cast<size_t>(head) * D * p.h + static_cast<size_t>(i) * p.h + hid;
  else if (m == 1) off = hdh + static_cast<size_t>(head) * D * p.h + static_cast<size_t>(i) * p.h + hid;
  else off = 2 * hdh + static_cast<size_t>(head) * p.h * D + static_cast<size_t>(hid) * D + i;
  // the backward kernel accumulates 2 dW1^T (its chain rule runs on z1/2): halve it, exactly
  if (p.theta_in)
    p.theta_out[off] = p.theta_in[off] - (m == 0 ? 0.5f * p.scale : p.scale) * g;
  else
    p.theta_out[off] = p.scale * (m == 0 ? 0.5f * g : g);
}

// theta_out = theta_in - scale * sum_r grads[r * count + e], r in order.
__global__ void sgd_sum_kernel(const float* theta_in, const float* __restrict__ grads, int n_grads,
                               long long count, float scale, float* theta_out) {
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < count;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    float g = grads[e];
    for (int r = 1; r < n_grads; ++r) g += grads[static_cast<long long>(r) * count + e];
    theta_out[e] = theta_in[e] - scale * g;
  }
}

// bf16 -> f16 (round to nearest; exact in f16's normal range), 8 values per
// thread and iteration.
__global__ void bf16_to_f16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, long long n8) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 v = src[i];
    dst[i] = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
  }
}

struct PackParams {
  const float* theta;
  __nv_bfloat16* w13_img;
  __half* w2h_img;
  __half* wt_img;         // null: not written
  int heads, d, h, hidp;
};

// One thread per (image, head, row, element).
__global__ void pack_images_kernel(const PackParams p) {
  const int D = p.d, SW = 2 * D;
  const long long n13 = static_cast<long long>(p.heads) * 2 * p.hidp * D;
  const long long n2 = static_cast<long long>(p.heads) * p.hidp * D;
  const long long nt = p.wt_img ? 3 * n2 : 0;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n13 + n2 + nt) return;
  const size_t hdh = static_cast<size_t>(p.heads) * D * p.h;
  if (idx < n13) {
    const int col = static_cast<int>(idx % D);
    const long long r_all = idx / D;
    const int R = static_cast<int>(r_all % (2 * p.hidp));
    const int head = static_cast<int>(r_all / (2 * p.hidp));
    const int sub = R / 64, rr = R % 64;
    const int hid = sub * 32 + (rr & 31);
    float v = 0.f;
    if (hid < p.h) {
      const float* w = p.theta + (rr < 32 ? 0 : hdh);
      v = w[static_cast<size_t>(head) * D * p.h + static_cast<size_t>(col) * p.h + hid];
      if (rr < 32) v *= 0.5f;   // W1 halved (exact): the forward gate reads u = z1/2
    }
    const uint32_t off = swz(static_cast<uint32_t>(R) * SW + col * 2, SW);
    *reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(p.w13_img + static_cast<size_t>(head) * 2 * p.hidp * D) + off) =
        __float2bfloat16_rn(v);
  } else if (idx < n13 + n2) {
    const long long k = idx - n13;
    const int col = static_cast<int>(k % D);
    const long long r_all = k / D;
    const int R = static_cast<int>(r_all % p.hidp);
    const int head = static_cast<int>(r_all / p.hidp);
    float v = 0.f;
    if (R < p.h) v = p.theta[2 * hdh + static_cast<size_t>(head) * p.h * D + static_cast<size_t>(R) * D + col];
    const uint32_t off = swz(static_cast<uint32_t>(R) * SW + col * 2, SW);
    *reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(p.w2h_img + static_cast<size_t>(head) * p.hidp * D) + off) =
        __float2half_rn(v);
  } else {
    // WT: element idx = ((head * HIDP + r) * 3 + m) * D + col
    const long long k = idx - n13 - n2;
    const int col = static_cast<int>(k % D);
    const int m = static_cast<int>((k / D) % 3);
    const long long hr = k / (3LL * D);
    const int r = static_cast<int>(hr % p.hidp);
    const int head = static_cast<int>(hr / p.hidp);
    float v = 0.f;
    if (r < p.h) {
      if (m < 2) {
        v = p.theta[m * hdh + static_cast<size_t>(head) * D * p.h + static_cast<size_t>(col) * p.h + r];
        if (m == 0) v *= 0.5f;   // W1^T / 2: the backward kernel's products give z1/2 directly
      } else {
        v = p.theta[2 * hdh + static_cast<size_t>(head) * p.h * D + static_cast<size_t>(r) * D + col];
      }
    }
    p.wt_img[k] = __float2half_rn(v);
  }
}

// ------------------------------------------------------------------ Muon
// The pages' inner optimiser (VGG-T$^3$: Offline Feed-Forward 3D
// Reconstruction at Scale, Sec. 3.4, "TTT MLP Architecture and Inner
// Optimization": Muon, 5 Newton-Schulz iterations): per weight matrix G of a
// head, X_0 = G / ||G||_F, then X <- 1.5 X - 0.5 X X^T X five times (the
// cubic iteration for the orthogonal polar factor; the pages give no
// polynomial), and theta <- theta - lr * X_5.
//
// One CTA per (head, matrix).  X is held as d x h (W2's h x d gradient
// transposed: the iteration commutes with transposition), in shared memory
// transposed, Xt[c][i] (c < h, i < d), so both products read float4 rows:
//   Gram = X X^T        (d x d): Gram[i][j] = sum_c Xt[c][i] Xt[c][j]
//   X   <- 1.5 X - 0.5 Gram X:   Xt[c][i] = 1.5 Xt[c][i] - 0.5 sum_j Gram[j][i] Xt[c][j]
// FP32 FMAs; the whole iteration is ~10 MFLOP per matrix at d=64, h=256,
// too small for the tensor cores to pay off.
constexpr int kNsThreads = 256;
constexpr int kNsIters = 5;

__host__ __device__ constexpr size_t ns_smem_bytes(int d, int h) {
  return (static_cast<size_t>(h) * d + static_cast<size_t>(d) * d + 32) * sizeof(float);
}

struct MuonParams {
  const float* theta_in;
  const float* grads;     // n_grads gradients in theta's layout, summed in order
  float* theta_out;
  int n_grads, heads, d, h;
  float lr;
};

__global__ void __launch_bounds__(kNsThreads) muon_update_kernel(const MuonParams p) {
  extern __shared__ __align__(16) float ns_smem[];
  const int D = p.d, Hh = p.h;
  const int head = blockIdx.x / 3, m = blockIdx.x % 3;
  float* Xt = ns_smem;                       // [h][d]
  float* gram = ns_smem + Hh * D;            // [d][d]
  float* red = gram + D * D;                 // 32 partial sums
  const long long per = static_cast<long long>(D) * Hh;
  const long long count = 3LL * p.heads * per;
  const long long base = m * p.heads * per + head * per;
  // element (i, c) of X = G (m < 2, G is [d][h]) or G^T (m == 2, G is [h][d])
  auto goff = [&](int i, int c) -> long long {
    return base + (m < 2 ? static_cast<long long>(i) * Hh + c : static_cast<long long>(c) * D + i);
  };
  float ss = 0.f;
  for (int e = threadIdx.x; e < D * Hh; e += blockDim.x) {
    const int c = e / D, i = e % D;
    const long long o = goff(i, c);
    float g = p.grads[o];
    for (int r = 1; r < p.n_grads; ++r) g += p.grads[static_cast<long long>(r) * count + o];
    Xt[c * D + i] = g;
    ss = fmaf(g, g, ss);
  }
  // ||G||_F
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float nrm = sqrtf(red[0]);
  const float inv = nrm > 0.f ? 1.f / nrm : 0.f;
  for (int e = threadIdx.x; e < D * Hh; e += blockDim.x) Xt[e] *= inv;
  __syncthreads();

  const int D4 = D / 4;
  for (int it = 0; it < kNsIters; ++it) {
    // Gram[i][j0..j0+3] = sum_c Xt[c][i] * Xt[c][j0..j0+3]
    for (int t = threadIdx.x; t < D * D4; t += blockDim.x) {
      const int i = t / D4, j0 = (t % D4) * 4;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      for (int c = 0; c < Hh; ++c) {
        const float xi = Xt[c * D + i];
        const float4 xj = *reinterpret_cast<const float4*>(Xt + c * D + j0);
        a0 = fmaf(xi, xj.x, a0); a1 = fmaf(xi, xj.y, a1); a2 = fmaf(xi, xj.z, a2); a3 = fmaf(xi, xj.w, a3);
      }
      *reinterpret_cast<float4*>(gram + i * D + j0) = make_float4(a0, a1, a2, a3);
    }
    __syncthreads();
    // new Xt[c][i0..i0+3] = 1.5 Xt - 0.5 sum_j Gram[j][i0..i0+3] Xt[c][j]  (Gram is symmetric)
    constexpr int kMaxItems = 16;   // (h * d / 4) / kNsThreads at d = 64, h = 256 (the host checks d, h)
    float4 acc[kMaxItems];
#pragma unroll
    for (int k = 0; k < kMaxItems; ++k) {
      const int t = threadIdx.x + k * kNsThreads;
      if (t < Hh * D4) {
        const int c = t / D4, i0 = (t % D4) * 4;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        for (int j = 0; j < D; ++j) {
          const float xj = Xt[c * D + j];
          const float4 gj = *reinterpret_cast<const float4*>(gram + j * D + i0);
          a0 = fmaf(gj.x, xj, a0); a1 = fmaf(gj.y, xj, a1); a2 = fmaf(gj.z, xj, a2); a3 = fmaf(gj.w, xj, a3);
        }
        const float4 x = *reinterpret_cast<const float4*>(Xt + c * D + i0);
        acc[k] = make_float4(1.5f * x.x - 0.5f * a0, 1.5f * x.y - 0.5f * a1, 1.5f * x.z - 0.5f * a2,
                             1.5f * x.w - 0.5f * a3);
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kMaxItems; ++k) {
      const int t = threadIdx.x + k * kNsThreads;
      if (t < Hh * D4) *reinterpret_cast<float4*>(Xt + (t / D4) * D + (t % D4) * 4) = acc[k];
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < D * Hh; e += blockDim.x) {
    const int c = e / D, i = e % D;
    const long long o = goff(i, c);
    p.theta_out[o] = p.theta_in[o] - p.lr * Xt[c * D + i];
  }
}

}  // namespace ttt
