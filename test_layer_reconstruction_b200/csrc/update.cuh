// update.cuh — the SGD step on the fast weights and the bf16 operand images.
//
// reduce_sgd: g = sum of the backward kernel's partials of a (head, hidden
// slice) in CTA-group order (a fixed order, so the step is deterministic; Eq. 5 of
// VGG-T$^3$: Offline Feed-Forward 3D Reconstruction at Scale says the full
// gradient is exactly the sum of the chunk gradients), then
//   theta_out = theta_in - lr * (2/n) * g
// (plain SGD on the mean-squared loss; the 2/n of its gradient is applied
// here).  theta_out may alias theta_in: each element is read and written by
// one thread.  With theta_in null the kernel writes g itself (the gradient of
// (1/2) sum_i ||T(k_i) - v'_i||^2 over the call's tokens) into theta_out, for
// a write whose tokens are sharded over several processes.
//
// sgd_sum: theta_out = theta_in - scale * (g_0 + g_1 + ... + g_{r-1}) over r
// gathered gradients, summed in index order for every element, so every
// process that applies it gets the same bits.
//
// pack_images: theta (f32) -> round-to-nearest-even operand images, hidden
// units padded with zeros up to HIDP:
//   W13 image (bf16), per head, laid out as the forward kernel's shared-memory
//     tile (rows of D elements, swizzled by 8-row atoms): for every 32-unit
//     sub-chunk s, 32 rows of W1^T (hidden s*32+r) then 32 rows of W3^T.
//   W2 image (f16, same tiling), per head: row j = W2[j][:]; the forward
//     kernel's gate operand is f16.
//   WT image (bf16, plain rows; write path only), per head and hidden unit r:
//     [W1^T row r / 2 | W3^T row r | W2 row r], the backward kernel's weight
//     rows (halving is exact in bf16).
#pragma once
#include "bwd.cuh"

namespace ttt {

struct UpdateParams {
  const float* partials;
  const float* theta_in;   // null: write the gradient itself
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
    p.theta_out[off] = m == 0 ? 0.5f * g : g;
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

struct PackParams {
  const float* theta;
  __nv_bfloat16* w13_img;
  __half* w2h_img;
  __nv_bfloat16* wt_img;  // null: not written
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
    p.wt_img[k] = __float2bfloat16_rn(v);
  }
}

}  // namespace ttt
