// bwd.cuh — gradient of the mean-squared TTT loss w.r.t. the SwiGLU fast
// weights, as split-K partial sums over token ranges.
//
// For the loss L = (1/n) sum_i ||T(k_i) - v'_i||^2 (VGG-T$^3$: Offline
// Feed-Forward 3D Reconstruction at Scale, Sec. 3.4, Eq. 3; the gradient is a
// sum of per-token terms, Eq. 5) with residual E = T(K) - V' from the forward
// kernel, the chain rule through T(x) = (silu(x W1) * (x W3)) W2 gives, per
// token (G = (2/n) E; the 2/n is applied in the update):
//   Z1 = K W1, Z3 = K W3, S = sigmoid(Z1)                      (recomputed)
//   dA = E W2^T
//   dZ1 = dA * Z3 * S * (1 + Z1 (1 - S)),  dZ3 = dA * Z1 * S,  A = Z1 S Z3
//   dW1^T += dZ1^T K,  dW3^T += dZ3^T K,  dW2 += A^T E
//
// Hidden-major formulation.  All products are taken with the hidden units on
// the 128 TMEM lanes (M=128 hidden, N=48 tokens, K=d; f16 operands, FP32
// accumulators):
//   U^T = (W1/2)^T K^T   A = the slice's W1^T/2 rows kept in TMEM (TS)
//   Z3^T = W3^T K^T      A = the slice's W3^T rows in shared memory (SS)
//   dA^T = W2 E^T        A = the slice's W2 rows in shared memory (SS)
// The epilogue thread of hidden unit r evaluates the chain rule for 16 tokens
// and writes 2*dZ1^T, dZ3^T and A^T back to TMEM as packed f16 (2 dZ1^T and
// dZ3^T over the U columns it has just read, A^T into a small ring); that is
// exactly the A operand layout of
//   dW1^T += (2 dZ1^T) K, dW3^T += dZ3^T K, dW2 += A^T E   (M=128 hidden, N=d,
//        K=16 tokens; B = the same K/E tile, read MN-major)
// (the factor 2 is removed in the update), so no intermediate goes through
// shared memory.  With u = z1/2 and t = tanh(u): sigmoid(z1) = (1+t)/2,
// silu(z1) = u (1+t) and 2 d silu/dz1 = (1+t) + u (1 - t^2).
//
// Buffering (TMEM, 512 columns at d=64): U is triple buffered and is the only
// buffer whose reuse waits for the dW MMAs, so a unit's epilogue never waits
// on the dW products of the unit before; Z3^T and dA^T are single buffered
// (the epilogue empties them as soon as a unit is ready); A^T has two slots.
//
// CTA work = (head, 128-wide slice of the hidden units, contiguous range of
// 48-token units); the CTAs of one group share the unit range, one slice
// each.  dW of the slice stays in TMEM for the whole range and is written once
// per (head, slice) segment to a partial buffer; the update kernel sums the
// partials of a (head, slice) in group order, so the result is deterministic.
//
// Warp roles: warp 0 TMA producer; warp 1 TMEM allocator and U/Z3/dA issuer;
// warp 2 dW issuer; warp 3 converts each landed K tile to f16 in place; warps
// 4-15 three epilogue warpgroups, group g owning tokens 16g..16g+15 of every
// unit.  Both issuers run warp-uniform loops
// with precomputed descriptors and issue from one elected lane.
#pragma once
#include "fwd.cuh"

namespace ttt {

constexpr int kUnit = 48;             // tokens per backward unit (N of the U/Z3/dA products)
constexpr int kBwdThreads = 512;      // 16 warps
constexpr int kBwdZWarp = 1;
constexpr int kBwdDwWarp = 2;
constexpr int kBwdCvtWarp = 3;
constexpr int kBwdEpiWarp0 = 4;
constexpr int kBwdStages = 6;         // K/E ring depth
constexpr int kBwdUBufs = 3;          // U^T buffers
constexpr int kBwdPaSlots = 2;        // A^T slots

struct BwdParams {
  // Per head, per hidden row r < HIDP: [W1^T row / 2 | W3^T row | W2 row], D
  // f16 each (zero for r >= h); read as pairs (element 2c in the low half).
  const uint32_t* wt_img;
  float* partials;               // [head*slices+slice][max_contrib][3][128][D] f32
  int n, heads, units, slices;   // units = ceil(n / kUnit); slices = HIDP / 128
  int max_contrib;
  unsigned int* status;
  long long wait_clocks;         // limit of a bounded wait (<= 0: the default)
};

template <int D>
struct BwdLayout {
  static constexpr int SW = 2 * D;
  static constexpr uint32_t kBox = 1u * kUnit * D * 2;                  // bytes of one TMA box
  static constexpr uint32_t kStage = (kBox + 1023u) / 1024u * 1024u;    // swizzle-period aligned
  static constexpr uint32_t kWRows = (128u * D * 2 + 1023u) / 1024u * 1024u;  // 128 weight rows (K-major)
  static constexpr uint32_t off_w3 = 0;
  static constexpr uint32_t off_w2 = off_w3 + kWRows;
  static constexpr uint32_t off_k = off_w2 + kWRows;
  static constexpr uint32_t off_e = off_k + kBwdStages * kStage;
  static constexpr uint32_t off_bar = off_e + kBwdStages * kStage;
  static constexpr int kNumBars = 48;
  static constexpr uint32_t bytes = off_bar + kNumBars * 8 + 16 + 1024;
  // TMEM columns
  static constexpr uint32_t cW1 = 0;                          // W1^T/2 rows: D/2 columns
  static constexpr uint32_t cDW = (D / 2 + 15) / 16 * 16;     // 2 dW1^T, dW3^T, dW2: D columns each
  static constexpr uint32_t cU = cDW + 3 * D;                 // kBwdUBufs x kUnit
  static constexpr uint32_t cZ3 = cU + kBwdUBufs * kUnit;     // kUnit
  static constexpr uint32_t cDA = cZ3 + kUnit;                // kUnit
  static constexpr uint32_t cPA = cDA + kUnit;                // kBwdPaSlots x 3 groups x 8
  static_assert(cPA + kBwdPaSlots * 24 <= 512, "tensor memory");
};

enum BwdBar {
  BB_KE_FULL = 0, BB_KC_FULL = kBwdStages, BB_KE_EMPTY = 2 * kBwdStages, BB_W_FULL = 3 * kBwdStages, BB_W_EMPTY, BB_FULL,
  BB_U_EMPTY = BB_FULL + kBwdUBufs, BB_ZD_EMPTY = BB_U_EMPTY + kBwdUBufs, BB_P_FULL,
  BB_PA_EMPTY = BB_P_FULL + 3 * kBwdUBufs, BB_ACC_FULL = BB_PA_EMPTY + kBwdPaSlots, BB_ACC_EMPTY, BB_DONE
};
static_assert(BB_DONE < 48, "barrier count");

constexpr uint32_t kHalf2One = 0x3C003C00u;   // (1, 1) in f16x2

// Two bf16 values (one 32-bit word) -> two f16 values (exact in f16's normal range).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  return pack_f16x2(bf16lo(v), bf16hi(v));
}

// Group (of CTAs) that owns flattened (head, unit) item i under the static
// partition [floor(g*N/G), floor((g+1)*N/G)).
__host__ __device__ inline long long owner_cta(long long i, long long n_items, long long grid) {
  return ((i + 1) * grid - 1) / n_items;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_e,
               const BwdParams p) {
  using L = BwdLayout<D>;
  constexpr int SW = L::SW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const Abort ab{abort_flag, p.status, p.wait_clocks};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // CTAs come in groups of `slices`: CTA group*slices + s handles hidden slice s
  // of the group's (head, unit) range, so the CTAs of a group read the same K/E
  // tiles at about the same time and all but the first find them in L2.
  const int slice_id = blockIdx.x % p.slices;
  const int group = blockIdx.x / p.slices;
  const int groups = gridDim.x / p.slices;
  const long long total = static_cast<long long>(p.heads) * p.units;
  const long long it0 = total * group / groups;
  const long long it1 = total * (group + 1) / groups;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(&bars[BB_KE_FULL + s], 1);
      mbar_init(&bars[BB_KC_FULL + s], 1);
      mbar_init(&bars[BB_KE_EMPTY + s], 1);
    }
    mbar_init(&bars[BB_W_FULL], 12);     // every epilogue warp writes part of the weights
    mbar_init(&bars[BB_W_EMPTY], 1);
    for (int b = 0; b < kBwdUBufs; ++b) {
      mbar_init(&bars[BB_FULL + b], 1);
      mbar_init(&bars[BB_U_EMPTY + b], 1);
    }
    mbar_init(&bars[BB_ZD_EMPTY], 12);
    // per (U buffer, token group): a warpgroup reuses buffer b only after the
    // dW MMAs of the unit that last used it have drained it, so no phase is
    // ever skipped
    for (int i = 0; i < 3 * kBwdUBufs; ++i) mbar_init(&bars[BB_P_FULL + i], 4);
    for (int i = 0; i < kBwdPaSlots; ++i) mbar_init(&bars[BB_PA_EMPTY + i], 1);
    mbar_init(&bars[BB_ACC_FULL], 1);
    mbar_init(&bars[BB_ACC_EMPTY], 12);
    mbar_init(&bars[BB_DONE], 2);
    fence_mbar_init();
  }
  if (warp == kBwdZWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      TTT_TR_DECL
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_e);
      Cursor cu;
      cu.init(it0, p.units);
      uint32_t s = 0, ph = 0, issued = 0;
      for (; cu.it < it1; cu.next(p.units), ++issued) {
        TTT_TR_LAP(0);
        if (!mbar_wait(&bars[BB_KE_EMPTY + s], ph ^ 1, ab)) break;
        TTT_TR_LAP(1);
        mbar_arrive_expect_tx(&bars[BB_KE_FULL + s], 2 * L::kBox);
        tma_load_2d(smem + L::off_k + s * L::kStage, &tm_k, &bars[BB_KE_FULL + s], cu.major * D, cu.tile * kUnit);
        tma_load_2d(smem + L::off_e + s * L::kStage, &tm_e, &bars[BB_KE_FULL + s], cu.major * D, cu.tile * kUnit);
        if (++s == kBwdStages) {
          s = 0;
          ph ^= 1;
        }
      }
      TTT_TR_LAP(0);
      TTT_TR_DUMP(2);
      // Drain: the last load issued into each stage has landed before exit.
      const uint32_t last = issued < static_cast<uint32_t>(kBwdStages) ? issued : kBwdStages;
      for (uint32_t b = 0; b < last; ++b) {
        const uint32_t jj = issued - 1 - b;
        mbar_drain(&bars[BB_KE_FULL + jj % kBwdStages], (jj / kBwdStages) & 1);
      }
    }
  } else if (warp == kBwdCvtWarp) {
    // ------------------------------------------------------------ K -> f16
    // In place over the landed bf16 tile (the swizzle permutes whole 16-byte
    // chunks, so converting every word keeps the layout), then a
    // generic-to-async proxy fence before the tensor core reads it.
    Cursor cu;
    cu.init(it0, p.units);
    uint32_t s = 0, ph = 0;
    for (; cu.it < it1; cu.next(p.units)) {
      if (!mbar_wait_warp(&bars[BB_KE_FULL + s], ph, ab)) break;
      const uint32_t base = smem_u32(smem + L::off_k + s * L::kStage);
#pragma unroll 2
      for (uint32_t off = lane * 16u; off < L::kBox; off += 32u * 16u) {
        uint32_t a, b, c, d;
        ld_shared_v4(base + off, a, b, c, d);
        st_shared_v4(base + off, bf16x2_to_f16x2(a), bf16x2_to_f16x2(b), bf16x2_to_f16x2(c), bf16x2_to_f16x2(d));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[BB_KC_FULL + s]);
      if (++s == kBwdStages) {
        s = 0;
        ph ^= 1;
      }
    }
  } else if (warp == kBwdZWarp) {
    // ------------------------------------------------------------ U / Z3 / dA issuer
    constexpr uint32_t kId = idesc_f16(128, kUnit, false, false);
    const uint64_t dk0 = smem_desc(smem_u32(smem + L::off_k), 0, 8 * SW, SW);
    const uint64_t de0 = smem_desc(smem_u32(smem + L::off_e), 0, 8 * SW, SW);
    const uint64_t dw3 = smem_desc(smem_u32(smem + L::off_w3), 0, 8 * SW, SW);
    const uint64_t dw2 = smem_desc(smem_u32(smem + L::off_w2), 0, 8 * SW, SW);
    const uint32_t tW1 = tbase + L::cW1, tZ3 = tbase + L::cZ3, tDA = tbase + L::cDA;
    TTT_TR_DECL
    Cursor zc;
    zc.init(it0, p.units);
    int cur_head = -1;
    uint32_t s = 0, ph = 0, j = 0, ub = 0, uph = 0, seg = 0;
    bool ok = true;
    for (; zc.it < it1 && ok; zc.next(p.units), ++j) {
      if (zc.major != cur_head) {
        if (seg > 0) mma_commit_warp(&bars[BB_W_EMPTY]);
        TTT_TR_LAP(0);
        if (!(ok = mbar_wait_warp(&bars[BB_W_FULL], seg & 1, ab))) break;
        TTT_TR_LAP(4);
        ++seg;
        cur_head = zc.major;
      }
      TTT_TR_LAP(0);
      if (!(ok = mbar_wait_warp(&bars[BB_KC_FULL + s], ph, ab))) break;
      TTT_TR_LAP(1);
      const uint64_t soff = (s * L::kStage) >> 4;
      const uint64_t dk = dk0 + soff, de = de0 + soff;
      // U^T into buffer ub once the dW MMAs of unit j-3 have read it (early:
      // this wait is off the critical path, so U goes first).
      if (!(ok = mbar_wait_warp(&bars[BB_U_EMPTY + ub], uph ^ 1, ab))) break;
      TTT_TR_LAP(5);
      tc_fence_after();
      const uint32_t tu = tbase + L::cU + ub * kUnit;
#pragma unroll
      for (int k = 0; k < D / 16; ++k) mma_bf16_ts_warp(tu, tW1 + 8 * k, dk + 2 * k, kId, k > 0 ? 1u : 0u);
      // Z3^T and dA^T of this unit once the epilogue has read the previous ones.
      if (!(ok = mbar_wait_warp(&bars[BB_ZD_EMPTY], (j & 1) ^ 1, ab))) break;
      TTT_TR_LAP(2);
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < D / 16; ++k) mma_bf16_warp(tDA, dw2 + 2 * k, de + 2 * k, kId, k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) mma_bf16_warp(tZ3, dw3 + 2 * k, dk + 2 * k, kId, k > 0 ? 1u : 0u);
      mma_commit_warp(&bars[BB_FULL + ub]);
      TTT_TR_LAP(3);
      if (++s == kBwdStages) {
        s = 0;
        ph ^= 1;
      }
      if (++ub == kBwdUBufs) {
        ub = 0;
        uph ^= 1;
      }
    }
    TTT_TR_DUMP(2);
    mma_commit_warp(&bars[BB_DONE]);
    mbar_drain(&bars[BB_DONE], 0);
  } else if (warp == kBwdDwWarp) {
    // ------------------------------------------------------------ dW issuer
    // dW1^T += (2 dZ1^T) K, dW3^T += dZ3^T K, dW2 += A^T E per 16-token group
    // as soon as its epilogue warpgroup has written it.  The unit's last
    // commits release its U buffer, its A^T slot and its K/E stage: the unit's
    // other MMAs completed before the epilogue could read their results, so
    // every reader of the stage is done.
    constexpr uint32_t kIdW = idesc_f16(128, D, false, true);
    const uint64_t dk0 = smem_desc(smem_u32(smem + L::off_k), 0, 8 * SW, SW);
    const uint64_t de0 = smem_desc(smem_u32(smem + L::off_e), 0, 8 * SW, SW);
    const uint32_t tDW = tbase + L::cDW;
    TTT_TR_DECL
    Cursor wc;
    wc.init(it0, p.units);
    uint32_t s = 0, ub = 0, uph = 0, pa = 0, seg = 0;
    bool ok = true;
    for (; wc.it < it1 && ok; wc.next(p.units)) {
      const bool first = (wc.it == it0) || wc.tile == 0;
      const bool last = (wc.it == it1 - 1) || wc.tile == p.units - 1;
      if (first && seg > 0) {
        TTT_TR_LAP(0);
        if (!(ok = mbar_wait_warp(&bars[BB_ACC_EMPTY], (seg - 1) & 1, ab))) break;
        TTT_TR_LAP(4);
      }
      const uint32_t tu = tbase + L::cU + ub * kUnit, tpa = tbase + L::cPA + pa * 24;
      const uint64_t soff = (s * L::kStage) >> 4;
      const uint64_t dk = dk0 + soff, de = de0 + soff;
#pragma unroll
      for (int g = 0; g < 3; ++g) {
        TTT_TR_LAP(0);
        if (!(ok = mbar_wait_warp(&bars[BB_P_FULL + 3 * ub + g], uph, ab))) break;
        TTT_TR_LAP(1);
        tc_fence_after();
        const uint32_t acc = (first && g == 0) ? 0u : 1u;
        const uint64_t go = (16u * g * SW) >> 4;
        mma_bf16_ts_warp(tDW, tu + 16 * g, dk + go, kIdW, acc);
        mma_bf16_ts_warp(tDW + D, tu + 16 * g + 8, dk + go, kIdW, acc);
        mma_bf16_ts_warp(tDW + 2 * D, tpa + 8 * g, de + go, kIdW, acc);
        TTT_TR_LAP(2);
      }
      if (!ok) break;
      mma_commit_warp(&bars[BB_U_EMPTY + ub]);
      mma_commit_warp(&bars[BB_PA_EMPTY + pa]);
      mma_commit_warp(&bars[BB_KE_EMPTY + s]);
      if (last) {
        mma_commit_warp(&bars[BB_ACC_FULL]);   // segment done: the epilogue dumps dW
        ++seg;
      }
      if (++s == kBwdStages) s = 0;
      if (++ub == kBwdUBufs) {
        ub = 0;
        uph ^= 1;
      }
      pa ^= 1;
    }
    TTT_TR_DUMP(2);
    mma_commit_warp(&bars[BB_DONE]);
    mbar_drain(&bars[BB_DONE], 0);
  } else if (warp >= kBwdEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int g = (warp - kBwdEpiWarp0) >> 2;  // token group of every unit; weight / dW matrix it moves
    const int q = warp & 3;                    // TMEM lane quadrant
    const int row = q * 32 + lane;             // hidden unit within the slice
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t j = 0, ub = 0, uph = 0, seg = 0, dumps = 0;
    long long cur_pair = -1;
    bool ok = true;
    TTT_TR_DECL

    // Write dW of the finished segment (pair) to its partial slot: warpgroup g
    // moves matrix g (2 dW1^T, dW3^T, dW2), row = hidden unit.
    auto dump = [&](long long pair) -> bool {
      TTT_TR_LAP(0);
      if (!mbar_wait_warp(&bars[BB_ACC_FULL], dumps & 1, ab)) return false;
      TTT_TR_LAP(5);
      tc_fence_after();
      const long long first_item = (pair / p.slices) * static_cast<long long>(p.units);
      const long long contrib = group - owner_cta(first_item, total, groups);
      float* dst = p.partials + (static_cast<size_t>(pair) * p.max_contrib + contrib) * (3u * 128u * D) +
                   (static_cast<size_t>(g) * 128 + row) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(tbase + L::cDW + g * D + c0 + lane_off, r);
        tmem_wait_ld();
        float4* o = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          o[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]), __uint_as_float(r[4 * v + 2]),
                             __uint_as_float(r[4 * v + 3]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[BB_ACC_EMPTY]);
      ++dumps;
      TTT_TR_LAP(6);
      return true;
    };

    // Weights of a (head, slice): warpgroup 0 writes the W1^T/2 rows into TMEM,
    // warpgroups 1 and 2 the W3^T and W2 rows into shared memory (the K-major,
    // swizzled A operands of Z3^T and dA^T).
    auto load_weights = [&](int head) -> bool {
      if (seg > 0 && !mbar_wait_warp(&bars[BB_W_EMPTY], (seg - 1) & 1, ab)) return false;
      tc_fence_after();
      const size_t hidp = static_cast<size_t>(p.slices) * 128;
      const uint4* src = reinterpret_cast<const uint4*>(
          p.wt_img + ((static_cast<size_t>(head) * hidp + slice_id * 128 + row) * 3 + g) * (D / 2));
      if (g > 0) {
        const uint32_t base = smem_u32(smem + (g == 1 ? L::off_w3 : L::off_w2));
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 x = __ldg(src + c);
          st_shared_v4(base + swz(static_cast<uint32_t>(row) * SW + c * 16, SW), x.x, x.y, x.z, x.w);
        }
        fence_proxy_async_smem();
      } else if constexpr (D >= 32) {
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 16) {
          uint32_t w[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 x = __ldg(src + c0 / 4 + v);
            w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
          }
          tmem_st16(tbase + L::cW1 + c0 + lane_off, w);
        }
        tmem_wait_st();
      } else {
        uint32_t w[8];
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const uint4 x = __ldg(src + v);
          w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
        }
        tmem_st8(tbase + L::cW1 + lane_off, w);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[BB_W_FULL]);
      ++seg;
      return true;
    };

    Cursor cu;
    cu.init(it0, p.units);
    for (; cu.it < it1 && ok; cu.next(p.units), ++j) {
      const long long pair = static_cast<long long>(cu.major) * p.slices + slice_id;
      if (pair != cur_pair) {
        if (cur_pair >= 0 && !(ok = dump(cur_pair))) break;
        if (!(ok = load_weights(cu.major))) break;
        cur_pair = pair;
      }
      const uint32_t pa = j & 1;
      TTT_TR_LAP(0);
      if (!(ok = mbar_wait_warp(&bars[BB_FULL + ub], uph, ab))) break;
      TTT_TR_LAP(1);
      tc_fence_after();
      uint32_t zu[16], z3[16], da[16];
      const uint32_t tu = tbase + L::cU + ub * kUnit + 16 * g + lane_off;
      // The single-buffered Z3^T / dA^T columns first: the next unit's MMAs
      // into them wait for this release.
      tmem_ld16(tbase + L::cZ3 + 16 * g + lane_off, z3);
      tmem_ld16(tbase + L::cDA + 16 * g + lane_off, da);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[BB_ZD_EMPTY]);
      tmem_ld16(tu, zu);
      tmem_wait_ld();
      TTT_TR_LAP(2);
      uint32_t pz1[8], pz3[8], pav[8];
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        // Packed f16 arithmetic on two tokens of this hidden unit (the outputs
        // are the f16 A operands of the dW MMAs), with u = z1/2, t = tanh(u):
        //   silu = u (1+t),  2 dsilu/dz1 = (1+t) + u (1 - t^2),
        //   2 dZ1 = dA z3 (2 dsilu/dz1),  dZ3 = dA silu,  A = silu z3.
        const uint32_t bu = pack_f16x2(__uint_as_float(zu[i]), __uint_as_float(zu[i + 1]));
        const uint32_t b3 = pack_f16x2(__uint_as_float(z3[i]), __uint_as_float(z3[i + 1]));
        const uint32_t bd = pack_f16x2(__uint_as_float(da[i]), __uint_as_float(da[i + 1]));
        const uint32_t t = htanh2(bu);
        const uint32_t s2 = hfma2(t, kHalf2One, kHalf2One);              // 1 + t
        const uint32_t silu = hmul2(bu, s2);
        const uint32_t om = hfma2(t ^ 0x80008000u, t, kHalf2One);         // 1 - t^2
        const uint32_t q2 = hfma2(bu, om, s2);                          // 2 dsilu/dz1
        pz1[i / 2] = hmul2(hmul2(bd, b3), q2);
        pz3[i / 2] = hmul2(bd, silu);
        pav[i / 2] = hmul2(silu, b3);
      }
      TTT_TR_LAP(3);
      // 2 dZ1^T, dZ3^T over this warpgroup's U columns (read above); A^T into
      // its slot once the dW MMAs of unit j-2 have read it.
      tmem_st8(tu, pz1);
      tmem_st8(tu + 8, pz3);
      if (!(ok = mbar_wait_warp(&bars[BB_PA_EMPTY + pa], ((j >> 1) & 1) ^ 1, ab))) break;
      TTT_TR_LAP(4);
      tc_fence_after();
      tmem_st8(tbase + L::cPA + pa * 24 + 8 * g + lane_off, pav);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[BB_P_FULL + 3 * ub + g]);
      TTT_TR_LAP(7);
      if (++ub == kBwdUBufs) {
        ub = 0;
        uph ^= 1;
      }
    }
    if (ok && cur_pair >= 0) dump(cur_pair);
    TTT_TR_LAP(0);
    TTT_TR_DUMP(2);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdZWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace ttt
