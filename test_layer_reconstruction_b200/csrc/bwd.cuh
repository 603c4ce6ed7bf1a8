// bwd.cuh — gradient of the mean-squared TTT loss w.r.t. the SwiGLU fast
// weights, as split-K partial sums over token ranges.
//
// For the loss L = (1/n) sum_i ||T(k_i) - v'_i||^2 (VGG-T$^3$: Offline
// Feed-Forward 3D Reconstruction at Scale, Sec. 3.4, Eq. 3; the gradient is a
// sum of per-token terms, Eq. 5) with residual E = T(K) - V' from the forward
// kernel, the chain rule through T(x) = (silu(x W1) * (x W3)) W2 gives, per
// token tile (G = (2/n) E; the 2/n is applied in the update):
//   Z1 = K W1, Z3 = K W3, S = sigmoid(Z1)                      (recomputed)
//   dA = E W2^T
//   dZ1 = dA * Z3 * S * (1 + Z1 (1 - S)),  dZ3 = dA * Z1 * S,  A = Z1 S Z3
//   dW1^T += dZ1^T K,  dW3^T += dZ3^T K,  dW2 += A^T E
// CTA work = (head, 128-wide slice of the hidden units, contiguous range of
// 128-token tiles); the CTAs of one group share the tile range, one slice
// each.  dW for the slice stays in TMEM for the whole range and is written
// once per (head, slice) segment to a partial buffer.  The update kernel sums
// the partials of a (head, slice) in group order, so the result is
// deterministic.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator + sub-chunk MMA
// issuer, warp 10 dW MMA issuer, warps 2-9 two epilogue warpgroups.  Per tile the
// slice is walked in 4 sub-chunks of 32 hidden units, each with
//   Z  = K * [W1 | W3]_sub   (M=128 tokens, N=64, K=d)
//   dA = E * W2_sub^T        (M=128 tokens, N=32, K=d)
// in one of 3 TMEM slots; the epilogue writes A, dZ1, dZ3 (bf16) to shared
// memory and the dW MMAs (M=128 hidden, N=d, K=128 tokens, both operands
// MN-major) of a tile go out as soon as that is done.
#pragma once
#include "fwd.cuh"

namespace ttt {

constexpr int kBwdThreads = 352;    // 11 warps: 0 producer, 1 sub-chunk issuer, 2-9 epilogue, 10 dW issuer
constexpr int kBwdDwWarp = 10;

struct BwdParams {
  const __nv_bfloat16* w13_img;  // per head: 2*HIDP rows of D bf16 (sw-swizzled)
  const __nv_bfloat16* w2_img;   // per head: HIDP rows of D bf16 (sw-swizzled)
  float* partials;               // [head*slices+slice][max_contrib][3][128][D] f32
  int n, heads, tiles, slices;   // slices = HIDP / 128
  int max_contrib;
  unsigned int* status;
};

template <int D>
struct BwdLayout {
  static constexpr int SW = 2 * D;
  static constexpr uint32_t kW13 = 2u * 128 * D * 2;  // rows of one 128-wide slice
  static constexpr uint32_t kW2 = 1u * 128 * D * 2;
  static constexpr uint32_t kTile = 1u * kTileM * D * 2;
  static constexpr uint32_t kBuf = 2u * kTileM * 64 * 2;  // [128 tok][128 hid] as 2 atoms of 64
  static constexpr uint32_t off_w13 = 0;
  static constexpr uint32_t off_w2 = off_w13 + kW13;
  static constexpr uint32_t off_k = off_w2 + kW2;
  static constexpr uint32_t off_e = off_k + 2 * kTile;
  static constexpr uint32_t off_a = off_e + 2 * kTile;
  static constexpr uint32_t off_dz1 = off_a + kBuf;
  static constexpr uint32_t off_dz3 = off_dz1 + kBuf;
  static constexpr uint32_t off_bar = off_dz3 + kBuf;
  static constexpr int kNumBars = 24;
  static constexpr uint32_t bytes = off_bar + kNumBars * 8 + 16 + 1024;
  static_assert(off_k % 1024 == 0 && off_e % 1024 == 0 && off_a % 1024 == 0, "1 KiB alignment");
};

enum BwdBar {
  BB_W_FULL = 0, BB_W_EMPTY = 1, BB_KE_FULL = 2, BB_KE_EMPTY = 4, BB_SL_FULL = 6, BB_SL_EMPTY = 9,
  BB_DZ_FULL = 12, BB_DZ_EMPTY = 13, BB_ACC_FULL = 14, BB_ACC_EMPTY = 15, BB_DONE = 16
};

// Group (of CTAs) that owns flattened (head, tile) item i under the static
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
  constexpr uint32_t kSlot = 96;       // TMEM columns per sub-chunk slot
  constexpr uint32_t kDw = 288;        // first dW column
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const Abort ab{abort_flag, p.status};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // CTAs come in groups of `slices`: CTA group*slices + s handles hidden slice s
  // of the group's (head, tile) range, so the CTAs of a group read the same K/E
  // tiles at about the same time and all but the first find them in L2.
  const int slice_id = blockIdx.x % p.slices;
  const int group = blockIdx.x / p.slices;
  const int groups = gridDim.x / p.slices;
  const long long total = static_cast<long long>(p.heads) * p.tiles;
  const long long it0 = total * group / groups;
  const long long it1 = total * (group + 1) / groups;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(&bars[BB_W_FULL], 1);
    mbar_init(&bars[BB_W_EMPTY], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[BB_KE_FULL + s], 1);
      mbar_init(&bars[BB_KE_EMPTY + s], 1);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bars[BB_SL_FULL + s], 1);
      mbar_init(&bars[BB_SL_EMPTY + s], 4);
    }
    mbar_init(&bars[BB_DZ_FULL], 8);
    mbar_init(&bars[BB_DZ_EMPTY], 1);
    mbar_init(&bars[BB_ACC_FULL], 1);
    mbar_init(&bars[BB_ACC_EMPTY], 8);
    mbar_init(&bars[BB_DONE], 2);
    fence_mbar_init();
  }
  if (warp == 1) {
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
      long long cur_pair = -1;
      int head = 0, slice = 0;
      uint32_t wl = 0, j = 0;
      Cursor pf;
      pf.init(it0, p.tiles);
      for (int k = 0; k < kPrefetchAhead && pf.it < it1; ++k, pf.next(p.tiles)) {
        tma_prefetch_l2_2d(&tm_k, pf.major * D, pf.tile * kTileM);
        tma_prefetch_l2_2d(&tm_e, pf.major * D, pf.tile * kTileM);
      }
      Cursor cu;
      cu.init(it0, p.tiles);
      for (; cu.it < it1; cu.next(p.tiles), ++j) {
        const int pair = cu.major * p.slices + slice_id;
        const int tile = cu.tile;
        if (pair != cur_pair) {
          head = cu.major;
          slice = slice_id;
          TTT_TR_LAP(0);
          if (wl > 0 && !mbar_wait(&bars[BB_W_EMPTY], (wl - 1) & 1, ab)) break;
          TTT_TR_LAP(2);
          mbar_arrive_expect_tx(&bars[BB_W_FULL], L::kW13 + L::kW2);
          const size_t hidp = static_cast<size_t>(p.slices) * 128;
          const __nv_bfloat16* w13 = p.w13_img + (static_cast<size_t>(head) * 2 * hidp + slice * 256) * D;
          const __nv_bfloat16* w2 = p.w2_img + (static_cast<size_t>(head) * hidp + slice * 128) * D;
          bulk_load_pieces(smem + L::off_w13, w13, L::kW13, &bars[BB_W_FULL]);
          bulk_load_pieces(smem + L::off_w2, w2, L::kW2, &bars[BB_W_FULL]);
          ++wl;
          cur_pair = pair;
        }
        const int s = j & 1;
        if (pf.it < it1) {
          tma_prefetch_l2_2d(&tm_k, pf.major * D, pf.tile * kTileM);
          tma_prefetch_l2_2d(&tm_e, pf.major * D, pf.tile * kTileM);
          pf.next(p.tiles);
        }
        TTT_TR_LAP(0);
        if (!mbar_wait(&bars[BB_KE_EMPTY + s], ((j >> 1) & 1) ^ 1, ab)) break;
        TTT_TR_LAP(1);
        mbar_arrive_expect_tx(&bars[BB_KE_FULL + s], 2 * L::kTile);
        tma_load_2d(smem + L::off_k + s * L::kTile, &tm_k, &bars[BB_KE_FULL + s], head * D, tile * kTileM);
        tma_load_2d(smem + L::off_e + s * L::kTile, &tm_e, &bars[BB_KE_FULL + s], head * D, tile * kTileM);
      }
      TTT_TR_LAP(0);
      TTT_TR_DUMP(2);
      if (wl > 0) mbar_drain(&bars[BB_W_FULL], (wl - 1) & 1);
      for (uint32_t jj = (j >= 2 ? j - 2 : 0); jj < j; ++jj) mbar_drain(&bars[BB_KE_FULL + (jj & 1)], (jj >> 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ sub-chunk issuer
    // Z = K * [W1 | W3]_sub and dA = E * W2_sub^T into one of 3 TMEM slots.
    constexpr uint32_t kIdZ = idesc_bf16(128, 64, false, false);
    constexpr uint32_t kIdDA = idesc_bf16(128, 32, false, false);
    const uint32_t w13 = smem_u32(smem + L::off_w13);
    const uint32_t w2 = smem_u32(smem + L::off_w2);
    TTT_TR_DECL
    Cursor sc;
    sc.init(it0, p.tiles);
    int cur_pair = -1;
    uint32_t sj = 0, kc = 0, wl = 0;
    bool ok = true;
    for (; sc.it < it1 && ok; sc.next(p.tiles), ++sj) {
      if (sc.major != cur_pair) {
        if (cur_pair >= 0) mma_commit_warp(&bars[BB_W_EMPTY]);
        if (!(ok = mbar_wait_warp(&bars[BB_W_FULL], wl & 1, ab))) break;
        ++wl;
        cur_pair = sc.major;
      }
      const int s = sj & 1;
      TTT_TR_LAP(0);
      if (!(ok = mbar_wait_warp(&bars[BB_KE_FULL + s], (sj >> 1) & 1, ab))) break;
      TTT_TR_LAP(1);
      const uint32_t ks = smem_u32(smem + L::off_k + s * L::kTile);
      const uint32_t es = smem_u32(smem + L::off_e + s * L::kTile);
      for (int ssc = 0; ssc < 4; ++ssc, ++kc) {
        const uint32_t slot = kc % 3, use = kc / 3;
        TTT_TR_LAP(0);
        if (!(ok = mbar_wait_warp(&bars[BB_SL_EMPTY + slot], (use & 1) ^ 1, ab))) break;
        TTT_TR_LAP(2);
        tc_fence_after();
        const uint32_t tsl = tbase + slot * kSlot;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_warp(tsl, smem_desc(ks + 32 * k, 0, 8 * SW, SW),
                        smem_desc(w13 + 64 * ssc * SW + 32 * k, 0, 8 * SW, SW), kIdZ, k > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_warp(tsl + 64, smem_desc(es + 32 * k, 0, 8 * SW, SW),
                        smem_desc(w2 + 32 * ssc * SW + 32 * k, 0, 8 * SW, SW), kIdDA, k > 0 ? 1u : 0u);
        mma_commit_warp(&bars[BB_SL_FULL + slot]);
        TTT_TR_LAP(3);
      }
    }
    TTT_TR_DUMP(2);
    mma_commit_warp(&bars[BB_DONE]);
    mbar_drain(&bars[BB_DONE], 0);
  } else if (warp == kBwdDwWarp) {
    // ------------------------------------------------------------ dW issuer
    // dW1^T += dZ1^T K, dW3^T += dZ3^T K, dW2 += A^T E once the epilogue has
    // written A, dZ1, dZ3 of the tile.  This warp's commit releases the K/E
    // stage: the tile's sub-chunk MMAs completed before the epilogue could
    // write its dZ, so every reader of the stage is done.
    constexpr uint32_t kIdW = idesc_bf16(128, D, true, true);
    const uint32_t sa = smem_u32(smem + L::off_a);
    const uint32_t sdz1 = smem_u32(smem + L::off_dz1);
    const uint32_t sdz3 = smem_u32(smem + L::off_dz3);
    Cursor wc;
    wc.init(it0, p.tiles);
    uint32_t wj = 0, wseg = 0;
    bool ok = true;
    for (; wc.it < it1 && ok; wc.next(p.tiles), ++wj) {
      const bool first = (wc.it == it0) || wc.tile == 0;
      const bool last = (wc.it == it1 - 1) || wc.tile == p.tiles - 1;
      if (!(ok = mbar_wait_warp(&bars[BB_DZ_FULL], wj & 1, ab))) break;
      if (first && wseg > 0 && !(ok = mbar_wait_warp(&bars[BB_ACC_EMPTY], (wseg - 1) & 1, ab))) break;
      tc_fence_after();
      const int s = wj & 1;
      const uint32_t ks = smem_u32(smem + L::off_k + s * L::kTile);
      const uint32_t es = smem_u32(smem + L::off_e + s * L::kTile);
#pragma unroll
      for (int k = 0; k < kTileM / 16; ++k) {
        const uint32_t acc = (first && k == 0) ? 0u : 1u;
        const uint64_t bk = smem_desc(ks + k * 16 * SW, 0, 8 * SW, SW);
        const uint64_t be = smem_desc(es + k * 16 * SW, 0, 8 * SW, SW);
        mma_bf16_warp(tbase + kDw, smem_desc(sdz1 + k * 2048, 16384, 1024, 128), bk, kIdW, acc);
        mma_bf16_warp(tbase + kDw + D, smem_desc(sdz3 + k * 2048, 16384, 1024, 128), bk, kIdW, acc);
        mma_bf16_warp(tbase + kDw + 2 * D, smem_desc(sa + k * 2048, 16384, 1024, 128), be, kIdW, acc);
      }
      mma_commit_warp(&bars[BB_DZ_EMPTY]);
      mma_commit_warp(&bars[BB_KE_EMPTY + s]);
      if (last) {
        mma_commit_warp(&bars[BB_ACC_FULL]);   // segment done: the epilogue dumps dW
        ++wseg;
      }
    }
    mma_commit_warp(&bars[BB_DONE]);
    mbar_drain(&bars[BB_DONE], 0);
  } else if (warp >= 2 && warp <= 9) {
    // ------------------------------------------------------------ epilogue
    const int g = (warp - 2) >> 2;
    const int q = warp & 3;
    const int row = q * 32 + lane;            // token row (sub-chunks), hidden row (dW dump)
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t sa = smem_u32(smem + L::off_a);
    const uint32_t sdz1 = smem_u32(smem + L::off_dz1);
    const uint32_t sdz3 = smem_u32(smem + L::off_dz3);
    uint32_t j = 0, seg = 0;
    long long cur_pair = -1;
    bool ok = true;
    TTT_TR_DECL

    // Write dW of the finished segment (pair) to its partial slot.
    auto dump = [&](long long pair) -> bool {
      TTT_TR_LAP(0);
      if (!mbar_wait(&bars[BB_ACC_FULL], seg & 1, ab)) return false;
      TTT_TR_LAP(5);
      tc_fence_after();
      const long long first_item = (pair / p.slices) * static_cast<long long>(p.tiles);
      const long long contrib = group - owner_cta(first_item, total, groups);
      float* dst = p.partials + (static_cast<size_t>(pair) * p.max_contrib + contrib) * (3u * 128u * D);
      for (int grp = g; grp < 3 * D / 16; grp += 2) {
        uint32_t r[16];
        tmem_ld16(tbase + kDw + grp * 16 + lane_off, r);
        tmem_wait_ld();
        const int m = grp * 16 / D, col = grp * 16 % D;
        float4* o = reinterpret_cast<float4*>(dst + (static_cast<size_t>(m) * 128 + row) * D + col);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          o[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]), __uint_as_float(r[4 * v + 2]),
                             __uint_as_float(r[4 * v + 3]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[BB_ACC_EMPTY]);
      ++seg;
      TTT_TR_LAP(6);
      return true;
    };

    Cursor cu;
    cu.init(it0, p.tiles);
    for (; cu.it < it1 && ok; cu.next(p.tiles), ++j) {
      const long long pair = static_cast<long long>(cu.major) * p.slices + slice_id;
      if (pair != cur_pair) {
        if (cur_pair >= 0 && !(ok = dump(cur_pair))) break;
        cur_pair = pair;
      }
      bool waited_buf = false;
      for (int sc = g; sc < 4; sc += 2) {
        const uint32_t kc = j * 4 + sc;
        const uint32_t slot = kc % 3, use = kc / 3;
        TTT_TR_LAP(0);
        if (!(ok = mbar_wait(&bars[BB_SL_FULL + slot], use & 1, ab))) break;
        TTT_TR_LAP(1);
        tc_fence_after();
        const uint32_t tsl = tbase + slot * kSlot + lane_off;
        // Load the whole sub-chunk (Z1, Z3, dA), return the slot to the MMA
        // issuer at once, then compute from registers.
        uint32_t zz1[2][16], zz3[2][16], zda[2][16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          tmem_ld16(tsl + half * 16, zz1[half]);
          tmem_ld16(tsl + 32 + half * 16, zz3[half]);
          tmem_ld16(tsl + 64 + half * 16, zda[half]);
        }
        tmem_wait_ld();
        TTT_TR_LAP(7);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[BB_SL_EMPTY + slot]);
        uint32_t pa[16], pz1[16], pz3[16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t (&z1)[16] = zz1[half];
          const uint32_t (&z3)[16] = zz3[half];
          const uint32_t (&da)[16] = zda[half];
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            // Packed bf16 arithmetic on two hidden units (the outputs are the
            // bf16 operands of the dW MMAs): with s = sigmoid(z1) =
            // (1 + tanh(z1/2))/2, silu = z1 s, A = silu z3, and
            // d silu/dz1 = s (1 + z1 (1 - s)):
            //   dZ1 = dA * (z3 s + z3 s * z1 (1 - s)),  dZ3 = dA * silu.
            const uint32_t b1 = pack_bf16x2(__uint_as_float(z1[i]), __uint_as_float(z1[i + 1]));
            const uint32_t b3 = pack_bf16x2(__uint_as_float(z3[i]), __uint_as_float(z3[i + 1]));
            const uint32_t bd = pack_bf16x2(__uint_as_float(da[i]), __uint_as_float(da[i + 1]));
            const uint32_t sg = bfma2(btanh2(bmul2(b1, kBf2Half)), kBf2Half, kBf2Half);
            const uint32_t silu = bmul2(b1, sg);
            const uint32_t tt = bmul2(b3, sg);
            const uint32_t w = bmul2(b1, bfma2(sg, kBf2NegOne, kBf2One));
            pa[half * 8 + i / 2] = bmul2(silu, b3);
            pz1[half * 8 + i / 2] = bmul2(bd, bfma2(tt, w, tt));
            pz3[half * 8 + i / 2] = bmul2(bd, silu);
          }
        }
        TTT_TR_LAP(2);
        if (!waited_buf) {
          if (!(ok = mbar_wait(&bars[BB_DZ_EMPTY], (j & 1) ^ 1, ab))) break;
          waited_buf = true;
        }
        TTT_TR_LAP(3);
        // hidden unit (within the slice) sc*32 + 8v + e  ->  atom sc/2, 16-byte chunk (sc%2)*4 + v
        const uint32_t base = (sc >> 1) * 16384u;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint32_t off = base + swz(row * 128 + ((sc & 1) * 4 + v) * 16, 128);
          st_shared_v4(sa + off, pa[4 * v], pa[4 * v + 1], pa[4 * v + 2], pa[4 * v + 3]);
          st_shared_v4(sdz1 + off, pz1[4 * v], pz1[4 * v + 1], pz1[4 * v + 2], pz1[4 * v + 3]);
          st_shared_v4(sdz3 + off, pz3[4 * v], pz3[4 * v + 1], pz3[4 * v + 2], pz3[4 * v + 3]);
        }
      }
      if (!ok) break;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[BB_DZ_FULL]);
      TTT_TR_LAP(4);
    }
    if (ok && cur_pair >= 0) dump(cur_pair);
    TTT_TR_LAP(0);
    TTT_TR_DUMP(2);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace ttt
