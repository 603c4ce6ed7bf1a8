// fwd.cuh — SwiGLU forward over token tiles on the 5th-gen tensor cores.
//
// Y = T_theta(X) = (silu(X W1) * (X W3)) W2 per head, for all n tokens
// (VGG-T$^3$: Offline Feed-Forward 3D Reconstruction at Scale, Sec. 3.4,
// Eq. 4 and "TTT MLP Architecture and Inner Optimization").
//   READ mode : X = Q, writes O = Y (bf16).
//   WRITE mode: X = K, writes the residual E = Y - V' (f16); the backward
//               kernel turns it into the gradient, the factor 2/n of the
//               mean-squared loss is applied in the update.
//
// One persistent CTA per SM walks a contiguous range of (head, 128-token
// tile) items.  Warp roles:
//   warp 0   : TMA producer (weights of the current head by bulk copy, X and
//              V' tiles by 2-D TMA, two stages each, L2 prefetch ahead)
//   warp 1   : TMEM allocator and Z issuer
//   warp 2   : Y issuer (warp 3 idles)
//   warps 4-19: four epilogue warpgroups; warpgroups 2p and 2p+1 share the
//              chunks c with c % 2 == p, one 32-unit half of the chunk each
// Both issuers run in uniform control flow and issue from one elected lane.
// Per tile the hidden dimension is walked in chunks of 64 units:
//   Z = X * [W1/2 | W3]_chunk      (M=128 tokens, N=128, K=d, A and B in smem)
//                                    -> TMEM Z slot c % 2
//   gate = silu(Z1) * Z3           (epilogue warpgroups 2(c%2), 2(c%2)+1, packed
//                                    f16 arithmetic on Z1/2) -> TMEM gate slot
//                                    (three, taken in turn by every chunk of every tile)
//   Y += gate * W2_chunk           (M=128, N=d, K=64, A from TMEM, B = f16 W2
//                                    image in smem) -> TMEM Y slot j % 2
// Keeping the gate in tensor memory avoids a shared-memory round trip and
// lets the N=d MMA run at full rate.  The Y epilogue of tile j runs in the
// warpgroup pair j % 2 (one half of the columns each) after that pair's
// chunks of tile j+1.
#pragma once
#include "sm100.cuh"

namespace ttt {

constexpr int kTileM = 128;
constexpr int kThreads = 640;        // 20 warps: 0 producer, 1 Z issuer, 2 Y issuer, 3 idle, 4-19 epilogue
constexpr int kYWarp = 2;            // second MMA-issuing warp
constexpr int kEpiWarp0 = 4;         // first epilogue warp (4 warpgroups of 4)
constexpr int kPrefetchAhead = 3;    // items whose tiles the producer prefetches into L2

struct FwdParams {
  const __nv_bfloat16* w13_img;  // per head: 2*HIDP rows of D bf16 (sw-swizzled)
  const __half* w2_img;          // per head: HIDP rows of D f16 (sw-swizzled)
  __nv_bfloat16* out;            // [n][heads][D]: O (bf16) or, in WRITE mode, E (f16 bits)
  int n, heads, tiles;
  unsigned int* status;
  long long wait_clocks;         // limit of a bounded wait (<= 0: the default)
};

template <int D, int HIDP>
struct FwdLayout {
  static constexpr int SW = 2 * D;
  static constexpr uint32_t kW13 = 2u * HIDP * D * 2;
  static constexpr uint32_t kW2 = 1u * HIDP * D * 2;
  static constexpr uint32_t kTile = 1u * kTileM * D * 2;
  static constexpr uint32_t off_w13 = 0;
  static constexpr uint32_t off_w2 = off_w13 + kW13;
  static constexpr uint32_t off_x = off_w2 + kW2;
  static constexpr uint32_t off_vp = off_x + 2 * kTile;
  static constexpr uint32_t off_bar = off_vp + 2 * kTile;
  static constexpr int kNumBars = 30;
  static constexpr uint32_t bytes = off_bar + kNumBars * 8 + 16 + 1024;
  static_assert(off_x % 1024 == 0 && off_vp % 1024 == 0, "1 KiB alignment");
};

// TMEM columns
constexpr uint32_t kFwdZCols = 0;      // 2 Z slots x 128
constexpr uint32_t kFwdGateCols = 256; // kFwdGateSlots gate slots x 32 (64 f16 per row)
constexpr int kFwdGateSlots = 3;       // taken in turn by the chunks of all tiles
constexpr uint32_t kFwdYCols = 352;    // 2 Y slots x D

// barrier indices
enum FwdBar {
  FB_W_FULL = 0, FB_W_EMPTY = 1, FB_X_FULL = 2, FB_X_EMPTY = 4, FB_VP_FULL = 6, FB_VP_EMPTY = 8,
  FB_Z_FULL = 10, FB_Z_EMPTY = 12, FB_Y_FULL = 18, FB_Y_EMPTY = 20,
  FB_DONE = 22, FB_G_FULL = 24, FB_G_EMPTY = FB_G_FULL + kFwdGateSlots
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Copy `bytes` (multiple of 16) from global to shared in 16 KiB bulk pieces.
__device__ __forceinline__ void bulk_load_pieces(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  for (uint32_t o = 0; o < bytes; o += 16384u) {
    const uint32_t len = bytes - o < 16384u ? bytes - o : 16384u;
    bulk_load(static_cast<uint8_t*>(dst) + o, static_cast<const uint8_t*>(src) + o, len, bar);
  }
}

// Position in the flattened (major, tile) work space (major = head in the
// forward kernel, (head, hidden slice) pair in the backward kernel), advanced
// without integer division: the issuing loops run once per MMA group and a
// 64-bit division costs hundreds of clocks there.
struct Cursor {
  long long it;
  int major, tile;
  __device__ __forceinline__ void init(long long i, int tiles) {
    it = i;
    major = static_cast<int>(i / tiles);
    tile = static_cast<int>(i % tiles);
  }
  __device__ __forceinline__ void next(int tiles) {
    ++it;
    if (++tile == tiles) {
      tile = 0;
      ++major;
    }
  }
};

// Bounded wait that ignores the abort flag (used only while draining).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitClockLimit) break;
  }
}

// Gate of two hidden units in packed f16: silu(z1) * z3.  The Z1 columns
// hold u = z1/2 (the W1 operand image is halved, exactly), and with
// t = tanh(u): sigmoid(z1) = (1 + t)/2, so silu(z1) = u (1 + t) = u + u t.
__device__ __forceinline__ uint32_t gate_f16x2(float ua, float ub, float z3a, float z3b) {
  const uint32_t hu = pack_f16x2(ua, ub);
  const uint32_t h3 = pack_f16x2(z3a, z3b);
  const uint32_t t = htanh2(hu);
  return hmul2(hfma2(hu, t, hu), h3);
}

template <int D, int HIDP, bool WRITE>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_vp,
               const FwdParams p) {
  using L = FwdLayout<D, HIDP>;
  constexpr int SW = L::SW;
  constexpr int NC = HIDP / 64;
  static_assert(NC % 2 == 0, "hidden chunks are split between two warpgroups");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const Abort ab{abort_flag, p.status, p.wait_clocks};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const long long total = static_cast<long long>(p.heads) * p.tiles;
  const long long it0 = total * blockIdx.x / gridDim.x;
  const long long it1 = total * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(&bars[FB_W_FULL], 1);
    mbar_init(&bars[FB_W_EMPTY], 2);    // released by both issuing warps
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[FB_X_FULL + s], 1);
      mbar_init(&bars[FB_X_EMPTY + s], 1);
      mbar_init(&bars[FB_VP_FULL + s], 1);
      mbar_init(&bars[FB_VP_EMPTY + s], 8);
      mbar_init(&bars[FB_Z_FULL + s], 1);
      mbar_init(&bars[FB_Z_EMPTY + s], 8);
      mbar_init(&bars[FB_Y_FULL + s], 1);
      mbar_init(&bars[FB_Y_EMPTY + s], 8);
    }
    for (int s = 0; s < kFwdGateSlots; ++s) {
      mbar_init(&bars[FB_G_FULL + s], 8);    // the eight warps of the pair that gated the chunk
      mbar_init(&bars[FB_G_EMPTY + s], 1);
    }
    mbar_init(&bars[FB_DONE], 2);
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
  const uint32_t tz = tbase + kFwdZCols;
  const uint32_t tg = tbase + kFwdGateCols;
  const uint32_t ty = tbase + kFwdYCols;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      TTT_TR_DECL
      tma_prefetch_desc(&tm_x);
      if (WRITE) tma_prefetch_desc(&tm_vp);
      int cur_head = -1;
      uint32_t wl = 0, j = 0, nx = 0, nvp = 0;
      Cursor pf;
      pf.init(it0, p.tiles);
      for (int k = 0; k < kPrefetchAhead && pf.it < it1; ++k, pf.next(p.tiles)) {
        tma_prefetch_l2_2d(&tm_x, pf.major * D, pf.tile * kTileM);
        if (WRITE) tma_prefetch_l2_2d(&tm_vp, pf.major * D, pf.tile * kTileM);
      }
      Cursor cu;
      cu.init(it0, p.tiles);
      for (; cu.it < it1; cu.next(p.tiles), ++j) {
        const int head = cu.major;
        const int tile = cu.tile;
        if (head != cur_head) {
          if (wl > 0 && !mbar_wait(&bars[FB_W_EMPTY], (wl - 1) & 1, ab)) break;
          mbar_arrive_expect_tx(&bars[FB_W_FULL], L::kW13 + L::kW2);
          bulk_load_pieces(smem + L::off_w13, p.w13_img + static_cast<size_t>(head) * (L::kW13 / 2), L::kW13,
                           &bars[FB_W_FULL]);
          bulk_load_pieces(smem + L::off_w2, p.w2_img + static_cast<size_t>(head) * (L::kW2 / 2), L::kW2,
                           &bars[FB_W_FULL]);
          ++wl;
          cur_head = head;
        }
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        // Warm L2 with the tiles a few items ahead so the shared-memory loads hit L2.
        if (pf.it < it1) {
          tma_prefetch_l2_2d(&tm_x, pf.major * D, pf.tile * kTileM);
          if (WRITE) tma_prefetch_l2_2d(&tm_vp, pf.major * D, pf.tile * kTileM);
          pf.next(p.tiles);
        }
        TTT_TR_LAP(0);
        if (!mbar_wait(&bars[FB_X_EMPTY + s], ph ^ 1, ab)) break;
        TTT_TR_LAP(1);
        mbar_arrive_expect_tx(&bars[FB_X_FULL + s], L::kTile);
        tma_load_2d(smem + L::off_x + s * L::kTile, &tm_x, &bars[FB_X_FULL + s], head * D, tile * kTileM);
        ++nx;
        if (WRITE) {
          TTT_TR_LAP(0);
          if (!mbar_wait(&bars[FB_VP_EMPTY + s], ph ^ 1, ab)) break;
          TTT_TR_LAP(2);
          mbar_arrive_expect_tx(&bars[FB_VP_FULL + s], L::kTile);
          tma_load_2d(smem + L::off_vp + s * L::kTile, &tm_vp, &bars[FB_VP_FULL + s], head * D, tile * kTileM);
          ++nvp;
        }
      }
      TTT_TR_LAP(0);
      TTT_TR_DUMP(WRITE ? 0 : 1);
      // Drain: the last load issued into each barrier has landed before exit
      // (after an abort the X load of an item may have gone out without its V').
      if (wl > 0) mbar_drain(&bars[FB_W_FULL], (wl - 1) & 1);
      for (uint32_t jj = (nx >= 2 ? nx - 2 : 0); jj < nx; ++jj) mbar_drain(&bars[FB_X_FULL + (jj & 1)], (jj >> 1) & 1);
      for (uint32_t jj = (nvp >= 2 ? nvp - 2 : 0); jj < nvp; ++jj)
        mbar_drain(&bars[FB_VP_FULL + (jj & 1)], (jj >> 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ Z issuer
    // Z = X * [W1 | W3]_chunk into TMEM slot c % 2 as soon as the slot is free.
    constexpr uint32_t kIdZ = idesc_bf16(128, 128, false, false);
    const uint32_t w13 = smem_u32(smem + L::off_w13);
    TTT_TR_DECL
    Cursor zc;
    zc.init(it0, p.tiles);
    int cur_head = -1;
    uint32_t zj = 0, zcount = 0, wl = 0;
    bool ok = true;
    for (; zc.it < it1 && ok; zc.next(p.tiles), ++zj) {
      if (zc.major != cur_head) {
        if (cur_head >= 0) mma_commit_warp(&bars[FB_W_EMPTY]);
        if (!(ok = mbar_wait_warp(&bars[FB_W_FULL], wl & 1, ab))) break;
        ++wl;
        cur_head = zc.major;
      }
      const int s = zj & 1;
      TTT_TR_LAP(0);
      if (!(ok = mbar_wait_warp(&bars[FB_X_FULL + s], (zj >> 1) & 1, ab))) break;
      TTT_TR_LAP(1);
      const uint32_t xa = smem_u32(smem + L::off_x + s * L::kTile);
      for (int c = 0; c < NC; ++c, ++zcount) {
        const int zs = c & 1;
        TTT_TR_LAP(0);
        if (!(ok = mbar_wait_warp(&bars[FB_Z_EMPTY + zs], ((zcount >> 1) & 1) ^ 1, ab))) break;
        TTT_TR_LAP(2);
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t ad = smem_desc(xa + 32 * k, 0, 8 * SW, SW);
          const uint64_t bd = smem_desc(w13 + 128 * c * SW + 32 * k, 0, 8 * SW, SW);
          mma_bf16_warp(tz + zs * 128, ad, bd, kIdZ, k > 0 ? 1u : 0u);
        }
        mma_commit_warp(&bars[FB_Z_FULL + zs]);
        TTT_TR_LAP(3);
      }
      if (ok) mma_commit_warp(&bars[FB_X_EMPTY + s]);
    }
    TTT_TR_DUMP(WRITE ? 0 : 1);
    // All issued MMAs have completed before TMEM is released.
    mma_commit_warp(&bars[FB_DONE]);
    mbar_drain(&bars[FB_DONE], 0);
  } else if (warp == kYWarp) {
    // ------------------------------------------------------------ Y issuer
    // Y += gate_chunk * W2_chunk once the gate of the chunk is in TMEM.
    constexpr uint32_t kIdY = idesc_f16(128, D, false, true);
    const uint32_t w2 = smem_u32(smem + L::off_w2);
    Cursor yc;
    yc.init(it0, p.tiles);
    int cur_head = -1;
    uint32_t yj = 0, wl = 0;
    bool ok = true;
    for (; yc.it < it1 && ok; yc.next(p.tiles), ++yj) {
      if (yc.major != cur_head) {
        if (cur_head >= 0) mma_commit_warp(&bars[FB_W_EMPTY]);
        if (!(ok = mbar_wait_warp(&bars[FB_W_FULL], wl & 1, ab))) break;
        ++wl;
        cur_head = yc.major;
      }
      const uint32_t ys = yj & 1;
      if (!(ok = mbar_wait_warp(&bars[FB_Y_EMPTY + ys], ((yj >> 1) & 1) ^ 1, ab))) break;
      for (int c = 0; c < NC; ++c) {
        const uint32_t gc = yj * NC + c;   // chunk counter: gate slot gc % kFwdGateSlots
        const uint32_t gs = gc % kFwdGateSlots;
        if (!(ok = mbar_wait_warp(&bars[FB_G_FULL + gs], (gc / kFwdGateSlots) & 1, ab))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t bd = smem_desc(w2 + (64 * c + 16 * k) * SW, HIDP * SW, 8 * SW, SW);
          mma_bf16_ts_warp(ty + ys * D, tg + gs * 32 + 8 * k, bd, kIdY, (c > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit_warp(&bars[FB_G_EMPTY + gs]);
      }
      if (ok) mma_commit_warp(&bars[FB_Y_FULL + ys]);
    }
    mma_commit_warp(&bars[FB_DONE]);
    mbar_drain(&bars[FB_DONE], 0);
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int e = (warp - kEpiWarp0) >> 2;  // warpgroup 0..3
    const int pr = e >> 1;                  // pair: chunks c % 2 == pr, Y of tiles j % 2 == pr
    const int hf = e & 1;                   // half of the chunk (32 hidden) / of the Y columns
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;          // token row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    constexpr int kYHalf = D / 2;           // Y columns per warpgroup
    uint32_t j = 0, u = 0;
    TTT_TR_DECL

    // Y epilogue of tile jj (head, tile): columns [hf*D/2, (hf+1)*D/2).
    auto y_epilogue = [&](uint32_t jj, int head, int tile) -> bool {
      const uint32_t ys = jj & 1;
      TTT_TR_LAP(0);
      if (!mbar_wait_warp(&bars[FB_Y_FULL + ys], (jj >> 1) & 1, ab)) return false;
      TTT_TR_LAP(5);
      tc_fence_after();
      float y[kYHalf];
      const uint32_t yb = ty + ys * D + hf * kYHalf + lane_off;
      if (kYHalf >= 16) {
#pragma unroll
        for (int c0 = 0; c0 < kYHalf; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(yb + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) y[c0 + i] = __uint_as_float(r[i]);
        }
      } else {
        uint32_t r[8];
        tmem_ld8(yb, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = __uint_as_float(r[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[FB_Y_EMPTY + ys]);
      if (WRITE) {
        if (!mbar_wait_warp(&bars[FB_VP_FULL + ys], (jj >> 1) & 1, ab)) return false;
        const uint32_t vb = smem_u32(smem + L::off_vp + ys * L::kTile);
#pragma unroll
        for (int ch = 0; ch < kYHalf / 8; ++ch) {
          uint32_t v0, v1, v2, v3;
          ld_shared_v4(vb + swz(row * SW + (hf * kYHalf / 8 + ch) * 16, SW), v0, v1, v2, v3);
          y[8 * ch + 0] -= bf16lo(v0); y[8 * ch + 1] -= bf16hi(v0);
          y[8 * ch + 2] -= bf16lo(v1); y[8 * ch + 3] -= bf16hi(v1);
          y[8 * ch + 4] -= bf16lo(v2); y[8 * ch + 5] -= bf16hi(v2);
          y[8 * ch + 6] -= bf16lo(v3); y[8 * ch + 7] -= bf16hi(v3);
        }
      }
      const long long tok = static_cast<long long>(tile) * kTileM + row;
      if (tok < p.n) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + (tok * p.heads + head) * D + hf * kYHalf);
        // O in bf16; the residual E in f16, the backward kernel's operand type
        auto pk = [](float a, float b) { return WRITE ? pack_f16x2(a, b) : pack_bf16x2(a, b); };
#pragma unroll
        for (int ch = 0; ch < kYHalf / 8; ++ch) {
          uint4 v;
          v.x = pk(y[8 * ch + 0], y[8 * ch + 1]);
          v.y = pk(y[8 * ch + 2], y[8 * ch + 3]);
          v.z = pk(y[8 * ch + 4], y[8 * ch + 5]);
          v.w = pk(y[8 * ch + 6], y[8 * ch + 7]);
          dst[ch] = v;
        }
      }
      if (WRITE) {
        // The V' stage is refilled by TMA (async proxy) once all eight warps
        // have arrived.  An arrive right after the shared loads let the refill
        // land before the last loads of some lanes had returned, so the stage
        // is released only after the residual has been stored (the stores
        // consume every loaded value), behind a generic-to-async proxy fence.
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[FB_VP_EMPTY + ys]);
      }
      TTT_TR_LAP(6);
      return true;
    };

    bool ok = true;
    int prev_head = 0, prev_tile = 0;
    Cursor cu;
    cu.init(it0, p.tiles);
    for (; cu.it < it1 && ok; cu.next(p.tiles), ++j) {
      for (int c = pr; c < NC; c += 2, ++u) {
        TTT_TR_LAP(0);
        if (!(ok = mbar_wait_warp(&bars[FB_Z_FULL + pr], u & 1, ab))) break;
        TTT_TR_LAP(1);
        tc_fence_after();
        // Z slot columns: [Z1 (32) | Z3 (32)] of hidden 64c + 0..31, then of 64c + 32..63;
        // this warpgroup's half hf is columns 64*hf .. 64*hf + 63.
        const uint32_t zb = tz + pr * 128 + hf * 64 + lane_off;
        uint32_t gk[16];  // 32 gate values of this row as f16 pairs
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          uint32_t z1[16], z3[16];
          tmem_ld16(zb + part * 16, z1);
          tmem_ld16(zb + 32 + part * 16, z3);
          tmem_wait_ld();
          TTT_TR_LAP(7);
#pragma unroll
          for (int i = 0; i < 16; i += 2)
            gk[part * 8 + i / 2] = gate_f16x2(__uint_as_float(z1[i]), __uint_as_float(z1[i + 1]),
                                              __uint_as_float(z3[i]), __uint_as_float(z3[i + 1]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[FB_Z_EMPTY + pr]);
        TTT_TR_LAP(2);
        const uint32_t gc = j * NC + c;   // chunk counter: gate slot gc % kFwdGateSlots
        const uint32_t gs = gc % kFwdGateSlots;
        if (!(ok = mbar_wait_warp(&bars[FB_G_EMPTY + gs], ((gc / kFwdGateSlots) & 1) ^ 1, ab))) break;
        TTT_TR_LAP(3);
        tc_fence_after();
        tmem_st16(tg + gs * 32 + hf * 16 + lane_off, gk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[FB_G_FULL + gs]);
        TTT_TR_LAP(4);
      }
      if (!ok) break;
      if (j >= 1 && ((j - 1) & 1) == static_cast<uint32_t>(pr)) ok = y_epilogue(j - 1, prev_head, prev_tile);
      prev_head = cu.major;
      prev_tile = cu.tile;
    }
    if (ok && j >= 1 && ((j - 1) & 1) == static_cast<uint32_t>(pr)) y_epilogue(j - 1, prev_head, prev_tile);
    TTT_TR_LAP(0);
    if (hf == 0 && pr == 0) TTT_TR_DUMP(WRITE ? 0 : 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace ttt
