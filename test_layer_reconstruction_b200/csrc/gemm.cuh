// gemm.cuh — persistent bf16 GEMM on the 5th-generation tensor cores with
// fused epilogues, for the products that are plain dense GEMMs:
//   * the wide-head layer (one head with d = 1024, h = 2048; VGG-T$^3$:
//     Offline Feed-Forward 3D Reconstruction at Scale, Sec. 3.4, Eq. 3-5),
//     where one head's fast weights no longer fit on chip, and
//   * the layer's surround: the QKV projection with the per-head L2
//     normalisation of q and k in its epilogue (Sec. 3, Eq. 1, and "The
//     LayerNorm removal"), and the output projection.
//
// C[m][n] = sum_k A[m][k] B[k][n] with bf16 operands and FP32 accumulation
// in tensor memory.  Each operand is read by TMA from a 2-D bf16 tensor in
// one of two layouts:
//   K-major : the operand's rows are M (or N) and K is contiguous (A stored
//             [M][K], B stored [N][K]); TMA box 64 (K) x 128 rows.
//   MN-major: the rows are K and M (or N) is contiguous (A stored [K][M],
//             B stored [K][N]); TMA box 64 (M or N) x 64 (K rows).
// Both use the 128-byte swizzle.
//
// CTA pairs (clusters of two) share each 256 x 256 tile through the
// tensor cores' two-CTA form (cta_group::2): CTA r of the pair loads rows
// 128r..128r+127 of the tile's A and columns 128r..128r+127 of its B (16 KiB
// each per K step of 64), the leader issues M=256, N=256, K=16 MMAs that read
// both CTAs' shared memory, and each CTA's tensor memory holds its own 128
// rows of the accumulator.  Per SM and K step that is 32 KiB of operands for
// 2 x 128 x 256 x 64 FLOPs, a third less than a one-CTA 128 x 256 tile, which
// leaves shared-memory bandwidth for the epilogue and fits six stages.  Both
// CTAs' loads complete on the leader's stage barrier; the leader's commits
// reach both CTAs' barriers (multicast to the pair); each CTA's epilogue
// arrives on the leader's accumulator-free barrier.
//
// Each pair walks the work items (problem, 256-row M tile, N tile, K split)
// of up to three problems with a static stride.  Warp roles, in both CTAs:
//   warp 0     TMA producer
//   warp 1     TMEM allocator; in the leader also the MMA issuer
//              (warp-uniform, one elected lane)
//   warps 4-11 epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (rows of
//              the CTA's half tile); warps 4-7 take the first half of the
//              tile's columns, warps 8-11 the second.
// The accumulator is double buffered in TMEM (2 x 256 columns), so the
// epilogue of one tile overlaps the MMAs of the next.  Rows and columns past
// a problem's M and N are computed on TMA's zero fill and not stored.
//
// Epilogues (template parameter):
//   kEpiStore    out = bf16(C) (a column offset lets a tile land inside a
//                wider row, e.g. one head's columns of [n][heads*d]).
//   kEpiResidual out = bf16(C - R) with R a bf16 tensor of out's shape.
//   kEpiL2Heads  the tile's columns are heads of 64: columns below
//                `norm_cols` are divided by the L2 norm of their 64-column
//                row segment (a zero segment stays zero), then bf16.
//   kEpiGate     the tile's columns are [Z1 of 128 hidden units | Z3 of the
//                same units]: A = silu(Z1) Z3, F1 = Z3 s (1 + Z1 (1 - s)) and
//                F3 = silu(Z1) with s = sigmoid(Z1), each bf16 [rows][hidden]
//                (F1 and F3 optional): A feeds the next products, and
//                dZ1 = dA F1, dZ3 = dA F3 is the chain rule of the backward.
//   kEpiDz       C = dA (columns = hidden units): dZ1 = dA F1, dZ3 = dA F3
//                written in place over F1 and F3.
//   kEpiAccF32   f32 [M][N] at out + split * split_stride = C, or += C when
//                `accumulate`: the split-K partial sums of the weight
//                gradients, each element owned by one CTA per launch, so the
//                sums are deterministic.
#pragma once
#include "fwd.cuh"

namespace ttt {

constexpr int kGemmBM = 256, kGemmBN = 256, kGemmBK = 64;   // tile of a CTA pair
constexpr int kGemmHalfM = kGemmBM / 2, kGemmHalfN = kGemmBN / 2; // loaded by each CTA
constexpr int kGemmStages = 6;
constexpr int kGemmThreads = 384;    // 12 warps
constexpr int kGemmEpiWarp0 = 4;
constexpr int kGemmMaxProblems = 3;

enum GemmEpilogue { kEpiStore = 0, kEpiResidual = 1, kEpiL2Heads = 2, kEpiGate = 3, kEpiDz = 4, kEpiAccF32 = 5 };

struct GemmProblem {
  int M, N;          // output extent
  int K;             // reduction length (the maps' extent along K; TMA zero-fills past it)
  int splits;        // K splits (kEpiAccF32 only; otherwise 1)
  int k_per_split;   // multiple of kGemmBK
  int a_mn, b_mn;    // operand layouts: 1 = MN-major
  int a_x0, a_y0;    // coordinate offsets of the A map (x = inner dimension)
  int b_x0, b_y0;    // likewise B
  // epilogue operands
  void* out;         // bf16, or f32 for kEpiAccF32
  long long ldo;     // row pitch of out in elements
  int out_col0;      // column offset inside out's rows
  const __nv_bfloat16* res;   // kEpiResidual: [rows][ldr] at column res_col0
  long long ldr;
  int res_col0;
  __nv_bfloat16* f1;          // kEpiGate: F1 out (may be null); kEpiDz: F1 in / dZ1 out
  __nv_bfloat16* f3;          // likewise F3 / dZ3
  long long ldf;              // row pitch of A, F1, F3 (hidden units)
  int norm_cols;              // kEpiL2Heads: columns [0, norm_cols) are normalised per 64
  int accumulate;             // kEpiAccF32: add to out instead of overwriting
  long long split_stride;     // kEpiAccF32: elements between the partials of consecutive splits
  int tiles_m, tiles_n;       // filled by the host
  long long items;            // tiles_m * tiles_n * splits
};

struct GemmParams {
  GemmProblem prob[kGemmMaxProblems];
  int n_problems;
  long long total_items;
  unsigned int* status;
  long long wait_clocks;      // limit of a bounded wait (<= 0: the default)
};

struct GemmLayout {
  static constexpr uint32_t kA = kGemmHalfM * kGemmBK * 2;   // 16 KiB: this CTA's A rows
  static constexpr uint32_t kB = kGemmHalfN * kGemmBK * 2;   // 16 KiB: this CTA's B columns
  static constexpr uint32_t kStage = kA + kB;
  // per epilogue warp: 32 rows x 64 bytes, rows padded to 80 bytes (no bank conflicts)
  static constexpr uint32_t kStgPitch = 80, kStgBytes = 32 * kStgPitch;
  static constexpr uint32_t off_stg = kGemmStages * kStage;
  static constexpr uint32_t off_bar = off_stg + 8 * kStgBytes;
  static constexpr int kNumBars = 2 * kGemmStages + 4 + 1;
  static constexpr uint32_t bytes = off_bar + kNumBars * 8 + 16 + 1024;
};

// Work item -> (problem, tile m, tile n, split); tiles of one M row are
// consecutive, so the CTAs that run at the same time share their A rows in L2.
struct GemmItem {
  int p, tm, tn, s;
};
__device__ __forceinline__ GemmItem gemm_item(const GemmParams& P, long long it) {
  GemmItem w{0, 0, 0, 0};
  int p = 0;
  while (p + 1 < P.n_problems && it >= P.prob[p].items) {
    it -= P.prob[p].items;
    ++p;
  }
  const GemmProblem& q = P.prob[p];
  w.p = p;
  const long long per_s = static_cast<long long>(q.tiles_m) * q.tiles_n;
  w.s = static_cast<int>(it / per_s);
  const long long r = it % per_s;
  w.tm = static_cast<int>(r / q.tiles_n);
  w.tn = static_cast<int>(r % q.tiles_n);
  return w;
}

__device__ __forceinline__ void gemm_k_range(const GemmProblem& q, int s, int* k0, int* nkb) {
  const int lo = s * q.k_per_split;
  int hi = lo + q.k_per_split;
  if (hi > q.K) hi = q.K;
  *k0 = lo;
  *nkb = hi > lo ? (hi - lo + kGemmBK - 1) / kGemmBK : 0;
}

__device__ __forceinline__ uint32_t gemm_idesc(int a_mn, int b_mn) {
  return idesc_bf16(kGemmBM, kGemmBN, a_mn != 0, b_mn != 0);
}

// ------------------------------------------------------------------ CTA pairs
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on an mbarrier given by its cluster address (this CTA's or the peer's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
// 2-D TMA load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem, both CTAs] (+)= A[smem, both CTAs] * B[smem, both CTAs], issued by one elected lane.
__device__ __forceinline__ void mma_pair_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this address in both CTAs of the pair when
// every MMA issued so far by this thread completes.
__device__ __forceinline__ void mma_commit_pair_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b16 m;\n\t"
      "mov.b16 m, 3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 bits, 32 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// One MUFU operation per element: sigmoid(z) = (1 + tanh(z/2)) / 2.
__device__ __forceinline__ float gemm_sigmoid(float z) { return sigmoid_fast(z); }

__device__ __forceinline__ void store_bf16x8(__nv_bfloat16* dst, const float* v) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(dst) = u;
}
__device__ __forceinline__ void load_bf16x8(const __nv_bfloat16* src, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x);
  v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
  v[4] = bf16lo(u.z); v[5] = bf16hi(u.z);
  v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}

// Coalesced epilogue I/O.  A warp's 32 threads own 32 rows of the tile (one
// row each, the layout of the tensor-memory loads); written straight to
// global memory, one instruction would touch 32 rows.  Staged through the
// warp's 32 x 64-byte shared buffer instead, each instruction moves 64
// contiguous bytes of 8 rows.  `m0` is the warp's first row; rows at or past
// `M` and 8-column groups at or past `N` are skipped.
struct StageIO {
  uint32_t buf;   // this warp's staging buffer (shared address)
  int lane;
  // This thread's 32 bf16 (four 16-byte vectors) of its row -> rows m0.. of
  // `dst` (row pitch `ld` elements) at column `col`.
  __device__ __forceinline__ void store_bf16(const uint4 (&v)[4], __nv_bfloat16* dst, long long ld, long long m0,
                                             long long M, int col, int N) const {
#pragma unroll
    for (int c = 0; c < 4; ++c) st_shared_v4(buf + lane * GemmLayout::kStgPitch + c * 16, v[c].x, v[c].y, v[c].z, v[c].w);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = i * 8 + (lane >> 2), c = lane & 3;
      uint4 x;
      ld_shared_v4(buf + r * GemmLayout::kStgPitch + c * 16, x.x, x.y, x.z, x.w);
      if (m0 + r < M && col + 8 * c < N) *reinterpret_cast<uint4*>(dst + (m0 + r) * ld + col + 8 * c) = x;
    }
    __syncwarp();
  }
  // The reverse: rows m0.. of `src` at column `col` -> this thread's row (32 bf16).
  __device__ __forceinline__ void load_bf16(uint4 (&v)[4], const __nv_bfloat16* src, long long ld, long long m0,
                                            long long M, int col, int N) const {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = i * 8 + (lane >> 2), c = lane & 3;
      uint4 x = make_uint4(0u, 0u, 0u, 0u);
      if (m0 + r < M && col + 8 * c < N) x = *reinterpret_cast<const uint4*>(src + (m0 + r) * ld + col + 8 * c);
      st_shared_v4(buf + r * GemmLayout::kStgPitch + c * 16, x.x, x.y, x.z, x.w);
    }
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 4; ++c) ld_shared_v4(buf + lane * GemmLayout::kStgPitch + c * 16, v[c].x, v[c].y, v[c].z, v[c].w);
    __syncwarp();
  }
  // f32 versions: 16 floats (64 bytes) of the row.
  __device__ __forceinline__ void store_f32(const float4 (&v)[4], float* dst, long long ld, long long m0, long long M,
                                            int col, int N) const {
    store_bf16(reinterpret_cast<const uint4(&)[4]>(v), reinterpret_cast<__nv_bfloat16*>(dst), 2 * ld, m0, M, 2 * col,
               2 * N);
  }
  __device__ __forceinline__ void load_f32(float4 (&v)[4], const float* src, long long ld, long long m0, long long M,
                                           int col, int N) const {
    load_bf16(reinterpret_cast<uint4(&)[4]>(v), reinterpret_cast<const __nv_bfloat16*>(src), 2 * ld, m0, M, 2 * col,
              2 * N);
  }
};

__device__ __forceinline__ uint4 pack_bf16x8(const float* v) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}
__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float* v) {
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x);
  v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
  v[4] = bf16lo(u.z); v[5] = bf16hi(u.z);
  v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tma0, const __grid_constant__ CUtensorMap tmb0,
                const __grid_constant__ CUtensorMap tma1, const __grid_constant__ CUtensorMap tmb1,
                const __grid_constant__ CUtensorMap tma2, const __grid_constant__ CUtensorMap tmb2,
                const __grid_constant__ GemmParams P) {
  using L = GemmLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kGemmStages;
  uint64_t* acc_full = bars + 2 * kGemmStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const Abort ab{abort_flag, P.status, P.wait_clocks};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();           // 0: the pair's leader
  const long long pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&full[s], 1);     // the leader's expect_tx; both CTAs' loads complete on it
      mbar_init(&empty[s], 1);    // the leader's commit, multicast to both CTAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 16);   // the epilogue warps of both CTAs (the leader's is used)
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers exist before either CTA signals the other's
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const CUtensorMap* ma[3] = {&tma0, &tma1, &tma2};
      const CUtensorMap* mb[3] = {&tmb0, &tmb1, &tmb2};
      for (int p = 0; p < P.n_problems; ++p) {
        tma_prefetch_desc(ma[p]);
        tma_prefetch_desc(mb[p]);
      }
      const uint32_t full_leader = map_to_rank(smem_u32(full), 0);
      uint32_t stage = 0, ph = 0, issued = 0;
      bool ok = true;
      for (long long it = pair; it < P.total_items && ok; it += npairs) {
        const GemmItem w = gemm_item(P, it);
        const GemmProblem& q = P.prob[w.p];
        int k0, nkb;
        gemm_k_range(q, w.s, &k0, &nkb);
        const int m0 = w.tm * kGemmBM + rank * kGemmHalfM, n0 = w.tn * kGemmBN + rank * kGemmHalfN;
        for (int kb = 0; kb < nkb; ++kb) {
          const int k = k0 + kb * kGemmBK;
          if (!(ok = mbar_wait(&empty[stage], ph ^ 1, ab))) break;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * L::kStage);
          const uint32_t bar = full_leader + stage * 8;
          uint8_t* sa = smem + stage * L::kStage;
          uint8_t* sb = sa + L::kA;
          if (q.a_mn) {
            tma_load_2d_pair(sa, ma[w.p], bar, q.a_x0 + m0, q.a_y0 + k);
            tma_load_2d_pair(sa + 8192, ma[w.p], bar, q.a_x0 + m0 + 64, q.a_y0 + k);
          } else {
            tma_load_2d_pair(sa, ma[w.p], bar, q.a_x0 + k, q.a_y0 + m0);
          }
          if (q.b_mn) {
            tma_load_2d_pair(sb, mb[w.p], bar, q.b_x0 + n0, q.b_y0 + k);
            tma_load_2d_pair(sb + 8192, mb[w.p], bar, q.b_x0 + n0 + 64, q.b_y0 + k);
          } else {
            tma_load_2d_pair(sb, mb[w.p], bar, q.b_x0 + k, q.b_y0 + n0);
          }
          ++issued;
          if (++stage == kGemmStages) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      // Drain (leader): the stage barriers count both CTAs' loads, so the last
      // load issued into each stage by either CTA has landed before exit.  The
      // peer cannot wait on the leader's barriers; it leaves only after the
      // closing cluster barrier, which the leader reaches after this drain.
      if (rank == 0) {
        const uint32_t last = issued < static_cast<uint32_t>(kGemmStages) ? issued : kGemmStages;
        for (uint32_t b = 0; b < last; ++b) {
          const uint32_t jj = issued - 1 - b;
          mbar_drain(&full[jj % kGemmStages], (jj / kGemmStages) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (rank == 0) {
      const uint32_t sbase = smem_u32(smem);
      uint32_t stage = 0, ph = 0, local = 0;
      bool ok = true;
      for (long long it = pair; it < P.total_items && ok; it += npairs, ++local) {
        const GemmItem w = gemm_item(P, it);
        const GemmProblem& q = P.prob[w.p];
        int k0, nkb;
        gemm_k_range(q, w.s, &k0, &nkb);
        const uint32_t buf = local & 1;
        if (!(ok = mbar_wait_warp(&acc_empty[buf], ((local >> 1) & 1) ^ 1, ab))) break;
        tc_fence_after();
        const uint32_t idesc = gemm_idesc(q.a_mn, q.b_mn);
        // per K=16 step: K-major operands advance 32 bytes, MN-major ones 16 rows of 128 bytes
        const uint32_t a_step = q.a_mn ? 2048u : 32u, b_step = q.b_mn ? 2048u : 32u;
        const uint32_t a_lbo = q.a_mn ? 8192u : 16u, b_lbo = q.b_mn ? 8192u : 16u;
        const uint32_t tacc = tbase + buf * kGemmBN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!(ok = mbar_wait_warp(&full[stage], ph, ab))) break;
          tc_fence_after();
          const uint32_t sa = sbase + stage * L::kStage, sb = sa + L::kA;
          const uint64_t ad = smem_desc(sa, a_lbo, 1024, 128), bd = smem_desc(sb, b_lbo, 1024, 128);
#pragma unroll
          for (int k = 0; k < kGemmBK / 16; ++k)
            mma_pair_warp(tacc, ad + ((k * a_step) >> 4), bd + ((k * b_step) >> 4), idesc,
                          (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit_pair_warp(&empty[stage]);
          if (++stage == kGemmStages) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (ok) mma_commit_pair_warp(&acc_full[buf]);
      }
      // All issued MMAs (which write both CTAs' tensor memory) have completed
      // before either CTA releases it.
      mma_commit_pair_warp(done);
    }
    mbar_drain(done, 0);
  } else if (warp >= kGemmEpiWarp0) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int e = warp - kGemmEpiWarp0;      // 0..7
    const int quad = warp & 3;               // TMEM lane quadrant
    const int hf = e >> 2;                   // column half of the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t acc_empty_leader = map_to_rank(smem_u32(acc_empty), 0);
    const StageIO io{smem_u32(smem + L::off_stg + e * L::kStgBytes), lane};
    uint32_t local = 0;
    for (long long it = pair; it < P.total_items; it += npairs, ++local) {
      const GemmItem w = gemm_item(P, it);
      const GemmProblem& q = P.prob[w.p];
      const uint32_t buf = local & 1;
      if (!mbar_wait_warp(&acc_full[buf], (local >> 1) & 1, ab)) break;
      tc_fence_after();
      const uint32_t tacc = tbase + buf * kGemmBN + lane_off;
      const int n0 = w.tn * kGemmBN;
      const long long m0 = static_cast<long long>(w.tm) * kGemmBM + rank * kGemmHalfM + quad * 32;
      if (EPI == kEpiGate) {
        // hidden units [64 hf, 64 hf + 64) of this tile: Z1 at columns c, Z3 at 128 + c
        const int hid0 = w.tn * 128 + hf * 64;
        const int nh = q.N / 2;   // hidden units (padded) = row length of A, F1, F3
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          uint32_t z1[32], z3[32];
          tmem_ld32(tacc + hf * 64 + c0, z1);
          tmem_ld32(tacc + 128 + hf * 64 + c0, z3);
          tmem_wait_ld();
          const int hid = hid0 + c0;
          uint4 a[4], f1[4], f3[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            float va[8], v1[8], v3[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float x1 = __uint_as_float(z1[8 * g + i]), x3 = __uint_as_float(z3[8 * g + i]);
              const float sg = gemm_sigmoid(x1);
              const float silu = x1 * sg;
              va[i] = silu * x3;
              v3[i] = silu;
              v1[i] = x3 * sg * (1.f + x1 * (1.f - sg));
            }
            a[g] = pack_bf16x8(va);
            f1[g] = pack_bf16x8(v1);
            f3[g] = pack_bf16x8(v3);
          }
          io.store_bf16(a, reinterpret_cast<__nv_bfloat16*>(q.out), q.ldf, m0, q.M, hid, nh);
          if (q.f1) io.store_bf16(f1, q.f1, q.ldf, m0, q.M, hid, nh);
          if (q.f3) io.store_bf16(f3, q.f3, q.ldf, m0, q.M, hid, nh);
        }
      } else if (EPI == kEpiAccF32) {
        float* out = reinterpret_cast<float*>(q.out) + static_cast<long long>(w.s) * q.split_stride;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(tacc + hf * 128 + c0, r);
          tmem_wait_ld();
          const int col = n0 + hf * 128 + c0;
          float4 x[4];
#pragma unroll
          for (int v = 0; v < 4; ++v)
            x[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]), __uint_as_float(r[4 * v + 2]),
                               __uint_as_float(r[4 * v + 3]));
          if (q.accumulate) {
            float4 o[4];
            io.load_f32(o, out, q.ldo, m0, q.M, col, q.N);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              x[v].x += o[v].x; x[v].y += o[v].y; x[v].z += o[v].z; x[v].w += o[v].w;
            }
          }
          io.store_f32(x, out, q.ldo, m0, q.M, col, q.N);
        }
      } else if (EPI == kEpiL2Heads) {
        // two heads of 64 columns per half
#pragma unroll 1
        for (int hd = 0; hd < 2; ++hd) {
          uint32_t r0[32], r1[32];
          const int c = hf * 128 + hd * 64;
          tmem_ld32(tacc + c, r0);
          tmem_ld32(tacc + c + 32, r1);
          tmem_wait_ld();
          const int col = n0 + c;
          float scale = 1.f;
          if (col < q.norm_cols) {
            float ss = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float x0 = __uint_as_float(r0[i]), x1 = __uint_as_float(r1[i]);
              ss = fmaf(x0, x0, ss);
              ss = fmaf(x1, x1, ss);
            }
            scale = ss > 0.f ? rsqrtf(ss) : 0.f;
          }
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(q.out) + q.out_col0;
          uint4 v[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            float t[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) t[i] = __uint_as_float(r0[8 * g + i]) * scale;
            v[g] = pack_bf16x8(t);
          }
          io.store_bf16(v, dst, q.ldo, m0, q.M, col, q.N);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            float t[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) t[i] = __uint_as_float(r1[8 * g + i]) * scale;
            v[g] = pack_bf16x8(t);
          }
          io.store_bf16(v, dst, q.ldo, m0, q.M, col + 32, q.N);
        }
      } else {
        // kEpiStore, kEpiResidual, kEpiDz: 128 columns of this half in chunks of 32
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tacc + hf * 128 + c0, r);
          tmem_wait_ld();
          const int col = n0 + hf * 128 + c0;
          if (EPI == kEpiDz) {
            uint4 f1[4], f3[4];
            io.load_bf16(f1, q.f1, q.ldf, m0, q.M, col, q.N);
            io.load_bf16(f3, q.f3, q.ldf, m0, q.M, col, q.N);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              float a1[8], a3[8];
              unpack_bf16x8(f1[g], a1);
              unpack_bf16x8(f3[g], a3);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float da = __uint_as_float(r[8 * g + i]);
                a1[i] *= da;
                a3[i] *= da;
              }
              f1[g] = pack_bf16x8(a1);
              f3[g] = pack_bf16x8(a3);
            }
            io.store_bf16(f1, q.f1, q.ldf, m0, q.M, col, q.N);
            io.store_bf16(f3, q.f3, q.ldf, m0, q.M, col, q.N);
          } else {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
            if (EPI == kEpiResidual) {
              uint4 rr[4];
              io.load_bf16(rr, q.res + q.res_col0, q.ldr, m0, q.M, col, q.N);
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                float t[8];
                unpack_bf16x8(rr[g], t);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[8 * g + i] -= t[i];
              }
            }
            uint4 o[4];
#pragma unroll
            for (int g = 0; g < 4; ++g) o[g] = pack_bf16x8(v + 8 * g);
            io.store_bf16(o, reinterpret_cast<__nv_bfloat16*>(q.out) + q.out_col0, q.ldo, m0, q.M, col, q.N);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader + buf * 8);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no signal to the peer is still on its way, and no MMA writes TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, 512);
  }
}

}  // namespace ttt
