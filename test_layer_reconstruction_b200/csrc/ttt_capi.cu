// ttt_capi.cu — the C ABI declared in include/ttt.h: host-side validation,
// workspace layout, TMA descriptors and the launch sequence of the layer
//   conv -> steps x [pack theta -> forward (residual) -> backward (partials)
//   -> reduce + SGD] -> pack theta* -> forward (read)
// for head widths 16, 32, 64 (h <= 256), and the wide-head sequence (token
// chunks of the tensor-core GEMM of gemm.cuh with fused epilogues, and the
// small kernels of wide.cuh) for head widths and hidden widths that are
// multiples of 64 beyond that.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/ttt.h"
#include "conv.cuh"
#include "gemm.cuh"
#include "update.cuh"
#include "wide.cuh"

using namespace ttt;

namespace {

constexpr size_t kAlign = 1024;
size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

struct Shape {
  long long n;   // tokens
  int H, D, h, hidp, tiles, slices, units;
  long long C;   // H * D channels
  bool wide;     // wide-head path (tensor-core GEMMs over token chunks)
};

constexpr long long kWideChunk = 262144;   // tokens per GEMM chunk of the wide path
constexpr int kWideMaxSplits = 8;          // most K splits of the weight-gradient GEMMs

int check_dims(const ttt_dims* dm, Shape* s) {
  if (!dm) return TTT_EINVAL;
  if (dm->n_views < 1 || dm->grid_h < 1 || dm->grid_w < 1 || dm->n_special < 0 || dm->heads < 1 || dm->d < 1 ||
      dm->h < 1)
    return TTT_EINVAL;
  const bool fused = (dm->d == 16 || dm->d == 32 || dm->d == 64) && dm->h <= 256;
  const bool wide = dm->d % 64 == 0 && dm->h % 64 == 0 && dm->d <= 8192 && dm->h <= 32768;
  if (!fused && !wide) return TTT_EUNSUPPORTED;
  s->wide = !fused;
  const long long T = static_cast<long long>(dm->n_special) + static_cast<long long>(dm->grid_h) * dm->grid_w;
  const long long n = T * dm->n_views;
  if (n <= 0 || n > (1LL << 31) - 1 - 128) return TTT_EUNSUPPORTED;   // TMA coordinates are int32
  if (dm->n_views > 65535 || dm->grid_h > 65534) return TTT_EUNSUPPORTED;  // conv grid limits
  s->n = n;
  s->H = dm->heads;
  s->D = dm->d;
  s->h = dm->h;
  s->hidp = (dm->h + 127) / 128 * 128;
  s->slices = s->hidp / 128;
  s->tiles = static_cast<int>((n + kTileM - 1) / kTileM);
  s->units = static_cast<int>((n + kUnit - 1) / kUnit);
  s->C = static_cast<long long>(dm->heads) * dm->d;
  return TTT_OK;
}

int num_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

struct Grids {
  int fwd, bwd, bwd_groups, max_contrib;
};

// Forward: one CTA per SM over (head, 128-token tile) items.  Backward: groups
// of `slices` CTAs over (head, 48-token unit) items, one hidden slice per CTA
// of a group.
Grids grids_for(const Shape& s, int sms) {
  Grids g;
  const long long items = static_cast<long long>(s.H) * s.tiles;
  g.fwd = static_cast<int>(std::min<long long>(sms, items));
  const long long units = static_cast<long long>(s.H) * s.units;
  g.bwd_groups = static_cast<int>(std::max<long long>(1, std::min<long long>(sms / s.slices, units)));
  g.bwd = g.bwd_groups * s.slices;
  int mc = 1;
  for (long long head = 0; head < s.H; ++head) {
    const long long lo = owner_cta(head * s.units, units, g.bwd_groups);
    const long long hi = owner_cta(head * s.units + s.units - 1, units, g.bwd_groups);
    mc = std::max<int>(mc, static_cast<int>(hi - lo + 1));
  }
  g.max_contrib = mc;
  return g;
}

struct Ws {
  size_t status, w13, w2h, wt, vp, e, part, grad, q, k, v, o, convw, th0, thout, total;
  size_t img, img2, acc, z1, z3, ab, eb;   // wide path
  size_t nsx, nsy, nsg, nsxh, nsxl, nsgh, nsgl, nsp;   // wide path: Newton-Schulz scratch
};

Ws ws_layout(const Shape& s, const Grids& g, int op) {
  Ws w;
  memset(&w, 0, sizeof(w));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t r = off;
    off = align_up(off + bytes);
    return r;
  };
  const size_t tok_bytes = static_cast<size_t>(s.n) * s.C * 2;
  const size_t theta_bytes = 3ull * s.H * s.D * s.h * 4;
  w.status = take(256);
  if (s.wide) {
    const bool writes = op == TTT_OP_WRITE || op == TTT_OP_LAYER || op == TTT_OP_LAYER_HOST;
    const size_t nc = static_cast<size_t>(std::min<long long>(s.n, kWideChunk));
    w.img = take(static_cast<size_t>(s.H) * s.D * 2 * s.hidp * 2);   // per head [d][2 hidp]: W1 | W3 by 128
    w.img2 = take(static_cast<size_t>(s.H) * s.h * s.D * 2);         // per head [h][d]: W2
    w.ab = take(nc * s.hidp * 2);                                     // A = silu(Z1) Z3
    if (writes) {
      w.z1 = take(nc * s.hidp * 2);                                   // F1, then dZ1
      w.z3 = take(nc * s.hidp * 2);                                   // F3, then dZ3
      w.eb = take(nc * s.D * 2);                                      // E = Y - V'
      w.acc = take(static_cast<size_t>(kWideMaxSplits) * 3 * s.D * s.h * 4);
      w.vp = take(tok_bytes);
      // Muon steps: the gradient, then Newton-Schulz on one d x h matrix at a time
      const size_t dh = static_cast<size_t>(s.D) * s.h, dd = static_cast<size_t>(s.D) * s.D;
      w.grad = take(theta_bytes);
      w.nsx = take(dh * 4);
      w.nsy = take(dh * 4);
      w.nsg = take(dd * 4);
      w.nsxh = take(dh * 2);
      w.nsxl = take(dh * 2);
      w.nsgh = take(dd * 2);
      w.nsgl = take(dd * 2);
      w.nsp = take(kNsParts * 4);
    }
    if (op == TTT_OP_LAYER_HOST) {
      w.q = take(tok_bytes);
      w.k = take(tok_bytes);
      w.v = take(tok_bytes);
      w.o = take(tok_bytes);
      w.convw = take(static_cast<size_t>(s.C) * 9 * 4);
      w.th0 = take(theta_bytes);
      w.thout = take(theta_bytes);
    }
    w.total = off;
    return w;
  }
  w.w13 = take(static_cast<size_t>(s.H) * 2 * s.hidp * s.D * 2);
  w.w2h = take(static_cast<size_t>(s.H) * s.hidp * s.D * 2);
  if (op == TTT_OP_WRITE || op == TTT_OP_LAYER || op == TTT_OP_LAYER_HOST || op == TTT_OP_ATTENTION) {
    w.wt = take(static_cast<size_t>(s.H) * s.hidp * 3 * s.D * 2);
    w.vp = take(tok_bytes);
    w.e = take(tok_bytes);
    w.part = take(static_cast<size_t>(s.H) * s.slices * g.max_contrib * 3ull * 128 * s.D * 4);
    w.grad = take(theta_bytes);   // the gradient of a Muon step
  }
  if (op == TTT_OP_LAYER_HOST) {
    w.q = take(tok_bytes);
    w.k = take(tok_bytes);
    w.v = take(tok_bytes);
    w.o = take(tok_bytes);
    w.convw = take(static_cast<size_t>(s.C) * 9 * 4);
    w.th0 = take(theta_bytes);
    w.thout = take(theta_bytes);
  }
  if (op == TTT_OP_ATTENTION) {   // q, k, v of the projection and the layer's read O
    w.q = take(tok_bytes);
    w.k = take(tok_bytes);
    w.v = take(tok_bytes);
    w.o = take(tok_bytes);
  }
  w.total = off;
  return w;
}

// ------------------------------------------------------------------ TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D view [n rows][C bf16] of a token tensor; box = D columns x `rows` rows,
// swizzled by rows of 2*D bytes (the layout the kernels' descriptors expect).
bool make_token_map(CUtensorMap* m, const void* base, const Shape& s, int rows = kTileM) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(s.C), static_cast<cuuint64_t>(s.n)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(s.C) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(s.D), static_cast<cuuint32_t>(rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = s.D == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                          : (s.D == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ profiling
enum KernelKind {
  KK_CONV = 0, KK_PACK = 1, KK_FWD_WRITE = 2, KK_BWD = 3, KK_REDUCE = 4, KK_FWD_READ = 5,
  KK_GEMM_GATE = 6, KK_GEMM_RESIDUAL = 7, KK_GEMM_DZ = 8, KK_GEMM_WGRAD = 9, KK_GEMM_STORE = 10, KK_GEMM_QKV = 11
};
const char* const kKernelNames[TTT_KERNEL_KINDS] = {
    "shortconv2d", "pack_theta", "swiglu_fwd_residual", "swiglu_bwd_partials", "reduce_sgd", "swiglu_fwd_read",
    "gemm_gate", "gemm_residual", "gemm_dz", "gemm_wgrad", "gemm_store", "gemm_qkv_l2norm"};
constexpr size_t kMaxProfiled = 65536;

struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> ev;   // 2 per launch
  std::vector<int> kind;
  size_t used = 0;
  int dropped = 0;
};
Profiler& profiler() {
  static Profiler p;
  return p;
}

// Records an event pair around one launch when profiling is on.
struct ProfScope {
  cudaEvent_t end = nullptr;
  cudaStream_t st;
  ProfScope(int k, cudaStream_t s) : st(s) {
    Profiler& p = profiler();
    std::lock_guard<std::mutex> lock(p.mu);
    if (!p.on) return;
    if (p.used >= kMaxProfiled) {
      ++p.dropped;
      return;
    }
    while (p.ev.size() < 2 * (p.used + 1)) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return;
      p.ev.push_back(e);
    }
    if (p.kind.size() < p.used + 1) p.kind.resize(p.used + 1);
    p.kind[p.used] = k;
    cudaEventRecord(p.ev[2 * p.used], st);
    end = p.ev[2 * p.used + 1];
    ++p.used;
  }
  ~ProfScope() {
    if (end) cudaEventRecord(end, st);
  }
};

// Limit (SM clocks) of every bounded wait in the kernels launched from now
// on; 0 selects the built-in limit.  Set by ttt_set_wait_limit.
std::atomic<long long>& wait_clock_setting() {
  static std::atomic<long long> v{0};
  return v;
}
long long wait_clocks() { return wait_clock_setting().load(std::memory_order_relaxed); }

bool aligned(const void* p, size_t a = 16) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int launch_status() { return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ECUDA; }

// ------------------------------------------------------------------ launches
// V' = ShortConv2D(V), stored as bf16, or as f16 with `f16out` (the
// backward kernel's operand type, for the dot-product-loss path).
int run_conv(const Shape& s, const ttt_dims* dm, const uint16_t* V, const float* w, uint16_t* out,
             cudaStream_t st, bool f16out = false) {
  ConvParams p;
  p.V = reinterpret_cast<const uint2*>(V);
  p.w = w;
  p.out = reinterpret_cast<uint2*>(out);
  p.n_views = dm->n_views;
  p.gh = dm->grid_h;
  p.gw = dm->grid_w;
  p.n_special = dm->n_special;
  p.C = static_cast<int>(s.C);
  const int g4 = p.C / 4;
  const int block = std::min(kConvThreads, (g4 + 31) / 32 * 32);
  const long long items = static_cast<long long>(dm->n_views) * ((dm->grid_h + kConvBand - 1) / kConvBand + 1);
  const int sms = num_sms();
  const long long persistent = static_cast<long long>(sms > 0 ? sms : 148) * 2;
  dim3 grid(static_cast<unsigned>(std::min(items, persistent)), (g4 + block - 1) / block, 1);
  const size_t smem = conv_smem_bytes(block);
  auto k = f16out ? shortconv_kernel<kConvBand, true> : shortconv_kernel<kConvBand, false>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return TTT_ECUDA;
  ProfScope prof(KK_CONV, st);
  k<<<grid, block, smem, st>>>(p);
  return launch_status();
}

// Operand images of theta; the backward kernel's weight rows only when `with_wt`.
int run_pack(const Shape& s, const float* theta, const Ws& w, uint8_t* ws, bool with_wt, cudaStream_t st) {
  PackParams p;
  p.theta = theta;
  p.w13_img = reinterpret_cast<__nv_bfloat16*>(ws + w.w13);
  p.w2h_img = reinterpret_cast<__half*>(ws + w.w2h);
  p.wt_img = with_wt ? reinterpret_cast<__half*>(ws + w.wt) : nullptr;
  p.heads = s.H;
  p.d = s.D;
  p.h = s.h;
  p.hidp = s.hidp;
  const long long total = static_cast<long long>(s.H) * (with_wt ? 6 : 3) * s.hidp * s.D;
  ProfScope prof(KK_PACK, st);
  pack_images_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(p);
  return launch_status();
}

// The tensor-core kernels allocate all 512 TMEM columns of their SM; asking
// for more than half of the SM's shared memory keeps their residency at one
// CTA per SM, so an allocation never waits for a co-resident CTA.
constexpr uint32_t kHalfSmem = 116u * 1024u;
uint32_t one_cta_per_sm(uint32_t bytes) { return bytes > kHalfSmem ? bytes : kHalfSmem; }

template <int D, int HIDP, bool WRITE>
int launch_fwd_t(const CUtensorMap& tx, const CUtensorMap& tvp, const FwdParams& p, int grid, cudaStream_t st) {
  using L = FwdLayout<D, HIDP>;
  auto k = fwd_kernel<D, HIDP, WRITE>;
  const uint32_t smem = one_cta_per_sm(L::bytes);
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TTT_ECUDA;
  ProfScope prof(WRITE ? KK_FWD_WRITE : KK_FWD_READ, st);
  k<<<grid, kThreads, smem, st>>>(tx, tvp, p);
  return launch_status();
}

template <bool WRITE>
int launch_fwd(const Shape& s, const CUtensorMap& tx, const CUtensorMap& tvp, const FwdParams& p, int grid,
               cudaStream_t st) {
#define TTT_FWD_CASE(DD, HH) \
  if (s.D == DD && s.hidp == HH) return launch_fwd_t<DD, HH, WRITE>(tx, tvp, p, grid, st);
  TTT_FWD_CASE(16, 128) TTT_FWD_CASE(16, 256) TTT_FWD_CASE(32, 128) TTT_FWD_CASE(32, 256)
  TTT_FWD_CASE(64, 128) TTT_FWD_CASE(64, 256)
#undef TTT_FWD_CASE
  return TTT_EUNSUPPORTED;
}

template <int D>
int launch_bwd_t(const CUtensorMap& tk, const CUtensorMap& te, const BwdParams& p, int grid, cudaStream_t st) {
  using L = BwdLayout<D>;
  auto k = bwd_kernel<D>;
  const uint32_t smem = one_cta_per_sm(L::bytes);
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TTT_ECUDA;
  ProfScope prof(KK_BWD, st);
  k<<<grid, kBwdThreads, smem, st>>>(tk, te, p);
  return launch_status();
}

int launch_bwd(const Shape& s, const CUtensorMap& tk, const CUtensorMap& te, const BwdParams& p, int grid,
               cudaStream_t st) {
  if (s.D == 16) return launch_bwd_t<16>(tk, te, p, grid, st);
  if (s.D == 32) return launch_bwd_t<32>(tk, te, p, grid, st);
  if (s.D == 64) return launch_bwd_t<64>(tk, te, p, grid, st);
  return TTT_EUNSUPPORTED;
}

struct Call {
  Shape s;
  Grids g;
  Ws w;
  uint8_t* ws;
  cudaStream_t st;
};

// Host-side validation first (no CUDA call), then the device-dependent sizes.
int prepare(const ttt_dims* dm, int op, void* workspace, size_t ws_bytes, void* stream, Call* c) {
  int rc = check_dims(dm, &c->s);
  if (rc != TTT_OK) return rc;
  if (!workspace) return TTT_EINVAL;
  if (!aligned(workspace, 256)) return TTT_EALIGN;
  const int sms = num_sms();
  if (sms <= 0) return TTT_ECUDA;
  c->g = grids_for(c->s, sms);
  c->w = ws_layout(c->s, c->g, op);
  if (ws_bytes < c->w.total) return TTT_EWORKSPACE;
  c->ws = static_cast<uint8_t*>(workspace);
  c->st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(c->ws + c->w.status, 0, 4, c->st) != cudaSuccess) return TTT_ECUDA;
  return TTT_OK;
}

// ------------------------------------------------------------------ tensor-core GEMM
// 2-D bf16 tensor [rows][cols] (row pitch `pitch` elements) for the GEMM's
// operand loads: K-major boxes are 64 columns x 128 rows, MN-major boxes 64
// columns x 64 rows, both with the 128-byte swizzle.
bool make_gemm_map(CUtensorMap* m, const void* base, long long rows, long long cols, long long pitch, bool mn) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows < 1 || cols < 1) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(pitch) * 2};
  cuuint32_t box[2] = {64u, mn ? 64u : 128u};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One launch of gemm_kernel: up to three problems with their operand maps.
struct GemmLaunch {
  GemmParams P;
  CUtensorMap ma[kGemmMaxProblems], mb[kGemmMaxProblems];
  GemmLaunch() {
    memset(&P, 0, sizeof(P));
    memset(ma, 0, sizeof(ma));
    memset(mb, 0, sizeof(mb));
  }
  // A problem of M x N with reduction length K; `splits` > 1 only for kEpiAccF32.
  GemmProblem& add(int M, int N, int K, bool a_mn, bool b_mn, int splits = 1) {
    GemmProblem& q = P.prob[P.n_problems++];
    q.M = M;
    q.N = N;
    q.K = K;
    q.a_mn = a_mn;
    q.b_mn = b_mn;
    const int kblocks = (K + kGemmBK - 1) / kGemmBK;
    splits = std::max(1, std::min(splits, kblocks));
    q.k_per_split = (kblocks + splits - 1) / splits * kGemmBK;
    q.splits = (K + q.k_per_split - 1) / q.k_per_split;
    q.tiles_m = (M + kGemmBM - 1) / kGemmBM;
    q.tiles_n = (N + kGemmBN - 1) / kGemmBN;
    q.items = static_cast<long long>(q.tiles_m) * q.tiles_n * q.splits;
    return q;
  }
};

template <int EPI>
int launch_gemm(GemmLaunch& g, unsigned int* status, int kind, cudaStream_t st) {
  g.P.status = status;
  g.P.wait_clocks = wait_clocks();
  g.P.total_items = 0;
  for (int p = 0; p < g.P.n_problems; ++p) g.P.total_items += g.P.prob[p].items;
  if (g.P.total_items == 0) return TTT_OK;
  for (int p = g.P.n_problems; p < kGemmMaxProblems; ++p) {
    g.ma[p] = g.ma[0];
    g.mb[p] = g.mb[0];
  }
  // one CTA pair (a cluster of two) per two SMs
  const int sms = num_sms();
  const long long pairs = std::min<long long>((sms > 1 ? sms : 148) / 2, g.P.total_items);
  auto k = gemm_kernel<EPI>;
  const uint32_t smem = GemmLayout::bytes;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return TTT_ECUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ProfScope prof(kind, st);
  if (cudaLaunchKernelEx(&cfg, k, g.ma[0], g.mb[0], g.ma[1], g.mb[1], g.ma[2], g.mb[2], g.P) != cudaSuccess)
    return TTT_ECUDA;
  return launch_status();
}

// K splits of the weight-gradient launch: enough items for about three waves
// of one CTA pair per two SMs.
int wgrad_splits(const Shape& s, long long nc) {
  const int sms = std::max(2, num_sms()) / 2;
  const long long tiles = 2LL * ((s.D + kGemmBM - 1) / kGemmBM) * ((s.h + kGemmBN - 1) / kGemmBN) +
                          static_cast<long long>((s.h + kGemmBM - 1) / kGemmBM) * ((s.D + kGemmBN - 1) / kGemmBN);
  const long long want = (3LL * sms + tiles - 1) / tiles;
  const long long kblocks = (nc + kGemmBK - 1) / kGemmBK;
  return static_cast<int>(std::max<long long>(1, std::min<long long>({want, kWideMaxSplits, kblocks})));
}

// ------------------------------------------------------------------ the layer's surround
// q = L2(X Wq), k = L2(X Wk) per (token, head) row of 64, v = X Wv: one launch
// of three problems sharing the A operand X.
int run_qkv(const Call& c, const uint16_t* X, const uint16_t* Wq, const uint16_t* Wk, const uint16_t* Wv,
            uint16_t* q, uint16_t* k, uint16_t* v) {
  const Shape& s = c.s;
  GemmLaunch g;
  const uint16_t* W[3] = {Wq, Wk, Wv};
  uint16_t* out[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    if (!make_gemm_map(&g.ma[i], X, s.n, s.C, s.C, false) || !make_gemm_map(&g.mb[i], W[i], s.C, s.C, s.C, true))
      return TTT_ECUDA;
    GemmProblem& p = g.add(static_cast<int>(s.n), static_cast<int>(s.C), static_cast<int>(s.C), false, true);
    p.out = out[i];
    p.ldo = s.C;
    p.norm_cols = i < 2 ? static_cast<int>(s.C) : 0;
  }
  return launch_gemm<kEpiL2Heads>(g, reinterpret_cast<unsigned int*>(c.ws + c.w.status), KK_GEMM_QKV, c.st);
}

// out = O Wo.
int run_out_proj(const Call& c, const uint16_t* O, const uint16_t* Wo, uint16_t* out) {
  const Shape& s = c.s;
  GemmLaunch g;
  if (!make_gemm_map(&g.ma[0], O, s.n, s.C, s.C, false) || !make_gemm_map(&g.mb[0], Wo, s.C, s.C, s.C, true))
    return TTT_ECUDA;
  GemmProblem& p = g.add(static_cast<int>(s.n), static_cast<int>(s.C), static_cast<int>(s.C), false, true);
  p.out = out;
  p.ldo = s.C;
  return launch_gemm<kEpiStore>(g, reinterpret_cast<unsigned int*>(c.ws + c.w.status), KK_GEMM_STORE, c.st);
}

// ------------------------------------------------------------------ wide path
unsigned elementwise_grid(long long n) {
  const int sms = num_sms();
  return static_cast<unsigned>(std::max<long long>(1, std::min<long long>((n + 255) / 256, 8LL * (sms > 0 ? sms : 148))));
}

// Operand images of theta for the wide path: per head W13 [d][2 hidp] (hidden
// block j of 128 units: W1 columns, then W3 columns) and W2 [h][d], bf16.
int wide_pack(const Call& c, const float* theta) {
  const Shape& s = c.s;
  const long long count = static_cast<long long>(s.H) * s.D * (2LL * s.hidp + s.h);
  ProfScope prof(KK_PACK, c.st);
  wide_pack_kernel<<<elementwise_grid(count), 256, 0, c.st>>>(
      theta, reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.img), reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.img2),
      s.H, s.D, s.h, s.hidp);
  return launch_status();
}

struct WideOperands {
  const __nv_bfloat16* img13;   // this head's W13 image
  const __nv_bfloat16* img2;    // this head's W2 image
};
WideOperands wide_head(const Call& c, int head) {
  const Shape& s = c.s;
  WideOperands o;
  o.img13 = reinterpret_cast<const __nv_bfloat16*>(c.ws + c.w.img) + static_cast<size_t>(head) * s.D * 2 * s.hidp;
  o.img2 = reinterpret_cast<const __nv_bfloat16*>(c.ws + c.w.img2) + static_cast<size_t>(head) * s.h * s.D;
  return o;
}

// Gate of rows [t0, t0 + nc) of head `head` of X: A = silu(X W1) (X W3), and
// with `chain` also F1, F3 (the backward's chain-rule factors).
int wide_gate_chunk(const Call& c, const uint16_t* X, int head, long long t0, int nc, bool chain) {
  const Shape& s = c.s;
  const WideOperands w = wide_head(c, head);
  GemmLaunch g;
  if (!make_gemm_map(&g.ma[0], X + static_cast<size_t>(t0) * s.C, nc, s.C, s.C, false) ||
      !make_gemm_map(&g.mb[0], w.img13, s.D, 2LL * s.hidp, 2LL * s.hidp, true))
    return TTT_ECUDA;
  GemmProblem& q = g.add(nc, 2 * s.hidp, s.D, false, true);
  q.a_x0 = head * s.D;
  q.out = c.ws + c.w.ab;
  q.ldf = s.hidp;
  q.f1 = chain ? reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.z1) : nullptr;
  q.f3 = chain ? reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.z3) : nullptr;
  return launch_gemm<kEpiGate>(g, reinterpret_cast<unsigned int*>(c.ws + c.w.status), KK_GEMM_GATE, c.st);
}

// dW of one head of the wide path over all tokens, per token chunk:
//   A, F1, F3 (gate GEMM) -> E = A W2 - V' -> dA = E W2^T, dZ1 = dA F1, dZ3 = dA F3
//   -> dW1 += K^T dZ1, dW3 += K^T dZ3, dW2 += A^T E   (FP32 split-K partials, Eq. 5)
// into the workspace accumulator [splits][dW1 | dW3 | dW2]; returns the split count.
// With `dot` (the dot-product loss, whose output gradient is the constant
// -V'/n) the residual GEMM is skipped and V' itself stands where E stands;
// the caller negates.
int wide_grad_head(const Call& c, const uint16_t* K, const uint16_t* vp, int head, int* splits_out, bool dot = false) {
  const Shape& s = c.s;
  const WideOperands w = wide_head(c, head);
  unsigned int* status = reinterpret_cast<unsigned int*>(c.ws + c.w.status);
  float* acc = reinterpret_cast<float*>(c.ws + c.w.acc);
  __nv_bfloat16* ab = reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.ab);
  __nv_bfloat16* f1 = reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.z1);
  __nv_bfloat16* f3 = reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.z3);
  __nv_bfloat16* eb = reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.eb);
  const long long per = static_cast<long long>(s.D) * s.h;
  int rc, splits = 1;
  for (long long t0 = 0; t0 < s.n; t0 += kWideChunk) {
    const int nc = static_cast<int>(std::min<long long>(kWideChunk, s.n - t0));
    if ((rc = wide_gate_chunk(c, K, head, t0, nc, true)) != TTT_OK) return rc;
    // E: [nc][d] in the chunk buffer (pitch d), or V' in place (pitch C, the head's columns)
    const __nv_bfloat16* e_src = dot ? reinterpret_cast<const __nv_bfloat16*>(vp) + static_cast<size_t>(t0) * s.C : eb;
    const long long e_pitch = dot ? s.C : s.D, e_cols = dot ? s.C : s.D;
    const int e_x0 = dot ? head * s.D : 0;
    if (!dot) {  // E = A W2 - V'
      GemmLaunch g;
      if (!make_gemm_map(&g.ma[0], ab, nc, s.hidp, s.hidp, false) ||
          !make_gemm_map(&g.mb[0], w.img2, s.h, s.D, s.D, true))
        return TTT_ECUDA;
      GemmProblem& q = g.add(nc, s.D, s.h, false, true);
      q.out = eb;
      q.ldo = s.D;
      q.res = reinterpret_cast<const __nv_bfloat16*>(vp) + static_cast<size_t>(t0) * s.C;
      q.ldr = s.C;
      q.res_col0 = head * s.D;
      if ((rc = launch_gemm<kEpiResidual>(g, status, KK_GEMM_RESIDUAL, c.st)) != TTT_OK) return rc;
    }
    {  // dA = E W2^T, then dZ1 = dA F1, dZ3 = dA F3 in place
      GemmLaunch g;
      if (!make_gemm_map(&g.ma[0], e_src, nc, e_cols, e_pitch, false) ||
          !make_gemm_map(&g.mb[0], w.img2, s.h, s.D, s.D, false))
        return TTT_ECUDA;
      GemmProblem& q = g.add(nc, s.hidp, s.D, false, false);
      q.a_x0 = e_x0;
      q.f1 = f1;
      q.f3 = f3;
      q.ldf = s.hidp;
      if ((rc = launch_gemm<kEpiDz>(g, status, KK_GEMM_DZ, c.st)) != TTT_OK) return rc;
    }
    {  // dW1 = K^T dZ1, dW3 = K^T dZ3, dW2 = A^T E, split over the chunk's tokens
      GemmLaunch g;
      const uint16_t* kc = K + static_cast<size_t>(t0) * s.C;
      if (!make_gemm_map(&g.ma[0], kc, nc, s.C, s.C, true) || !make_gemm_map(&g.mb[0], f1, nc, s.hidp, s.hidp, true) ||
          !make_gemm_map(&g.ma[1], kc, nc, s.C, s.C, true) || !make_gemm_map(&g.mb[1], f3, nc, s.hidp, s.hidp, true) ||
          !make_gemm_map(&g.ma[2], ab, nc, s.hidp, s.hidp, true) ||
          !make_gemm_map(&g.mb[2], e_src, nc, e_cols, e_pitch, true))
        return TTT_ECUDA;
      // The first chunk is the largest and fixes the split count: every later
      // chunk adds its split s into partial s (it may have fewer splits,
      // whose partials then gain nothing), and the update sums the first
      // chunk's splits in order.
      const int sp = t0 == 0 ? wgrad_splits(s, nc) : splits;
      const int acc_flag = t0 > 0 ? 1 : 0;
      GemmProblem* qs[3] = {&g.add(s.D, s.h, nc, true, true, sp), &g.add(s.D, s.h, nc, true, true, sp),
                            &g.add(s.h, s.D, nc, true, true, sp)};
      if (t0 == 0) splits = qs[0]->splits;
      for (int m = 0; m < 3; ++m) {
        GemmProblem& q = *qs[m];
        q.a_x0 = m < 2 ? head * s.D : 0;
        if (m == 2) q.b_x0 = e_x0;
        q.out = acc + m * per;
        q.ldo = m < 2 ? s.h : s.D;
        q.split_stride = 3 * per;
        q.accumulate = acc_flag;
      }
      if ((rc = launch_gemm<kEpiAccF32>(g, status, KK_GEMM_WGRAD, c.st)) != TTT_OK) return rc;
    }
  }
  *splits_out = splits;
  return TTT_OK;
}

// The write of the wide path: per step and head, dW over all token chunks,
// then theta_out = theta_in - lr (2/n) dW for the head.
int run_write_wide(const Call& c, const ttt_dims* dm, const uint16_t* K, const uint16_t* V, const float* conv_w,
                   const float* theta0, float lr, int steps, float* theta_out) {
  const Shape& s = c.s;
  uint16_t* vp = reinterpret_cast<uint16_t*>(c.ws + c.w.vp);
  int rc = run_conv(s, dm, V, conv_w, vp, c.st);
  if (rc != TTT_OK) return rc;
  if (steps == 0) {
    if (theta_out != theta0 &&
        cudaMemcpyAsync(theta_out, theta0, 3ull * s.H * s.D * s.h * 4, cudaMemcpyDeviceToDevice, c.st) != cudaSuccess)
      return TTT_ECUDA;
    return TTT_OK;
  }
  const long long per = static_cast<long long>(s.D) * s.h;
  const float* acc = reinterpret_cast<const float*>(c.ws + c.w.acc);
  const float scale = lr * 2.0f / static_cast<float>(s.n);
  for (int step = 0; step < steps; ++step) {
    const float* th_in = step == 0 ? theta0 : theta_out;
    if ((rc = wide_pack(c, th_in)) != TTT_OK) return rc;
    for (int head = 0; head < s.H; ++head) {
      int splits = 1;
      if ((rc = wide_grad_head(c, K, vp, head, &splits)) != TTT_OK) return rc;
      ProfScope prof(KK_REDUCE, c.st);
      wide_sgd_kernel<<<elementwise_grid(3 * per), 256, 0, c.st>>>(th_in, theta_out, acc, splits, s.H, s.D, s.h,
                                                                    head, scale);
      if ((rc = launch_status()) != TTT_OK) return rc;
    }
  }
  return TTT_OK;
}

// The gradient (1/2) d/dtheta sum_i ||T(k_i) - v'_i||^2 of the wide path, or
// with `dot` that of -sum_i <T(k_i), v'_i>.
int run_grad_wide(const Call& c, const uint16_t* K, const uint16_t* vp, const float* theta, float* grad,
                  bool dot = false) {
  const Shape& s = c.s;
  const long long per = static_cast<long long>(s.D) * s.h;
  const float* acc = reinterpret_cast<const float*>(c.ws + c.w.acc);
  int rc = wide_pack(c, theta);
  if (rc != TTT_OK) return rc;
  for (int head = 0; head < s.H; ++head) {
    int splits = 1;
    if ((rc = wide_grad_head(c, K, vp, head, &splits, dot)) != TTT_OK) return rc;
    ProfScope prof(KK_REDUCE, c.st);
    wide_grad_kernel<<<elementwise_grid(3 * per), 256, 0, c.st>>>(grad, acc, splits, s.H, s.D, s.h, head,
                                                                   dot ? -1.f : 1.f);
    if ((rc = launch_status()) != TTT_OK) return rc;
  }
  return TTT_OK;
}

// out (f32 [M][N], row pitch ldo) = or += A B on the tensor-core GEMM, A and B
// bf16 in the given layouts (A: [M][K] K-major or [K][M]; B: [N][K] K-major
// or [K][N]).
int gemm_f32(const Call& c, const __nv_bfloat16* A, bool a_mn, const __nv_bfloat16* B, bool b_mn, int M, int N, int K,
             float* out, long long ldo, bool accumulate) {
  GemmLaunch g;
  if (!make_gemm_map(&g.ma[0], A, a_mn ? K : M, a_mn ? M : K, a_mn ? M : K, a_mn) ||
      !make_gemm_map(&g.mb[0], B, b_mn ? K : N, b_mn ? N : K, b_mn ? N : K, b_mn))
    return TTT_ECUDA;
  GemmProblem& q = g.add(M, N, K, a_mn, b_mn);
  q.out = out;
  q.ldo = ldo;
  q.accumulate = accumulate ? 1 : 0;
  return launch_gemm<kEpiAccF32>(g, reinterpret_cast<unsigned int*>(c.ws + c.w.status), KK_REDUCE, c.st);
}

// theta_out = theta_in - lr NS5(sum of n_grads gradients) on the wide path,
// per head and matrix (reading 10; products split into bf16 pairs, wide.cuh).
int run_muon_update_wide(const Call& c, const float* theta_in, const float* grads, int n_grads, float lr,
                         float* theta_out) {
  const Shape& s = c.s;
  const int d = s.D, h = s.h;
  const long long dh = static_cast<long long>(d) * h, dd = static_cast<long long>(d) * d;
  float* X = reinterpret_cast<float*>(c.ws + c.w.nsx);
  float* Y = reinterpret_cast<float*>(c.ws + c.w.nsy);
  float* G = reinterpret_cast<float*>(c.ws + c.w.nsg);
  __nv_bfloat16* xh = reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.nsxh);
  __nv_bfloat16* xl = reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.nsxl);
  __nv_bfloat16* gh = reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.nsgh);
  __nv_bfloat16* gl = reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.nsgl);
  float* part = reinterpret_cast<float*>(c.ws + c.w.nsp);
  int rc;
  for (int head = 0; head < s.H; ++head) {
    for (int m = 0; m < 3; ++m) {
      {
        ProfScope prof(KK_REDUCE, c.st);
        ns_load_kernel<<<kNsParts, 256, 0, c.st>>>(grads, n_grads, s.H, d, h, head, m, X, part);
        ns_normalise_kernel<<<elementwise_grid(dh), 256, 0, c.st>>>(X, part, dh, xh, xl);
      }
      if ((rc = launch_status()) != TTT_OK) return rc;
      for (int it = 0; it < kNsIters; ++it) {
        // Gram = X X^T (B = X read K-major), split; Y = Gram X (B = X read MN-major)
        if ((rc = gemm_f32(c, xh, false, xh, false, d, d, h, G, d, false)) != TTT_OK ||
            (rc = gemm_f32(c, xh, false, xl, false, d, d, h, G, d, true)) != TTT_OK ||
            (rc = gemm_f32(c, xl, false, xh, false, d, d, h, G, d, true)) != TTT_OK)
          return rc;
        {
          ProfScope prof(KK_REDUCE, c.st);
          ns_split_kernel<<<elementwise_grid(dd), 256, 0, c.st>>>(G, dd, gh, gl);
        }
        if ((rc = launch_status()) != TTT_OK) return rc;
        if ((rc = gemm_f32(c, gh, false, xh, true, d, h, d, Y, h, false)) != TTT_OK ||
            (rc = gemm_f32(c, gh, false, xl, true, d, h, d, Y, h, true)) != TTT_OK ||
            (rc = gemm_f32(c, gl, false, xh, true, d, h, d, Y, h, true)) != TTT_OK)
          return rc;
        {
          ProfScope prof(KK_REDUCE, c.st);
          ns_combine_kernel<<<elementwise_grid(dh), 256, 0, c.st>>>(X, Y, dh, xh, xl);
        }
        if ((rc = launch_status()) != TTT_OK) return rc;
      }
      {
        ProfScope prof(KK_REDUCE, c.st);
        ns_apply_kernel<<<elementwise_grid(dh), 256, 0, c.st>>>(theta_in, theta_out, X, s.H, d, h, head, m, lr);
      }
      if ((rc = launch_status()) != TTT_OK) return rc;
    }
  }
  return TTT_OK;
}

// The read of the wide path: per head and token chunk, the gate GEMM (A),
// then O = A W2 written straight into the head's columns of O.
int run_read_wide(const Call& c, const uint16_t* Q, const float* theta, uint16_t* O) {
  const Shape& s = c.s;
  int rc = wide_pack(c, theta);
  if (rc != TTT_OK) return rc;
  unsigned int* status = reinterpret_cast<unsigned int*>(c.ws + c.w.status);
  for (int head = 0; head < s.H; ++head) {
    const WideOperands w = wide_head(c, head);
    for (long long t0 = 0; t0 < s.n; t0 += kWideChunk) {
      const int nc = static_cast<int>(std::min<long long>(kWideChunk, s.n - t0));
      if ((rc = wide_gate_chunk(c, Q, head, t0, nc, false)) != TTT_OK) return rc;
      GemmLaunch g;
      if (!make_gemm_map(&g.ma[0], c.ws + c.w.ab, nc, s.hidp, s.hidp, false) ||
          !make_gemm_map(&g.mb[0], w.img2, s.h, s.D, s.D, true))
        return TTT_ECUDA;
      GemmProblem& q = g.add(nc, s.D, s.h, false, true);
      q.out = O + static_cast<size_t>(t0) * s.C;
      q.ldo = s.C;
      q.out_col0 = head * s.D;
      if ((rc = launch_gemm<kEpiStore>(g, status, KK_GEMM_STORE, c.st)) != TTT_OK) return rc;
    }
  }
  return TTT_OK;
}

// One gradient pass of the fused path over (K, V'): operand images of theta,
// forward (E = T(K) - V'), backward partials, and the fixed-order reduction.
struct GradPass {
  CUtensorMap tk, tvp, tku, teu;
  FwdParams fp;
  BwdParams bp;
  UpdateParams up;
  long long red_threads;
};

// dot: the dot-product loss, whose output gradient is the constant -V'; the
// backward then reads V' where it reads E (no forward pass) and the reduction
// negates.
bool setup_grad_pass(const Call& c, const uint16_t* K, const uint16_t* vp, GradPass* gp, bool dot = false) {
  const Shape& s = c.s;
  uint16_t* e = dot ? const_cast<uint16_t*>(vp) : reinterpret_cast<uint16_t*>(c.ws + c.w.e);
  unsigned int* status = reinterpret_cast<unsigned int*>(c.ws + c.w.status);
  if (!make_token_map(&gp->tk, K, s) || !make_token_map(&gp->tvp, vp, s) || !make_token_map(&gp->tku, K, s, kUnit) ||
      !make_token_map(&gp->teu, e, s, kUnit))
    return false;
  FwdParams& fp = gp->fp;
  fp.w13_img = reinterpret_cast<const __nv_bfloat16*>(c.ws + c.w.w13);
  fp.w2_img = reinterpret_cast<const __half*>(c.ws + c.w.w2h);
  fp.out = reinterpret_cast<__nv_bfloat16*>(e);
  fp.n = static_cast<int>(s.n);
  fp.heads = s.H;
  fp.tiles = s.tiles;
  fp.status = status;
  fp.wait_clocks = wait_clocks();
  BwdParams& bp = gp->bp;
  bp.wt_img = reinterpret_cast<const uint32_t*>(c.ws + c.w.wt);
  bp.partials = reinterpret_cast<float*>(c.ws + c.w.part);
  bp.n = fp.n;
  bp.heads = s.H;
  bp.units = s.units;
  bp.slices = s.slices;
  bp.max_contrib = c.g.max_contrib;
  bp.status = status;
  bp.wait_clocks = wait_clocks();
  UpdateParams& up = gp->up;
  up.partials = bp.partials;
  up.heads = s.H;
  up.d = s.D;
  up.h = s.h;
  up.slices = s.slices;
  up.units = s.units;
  up.max_contrib = c.g.max_contrib;
  up.n_items = static_cast<long long>(s.H) * s.units;
  up.grid = c.g.bwd_groups;
  gp->red_threads = static_cast<long long>(s.H) * s.slices * 3 * 128 * s.D;
  return true;
}

// With theta_in: out = theta_in - scale * g (one SGD step).  Without: out = scale * g.
int run_grad_pass(const Call& c, GradPass& gp, const float* theta, const float* theta_in, float scale, float* out,
                  bool dot = false) {
  const Shape& s = c.s;
  int rc;
  if ((rc = run_pack(s, theta, c.w, c.ws, true, c.st)) != TTT_OK) return rc;
  if (!dot && (rc = launch_fwd<true>(s, gp.tk, gp.tvp, gp.fp, c.g.fwd, c.st)) != TTT_OK) return rc;
  if ((rc = launch_bwd(s, gp.tku, gp.teu, gp.bp, c.g.bwd, c.st)) != TTT_OK) return rc;
  gp.up.theta_in = theta_in;
  gp.up.theta_out = out;
  gp.up.scale = scale;
  {
    ProfScope prof(KK_REDUCE, c.st);
    reduce_sgd_kernel<<<static_cast<unsigned>((gp.red_threads + 255) / 256), 256, 0, c.st>>>(gp.up);
  }
  return launch_status();
}

int run_write(const Call& c, const ttt_dims* dm, const uint16_t* K, const uint16_t* V, const float* conv_w,
              const float* theta0, float lr, int steps, float* theta_out) {
  const Shape& s = c.s;
  if (s.wide) return run_write_wide(c, dm, K, V, conv_w, theta0, lr, steps, theta_out);
  uint16_t* vp = reinterpret_cast<uint16_t*>(c.ws + c.w.vp);
  int rc = run_conv(s, dm, V, conv_w, vp, c.st);
  if (rc != TTT_OK) return rc;
  if (steps == 0) {
    if (theta_out != theta0 &&
        cudaMemcpyAsync(theta_out, theta0, 3ull * s.H * s.D * s.h * 4, cudaMemcpyDeviceToDevice, c.st) != cudaSuccess)
      return TTT_ECUDA;
    return TTT_OK;
  }
  GradPass gp;
  if (!setup_grad_pass(c, K, vp, &gp)) return TTT_ECUDA;
  const float scale = lr * 2.0f / static_cast<float>(s.n);
  for (int step = 0; step < steps; ++step) {
    const float* th_in = step == 0 ? theta0 : theta_out;
    if ((rc = run_grad_pass(c, gp, th_in, th_in, scale, theta_out)) != TTT_OK) return rc;
  }
  return TTT_OK;
}

// theta_out = theta_in - lr * NS5(sum of n_grads gradients), per (head, matrix).
int run_muon_update(const Shape& s, const float* theta_in, const float* grads, int n_grads, float lr,
                    float* theta_out, cudaStream_t st) {
  MuonParams mp;
  mp.theta_in = theta_in;
  mp.grads = grads;
  mp.theta_out = theta_out;
  mp.n_grads = n_grads;
  mp.heads = s.H;
  mp.d = s.D;
  mp.h = s.h;
  mp.lr = lr;
  const size_t smem = ns_smem_bytes(s.D, s.h);
  if (cudaFuncSetAttribute(muon_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return TTT_ECUDA;
  {
    ProfScope prof(KK_REDUCE, st);
    muon_update_kernel<<<3 * s.H, kNsThreads, smem, st>>>(mp);
  }
  return launch_status();
}

// The pages' inner loop: `steps` Muon steps on the dot-product loss.  The
// gradient's output factor is the constant -V', which the backward kernel
// reads where it reads E, so V' is stored in f16, its operand type.
int run_write_muon(const Call& c, const ttt_dims* dm, const uint16_t* K, const uint16_t* V, const float* conv_w,
                   const float* theta0, float lr, int steps, float* theta_out) {
  const Shape& s = c.s;
  uint16_t* vp = reinterpret_cast<uint16_t*>(c.ws + c.w.vp);
  float* grad = reinterpret_cast<float*>(c.ws + c.w.grad);
  // the wide path's GEMMs read V' in bf16; the fused backward in f16
  int rc = run_conv(s, dm, V, conv_w, vp, c.st, !s.wide);
  if (rc != TTT_OK) return rc;
  if (steps == 0) {
    if (theta_out != theta0 &&
        cudaMemcpyAsync(theta_out, theta0, 3ull * s.H * s.D * s.h * 4, cudaMemcpyDeviceToDevice, c.st) != cudaSuccess)
      return TTT_ECUDA;
    return TTT_OK;
  }
  if (s.wide) {
    for (int step = 0; step < steps; ++step) {
      const float* th_in = step == 0 ? theta0 : theta_out;
      if ((rc = run_grad_wide(c, K, vp, th_in, grad, true)) != TTT_OK) return rc;
      if ((rc = run_muon_update_wide(c, th_in, grad, 1, lr, theta_out)) != TTT_OK) return rc;
    }
    return TTT_OK;
  }
  GradPass gp;
  if (!setup_grad_pass(c, K, vp, &gp, true)) return TTT_ECUDA;
  for (int step = 0; step < steps; ++step) {
    const float* th_in = step == 0 ? theta0 : theta_out;
    if ((rc = run_grad_pass(c, gp, th_in, nullptr, -1.f, grad, true)) != TTT_OK) return rc;
    if ((rc = run_muon_update(s, th_in, grad, 1, lr, theta_out, c.st)) != TTT_OK) return rc;
  }
  return TTT_OK;
}

// The gradient of (1/2) sum_i ||T(k_i) - v'_i||^2 over the call's tokens.
int run_grad(const Call& c, const uint16_t* K, const uint16_t* vp, const float* theta, float* grad) {
  if (c.s.wide) return run_grad_wide(c, K, vp, theta, grad);
  GradPass gp;
  if (!setup_grad_pass(c, K, vp, &gp)) return TTT_ECUDA;
  return run_grad_pass(c, gp, theta, nullptr, 1.f, grad);
}

// Read of the nt tokens at Q (fused path), with the operand images of theta
// already packed in the workspace.
int launch_read_tokens(const Call& c, const uint16_t* Q, uint16_t* O, long long nt) {
  Shape s = c.s;
  s.n = nt;
  s.tiles = static_cast<int>((nt + kTileM - 1) / kTileM);
  CUtensorMap tq;
  if (!make_token_map(&tq, Q, s)) return TTT_ECUDA;
  FwdParams fp;
  fp.w13_img = reinterpret_cast<const __nv_bfloat16*>(c.ws + c.w.w13);
  fp.w2_img = reinterpret_cast<const __half*>(c.ws + c.w.w2h);
  fp.out = reinterpret_cast<__nv_bfloat16*>(O);
  fp.n = static_cast<int>(s.n);
  fp.heads = s.H;
  fp.tiles = s.tiles;
  fp.status = reinterpret_cast<unsigned int*>(c.ws + c.w.status);
  fp.wait_clocks = wait_clocks();
  const int grid = static_cast<int>(std::min<long long>(c.g.fwd, static_cast<long long>(s.H) * s.tiles));
  return launch_fwd<false>(s, tq, tq, fp, grid, c.st);
}

int run_read(const Call& c, const uint16_t* Q, const float* theta, uint16_t* O) {
  const Shape& s = c.s;
  if (s.wide) return run_read_wide(c, Q, theta, O);
  int rc = run_pack(s, theta, c.w, c.ws, false, c.st);
  if (rc != TTT_OK) return rc;
  return launch_read_tokens(c, Q, O, s.n);
}

// ------------------------------------------------------------------ host pipeline
constexpr int kHostChunks = 8;           // most Q/O chunks of ttt_layer_host
constexpr int kHostChunkMinTiles = 64;   // fewest 128-token tiles per chunk

// Helper streams and events of one ttt_layer_host call, created per call and
// destroyed once its work is enqueued (CUDA releases them when that work has
// completed).
struct HostPipe {
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t ev[4 + 2 * kHostChunks] = {};
  int n_ev = 0;
  ~HostPipe() {
    for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);
    if (up) cudaStreamDestroy(up);
    if (down) cudaStreamDestroy(down);
  }
  bool init(int events) {
    if (cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking) != cudaSuccess)
      return false;
    for (; n_ev < events; ++n_ev)
      if (cudaEventCreateWithFlags(&ev[n_ev], cudaEventDisableTiming) != cudaSuccess) return false;
    return true;
  }
};

// ------------------------------------------------------------------ fixed scratch
// Scratch of ttt_read_noalloc.  In host code `g_noalloc_scratch` is only a
// host-side stand-in for the symbol; kernels receive the device address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[TTT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current); nullptr on failure.
uint8_t* noalloc_scratch() {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return static_cast<uint8_t*>(addr[dev]);
}

// Host-only shape check of the entry points that have no wide-head path.
int fused_only(const ttt_dims* dims) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != TTT_OK) return rc;
  return s.wide ? TTT_EUNSUPPORTED : TTT_OK;
}

}  // namespace

extern "C" {

#ifdef TTT_TRACE
// Trace builds only: copy out (and with reset != 0, clear) the per-warp phase clocks.
int ttt_trace_read(unsigned long long* out, int reset) {
  if (cudaDeviceSynchronize() != cudaSuccess) return TTT_ECUDA;
  if (cudaMemcpyFromSymbol(out, ttt::g_ttt_trace, sizeof(ttt::g_ttt_trace)) != cudaSuccess) return TTT_ECUDA;
  if (reset) {
    static unsigned long long zeros[ttt::kTraceKernels * ttt::kTraceWarps * ttt::kTraceSlots] = {};
    if (cudaMemcpyToSymbol(ttt::g_ttt_trace, zeros, sizeof(zeros)) != cudaSuccess) return TTT_ECUDA;
  }
  return TTT_OK;
}
#endif

int ttt_read_noalloc_status(void* stream) {
  uint8_t* scratch = noalloc_scratch();
  if (!scratch) return TTT_ECUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TTT_ECUDA;
  // The status word is the first field of every workspace layout (offset 0).
  unsigned int v = 0;
  if (cudaMemcpy(&v, scratch, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return TTT_ECUDA;
  if (v != 0) {
    if (cudaMemset(scratch, 0, sizeof(v)) != cudaSuccess) return TTT_ECUDA;
    return TTT_EDEVICE;
  }
  return TTT_OK;
}

int ttt_read_noalloc(const ttt_dims* dims, const uint16_t* Q, const float* theta, uint16_t* O, void* stream) {
  if (!Q || !theta || !O) return TTT_EINVAL;
  if (!aligned(Q) || !aligned(theta) || !aligned(O)) return TTT_EALIGN;
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != TTT_OK) return rc;
  const int sms = num_sms();
  if (sms <= 0) return TTT_ECUDA;
  if (ws_layout(s, grids_for(s, sms), TTT_OP_READ).total > TTT_NOALLOC_SCRATCH_BYTES) return TTT_EWORKSPACE;
  uint8_t* scratch = noalloc_scratch();
  if (!scratch) return TTT_ECUDA;
  Call c;
  rc = prepare(dims, TTT_OP_READ, scratch, TTT_NOALLOC_SCRATCH_BYTES, stream, &c);
  if (rc != TTT_OK) return rc;
  return run_read(c, Q, theta, O);
}

size_t ttt_workspace_bytes(const ttt_dims* dims, int op) {
  Shape s;
  if (check_dims(dims, &s) != TTT_OK) return 0;
  if (op < TTT_OP_WRITE || op > TTT_OP_ATTENTION) return 0;
  const int sms = num_sms();
  if (sms <= 0) return 0;
  return ws_layout(s, grids_for(s, sms), op).total;
}

int ttt_shortconv2d(const ttt_dims* dims, const uint16_t* V, const float* conv_w, uint16_t* V_out, void* stream) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != TTT_OK) return rc;
  if (!V || !conv_w || !V_out) return TTT_EINVAL;
  if (!aligned(V) || !aligned(conv_w) || !aligned(V_out)) return TTT_EALIGN;
  return run_conv(s, dims, V, conv_w, V_out, static_cast<cudaStream_t>(stream));
}

int ttt_write(const ttt_dims* dims, const uint16_t* K, const uint16_t* V, const float* conv_w, const float* theta0,
              float lr, int steps, float* theta_out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!K || !V || !conv_w || !theta0 || !theta_out || steps < 0) return TTT_EINVAL;
  if (!aligned(K) || !aligned(V) || !aligned(conv_w) || !aligned(theta0) || !aligned(theta_out)) return TTT_EALIGN;
  Call c;
  int rc = prepare(dims, TTT_OP_WRITE, workspace, workspace_bytes, stream, &c);
  if (rc != TTT_OK) return rc;
  return run_write(c, dims, K, V, conv_w, theta0, lr, steps, theta_out);
}

int ttt_grad(const ttt_dims* dims, const uint16_t* K, const uint16_t* Vp, const float* theta, float* grad,
             void* workspace, size_t workspace_bytes, void* stream) {
  if (!K || !Vp || !theta || !grad) return TTT_EINVAL;
  if (!aligned(K) || !aligned(Vp) || !aligned(theta) || !aligned(grad)) return TTT_EALIGN;
  Call c;
  int rc = prepare(dims, TTT_OP_WRITE, workspace, workspace_bytes, stream, &c);
  if (rc != TTT_OK) return rc;
  return run_grad(c, K, Vp, theta, grad);
}

int ttt_grad_dot(const ttt_dims* dims, const uint16_t* K, const uint16_t* Vp, const float* theta, float* grad,
                 void* workspace, size_t workspace_bytes, void* stream) {
  if (!K || !Vp || !theta || !grad) return TTT_EINVAL;
  if (!aligned(K) || !aligned(Vp) || !aligned(theta) || !aligned(grad)) return TTT_EALIGN;
  Call c;
  int rc = prepare(dims, TTT_OP_WRITE, workspace, workspace_bytes, stream, &c);
  if (rc != TTT_OK) return rc;
  if (c.s.wide) return run_grad_wide(c, K, Vp, theta, grad, true);
  // the backward kernel reads V' in f16, its operand type
  uint16_t* vp16 = reinterpret_cast<uint16_t*>(c.ws + c.w.e);
  const long long count = c.s.n * c.s.C;
  bf16_to_f16_kernel<<<elementwise_grid(count / 8), 256, 0, c.st>>>(reinterpret_cast<const uint4*>(Vp),
                                                                     reinterpret_cast<uint4*>(vp16), count / 8);
  if ((rc = launch_status()) != TTT_OK) return rc;
  GradPass gp;
  if (!setup_grad_pass(c, K, vp16, &gp, true)) return TTT_ECUDA;
  return run_grad_pass(c, gp, theta, nullptr, -1.f, grad, true);
}

int ttt_muon_update(const ttt_dims* dims, const float* theta_in, const float* grads, int n_grads, float lr,
                    float* theta_out, void* stream) {
  int rc = fused_only(dims);
  if (rc != TTT_OK) return rc;
  Shape s;
  check_dims(dims, &s);
  if (!theta_in || !grads || !theta_out || n_grads < 1) return TTT_EINVAL;
  if (!aligned(theta_in) || !aligned(grads) || !aligned(theta_out)) return TTT_EALIGN;
  return run_muon_update(s, theta_in, grads, n_grads, lr, theta_out, static_cast<cudaStream_t>(stream));
}

int ttt_write_muon(const ttt_dims* dims, const uint16_t* K, const uint16_t* V, const float* conv_w,
                   const float* theta0, float lr, int steps, float* theta_out, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (!K || !V || !conv_w || !theta0 || !theta_out || steps < 0) return TTT_EINVAL;
  if (!aligned(K) || !aligned(V) || !aligned(conv_w) || !aligned(theta0) || !aligned(theta_out)) return TTT_EALIGN;
  Call c;
  int rc = prepare(dims, TTT_OP_WRITE, workspace, workspace_bytes, stream, &c);
  if (rc != TTT_OK) return rc;
  return run_write_muon(c, dims, K, V, conv_w, theta0, lr, steps, theta_out);
}

int ttt_layer_muon(const ttt_dims* dims, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                   const float* conv_w, const float* theta0, float lr, int steps, float* theta_out, uint16_t* O,
                   void* workspace, size_t workspace_bytes, void* stream) {
  if (!Q || !K || !V || !conv_w || !theta0 || !theta_out || !O || steps < 0) return TTT_EINVAL;
  if (!aligned(Q) || !aligned(K) || !aligned(V) || !aligned(conv_w) || !aligned(theta0) || !aligned(theta_out) ||
      !aligned(O))
    return TTT_EALIGN;
  Call c;
  int rc = prepare(dims, TTT_OP_LAYER, workspace, workspace_bytes, stream, &c);
  if (rc != TTT_OK) return rc;
  if ((rc = run_write_muon(c, dims, K, V, conv_w, theta0, lr, steps, theta_out)) != TTT_OK) return rc;
  return run_read(c, Q, theta_out, O);
}

int ttt_sgd_update(const ttt_dims* dims, const float* theta_in, const float* grads, int n_grads, float scale,
                   float* theta_out, void* stream) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != TTT_OK) return rc;
  if (!theta_in || !grads || !theta_out || n_grads < 1) return TTT_EINVAL;
  if (!aligned(theta_in) || !aligned(grads) || !aligned(theta_out)) return TTT_EALIGN;
  const long long count = 3LL * s.H * s.D * s.h;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    ProfScope prof(KK_REDUCE, st);
    sgd_sum_kernel<<<elementwise_grid(count), 256, 0, st>>>(theta_in, grads, n_grads, count, scale, theta_out);
  }
  return launch_status();
}

int ttt_read(const ttt_dims* dims, const uint16_t* Q, const float* theta, uint16_t* O, void* workspace,
             size_t workspace_bytes, void* stream) {
  if (!Q || !theta || !O) return TTT_EINVAL;
  if (!aligned(Q) || !aligned(theta) || !aligned(O)) return TTT_EALIGN;
  Call c;
  int rc = prepare(dims, TTT_OP_READ, workspace, workspace_bytes, stream, &c);
  if (rc != TTT_OK) return rc;
  return run_read(c, Q, theta, O);
}

int ttt_layer(const ttt_dims* dims, const uint16_t* Q, const uint16_t* K, const uint16_t* V, const float* conv_w,
              const float* theta0, float lr, int steps, float* theta_out, uint16_t* O, void* workspace,
              size_t workspace_bytes, void* stream) {
  if (!Q || !K || !V || !conv_w || !theta0 || !theta_out || !O || steps < 0) return TTT_EINVAL;
  if (!aligned(Q) || !aligned(K) || !aligned(V) || !aligned(conv_w) || !aligned(theta0) || !aligned(theta_out) ||
      !aligned(O))
    return TTT_EALIGN;
  Call c;
  int rc = prepare(dims, TTT_OP_LAYER, workspace, workspace_bytes, stream, &c);
  if (rc != TTT_OK) return rc;
  if ((rc = run_write(c, dims, K, V, conv_w, theta0, lr, steps, theta_out)) != TTT_OK) return rc;
  return run_read(c, Q, theta_out, O);
}

int ttt_attention(const ttt_dims* dims, const uint16_t* X, const uint16_t* Wq, const uint16_t* Wk,
                  const uint16_t* Wv, const uint16_t* Wo, const float* conv_w, const float* theta0, float lr,
                  int steps, int inner, float* theta_out, uint16_t* out, void* workspace, size_t workspace_bytes,
                  void* stream) {
  if (!X || !Wq || !Wk || !Wv || !Wo || !conv_w || !theta0 || !theta_out || !out || steps < 0) return TTT_EINVAL;
  if (inner != TTT_INNER_SGD && inner != TTT_INNER_MUON) return TTT_EINVAL;
  if (!aligned(X) || !aligned(Wq) || !aligned(Wk) || !aligned(Wv) || !aligned(Wo) || !aligned(conv_w) ||
      !aligned(theta0) || !aligned(theta_out) || !aligned(out))
    return TTT_EALIGN;
  int rc = fused_only(dims);
  if (rc != TTT_OK) return rc;
  if (dims->d != 64) return TTT_EUNSUPPORTED;   // the normalising epilogue takes heads of 64
  Call c;
  rc = prepare(dims, TTT_OP_ATTENTION, workspace, workspace_bytes, stream, &c);
  if (rc != TTT_OK) return rc;
  uint16_t* q = reinterpret_cast<uint16_t*>(c.ws + c.w.q);
  uint16_t* k = reinterpret_cast<uint16_t*>(c.ws + c.w.k);
  uint16_t* v = reinterpret_cast<uint16_t*>(c.ws + c.w.v);
  uint16_t* o = reinterpret_cast<uint16_t*>(c.ws + c.w.o);
  if ((rc = run_qkv(c, X, Wq, Wk, Wv, q, k, v)) != TTT_OK) return rc;
  rc = inner == TTT_INNER_SGD ? run_write(c, dims, k, v, conv_w, theta0, lr, steps, theta_out)
                              : run_write_muon(c, dims, k, v, conv_w, theta0, lr, steps, theta_out);
  if (rc != TTT_OK) return rc;
  if ((rc = run_read(c, q, theta_out, o)) != TTT_OK) return rc;
  return run_out_proj(c, o, Wo, out);
}

int ttt_gemm_bf16(int M, int N, int K, const uint16_t* A, int64_t lda, int a_layout, const uint16_t* B, int64_t ldb,
                  int b_layout, uint16_t* C, int64_t ldc, void* stream) {
  if (!A || !B || !C || M < 1 || N < 1 || K < 1) return TTT_EINVAL;
  if ((a_layout != 0 && a_layout != 1) || (b_layout != 0 && b_layout != 1)) return TTT_EINVAL;
  if (lda < (a_layout ? M : K) || ldb < (b_layout ? K : N) || ldc < N) return TTT_EINVAL;
  if (!aligned(A) || !aligned(B) || !aligned(C) || lda % 8 || ldb % 8 || ldc % 8 || N % 8) return TTT_EALIGN;
  GemmLaunch g;
  const bool a_mn = a_layout == 1, b_mn = b_layout == 0;
  if (!make_gemm_map(&g.ma[0], A, a_mn ? K : M, a_mn ? M : K, lda, a_mn) ||
      !make_gemm_map(&g.mb[0], B, b_mn ? K : N, b_mn ? N : K, ldb, b_mn))
    return TTT_ECUDA;
  GemmProblem& p = g.add(M, N, K, a_mn, b_mn);
  p.out = C;
  p.ldo = ldc;
  return launch_gemm<kEpiStore>(g, nullptr, KK_GEMM_STORE, static_cast<cudaStream_t>(stream));
}

int ttt_layer_host(const ttt_dims* dims, const uint16_t* Q_host, const uint16_t* K_host, const uint16_t* V_host,
                   const float* conv_w_host, const float* theta0_host, float lr, int steps, float* theta_out_host,
                   uint16_t* O_host, void* workspace, size_t workspace_bytes, void* stream) {
  if (!Q_host || !K_host || !V_host || !conv_w_host || !theta0_host || !theta_out_host || !O_host || steps < 0)
    return TTT_EINVAL;
  Call c;
  int rc = prepare(dims, TTT_OP_LAYER_HOST, workspace, workspace_bytes, stream, &c);
  if (rc != TTT_OK) return rc;
  const Shape& s = c.s;
  const size_t tok = static_cast<size_t>(s.n) * s.C * 2;
  const size_t thb = 3ull * s.H * s.D * s.h * 4;
  uint16_t* dq = reinterpret_cast<uint16_t*>(c.ws + c.w.q);
  uint16_t* dk = reinterpret_cast<uint16_t*>(c.ws + c.w.k);
  uint16_t* dv = reinterpret_cast<uint16_t*>(c.ws + c.w.v);
  uint16_t* dout = reinterpret_cast<uint16_t*>(c.ws + c.w.o);
  float* dw = reinterpret_cast<float*>(c.ws + c.w.convw);
  float* dth0 = reinterpret_cast<float*>(c.ws + c.w.th0);
  float* dthout = reinterpret_cast<float*>(c.ws + c.w.thout);
  const size_t convb = static_cast<size_t>(s.C) * 9 * 4;
  if (s.wide) {
    // wide-head path: one copy each, in order on the caller's stream
    if (cudaMemcpyAsync(dq, Q_host, tok, cudaMemcpyHostToDevice, c.st) != cudaSuccess ||
        cudaMemcpyAsync(dk, K_host, tok, cudaMemcpyHostToDevice, c.st) != cudaSuccess ||
        cudaMemcpyAsync(dv, V_host, tok, cudaMemcpyHostToDevice, c.st) != cudaSuccess ||
        cudaMemcpyAsync(dw, conv_w_host, convb, cudaMemcpyHostToDevice, c.st) != cudaSuccess ||
        cudaMemcpyAsync(dth0, theta0_host, thb, cudaMemcpyHostToDevice, c.st) != cudaSuccess)
      return TTT_ECUDA;
    if ((rc = run_write(c, dims, dk, dv, dw, dth0, lr, steps, dthout)) != TTT_OK) return rc;
    if ((rc = run_read(c, dq, dthout, dout)) != TTT_OK) return rc;
    if (cudaMemcpyAsync(theta_out_host, dthout, thb, cudaMemcpyDeviceToHost, c.st) != cudaSuccess ||
        cudaMemcpyAsync(O_host, dout, tok, cudaMemcpyDeviceToHost, c.st) != cudaSuccess)
      return TTT_ECUDA;
    return TTT_OK;
  }
  // Fused path, pipelined over the two copy directions: the upload stream
  // copies conv_w, theta0, V, K, then Q in chunks while the write runs; each
  // chunk of Q is read as soon as it has landed, and its O goes back on the
  // download stream while the next chunk is read.  Chunks are whole 128-token
  // tiles, so each read launch covers exactly its own tokens.
  const long long chunk_tiles =
      std::max<long long>(kHostChunkMinTiles, (static_cast<long long>(s.tiles) + kHostChunks - 1) / kHostChunks);
  const int chunks = static_cast<int>((s.tiles + chunk_tiles - 1) / chunk_tiles);
  HostPipe hp;
  if (!hp.init(4 + 2 * chunks)) return TTT_ECUDA;
  cudaEvent_t ev_start = hp.ev[0], ev_kv = hp.ev[1], ev_th = hp.ev[2], ev_done = hp.ev[3];
  cudaEvent_t* ev_q = hp.ev + 4;
  cudaEvent_t* ev_o = hp.ev + 4 + chunks;
  const size_t row_bytes = static_cast<size_t>(s.C) * 2;
  auto chunk_rows = [&](int i, long long* t0) {
    *t0 = i * chunk_tiles * kTileM;
    return std::min<long long>(chunk_tiles * kTileM, s.n - *t0);
  };
  // everything earlier on the caller's stream comes first
  if (cudaEventRecord(ev_start, c.st) != cudaSuccess || cudaStreamWaitEvent(hp.up, ev_start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp.down, ev_start, 0) != cudaSuccess)
    return TTT_ECUDA;
  if (cudaMemcpyAsync(dw, conv_w_host, convb, cudaMemcpyHostToDevice, hp.up) != cudaSuccess ||
      cudaMemcpyAsync(dth0, theta0_host, thb, cudaMemcpyHostToDevice, hp.up) != cudaSuccess ||
      cudaMemcpyAsync(dv, V_host, tok, cudaMemcpyHostToDevice, hp.up) != cudaSuccess ||
      cudaMemcpyAsync(dk, K_host, tok, cudaMemcpyHostToDevice, hp.up) != cudaSuccess ||
      cudaEventRecord(ev_kv, hp.up) != cudaSuccess)
    return TTT_ECUDA;
  for (int i = 0; i < chunks; ++i) {
    long long t0;
    const long long nt = chunk_rows(i, &t0);
    if (cudaMemcpyAsync(dq + t0 * s.C, Q_host + t0 * s.C, nt * row_bytes, cudaMemcpyHostToDevice, hp.up) !=
            cudaSuccess ||
        cudaEventRecord(ev_q[i], hp.up) != cudaSuccess)
      return TTT_ECUDA;
  }
  if (cudaStreamWaitEvent(c.st, ev_kv, 0) != cudaSuccess) return TTT_ECUDA;
  if ((rc = run_write(c, dims, dk, dv, dw, dth0, lr, steps, dthout)) != TTT_OK) return rc;
  if ((rc = run_pack(s, dthout, c.w, c.ws, false, c.st)) != TTT_OK) return rc;
  // theta* goes back once the write (and the pack that reads it) is done
  if (cudaEventRecord(ev_th, c.st) != cudaSuccess || cudaStreamWaitEvent(hp.down, ev_th, 0) != cudaSuccess ||
      cudaMemcpyAsync(theta_out_host, dthout, thb, cudaMemcpyDeviceToHost, hp.down) != cudaSuccess)
    return TTT_ECUDA;
  for (int i = 0; i < chunks; ++i) {
    long long t0;
    const long long nt = chunk_rows(i, &t0);
    if (cudaStreamWaitEvent(c.st, ev_q[i], 0) != cudaSuccess) return TTT_ECUDA;
    if ((rc = launch_read_tokens(c, dq + t0 * s.C, dout + t0 * s.C, nt)) != TTT_OK) return rc;
    if (cudaEventRecord(ev_o[i], c.st) != cudaSuccess || cudaStreamWaitEvent(hp.down, ev_o[i], 0) != cudaSuccess ||
        cudaMemcpyAsync(O_host + t0 * s.C, dout + t0 * s.C, nt * row_bytes, cudaMemcpyDeviceToHost, hp.down) !=
            cudaSuccess)
      return TTT_ECUDA;
  }
  if (cudaEventRecord(ev_done, hp.down) != cudaSuccess || cudaStreamWaitEvent(c.st, ev_done, 0) != cudaSuccess)
    return TTT_ECUDA;
  return TTT_OK;
}

int ttt_set_wait_limit(long long clocks) {
  if (clocks < 0) return TTT_EINVAL;
  wait_clock_setting().store(clocks, std::memory_order_relaxed);
  return TTT_OK;
}

int ttt_check_status(const void* workspace, void* stream) {
  if (!workspace) return TTT_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return TTT_ECUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, workspace, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return TTT_ECUDA;
  if (v != 0) {
    if (cudaMemset(const_cast<void*>(workspace), 0, 4) != cudaSuccess) return TTT_ECUDA;
    return TTT_EDEVICE;
  }
  return TTT_OK;
}

int ttt_profile_start(void) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> lock(p.mu);
  p.on = true;
  p.used = 0;
  p.dropped = 0;
  return TTT_OK;
}

int ttt_profile_stop(ttt_kernel_times* out) {
  if (!out) return TTT_EINVAL;
  Profiler& p = profiler();
  std::lock_guard<std::mutex> lock(p.mu);
  p.on = false;
  memset(out, 0, sizeof(*out));
  int rc = TTT_OK;
  for (size_t i = 0; i < p.used; ++i) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, p.ev[2 * i], p.ev[2 * i + 1]) != cudaSuccess) {
      rc = TTT_ECUDA;
      continue;
    }
    out->launches[p.kind[i]] += 1;
    out->total_ms[p.kind[i]] += ms;
  }
  out->dropped = p.dropped;
  p.used = 0;
  return rc;
}

const char* ttt_kernel_name(int kind) {
  return (kind >= 0 && kind < TTT_KERNEL_KINDS) ? kKernelNames[kind] : "unknown";
}

const char* ttt_status_str(int status) {
  switch (status) {
    case TTT_OK: return "ok";
    case TTT_EINVAL: return "invalid argument";
    case TTT_EALIGN: return "misaligned pointer";
    case TTT_EUNSUPPORTED: return "unsupported shape";
    case TTT_EWORKSPACE: return "workspace too small";
    case TTT_ECUDA: return "CUDA error";
    case TTT_EDEVICE: return "device-side fault recorded";
    default: return "unknown status";
  }
}

}  // extern "C"
