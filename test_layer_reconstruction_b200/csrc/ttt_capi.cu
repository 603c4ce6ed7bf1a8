// ttt_capi.cu — the C ABI declared in include/ttt.h: host-side validation,
// workspace layout, TMA descriptors and the launch sequence of the layer
//   conv -> steps x [pack theta -> forward (residual) -> backward (partials)
//   -> reduce + SGD] -> pack theta* -> forward (read)
// for head widths 16, 32, 64 (h <= 256), and the wide-head sequence (token
// chunks of bf16 library GEMMs and the elementwise kernels of wide.cuh) for
// head widths and hidden widths that are multiples of 64 beyond that.
#include <cublas_v2.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/ttt.h"
#include "conv.cuh"
#include "update.cuh"
#include "wide.cuh"

using namespace ttt;

namespace {

constexpr size_t kAlign = 1024;
constexpr int kMaxDevicesWide = 64;
size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

struct Shape {
  long long n;   // tokens
  int H, D, h, hidp, tiles, slices, units;
  long long C;   // H * D channels
  bool wide;     // wide-head path (library GEMMs over token chunks)
};

constexpr long long kWideChunk = 131072;           // tokens per GEMM chunk of the wide path
constexpr size_t kWideGemmWorkspace = 32u << 20;   // library GEMM workspace (bytes)

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
  size_t img, acc, z1, z3, da, ab, eb, gemm;   // wide path
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
    w.img = take(3ull * s.H * s.D * s.h * 2);
    w.z1 = take(nc * s.h * 2);
    w.z3 = take(nc * s.h * 2);
    w.ab = take(nc * s.h * 2);
    w.gemm = take(kWideGemmWorkspace);
    if (writes) {
      w.acc = take(3ull * s.D * s.h * 4);
      w.da = take(nc * s.h * 2);
      w.eb = take(nc * s.D * 2);
      w.vp = take(tok_bytes);
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
  if (op == TTT_OP_WRITE || op == TTT_OP_LAYER || op == TTT_OP_LAYER_HOST) {
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
enum KernelKind { KK_CONV = 0, KK_PACK = 1, KK_FWD_WRITE = 2, KK_BWD = 3, KK_REDUCE = 4, KK_FWD_READ = 5 };
const char* const kKernelNames[TTT_KERNEL_KINDS] = {"shortconv2d", "pack_theta", "swiglu_fwd_residual",
                                                     "swiglu_bwd_partials", "reduce_sgd", "swiglu_fwd_read"};
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

bool aligned(const void* p, size_t a = 16) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int launch_status() { return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ECUDA; }

// ------------------------------------------------------------------ launches
int run_conv(const Shape& s, const ttt_dims* dm, const uint16_t* V, const float* w, uint16_t* out,
             cudaStream_t st) {
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
  if (cudaFuncSetAttribute(shortconv_kernel<kConvBand>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return TTT_ECUDA;
  ProfScope prof(KK_CONV, st);
  shortconv_kernel<kConvBand><<<grid, block, smem, st>>>(p);
  return launch_status();
}

// Operand images of theta; the backward kernel's weight rows only when `with_wt`.
int run_pack(const Shape& s, const float* theta, const Ws& w, uint8_t* ws, bool with_wt, cudaStream_t st) {
  PackParams p;
  p.theta = theta;
  p.w13_img = reinterpret_cast<__nv_bfloat16*>(ws + w.w13);
  p.w2h_img = reinterpret_cast<__half*>(ws + w.w2h);
  p.wt_img = with_wt ? reinterpret_cast<__nv_bfloat16*>(ws + w.wt) : nullptr;
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

// ------------------------------------------------------------------ wide path
// One library GEMM handle per device, created on first use; enqueues of the
// wide path on a device are serialised because the handle's stream and
// workspace are set per call.
struct WideGemm {
  std::mutex mu;
  cublasHandle_t h[kMaxDevicesWide] = {};
};
WideGemm& wide_gemm() {
  static WideGemm g;
  return g;
}

// Row-major C[M x N] (ldc) = alpha op(A)[M x K] op(B)[K x N] + beta C, bf16 A and
// B, FP32 accumulation; op(A) = A^T when `ta` (A stored K x M), likewise B.
// Column-major view: C^T = op(B)^T op(A)^T.
bool gemm_rm(cublasHandle_t hd, bool ta, bool tb, int M, int N, int K, float alpha, const void* A, int lda,
             const void* B, int ldb, float beta, void* C, cudaDataType_t ctype, int ldc) {
  return cublasGemmEx(hd, tb ? CUBLAS_OP_T : CUBLAS_OP_N, ta ? CUBLAS_OP_T : CUBLAS_OP_N, N, M, K, &alpha, B,
                      CUDA_R_16BF, ldb, A, CUDA_R_16BF, lda, &beta, C, ctype, ldc, CUBLAS_COMPUTE_32F,
                      CUBLAS_GEMM_DEFAULT) == CUBLAS_STATUS_SUCCESS;
}

unsigned elementwise_grid(long long n8) {
  const int sms = num_sms();
  return static_cast<unsigned>(std::max<long long>(1, std::min<long long>((n8 + 255) / 256, 8LL * (sms > 0 ? sms : 148))));
}

// Takes the device's GEMM handle (created on first use) bound to this call's
// stream and workspace; holds the device's lock for the caller's enqueue.
struct WideCall {
  std::unique_lock<std::mutex> lock;
  cublasHandle_t hd = nullptr;
  bool ok = false;
  WideCall(const Call& c) : lock(wide_gemm().mu) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevicesWide) return;
    cublasHandle_t& h = wide_gemm().h[dev];
    if (!h && cublasCreate(&h) != CUBLAS_STATUS_SUCCESS) {
      h = nullptr;
      return;
    }
    if (cublasSetStream(h, c.st) != CUBLAS_STATUS_SUCCESS) return;
    if (cublasSetWorkspace(h, c.ws + c.w.gemm, kWideGemmWorkspace) != CUBLAS_STATUS_SUCCESS) return;
    hd = h;
    ok = true;
  }
};

int wide_cast(const Call& c, const float* theta) {
  const long long count = 3LL * c.s.H * c.s.D * c.s.h;
  wide_cast_kernel<<<elementwise_grid(count / 8), 256, 0, c.st>>>(
      theta, reinterpret_cast<__nv_bfloat16*>(c.ws + c.w.img), count);
  return launch_status();
}

// Z1, Z3 (bf16) of rows [t0, t0 + nc) of head hd of X, then A = silu(Z1) Z3.
int wide_forward_chunk(const Call& c, cublasHandle_t hd, const uint16_t* X, int head, long long t0, int nc) {
  const Shape& s = c.s;
  const size_t per = static_cast<size_t>(s.D) * s.h;
  const __nv_bfloat16* img = reinterpret_cast<const __nv_bfloat16*>(c.ws + c.w.img);
  const uint16_t* xc = X + (static_cast<size_t>(t0) * s.H + head) * s.D;
  const int ldx = s.H * s.D;
  if (!gemm_rm(hd, false, false, nc, s.h, s.D, 1.f, xc, ldx, img + head * per, s.h, 0.f, c.ws + c.w.z1, CUDA_R_16BF,
               s.h) ||
      !gemm_rm(hd, false, false, nc, s.h, s.D, 1.f, xc, ldx, img + (s.H + head) * per, s.h, 0.f, c.ws + c.w.z3,
               CUDA_R_16BF, s.h))
    return TTT_ECUDA;
  const long long n8 = static_cast<long long>(nc) * s.h / 8;
  wide_gate_kernel<<<elementwise_grid(n8), 256, 0, c.st>>>(reinterpret_cast<const uint4*>(c.ws + c.w.z1),
                                                           reinterpret_cast<const uint4*>(c.ws + c.w.z3),
                                                           reinterpret_cast<uint4*>(c.ws + c.w.ab), n8);
  return launch_status();
}

// dW of one head of the wide path over all tokens, per token chunk
//   Z1, Z3, A (forward) -> E = A W2 - V' -> dA = E W2^T -> dZ1, dZ3
//   -> dW1 += K^T dZ1, dW3 += K^T dZ3, dW2 += A^T E   (FP32, Eq. 5)
// into the workspace accumulator; the operand image of theta is current.
int wide_grad_head(const Call& c, cublasHandle_t hd, const uint16_t* K, const uint16_t* vp, int head) {
  const Shape& s = c.s;
  const size_t per = static_cast<size_t>(s.D) * s.h;
  const __nv_bfloat16* img = reinterpret_cast<const __nv_bfloat16*>(c.ws + c.w.img);
  float* acc = reinterpret_cast<float*>(c.ws + c.w.acc);
  uint8_t* eb = c.ws + c.w.eb;
  const int ldx = s.H * s.D;
  const __nv_bfloat16* w2 = img + (2 * static_cast<size_t>(s.H) + head) * per;   // [h][D]
  int rc;
  for (long long t0 = 0; t0 < s.n; t0 += kWideChunk) {
    const int nc = static_cast<int>(std::min<long long>(kWideChunk, s.n - t0));
    const float beta = t0 == 0 ? 0.f : 1.f;
    if ((rc = wide_forward_chunk(c, hd, K, head, t0, nc)) != TTT_OK) return rc;
    // E = A W2 - V' (the chunk's V' rows first copied into E)
    if (cudaMemcpy2DAsync(eb, static_cast<size_t>(s.D) * 2, vp + (static_cast<size_t>(t0) * s.H + head) * s.D,
                          static_cast<size_t>(ldx) * 2, static_cast<size_t>(s.D) * 2, nc, cudaMemcpyDeviceToDevice,
                          c.st) != cudaSuccess)
      return TTT_ECUDA;
    if (!gemm_rm(hd, false, false, nc, s.D, s.h, 1.f, c.ws + c.w.ab, s.h, w2, s.D, -1.f, eb, CUDA_R_16BF, s.D) ||
        !gemm_rm(hd, false, true, nc, s.h, s.D, 1.f, eb, s.D, w2, s.D, 0.f, c.ws + c.w.da, CUDA_R_16BF, s.h))
      return TTT_ECUDA;
    const long long n8 = static_cast<long long>(nc) * s.h / 8;
    wide_dz_kernel<<<elementwise_grid(n8), 256, 0, c.st>>>(reinterpret_cast<uint4*>(c.ws + c.w.z1),
                                                           reinterpret_cast<uint4*>(c.ws + c.w.z3),
                                                           reinterpret_cast<const uint4*>(c.ws + c.w.da), n8);
    if ((rc = launch_status()) != TTT_OK) return rc;
    const uint16_t* kc = K + (static_cast<size_t>(t0) * s.H + head) * s.D;
    if (!gemm_rm(hd, true, false, s.D, s.h, nc, 1.f, kc, ldx, c.ws + c.w.z1, s.h, beta, acc, CUDA_R_32F, s.h) ||
        !gemm_rm(hd, true, false, s.D, s.h, nc, 1.f, kc, ldx, c.ws + c.w.z3, s.h, beta, acc + per, CUDA_R_32F,
                 s.h) ||
        !gemm_rm(hd, true, false, s.h, s.D, nc, 1.f, c.ws + c.w.ab, s.h, eb, s.D, beta, acc + 2 * per, CUDA_R_32F,
                 s.D))
      return TTT_ECUDA;
  }
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
  WideCall wc(c);
  if (!wc.ok) return TTT_ECUDA;
  const size_t per = static_cast<size_t>(s.D) * s.h;
  const float* acc = reinterpret_cast<const float*>(c.ws + c.w.acc);
  const float scale = lr * 2.0f / static_cast<float>(s.n);
  for (int step = 0; step < steps; ++step) {
    const float* th_in = step == 0 ? theta0 : theta_out;
    if ((rc = wide_cast(c, th_in)) != TTT_OK) return rc;
    for (int head = 0; head < s.H; ++head) {
      if ((rc = wide_grad_head(c, wc.hd, K, vp, head)) != TTT_OK) return rc;
      wide_sgd_kernel<<<elementwise_grid(static_cast<long long>(3 * per) / 8), 256, 0, c.st>>>(
          th_in, theta_out, acc, s.H, s.D, s.h, head, scale);
      if ((rc = launch_status()) != TTT_OK) return rc;
    }
  }
  return TTT_OK;
}

// The gradient (1/2) d/dtheta sum_i ||T(k_i) - v'_i||^2 of the wide path.
int run_grad_wide(const Call& c, const uint16_t* K, const uint16_t* vp, const float* theta, float* grad) {
  const Shape& s = c.s;
  WideCall wc(c);
  if (!wc.ok) return TTT_ECUDA;
  const size_t per = static_cast<size_t>(s.D) * s.h;
  const float* acc = reinterpret_cast<const float*>(c.ws + c.w.acc);
  int rc = wide_cast(c, theta);
  if (rc != TTT_OK) return rc;
  for (int head = 0; head < s.H; ++head) {
    if ((rc = wide_grad_head(c, wc.hd, K, vp, head)) != TTT_OK) return rc;
    wide_grad_kernel<<<elementwise_grid(static_cast<long long>(3 * per) / 8), 256, 0, c.st>>>(grad, acc, s.H, s.D,
                                                                                              s.h, head);
    if ((rc = launch_status()) != TTT_OK) return rc;
  }
  return TTT_OK;
}

// The read of the wide path: per head and token chunk, Z1, Z3, A, then
// O = A W2 written straight into the head's columns of O.
int run_read_wide(const Call& c, const uint16_t* Q, const float* theta, uint16_t* O) {
  const Shape& s = c.s;
  WideCall wc(c);
  if (!wc.ok) return TTT_ECUDA;
  int rc = wide_cast(c, theta);
  if (rc != TTT_OK) return rc;
  const size_t per = static_cast<size_t>(s.D) * s.h;
  const __nv_bfloat16* img = reinterpret_cast<const __nv_bfloat16*>(c.ws + c.w.img);
  const int ldx = s.H * s.D;
  for (int head = 0; head < s.H; ++head) {
    const __nv_bfloat16* w2 = img + (2 * static_cast<size_t>(s.H) + head) * per;
    for (long long t0 = 0; t0 < s.n; t0 += kWideChunk) {
      const int nc = static_cast<int>(std::min<long long>(kWideChunk, s.n - t0));
      if ((rc = wide_forward_chunk(c, wc.hd, Q, head, t0, nc)) != TTT_OK) return rc;
      if (!gemm_rm(wc.hd, false, false, nc, s.D, s.h, 1.f, c.ws + c.w.ab, s.h, w2, s.D, 0.f,
                   O + (static_cast<size_t>(t0) * s.H + head) * s.D, CUDA_R_16BF, ldx))
        return TTT_ECUDA;
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
  BwdParams& bp = gp->bp;
  bp.wt_img = reinterpret_cast<const uint32_t*>(c.ws + c.w.wt);
  bp.partials = reinterpret_cast<float*>(c.ws + c.w.part);
  bp.n = fp.n;
  bp.heads = s.H;
  bp.units = s.units;
  bp.slices = s.slices;
  bp.max_contrib = c.g.max_contrib;
  bp.status = status;
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

// The pages' inner loop: `steps` Muon steps on the dot-product loss.
int run_write_muon(const Call& c, const ttt_dims* dm, const uint16_t* K, const uint16_t* V, const float* conv_w,
                   const float* theta0, float lr, int steps, float* theta_out) {
  const Shape& s = c.s;
  uint16_t* vp = reinterpret_cast<uint16_t*>(c.ws + c.w.vp);
  float* grad = reinterpret_cast<float*>(c.ws + c.w.grad);
  int rc = run_conv(s, dm, V, conv_w, vp, c.st);
  if (rc != TTT_OK) return rc;
  if (steps == 0) {
    if (theta_out != theta0 &&
        cudaMemcpyAsync(theta_out, theta0, 3ull * s.H * s.D * s.h * 4, cudaMemcpyDeviceToDevice, c.st) != cudaSuccess)
      return TTT_ECUDA;
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
  if (op < TTT_OP_WRITE || op > TTT_OP_LAYER_HOST) return 0;
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
  int rc = fused_only(dims);
  if (rc != TTT_OK) return rc;
  Call c;
  rc = prepare(dims, TTT_OP_WRITE, workspace, workspace_bytes, stream, &c);
  if (rc != TTT_OK) return rc;
  GradPass gp;
  if (!setup_grad_pass(c, K, Vp, &gp, true)) return TTT_ECUDA;
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
  int rc = fused_only(dims);
  if (rc != TTT_OK) return rc;
  Call c;
  rc = prepare(dims, TTT_OP_WRITE, workspace, workspace_bytes, stream, &c);
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
  int rc = fused_only(dims);
  if (rc != TTT_OK) return rc;
  Call c;
  rc = prepare(dims, TTT_OP_LAYER, workspace, workspace_bytes, stream, &c);
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
