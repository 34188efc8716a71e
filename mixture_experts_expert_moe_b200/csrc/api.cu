// Host side of the C ABI declared in include/moe_b200.h: argument checks,
// workspace carving and kernel launches.  No device memory is allocated and
// no call synchronises the host.
#include <cstdio>
#include <cstring>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "kernels.cuh"

namespace {
thread_local std::string g_last_cuda_error;
}  // namespace

namespace moe {
moe_status_t record_cuda_error(cudaError_t e, const char* where) {
  char buf[256];
  snprintf(buf, sizeof(buf), "%s: %s (%d)", where, cudaGetErrorString(e), (int)e);
  g_last_cuda_error = buf;
  return MOE_ERR_CUDA;
}
}  // namespace moe

namespace {

inline moe_status_t cuda_fail(cudaError_t e, const char* where) { return moe::record_cuda_error(e, where); }

#define MOE_CU(call)                                          \
  do {                                                        \
    cudaError_t _e = (call);                                  \
    if (_e != cudaSuccess) return cuda_fail(_e, #call);       \
  } while (0)

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// An NVTX range over a scope (entry points and the forward's stages show up
// by name in Nsight Systems / Compute timelines; a no-op without a tool).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

struct Carver {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  }
};

inline cudaError_t record(void** ev, int i, cudaStream_t s) {
  return ev ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) : cudaSuccess;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

moe_status_t check_device() {
  int dev = 0, major = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver) {
    cuda_fail(e, "cudaGetDevice");   // keeps the text for moe_last_cuda_error
    return MOE_ERR_DEVICE;           // no usable GPU at all: there is no CPU fallback
  }
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  return major == 10 ? MOE_OK : MOE_ERR_DEVICE;
}

// ---------------------------------------------------------------------------
// align & sort
// ---------------------------------------------------------------------------
constexpr int kMaxAlignCtas = 1024;
constexpr int kMinSlotsPerCta = 4096;
// up to this many slots the FP8 path quantises per sorted row (the token's k
// copies are quantised redundantly) instead of once per token plus a gather
constexpr int kFusedQuantSlots = 4096;
// tokens gated per CTA of the fused routing launch (at most one CTA per SM).
// Each warp gates its tokens one after another (k arg-max rounds each), so
// fewer tokens per CTA shorten the gating phase, while more CTAs lengthen the
// cross-CTA count merge.  Measured routing launch (T = 2048, top-8 of 256):
// 37.9 us at 64 tokens per CTA, 29.7 at 32, 26.8 at 16; 25.2 us at 16 vs 38.5
// at 64 for T = 256.
constexpr int kRouteTokensPerCta = 16;
constexpr long long kRouteZeroMaxFloats = 65536;   // 256 KB: a few us for one CTA

bool align_args_ok(int T, int k, int E, int bm) {
  return T >= 0 && k >= 1 && E >= 1 && E <= 1024 && bm >= 1 && bm <= 1024 &&
         (long long)T * k + (long long)E * (bm - 1) < 0x7FFFFFFFLL;
}

size_t align_ws_bytes(int E) { return 256 + (size_t)kMaxAlignCtas * E * sizeof(int32_t); }

moe_status_t run_align(const int32_t* ids, int T, int k, int E, int bm, int32_t* sorted, int32_t* expert_ids,
                       int32_t* num_post, void* ws, int32_t* status, cudaStream_t stream) {
  const int N = T * k;
  int err = 0;
  const int max_ctas = moe::align_max_ctas(E, &err);
  if (err) return cuda_fail((cudaError_t)err, "align occupancy");
  if (max_ctas < 1) return MOE_ERR_UNSUPPORTED;
  const int per_cta_unit = 32 * 32;  // warps x lanes
  int grid = (int)(((long long)N + kMinSlotsPerCta - 1) / kMinSlotsPerCta);
  grid = grid < 1 ? 1 : grid;
  grid = grid > max_ctas ? max_ctas : grid;
  grid = grid > kMaxAlignCtas ? kMaxAlignCtas : grid;
  int chunk = (N + grid - 1) / grid;
  chunk = (chunk + per_cta_unit - 1) / per_cta_unit * per_cta_unit;
  if (chunk < per_cta_unit) chunk = per_cta_unit;
  grid = N > 0 ? (N + chunk - 1) / chunk : 1;

  uint8_t* w = static_cast<uint8_t*>(ws);
  moe::AlignParams p;
  p.ids = ids;
  p.N = N;
  p.E = E;
  p.bm = bm;
  p.chunk = chunk;
  p.sorted = sorted;
  p.expert_ids = expert_ids;
  p.num_post = num_post;
  p.barrier = reinterpret_cast<int*>(w);
  p.hist = reinterpret_cast<int32_t*>(w + 256);
  p.status = status;
  p.timeout_ns = moe::kDefaultTimeoutNs;
  p.expected = grid;
  MOE_CU(cudaMemsetAsync(p.barrier, 0, sizeof(int), stream));
  MOE_CU(moe::launch_align_sort(p, grid, stream));
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// grouped FFN
// ---------------------------------------------------------------------------
struct FfnShape {
  int T, H, I, E, k, bm, fp8, tn;
  int mx, fp4;          // MX block-scaled operands; E2M1 weights
  long long P, NB, N;
  long long rows_max;   // bound on num_post: at most min(E, N) experts pad, each by < bm rows
};

int pick_tn(const FfnShape& s, int hint) {
  if (hint) return hint;
  const double avg = (double)s.N / s.E;  // slots per expert
  long long need = (long long)((avg * 1.25 + s.bm - 1) / s.bm) * s.bm;
  if (need < s.bm) need = s.bm;
  // MX tiles stage every stage's activation scales of two token tiles in
  // shared memory, which leaves room for at most 128 tokens per tile
  const int cap = s.mx ? 128 : 256;
  int tn = 16;
  while (tn < need && tn < cap) tn <<= 1;
  return tn;
}

moe_status_t ffn_shape(int T, int H, int I, int E, int k, int bm, int wdtype, int hint, FfnShape* s) {
  if (!align_args_ok(T, k, E, bm) || H <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
  if (k > 32 || k > E) return MOE_ERR_INVALID_ARG;
  if (wdtype != MOE_BF16 && wdtype != MOE_FP8_E4M3 && wdtype != MOE_MXFP8 && wdtype != MOE_MXFP4)
    return MOE_ERR_INVALID_ARG;
  if (hint != 0 && hint != 16 && hint != 32 && hint != 64 && hint != 128 && hint != 256)
    return MOE_ERR_INVALID_ARG;
  if (H % 128 || I % 128) return MOE_ERR_UNSUPPORTED;
  s->T = T; s->H = H; s->I = I; s->E = E; s->k = k; s->bm = bm;
  s->fp8 = wdtype == MOE_FP8_E4M3;
  s->mx = wdtype == MOE_MXFP8 || wdtype == MOE_MXFP4;
  s->fp4 = wdtype == MOE_MXFP4;
  if (s->mx && hint > 128) return MOE_ERR_UNSUPPORTED;
  s->N = (long long)T * k;
  s->P = s->N + (long long)E * (bm - 1);
  s->NB = (s->P + bm - 1) / bm;
  {
    const long long touched = s->N < E ? s->N : E;
    const long long bound = s->N + touched * (bm - 1);
    s->rows_max = bound < s->P ? bound : s->P;
  }
  s->tn = pick_tn(*s, hint);
  if ((long long)s->P * (s->H > s->I ? s->H : s->I) >= (1LL << 40)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

struct FfnWs {
  size_t plan, xq, sx, A, sA, h, hq, sH, total;
};

// Workspace: the tile plan; the sorted activations A (bf16, E4M3 + a scale
// per row, or MX: E4M3 + E8M0 per 32 elements); h (bf16), and in FP8 / MX
// its quantised copy hq with its scales (MX: h is quantised by the gate/up
// epilogue, so only hq exists).
FfnWs ffn_ws_layout(const FfnShape& s) {
  Carver c;
  FfnWs w;
  w.plan = c.take((size_t)moe::plan_ints(s.E) * 4);
  w.xq = c.take(s.fp8 ? (size_t)s.T * s.H : 0);
  w.sx = c.take(s.fp8 ? (size_t)s.T * 4 : 0);
  w.A = c.take((size_t)s.P * s.H * (s.fp8 || s.mx ? 1 : 2));
  w.sA = c.take(s.fp8 ? (size_t)s.P * 4 : s.mx ? (size_t)s.P * (s.H / 32) : 0);
  w.h = c.take(s.mx ? 0 : (size_t)s.P * s.I * 2);
  w.hq = c.take(s.fp8 || s.mx ? (size_t)s.P * s.I : 0);
  w.sH = c.take(s.fp8 ? (size_t)s.P * 4 : s.mx ? (size_t)s.P * (s.I / 32) : 0);
  w.total = c.off;
  return w;
}

moe_status_t gemm_fail(int r, const char* what) {
  if (r == -1) {
    g_last_cuda_error = std::string(what) + ": cuTensorMapEncodeTiled failed";
    return MOE_ERR_CUDA;
  }
  return cuda_fail((cudaError_t)r, what);
}

// Runs plan -> gather(+quant) -> gate/up GEMM -> (requant) -> down GEMM.
// Weight operands of one FFN call.
struct FfnWeights {
  const void* w13;
  const float* w13s;          // FP8: per-channel scales
  const void* w2;
  const float* w2s;
  const uint8_t* w13_mx;      // MX: tiled E8M0 scales
  const uint8_t* w2_mx;
};

moe_status_t run_ffn(const FfnShape& s, const void* x, const FfnWeights& W, const int32_t* sorted,
                     const int32_t* expert_ids, const int32_t* num_post, float* y, uint8_t* ws, int32_t* status,
                     cudaStream_t stream, void** ev = nullptr, bool plan_ready = false, float* comb_out = nullptr,
                     const float* comb_w = nullptr) {
  const void* w13 = W.w13;
  const void* w2 = W.w2;
  const float* w13s = W.w13s;
  const float* w2s = W.w2s;
  const FfnWs L = ffn_ws_layout(s);
  int32_t* plan = reinterpret_cast<int32_t*>(ws + L.plan);
  void* A = ws + L.A;
  float* sA = reinterpret_cast<float*>(ws + L.sA);
  void* xq = ws + L.xq;
  float* sx = reinterpret_cast<float*>(ws + L.sx);
  void* h = ws + L.h;
  void* hq = ws + L.hq;
  float* sH = reinterpret_cast<float*>(ws + L.sH);
  const int P = (int)s.P, N = (int)s.N;
  const int R = (int)s.rows_max;   // grid size of the row kernels (they read num_post on the device)

  if (!plan_ready) {
    NvtxRange nr("moe: tile plan");
    MOE_CU(moe::launch_plan(expert_ids, num_post, sorted, N, P, s.E, s.bm, s.tn, s.I / 128, (s.H + 255) / 256, plan,
                            status, stream));
  }
  MOE_CU(record(ev, MOE_STAGE_PLAN + 1, stream));
  {
    NvtxRange nr_gather("moe: gather");
    if (s.mx) {
      // every sorted row MX-quantises its token (codes + a scale per 32 elements)
      MOE_CU(moe::launch_mx_quant_rows(x, sorted, N, s.k, num_post, R, s.H, A, reinterpret_cast<uint8_t*>(sA),
                                       stream));
    } else if (s.fp8 && N <= kFusedQuantSlots) {
      // few slots: each sorted row quantises its token directly (one launch)
      MOE_CU(moe::launch_quant_rows(x, sorted, /*gather=*/true, N, s.k, num_post, R, s.H, A, sA, status, stream));
    } else if (s.fp8) {
      // quantise each token once, then gather codes and scales into sorted order
      MOE_CU(moe::launch_quant_rows(x, nullptr, false, N, s.k, nullptr, s.T, s.H, xq, sx, status, stream));
      MOE_CU(moe::launch_gather_rows(xq, sx, sorted, num_post, R, N, s.k, s.H, A, sA, stream));
    } else {
      MOE_CU(moe::launch_gather_rows(x, nullptr, sorted, num_post, R, N, s.k, s.H * 2, A, nullptr, stream));
    }
  }
  MOE_CU(record(ev, MOE_STAGE_GATHER + 1, stream));

  moe::GemmLaunch g1 = {};
  g1.w = w13;
  g1.w_rows = (long long)s.E * 2 * s.I;
  g1.x = A;
  g1.x_rows = s.P;
  g1.p.gateup = 1;
  g1.p.fp8 = s.fp8;
  g1.p.mx = s.mx;
  g1.p.w_fp4 = s.fp4;
  g1.p.w_sf = W.w13_mx;
  g1.p.x_sf = reinterpret_cast<const uint8_t*>(sA);
  g1.p.h_sf = reinterpret_cast<uint8_t*>(sH);
  g1.p.K = s.H;
  g1.p.n_out = s.I;
  g1.p.tn = s.tn;
  g1.p.E = s.E;
  g1.p.n_slots = N;
  g1.p.k = s.k;
  g1.p.plan = plan;
  g1.p.sorted = sorted;
  g1.p.a_scale = sA;
  g1.p.w_scale = w13s;
  g1.p.out = s.mx ? hq : h;   // MX: the epilogue writes the MXFP8 codes of h (+ their scales)
  g1.p.status = status;
  g1.p.timeout_ns = moe::kDefaultTimeoutNs;
  g1.p.tile_counter = plan + moe::plan_counter(s.E, true);
  int r;
  {
    NvtxRange nr("moe: gate/up GEMM");
    r = moe::launch_grouped_gemm(g1, stream);
  }
  if (r) return gemm_fail(r, "gate/up GEMM");
  MOE_CU(record(ev, MOE_STAGE_GATEUP + 1, stream));

  // padding rows of h are skipped: the gate/up GEMM does not write them, and
  // the down GEMM stores no column of a padding slot
  if (s.fp8)
    MOE_CU(moe::launch_quant_rows(h, sorted, /*gather=*/false, N, s.k, num_post, R, s.I, hq, sH, status, stream));
  MOE_CU(record(ev, MOE_STAGE_REQUANT + 1, stream));

  moe::GemmLaunch g2 = {};
  g2.w = w2;
  g2.w_rows = (long long)s.E * s.H;
  g2.x = s.fp8 || s.mx ? hq : h;
  g2.x_rows = s.P;
  g2.p.gateup = 0;
  g2.p.fp8 = s.fp8;
  g2.p.mx = s.mx;
  g2.p.w_fp4 = s.fp4;
  g2.p.w_sf = W.w2_mx;
  g2.p.x_sf = reinterpret_cast<const uint8_t*>(sH);
  g2.p.K = s.I;
  g2.p.n_out = s.H;
  g2.p.tn = s.tn;
  g2.p.E = s.E;
  g2.p.n_slots = N;
  g2.p.k = s.k;
  g2.p.plan = plan;
  g2.p.sorted = sorted;
  g2.p.a_scale = sH;
  g2.p.w_scale = w2s;
  g2.p.out = y;
  g2.p.status = status;
  g2.p.timeout_ns = moe::kDefaultTimeoutNs;
  g2.p.tile_counter = plan + moe::plan_counter(s.E, false);
  g2.p.comb_out = comb_out;   // non-null: out32[t] += w * y in the epilogue, y is not written
  g2.p.comb_w = comb_w;
  {
    NvtxRange nr("moe: down GEMM");
    r = moe::launch_grouped_gemm(g2, stream);
  }
  if (r) return gemm_fail(r, "down GEMM");
  MOE_CU(record(ev, MOE_STAGE_DOWN + 1, stream));
  return MOE_OK;
}

// The weight pointers and scales a weight type needs, aligned for TMA.
bool weights_ok(const FfnShape& s, const void* w13, const float* w13s, const void* w2, const float* w2s,
                       const uint8_t* w13_mx, const uint8_t* w2_mx) {
  if (!w13 || !w2) return false;
  if (s.fp8 && (!w13s || !w2s)) return false;
  if (s.mx && (!w13_mx || !w2_mx || !aligned16(w13_mx) || !aligned16(w2_mx))) return false;
  const uintptr_t a = s.fp4 ? 31 : 15;   // packed 4-bit tensor maps need 32-byte aligned bases
  return ((reinterpret_cast<uintptr_t>(w13) | reinterpret_cast<uintptr_t>(w2)) & a) == 0;
}

// Gate + align&sort + tile plan in one launch (moe_forward).
// s holds the expert and slot counts with the shared experts included
// (s.E = E_routed + n_shared, s.k = k_routed + n_shared).
moe_status_t run_route(const FfnShape& s, int n_shared, bool select_only, const float* logits, const float* bias,
                       int32_t* ids, float* w, int32_t* sorted, int32_t* expert_ids, int32_t* num_post,
                       void* align_ws, int32_t* plan, int32_t* status, cudaStream_t stream,
                       float* zero_out = nullptr, long long zero_n = 0) {
  const int N = (int)s.N;
  int err = 0;
  const int max_ctas = moe::align_max_ctas(s.E, &err);
  if (err) return cuda_fail((cudaError_t)err, "route occupancy");
  if (max_ctas < 1) return MOE_ERR_UNSUPPORTED;
  int g = 32, b = s.k;  // unit = lcm(32 warps, k): a CTA's slots are whole tokens
  while (b) {
    const int t = g % b;
    g = b;
    b = t;
  }
  const int unit = 32 / g * s.k;
  // the gating work is per token: spread the tokens over the SMs
  int grid = (s.T + kRouteTokensPerCta - 1) / kRouteTokensPerCta;
  grid = grid < 1 ? 1 : grid;
  grid = grid > max_ctas ? max_ctas : grid;
  grid = grid > kMaxAlignCtas ? kMaxAlignCtas : grid;
  long long chunk = ((long long)N + grid - 1) / grid;
  chunk = (chunk + unit - 1) / unit * unit;
  if (chunk < unit) chunk = unit;
  grid = N > 0 ? (int)((N + chunk - 1) / chunk) : 1;

  uint8_t* wsb = static_cast<uint8_t*>(align_ws);
  moe::AlignParams p;
  p.ids = ids;
  p.N = N;
  p.E = s.E;
  p.bm = s.bm;
  p.chunk = (int)chunk;
  p.sorted = sorted;
  p.expert_ids = expert_ids;
  p.num_post = num_post;
  p.barrier = reinterpret_cast<int*>(wsb);
  p.hist = reinterpret_cast<int32_t*>(wsb + 256);
  p.status = status;
  p.timeout_ns = moe::kDefaultTimeoutNs;
  p.expected = grid;
  moe::RouteExtra r;
  r.logits = logits;
  r.bias = bias;
  r.select_only = select_only ? 1 : 0;
  r.T = s.T;
  r.k = s.k - n_shared;
  r.E_routed = s.E - n_shared;
  r.n_shared = n_shared;
  r.ids_out = ids;
  r.w_out = w;
  r.plan = plan;
  r.tn = s.tn;
  r.nw_gu = s.I / 128;
  r.nw_dn = (s.H + 255) / 256;
  r.zero_out = nullptr;
  r.zero_n = 0;
  if (zero_out) {
    // the few-slot routing kernel (one CTA) zeroes a small buffer; otherwise
    // a memset does (spread over the GPU)
    if (moe::route_zeroes(N) && zero_n <= kRouteZeroMaxFloats) {
      r.zero_out = zero_out;
      r.zero_n = zero_n;
    } else {
      MOE_CU(cudaMemsetAsync(zero_out, 0, (size_t)zero_n * sizeof(float), stream));
    }
  }
  if (grid > 1 && !moe::route_zeroes(N)) MOE_CU(cudaMemsetAsync(p.barrier, 0, sizeof(int), stream));
  MOE_CU(moe::launch_route(p, r, grid, stream));
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(int s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
    default: return "MOE_ERR_UNKNOWN";
  }
}

const char* moe_last_cuda_error(void) { return g_last_cuda_error.c_str(); }

int moe_version(void) { return MOE_ABI_VERSION; }

moe_status_t moe_topk_gate(const float* logits, const float* bias, int bias_mode, int T, int E, int k,
                           int n_shared, int32_t* topk_ids, float* topk_w, void* stream) {
  NvtxRange nvtx_("moe_topk_gate");
  if (T < 0 || E < 1 || k < 1 || k > E || n_shared < 0 || k + n_shared > 32 || E + n_shared > 1024)
    return MOE_ERR_INVALID_ARG;
  if (bias_mode != MOE_BIAS_LOGITS && bias_mode != MOE_BIAS_SELECT) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_ids || !topk_w)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  moe_status_t st = check_device();
  if (st) return st;
  MOE_CU(moe::launch_topk_gate(logits, bias, bias_mode == MOE_BIAS_SELECT, T, E, k, n_shared, topk_ids, topk_w,
                               (cudaStream_t)stream));
  return MOE_OK;
}

moe_status_t moe_align_sort_sizes(int T, int k, int E, int block_size, size_t* P, size_t* NB, size_t* ws_bytes) {
  if (!align_args_ok(T, k, E, block_size)) return MOE_ERR_INVALID_ARG;
  const long long p = (long long)T * k + (long long)E * (block_size - 1);
  if (P) *P = (size_t)p;
  if (NB) *NB = (size_t)((p + block_size - 1) / block_size);
  if (ws_bytes) *ws_bytes = align_ws_bytes(E);
  return MOE_OK;
}

moe_status_t moe_align_sort(const int32_t* topk_ids, int T, int k, int E, int block_size, int32_t* sorted_ids,
                            int32_t* expert_ids, int32_t* num_post, void* ws, size_t ws_bytes,
                            int32_t* dev_status, void* stream) {
  NvtxRange nvtx_("moe_align_sort");
  if (!align_args_ok(T, k, E, block_size)) return MOE_ERR_INVALID_ARG;
  if (!sorted_ids || !expert_ids || !num_post || !ws || (T > 0 && !topk_ids)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < align_ws_bytes(E)) return MOE_ERR_WORKSPACE;
  moe_status_t st = check_device();
  if (st) return st;
  return run_align(topk_ids, T, k, E, block_size, sorted_ids, expert_ids, num_post, ws, dev_status,
                   (cudaStream_t)stream);
}

moe_status_t moe_ffn_workspace(const moe_ffn_args* a, size_t* ws_bytes) {
  if (!a || !ws_bytes) return MOE_ERR_INVALID_ARG;
  FfnShape s;
  moe_status_t st = ffn_shape(a->T, a->H, a->I, a->E, a->k, a->block_size, a->wdtype, a->tile_tokens, &s);
  if (st) return st;
  *ws_bytes = ffn_ws_layout(s).total;
  return MOE_OK;
}

moe_status_t moe_grouped_ffn(const moe_ffn_args* a, float* y, void* ws, size_t ws_bytes, int32_t* dev_status,
                             void* stream) {
  NvtxRange nvtx_("moe_grouped_ffn");
  if (!a) return MOE_ERR_INVALID_ARG;
  FfnShape s;
  moe_status_t st = ffn_shape(a->T, a->H, a->I, a->E, a->k, a->block_size, a->wdtype, a->tile_tokens, &s);
  if (st) return st;
  if (s.N == 0) return MOE_OK;
  if (!a->x || !a->w13 || !a->w2 || !a->sorted_ids || !a->expert_ids || !a->num_post || !y || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!weights_ok(s, a->w13, a->w13_scale, a->w2, a->w2_scale, a->w13_mx_scale, a->w2_mx_scale))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(a->x) || !aligned16(y) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ffn_ws_layout(s).total) return MOE_ERR_WORKSPACE;
  st = check_device();
  if (st) return st;
  const FfnWeights W = {a->w13, a->w13_scale, a->w2, a->w2_scale, a->w13_mx_scale, a->w2_mx_scale};
  return run_ffn(s, a->x, W, a->sorted_ids, a->expert_ids, a->num_post, y, static_cast<uint8_t*>(ws), dev_status,
                 (cudaStream_t)stream);
}

moe_status_t moe_combine(const float* y, const float* topk_w, int T, int k, int H, void* out, int out_dtype,
                         void* stream) {
  NvtxRange nvtx_("moe_combine");
  if (T < 0 || k < 1 || H < 1 || H % 4) return MOE_ERR_INVALID_ARG;
  if (out_dtype != MOE_BF16 && out_dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!y || !topk_w || !out || !aligned16(y) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st) return st;
  MOE_CU(moe::launch_combine(y, topk_w, T, k, H, out, out_dtype == MOE_BF16, (cudaStream_t)stream));
  return MOE_OK;
}

namespace {
// The combine is fused into the down GEMM's epilogue when a token has at
// least this many slots (then the per-slot outputs are >= 4x the token
// outputs).  With fewer slots the per-slot round trip is small, and the down
// GEMM's re-read operands (h, weights) need L2 more than an fp32 token
// accumulator does (measured: Mixtral, k = 2, is faster unfused; DeepSeek-V3,
// k = 8, fused).
constexpr int kFuseCombineMinSlots = 4;

bool fuse_combine(const FfnShape& s) { return s.k >= kFuseCombineMinSlots; }

struct FwdWs {
  size_t ids, w, sorted, eids, npost, align, ffn, acc, y, total;
};
FwdWs fwd_ws_layout(const FfnShape& s, int out_dtype) {
  Carver c;
  FwdWs w;
  w.ids = c.take((size_t)s.N * 4);
  w.w = c.take((size_t)s.N * 4);
  w.sorted = c.take((size_t)s.P * 4);
  w.eids = c.take((size_t)s.NB * 4);
  w.npost = c.take(4);
  w.align = c.take(align_ws_bytes(s.E));
  w.ffn = c.take(ffn_ws_layout(s).total);
  // fused combine: fp32 token accumulator (the output itself when it is f32);
  // otherwise one fp32 row per slot for the combine kernel
  const bool fused = fuse_combine(s);
  w.acc = c.take(fused && out_dtype == MOE_BF16 ? (size_t)s.T * s.H * 4 : 0);
  w.y = c.take(fused ? 0 : (size_t)s.N * s.H * 4);
  w.total = c.off;
  return w;
}
}  // namespace

// Shape of a forward call: the shared experts count as experts and as slots.
moe_status_t forward_shape(const moe_forward_args* a, FfnShape* s) {
  if (a->out_dtype != MOE_BF16 && a->out_dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (a->bias_mode != MOE_BIAS_LOGITS && a->bias_mode != MOE_BIAS_SELECT) return MOE_ERR_INVALID_ARG;
  if (a->n_shared < 0 || a->E < 1 || a->k < 1 || a->k > a->E || a->k + a->n_shared > 32 ||
      a->E + a->n_shared > 1024)
    return MOE_ERR_INVALID_ARG;
  return ffn_shape(a->T, a->H, a->I, a->E + a->n_shared, a->k + a->n_shared, a->block_size, a->wdtype,
                   a->tile_tokens, s);
}

moe_status_t moe_forward_workspace(const moe_forward_args* a, size_t* ws_bytes) {
  if (!a || !ws_bytes) return MOE_ERR_INVALID_ARG;
  FfnShape s;
  moe_status_t st = forward_shape(a, &s);
  if (st) return st;
  *ws_bytes = fwd_ws_layout(s, a->out_dtype).total;
  return MOE_OK;
}

moe_status_t moe_forward(const moe_forward_args* a, void* ws, size_t ws_bytes, int32_t* dev_status,
                         void* stream) {
  NvtxRange nvtx_("moe_forward");
  if (!a) return MOE_ERR_INVALID_ARG;
  FfnShape s;
  moe_status_t st = forward_shape(a, &s);
  if (st) return st;
  if (s.T == 0) return MOE_OK;
  if (!a->x || !a->logits || !a->out || !ws) return MOE_ERR_INVALID_ARG;
  if (!weights_ok(s, a->w13, a->w13_scale, a->w2, a->w2_scale, a->w13_mx_scale, a->w2_mx_scale))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(a->x) || !aligned16(a->out) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  const FwdWs L = fwd_ws_layout(s, a->out_dtype);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  st = check_device();
  if (st) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* ids = a->topk_ids ? a->topk_ids : reinterpret_cast<int32_t*>(w + L.ids);
  float* tw = a->topk_w ? a->topk_w : reinterpret_cast<float*>(w + L.w);
  int32_t* sorted = reinterpret_cast<int32_t*>(w + L.sorted);
  int32_t* eids = reinterpret_cast<int32_t*>(w + L.eids);
  int32_t* npost = reinterpret_cast<int32_t*>(w + L.npost);
  void** ev = a->stage_events;
  const bool out_bf16 = a->out_dtype == MOE_BF16;
  const bool fused = fuse_combine(s);
  float* out32 = !fused ? nullptr : out_bf16 ? reinterpret_cast<float*>(w + L.acc) : static_cast<float*>(a->out);
  float* y = fused ? nullptr : reinterpret_cast<float*>(w + L.y);
  MOE_CU(record(ev, 0, cs));
  // gate, align&sort and the GEMM tile plan are one launch: stages 0..2 end together
  uint8_t* ffn_ws = w + L.ffn;
  int32_t* plan = reinterpret_cast<int32_t*>(ffn_ws + ffn_ws_layout(s).plan);
  {
    NvtxRange nr("moe: route (gate, align & sort, plan)");
    // the fused combine's fp32 accumulator is zeroed by the routing step
    st = run_route(s, a->n_shared, a->bias_mode == MOE_BIAS_SELECT, a->logits, a->bias, ids, tw, sorted, eids,
                   npost, w + L.align, plan, dev_status, cs, fused ? out32 : nullptr,
                   fused ? (long long)s.T * s.H : 0);
  }
  if (st) return st;
  MOE_CU(record(ev, MOE_STAGE_GATE + 1, cs));
  MOE_CU(record(ev, MOE_STAGE_ALIGN + 1, cs));
  // fused: the down GEMM adds w * y of every slot into its token's fp32 row;
  // otherwise it writes y per slot and the combine kernel sums them
  const FfnWeights W = {a->w13, a->w13_scale, a->w2, a->w2_scale, a->w13_mx_scale, a->w2_mx_scale};
  st = run_ffn(s, a->x, W, sorted, eids, npost, y, ffn_ws, dev_status, cs, ev, /*plan_ready=*/true, out32, tw);
  if (st) return st;
  NvtxRange nr_combine("moe: combine");
  if (fused) {
    if (out_bf16) MOE_CU(moe::launch_cast_bf16(out32, (long long)s.T * s.H, a->out, cs));
  } else {
    MOE_CU(moe::launch_combine(y, tw, s.T, s.k, s.H, a->out, out_bf16, cs));
  }
  MOE_CU(record(ev, MOE_STAGE_COMBINE + 1, cs));
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// backward
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

struct BwdWs {
  size_t ids, w, sorted, eids, npost, align, plan, X, D, Z, hw, dgu, dwt, total;
};

moe_status_t bwd_shape(const moe_backward_args* a, FfnShape* s) {
  if (a->bias_mode != MOE_BIAS_LOGITS && a->bias_mode != MOE_BIAS_SELECT) return MOE_ERR_INVALID_ARG;
  if (a->n_shared < 0 || a->E < 1 || a->k < 1 || a->k > a->E || a->k + a->n_shared > 32 ||
      a->E + a->n_shared > 1024)
    return MOE_ERR_INVALID_ARG;
  moe_status_t st = ffn_shape(a->T, a->H, a->I, a->E + a->n_shared, a->k + a->n_shared, a->block_size, MOE_BF16,
                              0, s);
  if (st) return st;
  // the weight gradients multiply whole 16-row MMA steps of an expert's segment
  if (a->block_size % 16) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

BwdWs bwd_ws_layout(const FfnShape& s) {
  Carver c;
  BwdWs w;
  w.ids = c.take((size_t)s.N * 4);
  w.w = c.take((size_t)s.N * 4);
  w.sorted = c.take((size_t)s.P * 4);
  w.eids = c.take((size_t)s.NB * 4);
  w.npost = c.take(4);
  w.align = c.take(align_ws_bytes(s.E));
  w.plan = c.take((size_t)moe::plan_ints(s.E) * 4);
  w.X = c.take((size_t)s.P * s.H * 2);     // x rows in sorted order (bf16; padding rows zero)
  w.D = c.take((size_t)s.P * s.H * 2);     // dout rows in sorted order
  w.Z = c.take((size_t)s.P * s.I * 4);     // z = D . Wd (fp32)
  w.hw = c.take((size_t)s.P * s.I * 2);    // w * h (bf16)
  w.dgu = c.take((size_t)s.P * s.I * 4);   // [dg; du] (bf16, 2I per row)
  w.dwt = c.take((size_t)s.N * 4);         // combine-weight gradient per slot
  w.total = c.off;
  return w;
}

moe_status_t bwd_fail(int r, const char* what) {
  if (r == -1) {
    g_last_cuda_error = std::string(what) + ": cuTensorMapEncodeTiled failed";
    return MOE_ERR_CUDA;
  }
  return cuda_fail((cudaError_t)r, what);
}

}  // namespace

extern "C" {

moe_status_t moe_backward_workspace(const moe_backward_args* a, size_t* ws_bytes) {
  if (!a || !ws_bytes) return MOE_ERR_INVALID_ARG;
  FfnShape s;
  moe_status_t st = bwd_shape(a, &s);
  if (st) return st;
  *ws_bytes = bwd_ws_layout(s).total;
  return MOE_OK;
}

moe_status_t moe_backward(const moe_backward_args* a, void* ws, size_t ws_bytes, int32_t* dev_status,
                          void* stream) {
  NvtxRange nvtx_("moe_backward");
  if (!a) return MOE_ERR_INVALID_ARG;
  FfnShape s;
  moe_status_t st = bwd_shape(a, &s);
  if (st) return st;
  if (!a->w13 || !a->w2 || !a->dw13 || !a->dw2) return MOE_ERR_INVALID_ARG;
  if (!aligned16(a->w13) || !aligned16(a->w2) || !aligned16(a->dw13) || !aligned16(a->dw2))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t cs = (cudaStream_t)stream;
  const size_t EW = (size_t)s.E;
  if (s.T == 0) {
    st = check_device();
    if (st) return st;
    MOE_CU(cudaMemsetAsync(a->dw13, 0, EW * 2 * s.I * s.H * 4, cs));
    MOE_CU(cudaMemsetAsync(a->dw2, 0, EW * s.H * s.I * 4, cs));
    return MOE_OK;
  }
  if (!a->x || !a->logits || !a->dout || !a->dx || !a->dlogits || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(a->x) || !aligned16(a->dout) || !aligned16(a->dx) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  const BwdWs L = bwd_ws_layout(s);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  st = check_device();
  if (st) return st;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* ids = reinterpret_cast<int32_t*>(w + L.ids);
  float* tw = reinterpret_cast<float*>(w + L.w);
  int32_t* sorted = reinterpret_cast<int32_t*>(w + L.sorted);
  int32_t* eids = reinterpret_cast<int32_t*>(w + L.eids);
  int32_t* npost = reinterpret_cast<int32_t*>(w + L.npost);
  int32_t* plan = reinterpret_cast<int32_t*>(w + L.plan);
  void* X = w + L.X;
  void* D = w + L.D;
  float* Z = reinterpret_cast<float*>(w + L.Z);
  __nv_bfloat16* hw = reinterpret_cast<__nv_bfloat16*>(w + L.hw);
  __nv_bfloat16* dgu = reinterpret_cast<__nv_bfloat16*>(w + L.dgu);
  float* dwt = reinterpret_cast<float*>(w + L.dwt);
  const int N = (int)s.N, R = (int)s.rows_max;
  const int ks = s.k, kr = a->k;   // slots per token, routed choices

  // routing (gate + align & sort + tile plan), then the token rows in sorted order
  st = run_route(s, a->n_shared, a->bias_mode == MOE_BIAS_SELECT, a->logits, a->bias, ids, tw, sorted, eids, npost,
                 w + L.align, plan, dev_status, cs);
  if (st) return st;
  MOE_CU(moe::launch_gather_rows(a->x, nullptr, sorted, npost, R, N, ks, s.H * 2, X, nullptr, cs));
  MOE_CU(moe::launch_gather_rows(a->dout, nullptr, sorted, npost, R, N, ks, s.H * 2, D, nullptr, cs));

  moe::BwdLaunch g = {};
  g.p.E = s.E;
  g.p.k = ks;
  g.p.n_slots = N;
  g.p.plan = plan;
  g.p.sorted = sorted;
  g.p.status = dev_status;
  g.p.timeout_ns = moe::kDefaultTimeoutNs;
  g.p.tn = s.tn;
  // z = D . Wd (Wd read transposed)
  moe::BwdLaunch gz = g;
  gz.a = a->w2; gz.a_rows = (long long)EW * s.H; gz.a_cols = s.I;
  gz.b = D; gz.b_rows = s.P; gz.b_cols = s.H;
  gz.p.kind = moe::BWD_Z; gz.p.K = s.H; gz.p.n_out = s.I; gz.p.out = Z;
  int r = moe::launch_bwd_gemm(gz, cs);
  if (r) return bwd_fail(r, "backward z GEMM");
  // gate/up recomputed with the SwiGLU backward in the epilogue (padding rows of hw / dgu stay zero)
  MOE_CU(cudaMemsetAsync(hw, 0, (size_t)s.P * s.I * 2, cs));
  MOE_CU(cudaMemsetAsync(dgu, 0, (size_t)s.P * s.I * 4, cs));
  MOE_CU(cudaMemsetAsync(dwt, 0, (size_t)N * 4, cs));
  moe::BwdLaunch gg = g;
  gg.a = a->w13; gg.a_rows = (long long)EW * 2 * s.I; gg.a_cols = s.H;
  gg.b = X; gg.b_rows = s.P; gg.b_cols = s.H;
  gg.p.kind = moe::BWD_GUB; gg.p.K = s.H; gg.p.n_out = s.I;
  gg.p.topk_w = tw; gg.p.zbuf = Z; gg.p.hw = hw; gg.p.dgu = dgu; gg.p.dwt = dwt;
  r = moe::launch_bwd_gemm(gg, cs);
  if (r) return bwd_fail(r, "backward gate/up GEMM");
  // dx: per slot dgu . W13 (W13 read transposed), added into the token's row
  MOE_CU(cudaMemsetAsync(a->dx, 0, (size_t)s.T * s.H * 4, cs));
  moe::BwdLaunch gx = g;
  gx.a = a->w13; gx.a_rows = (long long)EW * 2 * s.I; gx.a_cols = s.H;
  gx.b = dgu; gx.b_rows = s.P; gx.b_cols = 2 * s.I;
  gx.p.kind = moe::BWD_DX; gx.p.K = 2 * s.I; gx.p.n_out = s.H; gx.p.dx = a->dx;
  r = moe::launch_bwd_gemm(gx, cs);
  if (r) return bwd_fail(r, "backward dx GEMM");
  // router logits
  MOE_CU(moe::launch_dlogits(ids, tw, dwt, s.T, a->E, kr, ks, a->dlogits, cs));
  // weight gradients, per expert over its sorted rows
  moe::BwdLaunch g2 = g;
  g2.a = D; g2.a_rows = s.P; g2.a_cols = s.H;
  g2.b = hw; g2.b_rows = s.P; g2.b_cols = s.I;
  g2.p.kind = moe::BWD_WG; g2.p.n_out = s.H; g2.p.n_cols = s.I; g2.p.out = a->dw2;
  g2.p.tn = s.I % 256 == 0 ? 256 : 128;
  r = moe::launch_bwd_gemm(g2, cs);
  if (r) return bwd_fail(r, "backward dW2 GEMM");
  moe::BwdLaunch g13 = g;
  g13.a = dgu; g13.a_rows = s.P; g13.a_cols = 2 * s.I;
  g13.b = X; g13.b_rows = s.P; g13.b_cols = s.H;
  g13.p.kind = moe::BWD_WG; g13.p.n_out = 2 * s.I; g13.p.n_cols = s.H; g13.p.out = a->dw13;
  g13.p.tn = s.H % 256 == 0 ? 256 : 128;
  r = moe::launch_bwd_gemm(g13, cs);
  if (r) return bwd_fail(r, "backward dW13 GEMM");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// expert parallelism: routing of slots to ranks, row permutations
// ---------------------------------------------------------------------------
static size_t ep_ws_layout(long long N, int R, size_t* dest, size_t* eids, size_t* npost, size_t* align) {
  Carver c;
  *dest = c.take((size_t)N * 4);
  *eids = c.take((size_t)N * 4);
  *npost = c.take(4);
  *align = c.take(align_ws_bytes(R));
  return c.off;
}

moe_status_t moe_ep_route_workspace(int T, int k, int R, size_t* ws_bytes) {
  if (!ws_bytes || !align_args_ok(T, k, R, 1)) return MOE_ERR_INVALID_ARG;
  size_t a, b, c, d;
  *ws_bytes = ep_ws_layout((long long)T * k, R, &a, &b, &c, &d);
  return MOE_OK;
}

moe_status_t moe_ep_route(const int32_t* topk_ids, int T, int k, int E, int R, int32_t* order, int32_t* send_counts,
                          int32_t* local_ids, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  NvtxRange nvtx_("moe_ep_route");
  if (!align_args_ok(T, k, R, 1) || E < R || E % R) return MOE_ERR_INVALID_ARG;
  if (!send_counts || (T > 0 && (!topk_ids || !order || !local_ids || !ws))) return MOE_ERR_INVALID_ARG;
  const long long N = (long long)T * k;
  size_t o_dest, o_eids, o_np, o_al;
  if (ws_bytes < ep_ws_layout(N, R, &o_dest, &o_eids, &o_np, &o_al) && T > 0) return MOE_ERR_WORKSPACE;
  moe_status_t st = check_device();
  if (st) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  MOE_CU(cudaMemsetAsync(send_counts, 0, (size_t)R * 4, cs));
  if (T == 0) return MOE_OK;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* dest = reinterpret_cast<int32_t*>(w + o_dest);
  MOE_CU(moe::launch_ep_dest(topk_ids, (int)N, E, E / R, dest, send_counts, dev_status, cs));
  // slots in destination-rank order: align & sort with the ranks as experts and blocks of one slot
  st = run_align(dest, T, k, R, 1, order, reinterpret_cast<int32_t*>(w + o_eids),
                 reinterpret_cast<int32_t*>(w + o_np), w + o_al, dev_status, cs);
  if (st) return st;
  MOE_CU(moe::launch_ep_local_ids(topk_ids, order, (int)N, E / R, local_ids, cs));
  return MOE_OK;
}

moe_status_t moe_permute_rows(const void* src, int row_bytes, const int32_t* map, int n, int div, int src_rows,
                              void* dst, void* stream) {
  if (n < 0 || div < 1 || src_rows < 0 || row_bytes <= 0 || row_bytes % 16) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (!src || !map || !dst || !aligned16(src) || !aligned16(dst)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st) return st;
  MOE_CU(moe::launch_permute_rows(src, row_bytes, map, n, div, src_rows, false, dst, (cudaStream_t)stream));
  return MOE_OK;
}

moe_status_t moe_scatter_rows(const void* src, int row_bytes, const int32_t* map, int n, int dst_rows, void* dst,
                              void* stream) {
  if (n < 0 || dst_rows < 0 || row_bytes <= 0 || row_bytes % 16) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (!src || !map || !dst || !aligned16(src) || !aligned16(dst)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st) return st;
  MOE_CU(moe::launch_permute_rows(src, row_bytes, map, n, 1, dst_rows, true, dst, (cudaStream_t)stream));
  return MOE_OK;
}

moe_status_t moe_mx_tile_scales(const uint8_t* sf, long long rows, int K, uint8_t* out, void* stream) {
  if (rows < 0 || K < 0 || rows % 128 || K % 128) return MOE_ERR_INVALID_ARG;
  if (rows == 0 || K == 0) return MOE_OK;
  if (!sf || !out || !aligned16(sf) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st) return st;
  MOE_CU(moe::launch_mx_tile_scales(sf, rows, K, out, (cudaStream_t)stream));
  return MOE_OK;
}

moe_status_t moe_mx_quantize_rows(const void* x, int R, int C, uint8_t* codes, uint8_t* scales, void* stream) {
  if (R < 0 || C < 0 || C % 32) return MOE_ERR_INVALID_ARG;
  if (R == 0 || C == 0) return MOE_OK;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(codes)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st) return st;
  MOE_CU(moe::launch_mx_quant_rows(x, nullptr, 0, 1, nullptr, R, C, codes, scales, (cudaStream_t)stream));
  return MOE_OK;
}

moe_status_t moe_test_wait_timeout(void* ws, int32_t* dev_status, long long timeout_ns, void* stream) {
  if (!ws || !dev_status || timeout_ns < 0) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  MOE_CU(cudaMemsetAsync(ws, 0, sizeof(int), cs));
  MOE_CU(moe::launch_wait_timeout(static_cast<int*>(ws), dev_status, timeout_ns, cs));
  return MOE_OK;
}

moe_status_t moe_test_quant_division(void* ws, void* stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  MOE_CU(cudaMemsetAsync(ws, 0, 32, cs));
  unsigned long long* counts = static_cast<unsigned long long*>(ws);
  MOE_CU(moe::launch_quant_division_check(counts, reinterpret_cast<unsigned int*>(counts + 2), cs));
  return MOE_OK;
}

}  // extern "C"
