// Kernel parameter blocks and launchers shared by the host API (api.cu).
#pragma once
#include "common.cuh"

namespace moe {

// Records "where: CUDA error text" for moe_last_cuda_error (this host thread)
// and returns MOE_ERR_CUDA.
moe_status_t record_cuda_error(cudaError_t e, const char* where);

struct AlignParams {
  const int32_t* ids;
  int N;            // T*k flat slots
  int E;
  int bm;
  int chunk;        // slots per CTA: a multiple of 32 and of the slots per token
  int32_t* sorted;
  int32_t* expert_ids;
  int32_t* num_post;
  int32_t* hist;    // [E][gridDim.x] per-CTA counts
  int* barrier;     // zeroed before launch
  int32_t* status;
  long long timeout_ns;
  int expected;     // arrivals to wait for (gridDim.x; larger only in the timeout test)
};

// Extra inputs of the fused routing launch (gating in front, tile plan behind).
struct RouteExtra {
  const float* logits;  // [T, E_routed]
  const float* bias;    // [E_routed] or null
  int select_only;      // the bias steers the selection only
  int T, k;             // tokens, routed choices per token
  int E_routed;         // routed experts; AlignParams::E = E_routed + n_shared
  int n_shared;         // shared experts (every token, weight 1)
  int32_t* ids_out;     // [T*(k+n_shared)] (the same buffer AlignParams::ids reads)
  float* w_out;         // [T*(k+n_shared)]
  int32_t* plan;        // plan layout below
  int tn, nw_gu, nw_dn;
  float* zero_out;      // few-slot routing only (route_zeroes(N)): zeroes [zero_n] floats
  long long zero_n;     // (a multiple of 4, 16-byte aligned), e.g. the fused combine's accumulator
};

size_t align_smem_bytes(int E);
cudaError_t launch_align_sort(const AlignParams& p, int grid, cudaStream_t stream);
// gate + align&sort + tile plan in one cooperative launch (p.chunk % (k + n_shared) == 0)
cudaError_t launch_route(const AlignParams& p, const RouteExtra& r, int grid, cudaStream_t stream);
// whether launch_route takes the few-slot kernel for N slots (which also
// zeroes RouteExtra::zero_out)
bool route_zeroes(long long N);
int align_max_ctas(int E, int* err_out);
cudaError_t launch_wait_timeout(int* counter, int32_t* status, long long timeout_ns, cudaStream_t stream);

// ids/w rows of k + n_shared entries (the shared experts E.. with weight 1)
cudaError_t launch_topk_gate(const float* logits, const float* bias, bool select_only, int T, int E, int k,
                             int n_shared, int32_t* ids, float* w, cudaStream_t s);
// dst row r < min(*num_post, P) = src row sorted[r]/k (row_bytes each, a
// multiple of 16), zero for padding (an id outside [0, N)); with scales also
// dst_scale[r] = src_scale[token] (1 for padding)
cudaError_t launch_gather_rows(const void* src, const float* src_scale, const int32_t* sorted,
                               const int32_t* num_post, int P, int N, int k, int row_bytes, void* dst,
                               float* dst_scale, cudaStream_t s);
// per-row E4M3 quantisation of bf16 rows of length C: rows
// [0, min(*nrows_dev, nrows)) (or [0, nrows) when nrows_dev is null) of
// src [.., C] -> E4M3 codes + fp32 scales.  With `sorted`, row r quantises
// token sorted[r] / k (gather) or src row r, and padding rows (an id outside
// [0, N)) are not written.
cudaError_t launch_quant_rows(const void* src, const int32_t* sorted, bool gather, int N, int k,
                              const int32_t* nrows_dev, int nrows, int C, void* q, float* scale, int32_t* status,
                              cudaStream_t s);
// MXFP8 quantisation of bf16 rows of length C (C % 32 == 0): E4M3 codes
// [rows, C] and E8M0 scales [rows, C/32]; rows and the gather row map as in
// launch_quant_rows (padding rows: zero codes, scale code 127)
cudaError_t launch_mx_quant_rows(const void* src, const int32_t* sorted, int N, int k, const int32_t* nrows_dev,
                                 int nrows, int C, void* codes, uint8_t* scales, cudaStream_t s);
// per-row E8M0 scales [rows, K/32] -> tiled chunks (rows % 128 == 0, K % 128 == 0)
cudaError_t launch_mx_tile_scales(const uint8_t* in, long long rows, int K, uint8_t* out, cudaStream_t s);
cudaError_t launch_quant_division_check(unsigned long long* counts, unsigned int* first_bad, cudaStream_t s);
cudaError_t launch_cast_bf16(const float* src, long long n, void* dst, cudaStream_t s);
// expert parallelism: dest[i] = ids[i] / E_loc, counts[dest] += 1 (counts zeroed by the caller)
cudaError_t launch_ep_dest(const int32_t* ids, int N, int E, int E_loc, int32_t* dest, int32_t* counts,
                           int32_t* status, cudaStream_t s);
// local_ids[i] = ids[order[i]] % E_loc
cudaError_t launch_ep_local_ids(const int32_t* ids, const int32_t* order, int N, int E_loc, int32_t* local_ids,
                                cudaStream_t s);
// gather: dst row i = src row map[i] / div; scatter: dst row map[i] / div = src row i (rows of row_bytes,
// a multiple of 16; map entries whose row falls outside [0, limit) move nothing)
cudaError_t launch_permute_rows(const void* src, int row_bytes, const int32_t* map, int n, int div, int limit,
                                bool scatter, void* dst, cudaStream_t s);
cudaError_t launch_combine(const float* y, const float* w, int T, int k, int H, void* out, bool bf16,
                           cudaStream_t s);

// Plan layout (int32, written by the routing kernel or plan_kernel, see plan.cuh):
//   [0] gate/up tiles  [1] down tiles  [2] tokens per tile  [3] padded rows
//   [4] gate/up tiles of the hot experts  [5] down tiles of the hot experts
//   [6] gate/up tile counter  [7] down tile counter (zeroed by the writer,
//       advanced by the GEMM launches as they claim tiles)
//   seg_start[E] @8, seg_rows[E] @8+E (padded), groups[E] @8+2E (by expert),
//   perm[E] @8+3E (expert at each list position: hot experts first),
//   pref_gu[E+1] @8+4E, pref_dn[E+1] @9+5E (tile prefix by list position),
//   seg_real[E] @10+6E (slots of the expert: its segment's rows that are not
//   padding, which come first in the segment)
enum {
  PLAN_TILES_GU = 0, PLAN_TILES_DN = 1, PLAN_TN = 2, PLAN_NUM_POST = 3, PLAN_HOT_GU = 4, PLAN_HOT_DN = 5,
  PLAN_COUNTER_GU = 6, PLAN_COUNTER_DN = 7, PLAN_HEADER = 8
};
__host__ __device__ inline int plan_ints(int E) { return 10 + 7 * E; }
__host__ __device__ inline int plan_start(int) { return PLAN_HEADER; }
__host__ __device__ inline int plan_rows(int E) { return PLAN_HEADER + E; }
__host__ __device__ inline int plan_groups(int E) { return PLAN_HEADER + 2 * E; }
__host__ __device__ inline int plan_perm(int E) { return PLAN_HEADER + 3 * E; }
__host__ __device__ inline int plan_pref(int E, bool gateup) { return gateup ? PLAN_HEADER + 4 * E : PLAN_HEADER + 5 * E + 1; }
__host__ __device__ inline int plan_real(int E) { return PLAN_HEADER + 6 * E + 2; }
__host__ __device__ inline int plan_counter(int, bool gateup) { return gateup ? PLAN_COUNTER_GU : PLAN_COUNTER_DN; }
cudaError_t launch_plan(const int32_t* expert_ids, const int32_t* num_post, const int32_t* sorted, int N, int P,
                        int E, int bm, int tn, int nw_gu, int nw_dn, int32_t* plan, int32_t* status, cudaStream_t s);

struct GemmParams {
  int gateup;          // 1: gate/up with SiLU*mul epilogue, 0: down projection
  int fp8;             // E4M3 operands (kind::f8f6f4) instead of bf16 (kind::f16)
  int K;               // reduction length (elements)
  int n_out;           // output features per expert: I (gate/up) or H (down)
  int tn;              // token tile (MMA N), multiple of 16, <= 256
  int stages;
  int n_acc;           // TMEM accumulator buffers
  int tmem_cols;       // allocated TMEM columns (power of two)
  int E;
  int n_slots;         // T*k
  int k;
  const int32_t* plan;
  const int32_t* sorted;
  const float* a_scale;  // [P] per sorted row (FP8)
  const float* w_scale;  // per weight row (FP8)
  void* out;             // gate/up: h bf16 [P, n_out]; down: y f32 [T*k, n_out] (one row per slot)
  int32_t* status;
  long long timeout_ns;
  int* tile_counter;     // next unclaimed tile of this launch (zero at launch)
  float* comb_out;       // down only, nullable: out32 [T, n_out] += comb_w[slot] * y instead of
  const float* comb_w;   //   writing y (top-k combine fused into the epilogue)
  // MX block-scaled operands (kind::mxf8f6f4 with E8M0 scales per 32 K-elements;
  // fp8 is 0 then, the scales are applied inside the MMA)
  int mx;                // 1: MX operands
  int w_fp4;             // MX weights are E2M1 codes packed two per byte (else E4M3)
  const uint8_t* w_sf;   // weight scales in the tiled layout of moe_mx_tile_scales
  const uint8_t* x_sf;   // activation scales [P, K/32]
  uint8_t* h_sf;         // gate/up: out holds E4M3 codes of h [P, n_out], these their scales [P, n_out/32]
};

struct GemmLaunch {
  const void* w;        // [E * w_rows_per_expert, K]
  long long w_rows;     // total weight rows
  const void* x;        // [P, K]
  long long x_rows;     // P
  GemmParams p;
};

// Backward GEMMs (bwd.cu): the tile kinds and their operands.
enum BwdKind {
  BWD_Z = 0,     // z [P, I] = D_r . Wd[e] (transposed weights): fp32 rows
  BWD_GUB = 1,   // gate/up recomputed; epilogue: SwiGLU backward -> dgu, w*h, combine-weight gradient
  BWD_DX = 2,    // dx [T, H] += dgu_r . W13[e] (transposed weights), fp32 additions per token
  BWD_WG = 3     // weight gradient of one expert: [M, N] = A^T B over its sorted token rows (fp32)
};
struct BwdParams {
  int kind;
  int K;              // reduction length (Z: H; GUB: H; DX: 2I; WG: the expert's rows)
  int n_out;          // M: output features (Z, GUB: I; DX: H) or rows of the weight gradient
  int n_cols;         // WG: columns of the weight gradient
  int tn;             // token tile (Z, GUB, DX) or column tile (WG, 128 or 256)
  int stages, n_acc, tmem_cols;
  int E, k, n_slots;
  const int32_t* plan;
  const int32_t* sorted;
  const float* topk_w;   // GUB: routing weights per slot
  const float* zbuf;     // GUB: z [P, I]
  float* out;            // Z: z [P, I]; WG: dW [E, n_out, n_cols]
  __nv_bfloat16* hw;     // GUB: w * h [P, I]
  __nv_bfloat16* dgu;    // GUB: [dg; du] [P, 2I]
  float* dwt;            // GUB: gradient of each slot's combine weight (atomic sums)
  float* dx;             // DX: [T, n_out] fp32
  int32_t* status;
  long long timeout_ns;
};
struct BwdLaunch {
  const void* a;             // A source [a_rows, a_cols] bf16 (K-major weights, or MN-major)
  long long a_rows, a_cols;
  const void* b;             // B source [b_rows, b_cols] bf16
  long long b_rows, b_cols;
  BwdParams p;
};
// returns 0 on success, -1 if a tensor map could not be encoded, else a cudaError_t
int launch_bwd_gemm(const BwdLaunch& L, cudaStream_t stream);
cudaError_t launch_dlogits(const int32_t* ids, const float* w, const float* dwt, int T, int E, int k, int kk,
                           float* dlogits, cudaStream_t s);

size_t gemm_smem_bytes(int tn, int stages, int E, bool mx);
int gemm_pick_stages(int tn, int E, bool mx);
// returns 0 on success, -1 if a tensor map could not be encoded, else a cudaError_t
int launch_grouped_gemm(GemmLaunch& L, cudaStream_t stream);

}  // namespace moe
