// Memory-bound steps of the MoE layer forward on sm_100a:
//   topk_gate      softmax top-k gating, one warp per token
//   gather_rows    token rows (bf16, or E4M3 codes + scale) into sorted
//                  (expert-grouped) order
//   quant_rows     per-row E4M3 quantisation (per-token activations, and the
//                  requantisation of h between the two GEMMs)
//   combine        top-k weighted sum of the per-slot expert outputs
#include <cfloat>

#include "gate.cuh"
#include "kernels.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Top-k gating, one warp per token (the per-token work is gate_token in
// gate.cuh).
// ---------------------------------------------------------------------------
template <int EPL>
__global__ void __launch_bounds__(256) topk_gate_kernel(const float* __restrict__ logits,
                                                        const float* __restrict__ bias, bool select_only, int T,
                                                        int E, int k, int n_shared, int32_t* __restrict__ ids,
                                                        float* __restrict__ w) {
  const long long t = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  gate_token<EPL>(logits, bias, select_only, t, E, k, n_shared, ids, w, threadIdx.x & 31);
}

cudaError_t launch_topk_gate(const float* logits, const float* bias, bool select_only, int T, int E, int k,
                             int n_shared, int32_t* ids, float* w, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int warps = 8;
  dim3 grid((unsigned)((T + warps - 1) / warps)), block(32 * warps);
  const int epl = (E + 31) / 32;
#define MOE_GATE(V) topk_gate_kernel<V><<<grid, block, 0, s>>>(logits, bias, select_only, T, E, k, n_shared, ids, w)
  if (epl <= 1) MOE_GATE(1);
  else if (epl <= 2) MOE_GATE(2);
  else if (epl <= 4) MOE_GATE(4);
  else if (epl <= 8) MOE_GATE(8);
  else if (epl <= 16) MOE_GATE(16);
  else MOE_GATE(32);
#undef MOE_GATE
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Gather of token rows into sorted order (MoE Align & Sort article,
// "FasterTransformer": permute before the group GEMM).  Row r of dst is the
// row of token sorted[r] / k (bf16 activations, or their E4M3 codes with the
// per-token scale); padding rows are zero (scale 1).  Rows >= num_post are not
// touched.  One warp per row, 16-byte vectors.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ src,
                                                          const float* __restrict__ src_scale,
                                                          const int32_t* __restrict__ sorted,
                                                          const int32_t* __restrict__ num_post, int P, int N,
                                                          int k, int vec, uint4* __restrict__ dst,
                                                          float* __restrict__ dst_scale) {
  const int np = min(*num_post, P);   // an invalid num_post (flagged by the plan) stays inside the buffers
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < np; r += gridDim.x * wpb) {
    const int slot = __ldg(sorted + r);
    const long long t = (unsigned)slot < (unsigned)N ? slot / k : -1;   // padding, or an invalid id: zeros
    const uint4* row = t >= 0 ? src + t * vec : nullptr;
    uint4* out = dst + (long long)r * vec;
    int c = lane;
    for (; c + 96 < vec; c += 128) {   // four independent 16-byte loads in flight per lane
      uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0, v2 = v0, v3 = v0;
      if (row) {
        v0 = __ldg(row + c);
        v1 = __ldg(row + c + 32);
        v2 = __ldg(row + c + 64);
        v3 = __ldg(row + c + 96);
      }
      out[c] = v0;
      out[c + 32] = v1;
      out[c + 64] = v2;
      out[c + 96] = v3;
    }
    for (; c < vec; c += 32) out[c] = row ? __ldg(row + c) : make_uint4(0, 0, 0, 0);
    if (dst_scale && lane == 0) dst_scale[r] = t >= 0 ? __ldg(src_scale + t) : 1.f;
  }
}

// ---------------------------------------------------------------------------
// Per-row E4M3 quantisation (aiter issue 1248: per-token FP8 activations;
// GC-MoE: requantisation between the GEMMs).  s = amax / 448 in fp32 (1 for
// an all-zero row); code = e4m3_rne_satfinite(v / s) with v / s the correctly
// rounded fp32 quotient.  One warp per row with the row held in registers (VPL
// 16-byte vectors of 8 bf16 per lane) below 4096 elements; longer rows are
// staged in shared memory by bulk copies (quant_rows_bulk_kernel), and rows
// too long for that (over 100K elements) take two passes.  With a row map the kernel also gathers (sorted row r quantises its
// token).
//
// The quotient comes from one reciprocal per row and a correction step per
// element (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Develop. 34(1), 1990): with r = RN(1/s)
// and q = RN(v r), the residual v - q s is exact under a fused multiply-add and
// RN(q + residual * r) = RN(v / s).  The residual is exact only while it does
// not underflow: for s >= 2^-90 that holds for every quotient of magnitude
// >= 2^-11, and smaller quotients all encode to a signed zero (their sign is
// carried over from q, since the sum can turn -0 into +0).  Rows with a
// smaller scale divide element by element.  moe_test_quant_division
// checks the resulting codes against a per-element IEEE division for every
// pair of bf16 values (v, amax) with |v| <= amax.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

struct RowScale {
  float s;     // the row's scale
  float r;     // RN(1 / s) when the correction step applies, else 0
};

__device__ __forceinline__ RowScale row_scale(float amax) {
  RowScale rs;
  rs.s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  rs.r = rs.s >= 0x1p-90f ? __frcp_rn(rs.s) : 0.f;
  return rs;
}

// RN(v / s): correction step (kFast, needs rs.r != 0) or IEEE division
template <bool kFast>
__device__ __forceinline__ float div_by_scale(float v, const RowScale& rs) {
  if (!kFast) return __fdiv_rn(v, rs.s);
  const float q = v * rs.r;
  const float res = fmaf(-q, rs.s, v);
  return copysignf(fmaf(res, rs.r, q), q);
}

// two quotients -> two E4M3 codes (a in the low byte)
__device__ __forceinline__ uint32_t e4m3_pack2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

template <bool kFast>
__device__ __forceinline__ uint32_t quant_pair(uint32_t u, const RowScale& rs) {
  return e4m3_pack2(div_by_scale<kFast>(bf16_lo(u), rs), div_by_scale<kFast>(bf16_hi(u), rs));
}

__device__ __forceinline__ float absmax8(const uint4& v) {
  return fmaxf(fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))), fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))),
               fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))), fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
}

template <bool kFast>
__device__ __forceinline__ uint2 quant8(const uint4& v, const RowScale& rs) {
  uint2 o;
  o.x = quant_pair<kFast>(v.x, rs) | (quant_pair<kFast>(v.y, rs) << 16);
  o.y = quant_pair<kFast>(v.z, rs) | (quant_pair<kFast>(v.w, rs) << 16);
  return o;
}

// the row's codes from n register-resident vectors v[i] -> dst[c0 + stride*i]
template <int V>
__device__ __forceinline__ void quant_store(const uint4 (&v)[V], const RowScale& rs, uint2* dst, int c0, int stride,
                                            int vec) {
  if (rs.r != 0.f) {
#pragma unroll
    for (int i = 0; i < V; ++i)
      if (c0 + stride * i < vec) dst[c0 + stride * i] = quant8<true>(v[i], rs);
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i)
      if (c0 + stride * i < vec) dst[c0 + stride * i] = quant8<false>(v[i], rs);
  }
}

// Source row of output row r.  Without a row map: src row r.  With the
// sorted slot ids as row map: the token sorted[r] / k (gather) or src row r,
// and -1 for a padding row (an id outside [0, N)), which is not written:
// nothing reads the codes of a padding row (the grouped GEMMs compute a
// padding row's column but store none of it).
__device__ __forceinline__ long long quant_src_row(const int32_t* sorted, bool gather, int r, int N, int k) {
  if (!sorted) return r;
  const int slot = __ldg(sorted + r);
  if ((unsigned)slot < (unsigned)N) return gather ? slot / k : r;
  return -1;
}

template <int VPL>
__global__ void __launch_bounds__(256) quant_rows_warp_kernel(const uint4* __restrict__ src,
                                                              const int32_t* __restrict__ sorted, bool gather,
                                                              int N, int k, const int32_t* __restrict__ nrows_dev,
                                                              int nrows, int vec, uint2* __restrict__ q,
                                                              float* __restrict__ scale) {
  const int n = nrows_dev ? min(*nrows_dev, nrows) : nrows;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < n; r += gridDim.x * wpb) {
    const long long sr = quant_src_row(sorted, gather, r, N, k);
    if (sr < 0) continue;
    uint2* dst = q + (long long)r * vec;
    const uint4* row = src + sr * vec;
    uint4 v[VPL];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int c = lane + 32 * i;
      v[i] = c < vec ? __ldg(row + c) : make_uint4(0, 0, 0, 0);
      amax = fmaxf(amax, absmax8(v[i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const RowScale rs = row_scale(amax);
    quant_store<VPL>(v, rs, dst, lane, 32, vec);
    if (lane == 0) scale[r] = rs.s;
  }
}

// Rows staged through shared memory: one warp per row, each warp with nb row
// buffers that lane 0 fills with 1-D bulk copies (completion on an mbarrier
// per buffer), so a warp keeps nb rows in flight without holding them in
// registers.  The row's amax is a warp max of the float bits (amax >= 0, so
// they order as integers; redux.sync), then each lane quantises its 16-byte
// vectors from shared memory.  Warp w of CTA c takes rows c*W + w + i*gridDim*W.
// A wait that runs out flags MOE_DEV_TIMEOUT, lets the warp's copies in flight
// land (bounded) and returns.
__global__ void __launch_bounds__(256, 1)
    quant_rows_bulk_kernel(const uint8_t* __restrict__ src, const int32_t* __restrict__ sorted, bool gather,
                           int N, int k,
                           const int32_t* __restrict__ nrows_dev, int nrows, int vec, int nb,
                           uint2* __restrict__ q, float* __restrict__ scale, int32_t* status,
                           long long timeout_ns) {
  extern __shared__ __align__(128) uint8_t smq[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, W = blockDim.x >> 5;
  const uint32_t row_bytes = (uint32_t)vec * 16u;
  uint8_t* buf = smq + (size_t)warp * nb * row_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smq + (size_t)W * nb * row_bytes) + warp * nb;
  const int n = nrows_dev ? min(*nrows_dev, nrows) : nrows;
  const int first = blockIdx.x * W + warp, stride = gridDim.x * W;
  if (lane == 0) {
    for (int b = 0; b < nb; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
  }
  __syncwarp();
  auto source = [&](int r) -> long long { return quant_src_row(sorted, gather, r, N, k); };
  // lane 0: the i-th row of this warp into buffer i % nb (a padding row only completes the phase)
  auto issue = [&](int i) {
    const int r = first + i * stride;
    if (r >= n) return;
    uint64_t* bar = &bars[i % nb];
    const long long sr = source(r);
    if (sr < 0) {
      mbar_arrive(bar);
      return;
    }
    mbar_arrive_expect_tx(bar, row_bytes);
    bulk_load(buf + (size_t)(i % nb) * row_bytes, src + sr * row_bytes, row_bytes, bar);
  };
  if (lane == 0)
    for (int i = 0; i < nb; ++i) issue(i);
  int i = 0;
  for (;; ++i) {
    const int r = first + i * stride;
    if (r >= n) break;
    const int b = i % nb;
    const bool ok = mbar_wait(&bars[b], (uint32_t)(i / nb) & 1u, timeout_ns);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) {
        dev_flag(status, MOE_DEV_TIMEOUT);
        // copies of rows i .. i+nb-1 may still be in flight: let them land
        for (int j = i; j < i + nb && first + j * stride < n; ++j)
          (void)mbar_wait(&bars[j % nb], (uint32_t)(j / nb) & 1u, 100000000LL);
      }
      __syncwarp();
      return;
    }
    const uint4* row = reinterpret_cast<const uint4*>(buf + (size_t)b * row_bytes);
    uint2* dst = q + (long long)r * vec;
    if (source(r) >= 0) {   // padding rows are not written
      float amax = 0.f;
      for (int c = lane; c < vec; c += 32) amax = fmaxf(amax, absmax8(row[c]));
      amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
      const RowScale rs = row_scale(amax);
      if (rs.r != 0.f)
        for (int c = lane; c < vec; c += 32) dst[c] = quant8<true>(row[c], rs);
      else
        for (int c = lane; c < vec; c += 32) dst[c] = quant8<false>(row[c], rs);
      if (lane == 0) scale[r] = rs.s;
    }
    __syncwarp();   // every lane is done with buffer b
    if (lane == 0) {
      fence_proxy_async();   // generic reads of the buffer before the bulk copy rewrites it
      issue(i + nb);
    }
  }
}

// Rows too long to stage (over 100K elements): one warp per row, two passes

// (the second pass re-reads the row from L1/L2).
__global__ void __launch_bounds__(256) quant_rows_2pass_kernel(const uint4* __restrict__ src,
                                                               const int32_t* __restrict__ sorted, bool gather,
                                                               int N, int k,
                                                               const int32_t* __restrict__ nrows_dev, int nrows,
                                                               int vec, uint2* __restrict__ q,
                                                               float* __restrict__ scale) {
  const int n = nrows_dev ? min(*nrows_dev, nrows) : nrows;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < n; r += gridDim.x * wpb) {
    const long long sr = quant_src_row(sorted, gather, r, N, k);
    if (sr < 0) continue;
    uint2* dst = q + (long long)r * vec;
    const uint4* row = src + sr * vec;
    float amax = 0.f;
    for (int c = lane; c < vec; c += 32) amax = fmaxf(amax, absmax8(__ldg(row + c)));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const RowScale rs = row_scale(amax);
    if (rs.r != 0.f)
      for (int c = lane; c < vec; c += 32) dst[c] = quant8<true>(__ldg(row + c), rs);
    else
      for (int c = lane; c < vec; c += 32) dst[c] = quant8<false>(__ldg(row + c), rs);
    if (lane == 0) scale[r] = rs.s;
  }
}

static int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// grid for one warp per row, 8 warps per CTA, at most 16 CTAs per SM
static int warp_rows_grid(long long rows) {
  const long long need = (rows + 7) / 8;
  const long long cap = (long long)sm_count() * 16;
  return (int)(need < 1 ? 1 : (need < cap ? need : cap));
}

cudaError_t launch_gather_rows(const void* src, const float* src_scale, const int32_t* sorted,
                               const int32_t* num_post, int P, int N, int k, int row_bytes, void* dst,
                               float* dst_scale, cudaStream_t s) {
  gather_rows_kernel<<<warp_rows_grid(P), 256, 0, s>>>((const uint4*)src, src_scale, sorted, num_post, P, N,
                                                        k, row_bytes / 16, (uint4*)dst, dst_scale);
  return cudaGetLastError();
}

cudaError_t launch_quant_rows(const void* src, const int32_t* sorted, bool gather, int N, int k,
                              const int32_t* nrows_dev, int nrows, int C, void* q, float* scale, int32_t* status,
                              cudaStream_t s) {
  const int vec = C / 8;
  if (C >= 4096) {
    // long rows, staged in shared memory: W warps x nb buffers of one row
    // each, <= 200 KB.  (Measured: Mixtral's 14336-wide h rows 81 -> 74 us;
    // 2048-wide rows are faster in registers, 34 vs 37 us.)
    constexpr size_t kBudget = 200 * 1024;
    const size_t row_bytes = (size_t)C * 2;
    int W = 8, nb = (int)(kBudget / (W * row_bytes));
    if (nb > 4) nb = 4;
    if (nb < 1) {
      nb = 1;
      W = (int)(kBudget / row_bytes);
    }
    if (W >= 1 && nrows > 0) {
      const size_t smem = (size_t)W * nb * (row_bytes + 8);
      const long long ctas = ((long long)nrows + W - 1) / W;
      const int sms = sm_count();
      const int g = (int)(ctas < sms ? ctas : sms);
      cudaError_t e = cudaFuncSetAttribute(quant_rows_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
      quant_rows_bulk_kernel<<<g, 32 * W, smem, s>>>((const uint8_t*)src, sorted, gather, N, k, nrows_dev, nrows,
                                                     vec, nb, (uint2*)q, scale, status, kDefaultTimeoutNs);
      return cudaGetLastError();
    }
  }
  const int vpl = (vec + 31) / 32;
  const int g = warp_rows_grid(nrows);
  const uint4* in = (const uint4*)src;
  uint2* out = (uint2*)q;
#define MOE_QUANT(V) \
  quant_rows_warp_kernel<V><<<g, 256, 0, s>>>(in, sorted, gather, N, k, nrows_dev, nrows, vec, out, scale)
  if (vpl <= 1) MOE_QUANT(1);
  else if (vpl <= 2) MOE_QUANT(2);
  else if (vpl <= 4) MOE_QUANT(4);
  else if (vpl <= 8) MOE_QUANT(8);
  else if (vpl <= 16) MOE_QUANT(16);
  else quant_rows_2pass_kernel<<<g, 256, 0, s>>>(in, sorted, gather, N, k, nrows_dev, nrows, vec, out, scale);
#undef MOE_QUANT
  return cudaGetLastError();
}

// Exhaustive check of the quotient path: block b takes amax = the positive
// bf16 with bit pattern b + 1 (up to the largest finite, 0x7F7F) and every
// bf16 v with |v| <= amax, both signs; the codes of quant_pair must equal
// e4m3(__fdiv_rn(v, s)).  counts[0] += pairs checked, counts[1] += mismatches;
// first_bad keeps one failing (v bits << 16 | amax bits).
__global__ void __launch_bounds__(256) quant_division_check_kernel(unsigned long long* counts,
                                                                   unsigned int* first_bad) {
  const uint32_t amax_bits = blockIdx.x + 1;
  const float amax = __uint_as_float(amax_bits << 16);
  const RowScale rs = row_scale(amax);
  unsigned long long bad = 0;
  for (uint32_t vb = threadIdx.x; vb <= amax_bits; vb += blockDim.x) {
    const uint32_t pos = vb, neg = vb | 0x8000u;
    const uint32_t packed = pos | (neg << 16);
    const uint32_t got = rs.r != 0.f ? quant_pair<true>(packed, rs) : quant_pair<false>(packed, rs);
    const uint32_t want = (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(__uint_as_float(pos << 16), rs.s), __NV_SATFINITE,
                                                          __NV_E4M3) |
                          ((uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(__uint_as_float(neg << 16), rs.s),
                                                           __NV_SATFINITE, __NV_E4M3)
                           << 8);
    if (got != want) {
      ++bad;
      atomicCAS(first_bad, 0u, (vb << 16) | amax_bits);
    }
  }
  for (int off = 16; off > 0; off >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, off);
  if ((threadIdx.x & 31) == 0 && bad) atomicAdd(counts + 1, bad);
  if (threadIdx.x == 0) atomicAdd(counts, 2ull * (amax_bits + 1));
}

cudaError_t launch_quant_division_check(unsigned long long* counts, unsigned int* first_bad, cudaStream_t s) {
  quant_division_check_kernel<<<0x7F7F, 256, 0, s>>>(counts, first_bad);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Combine (MoE Align & Sort article, "Megatron": unpermute):
// out[t] = sum_j w[t,j] * y[t*k+j], fp32 in ascending j, rounded once.
// ---------------------------------------------------------------------------
template <bool kBF16>
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y, const float* __restrict__ w,
                                                      int T, int k, int H, void* __restrict__ out) {
  const int t = blockIdx.y;
  const int h4 = blockIdx.x * blockDim.x + threadIdx.x;
  const int vec = H / 4;
  if (h4 >= vec) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const float wj = __ldg(w + (long long)t * k + j);
    const float4 v = __ldg(y + ((long long)t * k + j) * vec + h4);
    acc.x = fmaf(wj, v.x, acc.x);
    acc.y = fmaf(wj, v.y, acc.y);
    acc.z = fmaf(wj, v.z, acc.z);
    acc.w = fmaf(wj, v.w, acc.w);
  }
  if (kBF16) {
    __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y), b = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&a);
    o.y = *reinterpret_cast<uint32_t*>(&b);
    reinterpret_cast<uint2*>(out)[(long long)t * vec + h4] = o;
  } else {
    reinterpret_cast<float4*>(out)[(long long)t * vec + h4] = acc;
  }
}

// fp32 -> bf16 (round to nearest even), n a multiple of 4, 16-byte aligned
__global__ void __launch_bounds__(256) cast_bf16_kernel(const float4* __restrict__ src, long long n4,
                                                        uint2* __restrict__ dst) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 v = __ldg(src + i);
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&a);
    o.y = *reinterpret_cast<uint32_t*>(&b);
    dst[i] = o;
  }
}

cudaError_t launch_cast_bf16(const float* src, long long n, void* dst, cudaStream_t s) {
  const long long n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  const long long cap = (long long)sm_count() * 8;
  long long g = (n4 + 255) / 256;
  g = g < cap ? g : cap;
  cast_bf16_kernel<<<(unsigned)g, 256, 0, s>>>((const float4*)src, n4, (uint2*)dst);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* y, const float* w, int T, int k, int H, void* out, bool bf16,
                           cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  dim3 grid((unsigned)((H / 4 + 255) / 256), (unsigned)T), block(256);
  if (bf16) combine_kernel<true><<<grid, block, 0, s>>>((const float4*)y, w, T, k, H, out);
  else combine_kernel<false><<<grid, block, 0, s>>>((const float4*)y, w, T, k, H, out);
  return cudaGetLastError();
}

}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------
// Expert-parallel helpers: destination rank of every slot (and the number of
// slots per rank), the local expert ids of the slots in rank order, and row
// permutations by an index map.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) ep_dest_kernel(const int32_t* __restrict__ ids, int N, int E, int E_loc,
                                                      int32_t* __restrict__ dest, int32_t* __restrict__ counts,
                                                      int32_t* status) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
    const int e = ids[i];
    if (e < 0 || e >= E) {
      dev_flag(status, MOE_DEV_BAD_EXPERT_ID);
      dest[i] = -1;                 // align & sort skips it and flags it again
      continue;
    }
    const int r = e / E_loc;
    dest[i] = r;
    atomicAdd(counts + r, 1);
  }
}

__global__ void __launch_bounds__(256) ep_local_ids_kernel(const int32_t* __restrict__ ids,
                                                           const int32_t* __restrict__ order, int N, int E_loc,
                                                           int32_t* __restrict__ local_ids) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
    const int s = order[i];
    local_ids[i] = s >= 0 && s < N ? ids[s] % E_loc : 0;
  }
}

// dst row i = src row map[i] / div (gather) or dst row map[i] = src row i (scatter); 16-byte vectors, warp per row
template <bool kScatter>
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ src, int vec,
                                                           const int32_t* __restrict__ map, int n, int div,
                                                           int limit, uint4* __restrict__ dst) {
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < n; i += gridDim.x * wpb) {
    const int v = map[i];
    const int m = v / div;
    if (v < 0 || m >= limit) continue;          // out-of-range map entries move nothing
    const uint4* s = src + (long long)(kScatter ? i : m) * vec;
    uint4* d = dst + (long long)(kScatter ? m : i) * vec;
    for (int c = lane; c < vec; c += 32) d[c] = __ldg(s + c);
  }
}

static int grid_for(long long n, int per_block) {
  const long long need = (n + per_block - 1) / per_block;
  const long long cap = (long long)sm_count() * 16;
  return (int)(need < 1 ? 1 : (need < cap ? need : cap));
}

cudaError_t launch_ep_dest(const int32_t* ids, int N, int E, int E_loc, int32_t* dest, int32_t* counts,
                           int32_t* status, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  ep_dest_kernel<<<grid_for(N, 256), 256, 0, s>>>(ids, N, E, E_loc, dest, counts, status);
  return cudaGetLastError();
}

cudaError_t launch_ep_local_ids(const int32_t* ids, const int32_t* order, int N, int E_loc, int32_t* local_ids,
                                cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  ep_local_ids_kernel<<<grid_for(N, 256), 256, 0, s>>>(ids, order, N, E_loc, local_ids);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows(const void* src, int row_bytes, const int32_t* map, int n, int div, int limit,
                                bool scatter, void* dst, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int g = grid_for(n, 8);
  if (scatter)
    permute_rows_kernel<true><<<g, 256, 0, s>>>((const uint4*)src, row_bytes / 16, map, n, div, limit, (uint4*)dst);
  else
    permute_rows_kernel<false><<<g, 256, 0, s>>>((const uint4*)src, row_bytes / 16, map, n, div, limit, (uint4*)dst);
  return cudaGetLastError();
}

}  // namespace moe
