// Memory-bound steps of the MoE layer forward on sm_100a:
//   topk_gate      softmax top-k gating, one warp per token
//   permute        gather of token rows into sorted (expert-grouped) order
//   quant_rows     per-row E4M3 quantisation (per-token activations, and the
//                  requantisation of h between the two GEMMs), optionally
//                  fused with the gather
//   combine        top-k weighted sum of the per-slot expert outputs
#include <cfloat>

#include "kernels.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Top-k gating (MoE Align & Sort article, "FasterTransformer":
// moe_softmax + moe_top_k fused as topk_gating_softmax).  Lane l holds the
// logits of experts l, l+32, ...; k rounds of a warp arg-max (ties to the
// lower expert index) pick the experts in descending order.  The weights are
// exp(l_j - l_max) over the chosen experts, normalised by their sum, which is
// softmax over all E renormalised over the chosen k.
// ---------------------------------------------------------------------------
template <int EPL>
__global__ void __launch_bounds__(256) topk_gate_kernel(const float* __restrict__ logits,
                                                        const float* __restrict__ bias, int T, int E, int k,
                                                        int32_t* __restrict__ ids, float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  const long long t = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  float v[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    v[j] = -FLT_MAX;
    if (e < E) {
      float x = __ldg(logits + t * E + e);
      if (bias) x = __fadd_rn(x, __ldg(bias + e));
      v[j] = x;
    }
  }
  uint32_t taken = 0;
  float my_val = 0.f;
  int my_id = 0;
  for (int r = 0; r < k; ++r) {
    float best = -FLT_MAX;
    int be = INT_MAX;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((taken >> j) & 1u) && (be == INT_MAX || v[j] > best)) {
        best = v[j];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (oe != INT_MAX && (be == INT_MAX || ob > best || (ob == best && oe < be))) {
        best = ob;
        be = oe;
      }
    }
    if (lane == (be & 31)) taken |= 1u << (be >> 5);
    if (lane == r) {
      my_val = best;
      my_id = be;
    }
  }
  const float top = __shfl_sync(0xffffffffu, my_val, 0);
  const float ex = lane < k ? expf(my_val - top) : 0.f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < k) {
    ids[t * k + lane] = my_id;
    w[t * k + lane] = __fdiv_rn(ex, sum);
  }
}

cudaError_t launch_topk_gate(const float* logits, const float* bias, int T, int E, int k, int32_t* ids,
                             float* w, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int warps = 8;
  dim3 grid((unsigned)((T + warps - 1) / warps)), block(32 * warps);
  const int epl = (E + 31) / 32;
  if (epl <= 1) topk_gate_kernel<1><<<grid, block, 0, s>>>(logits, bias, T, E, k, ids, w);
  else if (epl <= 2) topk_gate_kernel<2><<<grid, block, 0, s>>>(logits, bias, T, E, k, ids, w);
  else if (epl <= 4) topk_gate_kernel<4><<<grid, block, 0, s>>>(logits, bias, T, E, k, ids, w);
  else if (epl <= 8) topk_gate_kernel<8><<<grid, block, 0, s>>>(logits, bias, T, E, k, ids, w);
  else if (epl <= 16) topk_gate_kernel<16><<<grid, block, 0, s>>>(logits, bias, T, E, k, ids, w);
  else topk_gate_kernel<32><<<grid, block, 0, s>>>(logits, bias, T, E, k, ids, w);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Gather of token rows into sorted order (MoE Align & Sort article,
// "FasterTransformer": permute before the group GEMM).  Row r of A is the
// token of slot sorted[r]; padding rows are zero.  Rows >= num_post are not
// touched.  16-byte vectors; H % 8 == 0.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) permute_bf16_kernel(const uint4* __restrict__ x,
                                                           const int32_t* __restrict__ sorted,
                                                           const int32_t* __restrict__ num_post, int N, int k,
                                                           int H, uint4* __restrict__ A) {
  const int np = *num_post;
  const int vec = H / 8;
  for (int r = blockIdx.x; r < np; r += gridDim.x) {
    const int slot = __ldg(sorted + r);
    const uint4* src = slot < N ? x + (long long)(slot / k) * vec : nullptr;
    uint4* dst = A + (long long)r * vec;
    for (int c = threadIdx.x; c < vec; c += blockDim.x) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (src) v = __ldg(src + c);
      dst[c] = v;
    }
  }
}

// ---------------------------------------------------------------------------
// Per-row E4M3 quantisation (aiter issue 1248: per-token FP8 activations;
// GC-MoE: requantisation between the GEMMs).  s = amax / 448 in fp32 (1 for
// an all-zero row); code = e4m3_rne_satfinite(v / s) with an IEEE fp32
// division.  In gather mode row r reads token sorted[r] / k of x (padding
// rows become zero codes with s = 1); otherwise it reads row r of src.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t e4m3_pack4(float a, float b, float c, float d) {
  const uint32_t qa = __nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3);
  const uint32_t qb = __nv_cvt_float_to_fp8(b, __NV_SATFINITE, __NV_E4M3);
  const uint32_t qc = __nv_cvt_float_to_fp8(c, __NV_SATFINITE, __NV_E4M3);
  const uint32_t qd = __nv_cvt_float_to_fp8(d, __NV_SATFINITE, __NV_E4M3);
  return qa | (qb << 8) | (qc << 16) | (qd << 24);
}

__global__ void __launch_bounds__(256) quant_rows_kernel(const uint4* __restrict__ src,
                                                         const int32_t* __restrict__ sorted,
                                                         const int32_t* __restrict__ num_post, int N, int k,
                                                         int C, uint2* __restrict__ q, float* __restrict__ scale) {
  __shared__ float s_red[8];
  const int np = *num_post;
  const int vec = C / 8;  // 8 bf16 per uint4 in, 8 codes per uint2 out
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r = blockIdx.x; r < np; r += gridDim.x) {
    const uint4* row;
    if (sorted) {
      const int slot = __ldg(sorted + r);
      row = slot < N ? src + (long long)(slot / k) * vec : nullptr;
    } else {
      row = src + (long long)r * vec;
    }
    uint2* dst = q + (long long)r * vec;
    if (!row) {
      for (int c = threadIdx.x; c < vec; c += blockDim.x) dst[c] = make_uint2(0, 0);
      if (threadIdx.x == 0) scale[r] = 1.f;
      continue;
    }
    float amax = 0.f;
    for (int c = threadIdx.x; c < vec; c += blockDim.x) {
      const uint4 v = __ldg(row + c);
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))),
                               fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))));
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))),
                               fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) s_red[warp] = amax;
    __syncthreads();
    amax = s_red[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) amax = fmaxf(amax, s_red[i]);
    __syncthreads();
    const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    for (int c = threadIdx.x; c < vec; c += blockDim.x) {
      const uint4 v = __ldg(row + c);
      uint2 o;
      o.x = e4m3_pack4(__fdiv_rn(bf16_lo(v.x), s), __fdiv_rn(bf16_hi(v.x), s), __fdiv_rn(bf16_lo(v.y), s),
                       __fdiv_rn(bf16_hi(v.y), s));
      o.y = e4m3_pack4(__fdiv_rn(bf16_lo(v.z), s), __fdiv_rn(bf16_hi(v.z), s), __fdiv_rn(bf16_lo(v.w), s),
                       __fdiv_rn(bf16_hi(v.w), s));
      dst[c] = o;
    }
    if (threadIdx.x == 0) scale[r] = s;
  }
}

static int rows_grid(int P) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long g = (long long)sms * 8;
  return (int)(P < g ? (P > 0 ? P : 1) : g);
}

cudaError_t launch_permute_bf16(const void* x, const int32_t* sorted, const int32_t* num_post, int P, int N,
                                int k, int H, void* A, cudaStream_t s) {
  permute_bf16_kernel<<<rows_grid(P), 256, 0, s>>>((const uint4*)x, sorted, num_post, N, k, H, (uint4*)A);
  return cudaGetLastError();
}

cudaError_t launch_quant_rows(const void* src, const int32_t* sorted, const int32_t* num_post, int P, int N,
                              int k, int C, void* q, float* scale, cudaStream_t s) {
  quant_rows_kernel<<<rows_grid(P), 256, 0, s>>>((const uint4*)src, sorted, num_post, N, k, C, (uint2*)q,
                                                 scale);
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

cudaError_t launch_combine(const float* y, const float* w, int T, int k, int H, void* out, bool bf16,
                           cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  dim3 grid((unsigned)((H / 4 + 255) / 256), (unsigned)T), block(256);
  if (bf16) combine_kernel<true><<<grid, block, 0, s>>>((const float4*)y, w, T, k, H, out);
  else combine_kernel<false><<<grid, block, 0, s>>>((const float4*)y, w, T, k, H, out);
  return cudaGetLastError();
}

}  // namespace moe
