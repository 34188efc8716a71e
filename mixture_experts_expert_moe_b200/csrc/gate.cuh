// Softmax top-k gating of one token by one warp (MoE Align & Sort article,
// "FasterTransformer": moe_softmax + moe_top_k fused as topk_gating_softmax;
// the opening definition: Top-K gating scores, with a gating bias in DeepSeek
// V3).  Shared by the stand-alone gate kernel and the fused routing kernel.
//
// Lane l holds the logits of experts l, l+32, ... (+ bias, added in fp32);
// k rounds of a warp arg-max (ties to the lower expert index) pick the experts
// in descending order.  The weights are exp(l_j - l_max) over the chosen
// experts normalised by their sum: softmax over all E renormalised over the
// chosen k (the full denominator cancels).
#pragma once
#include <cfloat>
#include <climits>

#include "common.cuh"

namespace moe {

template <int EPL>
__device__ __forceinline__ void gate_token(const float* __restrict__ logits, const float* __restrict__ bias,
                                           long long t, int E, int k, int32_t* __restrict__ ids,
                                           float* __restrict__ w, int lane) {
  float v[EPL], b[EPL];
  // all loads first, then the adds (a use right after a load would serialise them)
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < E ? __ldg(logits + t * E + e) : -FLT_MAX;
    b[j] = (bias && e < E) ? __ldg(bias + e) : 0.f;
  }
  if (bias) {
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (lane + 32 * j < E) v[j] = __fadd_rn(v[j], b[j]);
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

}  // namespace moe
