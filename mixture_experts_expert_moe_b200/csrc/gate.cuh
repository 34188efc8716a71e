// Softmax top-k gating of one token by one warp (MoE Align & Sort article,
// "FasterTransformer": moe_softmax + moe_top_k fused as topk_gating_softmax,
// and its biased variant; the opening definition: Top-K gating scores, with
// DeepSeek V3's gating bias and shared experts).  Shared by the stand-alone
// gate kernel and the fused routing kernel.
//
// Lane l holds the scores of experts l, l+32, ... (logit, + bias in fp32);
// k rounds of a warp arg-max (ties to the lower expert index) pick the
// experts in descending score order.  The weights are exp(l_j - max_j l_j)
// over the chosen experts normalised by their sum (softmax over all E
// renormalised over the chosen k: the full denominator cancels), where l is
// the biased logit, or with select_only the raw logit (the bias then only
// steers the choice, as in DeepSeek's auxiliary-loss-free balancing).
// Columns k..k+n_shared-1 of the token's row name the shared experts
// E..E+n_shared-1 with weight 1.
#pragma once
#include <cfloat>
#include <climits>

#include "common.cuh"

namespace moe {

template <int EPL>
__device__ __forceinline__ void gate_token(const float* __restrict__ logits, const float* __restrict__ bias,
                                           bool select_only, long long t, int E, int k, int n_shared,
                                           int32_t* __restrict__ ids, float* __restrict__ w, int lane) {
  float v[EPL], raw[EPL], b[EPL];
  // all loads first, then the adds (a use right after a load would serialise them)
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    raw[j] = e < E ? __ldg(logits + t * E + e) : -FLT_MAX;
    b[j] = (bias && e < E) ? __ldg(bias + e) : 0.f;
  }
#pragma unroll
  for (int j = 0; j < EPL; ++j) v[j] = (bias && lane + 32 * j < E) ? __fadd_rn(raw[j], b[j]) : raw[j];
  uint32_t taken = 0;
  float my_val = 0.f, my_raw = 0.f;
  int my_id = 0;
  for (int r = 0; r < k; ++r) {
    float best = -FLT_MAX, braw = 0.f;
    int be = INT_MAX;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((taken >> j) & 1u) && (be == INT_MAX || v[j] > best)) {
        best = v[j];
        braw = raw[j];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, off);
      const float oraw = __shfl_xor_sync(0xffffffffu, braw, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (oe != INT_MAX && (be == INT_MAX || ob > best || (ob == best && oe < be))) {
        best = ob;
        braw = oraw;
        be = oe;
      }
    }
    if (lane == (be & 31)) taken |= 1u << (be >> 5);
    if (lane == r) {
      my_val = best;
      my_raw = braw;
      my_id = be;
    }
  }
  const float l = lane < k ? (select_only ? my_raw : my_val) : -FLT_MAX;
  float top = l;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, off));
  const float ex = lane < k ? expf(l - top) : 0.f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const long long row = t * (k + n_shared);
  if (lane < k) {
    ids[row + lane] = my_id;
    w[row + lane] = __fdiv_rn(ex, sum);
  } else if (lane < k + n_shared) {
    ids[row + lane] = E + (lane - k);
    w[row + lane] = 1.f;
  }
}

}  // namespace moe
