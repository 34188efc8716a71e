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

// Order-preserving map of a finite float to uint32: a > b iff key(a) > key(b),
// and a == b (as floats) iff key(a) == key(b), so -0 maps like +0.
__device__ __forceinline__ uint32_t score_key(float f) {
  const uint32_t b = f == 0.f ? 0u : __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int EPL>
__device__ __forceinline__ void gate_token(const float* __restrict__ logits, const float* __restrict__ bias,
                                           bool select_only, long long t, int E, int k, int n_shared,
                                           int32_t* __restrict__ ids, float* __restrict__ w, int lane) {
  float v[EPL];
  {
    float b[EPL];
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
  }
  // Each round: the lane's best untaken score (first one on equal scores, so
  // the lowest expert index), a warp max of its order-preserving 32-bit key
  // (redux.sync), then a warp min of the expert index among the lanes that
  // hold that key (ties go to the lower index).  The winner's score is the
  // key inverted.
  uint32_t taken = 0;
  float my_val = 0.f;
  int my_id = 0;
  for (int r = 0; r < k; ++r) {
    uint32_t bkey = 0u;          // below every finite score's key
    int be = INT_MAX;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      const uint32_t key = score_key(v[j]);
      if (e < E && !((taken >> j) & 1u) && (be == INT_MAX || key > bkey)) {
        bkey = key;
        be = e;
      }
    }
    const uint32_t wkey = __reduce_max_sync(0xffffffffu, bkey);
    const int win = (int)__reduce_min_sync(0xffffffffu, (be != INT_MAX && bkey == wkey) ? (uint32_t)be : 0xffffffffu);
    if (lane == (win & 31)) taken |= 1u << (win >> 5);
    if (lane == r) {
      my_val = key_score(wkey);
      my_id = win;
    }
  }
  // selection-only bias: the weights use the chosen experts' raw logits
  float my_raw = my_val;
  if (select_only && bias && lane < k) my_raw = __ldg(logits + t * E + my_id);
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
