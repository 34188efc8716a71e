// Backward pass of the MoE layer's expert FFN and combine on sm_100a, bf16
// weights (MoE Align & Sort article, "Megatron": the combine's gradient is the
// unpermute of the output gradient; opening definition of the layer).  The
// gradients are the chain rule through the forward, recomputing what the
// forward does not keep:
//
//   D  = dout rows in sorted order                          (gather)
//   z  = Wd[e]^T D_r                 per sorted row, [P, I]  (BWD_Z)
//   g, u = W13[e] x_r (recomputed);  a = silu(g); h = bf16(a u)
//   dw_slot = <z, h>  (= <dout_t, y_slot>: the combine weight's gradient)
//   dh = w z (straight through the bf16 rounding of h);
//   dg = dh u s (1 + g (1 - s)), s = sigmoid(g);  du = dh a  (BWD_GUB)
//   dx_t += W13[e]^T [dg; du]                                 (BWD_DX)
//   dW2[e]  = sum_r D_r^T (w h)_r,  dW13[e] = sum_r [dg; du]_r^T x_r  (BWD_WG)
//
// One kernel, four tile kinds, the forward's warp roles (warp 0 TMA, warp 1
// tcgen05.mma, warps 2..9 epilogue) and a static round-robin tile schedule.
// Weights enter the gradient GEMMs transposed: they are read MN-major (TMA
// boxes of 64 features x 64 K-rows, the descriptor's MN-major 128-byte-swizzle
// layout), as are both operands of the per-expert weight gradients, whose
// reduction runs over the expert's sorted token rows.
#include "gemm_common.cuh"

namespace moe {

namespace {

constexpr int kKRows = 64;                       // K rows per stage of an MN-major operand (bf16: 128 B of K)
constexpr int kMnBox = 64 * kKRows * 2;          // one MN-major box: 64 features x 64 K-rows of bf16

struct BwdTile {
  int e, mt, r0, nrows, ncol0;   // expert, M tile, first token row (or K row), rows, first output column (WG)
  bool skip;                     // WG tile of an expert without tokens: the epilogue writes zeros
};

__device__ __forceinline__ BwdTile bwd_tile(const BwdParams& p, int t, const int* s_pref, const int* s_perm,
                                            const int* s_start, const int* s_rows, const int* s_groups,
                                            const int* s_prow) {
  BwdTile b;
  if (p.kind == BWD_WG) {
    const int nn = p.n_cols / p.tn, nm = (p.n_out + 2 * kWRows - 1) / (2 * kWRows);
    b.e = t / (nm * nn);
    const int rest = t - b.e * nm * nn;
    b.mt = rest / nn;
    b.ncol0 = (rest - b.mt * nn) * p.tn;
    b.r0 = s_start[b.e];
    b.nrows = s_prow[b.e];          // the expert's padded segment: K of this GEMM
    b.skip = b.nrows == 0;
  } else {
    const TileInfo ti = decode_tile(t, s_pref, s_perm, s_start, s_rows, s_groups, p.E, p.tn);
    b.e = ti.e;
    b.mt = ti.wt;
    b.r0 = ti.r0;
    b.nrows = ti.nrows;
    b.ncol0 = 0;
    b.skip = false;
  }
  return b;
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int E = p.E;
  const int a_bytes = 2 * kWTileBytes;                  // two 128-row A sub-tiles
  const int stage_bytes = a_bytes + p.tn * kStageK;     // + the B tile (tn rows or columns x 128 B)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)p.stages * stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + p.stages;
  uint64_t* acc_full = bars + 2 * p.stages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  int* s_abort = reinterpret_cast<int*>(s_tmem + 1);
  int* s_drain_fail = s_abort + 1;
  int* s_start = s_abort + 2;
  int* s_rows = s_start + E;       // real rows per expert
  int* s_prow = s_rows + E;        // padded rows per expert
  int* s_groups = s_prow + E;
  int* s_perm = s_groups + E;
  int* s_pref = s_perm + E;        // E + 1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    *s_drain_fail = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, p.tmem_cols);
    tmem_relinquish();
  }
  const bool gu_list = p.kind == BWD_Z || p.kind == BWD_GUB;
  const int pref_off = plan_pref(E, gu_list);
  for (int i = threadIdx.x; i < E; i += blockDim.x) {
    s_start[i] = p.plan[plan_start(E) + i];
    s_rows[i] = p.plan[plan_real(E) + i];
    s_prow[i] = p.plan[plan_rows(E) + i];
    s_groups[i] = p.plan[plan_groups(E) + i];
    s_perm[i] = p.plan[plan_perm(E) + i];
  }
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_pref[i] = p.plan[pref_off + i];
  int n_tiles;
  if (p.kind == BWD_WG)
    n_tiles = E * ((p.n_out + 2 * kWRows - 1) / (2 * kWRows)) * (p.n_cols / p.tn);
  else
    n_tiles = p.plan[gu_list ? PLAN_TILES_GU : PLAN_TILES_DN];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int cols_per_acc = 2 * p.tn;
  const int xb = x_box_rows(p.tn);
  volatile int* abort_flag = s_abort;
  // the A operand is MN-major in every kind but the gate/up recomputation;
  // B is MN-major in the weight gradients
  const bool a_mn = p.kind != BWD_GUB;
  const bool b_mn = p.kind == BWD_WG;
  const bool paired = p.kind != BWD_Z;    // BWD_Z: one 128-feature sub-tile per tile

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      long long armed = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const BwdTile bt = bwd_tile(p, t, s_pref, s_perm, s_start, s_rows, s_groups, s_prow);
        if (bt.skip) continue;
        if (!MOE_IN_BOUNDS(bt.e >= 0 && bt.e < E && bt.r0 >= 0 && bt.r0 + bt.nrows <= p.plan[PLAN_NUM_POST],
                           p.status)) {
          *abort_flag = 2;     // every role stops at its next wait (2: not a timeout)
          ok = false;
          break;
        }
        // A rows / columns of the two sub-tiles
        int a0, a1;            // K-major: weight rows; MN-major: first feature column
        bool has1 = paired;
        int abase = 0;         // MN-major: global row of the K origin
        if (p.kind == BWD_GUB) {
          a0 = bt.e * 2 * p.n_out + bt.mt * kWRows;      // gate rows, then up rows
          a1 = a0 + p.n_out;
        } else if (p.kind == BWD_Z) {
          a0 = bt.mt * kWRows;                            // Wd [E*H rows, I]: features are columns
          a1 = a0;
          abase = bt.e * p.K;
        } else if (p.kind == BWD_DX) {
          a0 = bt.mt * 2 * kWRows;                        // W13 [E*2I rows, H]: features are columns
          a1 = a0 + kWRows;
          has1 = a1 < p.n_out;
          abase = bt.e * p.K;
        } else {
          a0 = bt.mt * 2 * kWRows;                        // D or dgu [P, M]: features are columns
          a1 = a0 + kWRows;
          has1 = a1 < p.n_out;
          abase = bt.r0;
        }
        const int nk = p.kind == BWD_WG ? (bt.nrows + kKRows - 1) / kKRows : p.K / kKRows;
        const int nload = b_mn ? p.tn / 64 : (bt.nrows + xb - 1) / xb;
        const uint32_t tx = (has1 ? 2 : 1) * kWTileBytes + (b_mn ? p.tn * kStageK : nload * xb * kStageK);
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_or_abort(&empty[stage], phase ^ 1, p.timeout_ns, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sb = smem + (size_t)stage * stage_bytes;
          mbar_arrive_expect_tx(&full[stage], tx);
          const int kr = kb * kKRows;   // K offset (elements)
          if (a_mn) {
            // two boxes of 64 features per 128-row sub-tile
            tma_load_2d(sb, &tm_a, &full[stage], a0, abase + kr, pol_w);
            tma_load_2d(sb + kMnBox, &tm_a, &full[stage], a0 + 64, abase + kr, pol_w);
            if (has1) {
              tma_load_2d(sb + kWTileBytes, &tm_a, &full[stage], a1, abase + kr, pol_w);
              tma_load_2d(sb + kWTileBytes + kMnBox, &tm_a, &full[stage], a1 + 64, abase + kr, pol_w);
            }
          } else {
            tma_load_2d(sb, &tm_a, &full[stage], kr, a0, pol_w);
            tma_load_2d(sb + kWTileBytes, &tm_a, &full[stage], kr, a1, pol_w);
          }
          if (b_mn) {
            for (int c = 0; c < nload; ++c)
              tma_load_2d(sb + a_bytes + c * kMnBox, &tm_b, &full[stage], bt.ncol0 + 64 * c, bt.r0 + kr, pol_x);
          } else {
            for (int l = 0; l < nload; ++l)
              tma_load_2d(sb + a_bytes + l * xb * kStageK, &tm_b, &full[stage], kr, bt.r0 + l * xb, pol_x);
          }
          ++armed;
          if (++stage == p.stages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < p.stages; ++s) {
          if (armed > s) {
            const uint32_t par = s < stage ? phase : phase ^ 1;
            if (!mbar_wait(&full[s], par, kDrainTimeoutNs)) *s_drain_fail = 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int ia = 0;    // tiles that use an accumulator
      bool ok = true;
      bool issued = false;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const BwdTile bt = bwd_tile(p, t, s_pref, s_perm, s_start, s_rows, s_groups, s_prow);
        if (bt.skip) continue;
        const bool has1 = paired && (p.kind == BWD_GUB || bt.mt * 2 * kWRows + kWRows < p.n_out);
        const int acc = ia % p.n_acc;
        const uint32_t acc_phase = (uint32_t)(ia / p.n_acc) & 1u;
        ++ia;
        if (!wait_or_abort(&acc_empty[acc], acc_phase ^ 1, p.timeout_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * cols_per_acc);
        const uint32_t d1 = d0 + (uint32_t)p.tn;
        const int n_mma = b_mn ? p.tn : ((bt.nrows + 15) / 16) * 16;
        const uint32_t idesc = umma_idesc_bf16_major(kWRows, n_mma, a_mn ? 1u : 0u, b_mn ? 1u : 0u);
        const int nk = p.kind == BWD_WG ? (bt.nrows + kKRows - 1) / kKRows : p.K / kKRows;
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_or_abort(&full[stage], phase, p.timeout_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w0 = smem_u32(smem + (size_t)stage * stage_bytes);
          const uint32_t w1 = w0 + kWTileBytes;
          const uint32_t xa = w0 + (uint32_t)a_bytes;
          // MMA K-steps of 16 rows; a weight gradient's last stage stops at the
          // expert's padded segment end (a multiple of 16)
          const int ksteps = p.kind == BWD_WG ? min(4, (bt.nrows - kb * kKRows + 15) / 16) : 4;
          for (int kk = 0; kk < ksteps; ++kk) {
            const uint64_t adesc0 = a_mn ? umma_desc_mn_sw128(w0 + kk * 2048, kMnBox) : umma_desc_sw128(w0 + kk * 32);
            const uint64_t adesc1 = a_mn ? umma_desc_mn_sw128(w1 + kk * 2048, kMnBox) : umma_desc_sw128(w1 + kk * 32);
            const uint64_t bdesc = b_mn ? umma_desc_mn_sw128(xa + kk * 2048, kMnBox) : umma_desc_sw128(xa + kk * 32);
            const uint32_t accum = (kb | kk) != 0;
            mma_bf16(d0, adesc0, bdesc, idesc, accum);
            if (has1) mma_bf16(d1, adesc1, bdesc, idesc, accum);
          }
          issued = true;
          tc_commit(&empty[stage]);
          if (++stage == p.stages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
      }
      if (!ok && issued) {
        tc_commit(drain);
        if (!mbar_wait(drain, 0, kDrainTimeoutNs)) *s_drain_fail = 1;
      }
    }
  } else {
    // ---------------- epilogue: warps 2..9 ----------------
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int m = 32 * q + lane;
    int ia = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
      if (*abort_flag) break;
      const BwdTile bt = bwd_tile(p, t, s_pref, s_perm, s_start, s_rows, s_groups, s_prow);
      if (bt.skip) {
        // an expert without tokens: its weight gradient is zero
        const int r0 = bt.mt * 2 * kWRows + m;
        for (int sub = 0; sub < 2; ++sub) {
          const int row = r0 + sub * kWRows;
          if (row >= p.n_out) continue;
          float4* o = reinterpret_cast<float4*>(p.out + ((size_t)bt.e * p.n_out + row) * p.n_cols + bt.ncol0);
          for (int c = 4 * half; c < p.tn / 4; c += 8) {
            o[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            o[c + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
            o[c + 2] = make_float4(0.f, 0.f, 0.f, 0.f);
            o[c + 3] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        continue;
      }
      const int acc = ia % p.n_acc;
      const uint32_t acc_phase = (uint32_t)(ia / p.n_acc) & 1u;
      ++ia;
      if (!wait_or_abort(&acc_full[acc], acc_phase, p.timeout_ns, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * cols_per_acc);
      if (p.kind == BWD_Z) {
        const int n = bt.mt * kWRows + m;
        for (int c = 16 * half; c < bt.nrows; c += 32) {
          float v[16];
          tmem_ld16(tb + c, v);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c + i < bt.nrows) p.out[(size_t)(bt.r0 + c + i) * p.n_out + n] = v[i];
        }
      } else if (p.kind == BWD_GUB) {
        const int n = bt.mt * kWRows + m;
        const int I = p.n_out;
        for (int c = 16 * half; c < bt.nrows; c += 32) {
          float g[16], u[16];
          const bool in = lane < 16 && c + lane < bt.nrows;
          const int slot_l = in ? __ldg(p.sorted + bt.r0 + c + lane) : p.n_slots;
          const float w_l = (unsigned)slot_l < (unsigned)p.n_slots ? __ldg(p.topk_w + slot_l) : 0.f;
          tmem_ld16(tb + c, g);
          tmem_ld16(tb + p.tn + c, u);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int slot = __shfl_sync(0xffffffffu, slot_l, i);
            const float w = __shfl_sync(0xffffffffu, w_l, i);
            // uniform across the warp
            if (c + i < bt.nrows && MOE_IN_BOUNDS(slot >= 0, p.status) && (unsigned)slot < (unsigned)p.n_slots) {
              const size_t row = (size_t)(bt.r0 + c + i);
              const float gv = g[i], uv = u[i];
              const float s = 1.f / (1.f + expf(-gv));
              const float a = gv * s;
              const float h = __bfloat162float(__float2bfloat16_rn(a * uv));
              const float zz = p.zbuf[row * I + n];
              const float dh = w * zz;
              const float du = dh * a;
              const float dg = dh * uv * s * (1.f + gv * (1.f - s));
              p.dgu[row * 2 * I + n] = __float2bfloat16_rn(dg);
              p.dgu[row * 2 * I + I + n] = __float2bfloat16_rn(du);
              p.hw[row * I + n] = __float2bfloat16_rn(w * h);
              // the combine weight's gradient: <dout_t, y_slot> = <z, h>, summed over the features
              float part = zz * h;
#pragma unroll
              for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
              if (lane == 0) atomicAdd(p.dwt + slot, part);
            }
          }
        }
      } else if (p.kind == BWD_DX) {
        const int n0 = bt.mt * 2 * kWRows + m;
        const int n1 = n0 + kWRows;
        const bool has1 = n1 < p.n_out;
        const uint64_t pol = policy_evict_last();
        for (int c = 16 * half; c < bt.nrows; c += 32) {
          float v0[16], v1[16];
          const bool in = lane < 16 && c + lane < bt.nrows;
          const int slot_l = in ? __ldg(p.sorted + bt.r0 + c + lane) : p.n_slots;
          tmem_ld16(tb + c, v0);
          if (has1) tmem_ld16(tb + p.tn + c, v1);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int slot = __shfl_sync(0xffffffffu, slot_l, i);
            if (c + i < bt.nrows && MOE_IN_BOUNDS(slot >= 0, p.status) && (unsigned)slot < (unsigned)p.n_slots) {
              float* row = p.dx + (size_t)(slot / p.k) * p.n_out;
              red_add_f32(row + n0, v0[i], pol);
              if (has1) red_add_f32(row + n1, v1[i], pol);
            }
          }
        }
      } else {
        // weight gradient tile: rows m0 + m (and + 128) of dW[e], columns ncol0..+tn
        for (int sub = 0; sub < 2; ++sub) {
          const int row = bt.mt * 2 * kWRows + sub * kWRows + m;
          if (bt.mt * 2 * kWRows + sub * kWRows >= p.n_out) continue;   // uniform across the warp
          float* o = p.out + ((size_t)bt.e * p.n_out + row) * p.n_cols + bt.ncol0;
          for (int c = 16 * half; c < p.tn; c += 32) {
            float v[16];
            tmem_ld16(tb + sub * p.tn + c, v);
            float4* o4 = reinterpret_cast<float4*>(o + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) o4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag == 1) dev_flag(p.status, MOE_DEV_TIMEOUT);
  if (threadIdx.x == 0 && *s_drain_fail) dev_flag(p.status, MOE_DEV_DRAIN_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// MN-major bf16 operand [rows, cols] read in boxes of 64 columns x 64 rows.
bool make_map_mn(CUtensorMap* m, const void* base, long long rows, long long cols) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
  cuuint32_t box[2] = {64, (cuuint32_t)kKRows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Gradient of the renormalised top-k softmax (the combine weights) with
// respect to the router logits, one warp per token:
//   dl_j = w_j (dw_j - sum_i w_i dw_i) at the chosen experts, 0 elsewhere.
// The shared experts' constant weight 1 has no logit gradient.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dlogits_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w,
                                                      const float* __restrict__ dwt, int T, int E, int k, int kk,
                                                      float* __restrict__ dlogits) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  float* row = dlogits + (size_t)t * E;
  for (int e = lane; e < E; e += 32) row[e] = 0.f;
  const float wj = lane < k ? w[(size_t)t * kk + lane] : 0.f;
  const float gj = lane < k ? dwt[(size_t)t * kk + lane] : 0.f;
  float s = wj * gj;
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  __syncwarp();
  if (lane < k) row[ids[(size_t)t * kk + lane]] = wj * (gj - s);
}

}  // namespace

size_t bwd_smem_bytes(int tn, int stages, int E) {
  return 1024 + (size_t)stages * (2 * kWTileBytes + tn * kStageK) + (2 * stages + 5) * 8 + 16 +
         (size_t)(6 * E + 1) * 4;
}

int launch_bwd_gemm(const BwdLaunch& L, cudaStream_t stream) {
  BwdParams p = L.p;
  CUtensorMap ta, tb;
  const bool a_mn = p.kind != BWD_GUB, b_mn = p.kind == BWD_WG;
  if (a_mn ? !make_map_mn(&ta, L.a, L.a_rows, L.a_cols) : !make_map(&ta, L.a, L.a_rows, L.a_cols, 2, kWRows))
    return -1;
  if (b_mn ? !make_map_mn(&tb, L.b, L.b_rows, L.b_cols)
           : !make_map(&tb, L.b, L.b_rows, L.b_cols, 2, p.tn < 32 ? p.tn : 32))
    return -1;
  int s = 8;
  while (s > 2 && bwd_smem_bytes(p.tn, s, p.E) > 225 * 1024) --s;
  p.stages = s;
  const int cols = 2 * p.tn;
  p.n_acc = 2 * cols <= 512 ? 2 : 1;
  int need = p.n_acc * cols, alloc = 32;
  while (alloc < need) alloc <<= 1;
  p.tmem_cols = alloc;
  const size_t smem = bwd_smem_bytes(p.tn, p.stages, p.E);
  cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  bwd_gemm_kernel<<<sms, kGemmThreads, smem, stream>>>(ta, tb, p);
  return (int)cudaGetLastError();
}

cudaError_t launch_dlogits(const int32_t* ids, const float* w, const float* dwt, int T, int E, int k, int kk,
                           float* dlogits, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  dlogits_kernel<<<(T + 7) / 8, 256, 0, s>>>(ids, w, dwt, T, E, k, kk, dlogits);
  return cudaGetLastError();
}

}  // namespace moe
