// Grouped expert GEMMs of the MoE FFN on sm_100a: tcgen05 MMA with TMEM
// accumulators, operands staged by TMA into 128-byte-swizzled shared memory.
//
// What it computes (MoE Align & Sort article, opening definition and
// "AITER": each expert's FFN weights multiplied with a block of the tokens
// routed to it; aiter issue 1248: g1u1 SiLU, per-token FP8; GC-MoE: fused
// SwiGLU and requantisation):
//   gate/up : h[r, n] = bf16( silu(G) * U ),  G = Wg[e][n] . A[r],  U = Wu[e][n] . A[r]
//   down    : y[slot(r), n] = Wd[e][n] . h[r], or, fused with the combine
//             ("Megatron" unpermute), out32[slot(r) / k, n] += w[slot(r)] * y
//             (fp32 additions in L2, in no fixed order)
// for every sorted row r of expert e; FP8 operands are rescaled by the
// per-row activation scale and the per-channel weight scale after the fp32
// accumulation.
//
// Design (B200-first, not the pages' MI300 assembly tiles):
//   * operand swap (as the GC-MoE abstract describes for Blackwell decode):
//     128 weight rows fill the MMA M dimension and the expert's tokens are N
//     (16..256).  An expert's weight tile is streamed once for up to 256 of
//     its tokens, so weight traffic does not grow with the block size (the
//     lesson of the aiter issue's I/O table).
//   * persistent CTAs, one per SM, claim tiles from a global counter over a
//     device-built tile list ordered expert -> weight tile -> token group
//     (experts with several groups first, claims alternating between them
//     and the others; see plan.cuh), so CTAs that run at the same time share
//     weight tiles through L2 when an expert has several groups.  The TMA
//     warp claims; a 4-entry shared-memory ring hands the index to the MMA
//     and epilogue warps.
//   * warp roles: warp 0 issues TMA, warp 1 issues tcgen05.mma (one thread)
//     and owns the TMEM allocation, warps 2..9 drain TMEM (tcgen05.ld, two
//     warps per lane quarter on alternate column chunks) and run the
//     epilogue.  An S-stage shared-memory ring (full/empty
//     mbarriers) decouples TMA from MMA; two TMEM accumulator buffers
//     decouple MMA from the epilogue when they fit in 512 columns.
//   * every wait is bounded; on a timeout the CTA records MOE_DEV_TIMEOUT,
//     drains its copies and MMAs, frees TMEM and returns.
#include "gemm_common.cuh"
#include "plan.cuh"

namespace moe {

// Tile plan for the stand-alone FFN (moe_grouped_ffn), from the align & sort
// outputs; layout in kernels.cuh, ordering in plan.cuh.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ expert_ids,
                                                    const int32_t* __restrict__ num_post,
                                                    const int32_t* __restrict__ sorted, int N, int P, int E,
                                                    int bm, int tn, int nw_gu, int nw_dn,
                                                    int32_t* __restrict__ plan, int32_t* status) {
  extern __shared__ int sm[];
  int* s_first = sm;        // [E] first block of expert (-1: none)
  int* s_nblk = sm + E;     // [E] blocks of expert -> token groups
  int* sc = sm + 2 * E;     // [3E + 2] scratch of finish_plan
  int* s_bad = sm + 5 * E + 2;
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) {
    s_first[e] = -1;
    s_nblk[e] = 0;
  }
  if (tid == 0) *s_bad = 0;
  __syncthreads();
  int np = *num_post;
  if (np < 0 || np > P || np % bm != 0) {
    if (tid == 0) dev_flag(status, MOE_DEV_BAD_PLAN);
    np = 0;
  }
  const int nb = np / bm;
  for (int b = tid; b < nb; b += blockDim.x) {
    const int e = expert_ids[b];
    if (e < 0 || e >= E) {
      dev_flag(status, MOE_DEV_BAD_PLAN);
      continue;
    }
    atomicAdd(&s_nblk[e], 1);
    // the blocks of an expert form one run (a second run start would give a
    // segment reaching past num_post): anything else is an invalid plan
    if ((b == 0 || expert_ids[b - 1] != e) && atomicExch(&s_first[e], b) != -1) {
      dev_flag(status, MOE_DEV_BAD_PLAN);
      *s_bad = 1;
    }
  }
  __syncthreads();
  if (*s_bad) np = 0;       // an invalid plan runs no tiles
  for (int e = tid; e < E; e += blockDim.x) {
    const int rows = np ? s_nblk[e] * bm : 0;
    const int start = rows ? s_first[e] * bm : 0;
    // padding (slot id >= N) fills the end of the segment: count it in the last block
    int real = rows;
    for (int i = rows - 1; i >= 0 && i >= rows - bm; --i) {
      if ((unsigned)sorted[start + i] < (unsigned)N) break;
      --real;
    }
    plan[plan_start(E) + e] = start;
    plan[plan_rows(E) + e] = rows;
    plan[plan_real(E) + e] = real;
    s_nblk[e] = (rows + tn - 1) / tn;
  }
  __syncthreads();
  finish_plan(plan, s_nblk, E, nw_gu, nw_dn, tn, np, sc);
}

cudaError_t launch_plan(const int32_t* expert_ids, const int32_t* num_post, const int32_t* sorted, int N, int P,
                        int E, int bm, int tn, int nw_gu, int nw_dn, int32_t* plan, int32_t* status, cudaStream_t s) {
  plan_kernel<<<1, 1024, (5 * E + 3) * sizeof(int), s>>>(expert_ids, num_post, sorted, N, P, E, bm, tn, nw_gu,
                                                         nw_dn, plan, status);
  return cudaGetLastError();
}


// Shared-memory carve-up of one pipeline stage: two 128-row weight sub-tiles,
// the token rows, and with MX operands the weight sub-tiles' scale chunks and
// the token rows' scale chunks (stages stay 1024-byte aligned for the
// 128-byte swizzle).
struct GemmSmem {
  int stage_bytes;
  int nch;           // MX: 128-row scale chunks of the token tile
};
__host__ __device__ __forceinline__ GemmSmem gemm_smem_layout(int tn, bool mx) {
  GemmSmem g;
  g.nch = (tn + 127) / 128;
  const int b = 2 * kWTileBytes + tn * kStageK + (mx ? (2 + g.nch) * kSfChunk : 0);
  g.stage_bytes = (b + 1023) / 1024 * 1024;
  return g;
}

template <bool kMX>
__global__ void __launch_bounds__(kMX ? kGemmThreadsMx : kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                        GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int E = p.E;
  // stages per tile and elements per stage along K: one 128-byte swizzle row
  const bool byte_ops = kMX || p.fp8;
  const int nk = p.K * (byte_ops ? 1 : 2) / kStageK;
  const int k_elems = byte_ops ? kStageK : kStageK / 2;
  // every tile multiplies two 128-row weight sub-tiles with the same token
  // tile: gate and up rows (gate/up), or output rows n0 and n0+128 (down)
  const int w_bytes = 2 * kWTileBytes;
  const GemmSmem L = gemm_smem_layout(p.tn, kMX);
  const int stage_bytes = L.stage_bytes;
  const int sf_off = w_bytes + p.tn * kStageK;    // MX: weight scale chunks, then token scale chunks
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)p.stages * stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + p.stages;
  uint64_t* acc_full = bars + 2 * p.stages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* t_full = drain + 1;          // [kRing] a tile index was published
  uint64_t* t_empty = t_full + kRing;    // [kRing] every consumer has read it
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(t_empty + kRing);
  int* s_abort = reinterpret_cast<int*>(s_tmem + 1);
  int* s_drain_fail = s_abort + 1;   // a drain after an abort ran out of time
  int* s_ring = s_abort + 2;    // [kRing]
  int* s_start = s_ring + kRing + 1;
  int* s_rows = s_start + E;
  int* s_groups = s_rows + E;
  int* s_perm = s_groups + E;
  int* s_pref = s_perm + E;     // E + 1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < p.stages; ++s) {
      // MX: the 32 lanes of the scale warp also arrive, once their copies land
      mbar_init(&full[s], kMX ? 33 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);
    }
    mbar_init(drain, 1);
    for (int r = 0; r < kRing; ++r) {
      mbar_init(&t_full[r], 1);
      // the MMA thread, the 8 epilogue warps (and the MX scale warp)
      mbar_init(&t_empty[r], kMX ? 10 : 9);
    }
    *s_abort = 0;
    *s_drain_fail = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, p.tmem_cols);
    tmem_relinquish();
  }
  const int pref_off = plan_pref(E, p.gateup != 0);
  for (int i = threadIdx.x; i < E; i += blockDim.x) {
    s_start[i] = p.plan[plan_start(E) + i];
    s_rows[i] = p.plan[plan_real(E) + i];     // real rows per expert (padding excluded)
    s_groups[i] = p.plan[plan_groups(E) + i];
    s_perm[i] = p.plan[plan_perm(E) + i];
  }
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_pref[i] = p.plan[pref_off + i];
  const int n_tiles = p.plan[p.gateup ? PLAN_TILES_GU : PLAN_TILES_DN];
  const int n_hot = p.plan[p.gateup ? PLAN_HOT_GU : PLAN_HOT_DN];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  const int cols_per_acc = 2 * p.tn;
  const int xb = x_box_rows(p.tn);
  volatile int* abort_flag = s_abort;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      // L2 priorities: weights streamed once go first.  Re-read operands stay
      // (evict-last) in the gate/up GEMM; in the down GEMM with the fused
      // combine they are normal, so that the fp32 token rows the epilogue
      // adds into (evict-last) stay in L2.
      const bool keep_out = p.comb_out != nullptr;
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = keep_out ? policy_evict_normal() : policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      long long armed = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        // claim the next tile of the launch and publish it to the MMA and epilogue warps
        const int slot = it % kRing;
        if (!wait_or_abort(&t_empty[slot], ((uint32_t)(it / kRing) & 1u) ^ 1u, p.timeout_ns, abort_flag)) {
          ok = false;
          break;
        }
        const int t = claim_to_tile(atomicAdd(p.tile_counter, 1), n_hot, n_tiles);
        s_ring[slot] = t;
        mbar_arrive(&t_full[slot]);
        if (t >= n_tiles) break;
        const TileInfo ti = decode_tile(t, s_pref, s_perm, s_start, s_rows, s_groups, E, p.tn);
        if (!MOE_IN_BOUNDS(ti.e >= 0 && ti.e < E && ti.r0 >= 0 && ti.r0 + ti.nrows <= p.plan[PLAN_NUM_POST],
                           p.status)) {
          *abort_flag = 2;     // every role stops at its next wait (2: not a timeout)
          ok = false;
          break;
        }
        int row0, row1;
        bool has1 = true;
        if (p.gateup) {
          row0 = ti.e * 2 * p.n_out + ti.wt * kWRows;
          row1 = row0 + p.n_out;
        } else {
          row0 = ti.e * p.n_out + ti.wt * 2 * kWRows;
          row1 = row0 + kWRows;
          has1 = ti.wt * 2 * kWRows + kWRows < p.n_out;
        }
        const int nload = (ti.nrows + xb - 1) / xb;
        // a packed E2M1 weight box fills 16 KB of shared memory but completes
        // only its 8 KB of codes as transaction bytes
        const int w_tx = (kMX && p.w_fp4) ? kWTileBytes / 2 : kWTileBytes;
        const uint32_t tx = (has1 ? 2 : 1) * (w_tx + (kMX ? kSfChunk : 0)) + nload * xb * kStageK;
        // weights streamed once (one token group) go first; re-read ones stay in L2
        const uint64_t pol_wt = s_groups[ti.e] > 1 ? pol_x : pol_w;
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_or_abort(&empty[stage], phase ^ 1, p.timeout_ns, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sb = smem + (size_t)stage * stage_bytes;
          mbar_arrive_expect_tx(&full[stage], tx);
          const int kc = kb * k_elems;
          tma_load_2d(sb, &tm_w, &full[stage], kc, row0, pol_wt);
          if (has1) tma_load_2d(sb + kWTileBytes, &tm_w, &full[stage], kc, row1, pol_wt);
          for (int l = 0; l < nload; ++l)
            tma_load_2d(sb + w_bytes + l * xb * kStageK, &tm_x, &full[stage], kc, ti.r0 + l * xb, pol_x);
          if (kMX) {
            // the weight sub-tiles' scale chunks (128 rows x 4 K-blocks, 512 bytes each)
            uint8_t* sa = sb + sf_off;
            bulk_load(sa, p.w_sf + ((size_t)(row0 / kWRows) * nk + kb) * kSfChunk, kSfChunk, &full[stage]);
            if (has1)
              bulk_load(sa + kSfChunk, p.w_sf + ((size_t)(row1 / kWRows) * nk + kb) * kSfChunk, kSfChunk,
                        &full[stage]);
          }
          ++armed;
          if (++stage == p.stages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // let every copy already issued land before the CTA exits
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
      int it = 0;
      bool ok = true;
      bool issued = false;
      const uint32_t fmt = p.fp8 ? 0u : 1u;
      const uint32_t a_fmt_mx = p.w_fp4 ? 5u : 0u;   // E2M1 or E4M3 weights; activations E4M3
      // MX scale factors in TMEM after the accumulators: weight sub-tiles 0/1, then the token tile
      const uint32_t sf_col = tmem_base + (uint32_t)(p.n_acc * cols_per_acc);
      for (;; ++it) {
        const int slot = it % kRing;
        if (!wait_or_abort(&t_full[slot], (uint32_t)(it / kRing) & 1u, p.timeout_ns, abort_flag)) {
          ok = false;
          break;
        }
        const int t = s_ring[slot];
        mbar_arrive(&t_empty[slot]);
        if (t >= n_tiles) break;
        const TileInfo ti = decode_tile(t, s_pref, s_perm, s_start, s_rows, s_groups, E, p.tn);
        const bool has1 = p.gateup || ti.wt * 2 * kWRows + kWRows < p.n_out;
        const int acc = it % p.n_acc;
        const uint32_t acc_phase = (uint32_t)(it / p.n_acc) & 1u;
        if (!wait_or_abort(&acc_empty[acc], acc_phase ^ 1, p.timeout_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * cols_per_acc);
        const uint32_t d1 = d0 + (uint32_t)p.tn;
        const int n_mma = ((ti.nrows + 15) / 16) * 16;
        const uint32_t idesc = umma_idesc(kWRows, n_mma, fmt);
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_or_abort(&full[stage], phase, p.timeout_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w0 = smem_u32(smem + (size_t)stage * stage_bytes);
          const uint32_t w1 = w0 + kWTileBytes;
          const uint32_t xa = w0 + (uint32_t)w_bytes;
          if (kMX) {
            // this stage's scale factors into TMEM (executed in order with the MMAs below)
            const uint32_t sa = w0 + (uint32_t)sf_off;
            tmem_cp_32x128b_x4(sf_col, umma_desc_rows16(sa));
            if (has1) tmem_cp_32x128b_x4(sf_col + 4, umma_desc_rows16(sa + kSfChunk));
            for (int c = 0; c < L.nch; ++c)
              tmem_cp_32x128b_x4(sf_col + 8 + 4 * c, umma_desc_rows16(sa + (2 + c) * kSfChunk));
          }
#pragma unroll
          for (int kk = 0; kk < kStageK / 32; ++kk) {
            const uint64_t bdesc = umma_desc_sw128(xa + kk * 32);
            const uint32_t accum = (kb | kk) != 0;
            if (kMX) {
              const uint32_t idx = umma_idesc_mx(kWRows, n_mma, a_fmt_mx, 0u, (uint32_t)kk);
              const uint32_t sel = (uint32_t)kk << 30;     // byte kk of each scale word
              mma_mx(d0, umma_desc_sw128(w0 + kk * 32), bdesc, idx, sf_col | sel, (sf_col + 8) | sel, accum);
              if (has1)
                mma_mx(d1, umma_desc_sw128(w1 + kk * 32), bdesc, idx, (sf_col + 4) | sel, (sf_col + 8) | sel,
                       accum);
            } else {
              if (p.fp8) mma_e4m3(d0, umma_desc_sw128(w0 + kk * 32), bdesc, idesc, accum);
              else mma_bf16(d0, umma_desc_sw128(w0 + kk * 32), bdesc, idesc, accum);
              if (has1) {
                if (p.fp8) mma_e4m3(d1, umma_desc_sw128(w1 + kk * 32), bdesc, idesc, accum);
                else mma_bf16(d1, umma_desc_sw128(w1 + kk * 32), bdesc, idesc, accum);
              }
            }
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
        // wait for the MMAs in flight before TMEM is freed
        tc_commit(drain);
        if (!mbar_wait(drain, 0, kDrainTimeoutNs)) *s_drain_fail = 1;
      }
    }
  } else if (warp < 10) {
    // ---------------- epilogue: warps 2..9 ----------------
    // two warps per TMEM lane quarter (a warp may only read lanes 32*(warp%4)..+31);
    // they take alternate 16-column chunks
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int m = 32 * q + lane;
    for (int it = 0;; ++it) {
      const int slot = it % kRing;
      if (!wait_or_abort(&t_full[slot], (uint32_t)(it / kRing) & 1u, p.timeout_ns, abort_flag)) break;
      const int t = s_ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[slot]);
      if (t >= n_tiles) break;
      const TileInfo ti = decode_tile(t, s_pref, s_perm, s_start, s_rows, s_groups, E, p.tn);
      const int acc = it % p.n_acc;
      const uint32_t acc_phase = (uint32_t)(it / p.n_acc) & 1u;
      if (!wait_or_abort(&acc_full[acc], acc_phase, p.timeout_ns, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * cols_per_acc);
      if (p.gateup) {
        const int n = ti.wt * kWRows + m;
        float sg = 1.f, su = 1.f;
        if (p.fp8) {
          sg = __ldg(p.w_scale + (long long)ti.e * 2 * p.n_out + n);
          su = __ldg(p.w_scale + (long long)ti.e * 2 * p.n_out + p.n_out + n);
        }
        __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(p.out);
        for (int c = 16 * half; c < ti.nrows; c += 32) {
          float g[16], u[16];
          // lanes 0..15 fetch the chunk's row scales; shuffles broadcast them
          const float sa_l = (p.fp8 && lane < 16 && c + lane < ti.nrows) ? __ldg(p.a_scale + ti.r0 + c + lane) : 1.f;
          tmem_ld16(tb + c, g);
          tmem_ld16(tb + p.tn + c, u);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int j = c + i;
            const float sa = __shfl_sync(0xffffffffu, sa_l, i);
            if (j < ti.nrows) {
              const int row = ti.r0 + j;
              float gv = g[i], uv = u[i];
              if (p.fp8) {
                gv = gv * sa * sg;
                uv = uv * sa * su;
              }
              const float hv = __fdividef(gv, 1.f + __expf(-gv)) * uv;   // silu(g) * u
              if (kMX) {
                // h rounded to bf16, then MX-quantised: the warp's 32 lanes hold the
                // 32 consecutive features of one MX block of this row
                const float hb = __bfloat162float(__float2bfloat16_rn(hv));
                const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(hb) & 0x7FFFFFFFu);
                const int code = mx_e8m0_code(amax);
                const __nv_fp8_storage_t qv = __nv_cvt_float_to_fp8(hb * mx_inv_scale(code), __NV_SATFINITE,
                                                                   __NV_E4M3);
                reinterpret_cast<uint8_t*>(p.out)[(long long)row * p.n_out + n] = (uint8_t)qv;
                if (lane == 0) p.h_sf[(long long)row * (p.n_out / 32) + (n >> 5)] = (uint8_t)code;
              } else {
                h[(long long)row * p.n_out + n] = __float2bfloat16_rn(hv);
              }
            }
          }
        }
      } else {
        const int n0 = ti.wt * 2 * kWRows + m;
        const int n1 = n0 + kWRows;
        const bool has1 = n1 < p.n_out;   // uniform across the warp (n_out % 128 == 0)
        float sw0 = 1.f, sw1 = 1.f;
        if (p.fp8) {
          sw0 = __ldg(p.w_scale + (long long)ti.e * p.n_out + n0);
          if (has1) sw1 = __ldg(p.w_scale + (long long)ti.e * p.n_out + n1);
        }
        float* o = reinterpret_cast<float*>(p.out);
        const bool fused = p.comb_out != nullptr;
        const uint64_t pol_out = policy_evict_last();
        for (int c = 16 * half; c < ti.nrows; c += 32) {
          float v0[16], v1[16];
          // lanes 0..15 fetch the chunk's slots (row scales, routing weights); shuffles broadcast them
          const bool in = lane < 16 && c + lane < ti.nrows;
          const int slot_l = in ? __ldg(p.sorted + ti.r0 + c + lane) : p.n_slots;
          const float sa_l = (p.fp8 && in) ? __ldg(p.a_scale + ti.r0 + c + lane) : 1.f;
          // a negative slot id is invalid (debug builds report it); like padding it writes nothing
          const bool valid_l = (unsigned)slot_l < (unsigned)p.n_slots;
          const float wt_l = (fused && valid_l) ? __ldg(p.comb_w + slot_l) : 0.f;
          tmem_ld16(tb + c, v0);
          if (has1) tmem_ld16(tb + p.tn + c, v1);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int slot = __shfl_sync(0xffffffffu, slot_l, i);
            const float sa = __shfl_sync(0xffffffffu, sa_l, i);
            const float wt = __shfl_sync(0xffffffffu, wt_l, i);
            if (c + i < ti.nrows && MOE_IN_BOUNDS(slot >= 0, p.status) && (unsigned)slot < (unsigned)p.n_slots) {
              const float a0 = p.fp8 ? v0[i] * sa * sw0 : v0[i];
              const float a1 = p.fp8 ? v1[i] * sa * sw1 : v1[i];
              if (fused) {
                // the warp's 32 lanes add to 32 consecutive floats of the token's row
                float* orow = p.comb_out + (long long)(slot / p.k) * p.n_out;
                red_add_f32(orow + n0, wt * a0, pol_out);
                if (has1) red_add_f32(orow + n1, wt * a1, pol_out);
              } else {
                float* yr = o + (long long)slot * p.n_out;
                yr[n0] = a0;
                if (has1) yr[n1] = a1;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  } else if (kMX) {
    // ---------------- MX scale warp (warp 10) ----------------
    // For every stage the producer fills, copies the token rows' scales of
    // its 4 K-blocks (one 32-bit word per row) into the stage's token scale
    // chunks, in the layout tcgen05.cp reads: chunk c, byte
    // (n % 32) * 16 + ((n % 128) / 32) * 4 + b holds row 128c + n's scale of
    // K-block 4 * stage + b.  The copies are cp.async (fire and forget); each
    // lane's arrive on the stage's full barrier fires when its copies have
    // landed.  Rows past the token group are not written: the MMA columns
    // they scale are never read.
    int stage = 0;
    uint32_t phase = 0;
    for (int it = 0;; ++it) {
      const int slot = it % kRing;
      if (!wait_or_abort(&t_full[slot], (uint32_t)(it / kRing) & 1u, p.timeout_ns, abort_flag)) break;
      const int t = s_ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[slot]);
      if (t >= n_tiles) break;
      const TileInfo ti = decode_tile(t, s_pref, s_perm, s_start, s_rows, s_groups, E, p.tn);
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        if (!wait_or_abort(&empty[stage], phase ^ 1, p.timeout_ns, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t dst = smem_u32(smem + (size_t)stage * stage_bytes + sf_off + 2 * kSfChunk);
        for (int n = lane; n < ti.nrows; n += 32) {
          const uint32_t off = (uint32_t)((n >> 7) * kSfChunk + (n & 31) * 16 + ((n >> 5) & 3) * 4);
          cp_async_4(dst + off, p.x_sf + (size_t)(ti.r0 + n) * (p.K / 32) + (size_t)kb * 4);
        }
        cp_async_mbar_arrive_noinc(&full[stage]);
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
    }
    cp_async_wait_all();   // no copy of this warp may land after the CTA exits
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag == 1) dev_flag(p.status, MOE_DEV_TIMEOUT);
  if (threadIdx.x == 0 && *s_drain_fail) dev_flag(p.status, MOE_DEV_DRAIN_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t gemm_smem_bytes(int tn, int stages, int E, bool mx) {
  const GemmSmem L = gemm_smem_layout(tn, mx);
  return 1024 + (size_t)stages * L.stage_bytes + (2 * stages + 5 + 2 * kRing) * 8 + (kRing + 4) * 4 +
         (size_t)(5 * E + 1) * 4;
}

int gemm_pick_stages(int tn, int E, bool mx) {
  int s = 8;
  while (s > 2 && gemm_smem_bytes(tn, s, E, mx) > 225 * 1024) --s;
  return s;
}

int launch_grouped_gemm(GemmLaunch& L, cudaStream_t stream) {
  GemmParams& p = L.p;
  const bool mx = p.mx != 0;
  const int eb = (p.fp8 || mx) ? 1 : 2;
  CUtensorMap tw, tx;
  if (!make_map(&tw, L.w, L.w_rows, p.K, mx && p.w_fp4 ? 0 : eb, kWRows)) return -1;
  if (!make_map(&tx, L.x, L.x_rows, p.K, eb, p.tn < 32 ? p.tn : 32)) return -1;
  p.stages = gemm_pick_stages(p.tn, p.E, mx);
  const int cols = 2 * p.tn;
  const int sf_cols = mx ? 8 + 4 * ((p.tn + 127) / 128) : 0;   // MX scale factors after the accumulators
  p.n_acc = 2 * cols + sf_cols <= 512 ? 2 : 1;
  int need = p.n_acc * cols + sf_cols, alloc = 32;
  while (alloc < need) alloc <<= 1;
  p.tmem_cols = alloc;
  const size_t smem = gemm_smem_bytes(p.tn, p.stages, p.E, mx);
  const void* fn = mx ? (const void*)grouped_gemm_kernel<true> : (const void*)grouped_gemm_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (mx)
    grouped_gemm_kernel<true><<<sms, kGemmThreadsMx, smem, stream>>>(tw, tx, p);
  else
    grouped_gemm_kernel<false><<<sms, kGemmThreads, smem, stream>>>(tw, tx, p);
  return (int)cudaGetLastError();
}

}  // namespace moe
