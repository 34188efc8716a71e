// Tile plan of the grouped GEMMs, written on the device from the align & sort
// outputs (by the fused routing kernel's last step, or by plan_kernel for the
// stand-alone FFN), so that no host synchronisation sits between routing and
// the GEMMs.
//
// A tile is (expert, weight tile, token group): up to tn sorted rows of one
// expert times one weight tile.  Experts with at least two token groups
// ("hot": their weight tiles are re-read from L2 by the later groups, so
// their tiles are mostly tensor-bound) are listed first, the others ("cold":
// every tile streams its weights from HBM) after them; both in expert order.
// The GEMMs interleave the two lists (plan_claim_to_tile) so that hot and
// cold tiles run side by side instead of in separate phases.
#pragma once
#include "kernels.cuh"

namespace moe {

// Exclusive scan of a[0..n) in shared memory by the whole CTA; returns the total.
__device__ inline int block_exclusive_scan(int* a, int n) {
  __shared__ int s_warp[32];
  __shared__ int s_total;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthr = blockDim.x;
  const int ipt = (n + nthr - 1) / nthr;
  const int beg = min(n, tid * ipt), end = min(n, beg + ipt);
  int local = 0;
  for (int i = beg; i < end; ++i) local += a[i];
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int nw = nthr >> 5;
    int v = lane < nw ? s_warp[lane] : 0;
    int vi = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, vi, off);
      if (lane >= off) vi += u;
    }
    if (lane < nw) s_warp[lane] = vi - v;
    if (lane == nw - 1) s_total = vi;
  }
  __syncthreads();
  int run = s_warp[warp] + incl - local;
  for (int i = beg; i < end; ++i) {
    int v = a[i];
    a[i] = run;
    run += v;
  }
  __syncthreads();
  return s_total;
}

// Second half of the plan, by the whole CTA, once plan[PLAN_START..],
// plan[PLAN_ROWS..] and s_g[e] = token groups of expert e are in place.
// sc: shared scratch of at least 3E + 2 ints.
__device__ inline void finish_plan(int32_t* plan, const int* s_g, int E, int nw_gu, int nw_dn, int tn,
                                   int num_post, int* sc) {
  int* s_hot = sc;                 // [E] hot flag -> hot experts before e
  int* s_pg = sc + E;              // [E+1] per list position: gate/up tiles -> prefix
  int* s_pd = sc + 2 * E + 1;      // [E+1] down tiles -> prefix
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) {
    plan[plan_groups(E) + e] = s_g[e];
    s_hot[e] = s_g[e] >= 2 ? 1 : 0;
  }
  __syncthreads();
  const int n_hot = block_exclusive_scan(s_hot, E);
  for (int e = tid; e < E; e += blockDim.x) {
    const bool hot = s_g[e] >= 2;
    const int pos = hot ? s_hot[e] : n_hot + (e - s_hot[e]);
    plan[plan_perm(E) + pos] = e;
    s_pg[pos] = s_g[e] * nw_gu;
    s_pd[pos] = s_g[e] * nw_dn;
  }
  __syncthreads();
  const int tg = block_exclusive_scan(s_pg, E);
  const int td = block_exclusive_scan(s_pd, E);
  for (int i = tid; i < E; i += blockDim.x) {
    plan[plan_pref(E, true) + i] = s_pg[i];
    plan[plan_pref(E, false) + i] = s_pd[i];
  }
  if (tid == 0) {
    plan[plan_pref(E, true) + E] = tg;
    plan[plan_pref(E, false) + E] = td;
    plan[PLAN_TILES_GU] = tg;
    plan[PLAN_TILES_DN] = td;
    plan[PLAN_TN] = tn;
    plan[PLAN_NUM_POST] = num_post;
    plan[PLAN_HOT_GU] = n_hot < E ? s_pg[n_hot] : tg;
    plan[PLAN_HOT_DN] = n_hot < E ? s_pd[n_hot] : td;
    plan[PLAN_COUNTER_GU] = 0;
    plan[PLAN_COUNTER_DN] = 0;
  }
  __syncthreads();
}

}  // namespace moe
