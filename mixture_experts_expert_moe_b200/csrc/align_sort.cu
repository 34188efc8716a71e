// MoE Align & Sort on sm_100a: one cooperative launch, one grid-wide wait.
//
// Follows the D-C-P structure of the MoE Align & Sort article (dignews.cc,
// section "Writing AMD-friendly CUDA code with 3x~7x speed-up"):
//   (D) distributed concurrent counting: every CTA counts the expert ids of
//       its contiguous chunk of flat slots.  Inside a CTA every warp owns a
//       contiguous sub-chunk and a private histogram row in shared memory
//       (shared-memory atomics; counting needs no order).
//   (C) cumulative sums: the warp rows are scanned into per-warp exclusive
//       prefixes (the article's "unaligned local cumsum"), the CTA totals go
//       to a global matrix hist[expert][cta] (the "merge" through a
//       preallocated HBM buffer), and after the single grid-wide wait every
//       CTA reads each expert's row with coalesced warp loads to get its own
//       prefix and the expert totals, pads the totals to the block size and
//       scans them (the "aligned global cumsum").
//   (P) parallel placement: each warp re-reads its sub-chunk and writes every
//       slot to  offset[e] + (slots of e in earlier CTAs) + (in earlier warps)
//       + (earlier in this warp), which is the stable counting-sort position.
//       Block expert ids and the sentinel padding (only in an expert's last
//       block) are written by the CTA that owns the block.
// Unlike the article's design there is no second kernel and no single-block
// alignment step: every CTA redoes the small E-wide scan itself, which costs
// less than another launch or grid-wide wait.  The same kernel, instantiated
// with gating in front and the GEMM tile plan behind, is the single routing
// launch of moe_forward; with one CTA (small batches) it needs no grid-wide
// wait at all.
#include <atomic>

#include "gate.cuh"
#include "kernels.cuh"
#include "plan.cuh"

namespace moe {

constexpr int kAlignThreads = 1024;
constexpr int kAlignWarps = kAlignThreads / 32;
constexpr int kSub = 8;  // 32-slot sub-steps a warp loads before it processes them

// Grid-wide wait with a time limit; returns false if it ran out.
__device__ bool grid_wait(int* counter, int expected, long long timeout_ns) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(counter, 1);
    int ok = 1;
    unsigned long long t0 = globaltimer_ns();
    while (ld_acquire_gpu(counter) < expected) {
      __nanosleep(64);
      if ((long long)(globaltimer_ns() - t0) > timeout_ns) {
        ok = 0;
        break;
      }
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// Issues the loads of kSub sub-steps (32 consecutive slots each) of a warp's
// sub-chunk without using the values, so they can be in flight while the
// previous sub-steps are processed.  Plain (L2) loads: in the fused routing
// kernel the ids were written earlier in the same launch.
__device__ __forceinline__ void load_raw(const int32_t* ids, long long base, long long end, int lane,
                                         int (&key)[kSub]) {
#pragma unroll
  for (int q = 0; q < kSub; ++q) {
    const long long i = base + q * 32 + lane;
    key[q] = i < end ? __ldcg(ids + i) : -1;
  }
}

// Lanes of the warp holding the same value v in [0, 2^kBits): one ballot per
// bit, all independent, so they issue back to back.
template <int kBits>
__device__ __forceinline__ unsigned match_peers(int v) {
  unsigned ones[kBits];
#pragma unroll
  for (int b = 0; b < kBits; ++b) ones[b] = __ballot_sync(0xffffffffu, (v >> b) & 1);
  unsigned peers = 0xffffffffu;
#pragma unroll
  for (int b = 0; b < kBits; ++b) peers &= ((v >> b) & 1) ? ones[b] : ~ones[b];
  return peers;
}

template <int N>
struct Log2 {
  static constexpr int value = 1 + Log2<N / 2>::value;
};
template <>
struct Log2<1> {
  static constexpr int value = 0;
};

// ids outside [0, E) and slots past the end become -1; returns whether an id
// was out of range.
__device__ __forceinline__ bool validate_keys(long long base, long long end, int lane, int E, int (&key)[kSub]) {
  bool bad = false;
#pragma unroll
  for (int q = 0; q < kSub; ++q) {
    const long long i = base + q * 32 + lane;
    if (i < end && (key[q] < 0 || key[q] >= E)) {
      bad = true;
      key[q] = -1;
    }
  }
  return bad;
}

// EPL = ceil(E/32) rounded up to a power of two (the gating's logits per lane
// and the width of the id matching).  kGate: the CTA first gates the tokens
// whose slots it owns (its chunk is a multiple of the slots per token) and
// writes ids/weights.  kPlan: CTA 0 finally writes the
// grouped GEMMs' tile plan from the padded offsets.  With one CTA there is no
// grid-wide wait.
template <int EPL, bool kGate, bool kPlan>
__global__ void __launch_bounds__(kAlignThreads, 1) route_kernel(AlignParams p, RouteExtra r) {
  extern __shared__ int smem[];
  const int E = p.E;
  const int G = gridDim.x;
  int* wcnt = smem;                       // [kAlignWarps][E] per-warp counts, then prefixes
  int* s_off = wcnt + kAlignWarps * E;    // [E] padded segment offsets
  int* s_base = s_off + E;                // [E] this CTA's first position per expert
  int* s_tot = s_base + E;                // [E] expert totals
  __shared__ int s_bad;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kAlignWarps * E; i += blockDim.x) wcnt[i] = 0;
  if (tid == 0) s_bad = 0;

  const long long cta_begin = (long long)blockIdx.x * p.chunk;
  if (kGate) {
    // ---- gating of this CTA's tokens (warp per token) ----------------------
    const int kk = r.k + r.n_shared;   // slots per token
    const long long t0 = cta_begin / kk;
    const long long t1 = min((long long)r.T, (cta_begin + p.chunk) / kk);
    for (long long t = t0 + warp; t < t1; t += kAlignWarps)
      gate_token<EPL>(r.logits, r.bias, r.select_only != 0, t, r.E_routed, r.k, r.n_shared, r.ids_out, r.w_out,
                      lane);
  }
  __syncthreads();

  const int wsub = p.chunk / kAlignWarps;
  const long long w_begin = cta_begin + (long long)warp * wsub;
  const long long w_end = min((long long)p.N, w_begin + wsub);
  int* my = wcnt + warp * E;

  // ---- (D) count: each warp into its own row (shared-memory atomics) -----
  // the next step's ids are loaded while the current ones are counted
  bool bad = false;
  {
    int key[kSub], nxt[kSub];
    if (w_begin < w_end) load_raw(p.ids, w_begin, w_end, lane, key);
    for (long long base = w_begin; base < w_end; base += 32 * kSub) {
      if (base + 32 * kSub < w_end) load_raw(p.ids, base + 32 * kSub, w_end, lane, nxt);
      bad |= validate_keys(base, w_end, lane, E, key);
#pragma unroll
      for (int q = 0; q < kSub; ++q)
        if (key[q] >= 0) atomicAdd(&my[key[q]], 1);
#pragma unroll
      for (int q = 0; q < kSub; ++q) key[q] = nxt[q];
    }
  }
  if (bad) s_bad = 1;
  __syncthreads();
  if (tid == 0 && s_bad) dev_flag(p.status, MOE_DEV_BAD_EXPERT_ID);

  // per-warp exclusive prefixes inside the CTA; CTA totals to column b of hist[e][b]
  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll 8
    for (int w = 0; w < kAlignWarps; ++w) {
      const int c = wcnt[w * E + e];
      wcnt[w * E + e] = run;
      run += c;
    }
    if (G > 1) p.hist[(long long)e * G + blockIdx.x] = run;
    else {
      s_tot[e] = run;
      s_base[e] = 0;
      s_off[e] = (run + p.bm - 1) / p.bm * p.bm;
    }
  }

  if (G > 1) {
    if (!grid_wait(p.barrier, p.expected, p.timeout_ns)) {
      if (tid == 0) dev_flag(p.status, MOE_DEV_TIMEOUT);
      return;
    }
    // ---- (C) own prefix and expert totals from row e of hist ----------------
    // warp w reduces experts w, w+32, ...; lane l reads CTAs l, l+32, ...
    for (int e0 = warp; e0 < E; e0 += kAlignWarps * 8) {
      int pre[8], tot[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) pre[u] = tot[u] = 0;
      for (int c = 0; c < G; c += 32) {
        const int b = c + lane;
        int v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = e0 + u * kAlignWarps;
          v[u] = (e < E && b < G) ? __ldcg(p.hist + (long long)e * G + b) : 0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          pre[u] += b < (int)blockIdx.x ? v[u] : 0;
          tot[u] += v[u];
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          pre[u] += __shfl_xor_sync(0xffffffffu, pre[u], off);
          tot[u] += __shfl_xor_sync(0xffffffffu, tot[u], off);
        }
        const int e = e0 + u * kAlignWarps;
        if (lane == 0 && e < E) {
          s_tot[e] = tot[u];
          s_base[e] = pre[u];
          s_off[e] = (tot[u] + p.bm - 1) / p.bm * p.bm;
        }
      }
    }
  }
  __syncthreads();
  const int total_post = block_exclusive_scan(s_off, E);
  for (int e = tid; e < E; e += blockDim.x) s_base[e] += s_off[e];
  if (blockIdx.x == 0 && tid == 0) *p.num_post = total_post;
  __syncthreads();

  // ---- block expert ids and sentinel padding for this CTA's blocks -------
  const int nblk = total_post / p.bm;
  const int bpc = (nblk + G - 1) / G;
  const int j0 = blockIdx.x * bpc;
  const int j1 = min(nblk, j0 + bpc);
  for (int j = j0 + tid; j < j1; j += blockDim.x) {   // one thread per block
    const int pos = j * p.bm;
    int lo = 0, hi = E - 1;  // last expert whose segment starts at or before pos
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= pos) lo = mid; else hi = mid - 1;
    }
    p.expert_ids[j] = lo;
  }
  // padding (only in an expert's last block): the part inside this CTA's blocks
  for (int e = warp; e < E; e += kAlignWarps) {
    const int beg = max(s_off[e] + s_tot[e], j0 * p.bm);
    const int end = min(s_off[e] + (s_tot[e] + p.bm - 1) / p.bm * p.bm, j1 * p.bm);
    for (int q = beg + lane; q < end; q += 32) p.sorted[q] = p.N;
  }

  // ---- (P) stable placement ------------------------------------------------
  // Ranks: the lowest lane of each group of equal ids takes the group's
  // positions with one shared-memory atomicAdd on the warp's row (it returns
  // the running count) and shares it by a shuffle.  Leaders of one expert in
  // consecutive sub-steps can be different lanes: a __syncwarp between the
  // sub-steps orders their atomics (it is a memory fence among the warp's
  // lanes), so equal ids keep the order of the sub-steps.
  {
    int key[kSub], nxt[kSub];
    if (w_begin < w_end) load_raw(p.ids, w_begin, w_end, lane, key);
    for (long long base = w_begin; base < w_end; base += 32 * kSub) {
      if (base + 32 * kSub < w_end) load_raw(p.ids, base + 32 * kSub, w_end, lane, nxt);
      validate_keys(base, w_end, lane, E, key);
      int dest[kSub];
#pragma unroll
      for (int q = 0; q < kSub; ++q) {
        const int kq = key[q];
        // ids + 1 are in [0, 32*EPL]: Log2<32*EPL> + 1 bits (-1, no slot, becomes 0)
        const unsigned peers = match_peers<Log2<32 * EPL>::value + 1>(kq + 1);
        const int leader = __ffs(peers) - 1;
        int old = 0;
        if (kq >= 0 && lane == leader) old = atomicAdd(&my[kq], __popc(peers));
        old = __shfl_sync(0xffffffffu, old, leader);
        dest[q] = kq >= 0 ? s_base[kq] + old + __popc(peers & lanemask_lt()) : -1;
        __syncwarp();
      }
#pragma unroll
      for (int q = 0; q < kSub; ++q)
        if (dest[q] >= 0 && MOE_IN_BOUNDS(dest[q] < p.N + p.E * (p.bm - 1), p.status))
          p.sorted[dest[q]] = (int)(base + q * 32 + lane);
#pragma unroll
      for (int q = 0; q < kSub; ++q) key[q] = nxt[q];
    }
  }

  if (kPlan && blockIdx.x == 0) {
    // ---- tile plan of the grouped GEMMs (layout in kernels.cuh) --------------
    __syncthreads();
    int* s_g = wcnt;               // token groups per expert
    int* sc = wcnt + E;            // 3E + 2 ints of scratch (wcnt holds 32E)
    for (int e = tid; e < E; e += blockDim.x) {
      const int rows = (s_tot[e] + p.bm - 1) / p.bm * p.bm;
      r.plan[plan_start(E) + e] = s_off[e];
      r.plan[plan_rows(E) + e] = rows;
      r.plan[plan_real(E) + e] = s_tot[e];
      s_g[e] = (rows + r.tn - 1) / r.tn;
    }
    __syncthreads();
    finish_plan(r.plan, s_g, E, r.nw_gu, r.nw_dn, r.tn, total_post, sc);
  }
}

// Routing of at most 32 slots (decode: a few tokens), one CTA of 8 warps.
// The same outputs as route_kernel<EPL, true, true> with one CTA, in fewer
// steps: warps gate the tokens; warp 0 holds slot l in lane l, groups equal
// expert ids with one match (the group size is the expert's count, the
// lanes below in the group give the stable rank); the padded counts of all
// E experts are scanned into segment offsets; block ids, sentinels and the
// placement follow; the tile plan as in route_kernel.
constexpr int kSmallRouteSlots = 32;
constexpr int kSmallRouteThreads = 256;

template <int EPL>
__global__ void __launch_bounds__(kSmallRouteThreads, 1) route_small_kernel(AlignParams p, RouteExtra r) {
  extern __shared__ int smem[];
  const int E = p.E;
  int* s_tot = smem;         // [E] slots per expert
  int* s_off = s_tot + E;    // [E] padded counts, then segment offsets
  int* s_g = s_off + E;      // [E] padded counts, then token groups per expert
  int* sc = s_g + E;         // [3E + 2] scratch of finish_plan
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  for (int e = tid; e < E; e += blockDim.x) s_tot[e] = 0;
  if (r.zero_out) {   // in place of a memset launch
    float4* z = reinterpret_cast<float4*>(r.zero_out);
    for (long long i = tid; i < r.zero_n / 4; i += blockDim.x) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int t = warp; t < r.T; t += nwarps)
    gate_token<EPL>(r.logits, r.bias, r.select_only != 0, t, r.E_routed, r.k, r.n_shared, r.ids_out, r.w_out,
                    lane);
  __syncthreads();   // the ids (global, written by this CTA) and the zeroed counts

  // warp 0: slot `lane`'s expert, its stable rank among the slots of that expert
  int key = -1, rank = 0;
  if (warp == 0) {
    key = lane < p.N ? __ldcg(p.ids + lane) : -1;
    const bool bad = lane < p.N && (key < 0 || key >= E);
    if (bad) key = -1;
    if (__any_sync(0xffffffffu, bad) && lane == 0) dev_flag(p.status, MOE_DEV_BAD_EXPERT_ID);
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    rank = __popc(peers & lanemask_lt());
    if (key >= 0 && rank == 0) s_tot[key] = __popc(peers);   // one lane per expert
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    const int rows = (s_tot[e] + p.bm - 1) / p.bm * p.bm;
    s_off[e] = rows;
    s_g[e] = rows;
  }
  __syncthreads();   // the scan reads other threads' entries
  const int total_post = block_exclusive_scan(s_off, E);
  if (tid == 0) *p.num_post = total_post;

  // block expert ids: the last expert whose segment starts at or before the block
  const int nblk = total_post / p.bm;
  for (int j = tid; j < nblk; j += blockDim.x) {
    const int pos = j * p.bm;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= pos) lo = mid; else hi = mid - 1;
    }
    p.expert_ids[j] = lo;
  }
  if (warp == 0 && key >= 0 && MOE_IN_BOUNDS(s_off[key] + rank < p.N + p.E * (p.bm - 1), p.status))
    p.sorted[s_off[key] + rank] = lane;
  // per expert (one thread each): the sentinel padding at the end of its
  // segment (at most block_size - 1 entries; none for most experts) and its
  // entries of the tile plan
  for (int e = tid; e < E; e += blockDim.x) {
    const int start = s_off[e], real = s_tot[e], rows = s_g[e];
    for (int q = start + real; q < start + rows; ++q) p.sorted[q] = p.N;
    r.plan[plan_start(E) + e] = start;
    r.plan[plan_rows(E) + e] = rows;
    r.plan[plan_real(E) + e] = real;
    s_g[e] = (rows + r.tn - 1) / r.tn;
  }
  __syncthreads();
  finish_plan(r.plan, s_g, E, r.nw_gu, r.nw_dn, r.tn, total_post, sc);
}

size_t align_smem_bytes(int E) { return (size_t)(kAlignWarps + 3) * E * sizeof(int); }

template <typename K>
static cudaError_t launch_route_impl(K kernel, const AlignParams& p, const RouteExtra& r, int grid,
                                     cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)align_smem_bytes(1024));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kAlignThreads);
  cfg.dynamicSmemBytes = align_smem_bytes(p.E);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p, r);
}

cudaError_t launch_align_sort(const AlignParams& p, int grid, cudaStream_t stream) {
  RouteExtra r = {};
  const int epl = (p.E + 31) / 32;
  if (epl <= 1) return launch_route_impl(route_kernel<1, false, false>, p, r, grid, stream);
  if (epl <= 2) return launch_route_impl(route_kernel<2, false, false>, p, r, grid, stream);
  if (epl <= 4) return launch_route_impl(route_kernel<4, false, false>, p, r, grid, stream);
  if (epl <= 8) return launch_route_impl(route_kernel<8, false, false>, p, r, grid, stream);
  if (epl <= 16) return launch_route_impl(route_kernel<16, false, false>, p, r, grid, stream);
  return launch_route_impl(route_kernel<32, false, false>, p, r, grid, stream);
}

template <typename K>
static cudaError_t launch_route_small(K kernel, const AlignParams& p, const RouteExtra& r, cudaStream_t stream) {
  const size_t smem = (size_t)(6 * p.E + 2) * sizeof(int);   // <= 24.6 KB at E = 1024
  kernel<<<1, kSmallRouteThreads, smem, stream>>>(p, r);
  return cudaGetLastError();
}

bool route_zeroes(long long N) { return N <= kSmallRouteSlots; }

cudaError_t launch_route(const AlignParams& p, const RouteExtra& r, int grid, cudaStream_t stream) {
  const int epl = (p.E + 31) / 32;
  if (route_zeroes(p.N)) {
    if (epl <= 1) return launch_route_small(route_small_kernel<1>, p, r, stream);
    if (epl <= 2) return launch_route_small(route_small_kernel<2>, p, r, stream);
    if (epl <= 4) return launch_route_small(route_small_kernel<4>, p, r, stream);
    if (epl <= 8) return launch_route_small(route_small_kernel<8>, p, r, stream);
    if (epl <= 16) return launch_route_small(route_small_kernel<16>, p, r, stream);
    return launch_route_small(route_small_kernel<32>, p, r, stream);
  }
  if (epl <= 1) return launch_route_impl(route_kernel<1, true, true>, p, r, grid, stream);
  if (epl <= 2) return launch_route_impl(route_kernel<2, true, true>, p, r, grid, stream);
  if (epl <= 4) return launch_route_impl(route_kernel<4, true, true>, p, r, grid, stream);
  if (epl <= 8) return launch_route_impl(route_kernel<8, true, true>, p, r, grid, stream);
  if (epl <= 16) return launch_route_impl(route_kernel<16, true, true>, p, r, grid, stream);
  return launch_route_impl(route_kernel<32, true, true>, p, r, grid, stream);
}

// Largest cooperative grid: one CTA per SM (the column reads of phase C grow
// with the grid).  The function attribute and occupancy are set up once per
// device (they depend only on the device and the kernel).
int align_max_ctas(int E, int* err_out) {
  // per device: SM count once the attribute and occupancy check succeeded
  // (atomic: host threads may race here; they all store the same value)
  static std::atomic<int> cached_sms[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  *err_out = (int)e;
  if (e != cudaSuccess) return 0;
  const int need = (int)align_smem_bytes(1024);
  if (dev < 64) {
    const int c = cached_sms[dev].load(std::memory_order_acquire);
    if (c > 0) return c;
  }
  int sms = 0, per_sm = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(route_kernel<32, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, need);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_kernel<32, true, true>, kAlignThreads, need);
  *err_out = (int)e;
  if (e != cudaSuccess || per_sm < 1) return 0;
  (void)E;
  if (dev < 64) cached_sms[dev].store(sms, std::memory_order_release);
  return sms;
}

// Timeout test: the same wait on a counter that can never fill.
__global__ void wait_timeout_kernel(int* counter, int32_t* status, long long timeout_ns) {
  if (!grid_wait(counter, gridDim.x + 1, timeout_ns)) {
    if (threadIdx.x == 0) dev_flag(status, MOE_DEV_TIMEOUT);
  }
}

cudaError_t launch_wait_timeout(int* counter, int32_t* status, long long timeout_ns, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(counter, status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace moe
