// MoE Align & Sort on sm_100a: one cooperative launch, one grid-wide wait.
//
// Follows the D-C-P structure of the MoE Align & Sort article (dignews.cc,
// section "Writing AMD-friendly CUDA code with 3x~7x speed-up"):
//   (D) distributed concurrent counting: every CTA counts the expert ids of
//       its contiguous chunk of flat slots.  Inside a CTA every warp owns a
//       contiguous sub-chunk and a private histogram row in shared memory;
//       lanes that hold the same expert are grouped with __match_any_sync so
//       one leader updates the row (no atomics, and the order is fixed).
//   (C) cumulative sums: the warp rows are scanned into per-warp exclusive
//       prefixes (the article's "unaligned local cumsum"), the CTA totals go
//       to a global matrix hist[cta][expert] (the "merge" through a
//       preallocated HBM buffer), and after the single grid-wide wait every
//       CTA reads the matrix column-wise to get its own prefix and the
//       expert totals, pads the totals to the block size and scans them (the
//       "aligned global cumsum").
//   (P) parallel placement: each warp re-reads its sub-chunk and writes every
//       slot to  offset[e] + (slots of e in earlier CTAs) + (in earlier warps)
//       + (earlier in this warp), which is the stable counting-sort position.
//       Block expert ids and sentinel padding are written by the CTA that
//       owns the block.
// Unlike the article's design there is no second kernel and no single-block
// alignment step: every CTA redoes the small E-wide scan itself, which costs
// less than another launch or grid-wide wait.
#include "kernels.cuh"

namespace moe {

constexpr int kAlignThreads = 512;
constexpr int kAlignWarps = kAlignThreads / 32;


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
      __nanosleep(100);
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

// Exclusive scan of a[0..n) in shared memory by the whole CTA; returns the total.
__device__ int block_exclusive_scan(int* a, int n) {
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

__global__ void __launch_bounds__(kAlignThreads) align_sort_kernel(AlignParams p) {
  extern __shared__ int smem[];
  const int E = p.E;
  int* wcnt = smem;                       // [kAlignWarps][E] per-warp counts, then prefixes
  int* s_off = wcnt + kAlignWarps * E;    // [E] padded segment offsets
  int* s_base = s_off + E;                // [E] this CTA's first position per expert
  int* s_tot = s_base + E;                // [E] expert totals
  __shared__ int s_bad;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kAlignWarps * E; i += blockDim.x) wcnt[i] = 0;
  if (tid == 0) s_bad = 0;
  __syncthreads();

  const long long cta_begin = (long long)blockIdx.x * p.chunk;
  const int wsub = p.chunk / kAlignWarps;
  const long long w_begin = cta_begin + (long long)warp * wsub;
  const long long w_end = min((long long)p.N, w_begin + wsub);
  int* my = wcnt + warp * E;

  // ---- (D) count ----------------------------------------------------------
  bool bad = false;
  for (long long base = w_begin; base < w_end; base += 128) {
    int key[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      long long i = base + q * 32 + lane;
      int v = -1;
      if (i < w_end) {
        v = __ldg(p.ids + i);
        if (v < 0 || v >= E) {
          bad = true;
          v = -1;
        }
      }
      key[q] = v;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      unsigned peers = __match_any_sync(0xffffffffu, key[q]);
      if (key[q] >= 0 && (peers & lanemask_lt()) == 0) my[key[q]] += __popc(peers);
      __syncwarp();
    }
  }
  if (bad) s_bad = 1;
  __syncthreads();
  if (tid == 0 && s_bad) dev_flag(p.status, MOE_DEV_BAD_EXPERT_ID);

  // per-warp exclusive prefixes inside the CTA; CTA totals to the matrix
  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll 4
    for (int w = 0; w < kAlignWarps; ++w) {
      int c = wcnt[w * E + e];
      wcnt[w * E + e] = run;
      run += c;
    }
    p.hist[(long long)blockIdx.x * E + e] = run;
  }

  if (!grid_wait(p.barrier, p.expected, p.timeout_ns)) {
    if (tid == 0) dev_flag(p.status, MOE_DEV_TIMEOUT);
    return;
  }

  // ---- (C) this CTA's prefix, totals, padded offsets ----------------------
  const int ncta = gridDim.x;
  for (int e = tid; e < E; e += blockDim.x) {
    int pre = 0, tot = 0;
    int b = 0;
    for (; b + 8 <= ncta; b += 8) {
      int c[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) c[u] = __ldcg(p.hist + (long long)(b + u) * E + e);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        pre += (b + u < (int)blockIdx.x) ? c[u] : 0;
        tot += c[u];
      }
    }
    for (; b < ncta; ++b) {
      int c = __ldcg(p.hist + (long long)b * E + e);
      pre += (b < (int)blockIdx.x) ? c : 0;
      tot += c;
    }
    s_tot[e] = tot;
    s_base[e] = pre;
    s_off[e] = (tot + p.bm - 1) / p.bm * p.bm;
  }
  __syncthreads();
  const int total_post = block_exclusive_scan(s_off, E);
  for (int e = tid; e < E; e += blockDim.x) s_base[e] += s_off[e];
  if (blockIdx.x == 0 && tid == 0) *p.num_post = total_post;
  __syncthreads();

  // ---- block expert ids and sentinel padding for this CTA's blocks -------
  const int nblk = total_post / p.bm;
  const int bpc = (nblk + ncta - 1) / ncta;
  const int j0 = blockIdx.x * bpc;
  const int j1 = min(nblk, j0 + bpc);
  if (j1 > j0) {
    const long long npos = (long long)(j1 - j0) * p.bm;
    for (long long idx = tid; idx < npos; idx += blockDim.x) {
      const long long pos = (long long)j0 * p.bm + idx;
      int lo = 0, hi = E - 1;  // last expert whose segment starts at or before pos
      while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= pos) lo = mid; else hi = mid - 1;
      }
      if (idx % p.bm == 0) p.expert_ids[pos / p.bm] = lo;
      if (pos >= (long long)s_off[lo] + s_tot[lo]) p.sorted[pos] = p.N;
    }
  }

  // ---- (P) stable placement ------------------------------------------------
  for (long long base = w_begin; base < w_end; base += 128) {
    int key[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      long long i = base + q * 32 + lane;
      int v = -1;
      if (i < w_end) {
        v = __ldg(p.ids + i);
        if (v < 0 || v >= E) v = -1;
      }
      key[q] = v;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int kq = key[q];
      unsigned peers = __match_any_sync(0xffffffffu, kq);
      int cnt = kq >= 0 ? my[kq] : 0;
      __syncwarp();
      if (kq >= 0) {
        const unsigned below = peers & lanemask_lt();
        p.sorted[s_base[kq] + cnt + __popc(below)] = (int)(base + q * 32 + lane);
        if (below == 0) my[kq] = cnt + __popc(peers);
      }
      __syncwarp();
    }
  }
}

size_t align_smem_bytes(int E) { return (size_t)(kAlignWarps + 3) * E * sizeof(int); }

cudaError_t launch_align_sort(const AlignParams& p, int grid, cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(align_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)align_smem_bytes(p.E));
  if (err != cudaSuccess) return err;
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
  return cudaLaunchKernelEx(&cfg, align_sort_kernel, p);
}

int align_max_ctas(int E, int* err_out) {
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(align_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)align_smem_bytes(E));
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, align_sort_kernel, kAlignThreads,
                                                      align_smem_bytes(E));
  *err_out = (int)e;
  if (e != cudaSuccess) return 0;
  return sms * (per_sm < 1 ? 0 : 1);  // one CTA per SM: the column reads grow with the grid
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
