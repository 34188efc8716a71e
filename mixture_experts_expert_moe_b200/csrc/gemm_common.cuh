// Pieces shared by the grouped GEMM kernels of the forward (grouped_gemm.cu)
// and the backward (bwd.cu): tile geometry, the tile plan's decoding, bounded
// mbarrier waits that honour a CTA-wide abort flag, and TMA tensor maps.
#pragma once
#include "kernels.cuh"

namespace moe {

constexpr int kGemmThreads = 320;   // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kGemmThreadsMx = 352; // + warp 10: MX activation scales
constexpr int kSfChunk = 512;       // MX scale chunk: 128 rows x 4 K-blocks of E8M0
constexpr int kWRows = 128;      // weight rows per tile = MMA M
constexpr int kStageK = 128;     // bytes of K per stage (one swizzle row)
constexpr int kWTileBytes = kWRows * kStageK;
constexpr int kRing = 4;         // tile indices in flight from the producer to the other warps
// after an abort, how long a CTA waits for its own copies and MMAs in flight
// before it gives up (and reports MOE_DEV_DRAIN_TIMEOUT)
constexpr long long kDrainTimeoutNs = 100000000LL;

struct TileInfo {
  int e, wt, r0, nrows;
};

// Tile t of the list: the list position of its expert (last position whose
// tile range starts at or before t), then weight tile and token group.
// nrows counts the group's real rows only (the expert's padding rows, at the
// end of its segment, are neither loaded nor multiplied); a group of padding
// alone keeps one row, which every epilogue skips as padding.
__device__ __forceinline__ TileInfo decode_tile(int t, const int* s_pref, const int* s_perm, const int* s_start,
                                                const int* s_rows, const int* s_groups, int E, int tn) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_pref[mid] <= t) lo = mid; else hi = mid - 1;
  }
  TileInfo ti;
  ti.e = s_perm[lo];
  const int local = t - s_pref[lo];
  const int G = s_groups[ti.e];
  ti.wt = local / G;
  const int g = local - ti.wt * G;
  ti.r0 = s_start[ti.e] + g * tn;
  ti.nrows = max(1, min(tn, s_rows[ti.e] - g * tn));
  return ti;
}

// The c-th claimed tile: hot-list tiles [0, hot) and cold-list tiles
// [hot, n) alternate while both last, then the rest of the longer list (a
// bijection on [0, n); claims past the end stay past the end).
__device__ __forceinline__ int claim_to_tile(int c, int hot, int n) {
  if (c >= n) return c;
  const int cold = n - hot;
  const int m = min(hot, cold);
  if (c < 2 * m) return (c & 1) ? hot + (c >> 1) : (c >> 1);
  const int r = c - 2 * m;
  return hot > cold ? m + r : hot + m + r;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, long long timeout_ns,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*abort_flag) return false;
      if ((long long)(globaltimer_ns() - t0) > timeout_ns) {
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Token rows of the tile are loaded in boxes of x_box rows, only as many as
// the token group has (rounded up to x_box).
__device__ __forceinline__ int x_box_rows(int tn) { return tn < 32 ? tn : 32; }

// ---------------------------------------------------------------------------
// host: TMA tensor maps
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (thread-safe static
// initialisation); null if the driver does not provide it.
inline EncodeTiledFn get_encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return nullptr;
  }();
  return fn;
}

// 2-D K-major tensor [rows, K] with a box of (128 bytes of K) x box_rows,
// 128-byte swizzle.  elem_bytes 2: bf16; 1: one-byte codes; 0: E2M1 codes
// packed two per byte in global memory, unpacked by TMA to one 16-byte chunk
// per 16 elements (8 bytes of codes, 8 bytes of gap) in shared memory, the
// operand layout of the block-scaled MMA for 4-bit A.
inline bool make_map(CUtensorMap* m, const void* base, long long rows, long long K, int elem_bytes,
                     int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(elem_bytes == 0 ? K / 2 : K * elem_bytes)};
  cuuint32_t box[2] = {(cuuint32_t)(elem_bytes == 0 ? kStageK : kStageK / elem_bytes), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = elem_bytes == 2   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                   : CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}



}  // namespace moe
