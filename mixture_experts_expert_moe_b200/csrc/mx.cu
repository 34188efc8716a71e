// MX (OCP Microscaling) operand preparation for the block-scaled grouped GEMM
// on sm_100a (GC-MoE abstract: block-scaled tensor-core MMAs with FP4/FP8
// operands on Blackwell; the pages leave the formats open, the OCP MX formats
// are used):
//   mx_quant_rows    bf16 rows -> MXFP8: per 32 consecutive elements an E8M0
//                    scale X = 2^(floor(log2 amax) - 8) (clamped to
//                    2^-127..2^127; 1 for an all-zero block) and E4M3 codes of
//                    v / X (round to nearest even, saturating).  With a row map
//                    it also gathers: sorted row r quantises token sorted[r]/k.
//   mx_tile_scales   per-row scales [rows, K/32] -> the tiled layout the MMA's
//                    scale-factor copies read (a 512-byte chunk per 128 rows and
//                    128 K-elements).
#include "kernels.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// MXFP8 quantisation, one warp per row; each lane takes 8 consecutive
// elements (one 16-byte vector), so 4 lanes hold one 32-element block.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t abs_bits_bf16_pair_max(uint32_t u) {
  const uint32_t lo = (u << 16) & 0x7FFFFFFFu, hi = u & 0x7FFF0000u;
  return lo > hi ? lo : hi;
}

__global__ void __launch_bounds__(256) mx_quant_rows_kernel(const uint4* __restrict__ src,
                                                            const int32_t* __restrict__ sorted, int N, int k,
                                                            const int32_t* __restrict__ nrows_dev, int nrows,
                                                            int C, uint2* __restrict__ codes,
                                                            uint8_t* __restrict__ scales) {
  const int rows = nrows_dev ? min(*nrows_dev, nrows) : nrows;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int vec = C / 8;             // 16-byte vectors per row
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < rows; r += gridDim.x * wpb) {
    long long t = r;
    if (sorted) {
      const int slot = __ldg(sorted + r);
      t = (unsigned)slot < (unsigned)N ? slot / k : -1;
    }
    const uint4* row = t >= 0 ? src + t * vec : nullptr;
    uint2* out = codes + (long long)r * vec;
    uint8_t* sc = scales + (long long)r * (C / 32);
    for (int c = lane; c < vec; c += 32) {     // vec % 4 == 0: the 4 lanes of a block stay together
      const uint4 v = row ? __ldg(row + c) : make_uint4(0, 0, 0, 0);
      uint32_t a = max(max(abs_bits_bf16_pair_max(v.x), abs_bits_bf16_pair_max(v.y)),
                       max(abs_bits_bf16_pair_max(v.z), abs_bits_bf16_pair_max(v.w)));
      const unsigned grp = 0xFu << (lane & ~3);
      a = max(a, __shfl_xor_sync(grp, a, 1));
      a = max(a, __shfl_xor_sync(grp, a, 2));
      const int code = mx_e8m0_code(a);
      const float inv = mx_inv_scale(code);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t q[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t p0 = (uint32_t)__nv_cvt_float2_to_fp8x2(
            make_float2(__uint_as_float(w[2 * i] << 16) * inv, __uint_as_float(w[2 * i] & 0xFFFF0000u) * inv),
            __NV_SATFINITE, __NV_E4M3);
        const uint32_t p1 = (uint32_t)__nv_cvt_float2_to_fp8x2(
            make_float2(__uint_as_float(w[2 * i + 1] << 16) * inv,
                        __uint_as_float(w[2 * i + 1] & 0xFFFF0000u) * inv),
            __NV_SATFINITE, __NV_E4M3);
        q[i] = p0 | (p1 << 16);
      }
      out[c] = make_uint2(q[0], q[1]);
      if ((lane & 3) == 0) sc[c >> 2] = (uint8_t)code;
    }
  }
}

cudaError_t launch_mx_quant_rows(const void* src, const int32_t* sorted, int N, int k, const int32_t* nrows_dev,
                                 int nrows, int C, void* codes, uint8_t* scales, cudaStream_t s) {
  if (nrows <= 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int warps = 8;
  long long blocks = ((long long)nrows + warps - 1) / warps;
  if (blocks > 16LL * sms) blocks = 16LL * sms;
  mx_quant_rows_kernel<<<(unsigned)blocks, 32 * warps, 0, s>>>(static_cast<const uint4*>(src), sorted, N, k,
                                                               nrows_dev, nrows, C, static_cast<uint2*>(codes),
                                                               scales);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Scale tiling: word (row r, K-blocks 4w..4w+3) of the per-row layout goes to
// word (r % 32) * 4 + (r % 128) / 32 of chunk (r / 128, w).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) mx_tile_scales_kernel(const uint32_t* __restrict__ in, long long rows,
                                                             int nk, uint32_t* __restrict__ out) {
  const long long total = rows * nk;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / nk;
    const int w = (int)(i - r * nk);
    const long long chunk = (r >> 7) * nk + w;
    out[chunk * 128 + (r & 31) * 4 + ((r >> 5) & 3)] = __ldg(in + i);
  }
}

cudaError_t launch_mx_tile_scales(const uint8_t* in, long long rows, int K, uint8_t* out, cudaStream_t s) {
  const long long total = rows * (K / 128);
  if (total == 0) return cudaSuccess;
  long long blocks = (total + 255) / 256;
  if (blocks > 65535) blocks = 65535;
  mx_tile_scales_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(in), rows, K / 128,
                                                         reinterpret_cast<uint32_t*>(out));
  return cudaGetLastError();
}

}  // namespace moe
