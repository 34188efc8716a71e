// Shared device helpers for the sm_100a MoE kernels: status reporting,
// bounded waits, mbarriers, TMA and tcgen05 (UMMA / TMEM) wrappers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

constexpr long long kDefaultTimeoutNs = 2000000000LL;  // 2 s per bounded wait

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void dev_flag(int32_t* st, int bits) {
  if (st) atomicOr(st, bits);
}

// Bounds checks of the MOE_DEBUG build (the stand-in for a memory checker):
// MOE_IN_BOUNDS(cond, status) is cond, and flags MOE_DEV_BOUNDS when cond is
// false; without MOE_DEBUG it is true and compiles away.
#ifdef MOE_DEBUG
__device__ __forceinline__ bool moe_in_bounds(bool ok, int32_t* st) {
  if (!ok) dev_flag(st, MOE_DEV_BOUNDS);
  return ok;
}
#define MOE_IN_BOUNDS(cond, st) moe_in_bounds((cond), (st))
#else
#define MOE_IN_BOUNDS(cond, st) true
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of parity `parity` to complete, for at most timeout_ns.
// Returns false if the wait ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0 && (long long)(globaltimer_ns() - t0) > timeout_ns) return false;
  }
}

// ---------------------------------------------------------------------------
// TMA (no multicast anywhere in this library)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
// 1-D bulk copy global -> this CTA's shared memory, completion counted on an
// mbarrier (both addresses 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// 4-byte asynchronous copy global -> shared (cp.async, non-bulk); completion is
// tracked by cp_async_mbar_arrive_noinc or cp_async_wait_all of this thread.
__device__ __forceinline__ void cp_async_4(uint32_t dst_smem, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst_smem), "l"(reinterpret_cast<uint64_t>(src))
               : "memory");
}
// Arrive on the mbarrier once every cp.async this thread issued so far has
// completed; the arrival is counted in the barrier's expected count (noinc).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// fire-and-forget fp32 add in L2 with a cache-eviction priority
__device__ __forceinline__ void red_add_f32(float* addr, float v, uint64_t policy) {
  asm volatile("red.global.add.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(addr), "f"(v), "l"(policy) : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, MMA, commit, loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 operands, fp32 accumulator.
__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// Same with E4M3 operands (kind::f8f6f4), fp32 accumulator.
__device__ __forceinline__ void mma_e4m3(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// MX block-scaled MMA (kind::mxf8f6f4, one E8M0 scale per 32 K-elements of
// every row of A and of B): D[tmem] (+)= (A * SFA) * (B * SFB)^T.  sfa / sfb
// are the TMEM addresses of the scale factors; their top two bits pick the
// byte (the K-block of this MMA) inside each 32-bit TMEM word, and must
// agree with the scale-factor ids in the instruction descriptor.
__device__ __forceinline__ void mma_mx(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"(acc)
      : "memory");
}
// Copy a 32-row x 16-byte shared-memory block (descriptor sdesc) into TMEM
// columns taddr..taddr+3 of lanes 0..31, replicated to all four 32-lane
// quarters (the layout the block-scaled MMA reads its scale factors from).
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzle: rows of 128 bytes, 8-row (1024-byte) swizzle atoms
// stacked along M/N (stride-dimension byte offset 1024).  The tile base must
// be 1024-byte aligned; advancing along K inside the atom adds to the start
// address.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;                 // leading byte offset (unused for SW128 K-major)
  d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset
  d |= (uint64_t)1 << 46;                 // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                 // layout: 128-byte swizzle
  return d;
}

// MX (OCP Microscaling) block scale: E8M0 code of a 32-element block whose
// largest magnitude has the float bits amax_bits (non-negative, finite):
// 127 + floor(log2 amax) - 8 (8 = exponent of E4M3's largest normal, 448 =
// 1.75 * 2^8), clamped below at 0 (2^-127); 127 (X = 1) for an all-zero block.
// A subnormal amax has exponent field 0 and clamps as floor(log2) would.
__device__ __forceinline__ int mx_e8m0_code(uint32_t amax_bits) {
  if (amax_bits == 0) return 127;
  const int e = (int)(amax_bits >> 23) - 127;
  return max(e - 8, -127) + 127;
}
// 1 / X = 2^-(code - 127) as a float: biased exponent 254 - code, in [8, 254]
// for the codes mx_e8m0_code returns, so always an exact normal float.
__device__ __forceinline__ float mx_inv_scale(int code) { return __uint_as_float((uint32_t)(254 - code) << 23); }

// Shared-memory descriptor of an unswizzled K-major block of 8-row x 16-byte
// core matrices stacked along the rows (16 bytes per row, 128 bytes per core
// matrix): the source of tcgen05.cp's 32x128b shape.
__device__ __forceinline__ uint64_t umma_desc_rows16(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
  d |= (uint64_t)(128 >> 4) << 32;        // stride byte offset: next 8 rows
  d |= (uint64_t)1 << 46;                 // descriptor version (sm_100)
  return d;                               // layout type 0: no swizzle
}

// Instruction descriptor of the block-scaled MMA (kind::mxf8f6f4, E8M0 scale
// factors, fp32 accumulator, A/B K-major, shape M x N).  a_fmt / b_fmt: 0 =
// E4M3, 5 = E2M1; sf_id: the byte of the scale-factor words this MMA uses
// (for both A and B).
__host__ __device__ __forceinline__ uint32_t umma_idesc_mx(int M, int N, uint32_t a_fmt, uint32_t b_fmt,
                                                           uint32_t sf_id) {
  return (sf_id << 4) | (a_fmt << 7) | (b_fmt << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
         ((uint32_t)(M >> 4) << 24) | (sf_id << 29);
}

// Shared-memory descriptor of an MN-major operand tile with 128-byte swizzle,
// as TMA writes it from boxes of 64 bf16 along M (or N) by K rows: box c
// (elements 64c..64c+63 along M/N) at offset c * box_bytes, K-row k of a box
// at k * 128 bytes (swizzle atoms of 8 K-rows = 1024 bytes).  The leading
// byte offset steps to the next 64 elements along M/N, the stride byte offset
// to the next 8 K-rows; one MMA K-step of 16 rows advances the start address
// by 2048 bytes.
__device__ __forceinline__ uint64_t umma_desc_mn_sw128(uint32_t smem_addr, uint32_t box_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
  d |= (uint64_t)((box_bytes >> 4) & 0x3FFF) << 16;  // leading byte offset: next 64 M/N elements
  d |= (uint64_t)(1024 >> 4) << 32;                   // stride byte offset: next 8 K-rows
  d |= (uint64_t)1 << 46;                             // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                             // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16 with operand majors: a_mn / b_mn = 1 for
// an MN-major A / B (0 = K-major), bf16 operands, fp32 accumulator.
__host__ __device__ __forceinline__ uint32_t umma_idesc_bf16_major(int M, int N, uint32_t a_mn, uint32_t b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn << 15) | (b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor: fp32 accumulator, A/B K-major, shape M x N.
// fmt: 1 = bf16 (kind::f16), 0 = E4M3 (kind::f8f6f4).
__host__ __device__ __forceinline__ uint32_t umma_idesc(int M, int N, uint32_t fmt) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace moe
