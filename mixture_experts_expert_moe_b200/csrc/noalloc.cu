// moe_align_sort_noalloc: MoE Align & Sort for callers that cannot allocate
// device memory.
//
// The regular moe_align_sort needs a caller-provided device workspace for the
// per-CTA expert counts and the grid-wide wait counter.  Some callers cannot
// provide one: code running inside another framework's allocator-free region
// (for example a custom op invoked while a memory pool is frozen), a plain C
// host program that only holds pointers handed to it by someone else, or an
// embedded runtime that forbids cudaMalloc after start-up.  This entry point
// keeps that scratch in a fixed array inside the library instead.
//
// The scratch is a file-scope device array of kScratchBytes (256 KB plus a
// 256-byte header) that every GPU which loads this library holds until the
// process exits.  It fits E <= 256 experts times up to 256 CTAs of counters
// (B200 has 148 SMs, and the kernel uses at most one CTA per SM).  Larger E is
// rejected with MOE_ERR_UNSUPPORTED before anything is launched.
//
// Set-up: the first call on each device (with that device current) looks up
// the array's device address with cudaGetSymbolAddress and caches it per
// device ordinal; make that first call before any stream capture.  The cached
// address belongs to the device's primary context (the runtime API's
// default): callers working in another context of the same device, or after
// cudaDeviceReset on it, must not use this entry point (the address would
// name memory of a context that is gone or not current).  Every later call on the device
// reuses the same array, which keeps the previous call's contents: the
// wait counter is cleared on the stream at the start of each call, and the
// count matrix is fully rewritten before it is read.  Because all calls share
// one array, calls that overlap on the GPU (on different streams, or from
// different host threads without ordering) race and give wrong results;
// serialise them.  No cudaMalloc, cudaFree or allocating library routine is
// called.
#include <mutex>

#include "kernels.cuh"

namespace moe {

constexpr int kNoallocMaxExperts = 256;
constexpr int kNoallocMaxCtas = 256;
constexpr size_t kScratchHeader = 256;  // the wait counter lives here
constexpr size_t kScratchBytes = kScratchHeader + (size_t)kNoallocMaxExperts * kNoallocMaxCtas * sizeof(int32_t);

static __device__ __align__(256) unsigned char g_align_scratch[kScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_align_scratch on the current device (looked up once
// per device).  In host code the symbol itself is only a stand-in and must
// never be passed to a kernel.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_align_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

extern "C" MOE_API moe_status_t moe_align_sort_noalloc(const int32_t* topk_ids, int T, int k, int E,
                                                       int block_size, int32_t* sorted_ids,
                                                       int32_t* expert_ids, int32_t* num_post,
                                                       int32_t* dev_status, void* stream) {
  if (T < 0 || k < 1 || E < 1 || block_size < 1 || block_size > 1024 ||
      (long long)T * k + (long long)E * (block_size - 1) >= 0x7FFFFFFFLL)
    return MOE_ERR_INVALID_ARG;
  if (!sorted_ids || !expert_ids || !num_post || (T > 0 && !topk_ids)) return MOE_ERR_INVALID_ARG;
  if (E > moe::kNoallocMaxExperts) return MOE_ERR_UNSUPPORTED;  // beyond the built-in scratch

  int dev = 0, major = 0;
  const cudaError_t ge = cudaGetDevice(&dev);
  if (ge == cudaErrorNoDevice || ge == cudaErrorInsufficientDriver) {
    moe::record_cuda_error(ge, "cudaGetDevice");
    return MOE_ERR_DEVICE;
  }
  if (ge != cudaSuccess) return moe::record_cuda_error(ge, "cudaGetDevice");
  cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return moe::record_cuda_error(e, "cudaDeviceGetAttribute");
  if (major != 10) return MOE_ERR_DEVICE;

  void* scratch = nullptr;
  e = moe::scratch_address(&scratch);
  if (e != cudaSuccess) return moe::record_cuda_error(e, "cudaGetSymbolAddress(align scratch)");

  // grid: one CTA per 4096 slots, at most one per SM (the kernel's co-residency rule)
  const int N = T * k;
  int err = 0;
  const int max_ctas = moe::align_max_ctas(E, &err);
  if (err) return moe::record_cuda_error((cudaError_t)err, "align occupancy");
  if (max_ctas < 1) return MOE_ERR_UNSUPPORTED;
  const int unit = 32 * 32;
  int grid = (int)(((long long)N + 4095) / 4096);
  grid = grid < 1 ? 1 : grid;
  grid = grid > max_ctas ? max_ctas : grid;
  grid = grid > moe::kNoallocMaxCtas ? moe::kNoallocMaxCtas : grid;
  int chunk = (N + grid - 1) / grid;
  chunk = (chunk + unit - 1) / unit * unit;
  if (chunk < unit) chunk = unit;
  grid = N > 0 ? (N + chunk - 1) / chunk : 1;

  unsigned char* base = static_cast<unsigned char*>(scratch);
  moe::AlignParams p;
  p.ids = topk_ids;
  p.N = N;
  p.E = E;
  p.bm = block_size;
  p.chunk = chunk;
  p.sorted = sorted_ids;
  p.expert_ids = expert_ids;
  p.num_post = num_post;
  p.barrier = reinterpret_cast<int*>(base);
  p.hist = reinterpret_cast<int32_t*>(base + moe::kScratchHeader);
  p.status = dev_status;
  p.timeout_ns = moe::kDefaultTimeoutNs;
  p.expected = grid;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the shared wait counter must start at zero for every call
  e = cudaMemsetAsync(p.barrier, 0, sizeof(int), s);
  if (e != cudaSuccess) return moe::record_cuda_error(e, "cudaMemsetAsync(align scratch counter)");
  e = moe::launch_align_sort(p, grid, s);
  if (e != cudaSuccess) return moe::record_cuda_error(e, "align & sort launch");
  return MOE_OK;
}
