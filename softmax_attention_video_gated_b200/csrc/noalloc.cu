// noalloc.cu -- gated linear attention for callers that cannot allocate.
//
// sva_linear_attn_fwd needs a caller-provided workspace for its per-chunk
// partial states. Some callers have no way to provide one: an engine that
// plans every byte of device memory at start-up and forbids allocation once
// it serves requests, a plugin that is handed a stream but no allocator, or a
// host program whose memory pool belongs to another framework. For them this
// file keeps the scratch in one file-scope device array of fixed size, so the
// call needs nothing but its inputs and outputs.
//
// Rules of this entry point:
//  * The array is kStaticScratchBytes (16 MiB) and lives on every GPU that
//    loads the library, until the process exits.
//  * Calls that would need more scratch than that are refused on the host
//    with SVA_ERR_WORKSPACE before anything is launched.
//  * The array's device address is looked up once per device (with that
//    device current) on the first call there; make that first call before any
//    stream capture. The address is cached with the device's current context:
//    after cudaDeviceReset (a new context) the next call looks it up again.
//  * Every call on a device shares the one array, and it keeps the previous
//    call's contents. Each call clears the status word at its start and
//    overwrites all the scratch it reads, so back-to-back calls on one stream
//    are correct; calls that overlap on the GPU (other streams, other host
//    threads) race on the array and must be serialised by the caller.
//  * Device-side wait timeouts are recorded in the array's first bytes; this
//    entry point never synchronises and does not report them.
//  * Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;

__device__ __align__(256) unsigned char g_linear_scratch[kStaticScratchBytes];

struct CachedAddr {
  CUcontext ctx = nullptr;  // the context the address was looked up in
  void* addr = nullptr;     // device address of g_linear_scratch there
};
std::mutex g_scratch_mu;
CachedAddr g_scratch_addr[64];  // per device

PFN_cuCtxGetCurrent_v4000 ctx_get_current_fn() {
  static void* fn = nullptr;  // guarded by g_scratch_mu
  if (fn == nullptr) {
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      fn = nullptr;
  }
  return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
}

// Host code may not use g_linear_scratch as a pointer (it names a host-side
// shadow); ask the runtime for the device address, once per device and
// context.
sva_status_t static_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return sva::cuda_fail(e);
  if (dev < 0 || dev >= 64) return SVA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  PFN_cuCtxGetCurrent_v4000 get_ctx = ctx_get_current_fn();
  if (get_ctx == nullptr) return SVA_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return SVA_ERR_CUDA;
  CachedAddr& c = g_scratch_addr[dev];
  if (ctx == nullptr || c.addr == nullptr || c.ctx != ctx) {
    // the lookup also makes the runtime's context current when none is yet
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_linear_scratch)) != cudaSuccess) return sva::cuda_fail(e);
    if (p == nullptr || get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return SVA_ERR_CUDA;
    c.ctx = ctx;
    c.addr = p;
  }
  *out = c.addr;
  return SVA_OK;
}

}  // namespace

extern "C" sva_status_t sva_linear_attn_fwd_noalloc(const sva_attn_args* a, sva_stream_t stream) {
  sva_status_t st = sva::check_attn(a, /*linear=*/true);
  if (st != SVA_OK) return st;

  const sva::LinearPlan plan = sva::linear_plan(a->B, a->N, a->H, a->d, a->dtype);
  if (SVA_STATUS_BYTES + plan.total > kStaticScratchBytes) return SVA_ERR_WORKSPACE;

  void* base = nullptr;
  st = static_scratch(&base);
  if (st != SVA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(base, 0, SVA_STATUS_BYTES, s);
  if (e != cudaSuccess) return sva::cuda_fail(e);
  int* status = static_cast<int*>(base);
  void* scratch = static_cast<char*>(base) + SVA_STATUS_BYTES;
  e = a->dtype == SVA_BF16 ? sva::linear_bf16(*a, status, scratch, s, nullptr)
                           : sva::linear_f32(*a, status, scratch, s, nullptr);
  return e == cudaSuccess ? SVA_OK : sva::cuda_fail(e);
}
