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
//    stream capture.
//  * Every call on a device shares the one array, and it keeps the previous
//    call's contents. Each call clears the status word at its start and
//    overwrites all the scratch it reads, so back-to-back calls on one stream
//    are correct; calls that overlap on the GPU (other streams, other host
//    threads) race on the array and must be serialised by the caller.
//  * Device-side wait timeouts are recorded in the array's first bytes; this
//    entry point never synchronises and does not report them.
//  * Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library.
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;

__device__ __align__(256) unsigned char g_linear_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};  // per device: address of g_linear_scratch

// Host code may not use g_linear_scratch as a pointer (it names a host-side
// shadow); ask the runtime for the device address, once per device.
sva_status_t static_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SVA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || p == nullptr)
      return SVA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SVA_OK;
}

bool ptr_ok(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool row_ok(int64_t ld, int64_t width, size_t esize) {
  return ld >= width && (static_cast<size_t>(ld) * esize) % 16 == 0;
}

}  // namespace

extern "C" sva_status_t sva_linear_attn_fwd_noalloc(const sva_attn_args* a, sva_stream_t stream) {
  if (a == nullptr) return SVA_ERR_INVALID_ARGUMENT;
  if (a->dtype != SVA_F32 && a->dtype != SVA_BF16) return SVA_ERR_INVALID_ARGUMENT;
  if (a->B < 1 || a->N < 1 || a->H < 1 || a->d < 1) return SVA_ERR_INVALID_ARGUMENT;
  const size_t es = a->dtype == SVA_BF16 ? 2 : 4;
  const int64_t D = static_cast<int64_t>(a->H) * a->d;
  if (!ptr_ok(a->q) || !ptr_ok(a->k) || !ptr_ok(a->v) || !ptr_ok(a->gate) || !ptr_ok(a->out))
    return SVA_ERR_INVALID_ARGUMENT;
  if (!row_ok(a->ldq, D, es) || !row_ok(a->ldk, D, es) || !row_ok(a->ldv, D, es) ||
      !row_ok(a->ldg, D, es) || !row_ok(a->ldo, D, es))
    return SVA_ERR_INVALID_ARGUMENT;
  if (a->residual != nullptr && (!ptr_ok(a->residual) || !row_ok(a->ldr, D, es)))
    return SVA_ERR_INVALID_ARGUMENT;
  if (!(a->eps >= 0.f && std::isfinite(a->eps))) return SVA_ERR_INVALID_ARGUMENT;
  if (a->n_keys != 0) return SVA_ERR_INVALID_ARGUMENT;  // a key count is for anchors only
  if (a->wgate != nullptr &&
      (a->ldw < a->H || reinterpret_cast<uintptr_t>(a->wgate) % es != 0))
    return SVA_ERR_INVALID_ARGUMENT;
  if (static_cast<int64_t>(a->B) * a->N > (int64_t(1) << 31)) return SVA_ERR_UNSUPPORTED;
  if (a->dtype == SVA_BF16 && a->d != 128) return SVA_ERR_UNSUPPORTED;
  if (a->dtype == SVA_F32 && a->d != 64 && a->d != 128) return SVA_ERR_UNSUPPORTED;

  const sva::LinearPlan plan = sva::linear_plan(a->B, a->N, a->H, a->d, a->dtype);
  if (SVA_STATUS_BYTES + plan.total > kStaticScratchBytes) return SVA_ERR_WORKSPACE;

  void* base = nullptr;
  sva_status_t st = static_scratch(&base);
  if (st != SVA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(base, 0, SVA_STATUS_BYTES, s) != cudaSuccess) return SVA_ERR_CUDA;
  int* status = static_cast<int*>(base);
  void* scratch = static_cast<char*>(base) + SVA_STATUS_BYTES;
  const cudaError_t e = a->dtype == SVA_BF16 ? sva::linear_bf16(*a, status, scratch, s, nullptr)
                                             : sva::linear_f32(*a, status, scratch, s, nullptr);
  return e == cudaSuccess ? SVA_OK : SVA_ERR_CUDA;
}
