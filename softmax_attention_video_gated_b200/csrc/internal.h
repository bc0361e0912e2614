// internal.h -- host-side interface between the C ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sva.h"

namespace sva {

// Launch bracketing for the stack's optional per-launch CUDA-event profile.
struct Prof {
  cudaEvent_t* events = nullptr;  // 2 * capacity
  int capacity = 0;
  int* kinds = nullptr;           // host, capacity
  int count = 0;
  int launches = 0;  // kernels launched (a scope may launch more than one)
  int cur_kind = SVA_KERNEL_OTHER;
  void before(cudaStream_t s, int kind) {
    cur_kind = kind;
    if (events != nullptr && count < capacity) cudaEventRecord(events[2 * count], s);
  }
  void after(cudaStream_t s) {
    if (events != nullptr && count < capacity) {
      cudaEventRecord(events[2 * count + 1], s);
      if (kinds != nullptr) kinds[count] = cur_kind;
    }
    ++count;
    ++launches;
  }
  void extra_launch() { ++launches; }  // a second kernel inside one scope
};

struct ProfScope {
  Prof* p;
  cudaStream_t s;
  ProfScope(Prof* p_, cudaStream_t s_, int kind) : p(p_), s(s_) {
    if (p) p->before(s, kind);
  }
  ~ProfScope() {
    if (p) p->after(s);
  }
};

// ---------------------------------------------------------------- utilities
// Records the CUDA error's text for sva_last_cuda_error and returns SVA_ERR_CUDA.
sva_status_t cuda_fail(cudaError_t e);
// Host-side validation of an attention call (null and misaligned pointers,
// row strides, sizes, eps / scale, supported head sizes). need_kv: k, v (and
// the write gate) are read; need_qgo: q, gate, out (and the residual) are used.
sva_status_t check_attn(const sva_attn_args* a, bool linear, bool need_kv = true,
                        bool need_qgo = true);
int device_sm_count();
int device_index();
bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes /* rank-1 */,
                 const uint32_t* box, CUtensorMapSwizzle swizzle);

constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- projections
enum GemmEpi { EPI_STORE = 0, EPI_RESIDUAL = 1 };

struct GemmArgs {
  const void* a = nullptr;  int64_t lda = 0;   // [M, K]
  const void* b = nullptr;  int64_t ldb = 0;   // [N, K]
  // optional second weight: output columns n >= n_split take row n - n_split
  // of b2 ([N - n_split, K], row stride ldb) instead of row n of b; n_split is
  // a multiple of 256 (the tile width of the tensor-core path)
  const void* b2 = nullptr; int64_t n_split = 0;
  int64_t M = 0, N = 0, K = 0;
  int epi = EPI_STORE;
  void* c = nullptr;        int64_t ldc = 0;   // EPI_STORE: [M, N] output
  int relu_cols = 0;
  float* h = nullptr;       int64_t ldh = 0;   // EPI_RESIDUAL: fp32 stream
  void* h_copy = nullptr;   int64_t ldhc = 0;  // EPI_RESIDUAL: optional copy
  // EPI_RESIDUAL, bf16: 0 = the copy is rounded to nearest; otherwise it is
  // rounded without bias (pack_bf16x2_unbiased), the random bits hashed from
  // this seed, the row and the column pair (deterministic)
  uint32_t copy_dither = 0;
  int* status = nullptr;
};

cudaError_t gemm_bf16(const GemmArgs& g, cudaStream_t s);
cudaError_t gemm_f32(const GemmArgs& g, cudaStream_t s);
cudaError_t transpose_2d(const void* src, void* dst, int64_t rows, int64_t cols, sva_dtype_t dt,
                         cudaStream_t s);  // dst[c][r] = src[r][c]

// ---------------------------------------------------------------- linear attention
// Scratch of one linear-attention call (offsets from the scratch base):
// fp32 per-chunk partial states, then (fp32 path only) the reduced state.
struct LinearPlan {
  int tiles_per_chunk = 0;  // 128-token tiles per state chunk (bf16) / tokens per chunk (f32)
  int n_chunks = 0;
  size_t partial_off = 0, state_off = 0, total = 0;
};
LinearPlan linear_plan(int B, int N, int H, int d, sva_dtype_t dt);
// Gated linear attention. With state_out, only the state pass runs and the
// fp32 state [B*H][d*d + d] (S row-major d_k x d_v, then z) is written there;
// with state_in, the state pass is skipped and the read-out uses that state;
// with neither, the fused layer.
cudaError_t linear_bf16(const sva_attn_args& a, int* status, void* scratch, cudaStream_t s,
                        Prof* prof, float* state_out = nullptr, const float* state_in = nullptr);
cudaError_t linear_f32(const sva_attn_args& a, int* status, void* scratch, cudaStream_t s,
                       Prof* prof, float* state_out = nullptr, const float* state_in = nullptr);

// ---------------------------------------------------------------- softmax anchor
// Anchor launch plan: units of 512 queries (one CTA pair each), key blocks,
// and the split of the last wave's units along the keys (partial_bytes of
// scratch for their parts).
struct AnchorPlan {
  int n_qunits = 0, nkv_total = 0, n_full = 0, n_split_units = 0, split = 0;
  size_t partial_bytes = 0;
};
AnchorPlan anchor_plan(int B, int N, int H, int n_keys);
cudaError_t anchor_bf16(const sva_attn_args& a, int* status, void* scratch, cudaStream_t s,
                        Prof* prof = nullptr);
cudaError_t anchor_f32(const sva_attn_args& a, int* status, cudaStream_t s);

// ---------------------------------------------------------------- router
cudaError_t route(const float* h, const void* const* keys, const void* const* summaries,
                  int n_blocks, void* u, float* alpha, int64_t rows, int D, sva_dtype_t dt,
                  cudaStream_t s);

// ---------------------------------------------------------------- misc
cudaError_t selftest_wait(int* status, unsigned timeout_us, cudaStream_t s);
cudaError_t cast_f32(const float* src, void* dst, int64_t n, sva_dtype_t dt, cudaStream_t s);
cudaError_t upcast_to_f32(const void* src, float* dst, int64_t n, sva_dtype_t dt, cudaStream_t s);
cudaError_t sub_inplace(const float* a, float* out, int64_t n, cudaStream_t s);  // out = a - out

}  // namespace sva
