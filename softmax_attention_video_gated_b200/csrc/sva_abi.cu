// sva_abi.cu -- the C ABI: host-side validation, status handling, tensor-map
// encoding, and the hybrid stack orchestrator. Every entry point checks its
// arguments before launching anything, launches only on the caller's stream,
// and never allocates device memory.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace sva {

// ---------------------------------------------------------------------------
// utilities
// ---------------------------------------------------------------------------

namespace {
thread_local char g_last_cuda_error[256] = "";
std::atomic<int> g_sm_count[64];

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static std::atomic<void*> fn{nullptr};
  void* p = fn.load();
  if (p == nullptr) {
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn.store(p);
  }
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t esize(sva_dtype_t dt) { return dt == SVA_BF16 ? 2 : 4; }
bool ld_ok(int64_t ld, int64_t width, sva_dtype_t dt) {
  return ld >= width && (static_cast<size_t>(ld) * esize(dt)) % 16 == 0;
}
}  // namespace

sva_status_t cuda_fail(cudaError_t e) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
           cudaGetErrorString(e));
  return SVA_ERR_CUDA;
}

int device_index() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

int device_sm_count() {
  const int d = device_index();
  if (d < 0 || d >= 64) return 148;
  int v = g_sm_count[d].load();
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || v <= 0)
      v = 148;
    g_sm_count[d].store(v);
  }
  return v;
}

bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle) {
  auto fn = get_encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(map, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                        reinterpret_cast<const cuuint64_t*>(dims),
                        reinterpret_cast<const cuuint64_t*>(strides_bytes),
                        reinterpret_cast<const cuuint32_t*>(box), elem_strides,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sva

using namespace sva;

// ---------------------------------------------------------------------------
// validation
// ---------------------------------------------------------------------------

// need_kv: k, v (and the write gate) are read; need_qgo: q, gate, out (and the
// residual) are used. The fused calls need both; the two linear-attention
// phases one each.
sva_status_t sva::check_attn(const sva_attn_args* a, bool linear, bool need_kv, bool need_qgo) {
  if (a == nullptr) return SVA_ERR_INVALID_ARGUMENT;
  if (a->dtype != SVA_F32 && a->dtype != SVA_BF16) return SVA_ERR_INVALID_ARGUMENT;
  if (a->B < 1 || a->N < 1 || a->H < 1 || a->d < 1) return SVA_ERR_INVALID_ARGUMENT;
  const int64_t D = static_cast<int64_t>(a->H) * a->d;
  const void* ptrs[6] = {a->k, a->v, a->q, a->gate, a->out, a->residual};
  const int64_t lds[6] = {a->ldk, a->ldv, a->ldq, a->ldg, a->ldo, a->ldr};
  for (int i = 0; i < 6; ++i) {
    if (i < 2 && !need_kv) continue;
    if (i >= 2 && !need_qgo) break;
    if (i == 5 && a->residual == nullptr) break;
    if (ptrs[i] == nullptr || !aligned16(ptrs[i]) || !ld_ok(lds[i], D, a->dtype))
      return SVA_ERR_INVALID_ARGUMENT;
  }
  if (linear && !(a->eps >= 0.f && std::isfinite(a->eps))) return SVA_ERR_INVALID_ARGUMENT;
  if (a->n_keys < 0 || (linear && a->n_keys != 0)) return SVA_ERR_INVALID_ARGUMENT;
  if (static_cast<int64_t>(a->B) * a->n_keys > (int64_t(1) << 31)) return SVA_ERR_UNSUPPORTED;
  if (linear && need_kv && a->wgate != nullptr &&
      (a->ldw < a->H || reinterpret_cast<uintptr_t>(a->wgate) % esize(a->dtype) != 0))
    return SVA_ERR_INVALID_ARGUMENT;
  if (!linear && !(std::isfinite(a->scale) && a->scale >= 0.f)) return SVA_ERR_INVALID_ARGUMENT;
  if (static_cast<int64_t>(a->B) * a->N > (int64_t(1) << 31)) return SVA_ERR_UNSUPPORTED;
  if (a->dtype == SVA_BF16 && a->d != 128) return SVA_ERR_UNSUPPORTED;
  if (a->dtype == SVA_F32 && a->d != 64 && a->d != 128) return SVA_ERR_UNSUPPORTED;
  return SVA_OK;
}

namespace {

sva_status_t clear_status(void* ws, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(ws, 0, SVA_STATUS_BYTES, s);
  return e == cudaSuccess ? SVA_OK : cuda_fail(e);
}

sva_status_t check_gemm(const void* x, int64_t ldx, const void* w, int64_t M, int64_t Nout,
                        int64_t K, sva_dtype_t dt) {
  if (x == nullptr || w == nullptr) return SVA_ERR_INVALID_ARGUMENT;
  if (dt != SVA_F32 && dt != SVA_BF16) return SVA_ERR_INVALID_ARGUMENT;
  if (M < 1 || Nout < 1 || K < 1) return SVA_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(w) || !ld_ok(ldx, K, dt) || !ld_ok(K, K, dt))
    return SVA_ERR_INVALID_ARGUMENT;
  if (M > (int64_t(1) << 31) || Nout > (int64_t(1) << 31) || K > (int64_t(1) << 31))
    return SVA_ERR_UNSUPPORTED;
  return SVA_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// attention cores
// ---------------------------------------------------------------------------

extern "C" size_t sva_linear_attn_workspace_bytes(int B, int N, int H, int d, sva_dtype_t dtype) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return 0;
  return SVA_STATUS_BYTES + linear_plan(B, N, H, d, dtype).total;
}

extern "C" sva_status_t sva_linear_attn_fwd(const sva_attn_args* args, void* ws, size_t ws_bytes,
                                            sva_stream_t stream) {
  sva_status_t st = check_attn(args, true);
  if (st != SVA_OK) return st;
  if (ws == nullptr || !aligned16(ws) ||
      ws_bytes < sva_linear_attn_workspace_bytes(args->B, args->N, args->H, args->d, args->dtype))
    return SVA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != SVA_OK) return st;
  int* status = static_cast<int*>(ws);
  void* scratch = static_cast<char*>(ws) + SVA_STATUS_BYTES;
  cudaError_t e = args->dtype == SVA_BF16 ? linear_bf16(*args, status, scratch, s, nullptr)
                                          : linear_f32(*args, status, scratch, s, nullptr);
  return e == cudaSuccess ? SVA_OK : cuda_fail(e);
}

extern "C" size_t sva_linear_attn_state_bytes(int B, int H, int d) {
  if (B < 1 || H < 1 || d < 1) return 0;
  return static_cast<size_t>(B) * H * (static_cast<size_t>(d) * d + d) * sizeof(float);
}

extern "C" sva_status_t sva_linear_attn_state_fwd(const sva_attn_args* args, float* state,
                                                  void* ws, size_t ws_bytes,
                                                  sva_stream_t stream) {
  sva_status_t st = check_attn(args, true, true, false);
  if (st != SVA_OK) return st;
  if (state == nullptr || !aligned16(state)) return SVA_ERR_INVALID_ARGUMENT;
  if (ws == nullptr || !aligned16(ws) ||
      ws_bytes < sva_linear_attn_workspace_bytes(args->B, args->N, args->H, args->d, args->dtype))
    return SVA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != SVA_OK) return st;
  int* status = static_cast<int*>(ws);
  void* scratch = static_cast<char*>(ws) + SVA_STATUS_BYTES;
  const cudaError_t e = args->dtype == SVA_BF16
                            ? linear_bf16(*args, status, scratch, s, nullptr, state, nullptr)
                            : linear_f32(*args, status, scratch, s, nullptr, state, nullptr);
  return e == cudaSuccess ? SVA_OK : cuda_fail(e);
}

extern "C" sva_status_t sva_linear_attn_readout_fwd(const sva_attn_args* args, const float* state,
                                                    void* ws, size_t ws_bytes,
                                                    sva_stream_t stream) {
  sva_status_t st = check_attn(args, true, false, true);
  if (st != SVA_OK) return st;
  if (state == nullptr || !aligned16(state)) return SVA_ERR_INVALID_ARGUMENT;
  if (ws == nullptr || !aligned16(ws) ||
      ws_bytes < sva_linear_attn_workspace_bytes(args->B, args->N, args->H, args->d, args->dtype))
    return SVA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != SVA_OK) return st;
  int* status = static_cast<int*>(ws);
  void* scratch = static_cast<char*>(ws) + SVA_STATUS_BYTES;
  const cudaError_t e = args->dtype == SVA_BF16
                            ? linear_bf16(*args, status, scratch, s, nullptr, nullptr, state)
                            : linear_f32(*args, status, scratch, s, nullptr, nullptr, state);
  return e == cudaSuccess ? SVA_OK : cuda_fail(e);
}

extern "C" size_t sva_softmax_anchor_workspace_bytes(int B, int N, int H, int d,
                                                     sva_dtype_t dtype) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return 0;
  if (dtype != SVA_BF16) return SVA_STATUS_BYTES;
  // the split parts of the last wave (bounded over every key count)
  return SVA_STATUS_BYTES + anchor_plan(B, N, H, 1 << 30).partial_bytes;
}

extern "C" sva_status_t sva_softmax_anchor_fwd(const sva_attn_args* args, void* ws, size_t ws_bytes,
                                               sva_stream_t stream) {
  sva_status_t st = check_attn(args, false);
  if (st != SVA_OK) return st;
  const size_t need =
      SVA_STATUS_BYTES +
      (args->dtype == SVA_BF16 ? anchor_plan(args->B, args->N, args->H, args->n_keys).partial_bytes
                               : 0);
  if (ws == nullptr || !aligned16(ws) || ws_bytes < need) return SVA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != SVA_OK) return st;
  int* status = static_cast<int*>(ws);
  cudaError_t e = args->dtype == SVA_BF16
                      ? anchor_bf16(*args, status, static_cast<char*>(ws) + SVA_STATUS_BYTES, s)
                      : anchor_f32(*args, status, s);
  return e == cudaSuccess ? SVA_OK : cuda_fail(e);
}

// ---------------------------------------------------------------------------
// projections
// ---------------------------------------------------------------------------

extern "C" size_t sva_projection_workspace_bytes(void) { return SVA_STATUS_BYTES; }

extern "C" sva_status_t sva_projection_fwd(const void* x, int64_t ldx, const void* w, int64_t M,
                                           int64_t Nout, int64_t K, void* y, int64_t ldy,
                                           int relu_cols, sva_dtype_t dtype, void* ws,
                                           size_t ws_bytes, sva_stream_t stream) {
  sva_status_t st = check_gemm(x, ldx, w, M, Nout, K, dtype);
  if (st != SVA_OK) return st;
  if (y == nullptr || !aligned16(y) || !ld_ok(ldy, Nout, dtype) || relu_cols < 0)
    return SVA_ERR_INVALID_ARGUMENT;
  if (ws == nullptr || !aligned16(ws) || ws_bytes < SVA_STATUS_BYTES) return SVA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != SVA_OK) return st;
  GemmArgs g;
  g.a = x; g.lda = ldx; g.b = w; g.ldb = K; g.M = M; g.N = Nout; g.K = K;
  g.epi = EPI_STORE; g.c = y; g.ldc = ldy; g.relu_cols = relu_cols;
  g.status = static_cast<int*>(ws);
  cudaError_t e = dtype == SVA_BF16 ? gemm_bf16(g, s) : gemm_f32(g, s);
  return e == cudaSuccess ? SVA_OK : cuda_fail(e);
}

extern "C" sva_status_t sva_projection_residual_fwd(const void* x, int64_t ldx, const void* w,
                                                    int64_t M, int64_t Nout, int64_t K, float* h,
                                                    int64_t ldh, void* h_copy, int64_t ldc,
                                                    sva_dtype_t dtype, void* ws, size_t ws_bytes,
                                                    sva_stream_t stream) {
  sva_status_t st = check_gemm(x, ldx, w, M, Nout, K, dtype);
  if (st != SVA_OK) return st;
  if (h == nullptr || !aligned16(h) || !ld_ok(ldh, Nout, SVA_F32)) return SVA_ERR_INVALID_ARGUMENT;
  if (h_copy != nullptr && (!aligned16(h_copy) || !ld_ok(ldc, Nout, dtype)))
    return SVA_ERR_INVALID_ARGUMENT;
  if (ws == nullptr || !aligned16(ws) || ws_bytes < SVA_STATUS_BYTES) return SVA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != SVA_OK) return st;
  GemmArgs g;
  g.a = x; g.lda = ldx; g.b = w; g.ldb = K; g.M = M; g.N = Nout; g.K = K;
  g.epi = EPI_RESIDUAL; g.h = h; g.ldh = ldh; g.h_copy = h_copy; g.ldhc = ldc;
  g.status = static_cast<int*>(ws);
  cudaError_t e = dtype == SVA_BF16 ? gemm_bf16(g, s) : gemm_f32(g, s);
  return e == cudaSuccess ? SVA_OK : cuda_fail(e);
}

// ---------------------------------------------------------------------------
// AttnRes
// ---------------------------------------------------------------------------

extern "C" size_t sva_attnres_keys_workspace_bytes(int D, sva_dtype_t dtype) {
  if (D < 1) return 0;
  return SVA_STATUS_BYTES + align_up(static_cast<size_t>(D) * D * esize(dtype), 1024);
}

namespace {
cudaError_t keys_launch(const void* s_b, const void* w_r, void* k_b, int64_t rows, int D,
                        sva_dtype_t dtype, int* status, void* wr_t, bool transpose,
                        cudaStream_t s) {
  // k_b = s_b W_r = s_b (W_r^T)^T: the GEMM's [out, in] operand is W_r^T
  cudaError_t e = cudaSuccess;
  if (transpose) {
    e = transpose_2d(w_r, wr_t, D, D, dtype, s);
    if (e != cudaSuccess) return e;
  }
  GemmArgs g;
  g.a = s_b; g.lda = D; g.b = wr_t; g.ldb = D; g.M = rows; g.N = D; g.K = D;
  g.epi = EPI_STORE; g.c = k_b; g.ldc = D; g.status = status;
  return dtype == SVA_BF16 ? gemm_bf16(g, s) : gemm_f32(g, s);
}
}  // namespace

extern "C" sva_status_t sva_attnres_keys(const void* s_b, const void* w_r, void* k_b, int64_t rows,
                                         int D, sva_dtype_t dtype, void* ws, size_t ws_bytes,
                                         sva_stream_t stream) {
  sva_status_t st = check_gemm(s_b, D, w_r, rows, D, D, dtype);
  if (st != SVA_OK) return st;
  if (k_b == nullptr || !aligned16(k_b)) return SVA_ERR_INVALID_ARGUMENT;
  if (ws == nullptr || !aligned16(ws) || ws_bytes < sva_attnres_keys_workspace_bytes(D, dtype))
    return SVA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != SVA_OK) return st;
  cudaError_t e = keys_launch(s_b, w_r, k_b, rows, D, dtype, static_cast<int*>(ws),
                              static_cast<char*>(ws) + SVA_STATUS_BYTES, true, s);
  return e == cudaSuccess ? SVA_OK : cuda_fail(e);
}

extern "C" sva_status_t sva_attnres_route(const float* h, const void* const* keys,
                                          const void* const* summaries, int n_blocks, void* u,
                                          float* alpha, int64_t rows, int D, sva_dtype_t dtype,
                                          sva_stream_t stream) {
  if (h == nullptr || keys == nullptr || summaries == nullptr || u == nullptr)
    return SVA_ERR_INVALID_ARGUMENT;
  if (dtype != SVA_F32 && dtype != SVA_BF16) return SVA_ERR_INVALID_ARGUMENT;
  if (n_blocks < 1 || n_blocks > 8 || rows < 1 || D < 1) return SVA_ERR_INVALID_ARGUMENT;
  if (D % static_cast<int>(16 / esize(dtype)) != 0 || D % 4 != 0) return SVA_ERR_INVALID_ARGUMENT;
  if (!aligned16(h) || !aligned16(u) || (alpha != nullptr && (reinterpret_cast<uintptr_t>(alpha) & 3)))
    return SVA_ERR_INVALID_ARGUMENT;
  for (int b = 0; b < n_blocks; ++b)
    if (keys[b] == nullptr || summaries[b] == nullptr || !aligned16(keys[b]) ||
        !aligned16(summaries[b]))
      return SVA_ERR_INVALID_ARGUMENT;
  cudaError_t e = route(h, keys, summaries, n_blocks, u, alpha, rows, D, dtype,
                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SVA_OK : cuda_fail(e);
}

// ---------------------------------------------------------------------------
// the hybrid stack
// ---------------------------------------------------------------------------

namespace {

struct StackLayout {
  size_t h, u, qkvg, y, lin, wrt, summ, keys, total;
  int n_summ;  // summaries kept (completed blocks that feed a later block)
};

bool layer_is_anchor(const sva_stack_desc& d, int l) {
  return d.all_softmax || (d.softmax_period > 0 && l % d.softmax_period == 0);
}
int block_of(const sva_stack_desc& d, int l) {
  return d.attnres_block > 0 ? (l + d.attnres_block - 1) / d.attnres_block : 1;
}
bool layer_is_routed(const sva_stack_desc& d, int l) {
  return d.attnres_block > 0 && !layer_is_anchor(d, l) && block_of(d, l) >= 2;
}
int summaries_needed(const sva_stack_desc& d) {
  // summary c is needed iff some routed layer lies in a block > c
  int need = 0;
  for (int l = 1; l <= d.L; ++l)
    if (layer_is_routed(d, l)) need = std::max(need, block_of(d, l) - 1);
  return need;
}

// Row stride of the fused projection output [Q | K | V | G (| W)]: 4D, plus,
// for write-gated stacks, the H write-gate logits padded to 8 elements so
// rows stay 16-byte aligned for the TMA maps that read Q, K, V and G.
int64_t qkvg_ld(const sva_stack_desc& d) {
  const int64_t D = static_cast<int64_t>(d.H) * d.d;
  return 4 * D + (d.w_wg != nullptr ? (static_cast<int64_t>(d.H) + 7) / 8 * 8 : 0);
}

StackLayout stack_layout(const sva_stack_desc& d) {
  StackLayout s{};
  const size_t rows = static_cast<size_t>(d.B) * d.N;
  const size_t D = static_cast<size_t>(d.H) * d.d;
  const size_t es = esize(d.dtype);
  size_t off = SVA_STATUS_BYTES;
  auto take = [&](size_t bytes) {
    off = align_up(off, 1024);
    const size_t at = off;
    off += bytes;
    return at;
  };
  s.h = take(rows * D * 4);
  s.u = take(rows * D * es);
  s.qkvg = take(rows * static_cast<size_t>(qkvg_ld(d)) * es);
  s.y = take(rows * D * es);
  // attention scratch: the linear layers' partial states, or the anchors' split parts
  s.lin = take(std::max(linear_plan(d.B, d.N, d.H, d.d, d.dtype).total,
                        d.dtype == SVA_BF16 ? anchor_plan(d.B, d.N, d.H, 0).partial_bytes : 0));
  s.n_summ = summaries_needed(d);
  s.wrt = take(s.n_summ > 0 ? D * D * es : 0);
  s.summ = take(static_cast<size_t>(s.n_summ) * rows * D * es);
  s.keys = take(static_cast<size_t>(s.n_summ) * rows * D * es);
  s.total = align_up(off, 1024);
  return s;
}

sva_status_t check_stack(const sva_stack_desc* d) {
  if (d == nullptr) return SVA_ERR_INVALID_ARGUMENT;
  if (d->dtype != SVA_F32 && d->dtype != SVA_BF16) return SVA_ERR_INVALID_ARGUMENT;
  if (d->B < 1 || d->N < 1 || d->H < 1 || d->d < 1 || d->L < 1) return SVA_ERR_INVALID_ARGUMENT;
  if (d->softmax_period < 0 || d->attnres_block < 0) return SVA_ERR_INVALID_ARGUMENT;
  if (!(d->eps >= 0.f && std::isfinite(d->eps))) return SVA_ERR_INVALID_ARGUMENT;
  if (d->w_qkvg == nullptr || d->w_o == nullptr) return SVA_ERR_INVALID_ARGUMENT;
  for (int l = 0; l < d->L; ++l)
    if (d->w_qkvg[l] == nullptr || d->w_o[l] == nullptr || !aligned16(d->w_qkvg[l]) ||
        !aligned16(d->w_o[l]))
      return SVA_ERR_INVALID_ARGUMENT;
  if (d->dtype == SVA_BF16 && d->d != 128) return SVA_ERR_UNSUPPORTED;
  if (d->dtype == SVA_F32 && d->d != 64 && d->d != 128) return SVA_ERR_UNSUPPORTED;
  const int n_summ = summaries_needed(*d);
  if (n_summ > 8) return SVA_ERR_UNSUPPORTED;
  if (n_summ > 0 && (d->w_r == nullptr || !aligned16(d->w_r))) return SVA_ERR_INVALID_ARGUMENT;
  if (d->prof_events != nullptr && d->prof_capacity < 0) return SVA_ERR_INVALID_ARGUMENT;
  if (d->w_wg != nullptr)
    for (int l = 1; l <= d->L; ++l)
      if (!layer_is_anchor(*d, l) && (d->w_wg[l - 1] == nullptr || !aligned16(d->w_wg[l - 1])))
        return SVA_ERR_INVALID_ARGUMENT;
  return SVA_OK;
}

}  // namespace

extern "C" size_t sva_hybrid_stack_workspace_bytes(const sva_stack_desc* desc) {
  if (check_stack(desc) != SVA_OK) return 0;
  return stack_layout(*desc).total;
}

namespace {

// one stack pass; clear_first resets the workspace status word (a caller
// running several passes clears it once, so an early device error is kept)
sva_status_t stack_pass(const sva_stack_desc* desc, const void* x, void* y, void* ws,
                        size_t ws_bytes, sva_stream_t stream, bool clear_first) {
  sva_status_t st = check_stack(desc);
  if (st != SVA_OK) return st;
  const sva_stack_desc& d = *desc;
  if (x == nullptr || y == nullptr || !aligned16(x) || !aligned16(y)) return SVA_ERR_INVALID_ARGUMENT;
  const StackLayout lay = stack_layout(d);
  if (ws == nullptr || !aligned16(ws) || ws_bytes < lay.total) return SVA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // launches are counted whenever the caller asks for the count; events are
  // recorded only when it hands some over
  Prof prof_obj;
  Prof* prof = nullptr;
  if (d.prof_events != nullptr || d.launch_count != nullptr) {
    if (d.prof_events != nullptr) {
      prof_obj.events = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(d.prof_events));
      prof_obj.capacity = d.prof_capacity;
      prof_obj.kinds = d.prof_kind;
    }
    prof = &prof_obj;
  }

  char* base = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(base);
  float* h = reinterpret_cast<float*>(base + lay.h);
  char* u = base + lay.u;
  char* qkvg = base + lay.qkvg;
  char* ybuf = base + lay.y;
  void* lin_scratch = base + lay.lin;
  char* wrt = base + lay.wrt;
  const int64_t rows = static_cast<int64_t>(d.B) * d.N;
  const int D = d.H * d.d;
  const size_t es = esize(d.dtype);
  const size_t act_bytes = static_cast<size_t>(rows) * D * es;
  auto summ = [&](int c) { return base + lay.summ + static_cast<size_t>(c - 1) * act_bytes; };
  auto keyb = [&](int c) { return base + lay.keys + static_cast<size_t>(c - 1) * act_bytes; };
  const bool bf16 = d.dtype == SVA_BF16;
  const int64_t ldp = qkvg_ld(d);

  cudaError_t e = cudaSuccess;
#define SVA_TRY(expr)                          \
  do {                                         \
    if ((e = (expr)) != cudaSuccess) return cuda_fail(e); \
  } while (0)

  if (clear_first && (st = clear_status(ws, s)) != SVA_OK) return st;
  {
    ProfScope ps(prof, s, SVA_KERNEL_OTHER);
    SVA_TRY(upcast_to_f32(x, h, rows * D, d.dtype, s));
  }
  if (lay.n_summ > 0) {
    ProfScope ps(prof, s, SVA_KERNEL_OTHER);
    SVA_TRY(transpose_2d(d.w_r, wrt, D, D, d.dtype, s));
  }

  // input of the next layer's projection when it is not routed
  const void* in = bf16 ? x : static_cast<const void*>(h);
  for (int l = 1; l <= d.L; ++l) {
    const bool anchor = layer_is_anchor(d, l);
    const bool routed = layer_is_routed(d, l);
    if (routed) {
      const int c = block_of(d, l);
      const void* ks[8];
      const void* ss[8];
      for (int b = 1; b < c; ++b) {
        ks[b - 1] = keyb(b);
        ss[b - 1] = summ(b);
      }
      float* alpha = d.trace_alpha != nullptr ? static_cast<float*>(d.trace_alpha[l - 1]) : nullptr;
      ProfScope ps(prof, s, SVA_KERNEL_ROUTE);
      SVA_TRY(route(h, ks, ss, c - 1, u, alpha, rows, D, d.dtype, s));
      in = u;
    }
    const bool write_gated = !anchor && d.w_wg != nullptr;
    {
      // [Q | K | V | G] = u W_qkvg^T; the linear layers take phi(Q), phi(K) from
      // the epilogue; a write-gated layer's logits u W_wg^T follow in the same
      // GEMM as columns 4D .. 4D + H
      GemmArgs g;
      g.a = in; g.lda = D; g.b = d.w_qkvg[l - 1]; g.ldb = D;
      g.M = rows; g.N = 4 * static_cast<int64_t>(D); g.K = D;
      if (write_gated) {
        g.b2 = d.w_wg[l - 1];
        g.n_split = g.N;
        g.N += d.H;
      }
      g.epi = EPI_STORE; g.c = qkvg; g.ldc = ldp;
      g.relu_cols = anchor ? 0 : 2 * D;
      g.status = status;
      ProfScope ps(prof, s, SVA_KERNEL_PROJ_QKVG);
      SVA_TRY(bf16 ? gemm_bf16(g, s) : gemm_f32(g, s));
    }
    sva_attn_args a{};
    a.B = d.B; a.N = d.N; a.H = d.H; a.d = d.d; a.dtype = d.dtype;
    a.q = qkvg; a.k = qkvg + D * es; a.v = qkvg + 2 * D * es; a.gate = qkvg + 3 * D * es;
    a.ldq = a.ldk = a.ldv = a.ldg = ldp;
    a.residual = nullptr; a.ldr = 0;
    a.out = ybuf; a.ldo = D;
    a.eps = d.eps; a.scale = 0.f;
    a.flags = anchor ? 0u : SVA_FLAG_QK_FEATURES;
    if (write_gated) {
      a.wgate = qkvg + 4 * D * es;
      a.ldw = ldp;
    }
    if (anchor) {
      ProfScope ps(prof, s, SVA_KERNEL_ANCHOR);
      SVA_TRY(bf16 ? anchor_bf16(a, status, lin_scratch, s, prof) : anchor_f32(a, status, s));
    } else {
      SVA_TRY(bf16 ? linear_bf16(a, status, lin_scratch, s, prof)
                   : linear_f32(a, status, lin_scratch, s, prof));
    }
    if (d.trace_y != nullptr && d.trace_y[l - 1] != nullptr)
      SVA_TRY(cudaMemcpyAsync(d.trace_y[l - 1], ybuf, act_bytes, cudaMemcpyDeviceToDevice, s));
    float* tro = d.trace_o != nullptr ? static_cast<float*>(d.trace_o[l - 1]) : nullptr;
    if (tro != nullptr)
      SVA_TRY(cudaMemcpyAsync(tro, h, static_cast<size_t>(rows) * D * 4, cudaMemcpyDeviceToDevice, s));

    // where the updated stream's dtype copy goes
    const bool ends_block = d.attnres_block > 0 && l % d.attnres_block == 0 &&
                            l / d.attnres_block <= lay.n_summ;
    void* copy = nullptr;
    if (l == d.L) {
      copy = y;  // y = dtype(h_L)
    } else if (ends_block) {
      copy = summ(l / d.attnres_block);
    } else if (!layer_is_routed(d, l + 1) && bf16) {
      copy = u;
    }
    {
      GemmArgs g;
      g.a = ybuf; g.lda = D; g.b = d.w_o[l - 1]; g.ldb = D;
      g.M = rows; g.N = D; g.K = D;
      g.epi = EPI_RESIDUAL; g.h = h; g.ldh = D; g.h_copy = copy; g.ldhc = D;
      // A copy that a later projection reads (the next layer's input, a block
      // summary) is rounded without bias: h = x + (small updates) with x a
      // bf16 number, and round-to-nearest would drop every update below half
      // a bf16 step of x, the same way for every token; the linear layers
      // average over all tokens, so that bias would reach their outputs (a
      // 1.6% error in layer 2 at 19,320 tokens against 0.3% unbiased). The
      // stack's output y is rounded to nearest.
      if (copy != nullptr && copy != y) g.copy_dither = 0x9E3779B9u * static_cast<uint32_t>(l) | 1u;
      g.status = status;
      ProfScope ps(prof, s, SVA_KERNEL_PROJ_OUT);
      SVA_TRY(bf16 ? gemm_bf16(g, s) : gemm_f32(g, s));
    }
    if (tro != nullptr) SVA_TRY(sub_inplace(h, tro, rows * D, s));
    if (l < d.L) {
      if (ends_block) {
        const int c = l / d.attnres_block;
        ProfScope ps(prof, s, SVA_KERNEL_KEYS);
        SVA_TRY(keys_launch(summ(c), d.w_r, keyb(c), rows, D, d.dtype, status, wrt, false, s));
        in = bf16 ? static_cast<const void*>(summ(c)) : static_cast<const void*>(h);
      } else {
        in = bf16 ? static_cast<const void*>(u) : static_cast<const void*>(h);
      }
    }
  }
#undef SVA_TRY
  if (d.prof_count != nullptr) *d.prof_count = prof != nullptr ? prof->count : 0;
  if (d.launch_count != nullptr) *d.launch_count = prof != nullptr ? prof->launches : 0;
  return SVA_OK;
}

size_t act_slot_bytes(const sva_stack_desc& d) {
  return align_up(static_cast<size_t>(d.B) * d.N * d.H * d.d * esize(d.dtype), 256);
}

// streams and events of one host-batch call, released on every exit path
// (the runtime frees them once the work queued on them is done)
struct CopyPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, in_done[2] = {}, pass_done[2] = {}, out_done[2] = {};
  ~CopyPipe() {
    for (cudaEvent_t* e : {&start, &in_done[0], &in_done[1], &pass_done[0], &pass_done[1],
                           &out_done[0], &out_done[1]})
      if (*e != nullptr) cudaEventDestroy(*e);
    if (h2d != nullptr) cudaStreamDestroy(h2d);
    if (d2h != nullptr) cudaStreamDestroy(d2h);
  }
  cudaError_t create() {
    cudaError_t e = cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking);
    for (cudaEvent_t* ev : {&start, &in_done[0], &in_done[1], &pass_done[0], &pass_done[1],
                            &out_done[0], &out_done[1]})
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    return e;
  }
};

}  // namespace

extern "C" sva_status_t sva_hybrid_stack_fwd(const sva_stack_desc* desc, const void* x, void* y,
                                             void* ws, size_t ws_bytes, sva_stream_t stream) {
  return stack_pass(desc, x, y, ws, ws_bytes, stream, true);
}

extern "C" size_t sva_hybrid_stack_host_staging_bytes(const sva_stack_desc* desc) {
  if (check_stack(desc) != SVA_OK) return 0;
  return 4 * act_slot_bytes(*desc);  // two slots, each an input and an output
}

extern "C" sva_status_t sva_hybrid_stack_fwd_host(const sva_stack_desc* desc,
                                                  const void* const* x_host, void* const* y_host,
                                                  int n, void* ws, size_t ws_bytes, void* staging,
                                                  size_t staging_bytes, sva_stream_t stream) {
  sva_status_t st = check_stack(desc);
  if (st != SVA_OK) return st;
  if (n < 0 || (n > 0 && (x_host == nullptr || y_host == nullptr)))
    return SVA_ERR_INVALID_ARGUMENT;
  for (int i = 0; i < n; ++i)
    if (x_host[i] == nullptr || y_host[i] == nullptr) return SVA_ERR_INVALID_ARGUMENT;
  const sva_stack_desc& d = *desc;
  const size_t slot = act_slot_bytes(d);
  if (staging == nullptr || !aligned16(staging) || staging_bytes < 4 * slot)
    return SVA_ERR_WORKSPACE;
  if (ws == nullptr || !aligned16(ws) || ws_bytes < stack_layout(d).total) return SVA_ERR_WORKSPACE;
  if (n == 0) return SVA_OK;
  const size_t bytes = static_cast<size_t>(d.B) * d.N * d.H * d.d * esize(d.dtype);
  char* sb = static_cast<char*>(staging);
  void* xs[2] = {sb, sb + slot};
  void* ys[2] = {sb + 2 * slot, sb + 3 * slot};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CopyPipe cp;
  cudaError_t e = cp.create();
  if (e != cudaSuccess) return cuda_fail(e);
  if ((st = clear_status(ws, s)) != SVA_OK) return st;
#define SVA_TRY(expr)                                     \
  do {                                                    \
    if ((e = (expr)) != cudaSuccess) return cuda_fail(e); \
  } while (0)
  // the copy streams start after the work already queued on `stream`
  SVA_TRY(cudaEventRecord(cp.start, s));
  SVA_TRY(cudaStreamWaitEvent(cp.h2d, cp.start, 0));
  SVA_TRY(cudaStreamWaitEvent(cp.d2h, cp.start, 0));
  for (int i = 0; i < n; ++i) {
    const int k = i & 1;
    // slot k's input is free once the pass of batch i - 2 has finished
    if (i >= 2) SVA_TRY(cudaStreamWaitEvent(cp.h2d, cp.pass_done[k], 0));
    SVA_TRY(cudaMemcpyAsync(xs[k], x_host[i], bytes, cudaMemcpyHostToDevice, cp.h2d));
    SVA_TRY(cudaEventRecord(cp.in_done[k], cp.h2d));
    // the pass needs its input in and slot k's previous output copied out
    SVA_TRY(cudaStreamWaitEvent(s, cp.in_done[k], 0));
    if (i >= 2) SVA_TRY(cudaStreamWaitEvent(s, cp.out_done[k], 0));
    if ((st = stack_pass(desc, xs[k], ys[k], ws, ws_bytes, stream, false)) != SVA_OK) return st;
    SVA_TRY(cudaEventRecord(cp.pass_done[k], s));
    SVA_TRY(cudaStreamWaitEvent(cp.d2h, cp.pass_done[k], 0));
    SVA_TRY(cudaMemcpyAsync(y_host[i], ys[k], bytes, cudaMemcpyDeviceToHost, cp.d2h));
    SVA_TRY(cudaEventRecord(cp.out_done[k], cp.d2h));
  }
  // `stream` completes only after every output has reached the host
  SVA_TRY(cudaStreamWaitEvent(s, cp.out_done[(n - 1) & 1], 0));
  if (n >= 2) SVA_TRY(cudaStreamWaitEvent(s, cp.out_done[n & 1], 0));
#undef SVA_TRY
  return SVA_OK;
}

// ---------------------------------------------------------------------------
// status
// ---------------------------------------------------------------------------

extern "C" sva_status_t sva_check_device_status(const void* ws, sva_stream_t stream) {
  if (ws == nullptr) return SVA_ERR_INVALID_ARGUMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  int word[2] = {0, 0};
  e = cudaMemcpy(word, ws, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  return static_cast<sva_status_t>(word[0]);
}

extern "C" sva_status_t sva_selftest_bounded_wait(void* ws, size_t ws_bytes, unsigned timeout_us,
                                                  sva_stream_t stream) {
  if (ws == nullptr || !aligned16(ws) || ws_bytes < SVA_STATUS_BYTES) return SVA_ERR_WORKSPACE;
  if (timeout_us == 0 || timeout_us > 10000000u) return SVA_ERR_INVALID_ARGUMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  sva_status_t st = clear_status(ws, s);
  if (st != SVA_OK) return st;
  cudaError_t e = selftest_wait(static_cast<int*>(ws), timeout_us, s);
  return e == cudaSuccess ? SVA_OK : cuda_fail(e);
}

extern "C" const char* sva_status_string(sva_status_t status) {
  switch (status) {
    case SVA_OK: return "ok";
    case SVA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case SVA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case SVA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SVA_ERR_CUDA: return "CUDA error";
    case SVA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

extern "C" const char* sva_last_cuda_error(void) { return g_last_cuda_error; }

extern "C" int sva_version(void) { return 1; }
