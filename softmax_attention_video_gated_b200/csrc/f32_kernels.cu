// f32_kernels.cu -- fp32 kernels on the CUDA cores: the projections, gated
// linear attention and the gated softmax anchor for fp32 runs. The tensor-core
// paths are bf16; an fp32 run asks for fp32 arithmetic throughout (TF32 would
// not hold its accuracy), so these kernels use plain fp32 FMAs.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace sva {
namespace {

// ---------------------------------------------------------------------------
// projection: C = A B^T, A [M, K], B [N, K]
// ---------------------------------------------------------------------------

constexpr int GT = 64, GK = 16;

__global__ void __launch_bounds__(256) gemm_f32_kernel(GemmArgs g) {
  __shared__ float As[GK][GT + 4];
  __shared__ float Bs[GK][GT + 4];
  const float* A = static_cast<const float*>(g.a);
  const float* B = static_cast<const float*>(g.b);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * GT, n0 = static_cast<int64_t>(blockIdx.x) * GT;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < g.K; k0 += GK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = threadIdx.x + 256 * i;
      const int r = idx / GK, c = idx % GK;
      const int64_t m = m0 + r, n = n0 + r, k = k0 + c;
      As[c][r] = (m < g.M && k < g.K) ? A[m * g.lda + k] : 0.f;
      const float* Bn = (g.b2 != nullptr && n >= g.n_split)
                            ? static_cast<const float*>(g.b2) + (n - g.n_split) * g.ldb
                            : B + n * g.ldb;
      Bs[c][r] = (n < g.N && k < g.K) ? Bn[k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < GK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty + 16 * i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx + 16 * j;
      if (n >= g.N) continue;
      float v = acc[i][j];
      if (g.epi == EPI_STORE) {
        if (n < g.relu_cols) v = relu_f(v);
        static_cast<float*>(g.c)[m * g.ldc + n] = v;
      } else {
        float* hp = g.h + m * g.ldh + n;
        const float hv = *hp + v;
        *hp = hv;
        if (g.h_copy != nullptr) static_cast<float*>(g.h_copy)[m * g.ldhc + n] = hv;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// gated linear attention, fp32
// ---------------------------------------------------------------------------

constexpr int LT = 32;  // tokens per smem tile

// Partial state of one chunk of tokens of one (batch, head):
// S_c = sum_t phi(K_t)^T V_t and z_c = sum_t phi(K_t), each term times
// sigmoid(wgate[b, t, h]) in the write-gated variant.
template <int D_>
__global__ void __launch_bounds__(256) lin_state_f32_kernel(sva_attn_args a, float* partial,
                                                            int tokens_per_chunk, int n_chunks) {
  constexpr int R = D_ / 16;  // register tile is R x R
  __shared__ float Ks[LT][D_];
  __shared__ float Vs[LT][D_];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const float* K = static_cast<const float*>(a.k);
  const float* V = static_cast<const float*>(a.v);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int t_begin = c * tokens_per_chunk;
  const int t_end = min(a.N, t_begin + tokens_per_chunk);
  const bool features = (a.flags & SVA_FLAG_QK_FEATURES) != 0;
  const float* wg = static_cast<const float*>(a.wgate);
  float acc[R][R] = {};
  float zacc = 0.f;
  for (int t0 = t_begin; t0 < t_end; t0 += LT) {
    for (int idx = threadIdx.x; idx < LT * D_; idx += 256) {
      const int r = idx / D_, col = idx % D_;
      const int t = t0 + r;
      float kv = 0.f, vv = 0.f;
      if (t < t_end) {
        const int64_t row = static_cast<int64_t>(b) * a.N + t;
        kv = K[row * a.ldk + h * D_ + col];
        vv = V[row * a.ldv + h * D_ + col];
        if (!features) kv = relu_f(kv);
        if (wg != nullptr) kv *= 1.0f / (1.0f + expf(-wg[row * a.ldw + h]));  // write gate
      }
      Ks[r][col] = kv;
      Vs[r][col] = vv;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < LT; ++r) {
      float kk[R], vv[R];
#pragma unroll
      for (int i = 0; i < R; ++i) kk[i] = Ks[r][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < R; ++j) vv[j] = Vs[r][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) acc[i][j] = fmaf(kk[i], vv[j], acc[i][j]);
      if (threadIdx.x < D_) zacc += Ks[r][threadIdx.x];
    }
    __syncthreads();
  }
  float* out = partial + (static_cast<int64_t>(b * a.H + h) * n_chunks + c) * (D_ * D_ + D_);
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int j = 0; j < R; ++j) out[(ty + 16 * i) * D_ + tx + 16 * j] = acc[i][j];
  if (threadIdx.x < D_) out[D_ * D_ + threadIdx.x] = zacc;
}

// Sum of the chunk partials of one (batch, head), in chunk order.
__global__ void lin_reduce_f32_kernel(const float* partial, float* state, int n_chunks, int elems) {
  const int64_t bh = blockIdx.x;
  for (int e = threadIdx.x; e < elems; e += blockDim.x) {
    const float* p = partial + bh * n_chunks * elems + e;
    float s = 0.f;
    for (int c = 0; c < n_chunks; ++c) s += p[static_cast<int64_t>(c) * elems];
    state[bh * elems + e] = s;
  }
}

// Y_t = phi(Q_t) S / (phi(Q_t) . z + eps) * sigmoid(G_t) (+ residual)
template <int D_>
__global__ void __launch_bounds__(256) lin_readout_f32_kernel(sva_attn_args a, const float* state) {
  extern __shared__ float sm[];
  float* S = sm;                 // [D_][D_]
  float* z = S + D_ * D_;        // [D_]
  float* Qs = z + D_;            // [LT][D_]
  const int h = blockIdx.y, b = blockIdx.z;
  const int t0 = blockIdx.x * LT;
  const float* st = state + static_cast<int64_t>(b * a.H + h) * (D_ * D_ + D_);
  for (int e = threadIdx.x; e < D_ * D_ + D_; e += 256) S[e] = st[e];
  const float* Q = static_cast<const float*>(a.q);
  const bool features = (a.flags & SVA_FLAG_QK_FEATURES) != 0;
  for (int idx = threadIdx.x; idx < LT * D_; idx += 256) {
    const int r = idx / D_, col = idx % D_;
    const int t = t0 + r;
    float qv = 0.f;
    if (t < a.N) {
      qv = Q[(static_cast<int64_t>(b) * a.N + t) * a.ldq + h * D_ + col];
      if (!features) qv = relu_f(qv);
    }
    Qs[r * D_ + col] = qv;
  }
  __syncthreads();
  const int r = threadIdx.x >> 3, j0 = threadIdx.x & 7;
  const int t = t0 + r;
  if (t >= a.N) return;
  float den = 0.f;
  for (int i = 0; i < D_; ++i) den = fmaf(Qs[r * D_ + i], z[i], den);
  den += a.eps;
  const int64_t row = static_cast<int64_t>(b) * a.N + t;
  const float* G = static_cast<const float*>(a.gate);
  const float* Rz = static_cast<const float*>(a.residual);
  float* O = static_cast<float*>(a.out);
  for (int j = j0; j < D_; j += 8) {
    float num = 0.f;
    for (int i = 0; i < D_; ++i) num = fmaf(Qs[r * D_ + i], S[i * D_ + j], num);
    const int64_t col = h * D_ + j;
    const float gv = G[row * a.ldg + col];
    float y = num / den * (1.0f / (1.0f + expf(-gv)));
    if (Rz != nullptr) y += Rz[row * a.ldr + col];
    O[row * a.ldo + col] = y;
  }
}

// ---------------------------------------------------------------------------
// gated softmax anchor, fp32: one warp per query row, keys in tiles of 32
// ---------------------------------------------------------------------------

template <int D_>
__global__ void __launch_bounds__(256) anchor_f32_kernel(sva_attn_args a, float scale) {
  constexpr int C = D_ / 32;  // output columns per lane
  __shared__ float Ks[32][D_ + 1];
  __shared__ float Vs[32][D_];
  __shared__ float Qs[8][D_];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int t = blockIdx.x * 8 + w;
  const float* Q = static_cast<const float*>(a.q);
  const float* K = static_cast<const float*>(a.k);
  const float* V = static_cast<const float*>(a.v);
  const int64_t base = static_cast<int64_t>(b) * a.N;    // query rows of batch b
  const int Nk = a.n_keys > 0 ? a.n_keys : a.N;            // keys (all of them)
  const int64_t kbase = static_cast<int64_t>(b) * Nk;
  for (int i = lane; i < D_; i += 32)
    Qs[w][i] = (t < a.N) ? Q[(base + t) * a.ldq + h * D_ + i] : 0.f;
  float m = -INFINITY, l = 0.f;
  float o[C];
#pragma unroll
  for (int q = 0; q < C; ++q) o[q] = 0.f;
  for (int s0 = 0; s0 < Nk; s0 += 32) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < 32 * D_; idx += 256) {
      const int r = idx / D_, col = idx % D_;
      const int s = s0 + r;
      Ks[r][col] = (s < Nk) ? K[(kbase + s) * a.ldk + h * D_ + col] : 0.f;
      Vs[r][col] = (s < Nk) ? V[(kbase + s) * a.ldv + h * D_ + col] : 0.f;
    }
    __syncthreads();
    float sc = 0.f;
    for (int i = 0; i < D_; ++i) sc = fmaf(Qs[w][i], Ks[lane][i], sc);
    sc = (s0 + lane < Nk) ? sc * scale : -INFINITY;
    float mt = sc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
    const float mn = fmaxf(m, mt);
    const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
    const float p = (sc == -INFINITY) ? 0.f : expf(sc - mn);
    float ps = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * corr + ps;
#pragma unroll
    for (int q = 0; q < C; ++q) o[q] *= corr;
    for (int j = 0; j < 32; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
      for (int q = 0; q < C; ++q) o[q] = fmaf(pj, Vs[j][lane + 32 * q], o[q]);
    }
    m = mn;
  }
  if (t >= a.N) return;
  const float* G = static_cast<const float*>(a.gate);
  const float* Rz = static_cast<const float*>(a.residual);
  float* O = static_cast<float*>(a.out);
  const float inv = 1.0f / l;
#pragma unroll
  for (int q = 0; q < C; ++q) {
    const int64_t col = h * D_ + lane + 32 * q;
    const int64_t row = base + t;
    const float gv = G[row * a.ldg + col];
    float y = o[q] * inv * (1.0f / (1.0f + expf(-gv)));
    if (Rz != nullptr) y += Rz[row * a.ldr + col];
    O[row * a.ldo + col] = y;
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------

cudaError_t gemm_f32(const GemmArgs& g, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>((g.N + GT - 1) / GT), static_cast<unsigned>((g.M + GT - 1) / GT));
  gemm_f32_kernel<<<grid, 256, 0, s>>>(g);
  return cudaGetLastError();
}

cudaError_t linear_f32(const sva_attn_args& a, int* status, void* scratch, cudaStream_t s,
                       Prof* prof, float* state_out, const float* state_in) {
  (void)status;
  const LinearPlan p = linear_plan(a.B, a.N, a.H, a.d, SVA_F32);
  char* base = static_cast<char*>(scratch);
  float* partial = reinterpret_cast<float*>(base + p.partial_off);
  const float* state = state_in;
  const int elems = a.d * a.d + a.d;
  if (state_in == nullptr) {
    {
      ProfScope ps(prof, s, SVA_KERNEL_LINEAR_STATE);
      dim3 grid(p.n_chunks, a.H, a.B);
      if (a.d == 64)
        lin_state_f32_kernel<64><<<grid, 256, 0, s>>>(a, partial, p.tiles_per_chunk, p.n_chunks);
      else
        lin_state_f32_kernel<128><<<grid, 256, 0, s>>>(a, partial, p.tiles_per_chunk, p.n_chunks);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    // the state goes to the caller (state only) or to the scratch (fused)
    float* dst = state_out != nullptr ? state_out : reinterpret_cast<float*>(base + p.state_off);
    {
      ProfScope ps(prof, s, SVA_KERNEL_LINEAR_REDUCE);
      lin_reduce_f32_kernel<<<a.B * a.H, 256, 0, s>>>(partial, dst, p.n_chunks, elems);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    if (state_out != nullptr) return cudaSuccess;
    state = dst;
  }
  ProfScope ps(prof, s, SVA_KERNEL_LINEAR_READOUT);
  dim3 grid((a.N + LT - 1) / LT, a.H, a.B);
  if (a.d == 64) {
    const size_t smem = (64 * 64 + 64 + LT * 64) * sizeof(float);
    lin_readout_f32_kernel<64><<<grid, 256, smem, s>>>(a, state);
  } else {
    const size_t smem = (128 * 128 + 128 + LT * 128) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(lin_readout_f32_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    lin_readout_f32_kernel<128><<<grid, 256, smem, s>>>(a, state);
  }
  return cudaGetLastError();
}

cudaError_t anchor_f32(const sva_attn_args& a, int* status, cudaStream_t s) {
  (void)status;
  const float scale = a.scale != 0.f ? a.scale : 1.0f / sqrtf(static_cast<float>(a.d));
  dim3 grid((a.N + 7) / 8, a.H, a.B);
  if (a.d == 64)
    anchor_f32_kernel<64><<<grid, 256, 0, s>>>(a, scale);
  else
    anchor_f32_kernel<128><<<grid, 256, 0, s>>>(a, scale);
  return cudaGetLastError();
}

}  // namespace sva
