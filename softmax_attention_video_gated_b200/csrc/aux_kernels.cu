// aux_kernels.cu -- the AttnRes router, and small data-movement kernels
// (transpose, casts) plus the bounded-wait self test.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace sva {
namespace {

// ---------------------------------------------------------------------------
// AttnRes router [ai-papers.net summary, section "ブロックアテンション残差"]:
// one warp per token row. logits_b = h . k_b / sqrt(D) over the completed
// blocks, alpha = softmax_b(logits), u = h + sum_b alpha_b s_b.
// Streaming: h is read twice (the second pass mostly from L2), keys and
// summaries once, u written once.
// ---------------------------------------------------------------------------

constexpr int kMaxBlocks = 8;

template <typename T>
struct Vec;  // 16-byte vector of T, widened to fp32

template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const void* p, float (&f)[8]) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    f[0] = bf16lo_to_f32(v.x); f[1] = bf16hi_to_f32(v.x);
    f[2] = bf16lo_to_f32(v.y); f[3] = bf16hi_to_f32(v.y);
    f[4] = bf16lo_to_f32(v.z); f[5] = bf16hi_to_f32(v.z);
    f[6] = bf16lo_to_f32(v.w); f[7] = bf16hi_to_f32(v.w);
  }
  __device__ static void store(void* p, const float (&f)[8]) {
    uint4 v;
    v.x = pack_bf16x2(f[0], f[1]);
    v.y = pack_bf16x2(f[2], f[3]);
    v.z = pack_bf16x2(f[4], f[5]);
    v.w = pack_bf16x2(f[6], f[7]);
    *reinterpret_cast<uint4*>(p) = v;
  }
};

template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const void* p, float (&f)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
  __device__ static void store(void* p, const float (&f)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};

struct RoutePtrs {
  const void* keys[kMaxBlocks];
  const void* summaries[kMaxBlocks];
};

template <typename T>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ h, RoutePtrs p,
                                                    int n_blocks, T* __restrict__ u,
                                                    float* __restrict__ alpha, int64_t rows, int D,
                                                    float inv_sqrt_d) {
  constexpr int V = Vec<T>::N;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* hr = h + row * D;
  float dots[kMaxBlocks];
#pragma unroll
  for (int b = 0; b < kMaxBlocks; ++b) dots[b] = 0.f;
  for (int c = lane * V; c < D; c += 32 * V) {
    float hv[V];
#pragma unroll
    for (int i = 0; i < V; i += 4) {
      const float4 x = *reinterpret_cast<const float4*>(hr + c + i);
      hv[i] = x.x; hv[i + 1] = x.y; hv[i + 2] = x.z; hv[i + 3] = x.w;
    }
#pragma unroll
    for (int b = 0; b < kMaxBlocks; ++b) {
      if (b >= n_blocks) break;
      float kv[V];
      Vec<T>::load(static_cast<const T*>(p.keys[b]) + row * D + c, kv);
#pragma unroll
      for (int i = 0; i < V; ++i) dots[b] = fmaf(hv[i], kv[i], dots[b]);
    }
  }
  float wts[kMaxBlocks];
  float mx = -INFINITY;
#pragma unroll
  for (int b = 0; b < kMaxBlocks; ++b) {
    if (b >= n_blocks) break;
    float d = dots[b];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    wts[b] = d * inv_sqrt_d;
    mx = fmaxf(mx, wts[b]);
  }
  float sum = 0.f;
#pragma unroll
  for (int b = 0; b < kMaxBlocks; ++b) {
    if (b >= n_blocks) break;
    wts[b] = expf(wts[b] - mx);
    sum += wts[b];
  }
  const float inv = 1.0f / sum;
#pragma unroll
  for (int b = 0; b < kMaxBlocks; ++b) {
    if (b >= n_blocks) break;
    wts[b] *= inv;
    if (alpha != nullptr && lane == 0) alpha[row * n_blocks + b] = wts[b];
  }
  for (int c = lane * V; c < D; c += 32 * V) {
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; i += 4) {
      const float4 x = *reinterpret_cast<const float4*>(hr + c + i);
      acc[i] = x.x; acc[i + 1] = x.y; acc[i + 2] = x.z; acc[i + 3] = x.w;
    }
#pragma unroll
    for (int b = 0; b < kMaxBlocks; ++b) {
      if (b >= n_blocks) break;
      float sv[V];
      Vec<T>::load(static_cast<const T*>(p.summaries[b]) + row * D + c, sv);
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = fmaf(wts[b], sv[i], acc[i]);
    }
    Vec<T>::store(u + row * D + c, acc);
  }
}

// bf16 router with one group of D / 8 threads per row (D a multiple of 256):
// each thread keeps its 8 values of h in registers between the two steps, so h
// is read from HBM once, and every load of a step is issued before any is
// used (kept packed until then). The NB dot products are summed over the
// group's warps through shared memory; several groups may share a CTA.
template <int NB>
__global__ void __launch_bounds__(512) route_rows_kernel(const float* __restrict__ h, RoutePtrs p,
                                                         __nv_bfloat16* __restrict__ u,
                                                         float* __restrict__ alpha, int64_t rows,
                                                         int D, float inv_sqrt_d) {
  __shared__ float part[16][NB];  // per-warp partial dots (at most 16 warps)
  const int G = D >> 3;           // threads per row
  const int g = threadIdx.x / G, tg = threadIdx.x - g * G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / G) + g;
  const bool valid = row < rows;
  const int64_t off = (valid ? row : 0) * D + tg * 8;
  float4 ha = make_float4(0.f, 0.f, 0.f, 0.f), hb = ha;
  uint4 kq[NB];
  if (valid) {
    ha = *reinterpret_cast<const float4*>(h + off);
    hb = *reinterpret_cast<const float4*>(h + off + 4);
#pragma unroll
    for (int b = 0; b < NB; ++b)
      kq[b] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.keys[b]) + off);
  } else {
#pragma unroll
    for (int b = 0; b < NB; ++b) kq[b] = make_uint4(0u, 0u, 0u, 0u);
  }
  const float hv[8] = {ha.x, ha.y, ha.z, ha.w, hb.x, hb.y, hb.z, hb.w};
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const uint32_t kw[4] = {kq[b].x, kq[b].y, kq[b].z, kq[b].w};
    float d = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      d = fmaf(hv[2 * i], bf16lo_to_f32(kw[i]), d);
      d = fmaf(hv[2 * i + 1], bf16hi_to_f32(kw[i]), d);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    if (lane == 0) part[warp][b] = d;
  }
  __syncthreads();
  // the group's warps are [g * G / 32, (g + 1) * G / 32); every thread sums them
  const int w0 = (g * G) >> 5, nw = G >> 5;
  float wts[NB];
  float mx = -INFINITY;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    float d = 0.f;
    for (int w = 0; w < nw; ++w) d += part[w0 + w][b];
    wts[b] = d * inv_sqrt_d;
    mx = fmaxf(mx, wts[b]);
  }
  float sum = 0.f;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    wts[b] = expf(wts[b] - mx);
    sum += wts[b];
  }
  const float inv = 1.0f / sum;
  if (!valid) return;
  uint4 sq[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b)
    sq[b] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.summaries[b]) + off);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = hv[i];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const float wb = wts[b] * inv;
    if (alpha != nullptr && tg == 0) alpha[row * NB + b] = wb;
    const uint32_t sw[4] = {sq[b].x, sq[b].y, sq[b].z, sq[b].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(wb, bf16lo_to_f32(sw[i]), acc[2 * i]);
      acc[2 * i + 1] = fmaf(wb, bf16hi_to_f32(sw[i]), acc[2 * i + 1]);
    }
  }
  Vec<__nv_bfloat16>::store(u + off, acc);
}

template <int NB>
cudaError_t launch_route_rows(const float* h, const RoutePtrs& p, void* u, float* alpha,
                              int64_t rows, int D, float inv_sqrt_d, cudaStream_t s) {
  const int G = D / 8, per_cta = 512 / G;
  const unsigned grid = static_cast<unsigned>((rows + per_cta - 1) / per_cta);
  route_rows_kernel<NB><<<grid, G * per_cta, 0, s>>>(h, p, static_cast<__nv_bfloat16*>(u), alpha,
                                                     rows, D, inv_sqrt_d);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// transpose (32 x 32 tiles through shared memory) and casts
// ---------------------------------------------------------------------------

template <typename T>
__global__ void transpose_kernel(const T* __restrict__ src, T* __restrict__ dst, int64_t rows,
                                 int64_t cols) {
  __shared__ T tile[32][33];
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 32, r0 = static_cast<int64_t>(blockIdx.y) * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = src[r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) dst[c * rows + r] = tile[threadIdx.x][i];
  }
}

__global__ void cast_f32_to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                        int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

__global__ void upcast_bf16_kernel(const __nv_bfloat16* __restrict__ src, float* __restrict__ dst,
                                   int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = __bfloat162float(src[i]);
}

__global__ void sub_inplace_kernel(const float* __restrict__ a, float* __restrict__ out, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = a[i] - out[i];
}

// ---------------------------------------------------------------------------
// bounded-wait self test: a barrier nothing arrives at
// ---------------------------------------------------------------------------

__global__ void selftest_wait_kernel(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives: the wait must run out and report
    (void)mbar_wait(&bar, 0, &abort_flag, status, WHERE_SELFTEST, limit_ns);
  }
  __syncthreads();
}

}  // namespace

cudaError_t route(const float* h, const void* const* keys, const void* const* summaries,
                  int n_blocks, void* u, float* alpha, int64_t rows, int D, sva_dtype_t dt,
                  cudaStream_t s) {
  RoutePtrs p{};
  for (int b = 0; b < n_blocks; ++b) {
    p.keys[b] = keys[b];
    p.summaries[b] = summaries[b];
  }
  const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
  if (dt == SVA_BF16 && D % 256 == 0 && D / 8 <= 512) {
    switch (n_blocks) {
      case 1: return launch_route_rows<1>(h, p, u, alpha, rows, D, inv_sqrt_d, s);
      case 2: return launch_route_rows<2>(h, p, u, alpha, rows, D, inv_sqrt_d, s);
      case 3: return launch_route_rows<3>(h, p, u, alpha, rows, D, inv_sqrt_d, s);
      case 4: return launch_route_rows<4>(h, p, u, alpha, rows, D, inv_sqrt_d, s);
      default: break;  // more blocks: the warp-per-row kernel below
    }
  }
  const int warps = 8;
  const unsigned grid = static_cast<unsigned>((rows + warps - 1) / warps);
  if (dt == SVA_BF16)
    route_kernel<__nv_bfloat16><<<grid, 32 * warps, 0, s>>>(
        h, p, n_blocks, static_cast<__nv_bfloat16*>(u), alpha, rows, D, inv_sqrt_d);
  else
    route_kernel<float><<<grid, 32 * warps, 0, s>>>(h, p, n_blocks, static_cast<float*>(u), alpha,
                                                    rows, D, inv_sqrt_d);
  return cudaGetLastError();
}

cudaError_t transpose_2d(const void* src, void* dst, int64_t rows, int64_t cols, sva_dtype_t dt,
                         cudaStream_t s) {
  dim3 grid(static_cast<unsigned>((cols + 31) / 32), static_cast<unsigned>((rows + 31) / 32));
  dim3 block(32, 8);
  if (dt == SVA_BF16)
    transpose_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(
        static_cast<const __nv_bfloat16*>(src), static_cast<__nv_bfloat16*>(dst), rows, cols);
  else
    transpose_kernel<float><<<grid, block, 0, s>>>(static_cast<const float*>(src),
                                                   static_cast<float*>(dst), rows, cols);
  return cudaGetLastError();
}

cudaError_t cast_f32(const float* src, void* dst, int64_t n, sva_dtype_t dt, cudaStream_t s) {
  if (dt == SVA_F32) {
    if (src == dst) return cudaSuccess;
    return cudaMemcpyAsync(dst, src, n * sizeof(float), cudaMemcpyDeviceToDevice, s);
  }
  const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, 148 * 16));
  cast_f32_to_bf16_kernel<<<grid, 256, 0, s>>>(src, static_cast<__nv_bfloat16*>(dst), n);
  return cudaGetLastError();
}

cudaError_t upcast_to_f32(const void* src, float* dst, int64_t n, sva_dtype_t dt, cudaStream_t s) {
  if (dt == SVA_F32) return cudaMemcpyAsync(dst, src, n * sizeof(float), cudaMemcpyDeviceToDevice, s);
  const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, 148 * 16));
  upcast_bf16_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src), dst, n);
  return cudaGetLastError();
}

cudaError_t sub_inplace(const float* a, float* out, int64_t n, cudaStream_t s) {
  const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, 148 * 16));
  sub_inplace_kernel<<<grid, 256, 0, s>>>(a, out, n);
  return cudaGetLastError();
}

cudaError_t selftest_wait(int* status, unsigned timeout_us, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(status, static_cast<uint64_t>(timeout_us) * 1000ull);
  return cudaGetLastError();
}

}  // namespace sva
