// gemm_tc.cu -- bf16 projections of a mixer layer on the 5th-generation tensor
// cores: C = A B^T with A [M, K] (activations) and B [N, K] (weights in the
// [out, in] layout of a linear layer), both K-major, fp32 accumulation in TMEM.
//
// Persistent kernel, one CTA per SM, warp-specialised:
//   warp 0      TMA producer: 128x64 A and 256x64 B tiles (128-byte swizzle)
//               into a 4-stage shared-memory ring;
//   warp 1      allocates 512 TMEM columns; lane 0 issues tcgen05.mma
//               (M=128, N=256, K=16) into one of two 256-column accumulators;
//   warps 2..5  epilogue: tcgen05.ld of their 32-lane quadrant, then either a
//               bf16 store (optional ReLU on the leading columns, the feature
//               map phi of the linear layers) or the residual update
//               h += C (fp32) with an optional bf16 copy of h.
// Two accumulators let the epilogue of tile i overlap the main loop of i+1.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sva {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;              // 16 KB
constexpr int B_STAGE = BN * BK * 2;              // 32 KB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;    // 48 KB
constexpr int TMEM_COLS = 2 * BN;                 // two fp32 accumulators
constexpr int NUM_THREADS = 192;

struct GemmTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kGemmSmem = 1024 + STAGES * STAGE_BYTES + sizeof(GemmTail);

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  int never = 0;
  return mbar_wait(bar, parity, &never, nullptr, 0);
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap map_a,
                        const __grid_constant__ CUtensorMap map_b, GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE;
  GemmTail* tl = reinterpret_cast<GemmTail*>(smem + STAGES * STAGE_BYTES);

  const int warp = warp_id(), lane = lane_id();
  const int m_tiles = static_cast<int>((g.M + BM - 1) / BM);
  const int n_tiles = static_cast<int>((g.N + BN - 1) / BN);
  const int num_tiles = m_tiles * n_tiles;
  const int k_blocks = static_cast<int>((g.K + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&tl->full[s], 1);
      mbar_init(&tl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tl->acc_full[a], 1);
      mbar_init(&tl->acc_empty[a], 4);
    }
    mbar_init(&tl->drain, 1);
    tl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tl->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tl->tmem_base;
  volatile int* abort_flag = &tl->abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile / n_tiles, n_blk = tile % n_tiles;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&tl->empty[stage], phase ^ 1, abort_flag, g.status, WHERE_GEMM)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&tl->full[stage], STAGE_BYTES);
          tma_load_2d(&map_a, &tl->full[stage], sA + stage * A_STAGE, kb * BK, m_blk * BM);
          tma_load_2d(&map_b, &tl->full[stage], sB + stage * B_STAGE, kb * BK, n_blk * BN);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // abort: let every load still in flight land before the CTA exits
        for (int64_t i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
          (void)drain_wait(&tl->full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, false);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&tl->acc_empty[acc], acc_phase ^ 1, abort_flag, g.status, WHERE_GEMM)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&tl->full[stage], phase, abort_flag, g.status, WHERE_GEMM)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_STAGE);
          const uint32_t b_addr = smem_u32(sB + stage * B_STAGE);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = smem_desc(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc(b_addr + kk * 32, 16, 1024);
            umma_ss(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&tl->empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) umma_commit(&tl->acc_full[acc]);
      }
      // every MMA issued above completes before TMEM is released
      umma_commit(&tl->drain);
      (void)drain_wait(&tl->drain, 0);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quadrant of this warp
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const bool w = mbar_wait(&tl->acc_full[acc], acc_phase, abort_flag, g.status, WHERE_GEMM);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
      const int m_blk = tile / n_tiles, n_blk = tile % n_tiles;
      const int64_t row = static_cast<int64_t>(m_blk) * BM + q * 32 + lane;
      const bool row_ok = row < g.M;
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + cc, r);
        tmem_wait_ld();
        const int64_t col0 = static_cast<int64_t>(n_blk) * BN + cc;
        if (!row_ok || col0 >= g.N) continue;
        const bool full = col0 + 32 <= g.N;
        if (EPI == EPI_STORE) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            v[i] = __uint_as_float(r[i]);
            if (col0 + i < g.relu_cols) v[i] = relu_f(v[i]);
          }
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.c) + row * g.ldc + col0;
          if (full) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 w;
              w.x = pack_bf16x2(v[i], v[i + 1]);
              w.y = pack_bf16x2(v[i + 2], v[i + 3]);
              w.z = pack_bf16x2(v[i + 4], v[i + 5]);
              w.w = pack_bf16x2(v[i + 6], v[i + 7]);
              *reinterpret_cast<uint4*>(out + i) = w;
            }
          } else {
            for (int i = 0; col0 + i < g.N; ++i) out[i] = __float2bfloat16_rn(v[i]);
          }
        } else {
          float* hp = g.h + row * g.ldh + col0;
          float v[32];
          if (full) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              float4 x = *reinterpret_cast<const float4*>(hp + i);
              x.x += __uint_as_float(r[i]);
              x.y += __uint_as_float(r[i + 1]);
              x.z += __uint_as_float(r[i + 2]);
              x.w += __uint_as_float(r[i + 3]);
              *reinterpret_cast<float4*>(hp + i) = x;
              v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
            }
            if (g.h_copy != nullptr) {
              __nv_bfloat16* cp = static_cast<__nv_bfloat16*>(g.h_copy) + row * g.ldhc + col0;
#pragma unroll
              for (int i = 0; i < 32; i += 8) {
                uint4 w;
                w.x = pack_bf16x2(v[i], v[i + 1]);
                w.y = pack_bf16x2(v[i + 2], v[i + 3]);
                w.z = pack_bf16x2(v[i + 4], v[i + 5]);
                w.w = pack_bf16x2(v[i + 6], v[i + 7]);
                *reinterpret_cast<uint4*>(cp + i) = w;
              }
            }
          } else {
            for (int i = 0; col0 + i < g.N; ++i) {
              const float x = hp[i] + __uint_as_float(r[i]);
              hp[i] = x;
              if (g.h_copy != nullptr)
                static_cast<__nv_bfloat16*>(g.h_copy)[row * g.ldhc + col0 + i] =
                    __float2bfloat16_rn(x);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

cudaError_t gemm_bf16(const GemmArgs& g, cudaStream_t s) {
  CUtensorMap ma, mb;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(g.K), static_cast<uint64_t>(g.M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(g.lda) * 2};
    const uint32_t box[2] = {BK, BM};
    if (!encode_tmap(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.a, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(g.K), static_cast<uint64_t>(g.N)};
    const uint64_t strides[1] = {static_cast<uint64_t>(g.ldb) * 2};
    const uint32_t box[2] = {BK, BN};
    if (!encode_tmap(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.b, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const int64_t tiles = ((g.M + BM - 1) / BM) * ((g.N + BN - 1) / BN);
  const int grid = static_cast<int>(std::min<int64_t>(tiles, device_sm_count()));
  cudaError_t e;
  if (g.epi == EPI_STORE) {
    e = cudaFuncSetAttribute(gemm_bf16_tc_kernel<EPI_STORE>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kGemmSmem));
    if (e != cudaSuccess) return e;
    gemm_bf16_tc_kernel<EPI_STORE><<<grid, NUM_THREADS, kGemmSmem, s>>>(ma, mb, g);
  } else {
    e = cudaFuncSetAttribute(gemm_bf16_tc_kernel<EPI_RESIDUAL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kGemmSmem));
    if (e != cudaSuccess) return e;
    gemm_bf16_tc_kernel<EPI_RESIDUAL><<<grid, NUM_THREADS, kGemmSmem, s>>>(ma, mb, g);
  }
  return cudaGetLastError();
}

}  // namespace sva
