// anchor_tc.cu -- the gated softmax anchor, bf16, d = 128, on tcgen05/TMEM.
//
// Every fourth layer of the hybrid is gated softmax attention, which keeps the
// exact token relations the linear layers approximate [lode.cx summary, "How
// It Works"]: Y_t = sum_s softmax_s(scale Q_t . K_s) V_s * sigmoid(G_t),
// non-causal. FlashAttention-style: no N x N matrix is ever stored.
//
// One CTA per (128-query tile, head, batch); 6 warps:
//   warp 0      TMA: the Q tile once, then 128-key K and V tiles (2 stages)
//   warp 1      TMEM (512 columns: S0 | S1 | O); lane 0 issues the MMAs:
//               S_j = Q K_j^T (SS, M=128 N=128) into S[j%2] and
//               O += P_j V_j with P_j read from TMEM (TS, V MN-major)
//   warps 2..5  softmax: thread r owns query row r (its TMEM lane); loads S_j,
//               online max in the log2 domain, exp2, row sum, writes P_j as
//               bf16 over the first 64 columns of S[j%2]; rescales the O row
//               only when the running max grows by more than 2^8 (the stale
//               max keeps every p <= 2^8, exact after the final 1/l); then the
//               epilogue O / l * sigmoid(G) (+ residual) -> bf16.
// The MMA of S_{j+1} and of P_{j-1} V_{j-1} overlap the softmax of S_j.
#include <algorithm>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace sva {
namespace {

constexpr int HD = 128;
constexpr int BQ = 128, BKV = 128;
constexpr int BOX = 128 * 128;              // [64 cols x 128 rows] bf16 = 16 KB
constexpr int KV_STAGES = 2;
constexpr int Q_OFF = 0;                     // 32 KB
constexpr int KV_OFF = 2 * BOX;              // stage s: K at +s*64K, V at +s*64K+32K
constexpr int KV_STAGE_BYTES = 4 * BOX;
constexpr int TAIL_OFF = KV_OFF + KV_STAGES * KV_STAGE_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int S_COL0 = 0, O_COL = 256;
constexpr float kRescaleThreshold = 8.0f;    // log2 units

struct AnchorTail {
  uint64_t q_full;
  uint64_t k_full[KV_STAGES];
  uint64_t v_full[KV_STAGES];
  uint64_t kv_empty[KV_STAGES];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kAnchorSmem = 1024 + TAIL_OFF + sizeof(AnchorTail);

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  int never = 0;
  return mbar_wait(bar, parity, &never, nullptr, 0);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(192, 1)
    anchor_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                     const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, int N, float scale_log2,
                     const __nv_bfloat16* gate, int64_t ldg, const __nv_bfloat16* residual,
                     int64_t ldr, __nv_bfloat16* out, int64_t ldo, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  AnchorTail* tl = reinterpret_cast<AnchorTail*>(smem + TAIL_OFF);
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = warp_id(), lane = lane_id();
  const int nkv = (N + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(&tl->q_full, 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&tl->k_full[s], 1);
      mbar_init(&tl->v_full[s], 1);
      mbar_init(&tl->kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tl->s_full[i], 1);
      mbar_init(&tl->p_full[i], 128);
    }
    mbar_init(&tl->o_done, 1);
    mbar_init(&tl->drain, 1);
    tl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tl->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_q);
    tma_prefetch_desc(&map_k);
    tma_prefetch_desc(&map_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tl->tmem_base;
  volatile int* abort_flag = &tl->abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      mbar_arrive_expect_tx(&tl->q_full, 2 * BOX);
      tma_load_3d(&map_q, &tl->q_full, smem + Q_OFF, h * HD, qt * BQ, b);
      tma_load_3d(&map_q, &tl->q_full, smem + Q_OFF + BOX, h * HD + 64, qt * BQ, b);
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % KV_STAGES;
        const uint32_t ph = (j / KV_STAGES) & 1;
        if (!mbar_wait(&tl->kv_empty[st], ph ^ 1, abort_flag, status, WHERE_ANCHOR)) {
          ok = false;
          break;
        }
        uint8_t* kt = smem + KV_OFF + st * KV_STAGE_BYTES;
        mbar_arrive_expect_tx(&tl->k_full[st], 2 * BOX);
        tma_load_3d(&map_k, &tl->k_full[st], kt, h * HD, j * BKV, b);
        tma_load_3d(&map_k, &tl->k_full[st], kt + BOX, h * HD + 64, j * BKV, b);
        mbar_arrive_expect_tx(&tl->v_full[st], 2 * BOX);
        tma_load_3d(&map_v, &tl->v_full[st], kt + 2 * BOX, h * HD, j * BKV, b);
        tma_load_3d(&map_v, &tl->v_full[st], kt + 3 * BOX, h * HD + 64, j * BKV, b);
        ++issued;
      }
      (void)drain_wait(&tl->q_full, 0);
      if (!ok)
        for (int i = max(0, issued - KV_STAGES); i < issued; ++i) {
          (void)drain_wait(&tl->k_full[i % KV_STAGES], (i / KV_STAGES) & 1);
          (void)drain_wait(&tl->v_full[i % KV_STAGES], (i / KV_STAGES) & 1);
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_s = idesc_bf16_f32(BQ, BKV, false, false);  // Q, K: K-major
      constexpr uint32_t idesc_o = idesc_bf16_f32(BQ, HD, false, true);    // P (TMEM), V: MN-major
      const uint32_t qaddr = smem_u32(smem + Q_OFF);
      bool ok = mbar_wait(&tl->q_full, 0, abort_flag, status, WHERE_ANCHOR);
      auto issue_s = [&](int j) -> bool {
        const int st = j % KV_STAGES;
        if (!mbar_wait(&tl->k_full[st], (j / KV_STAGES) & 1, abort_flag, status, WHERE_ANCHOR))
          return false;
        tc_fence_after();
        const uint32_t kaddr = smem_u32(smem + KV_OFF + st * KV_STAGE_BYTES);
        const uint32_t d_tmem = tmem + S_COL0 + (j & 1) * BKV;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const int bx = kk >> 2, w = kk & 3;
          const uint64_t ad = smem_desc(qaddr + bx * BOX + w * 32, 16, 1024);
          const uint64_t bd = smem_desc(kaddr + bx * BOX + w * 32, 16, 1024);
          umma_ss(d_tmem, ad, bd, idesc_s, kk != 0 ? 1u : 0u);
        }
        umma_commit(&tl->s_full[j & 1]);
        return true;
      };
      if (ok && nkv > 0) ok = issue_s(0);
      for (int j = 0; j < nkv && ok; ++j) {
        if (j + 1 < nkv && !issue_s(j + 1)) {
          ok = false;
          break;
        }
        const int st = j % KV_STAGES;
        if (!mbar_wait(&tl->p_full[j & 1], (j >> 1) & 1, abort_flag, status, WHERE_ANCHOR) ||
            !mbar_wait(&tl->v_full[st], (j / KV_STAGES) & 1, abort_flag, status, WHERE_ANCHOR)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t vaddr = smem_u32(smem + KV_OFF + st * KV_STAGE_BYTES + 2 * BOX);
        const uint32_t p_tmem = tmem + S_COL0 + (j & 1) * BKV;
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint64_t bd = smem_desc(vaddr + kk * 2048, BOX, 1024);
          umma_ts(tmem + O_COL, p_tmem + kk * 8, bd, idesc_o, (j | kk) != 0 ? 1u : 0u);
        }
        umma_commit(&tl->o_done);
        umma_commit(&tl->kv_empty[st]);
      }
      umma_commit(&tl->drain);
      (void)drain_wait(&tl->drain, 0);
    }
  } else {
    // ------------------------------------------------ softmax + epilogue (warps 2..5)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    float m = -INFINITY;  // running (possibly stale) max of scaled logits, log2 units
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      bool w = mbar_wait(&tl->s_full[j & 1], (j >> 1) & 1, abort_flag, status, WHERE_ANCHOR);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sc = tmem + lane_base + S_COL0 + (j & 1) * BKV;
      float s[BKV];
#pragma unroll
      for (int c = 0; c < BKV; c += 32) {
        uint32_t v[32];
        tmem_ld32(sc + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c + i] = __uint_as_float(v[i]) * scale_log2;
      }
      const int valid = N - j * BKV;  // keys of this block inside the sequence
      if (valid < BKV) {
#pragma unroll
        for (int i = 0; i < BKV; ++i)
          if (i >= valid) s[i] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int i = 1; i < BKV; ++i) mx = fmaxf(mx, s[i]);
      float m_use = m;
      float factor = 1.f;
      const bool grow = mx > m + kRescaleThreshold;
      if (grow) {
        factor = (m == -INFINITY) ? 0.f : ex2(m - mx);
        m_use = mx;
      }
      // rescale the O row (only rows whose max grew; warps where none did skip it)
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        bool wo = mbar_wait(&tl->o_done, (j - 1) & 1, abort_flag, status, WHERE_ANCHOR);
        if (!__all_sync(0xffffffffu, wo)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < HD; c += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + O_COL + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * factor);
          tmem_st32(tmem + lane_base + O_COL + c, v);
        }
        tmem_wait_st();
      }
      l *= factor;
      m = m_use;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < BKV; c += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2(s[c + 2 * i] - m);
          const float p1 = ex2(s[c + 2 * i + 1] - m);
          rs += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(sc + c / 2, pk);
      }
      tmem_wait_st();
      l += rs;
      tc_fence_before();
      mbar_arrive(&tl->p_full[j & 1]);
    }
    if (ok && nkv > 0) {
      bool w = mbar_wait(&tl->o_done, (nkv - 1) & 1, abort_flag, status, WHERE_ANCHOR);
      ok = __all_sync(0xffffffffu, w);
    }
    if (ok) {
      tc_fence_after();
      const int t = qt * BQ + r;
      const float inv = 1.0f / l;
      const bool row_ok = t < N;
      const int64_t row = static_cast<int64_t>(b) * N + t;
#pragma unroll 1
      for (int c = 0; c < HD; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + O_COL + c, v);
        tmem_wait_ld();
        if (!row_ok) continue;
        const __nv_bfloat16* gp = gate + row * ldg + h * HD + c;
        __nv_bfloat16* op = out + row * ldo + h * HD + c;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 gv = *reinterpret_cast<const uint4*>(gp + 8 * k);
          const float gg[8] = {bf16lo_to_f32(gv.x), bf16hi_to_f32(gv.x), bf16lo_to_f32(gv.y),
                               bf16hi_to_f32(gv.y), bf16lo_to_f32(gv.z), bf16hi_to_f32(gv.z),
                               bf16lo_to_f32(gv.w), bf16hi_to_f32(gv.w)};
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            y[e] = __uint_as_float(v[8 * k + e]) * inv * fast_sigmoid(gg[e]);
          if (residual != nullptr) {
            const uint4 rv =
                *reinterpret_cast<const uint4*>(residual + row * ldr + h * HD + c + 8 * k);
            y[0] += bf16lo_to_f32(rv.x); y[1] += bf16hi_to_f32(rv.x);
            y[2] += bf16lo_to_f32(rv.y); y[3] += bf16hi_to_f32(rv.y);
            y[4] += bf16lo_to_f32(rv.z); y[5] += bf16hi_to_f32(rv.z);
            y[6] += bf16lo_to_f32(rv.w); y[7] += bf16hi_to_f32(rv.w);
          }
          uint4 o;
          o.x = pack_bf16x2(y[0], y[1]);
          o.y = pack_bf16x2(y[2], y[3]);
          o.z = pack_bf16x2(y[4], y[5]);
          o.w = pack_bf16x2(y[6], y[7]);
          *reinterpret_cast<uint4*>(op + 8 * k) = o;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

bool act_map(CUtensorMap* m, const void* base, int64_t ld, int B, int N, int D) {
  const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(N),
                            static_cast<uint64_t>(B)};
  const uint64_t strides[2] = {static_cast<uint64_t>(ld) * 2,
                               static_cast<uint64_t>(ld) * 2 * static_cast<uint64_t>(N)};
  const uint32_t box[3] = {64, 128, 1};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

cudaError_t anchor_bf16(const sva_attn_args& a, int* status, cudaStream_t s) {
  const int D = a.H * a.d;
  CUtensorMap mq, mk, mv;
  if (!act_map(&mq, a.q, a.ldq, a.B, a.N, D) || !act_map(&mk, a.k, a.ldk, a.B, a.N, D) ||
      !act_map(&mv, a.v, a.ldv, a.B, a.N, D))
    return cudaErrorInvalidValue;
  const float scale = a.scale != 0.f ? a.scale : 1.0f / sqrtf(static_cast<float>(a.d));
  const float scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e = cudaFuncSetAttribute(anchor_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kAnchorSmem));
  if (e != cudaSuccess) return e;
  dim3 grid((a.N + BQ - 1) / BQ, a.H, a.B);
  anchor_tc_kernel<<<grid, 192, kAnchorSmem, s>>>(
      mq, mk, mv, a.N, scale_log2, static_cast<const __nv_bfloat16*>(a.gate), a.ldg,
      static_cast<const __nv_bfloat16*>(a.residual), a.ldr, static_cast<__nv_bfloat16*>(a.out),
      a.ldo, status);
  return cudaGetLastError();
}

}  // namespace sva
