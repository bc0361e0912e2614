// anchor_tc.cu -- the gated softmax anchor, bf16, d = 128, on tcgen05/TMEM.
//
// Every fourth layer of the hybrid is gated softmax attention, which keeps the
// exact token relations the linear layers approximate [lode.cx summary, "How
// It Works"]: Y_t = sum_s softmax_s(scale Q_t . K_s) V_s * sigmoid(G_t),
// non-causal. FlashAttention-style: no N x N matrix is ever stored.
//
// One CTA per pair of 128-query tiles of one (head, batch); 12 warps in three
// warpgroups (the TMA and MMA warps run their loops with all 32 lanes, lane 0
// issuing; single-lane loops inside those warps, with the other 31 lanes
// parked at the end-of-kernel barrier, measured 1.7% slower at 720p: 3.89
// against 3.82 ms):
//   WG0  warp 0: TMA for both Q tiles once, then the 128-key K tiles (3-stage
//        ring), then, once the last S MMAs have read Q, the two tiles of the
//        gate G into Q's buffer, so the epilogue reads G from shared memory
//        (it used to wait on DRAM for each 32-column chunk: ~17,000 cycles of
//        a CTA's ~560,000 with the tensor pipe idle; 720p 3.87 -> 3.79 ms);
//        warp 2: TMA for the V tiles (2-stage ring); warp 3: checks that V_j and
//        K_{j+1} have landed and adds one arrival to each tile's P barrier, so
//        the MMA thread waits on P only and the softmax reports P without that
//        check on its chain (720p 3.75 -> 3.69-3.72 ms). K is released as
//        soon as both S MMAs of a block have read it, V after both P V MMAs,
//        so the next block's K is already resident when its S MMA is due.
//        warp 1: allocates all 512 TMEM columns (tile t: S_t at 256t, O_t at
//        256t+128) and issues every MMA from one thread. Registers shrink to 56.
//   WG1, WG2  softmax of tile 0 and tile 1: thread r owns query row r (its
//        TMEM lane). Registers grow to 224 so a row of S stays in registers.
// The MMA thread ping-pongs the tiles: O_0 += P_0 V_j, S_0 = Q_0 K_{j+1}, then
// O_1 += P_1 V_j, S_1 = Q_1 K_{j+1}, so the tensor core works on one tile while
// the other tile's softmax runs. P (bf16) is written over the first 64 columns
// of S and consumed straight from TMEM (A operand in TMEM); in-order execution
// of the MMAs keeps S_{j+1} from overwriting P_j before P_j V_j has read it,
// and the commit that reports S_{j+1} also covers P_j V_j, so a softmax warp
// that sees S_{j+1} may rescale O.
// Softmax per row: running max in the log2 domain, rescaled only when it grows
// by more than 8 (p <= 2^8 otherwise, exact after the final 1/l); the max uses
// three-input max, and the scale-and-shift and the row sum run on packed fp32
// pairs (one f32x2 FFMA or FADD per two keys). Exponentials run on the MUFU
// unit (sending a share of them to the FMA pipe as a polynomial was measured
// slower: the MUFU pipe is not what bounds this kernel).
// What bounds it (720p layer on B200, clock64 traces of one CTA, ncu): each
// tile's chain -- softmax of block j (about 1,700 cycles: S load 70, block
// max 350, exponentials and P stores 1,190, report 100), then the MMA warp
// noticing P (~350), P_j V_j and S_{j+1} on the tensor core (about 1,370; the
// S MMAs, both operands in shared memory, ~97 cycles each against 64 nominal),
// then the softmax seeing S_{j+1} (~150) -- sets the step at about 3,580
// cycles for two tiles. The exponential loop is near its minimum instruction
// count, and any instruction added to it lengthens it (a polynomial for part
// of the exponentials, or the block max folded into it). ncu against the
// library's sm100 flash kernel at the same shape shows the same MMA count and
// the same shared-memory and TMEM traffic; that kernel runs 16 warps and
// issues more per cycle. Descriptors are built once and offset by constants,
// since the MMA warp's own instruction count reaches the tensor pipe (8,190
// keys: 0.87 -> 0.79 ms; 720p: 3.94 -> 3.90 ms). Earlier steps: packed pairs
// 4.35 -> 4.02 ms; the waits for V_j and K_{j+1} moved from the MMA thread to
// a softmax warp of each tile, 3.94 ms; later to warp 3, with warp-uniform
// role loops and G prefetched for the epilogue: 3.66-3.72 ms.
#include <algorithm>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace sva {
namespace {

constexpr int HD = 128;
constexpr int BQ = 128, BKV = 128;
constexpr int BOX = 128 * 128;              // [64 cols x 128 rows] bf16 = 16 KB
constexpr int K_STAGES = 3, V_STAGES = 2;
constexpr int Q_OFF = 0;                     // tile t: 32 KB at Q_OFF + t * 2 * BOX
constexpr int K_OFF = 4 * BOX;               // K stage s: 32 KB at K_OFF + s * 2 * BOX
constexpr int V_OFF = K_OFF + K_STAGES * 2 * BOX;
constexpr int TAIL_OFF = V_OFF + V_STAGES * 2 * BOX;
constexpr int NUM_THREADS = 384;
constexpr int TMEM_COLS = 512;
constexpr float kRescaleThreshold = 8.0f;    // log2 units
// register split: 128 threads at 56 + 256 threads at 224 = 384 threads at 168
constexpr int kRegsProducer = 56, kRegsSoftmax = 224;

struct AnchorTail {
  uint64_t q_full;
  uint64_t k_full[K_STAGES];
  uint64_t k_empty[K_STAGES];
  uint64_t v_full[V_STAGES];
  uint64_t v_empty[V_STAGES];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t g_full;    // the gate tiles, loaded into the Q buffer once Q is no longer read
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kAnchorSmem = 1024 + TAIL_OFF + sizeof(AnchorTail);

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  int never = 0;
  return mbar_wait(bar, parity, &never, nullptr, 0);
}

__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Work of one launch: units (query-tile pair, head, batch), x fastest. The
// first n_full units run whole, one CTA each. The remaining units (the last,
// partial wave) are split `split` ways along the key blocks. Each part writes
// its unnormalised O, running max m and row sum l to `partial` and
// anchor_merge_kernel combines them. This shortens a last wave that would leave
// most SMs idle. 720p (1,824 units, 48 in the last wave, split 3): the span
// of the kernel drops from 3.95 to 3.85 ms on one B200, and launch to launch
// (merge included, 14 us) from 3.96-4.01 to 3.95-3.99 ms. It pays most when
// a call has fewer units than SMs.
struct AnchorWork {
  int n_qunits, H, n_full, n_split_units, split, nkv_total;
  float* partial;  // [n_split_units][split][2 tiles][BQ x HD O | BQ x (m, l)]
};
constexpr int PART_FLOATS = BQ * HD + 2 * BQ;

__global__ void __launch_bounds__(NUM_THREADS, 1)
    anchor_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                     const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v,
                     const __grid_constant__ CUtensorMap map_g, int N, int Nk,
                     float scale_log2, AnchorWork wk,
                     const __nv_bfloat16* gate, int64_t ldg, const __nv_bfloat16* residual,
                     int64_t ldr, __nv_bfloat16* out, int64_t ldo, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  AnchorTail* tl = reinterpret_cast<AnchorTail*>(smem + TAIL_OFF);
  // this CTA's unit and key blocks [kb0, kb0 + nkv)
  int unit = blockIdx.x, kb0 = 0, nkv = wk.nkv_total, part = -1, su = 0;
  if (unit >= wk.n_full) {
    const int sidx = unit - wk.n_full;
    su = sidx / wk.split;
    part = sidx - su * wk.split;
    unit = wk.n_full + su;
    kb0 = part * wk.nkv_total / wk.split;
    nkv = (part + 1) * wk.nkv_total / wk.split - kb0;
  }
  const int q0 = (unit % wk.n_qunits) * 2 * BQ;
  const int h = (unit / wk.n_qunits) % wk.H, b = unit / (wk.n_qunits * wk.H);
  const int warp = warp_id(), lane = lane_id();
  const int wg = warp >> 2;
  const bool has1 = q0 + BQ < N;  // the second tile holds at least one query

  if (threadIdx.x == 0) {
    mbar_init(&tl->q_full, 1);
    for (int s = 0; s < K_STAGES; ++s) {
      mbar_init(&tl->k_full[s], 1);
      mbar_init(&tl->k_empty[s], 1);
    }
    for (int s = 0; s < V_STAGES; ++s) {
      mbar_init(&tl->v_full[s], 1);
      mbar_init(&tl->v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tl->s_full[i], 1);
      mbar_init(&tl->p_full[i], 129);  // + warp 3: V_j, K_{j+1} resident
    }
    mbar_init(&tl->o_done, 1);
    mbar_init(&tl->g_full, 1);
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

  if (wg == 0) {
    warpgroup_reg_dec<kRegsProducer>();
    // The three role warps run their loops with all 32 lanes (warp-uniform
    // control flow); lane 0 alone issues the TMA copies, MMAs and commits.
    if (warp == 0) {
      // ------------------------------------------------ TMA producer: Q, then K
      if (lane == 0) {
        mbar_arrive_expect_tx(&tl->q_full, (has1 ? 4 : 2) * BOX);
        tma_load_3d(&map_q, &tl->q_full, smem + Q_OFF, h * HD, q0, b);
        tma_load_3d(&map_q, &tl->q_full, smem + Q_OFF + BOX, h * HD + 64, q0, b);
        if (has1) {
          tma_load_3d(&map_q, &tl->q_full, smem + Q_OFF + 2 * BOX, h * HD, q0 + BQ, b);
          tma_load_3d(&map_q, &tl->q_full, smem + Q_OFF + 3 * BOX, h * HD + 64, q0 + BQ, b);
        }
      }
      __syncwarp();
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % K_STAGES;
        const bool w = mbar_wait(&tl->k_empty[st], ((j / K_STAGES) & 1) ^ 1, abort_flag, status,
                                 WHERE_ANCHOR);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* kt = smem + K_OFF + st * 2 * BOX;
          mbar_arrive_expect_tx(&tl->k_full[st], 2 * BOX);
          tma_load_3d(&map_k, &tl->k_full[st], kt, h * HD, (kb0 + j) * BKV, b);
          tma_load_3d(&map_k, &tl->k_full[st], kt + BOX, h * HD + 64, (kb0 + j) * BKV, b);
        }
        __syncwarp();
        ++issued;
      }
      // The gate of both tiles goes into Q's buffer once the last S MMAs have
      // read Q (the commit that frees the last K stage covers them), so the
      // epilogue reads it from shared memory instead of waiting on DRAM.
      if (ok && part < 0 && nkv > 0) {
        const bool w = mbar_wait(&tl->k_empty[(nkv - 1) % K_STAGES], ((nkv - 1) / K_STAGES) & 1,
                                 abort_flag, status, WHERE_ANCHOR);
        ok = __all_sync(0xffffffffu, w);
        if (ok && lane == 0) {
          mbar_arrive_expect_tx(&tl->g_full, (has1 ? 4 : 2) * BOX);
          tma_load_3d(&map_g, &tl->g_full, smem + Q_OFF, h * HD, q0, b);
          tma_load_3d(&map_g, &tl->g_full, smem + Q_OFF + BOX, h * HD + 64, q0, b);
          if (has1) {
            tma_load_3d(&map_g, &tl->g_full, smem + Q_OFF + 2 * BOX, h * HD, q0 + BQ, b);
            tma_load_3d(&map_g, &tl->g_full, smem + Q_OFF + 3 * BOX, h * HD + 64, q0 + BQ, b);
          }
        }
        __syncwarp();
      }
      if (lane == 0) {
        (void)drain_wait(&tl->q_full, 0);
        if (ok && part < 0 && nkv > 0) (void)drain_wait(&tl->g_full, 0);
        if (!ok)
          for (int i = max(0, issued - K_STAGES); i < issued; ++i)
            (void)drain_wait(&tl->k_full[i % K_STAGES], (i / K_STAGES) & 1);
      }
      __syncwarp();
    } else if (warp == 2) {
      // ------------------------------------------------ TMA producer: V
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % V_STAGES;
        const bool w = mbar_wait(&tl->v_empty[st], ((j / V_STAGES) & 1) ^ 1, abort_flag, status,
                                 WHERE_ANCHOR);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* vt = smem + V_OFF + st * 2 * BOX;
          mbar_arrive_expect_tx(&tl->v_full[st], 2 * BOX);
          tma_load_3d(&map_v, &tl->v_full[st], vt, h * HD, (kb0 + j) * BKV, b);
          tma_load_3d(&map_v, &tl->v_full[st], vt + BOX, h * HD + 64, (kb0 + j) * BKV, b);
        }
        __syncwarp();
        ++issued;
      }
      if (lane == 0 && !ok)
        for (int i = max(0, issued - V_STAGES); i < issued; ++i)
          (void)drain_wait(&tl->v_full[i % V_STAGES], (i / V_STAGES) & 1);
      __syncwarp();
    } else if (warp == 3) {
      // ------------------------------------------------ residency of V_j and K_{j+1}
      // one arrival per tile and block on p_full once both have landed; it
      // waits for that phase to complete before checking the next block, so
      // it never arrives twice in one phase
      const int ntiles = has1 ? 2 : 1;
      for (int j = 0; j < nkv; ++j) {
        bool w = mbar_wait(&tl->v_full[j % V_STAGES], (j / V_STAGES) & 1, abort_flag, status,
                           WHERE_ANCHOR);
        if (j + 1 < nkv)
          w = w && mbar_wait(&tl->k_full[(j + 1) % K_STAGES], ((j + 1) / K_STAGES) & 1, abort_flag,
                             status, WHERE_ANCHOR);
        if (!__all_sync(0xffffffffu, w)) break;
        if (lane == 0)
          for (int t = 0; t < ntiles; ++t) mbar_arrive(&tl->p_full[t]);
        __syncwarp();
        bool wp = true;
        for (int t = 0; t < ntiles; ++t)
          wp = wp && mbar_wait(&tl->p_full[t], j & 1, abort_flag, status, WHERE_ANCHOR);
        if (!__all_sync(0xffffffffu, wp)) break;
      }
    } else if (warp == 1) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_s = idesc_bf16_f32(BQ, BKV, false, false);  // Q, K: K-major
      constexpr uint32_t idesc_o = idesc_bf16_f32(BQ, HD, false, true);    // P (TMEM), V: MN-major
      const int ntiles = has1 ? 2 : 1;
      bool ok = __all_sync(0xffffffffu,
                           mbar_wait(&tl->q_full, 0, abort_flag, status, WHERE_ANCHOR));
      // The MMA thread shares its SM sub-partition with two softmax warps, so
      // its own instruction count is on the critical path: descriptors are
      // built once and each MMA adds a compile-time offset to a stage's base
      // (start addresses stay below 256 KB, so the 14-bit field never carries).
      const uint64_t qd0 = smem_desc(smem_u32(smem + Q_OFF), 16, 1024);
      const uint64_t kd0 = smem_desc(smem_u32(smem + K_OFF), 16, 1024);
      const uint64_t vd0 = smem_desc(smem_u32(smem + V_OFF), BOX, 1024);
      auto issue_s = [&](int t, int kst) {
        const uint64_t qb = qd0 + static_cast<uint64_t>(t * (2 * BOX >> 4));
        const uint64_t kb = kd0 + static_cast<uint64_t>(kst * (2 * BOX >> 4));
        const uint32_t d_tmem = tmem + t * 256;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = static_cast<uint32_t>(((kk >> 2) * BOX + (kk & 3) * 32) >> 4);
          umma_ss(d_tmem, qb + off, kb + off, idesc_s, kk != 0 ? 1u : 0u);
        }
        umma_commit(&tl->s_full[t]);
      };
      auto issue_pv = [&](int t, int vst, bool first) {
        const uint64_t vb = vd0 + static_cast<uint64_t>(vst * (2 * BOX >> 4));
        const uint32_t p_tmem = tmem + t * 256;
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          umma_ts(p_tmem + 128, p_tmem + kk * 8, vb + static_cast<uint32_t>(kk * 2048 >> 4), idesc_o,
                  (kk != 0 || !first) ? 1u : 0u);
      };
      if (ok && nkv > 0) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&tl->k_full[0], 0, abort_flag, status, WHERE_ANCHOR));
        if (ok) {
          tc_fence_after();
          if (lane == 0) {
            for (int t = 0; t < ntiles; ++t) issue_s(t, 0);
            umma_commit(&tl->k_empty[0]);
          }
          __syncwarp();
        }
      }
      int vst = 0, kn = 1 % K_STAGES;  // stages of V_j and K_{j+1}
      for (int j = 0; j < nkv && ok; ++j) {
        const bool more = j + 1 < nkv;
        // V_j and K_{j+1} need no wait here: warp 3 saw them land before its
        // arrival on p_full, which the P_j wait below includes
        for (int t = 0; t < ntiles; ++t) {
          const bool w = mbar_wait(&tl->p_full[t], j & 1, abort_flag, status, WHERE_ANCHOR);
          if (!__all_sync(0xffffffffu, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            issue_pv(t, vst, j == 0);
            if (t == ntiles - 1) umma_commit(&tl->v_empty[vst]);
            if (more) {
              issue_s(t, kn);
              if (t == ntiles - 1) umma_commit(&tl->k_empty[kn]);
            }
          }
          __syncwarp();
        }
        vst = vst + 1 == V_STAGES ? 0 : vst + 1;
        kn = kn + 1 == K_STAGES ? 0 : kn + 1;
      }
      if (lane == 0) {
        if (ok) umma_commit(&tl->o_done);
        umma_commit(&tl->drain);
        (void)drain_wait(&tl->drain, 0);
      }
      __syncwarp();
    }
  } else {
    warpgroup_reg_inc<kRegsSoftmax>();
    // ------------------------------------------------ softmax + epilogue (WG1: tile 0, WG2: tile 1)
    const int t = wg - 1;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t s_col = tmem + lane_base + t * 256;
    const uint32_t o_col = s_col + 128;
    if (t == 0 || has1) {
      float m = -INFINITY;  // running (possibly stale) max of scaled logits, log2 units
      float l = 0.f;
      bool ok = true;
      for (int j = 0; j < nkv; ++j) {
        bool w = mbar_wait(&tl->s_full[t], j & 1, abort_flag, status, WHERE_ANCHOR);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[4][32];
        tmem_ld32(s_col, v[0]);
        tmem_ld32(s_col + 32, v[1]);
        tmem_ld32(s_col + 64, v[2]);
        tmem_ld32(s_col + 96, v[3]);
        tmem_wait_ld();
        float s[BKV];
#pragma unroll
        for (int i = 0; i < BKV; ++i) s[i] = __uint_as_float(v[i >> 5][i & 31]);
        const int valid = Nk - (kb0 + j) * BKV;  // keys of this block inside the sequence
        if (valid < BKV) {
#pragma unroll
          for (int i = 0; i < BKV; ++i)
            if (i >= valid) s[i] = -INFINITY;
        }
        // row max: eight chains of three-input max over the 128 keys
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = max3_f(s[k], s[k + 8], s[k + 16]);
#pragma unroll
        for (int base = 24; base + 16 <= BKV - 8; base += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = max3_f(mx8[k], s[base + k], s[base + 8 + k]);
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], s[BKV - 8 + k]);
        const float mx = fmaxf(max3_f(max3_f(mx8[0], mx8[1], mx8[2]),
                                      max3_f(mx8[3], mx8[4], mx8[5]), mx8[6]),
                               mx8[7]) *
                         scale_log2;
        const bool grow = mx > m + kRescaleThreshold;
        float factor = 1.f;
        if (grow) {
          factor = (m == -INFINITY) ? 0.f : ex2_mufu(m - mx);
          m = mx;
        }
        // O of this tile is complete up to block j-1 here: the commit that
        // reported S_j also covers P_{j-1} V_{j-1}
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < HD; c += 32) {
            uint32_t o[32];
            tmem_ld32(o_col + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
            tmem_st32(o_col + c, o);
          }
        }
        l *= factor;
        // x = s * scale - m and the row sum on packed pairs (f32x2)
        const uint64_t scale2 = f2pack(scale_log2, scale_log2), negm2 = f2pack(-m, -m);
        uint64_t acc2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc2[i] = f2pack(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1;
            f2unpack(fma_f2(f2pack(s[32 * c + 2 * i], s[32 * c + 2 * i + 1]), scale2, negm2), x0,
                     x1);
            const float p0 = ex2_mufu(x0);
            const float p1 = ex2_mufu(x1);
            acc2[i & 3] = add_f2(acc2[i & 3], f2pack(p0, p1));
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st16(s_col + 16 * c, pk);
        }
        tmem_wait_st();
        {
          float u0, u1;
          f2unpack(add_f2(add_f2(acc2[0], acc2[1]), add_f2(acc2[2], acc2[3])), u0, u1);
          l += u0 + u1;
        }
        tc_fence_before();
        mbar_arrive(&tl->p_full[t]);
      }
      if (ok && nkv > 0) {
        bool w = mbar_wait(&tl->o_done, 0, abort_flag, status, WHERE_ANCHOR);
        ok = __all_sync(0xffffffffu, w);
      }
      if (ok && part >= 0) {
        // one part of a split unit: unnormalised O, m and l for the merge
        tc_fence_after();
        float* pb = wk.partial + (static_cast<int64_t>(su * wk.split + part) * 2 + t) * PART_FLOATS;
#pragma unroll 1
        for (int c = 0; c < HD; c += 32) {
          uint32_t o[32];
          tmem_ld32(o_col + c, o);
          tmem_wait_ld();
          float4* dst = reinterpret_cast<float4*>(pb + r * HD + c);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(__uint_as_float(o[4 * k]), __uint_as_float(o[4 * k + 1]),
                                 __uint_as_float(o[4 * k + 2]), __uint_as_float(o[4 * k + 3]));
        }
        *reinterpret_cast<float2*>(pb + BQ * HD + 2 * r) = make_float2(m, l);
      } else if (ok) {
        tc_fence_after();
        {
          bool w = mbar_wait(&tl->g_full, 0, abort_flag, status, WHERE_ANCHOR);
          ok = __all_sync(0xffffffffu, w);
        }
        const int row_t = q0 + t * BQ + r;
        const float inv = 1.0f / l;
        const bool row_ok = row_t < N;
        const int64_t row = static_cast<int64_t>(b) * N + row_t;
#pragma unroll 1
        for (int c = 0; c < HD && ok; c += 32) {
          uint32_t o[32];
          tmem_ld32(o_col + c, o);
          tmem_wait_ld();
          if (!row_ok) continue;
          // row r of this tile's gate, 128-byte swizzle: chunk j of the row at j ^ (r & 7)
          const uint8_t* grow = smem + Q_OFF + (2 * t + (c >> 6)) * BOX + r * 128;
          __nv_bfloat16* op = out + row * ldo + h * HD + c;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int chunk = ((c & 63) >> 3) + k;
            const uint4 gv = *reinterpret_cast<const uint4*>(grow + ((chunk ^ (r & 7)) << 4));
            const float gg[8] = {bf16lo_to_f32(gv.x), bf16hi_to_f32(gv.x), bf16lo_to_f32(gv.y),
                                 bf16hi_to_f32(gv.y), bf16lo_to_f32(gv.z), bf16hi_to_f32(gv.z),
                                 bf16lo_to_f32(gv.w), bf16hi_to_f32(gv.w)};
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              y[e] = __uint_as_float(o[8 * k + e]) * inv * fast_sigmoid(gg[e]);
            if (residual != nullptr) {
              const uint4 rv =
                  *reinterpret_cast<const uint4*>(residual + row * ldr + h * HD + c + 8 * k);
              y[0] += bf16lo_to_f32(rv.x); y[1] += bf16hi_to_f32(rv.x);
              y[2] += bf16lo_to_f32(rv.y); y[3] += bf16hi_to_f32(rv.y);
              y[4] += bf16lo_to_f32(rv.z); y[5] += bf16hi_to_f32(rv.z);
              y[6] += bf16lo_to_f32(rv.w); y[7] += bf16hi_to_f32(rv.w);
            }
            uint4 ov;
            ov.x = pack_bf16x2(y[0], y[1]);
            ov.y = pack_bf16x2(y[2], y[3]);
            ov.z = pack_bf16x2(y[4], y[5]);
            ov.w = pack_bf16x2(y[6], y[7]);
            *reinterpret_cast<uint4*>(op + 8 * k) = ov;
          }
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

// Combines the parts of the split units: with M = max_p m_p and w_p =
// 2^(m_p - M), O = sum_p w_p O_p and l = sum_p w_p l_p (each part's O and l
// are relative to its own running max), then Y = O / l * sigmoid(G)
// (+ residual). One warp per query row, four columns per lane.
__global__ void __launch_bounds__(256) anchor_merge_kernel(AnchorWork wk, int N,
                                                           const __nv_bfloat16* gate, int64_t ldg,
                                                           const __nv_bfloat16* residual,
                                                           int64_t ldr, __nv_bfloat16* out,
                                                           int64_t ldo) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<int64_t>(wk.n_split_units) * 2 * BQ) return;
  const int su = static_cast<int>(wid / (2 * BQ));
  const int t = static_cast<int>((wid / BQ) & 1), r = static_cast<int>(wid % BQ);
  const int unit = wk.n_full + su;
  const int q0 = (unit % wk.n_qunits) * 2 * BQ;
  const int h = (unit / wk.n_qunits) % wk.H, b = unit / (wk.n_qunits * wk.H);
  const int row_t = q0 + t * BQ + r;
  if (row_t >= N) return;
  float mx = -INFINITY;
  for (int p = 0; p < wk.split; ++p) {
    const float* pb = wk.partial + (static_cast<int64_t>(su * wk.split + p) * 2 + t) * PART_FLOATS;
    mx = fmaxf(mx, pb[BQ * HD + 2 * r]);
  }
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, l = 0.f;
  for (int p = 0; p < wk.split; ++p) {
    const float* pb = wk.partial + (static_cast<int64_t>(su * wk.split + p) * 2 + t) * PART_FLOATS;
    const float2 ml = *reinterpret_cast<const float2*>(pb + BQ * HD + 2 * r);
    const float w = ml.x == -INFINITY ? 0.f : exp2f(ml.x - mx);
    const float4 o = *reinterpret_cast<const float4*>(pb + r * HD + 4 * lane);
    acc[0] = fmaf(w, o.x, acc[0]);
    acc[1] = fmaf(w, o.y, acc[1]);
    acc[2] = fmaf(w, o.z, acc[2]);
    acc[3] = fmaf(w, o.w, acc[3]);
    l = fmaf(w, ml.y, l);
  }
  const float inv = 1.0f / l;
  const int64_t row = static_cast<int64_t>(b) * N + row_t;
  const int col = h * HD + 4 * lane;
  const uint2 gv = *reinterpret_cast<const uint2*>(gate + row * ldg + col);
  const float gg[4] = {bf16lo_to_f32(gv.x), bf16hi_to_f32(gv.x), bf16lo_to_f32(gv.y),
                       bf16hi_to_f32(gv.y)};
  float y[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) y[e] = acc[e] * inv * fast_sigmoid(gg[e]);
  if (residual != nullptr) {
    const uint2 rv = *reinterpret_cast<const uint2*>(residual + row * ldr + col);
    y[0] += bf16lo_to_f32(rv.x); y[1] += bf16hi_to_f32(rv.x);
    y[2] += bf16lo_to_f32(rv.y); y[3] += bf16hi_to_f32(rv.y);
  }
  *reinterpret_cast<uint2*>(out + row * ldo + col) =
      make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
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

AnchorPlan anchor_plan(int B, int N, int H, int n_keys) {
  AnchorPlan p;
  const int Nk = n_keys > 0 ? n_keys : N;
  p.n_qunits = (N + 2 * BQ - 1) / (2 * BQ);
  p.nkv_total = (Nk + BKV - 1) / BKV;
  const int64_t units = static_cast<int64_t>(p.n_qunits) * H * B;
  const int sms = std::max(1, device_sm_count());  // one anchor CTA per SM
  const int tail = static_cast<int>(units % sms);
  p.n_full = static_cast<int>(units);
  // The last wave's `tail` units, split s ways along the keys, take about
  // ceil(tail * s / sms) / s of a whole unit's time. Take the best s <= 4 (and
  // <= the key blocks) when it saves at least a fifth of that wave.
  int best_s = 1;
  double best_t = 1.0;
  for (int sp = 2; sp <= std::min(4, p.nkv_total); ++sp) {
    const double t = static_cast<double>((tail * sp + sms - 1) / sms) / sp;
    if (t < best_t - 1e-9) {
      best_t = t;
      best_s = sp;
    }
  }
  if (tail > 0 && best_s > 1 && best_t <= 0.8) {
    p.split = best_s;
    p.n_split_units = tail;
    p.n_full = static_cast<int>(units - tail);
  }
  p.partial_bytes = static_cast<size_t>(p.n_split_units) * p.split * 2 * PART_FLOATS * sizeof(float);
  return p;
}

cudaError_t anchor_bf16(const sva_attn_args& a, int* status, void* scratch, cudaStream_t s,
                        Prof* prof) {
  const int D = a.H * a.d;
  CUtensorMap mq, mk, mv;
  const int Nk = a.n_keys > 0 ? a.n_keys : a.N;
  CUtensorMap mg;
  if (!act_map(&mq, a.q, a.ldq, a.B, a.N, D) || !act_map(&mk, a.k, a.ldk, a.B, Nk, D) ||
      !act_map(&mv, a.v, a.ldv, a.B, Nk, D) || !act_map(&mg, a.gate, a.ldg, a.B, a.N, D))
    return cudaErrorInvalidValue;
  const AnchorPlan p = anchor_plan(a.B, a.N, a.H, a.n_keys);
  if (p.partial_bytes > 0 && scratch == nullptr) return cudaErrorInvalidValue;
  AnchorWork wk;
  wk.n_qunits = p.n_qunits;
  wk.H = a.H;
  wk.n_full = p.n_full;
  wk.n_split_units = p.n_split_units;
  wk.split = p.split > 0 ? p.split : 1;
  wk.nkv_total = p.nkv_total;
  wk.partial = static_cast<float*>(scratch);
  const float scale = a.scale != 0.f ? a.scale : 1.0f / sqrtf(static_cast<float>(a.d));
  const float scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e = cudaFuncSetAttribute(anchor_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kAnchorSmem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(p.n_full + p.n_split_units * p.split);
  const auto* gate = static_cast<const __nv_bfloat16*>(a.gate);
  const auto* res = static_cast<const __nv_bfloat16*>(a.residual);
  auto* out = static_cast<__nv_bfloat16*>(a.out);
  anchor_tc_kernel<<<grid, NUM_THREADS, kAnchorSmem, s>>>(mq, mk, mv, mg, a.N, Nk, scale_log2, wk, gate,
                                                          a.ldg, res, a.ldr, out, a.ldo, status);
  if ((e = cudaGetLastError()) != cudaSuccess || p.n_split_units == 0) return e;
  const int64_t threads = static_cast<int64_t>(p.n_split_units) * 2 * BQ * 32;
  anchor_merge_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(
      wk, a.N, gate, a.ldg, res, a.ldr, out, a.ldo);
  if (prof != nullptr) prof->extra_launch();
  return cudaGetLastError();
}

}  // namespace sva
