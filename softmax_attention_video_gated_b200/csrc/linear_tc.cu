// linear_tc.cu -- gated linear attention, bf16, d = 128, on tcgen05/TMEM.
//
// The layer keeps a fixed-size state per (batch, head) and costs O(N)
// [ai-papers.net summary, section "ハイブリッド線形アテンション"]. With phi = ReLU:
//   S = sum_t phi(K_t)^T V_t,  z = sum_t phi(K_t),
//   Y_t = phi(Q_t) S / (phi(Q_t) . z + eps) * sigmoid(G_t)   (+ residual).
// In the write-gated variant token t's terms of S and z carry the factor
// sigmoid(W_t), one logit per token and head (same section: the gate sets how
// much each token writes into the state).
//
// Two kernels, both HBM-bound (the roofline is 10 B*N*D bytes of Q, K, V, G
// and Y traffic per layer):
//  1. lin_state_tc:  one CTA per (token chunk, head, batch). TMA streams
//     128-token K and V tiles into a 3-stage ring; four warps apply ReLU in
//     shared memory and accumulate z; one thread issues tcgen05.mma with
//     A = phi(K)^T and B = V, both read MN-major straight from the TMA layout,
//     accumulating the 128x128 fp32 partial state of the chunk in TMEM, which
//     goes to global memory (66 KB per chunk, read back from L2).
//  2. lin_readout_tc: persistent over the same chunks as the state pass. Its
//     epilogue warps first sum the head's chunk partials in chunk order
//     (deterministic, the same in every CTA of the head) into the read-out
//     operand [S^T | z_hi | z_lo | 0], bf16 [144 x 128] in shared memory (z
//     split in two bf16 rows keeps it to ~16 bits), while the first Q and G
//     tiles land. Q and G tiles stream through a 2-stage TMA ring; one M=128,
//     N=144, K=128 MMA per tile gives the numerator (columns 0..127) and
//     denominator (columns 128, 129) together into one of two TMEM
//     accumulators; eight epilogue warps divide, apply the sigmoid gate and
//     residual, and write Y through per-warp TMA stores.
//  Summing the partials in the read-out instead of a separate kernel removes
//  one launch and one kernel boundary per layer. In both kernels the TMA and
//  MMA warps run their loops with all 32 lanes and lane 0 issues (720p layer
//  133.0 -> 131.1 us against single-lane loops with 31 lanes parked).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sva {
namespace {

constexpr int HD = 128;                 // head dim of these kernels
constexpr int TT = 128;                 // tokens per tile
constexpr int BOX_BYTES = TT * 128;     // one [64 cols x 128 rows] bf16 box = 16 KB
constexpr int STATE_ROWS = HD + 16;     // read-out B operand rows: S^T, z_hi, z_lo, zeros
constexpr int STATE_BOX_BYTES = STATE_ROWS * 128;

// ------------------------------------------------------------------ state
constexpr int ST_STAGES = 3;
constexpr int ST_STAGE_BYTES = 4 * BOX_BYTES;  // K (2 boxes) + V (2 boxes)

struct StateTail {
  uint64_t full[ST_STAGES];
  uint64_t relu_done[ST_STAGES];
  uint64_t empty[ST_STAGES];
  uint64_t s_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  float zbuf[8][HD];
};
constexpr size_t kStateSmem = 1024 + ST_STAGES * ST_STAGE_BYTES + sizeof(StateTail);

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  int never = 0;
  return mbar_wait(bar, parity, &never, nullptr, 0);
}

// kWriteGate: token t's row of phi(K) is scaled by omega_t = sigmoid(wgate[b, t, h])
// before it enters S and z (the write-gated variant); wgate is [B, N, >=H], row
// stride ldw.
template <bool kWriteGate>
__global__ void __launch_bounds__(192, 1)
    lin_state_tc_kernel(const __grid_constant__ CUtensorMap map_k,
                        const __grid_constant__ CUtensorMap map_v, int N, int H,
                        int tiles_per_chunk, int n_chunks, unsigned flags,
                        const __nv_bfloat16* __restrict__ wgate, int64_t ldw, float* partial,
                        int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  StateTail* tl = reinterpret_cast<StateTail*>(smem + ST_STAGES * ST_STAGE_BYTES);
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = warp_id(), lane = lane_id();
  const int tiles_total = (N + TT - 1) / TT;
  const int tile0 = c * tiles_per_chunk;
  const int ntiles = max(0, min(tiles_per_chunk, tiles_total - tile0));

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST_STAGES; ++s) {
      mbar_init(&tl->full[s], 1);
      mbar_init(&tl->relu_done[s], 128);
      mbar_init(&tl->empty[s], 1);
    }
    mbar_init(&tl->s_full, 1);
    mbar_init(&tl->drain, 1);
    tl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tl->tmem_base, HD);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_k);
    tma_prefetch_desc(&map_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tl->tmem_base;
  volatile int* abort_flag = &tl->abort_flag;

  if (warp == 0) {
    {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < ntiles; ++i) {
        const bool w = mbar_wait(&tl->empty[stage], phase ^ 1, abort_flag, status, WHERE_LIN_STATE);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* st = smem + stage * ST_STAGE_BYTES;
          const int t0 = (tile0 + i) * TT;
          mbar_arrive_expect_tx(&tl->full[stage], ST_STAGE_BYTES);
          tma_load_3d(&map_k, &tl->full[stage], st, h * HD, t0, b);
          tma_load_3d(&map_k, &tl->full[stage], st + BOX_BYTES, h * HD + 64, t0, b);
          tma_load_3d(&map_v, &tl->full[stage], st + 2 * BOX_BYTES, h * HD, t0, b);
          tma_load_3d(&map_v, &tl->full[stage], st + 3 * BOX_BYTES, h * HD + 64, t0, b);
        }
        __syncwarp();
        ++issued;
        if (++stage == ST_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok && lane == 0)
        for (int i = max(0, issued - ST_STAGES); i < issued; ++i)
          (void)drain_wait(&tl->full[i % ST_STAGES], (i / ST_STAGES) & 1);
      __syncwarp();
    }
  } else if (warp == 1) {
    {
      // A = phi(K)^T: M = d (MN-major, the 64-wide d atoms 16 KB apart),
      // B = V: N = d (MN-major), K = tokens (8-token groups 1024 B apart).
      constexpr uint32_t idesc = idesc_bf16_f32(HD, HD, true, true);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < ntiles; ++i) {
        const bool w = mbar_wait(&tl->relu_done[stage], phase, abort_flag, status, WHERE_LIN_STATE);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t kaddr = smem_u32(smem + stage * ST_STAGE_BYTES);
          const uint32_t vaddr = kaddr + 2 * BOX_BYTES;
#pragma unroll
          for (int kk = 0; kk < TT / 16; ++kk) {
            const uint64_t ad = smem_desc(kaddr + kk * 2048, BOX_BYTES, 1024);
            const uint64_t bd = smem_desc(vaddr + kk * 2048, BOX_BYTES, 1024);
            umma_ss(tmem, ad, bd, idesc, (i | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&tl->empty[stage]);
        }
        __syncwarp();
        if (++stage == ST_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (lane == 0) {
        if (ok) umma_commit(&tl->s_full);
        umma_commit(&tl->drain);
        (void)drain_wait(&tl->drain, 0);
      }
      __syncwarp();
    }
  } else {
    // ---------------------------------------- ReLU + z workers, then epilogue
    const int wt = threadIdx.x - 64;          // 0..127
    const int ch = wt & 15;                   // logical 16-byte chunk of a row (8 columns)
    const int rc = wt >> 4;                   // row class: rows rc, rc+8, ...
    const int box = ch >> 3, cl = ch & 7;
    const uint32_t col_off = box * BOX_BYTES + ((cl ^ rc) << 4);
    const bool features = (flags & SVA_FLAG_QK_FEATURES) != 0;
    float z[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) z[i] = 0.f;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    // Write gate: a warp's threads touch 32 rows of a tile (row classes rc,
    // rc + 1 and every 8th row after them); lane L fetches the logit of the
    // row (rc & ~1) + (L & 1) + 8 (L >> 1) one tile ahead and the others read
    // its sigmoid by shuffle, so each tile costs one load per lane.
    const int my_row = (rc & ~1) + (lane & 1) + 8 * (lane >> 1);
    auto load_logit = [&](int tile) -> float {
      const int t = tile * TT + my_row;
      return t < N ? __bfloat162float(wgate[(static_cast<int64_t>(b) * N + t) * ldw + h]) : 0.f;
    };
    float next_logit = 0.f;
    if constexpr (kWriteGate) {
      if (ntiles > 0) next_logit = load_logit(tile0);
    }
    for (int i = 0; i < ntiles; ++i) {
      float om_lane = 1.f;
      if constexpr (kWriteGate) {
        om_lane = 1.0f / (1.0f + __expf(-next_logit));
        if (i + 1 < ntiles) next_logit = load_logit(tile0 + i + 1);
      }
      bool w = mbar_wait(&tl->full[stage], phase, abort_flag, status, WHERE_LIN_STATE);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      uint8_t* kt = smem + stage * ST_STAGE_BYTES + col_off;
#pragma unroll 4
      for (int j = 0; j < TT / 8; ++j) {
        uint4* p = reinterpret_cast<uint4*>(kt + (rc + 8 * j) * 128);
        uint4 v = *p;
        if constexpr (kWriteGate) {
          // phi(K) * omega, rounded once to bf16: S and z see the same values
          const float o = __shfl_sync(0xffffffffu, om_lane, (rc & 1) + 2 * j);
          const uint32_t in[4] = {v.x, v.y, v.z, v.w};
          uint32_t r4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t f = features ? in[e] : relu_bf16x2(in[e]);
            r4[e] = pack_bf16x2(bf16lo_to_f32(f) * o, bf16hi_to_f32(f) * o);
          }
          v = make_uint4(r4[0], r4[1], r4[2], r4[3]);
          *p = v;
        } else if (!features) {
          v.x = relu_bf16x2(v.x);
          v.y = relu_bf16x2(v.y);
          v.z = relu_bf16x2(v.z);
          v.w = relu_bf16x2(v.w);
          *p = v;
        }
        z[0] += bf16lo_to_f32(v.x); z[1] += bf16hi_to_f32(v.x);
        z[2] += bf16lo_to_f32(v.y); z[3] += bf16hi_to_f32(v.y);
        z[4] += bf16lo_to_f32(v.z); z[5] += bf16hi_to_f32(v.z);
        z[6] += bf16lo_to_f32(v.w); z[7] += bf16hi_to_f32(v.w);
      }
      fence_proxy_async_smem();
      mbar_arrive(&tl->relu_done[stage]);
      if (++stage == ST_STAGES) {
        stage = 0;
        phase ^= 1;
      }
    }
    // z: reduce the 8 row classes
#pragma unroll
    for (int i = 0; i < 8; ++i) tl->zbuf[rc][ch * 8 + i] = z[i];
    named_barrier_sync(1, 128);
    float* out = partial + (static_cast<int64_t>(b * H + h) * n_chunks + c) * (HD * HD + HD);
    {
      float zs = 0.f;
#pragma unroll
      for (int r = 0; r < 8; ++r) zs += tl->zbuf[r][wt];
      out[HD * HD + wt] = zs;
    }
    // partial state rows: TMEM lane = d_k index, column = d_v index
    const int q = warp & 3;
    const int row = q * 32 + lane;
    bool have = ok && ntiles > 0;
    if (have) {
      bool w = mbar_wait(&tl->s_full, 0, abort_flag, status, WHERE_LIN_STATE);
      have = __all_sync(0xffffffffu, w);
    }
    if (have) {
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < HD; cc += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + cc, r);
        tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(out + row * HD + cc);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          dst[k] = make_float4(__uint_as_float(r[4 * k]), __uint_as_float(r[4 * k + 1]),
                               __uint_as_float(r[4 * k + 2]), __uint_as_float(r[4 * k + 3]));
      }
    } else if (ntiles == 0) {
      float4* dst = reinterpret_cast<float4*>(out + row * HD);
      for (int k = 0; k < HD / 4; ++k) dst[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, HD);
  }
}

// ------------------------------------------------------------------ state only
// fp32 state of one (batch, head), [S (d_k rows x d_v) | z]: the chunk partials
// summed in chunk order (the same order as the read-out's own sum)
__global__ void __launch_bounds__(256) lin_sum_chunks_kernel(const float* __restrict__ partial,
                                                             float* __restrict__ state,
                                                             int n_chunks) {
  const int elems = HD * HD + HD;
  const int64_t bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= elems) return;
  const float* p = partial + bh * n_chunks * elems + e;
  float acc = 0.f;
  for (int c = 0; c < n_chunks; ++c) acc += p[static_cast<int64_t>(c) * elems];
  state[bh * elems + e] = acc;
}

// ------------------------------------------------------------------ read-out
// Persistent over the state pass's chunks (one CTA per (token chunk, head,
// batch), one wave). The head's read-out operand [S^T | z_hi | z_lo | 0] is
// built once (build_state_operand); 128-token tiles of Q and G stream through
// a 2-stage TMA ring.
// One M=128, N=144, K=128 MMA per tile gives numerator (columns 0..127) and
// denominator (128, 129) into one of two TMEM accumulators, so the MMA of the
// next tile runs during this tile's epilogue. Eight epilogue warps: warp w
// owns TMEM lane quadrant w % 4 (32 rows) and one 64-column half; each thread
// applies ReLU to its half-row of Q when the producer has not, and finishes
// its half-row of Y (divide, sigmoid(G), residual) into its warp's staging
// slot, which the warp stores by TMA. No barrier spans more than one warp
// inside the tile loop; a warp waits for its own previous store only before
// it reuses its slot.
constexpr int RO_STAGES = 2;
constexpr int RO_STAGE_BYTES = 4 * BOX_BYTES;          // Q (2 boxes) + G (2 boxes)
constexpr int RO_G = 2 * BOX_BYTES;                    // G's offset in a stage
constexpr int RO_S_OFF = RO_STAGES * RO_STAGE_BYTES;   // the state operand: 2 x [64 x 144]
constexpr int RO_Y_OFF = RO_S_OFF + 2 * STATE_BOX_BYTES;
constexpr int RO_Y_SLOT = 32 * 128;                    // one warp's [64 x 32] bf16 slot
constexpr int RO_TAIL_OFF = RO_Y_OFF + 8 * RO_Y_SLOT;
constexpr int RO_THREADS = 320;                        // producer, MMA, 8 epilogue warps
struct ReadoutTail {
  uint64_t full[RO_STAGES];
  uint64_t relu_done[RO_STAGES];
  uint64_t empty[RO_STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t s_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kReadoutSmem = 1024 + RO_TAIL_OFF + sizeof(ReadoutTail);
constexpr int RO_TMEM_COLS = 512;                      // two 256-column accumulators

// The read-out operand of head (b, h), built by the 256 epilogue threads
// straight into shared memory: [S^T | z_hi | z_lo | 0] as bf16 [144 x 128],
// K-major in two [64-column x 144-row] boxes with the 128-byte swizzle the MMA
// descriptor expects (16-byte chunk c of row r at chunk c ^ (r & 7)). S and z
// are the sums of the n_chunks fp32 partial states in chunk order (the same
// order for every CTA of the head, so they all build the same operand). The
// partials (66 KB each) are read from L2 with float4 loads: thread t sums
// columns n = 4 (t % 32) .. +3 of S (rows of S^T) over k in two 8-wide groups
// (t / 32 and t / 32 + 8).
__device__ __forceinline__ void build_state_operand(const float* __restrict__ part, int n_chunks,
                                                    uint8_t* op, int et) {
  constexpr int ELEMS = HD * HD + HD;
  const int nq = et & 31, kset = et >> 5;
  float acc[2][8][4];
#pragma unroll
  for (int g = 0; g < 2; ++g)
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[g][i][e] = 0.f;
#pragma unroll 1
  for (int c = 0; c < n_chunks; ++c) {
    const float* pc = part + static_cast<int64_t>(c) * ELEMS + 4 * nq;
    float4 v[2][8];
#pragma unroll
    for (int g = 0; g < 2; ++g)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        v[g][i] = *reinterpret_cast<const float4*>(pc + (8 * (kset + 8 * g) + i) * HD);
#pragma unroll
    for (int g = 0; g < 2; ++g)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[g][i][0] += v[g][i].x;
        acc[g][i][1] += v[g][i].y;
        acc[g][i][2] += v[g][i].z;
        acc[g][i][3] += v[g][i].w;
      }
  }
  // row n of S^T, k-group kg: 8 bf16 = one 16-byte chunk
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const int kg = kset + 8 * g;  // k = 8 kg .. 8 kg + 7
    uint8_t* box = op + (kg >> 3) * STATE_BOX_BYTES;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int n = 4 * nq + e;
      uint4 o;
      o.x = pack_bf16x2(acc[g][0][e], acc[g][1][e]);
      o.y = pack_bf16x2(acc[g][2][e], acc[g][3][e]);
      o.z = pack_bf16x2(acc[g][4][e], acc[g][5][e]);
      o.w = pack_bf16x2(acc[g][6][e], acc[g][7][e]);
      *reinterpret_cast<uint4*>(box + n * 128 + (((kg & 7) ^ (n & 7)) << 4)) = o;
    }
  }
  // rows 128, 129: z split into a bf16 head and its bf16 remainder; rows 130..143: 0
  if (et < 16) {
    const int kg = et;
    float z[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) z[i] = 0.f;
#pragma unroll 1
    for (int c = 0; c < n_chunks; ++c) {
      const float4* pz =
          reinterpret_cast<const float4*>(part + static_cast<int64_t>(c) * ELEMS + HD * HD + 8 * kg);
      const float4 a = pz[0], b = pz[1];
      z[0] += a.x; z[1] += a.y; z[2] += a.z; z[3] += a.w;
      z[4] += b.x; z[5] += b.y; z[6] += b.z; z[7] += b.w;
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hi[i] = pack_bf16x2(z[2 * i], z[2 * i + 1]);
      lo[i] = pack_bf16x2(z[2 * i] - bf16lo_to_f32(hi[i]), z[2 * i + 1] - bf16hi_to_f32(hi[i]));
    }
    uint8_t* box = op + (kg >> 3) * STATE_BOX_BYTES;
    *reinterpret_cast<uint4*>(box + HD * 128 + (((kg & 7) ^ (HD & 7)) << 4)) =
        make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(box + (HD + 1) * 128 + (((kg & 7) ^ ((HD + 1) & 7)) << 4)) =
        make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  for (int i = et; i < 2 * (STATE_ROWS - HD - 2) * 8; i += 256) {
    const int bx = i / ((STATE_ROWS - HD - 2) * 8), rem = i % ((STATE_ROWS - HD - 2) * 8);
    const int r = HD + 2 + rem / 8, ch = rem % 8;
    *reinterpret_cast<uint4*>(op + bx * STATE_BOX_BYTES + r * 128 + (ch << 4)) =
        make_uint4(0u, 0u, 0u, 0u);
  }
}

__global__ void __launch_bounds__(RO_THREADS, 1)
    lin_readout_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                          const __grid_constant__ CUtensorMap map_g,
                          const __grid_constant__ CUtensorMap map_o,
                          const float* __restrict__ partial, int n_chunks, int N, int H,
                          int tiles_per_chunk, float eps, unsigned flags,
                          const __nv_bfloat16* residual, int64_t ldr, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  ReadoutTail* tl = reinterpret_cast<ReadoutTail*>(smem + RO_TAIL_OFF);
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = warp_id(), lane = lane_id();
  const int tiles_total = (N + TT - 1) / TT;
  const int tile0 = c * tiles_per_chunk;
  const int ntiles = max(0, min(tiles_per_chunk, tiles_total - tile0));
  const bool features = (flags & SVA_FLAG_QK_FEATURES) != 0;

  if (threadIdx.x == 0) {
    for (int st = 0; st < RO_STAGES; ++st) {
      mbar_init(&tl->full[st], 1);
      mbar_init(&tl->relu_done[st], 256);
      mbar_init(&tl->empty[st], 8);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tl->acc_full[a], 1);
      mbar_init(&tl->acc_empty[a], 8);
    }
    mbar_init(&tl->s_full, 8);  // one arrival per epilogue warp once the operand is built
    mbar_init(&tl->drain, 1);
    tl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tl->tmem_base, RO_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tl->tmem_base;
  volatile int* abort_flag = &tl->abort_flag;

  if (warp == 0) {
    if (ntiles > 0) {
      // ------------------------------------------------ TMA producer (all lanes iterate)
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < ntiles; ++i) {
        const bool w =
            mbar_wait(&tl->empty[stage], phase ^ 1, abort_flag, status, WHERE_LIN_READOUT);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* sb = smem + stage * RO_STAGE_BYTES;
          const int t0 = (tile0 + i) * TT;
          mbar_arrive_expect_tx(&tl->full[stage], RO_STAGE_BYTES);
          tma_load_3d(&map_q, &tl->full[stage], sb, h * HD, t0, b);
          tma_load_3d(&map_q, &tl->full[stage], sb + BOX_BYTES, h * HD + 64, t0, b);
          tma_load_3d(&map_g, &tl->full[stage], sb + RO_G, h * HD, t0, b);
          tma_load_3d(&map_g, &tl->full[stage], sb + RO_G + BOX_BYTES, h * HD + 64, t0, b);
        }
        __syncwarp();
        ++issued;
        if (++stage == RO_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok && lane == 0)
        for (int i = max(0, issued - RO_STAGES); i < issued; ++i)
          (void)drain_wait(&tl->full[i % RO_STAGES], (i / RO_STAGES) & 1);
      __syncwarp();
    }
  } else if (warp == 1) {
    if (ntiles > 0) {
      // ------------------------------------------------ MMA issuer (all lanes iterate)
      constexpr uint32_t idesc = idesc_bf16_f32(128, STATE_ROWS, false, false);
      bool ok = __all_sync(0xffffffffu, mbar_wait(&tl->s_full, 0, abort_flag, status,
                                                  WHERE_LIN_READOUT));
      const uint32_t saddr = smem_u32(smem + RO_S_OFF);
      int stage = 0;
      uint32_t phase = 0;
      for (int i = 0; i < ntiles && ok; ++i) {
        const int acc = i & 1;
        const uint32_t acc_phase = (i >> 1) & 1;
        // Q is ready once loaded (features) or once the epilogue applied ReLU
        uint64_t* ready = features ? &tl->full[stage] : &tl->relu_done[stage];
        const bool w = mbar_wait(ready, phase, abort_flag, status, WHERE_LIN_READOUT) &&
                       mbar_wait(&tl->acc_empty[acc], acc_phase ^ 1, abort_flag, status,
                                 WHERE_LIN_READOUT);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t qaddr = smem_u32(smem + stage * RO_STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const int bx = kk >> 2, wk = kk & 3;
            const uint64_t ad = smem_desc(qaddr + bx * BOX_BYTES + wk * 32, 16, 1024);
            const uint64_t bd = smem_desc(saddr + bx * STATE_BOX_BYTES + wk * 32, 16, 1024);
            umma_ss(tmem + acc * 256, ad, bd, idesc, kk != 0 ? 1u : 0u);
          }
          umma_commit(&tl->acc_full[acc]);
        }
        __syncwarp();
        if (++stage == RO_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (lane == 0) {
        umma_commit(&tl->drain);
        (void)drain_wait(&tl->drain, 0);
      }
      __syncwarp();
    }
  } else if (ntiles > 0) {
    // ------------------------------------------------ epilogue: half a row per thread
    const int ew = warp - 2;                 // epilogue warp 0..7
    const int wq = warp & 3;                 // TMEM lane quadrant of this warp
    const int half = ew >> 2;                // 64-column half of the tile
    const int r = wq * 32 + lane;            // row of the tile
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    uint8_t* yslot = smem + RO_Y_OFF + ew * RO_Y_SLOT;
    // the head's read-out operand, while the producer's first Q and G tiles land
    build_state_operand(partial + static_cast<int64_t>(b * H + h) * n_chunks * (HD * HD + HD),
                        n_chunks, smem + RO_S_OFF, threadIdx.x - 64);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&tl->s_full);
    // ReLU on this thread's half-row of Q in tile k (its stage), then report it
    auto relu_tile = [&](int k) -> bool {
      const int st = k % RO_STAGES;
      const bool w = mbar_wait(&tl->full[st], (k / RO_STAGES) & 1, abort_flag, status,
                               WHERE_LIN_READOUT);
      if (!__all_sync(0xffffffffu, w)) return false;
      uint8_t* qrow = smem + st * RO_STAGE_BYTES + half * BOX_BYTES + r * 128;
#pragma unroll
      for (int cl = 0; cl < 8; ++cl) {
        uint4* p = reinterpret_cast<uint4*>(qrow + ((cl ^ (r & 7)) << 4));
        uint4 v = *p;
        v.x = relu_bf16x2(v.x);
        v.y = relu_bf16x2(v.y);
        v.z = relu_bf16x2(v.z);
        v.w = relu_bf16x2(v.w);
        *p = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(&tl->relu_done[st]);
      return true;
    };
    bool ok = features || relu_tile(0);
    for (int i = 0; i < ntiles && ok; ++i) {
      const int st = i % RO_STAGES, acc = i & 1;
      const uint32_t phase = (i / RO_STAGES) & 1, acc_phase = (i >> 1) & 1;
      const int t0 = (tile0 + i) * TT;
      {
        bool w = mbar_wait(&tl->full[st], phase, abort_flag, status, WHERE_LIN_READOUT);
        w = w && mbar_wait(&tl->acc_full[acc], acc_phase, abort_flag, status, WHERE_LIN_READOUT);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
      }
      tc_fence_after();
      const uint32_t trow = tmem + lane_base + acc * 256;
      uint32_t dd[16], num0[32], num1[32];
      tmem_ld16(trow + HD, dd);
      tmem_ld32(trow + half * 64, num0);
      tmem_ld32(trow + half * 64 + 32, num1);
      tmem_wait_ld();
      // the accumulator is read: hand it back to the MMA
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->acc_empty[acc]);
      const float inv = 1.0f / (__uint_as_float(dd[0]) + __uint_as_float(dd[1]) + eps);
      // this warp's previous store has read its slot before the slot is rewritten
      if (lane == 0) tma_store_wait_read0();
      __syncwarp();
      const int t = t0 + r;
      const __nv_bfloat16* res =
          (residual != nullptr && t < N)
              ? residual + (static_cast<int64_t>(b) * N + t) * ldr + h * HD + half * 64
              : nullptr;
      const uint8_t* grow = smem + st * RO_STAGE_BYTES + RO_G + half * BOX_BYTES + r * 128;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint4 gv = *reinterpret_cast<const uint4*>(grow + ((k ^ (r & 7)) << 4));
        const float gg[8] = {bf16lo_to_f32(gv.x), bf16hi_to_f32(gv.x), bf16lo_to_f32(gv.y),
                             bf16hi_to_f32(gv.y), bf16lo_to_f32(gv.z), bf16hi_to_f32(gv.z),
                             bf16lo_to_f32(gv.w), bf16hi_to_f32(gv.w)};
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          y[e] = __uint_as_float(k < 4 ? num0[8 * k + e] : num1[8 * (k - 4) + e]) * inv *
                 fast_sigmoid(gg[e]);
        if (res != nullptr) {
          const uint4 rv = *reinterpret_cast<const uint4*>(res + 8 * k);
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
        *reinterpret_cast<uint4*>(yslot + lane * 128 + ((k ^ (lane & 7)) << 4)) = o;
      }
      // G of this stage is read: release it (the MMA finished with Q at acc_full)
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->empty[st]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && t0 + wq * 32 < N) {
        tma_store_3d(&map_o, yslot, h * HD + half * 64, t0 + wq * 32, b);
        tma_store_commit();
      }
      // the next tile's ReLU after this epilogue: its load was issued when the
      // previous epilogue released the stage, so it has had this epilogue to land
      if (!features && i + 1 < ntiles && !relu_tile(i + 1)) {
        ok = false;
        break;
      }
    }
    // the slot stays valid until this warp's last store has read it
    if (lane == 0) tma_store_wait_read0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, RO_TMEM_COLS);
  }
}

bool act_map(CUtensorMap* m, const void* base, int64_t ld, int B, int N, int D) {
  const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(N),
                            static_cast<uint64_t>(B)};
  const uint64_t strides[2] = {static_cast<uint64_t>(ld) * 2,
                               static_cast<uint64_t>(ld) * 2 * static_cast<uint64_t>(N)};
  const uint32_t box[3] = {64, TT, 1};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

LinearPlan linear_plan(int B, int N, int H, int d, sva_dtype_t dt) {
  LinearPlan p;
  const int64_t work = static_cast<int64_t>(B) * H;
  const int sms = std::max(1, device_sm_count());
  if (dt == SVA_BF16) {
    // one wave: the fewest tiles per chunk with work * n_chunks <= #SMs
    const int tiles = (N + TT - 1) / TT;
    int ct = 1;
    while (ct < tiles && work * ((tiles + ct - 1) / ct) > sms) ++ct;
    p.tiles_per_chunk = ct;
    p.n_chunks = (tiles + ct - 1) / ct;
  } else {
    const int tokens = 256;
    p.tiles_per_chunk = tokens;
    p.n_chunks = (N + tokens - 1) / tokens;
  }
  const size_t elems = static_cast<size_t>(d) * d + d;
  p.partial_off = 0;
  p.state_off = align_up(p.partial_off + static_cast<size_t>(p.n_chunks) * work * elems * 4, 1024);
  // bf16: the read-out builds its operand in shared memory; fp32: the reduced state
  const size_t state_bytes = dt == SVA_BF16 ? 0 : static_cast<size_t>(work) * elems * 4;
  p.total = align_up(p.state_off + state_bytes, 1024);
  return p;
}

cudaError_t linear_bf16(const sva_attn_args& a, int* status, void* scratch, cudaStream_t s,
                        Prof* prof, float* state_out, const float* state_in) {
  const LinearPlan p = linear_plan(a.B, a.N, a.H, a.d, SVA_BF16);
  char* base = static_cast<char*>(scratch);
  float* partial = reinterpret_cast<float*>(base + p.partial_off);
  const int D = a.H * a.d;
  cudaError_t e;
  if (state_in == nullptr) {
    // ------------------------------------------------ state pass (K, V of these tokens)
    CUtensorMap mk, mv;
    if (!act_map(&mk, a.k, a.ldk, a.B, a.N, D) || !act_map(&mv, a.v, a.ldv, a.B, a.N, D))
      return cudaErrorInvalidValue;
    {
      ProfScope ps(prof, s, SVA_KERNEL_LINEAR_STATE);
      const bool wg = a.wgate != nullptr;
      auto kern = wg ? lin_state_tc_kernel<true> : lin_state_tc_kernel<false>;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kStateSmem));
      if (e != cudaSuccess) return e;
      dim3 grid(p.n_chunks, a.H, a.B);
      kern<<<grid, 192, kStateSmem, s>>>(mk, mv, a.N, a.H, p.tiles_per_chunk, p.n_chunks,
                                         a.flags, static_cast<const __nv_bfloat16*>(a.wgate),
                                         a.ldw, partial, status);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (state_out != nullptr) {
      // state only: the fp32 state, for the caller to sum over token shards
      ProfScope ps(prof, s, SVA_KERNEL_LINEAR_REDUCE);
      lin_sum_chunks_kernel<<<dim3((HD * HD + HD + 255) / 256, a.B * a.H), 256, 0, s>>>(
          partial, state_out, p.n_chunks);
      return cudaGetLastError();
    }
  }
  // ------------------------------------------------ read-out (Q, G, Y of these tokens)
  // Each read-out CTA sums its head's partial states itself (or takes a given
  // fp32 state, as one chunk) into the bf16 read-out operand in shared memory.
  const float* parts = state_in != nullptr ? state_in : partial;
  const int n_parts = state_in != nullptr ? 1 : p.n_chunks;
  CUtensorMap mq, mg, mo;
  if (!act_map(&mq, a.q, a.ldq, a.B, a.N, D) || !act_map(&mg, a.gate, a.ldg, a.B, a.N, D))
    return cudaErrorInvalidValue;
  {
    // Y: one [64 x 32] box per epilogue warp
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.N),
                              static_cast<uint64_t>(a.B)};
    const uint64_t strides[2] = {static_cast<uint64_t>(a.ldo) * 2,
                                 static_cast<uint64_t>(a.ldo) * 2 * static_cast<uint64_t>(a.N)};
    const uint32_t box[3] = {64, 32, 1};
    if (!encode_tmap(&mo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.out, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  ProfScope ps(prof, s, SVA_KERNEL_LINEAR_READOUT);
  e = cudaFuncSetAttribute(lin_readout_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kReadoutSmem));
  if (e != cudaSuccess) return e;
  lin_readout_tc_kernel<<<dim3(p.n_chunks, a.H, a.B), RO_THREADS, kReadoutSmem, s>>>(
      mq, mg, mo, parts, n_parts, a.N, a.H, p.tiles_per_chunk, a.eps, a.flags,
      static_cast<const __nv_bfloat16*>(a.residual), a.ldr, status);
  return cudaGetLastError();
}

}  // namespace sva
