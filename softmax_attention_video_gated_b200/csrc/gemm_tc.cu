// gemm_tc.cu -- bf16 projections of a mixer layer on the 5th-generation tensor
// cores: C = A B^T with A [M, K] (activations) and B [N, K] (weights in the
// [out, in] layout of a linear layer), both K-major, fp32 accumulation in TMEM.
//
// Persistent kernel on clusters of two CTAs (one CTA per SM). A cluster owns
// 256 x 256 output tiles; the pair shares each tcgen05.mma (cta_group::2):
// CTA r loads rows [128r, 128r+128) of the A tile and rows [128r, 128r+128) of
// the B tile (its half of N), so a 128-deep k-block costs each CTA 64 KB of
// shared memory instead of the 96 KB a single-CTA 128 x 256 tile needs. Per CTA:
//   warp 0      TMA producer: 128-row A and B boxes of 64 columns (128-byte
//               swizzle) into a ring of k-blocks; completion is counted on the
//               rank-0 CTA's barrier, which expects both CTAs' bytes;
//   warp 1      allocates 512 TMEM columns (pair allocation); on rank 0 one
//               lane issues M=256 N=256 K=16 MMAs into one of two 256-column
//               accumulators and multicasts its commits to both CTAs;
//   warps 2..5  epilogue of this CTA's 128 rows: tcgen05.ld, then either a bf16
//               store (ReLU on leading columns, the feature map phi of the
//               linear layers) through a swizzled slot and a TMA store per
//               32 x 32 chunk, or the residual update h += C (fp32) with an
//               optional bf16 copy of h. The main loop's TMA writes and MMA
//               operand reads already take about 128 bytes per clock of shared
//               memory, so the epilogues keep their own shared-memory traffic
//               low. Each warp releases the accumulator on rank 0's barrier.
// A k-block is 128 deep (two boxes per operand) in a 3-stage ring. Every
// k-block costs the MMA thread one barrier wait and one commit, and those
// stall its queue of MMAs, so 8 MMAs per k-block run faster than 4: the 720p
// QKVG projection takes 0.91 ms instead of 0.96 ms with 64-deep k-blocks. The
// residual epilogue moves h in 16-column chunks (6 KB of slots per warp) so
// that three 64 KB stages fit beside it (0.297 against 0.302 ms at 720p with
// 32-column chunks and five 32 KB stages).
// Tiles run in groups of whole M-tile columns so one wave touches few A rows
// and few B rows and both stay in L2 (the residual GEMM, with only a few N
// tiles, runs all N tiles of a few M tiles per wave and keeps its weight in L2
// with an evict-last hint, since the h stream passes through L2 beside it). A ragged last N tile issues MMAs only as
// wide as its columns (rounded up to 32), and the output columns from n_split
// on may come from a second weight (the write-gate projection appended to the
// fused [Q | K | V | G] projection, so the layer input is read once).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sva {
namespace {

constexpr int BM = 256, BN = 256, MAX_STAGES = 3;
constexpr int HALF = 128;                          // rows of A (and of B) per CTA
constexpr int KBOX = HALF * 64 * 2;                // one 128 x 64 bf16 box: 16 KB
constexpr int TMEM_COLS = 2 * BN;                  // two fp32 accumulators
constexpr int NUM_THREADS = 192;
// EPI_STORE epilogue: per warp two slots of a 32 x 32 bf16 chunk (64-byte swizzle)
constexpr int STO_SLOT_BYTES = 32 * 32 * 2;
constexpr int STO_WARP_BYTES = 2 * STO_SLOT_BYTES;
// EPI_RESIDUAL epilogue: per warp two slots of a 32-row x 16-column fp32 chunk
// of h (64-byte swizzle) and two of its bf16 copy (32-byte swizzle)
constexpr int RES_COLS = 16;                       // columns of h per chunk
constexpr int RES_H_BYTES = 32 * RES_COLS * 4, RES_C_BYTES = 32 * RES_COLS * 2;
constexpr int RES_WARP_BYTES = 2 * RES_H_BYTES + 2 * RES_C_BYTES;  // 6 KB

template <int EPI>
struct Layout {
  static constexpr int BK = 128;                              // k-block depth
  static constexpr int STAGES = 3;
  static constexpr int A_STAGE = HALF * BK * 2;                // 32 KB
  static constexpr int STAGE_BYTES = 2 * A_STAGE;              // A and B, per CTA
  static constexpr int EPI_OFF = STAGES * STAGE_BYTES;
  static_assert(STAGES <= MAX_STAGES, "barrier arrays hold every stage");
  static constexpr int TAIL_OFF = EPI_OFF + 4 * (EPI == EPI_STORE ? STO_WARP_BYTES : RES_WARP_BYTES);
};

struct GemmTail {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t hbar[4][2];  // EPI_RESIDUAL: h chunk loads, per epilogue warp and slot
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int EPI>
constexpr size_t gemm_smem() {
  return 1024 + Layout<EPI>::TAIL_OFF + sizeof(GemmTail);
}

// bulk stores: wait until at most one committed group still reads shared memory
__device__ __forceinline__ void tma_store_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  int never = 0;
  return mbar_wait(bar, parity, &never, nullptr, 0);
}

// MMA width of an N tile: the full BN, or for the ragged last tile its width
// rounded up to 32 (a legal N for M = 256 on a CTA pair), so a narrow tail
// costs tensor-core time in proportion to its width
__device__ __forceinline__ int tile_n_mma(int64_t N, int64_t n0) {
  const int64_t rem = N - n0;
  return rem >= BN ? BN : static_cast<int>((rem + 31) / 32 * 32);
}

__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int group,
                                            int& m_blk, int& n_blk) {
  const int per_group = group * n_tiles;
  const int g = tile / per_group, w = tile % per_group;
  const int m0 = g * group;
  const int gs = min(group, m_tiles - m0);
  m_blk = m0 + w % gs;
  n_blk = w / gs;
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap map_a,
                        const __grid_constant__ CUtensorMap map_b,
                        const __grid_constant__ CUtensorMap map_b2,
                        const __grid_constant__ CUtensorMap map_h,
                        const __grid_constant__ CUtensorMap map_c, GemmArgs g, int group) {
  constexpr int STAGES = Layout<EPI>::STAGES, BK = Layout<EPI>::BK;
  constexpr int A_STAGE = Layout<EPI>::A_STAGE, B_STAGE = A_STAGE;
  constexpr int STAGE_BYTES = Layout<EPI>::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE;
  GemmTail* tl = reinterpret_cast<GemmTail*>(smem + Layout<EPI>::TAIL_OFF);

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
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
      mbar_init(&tl->acc_empty[a], 8);  // 4 epilogue warps in each CTA of the pair
    }
    for (int w = 0; w < 4; ++w)
      for (int sl = 0; sl < 2; ++sl) mbar_init(&tl->hbar[w][sl], 1);
    mbar_init(&tl->drain, 1);
    tl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&tl->tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
    if (g.b2 != nullptr) tma_prefetch_desc(&map_b2);
    if (EPI == EPI_RESIDUAL) tma_prefetch_desc(&map_h);
    tma_prefetch_desc(&map_c);
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem_base = tl->tmem_base;
  volatile int* abort_flag = &tl->abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += n_clusters) {
        int m_blk, n_blk;
        tile_coords(tile, m_tiles, n_tiles, group, m_blk, n_blk);
        // each CTA of the pair holds half of the tile's MMA width of B rows
        const int64_t n0 = static_cast<int64_t>(n_blk) * BN;
        const bool second = g.b2 != nullptr && n0 >= g.n_split;
        const CUtensorMap* mb = second ? &map_b2 : &map_b;
        const int b_row = static_cast<int>(second ? n0 - g.n_split : n0) +
                          static_cast<int>(rank) * (tile_n_mma(g.N, n0) / 2);
        const uint64_t wpol = policy_evict_last();
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&tl->empty[stage], phase ^ 1, abort_flag, g.status, WHERE_GEMM)) {
            ok = false;
            break;
          }
          const uint32_t full0 = cluster_map(&tl->full[stage], 0);
          if (rank == 0) mbar_arrive_expect_tx(&tl->full[stage], 2 * STAGE_BYTES);
#pragma unroll
          for (int bx = 0; bx < BK / 64; ++bx) {
            tma_load_2d_pair(&map_a, full0, sA + stage * A_STAGE + bx * KBOX, kb * BK + 64 * bx,
                             m_blk * BM + rank * HALF);
            // the residual GEMM's weight (every wave reads all of it) is kept in
            // L2 ahead of the h stream: 473 -> 396 MB of DRAM reads, 266 -> 256 us
            if (EPI == EPI_RESIDUAL)
              tma_load_2d_pair_hint(mb, full0, sB + stage * B_STAGE + bx * KBOX, kb * BK + 64 * bx,
                                    b_row, wpol);
            else
              tma_load_2d_pair(mb, full0, sB + stage * B_STAGE + bx * KBOX, kb * BK + 64 * bx,
                               b_row);
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && rank == 0) {
        // abort: let the loads still in flight land before the CTA exits
        for (int64_t i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
          (void)drain_wait(&tl->full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1));
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------ MMA issuer (rank 0 only)
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += n_clusters, ++local) {
        int m_blk, n_blk;
        tile_coords(tile, m_tiles, n_tiles, group, m_blk, n_blk);
        const uint32_t idesc =
            idesc_bf16_f32(BM, tile_n_mma(g.N, static_cast<int64_t>(n_blk) * BN), false, false);
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
            const uint32_t off = static_cast<uint32_t>((kk >> 2) * KBOX + (kk & 3) * 32);
            const uint64_t ad = smem_desc(a_addr + off, 16, 1024);
            const uint64_t bd = smem_desc(b_addr + off, 16, 1024);
            umma_ss_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair(&tl->empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) umma_commit_pair(&tl->acc_full[acc], 0x3);
      }
      // every MMA issued above completes before TMEM is released
      umma_commit_pair(&tl->drain, 0x1);
      (void)drain_wait(&tl->drain, 0);
    }
  } else if (EPI == EPI_STORE) {
    // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
    // The thread owning a row packs 32 accumulator columns to bf16 (ReLU on the
    // leading relu_cols columns) into a 64-byte-swizzled slot, and one TMA
    // store per 32 x 32 chunk writes them out (TMA clips rows past M and
    // columns past N). Shared memory sees 2 KB written and 2 KB read per chunk.
    const int q = warp & 3;  // TMEM lane quadrant of this warp
    uint8_t* slots = smem + Layout<EPI>::EPI_OFF + q * STO_WARP_BYTES;
    const uint32_t acc_empty0[2] = {cluster_map(&tl->acc_empty[0], 0),
                                    cluster_map(&tl->acc_empty[1], 0)};
    int local = 0, sl = 0;
    for (int tile = cluster; tile < num_tiles; tile += n_clusters, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const bool w = mbar_wait(&tl->acc_full[acc], acc_phase, abort_flag, g.status, WHERE_GEMM);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
      int m_blk, n_blk;
      tile_coords(tile, m_tiles, n_tiles, group, m_blk, n_blk);
      const int64_t row0 = static_cast<int64_t>(m_blk) * BM + rank * HALF + q * 32;
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + cc, r);
        tmem_wait_ld();
        const int64_t col0 = static_cast<int64_t>(n_blk) * BN + cc;
        if (col0 >= g.N || row0 >= g.M) continue;  // warp-uniform
        // the store that used this slot two chunks ago has read it
        if (lane == 0) tma_store_wait_read1();
        __syncwarp();
        uint8_t* so = slots + sl * STO_SLOT_BYTES;
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          float a = __uint_as_float(r[2 * k]), bb = __uint_as_float(r[2 * k + 1]);
          if (col0 + 2 * k < g.relu_cols) a = relu_f(a);
          if (col0 + 2 * k + 1 < g.relu_cols) bb = relu_f(bb);
          pk[k] = pack_bf16x2(a, bb);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
          // 64-byte rows, 64-byte swizzle: chunk k of row r sits at k ^ ((r >> 1) & 3)
          *reinterpret_cast<uint4*>(so + lane * 64 + 16 * (k ^ ((lane >> 1) & 3))) =
              make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&map_c, so, static_cast<int>(col0), static_cast<int>(row0));
          tma_store_commit();
        }
        sl ^= 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0[acc]);
    }
    if (lane == 0) tma_store_wait0();
  } else {
    // ------------------------------------------------ residual epilogue (warps 2..5, both CTAs)
    // h += C for this warp's 32 rows, 16 columns at a time: TMA brings the h
    // chunk into a 64-byte-swizzled slot (prefetched two chunks ahead), the
    // thread owning a row adds its accumulator row in place (the swizzle keeps
    // the row-per-thread access free of bank conflicts), and TMA writes h and
    // its bf16 copy back.
    const int q = warp & 3;
    uint8_t* wbuf = smem + Layout<EPI>::EPI_OFF + q * RES_WARP_BYTES;
    uint64_t* hbar = tl->hbar[q];
    const uint32_t acc_empty0[2] = {cluster_map(&tl->acc_empty[0], 0),
                                    cluster_map(&tl->acc_empty[1], 0)};
    const bool copy = g.h_copy != nullptr;
    uint32_t hph[2] = {0u, 0u};
    bool pending[2] = {false, false};
    bool ok = true;
    int local = 0;
    for (int tile = cluster; tile < num_tiles && ok; tile += n_clusters, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      int m_blk, n_blk;
      tile_coords(tile, m_tiles, n_tiles, group, m_blk, n_blk);
      const int64_t row0 = static_cast<int64_t>(m_blk) * BM + rank * HALF + q * 32;
      const int64_t colT = static_cast<int64_t>(n_blk) * BN;
      const int64_t left = (g.N - colT + RES_COLS - 1) / RES_COLS;
      const int nch = row0 < g.M ? static_cast<int>(left < BN / RES_COLS ? left : BN / RES_COLS) : 0;
      if (lane == 0) {
        tma_store_wait_read0();  // both slots free again
        for (int c = 0; c < min(2, nch); ++c) {
          mbar_arrive_expect_tx(&hbar[c], RES_H_BYTES);
          tma_load_2d(&map_h, &hbar[c], wbuf + c * RES_H_BYTES, static_cast<int>(colT + RES_COLS * c),
                      static_cast<int>(row0));
          pending[c] = true;
        }
      }
      const bool w = mbar_wait(&tl->acc_full[acc], acc_phase, abort_flag, g.status, WHERE_GEMM);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < nch; ++c) {
        uint32_t r[RES_COLS];
        tmem_ld16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + RES_COLS * c, r);
        tmem_wait_ld();
        const int sl = c & 1;
        const bool wh = mbar_wait(&hbar[sl], hph[sl], abort_flag, g.status, WHERE_GEMM);
        if (!__all_sync(0xffffffffu, wh)) {
          ok = false;
          break;
        }
        hph[sl] ^= 1u;
        pending[sl] = false;
        float* hs = reinterpret_cast<float*>(wbuf + sl * RES_H_BYTES);
        uint8_t* cs = wbuf + 2 * RES_H_BYTES + sl * RES_C_BYTES;
        float hv[RES_COLS];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // 64-byte rows, 64-byte swizzle: 16-byte chunk k of row r sits at k ^ ((r >> 1) & 3)
          float4* a = reinterpret_cast<float4*>(hs + lane * 16 + 4 * (k ^ ((lane >> 1) & 3)));
          float4 x = *a;
          x.x += __uint_as_float(r[4 * k]);
          x.y += __uint_as_float(r[4 * k + 1]);
          x.z += __uint_as_float(r[4 * k + 2]);
          x.w += __uint_as_float(r[4 * k + 3]);
          *a = x;
          hv[4 * k] = x.x; hv[4 * k + 1] = x.y; hv[4 * k + 2] = x.z; hv[4 * k + 3] = x.w;
        }
        if (copy) {
          uint32_t pk[RES_COLS / 2];
          if (g.copy_dither != 0u) {
            // one hash per column pair of this row: (seed, row, pair) -> 32 bits
            const uint32_t rkey = g.copy_dither ^ (static_cast<uint32_t>(row0 + lane) * 0x9E3779B1u);
            const uint32_t pair0 = static_cast<uint32_t>((colT + RES_COLS * c) >> 1);
#pragma unroll
            for (int k = 0; k < RES_COLS / 2; ++k)
              pk[k] = pack_bf16x2_unbiased(hv[2 * k], hv[2 * k + 1],
                                           hash32(rkey + (pair0 + k) * 0x85EBCA77u));
          } else {
#pragma unroll
            for (int k = 0; k < RES_COLS / 2; ++k) pk[k] = pack_bf16x2(hv[2 * k], hv[2 * k + 1]);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k)
            // 32-byte rows, 32-byte swizzle: chunk k of row r sits at k ^ ((r >> 2) & 1)
            *reinterpret_cast<uint4*>(cs + lane * 32 + 16 * (k ^ ((lane >> 2) & 1))) =
                make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int x = static_cast<int>(colT + RES_COLS * c), y = static_cast<int>(row0);
          tma_store_2d(&map_h, hs, x, y);
          if (copy) tma_store_2d(&map_c, cs, x, y);
          tma_store_commit();
          if (c + 2 < nch) {
            tma_store_wait_read0();  // the slot's stores have read it
            mbar_arrive_expect_tx(&hbar[sl], RES_H_BYTES);
            tma_load_2d(&map_h, &hbar[sl], hs, x + 2 * RES_COLS, y);
            pending[sl] = true;
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0[acc]);
    }
    if (lane == 0) {
      for (int sl = 0; sl < 2; ++sl)
        if (pending[sl]) (void)drain_wait(&hbar[sl], hph[sl]);
      tma_store_wait0();
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the pair's MMAs may still read its tiles
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

template <int EPI>
cudaError_t launch(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb2,
                   const CUtensorMap& mh, const CUtensorMap& mc, const GemmArgs& g, int grid,
                   int group, cudaStream_t s) {
  auto kern = gemm_bf16_tc_kernel<EPI>;
  constexpr size_t kGemmSmem = gemm_smem<EPI>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kGemmSmem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = kGemmSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, ma, mb, mb2, mh, mc, g, group);
}

}  // namespace

cudaError_t gemm_bf16(const GemmArgs& g, cudaStream_t s) {
  CUtensorMap ma, mb, mb2;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(g.K), static_cast<uint64_t>(g.M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(g.lda) * 2};
    const uint32_t box[2] = {64, HALF};
    if (!encode_tmap(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.a, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  if (g.b2 != nullptr && (g.n_split <= 0 || g.n_split % BN != 0 || g.n_split >= g.N))
    return cudaErrorInvalidValue;
  const int64_t n_first = g.b2 != nullptr ? g.n_split : g.N;  // rows of b
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(g.K), static_cast<uint64_t>(n_first)};
    const uint64_t strides[1] = {static_cast<uint64_t>(g.ldb) * 2};
    const uint32_t box[2] = {64, HALF};
    if (!encode_tmap(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.b, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  mb2 = mb;
  if (g.b2 != nullptr) {
    const uint64_t dims[2] = {static_cast<uint64_t>(g.K), static_cast<uint64_t>(g.N - g.n_split)};
    const uint64_t strides[1] = {static_cast<uint64_t>(g.ldb) * 2};
    const uint32_t box[2] = {64, HALF};
    if (!encode_tmap(&mb2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.b2, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const int64_t m_tiles = (g.M + BM - 1) / BM, n_tiles = (g.N + BN - 1) / BN;
  const int64_t tiles = m_tiles * n_tiles;
  const int clusters = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(tiles, device_sm_count() / 2)));
  // A wave of clusters covers `group` M tiles by about four N tiles. The
  // residual GEMM (few N tiles, with h streamed through L2 beside it) covers
  // all N tiles of `group` M tiles instead, so each A tile is read by one wave
  // and leaves L2 with it: at 720p (M = 19,320, K = N = 3,072) DRAM reads fall
  // from 568 to 473 MB per launch and the launch from 277 to 266 us.
  const int64_t n_per_wave = (g.epi == EPI_RESIDUAL && 2 * n_tiles <= clusters)
                                 ? n_tiles
                                 : std::min<int64_t>(4, n_tiles);
  const int group = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(m_tiles, clusters / n_per_wave)));
  if (g.epi == EPI_STORE) {
    // bf16 output C [M, N] in 32 x 32 boxes with a 64-byte swizzle
    CUtensorMap mo;
    const uint64_t dims[2] = {static_cast<uint64_t>(g.N), static_cast<uint64_t>(g.M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(g.ldc) * 2};
    const uint32_t box[2] = {32, 32};
    if (!encode_tmap(&mo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.c, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
    return launch<EPI_STORE>(ma, mb, mb2, ma, mo, g, 2 * clusters, group, s);
  }
  // residual epilogue: h (fp32, 16-column x 32-row boxes, 64-byte swizzle) and
  // its bf16 copy (16 x 32 boxes, 32-byte swizzle); without a copy the h map
  // stands in
  CUtensorMap mh, mc;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(g.N), static_cast<uint64_t>(g.M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(g.ldh) * 4};
    const uint32_t box[2] = {RES_COLS, 32};
    if (!encode_tmap(&mh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, g.h, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  mc = mh;
  if (g.h_copy != nullptr) {
    const uint64_t dims[2] = {static_cast<uint64_t>(g.N), static_cast<uint64_t>(g.M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(g.ldhc) * 2};
    const uint32_t box[2] = {RES_COLS, 32};
    if (!encode_tmap(&mc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.h_copy, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_32B))
      return cudaErrorInvalidValue;
  }
  return launch<EPI_RESIDUAL>(ma, mb, mb2, mh, mc, g, 2 * clusters, group, s);
}

}  // namespace sva
