// Backward of one side of the layer (POET-X write-up, section 1: the block
// products of R or P) in one kernel on CTA pairs, for b = 256 bf16 layers:
//   O_j = D_j G_j^T              (dY = dV G_P^T, or dXg = dU G_R^T)
//   part[s][j] = X_j^T D_j       (dG_P = Y^T dV, or dG_R = Xg^T dU, over the
//                                 tokens of split s)
// where D is the incoming gradient and X the saved activation of that side,
// both [T][d] bf16 in the permuted frame, and block j holds columns
// 256j .. 256j+255.  Both products read the same D tile, so D crosses HBM
// once instead of twice.
//
// A pair of SMs takes a work item (block j, token split s) and walks its
// 256-token tiles.  Per tile, with tcgen05 cta_group::2 MMAs (M = N = 256):
//   MMA1: O tile = D tile G_j^T.  Each CTA supplies its 128 tokens of D
//         (K-major, 4 chunks of 64 features) and its 128 rows of G_j, which
//         stay resident in shared memory for the whole item; each CTA keeps
//         its 128 token rows of the accumulator (TMEM columns 0..255).
//   MMA2: acc_G += X tile^T D tile.  Each CTA supplies the tile's 256 tokens
//         of its 128 feature columns of X and of D (MN-major, 4 chunks of 64
//         tokens); each CTA keeps its 128 feature rows of dG_j (TMEM columns
//         256..511), accumulated over every tile of the item.
// The O epilogue reads the tile's accumulator rows into registers and
// releases TMEM at once (the next tile's MMA1 waits only for that), then
// stores them (bf16 -> swizzled smem boxes -> TMA store) while MMA2 of the
// tile and the next tile's loads proceed; the dG partial
// (fp32) is written once per item.  Out-of-range token rows of the last tile
// are zero-filled by TMA (no contribution to dG) and clipped by the TMA
// store.
//
//   warp 0: TMA producer (both CTAs; copies signal the leader's barriers)
//   warp 1: TMEM owner (both CTAs) and MMA issuer (leader only)
//   warps 2-5: epilogues (both CTAs)
// Every wait is bounded (ptx.cuh).  No load uses multicast.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "gemm2sm.cuh"

namespace poetx {
namespace bdg2 {

constexpr int BLK = 256;
constexpr int HALF = 128;
constexpr int CH = 64;
constexpr int UMMA_K = 16;
constexpr int TILE_BYTES = HALF * 128;          // 128 x 64 bf16 (or 64 x 2 x 64, MN-major)
constexpr int STAGE_BYTES = 2 * TILE_BYTES;
constexpr int STAGES = 4;
constexpr int G_BYTES = 4 * TILE_BYTES;         // this CTA's 128 rows of G_j
constexpr int EPI_BOX = 32 * 128;               // 32 rows x 64 bf16
constexpr int EPI_BYTES = 4 * 2 * EPI_BOX;      // two boxes per epilogue warp
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + G_BYTES + EPI_BYTES + 1024 + 256;
constexpr int NUM_THREADS = 192;

struct Params {
  int T;
  int nblk;
  int splits;
  int ntiles;          // 256-token tiles
  int want_o;          // 0: dG only (no O)
  uint32_t idesc_kk;   // MMA1: A K-major, B K-major, M = N = 256
  uint32_t idesc_mnmn; // MMA2: A MN-major, B MN-major
  float* part;         // [splits][nblk][BLK][BLK]
};

// Tiles of split s: [s * ntiles / splits, (s + 1) * ntiles / splits).
__device__ __forceinline__ void split_tiles(const Params& p, int s, int& t0, int& t1) {
  t0 = static_cast<int>(int64_t(s) * p.ntiles / p.splits);
  t1 = static_cast<int>(int64_t(s + 1) * p.ntiles / p.splits);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    bdg_pair_kernel(const __grid_constant__ CUtensorMap tmDk, const __grid_constant__ CUtensorMap tmDmn,
                    const __grid_constant__ CUtensorMap tmXmn, const __grid_constant__ CUtensorMap tmG,
                    const __grid_constant__ CUtensorMap tmO, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + G_BYTES + EPI_BYTES);
  // full[STAGES] (leader), empty[STAGES], gfull (leader), gempty, ofull, oempty (leader), afull, aempty (leader)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 6);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = tc2::cluster_rank();
  const bool leader = rank == 0;
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t sG = smem_base + STAGES * STAGE_BYTES;
  const uint32_t sEpi = sG + G_BYTES;
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = STAGES, GFULL = 2 * STAGES, GEMPTY = GFULL + 1, OFULL = GFULL + 2,
            OEMPTY = GFULL + 3, AFULL = GFULL + 4, AEMPTY = GFULL + 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(FULL + s), 1);
      mbar_init(bar(EMPTY + s), 1);
    }
    mbar_init(bar(GFULL), 1);
    mbar_init(bar(GEMPTY), 1);
    mbar_init(bar(OFULL), 1);
    mbar_init(bar(OEMPTY), 8);  // 4 epilogue warps x 2 CTAs
    mbar_init(bar(AFULL), 1);
    mbar_init(bar(AEMPTY), 8);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  tc2::cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int items = p.nblk * p.splits;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      prefetch_tmap(&tmDk);
      prefetch_tmap(&tmDmn);
      prefetch_tmap(&tmXmn);
      prefetch_tmap(&tmG);
      int stage = 0;
      uint32_t ring = 0;
      int local = 0;
      bool ok = true;
      auto next_stage = [&](uint32_t bytes_both) -> bool {
        if (!mbar_wait(bar(EMPTY + stage), ring ^ 1u, DERR_GEMM_WAIT)) return false;
        if (leader) mbar_arrive_expect_tx(bar(FULL + stage), bytes_both);
        return true;
      };
      auto advance = [&]() {
        if (++stage == STAGES) {
          stage = 0;
          ring ^= 1u;
        }
      };
      for (int item = pair; item < items && ok; item += npairs, ++local) {
        const int j = item % p.nblk, s = item / p.nblk;
        int ta, tb;
        split_tiles(p, s, ta, tb);
        const int fcol = j * BLK + int(rank) * HALF;  // this CTA's feature columns of block j
        if (p.want_o) {
          // this CTA's rows of G_j, resident for the item
          if (!mbar_wait(bar(GEMPTY), (local & 1) ^ 1u, DERR_GEMM_WAIT)) { ok = false; break; }
          const uint32_t gfull = tc2::map_to_rank(bar(GFULL), 0);
          if (leader) mbar_arrive_expect_tx(bar(GFULL), 2 * G_BYTES);
          for (int c = 0; c < 4; ++c) tc2::tma_load_2d_pair(sG + c * TILE_BYTES, &tmG, gfull, c * CH, fcol);
        }
        for (int tile = ta; tile < tb && ok; ++tile) {
          const int tok = tile * BLK;
          if (p.want_o) {
            for (int c = 0; c < 4; ++c) {
              if (!next_stage(2 * TILE_BYTES)) { ok = false; break; }
              const uint32_t full = tc2::map_to_rank(bar(FULL + stage), 0);
              tc2::tma_load_2d_pair(smem_base + stage * STAGE_BYTES, &tmDk, full, j * BLK + c * CH,
                                    tok + int(rank) * HALF);
              advance();
            }
          }
          for (int c = 0; c < 4 && ok; ++c) {
            if (!next_stage(2 * STAGE_BYTES)) { ok = false; break; }
            const uint32_t full = tc2::map_to_rank(bar(FULL + stage), 0);
            const uint32_t sa = smem_base + stage * STAGE_BYTES, sb = sa + TILE_BYTES;
            const int row = tok + c * CH;
            tc2::tma_load_2d_pair(sa, &tmXmn, full, fcol, row);
            tc2::tma_load_2d_pair(sa + CH * 128, &tmXmn, full, fcol + CH, row);
            tc2::tma_load_2d_pair(sb, &tmDmn, full, fcol, row);
            tc2::tma_load_2d_pair(sb + CH * 128, &tmDmn, full, fcol + CH, row);
            advance();
          }
        }
      }
      if (!ok) {
        const uint64_t t0 = global_ns();
        while (global_ns() - t0 < 100000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // ---------------- MMA issuer (leader, for both CTAs)
      const uint32_t accO = tmem_base, accG = tmem_base + BLK;
      int stage = 0;
      uint32_t ring = 0;
      int local = 0, otiles = 0;
      bool ok = true;
      for (int item = pair; item < items && ok; item += npairs, ++local) {
        const int s = item / p.nblk;
        int ta, tb;
        split_tiles(p, s, ta, tb);
        if (p.want_o && !mbar_wait(bar(GFULL), local & 1, DERR_GEMM_WAIT)) { ok = false; break; }
        if (!mbar_wait(bar(AEMPTY), (local & 1) ^ 1u, DERR_GEMM_WAIT)) { ok = false; break; }
        tc_fence_after();
        for (int tile = ta; tile < tb && ok; ++tile) {
          if (p.want_o) {
            if (!mbar_wait(bar(OEMPTY), (otiles & 1) ^ 1u, DERR_GEMM_WAIT)) { ok = false; break; }
            tc_fence_after();
            for (int c = 0; c < 4; ++c) {
              if (!mbar_wait(bar(FULL + stage), ring, DERR_GEMM_WAIT)) { ok = false; break; }
              tc_fence_after();
              const uint32_t sa = smem_base + stage * STAGE_BYTES, sg = sG + c * TILE_BYTES;
#pragma unroll
              for (int kk = 0; kk < CH / UMMA_K; ++kk)
                tc2::mma_pair(accO, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sg + kk * 32, 16, 1024),
                              p.idesc_kk, (c | kk) != 0 ? 1u : 0u);
              tc2::commit_pair(bar(EMPTY + stage));
              if (++stage == STAGES) { stage = 0; ring ^= 1u; }
            }
            if (!ok) break;
            tc2::commit_pair(bar(OFULL));
            ++otiles;
          }
          for (int c = 0; c < 4; ++c) {
            if (!mbar_wait(bar(FULL + stage), ring, DERR_GEMM_WAIT)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_base + stage * STAGE_BYTES, sb = sa + TILE_BYTES;
#pragma unroll
            for (int kk = 0; kk < CH / UMMA_K; ++kk)
              tc2::mma_pair(accG, smem_desc_sw128(sa + kk * (UMMA_K * 128), CH * 128, 1024),
                            smem_desc_sw128(sb + kk * (UMMA_K * 128), CH * 128, 1024), p.idesc_mnmn,
                            (tile != ta || c != 0 || kk != 0) ? 1u : 0u);
            tc2::commit_pair(bar(EMPTY + stage));
            if (++stage == STAGES) { stage = 0; ring ^= 1u; }
          }
        }
        if (!ok) break;
        if (p.want_o) tc2::commit_pair(bar(GEMPTY));  // G_j no longer read
        tc2::commit_pair(bar(AFULL));                  // also: every MMA of the item is done
      }
    }
  } else {
    // ---------------- epilogues (both CTAs): rows quarter*32 .. +31 of this CTA's 128
    const int quarter = warp & 3;
    const uint32_t my_boxes = sEpi + (warp - 2) * 2 * EPI_BOX;
    const uint32_t oempty_leader = tc2::map_to_rank(bar(OEMPTY), 0);
    const uint32_t aempty_leader = tc2::map_to_rank(bar(AEMPTY), 0);
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    int buf = 0;
    int local = 0, otiles = 0;
    bool ok = true;
    for (int item = pair; item < items && ok; item += npairs, ++local) {
      const int j = item % p.nblk, s = item / p.nblk;
      int ta, tb;
      split_tiles(p, s, ta, tb);
      if (p.want_o) {
        for (int tile = ta; tile < tb; ++tile, ++otiles) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(OFULL), otiles & 1, DERR_GEMM_WAIT));
          if (!ok) break;
          tc_fence_after();
          const int row0 = tile * BLK + int(rank) * HALF + quarter * 32;  // token rows of this warp
          const bool rows_in = row0 < p.T;
          // the whole 256-column row into registers (bf16 pairs), then release
          // the accumulator so the next tile's MMA1 can start while this tile
          // is stored
          uint32_t w[BLK / 2];
#pragma unroll
          for (int c = 0; c < BLK / 64; ++c) {
            float v[32], u[32];
            tmem_ld_32cols_x2(tl + 64 * c, tl + 64 * c + 32, v, u);  // one round trip per 64 columns
#pragma unroll
            for (int i = 0; i < 16; ++i) w[32 * c + i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
#pragma unroll
            for (int i = 0; i < 16; ++i) w[32 * c + 16 + i] = pack_bf16x2(u[2 * i], u[2 * i + 1]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) tc2::remote_arrive(oempty_leader);
          if (rows_in) {
#pragma unroll
            for (int c0 = 0; c0 < BLK / 64; ++c0) {
              if (lane == 0) bulk_wait_read<1>();
              __syncwarp();
              const uint32_t box = my_boxes + buf * EPI_BOX;
              const uint32_t rowp = box + lane * 128;
#pragma unroll
              for (int k = 0; k < 8; ++k)
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowp + ((k ^ (lane & 7)) << 4)),
                             "r"(w[32 * c0 + 4 * k]), "r"(w[32 * c0 + 4 * k + 1]), "r"(w[32 * c0 + 4 * k + 2]),
                             "r"(w[32 * c0 + 4 * k + 3])
                             : "memory");
              fence_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&tmO, box, j * BLK + 64 * c0, row0);
                bulk_commit();
              }
              buf ^= 1;
            }
          }
        }
        if (!ok) break;
      }
      // dG partial of this item: this CTA's 128 feature rows, fp32
      ok = __all_sync(0xffffffffu, mbar_wait(bar(AFULL), local & 1, DERR_GEMM_WAIT));
      if (!ok) break;
      tc_fence_after();
      float* dst = p.part + ((int64_t(s) * p.nblk + j) * BLK + int(rank) * HALF + quarter * 32 + lane) * BLK;
#pragma unroll 1
      for (int c0 = 0; c0 < BLK; c0 += 64) {
        float v[32], v2[32];
        tmem_ld_32cols_x2(tl + BLK + c0, tl + BLK + c0 + 32, v, v2);
        float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
        for (int u = 0; u < 8; ++u) d4[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
#pragma unroll
        for (int u = 0; u < 8; ++u) d4[8 + u] = make_float4(v2[4 * u], v2[4 * u + 1], v2[4 * u + 2], v2[4 * u + 3]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) tc2::remote_arrive(aempty_leader);
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  tc2::cluster_sync();  // every MMA into either CTA's TMEM and every remote arrive is done
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512) : "memory");
  }
  tc2::cluster_sync();
}

}  // namespace bdg2
}  // namespace poetx
