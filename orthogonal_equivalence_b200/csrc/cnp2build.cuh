// Cayley-Neumann build for b = 256 blocks on CTA pairs with the intermediate
// operands kept in shared memory (POET-X write-up, section 3:
// G = (I+Q)(I+Q+Q^2+Q^3) from the packed skew Q).
//
// With S = Q Q = -Q Q^T and H = 2Q + S, G = I + H + S + H S^T.  Both products
// of a block read only the rows each CTA of the pair already holds:
//   P1: acc0 = Q Q^T   A = this CTA's 128 rows of Q, B = the same rows (the
//                      pair's N half of Q^T is this CTA's rows of Q)
//   E1: S = -acc0, H = S + 2Q, both written as bf16 operand tiles into this
//       CTA's shared memory (the 128-byte swizzled K-major layout TMA uses)
//   P2: acc1 = H S^T   A = this CTA's rows of H, B = its rows of S
//   E2: G = I + H + S + acc1, rounded once to bf16, written over this
//       warp's rows of S and sent to global memory by TMA stores of
//       32-row x 64-column boxes
// so no operand leaves the SM between the phases (the kernel used for the
// backward stages S, H through L2).  Q of the next block is loaded as soon as
// E1 has read this block's Q, and P1 of the next block runs during E2 of this
// one (acc0 and acc1 are separate TMEM accumulators).
//
//   warp 0: TMA loads of Q (both CTAs; completion counted on the leader)
//   warp 1: TMEM owner (both CTAs) and MMA issuer (leader only)
//   warps 2-5: epilogues (both CTAs), rows 32 * quarter .. +31 of this CTA's 128
// Every wait is bounded (ptx.cuh); no load uses multicast.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "cnp2sm.cuh"

namespace poetx {
namespace cnp2b {

constexpr int BLK = cnp2::BLK;
constexpr int HALF = cnp2::HALF;
constexpr int CH = cnp2::CH;
constexpr int UMMA_K = cnp2::UMMA_K;
constexpr int TILE_BYTES = cnp2::TILE_BYTES;       // 128 rows x 64 bf16 columns
constexpr int MAT_BYTES = 4 * TILE_BYTES;          // this CTA's 128 rows x 256 columns
constexpr int NUM_THREADS = 192;
constexpr int NBARS = 6;
constexpr int SMEM_BYTES = 3 * MAT_BYTES + 1024 + 256;

struct Params {
  int nblk;
  uint32_t idesc;                 // A K-major, B K-major, M = N = 256
};

// One tensor map per segment over its G ([blocks * 256][256] bf16, boxes of
// 32 rows x 64 columns, 128-byte swizzle): E2 writes G with TMA stores.
struct GMaps {
  CUtensorMap m[kMaxSegs];
};

// 32 bf16 of row r, columns c0 .. c0+31 (c0 % 32 == 0), into the 128-byte
// swizzled K-major tiles of a 128 x 256 matrix (tile c0 / 64; 16-byte chunk u
// of a row sits at chunk u ^ (r % 8)).
__device__ __forceinline__ void tile_row_store_bf16x32(uint32_t mat, int r, int c0, const float* v) {
  const uint32_t rowp = mat + (c0 >> 6) * TILE_BYTES + r * 128;
  const int u0 = (c0 & 63) >> 3;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t w0 = pack_bf16x2(v[8 * u], v[8 * u + 1]), w1 = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
    const uint32_t w2 = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), w3 = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowp + (((u0 + u) ^ (r & 7)) << 4)), "r"(w0),
                 "r"(w1), "r"(w2), "r"(w3)
                 : "memory");
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    cnp_build_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ cnp2::PairSegs sg,
                          const __grid_constant__ GMaps gm, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 3 * MAT_BYTES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = tc2::cluster_rank();
  const bool leader = rank == 0;
  const uint32_t sQ = smem_u32(smem), sS = sQ + MAT_BYTES, sH = sS + MAT_BYTES;
  auto bar = [&](int i) { return smem_u32(bars + i); };
  // QFULL (leader, TMA bytes of both CTAs), QEMPTY (each CTA, its 4 epilogue
  // warps), A0FULL / A1FULL (each CTA, MMA commits), E1DONE / A1EMPTY (leader,
  // 4 epilogue warps x 2 CTAs)
  const int QFULL = 0, QEMPTY = 1, A0FULL = 2, A1FULL = 3, E1DONE = 4, A1EMPTY = 5;

  if (threadIdx.x == 0) {
    mbar_init(bar(QFULL), 1);
    mbar_init(bar(QEMPTY), 4);
    mbar_init(bar(A0FULL), 1);
    mbar_init(bar(A1FULL), 1);
    mbar_init(bar(E1DONE), 8);
    mbar_init(bar(A1EMPTY), 8);
    *s_abort = 0;
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
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- Q loads: this CTA's 128 rows of the block's bf16 Q
      prefetch_tmap(&tmQ);
      const uint32_t qfull_leader = tc2::map_to_rank(bar(QFULL), 0);
      int it = 0;
      for (int blk = pair; blk < p.nblk; blk += npairs, ++it) {
        // E1 of the previous block has read Q
        if (!mbar_wait(bar(QEMPTY), (it & 1) ^ 1u, DERR_GEMM_WAIT)) {
          *s_abort = 1;
          break;
        }
        if (leader) mbar_arrive_expect_tx(bar(QFULL), 2 * MAT_BYTES);
        for (int c = 0; c < 4; ++c)
          tc2::tma_load_2d_pair(sQ + c * TILE_BYTES, &tmQ, qfull_leader, c * CH, blk * BLK + int(rank) * HALF);
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // ---------------- MMA issuer (leader, for both CTAs)
      const uint32_t acc0 = tmem_base, acc1 = tmem_base + BLK;
      int it = 0;
      for (int blk = pair; blk < p.nblk; blk += npairs, ++it) {
        // P1: acc0 = Q Q^T (acc0 is free: E1 of the previous block was waited for below)
        if (!mbar_wait(bar(QFULL), it & 1, DERR_GEMM_WAIT)) {
          *s_abort = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int kk = 0; kk < CH / UMMA_K; ++kk) {
            const uint64_t d = smem_desc_sw128(sQ + c * TILE_BYTES + kk * 32, 16, 1024);
            tc2::mma_pair(acc0, d, d, p.idesc, (c | kk) != 0 ? 1u : 0u);
          }
        tc2::commit_pair(bar(A0FULL));
        // P2: acc1 = H S^T once both CTAs' E1 wrote H and S, and E2 of the
        // previous block has read acc1
        if (!mbar_wait(bar(E1DONE), it & 1, DERR_GEMM_WAIT) ||
            !mbar_wait(bar(A1EMPTY), (it & 1) ^ 1u, DERR_GEMM_WAIT)) {
          *s_abort = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int kk = 0; kk < CH / UMMA_K; ++kk)
            tc2::mma_pair(acc1, smem_desc_sw128(sH + c * TILE_BYTES + kk * 32, 16, 1024),
                          smem_desc_sw128(sS + c * TILE_BYTES + kk * 32, 16, 1024), p.idesc, (c | kk) != 0 ? 1u : 0u);
        tc2::commit_pair(bar(A1FULL));
      }
    }
  } else {
    // ---------------- epilogues (both CTAs)
    const int quarter = warp & 3;
    const int lrow = quarter * 32 + lane;            // row of this CTA's half
    const int row = int(rank) * HALF + lrow;         // row of the block
    const uint32_t t0 = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t e1done_leader = tc2::map_to_rank(bar(E1DONE), 0);
    const uint32_t a1empty_leader = tc2::map_to_rank(bar(A1EMPTY), 0);
    int it = 0;
    for (int blk = pair; blk < p.nblk; blk += npairs, ++it) {
      const int s = cnp2::pair_seg_of(sg, blk);
      const int lt = blk - sg.start[s];
      // E1: S = -acc0, H = S + 2Q into the operand tiles
      bool ok = !*s_abort && mbar_wait(bar(A0FULL), it & 1, DERR_GEMM_WAIT);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) *s_abort = 1;
        break;
      }
      tc_fence_after();
      for (int c0 = 0; c0 < BLK; c0 += 64) {
        float a[32], b[32], q[32];
        tmem_ld_32cols_x2(t0 + c0, t0 + c0 + 32, a, b);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int cc = c0 + 32 * h;
          float* v = h ? b : a;
          cnp2::tile_row_bf16x32(sQ + (cc >> 6) * TILE_BYTES, lrow, cc, q);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            v[e] = -v[e];             // S
            q[e] = v[e] + 2.f * q[e];  // H = S + 2Q
          }
          tile_row_store_bf16x32(sS, lrow, cc, v);
          tile_row_store_bf16x32(sH, lrow, cc, q);
        }
      }
      // the tiles are read by the tensor cores (async proxy) next; Q and acc0 are free
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(QEMPTY));
        tc2::remote_arrive(e1done_leader);
      }
      // E2: G = I + H + S + acc1
      ok = mbar_wait(bar(A1FULL), it & 1, DERR_GEMM_WAIT);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) *s_abort = 1;
        break;
      }
      tc_fence_after();
      // G replaces S in this warp's 32 rows of each tile (S and H of a row are
      // read before its G is written), and each 32-row x 64-column box goes
      // out with one TMA store
      for (int c0 = 0; c0 < BLK; c0 += 64) {
        float a[32], b[32], hs[32], sv[32];
        tmem_ld_32cols_x2(t0 + BLK + c0, t0 + BLK + c0 + 32, a, b);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int cc = c0 + 32 * h;
          float* v = h ? b : a;
          cnp2::tile_row_bf16x32(sH + (cc >> 6) * TILE_BYTES, lrow, cc, hs);
          cnp2::tile_row_bf16x32(sS + (cc >> 6) * TILE_BYTES, lrow, cc, sv);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = ((cc + e == row ? 1.f : 0.f) + (hs[e] + sv[e])) + v[e];
          tile_row_store_bf16x32(sS, lrow, cc, v);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&gm.m[s], sS + (c0 >> 6) * TILE_BYTES + quarter * 32 * 128, c0, lt * BLK + row - lane);
          bulk_commit();
        }
      }
      // the next block's E1 writes S again: the stores have read it
      if (lane == 0) bulk_wait_read<0>();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) tc2::remote_arrive(a1empty_leader);
    }
    if (lane == 0) bulk_wait_all();  // G is in global memory before the block leaves
  }

  if (*s_abort && threadIdx.x == 0) {
    // give copies already issued time to land before the block leaves
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < 100000ull) {
    }
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

}  // namespace cnp2b
}  // namespace poetx
