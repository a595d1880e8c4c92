// W0 GEMM on CTA pairs (tcgen05 cta_group::2): a 256 x 256 output tile per
// pair of SMs.  Each CTA of the pair loads its 128 rows of A and its 128
// columns of B, so every SM stages and reads half of the B tile it would need
// alone; the leader CTA issues the MMAs for both, each CTA keeps the
// accumulator rows of its half in its own TMEM and stores them with TMA.
//
//   warp 0: TMA producer (both CTAs; copies signal the leader's barrier)
//   warp 1: TMEM owner (both CTAs) and MMA issuer (leader only)
//   warps 2-5: epilogue (both CTAs): TMEM -> registers -> smem box -> TMA store
//
// bf16 operands, fp32 accumulation, plain output (no addends), batch 1.
// Every wait is bounded (see ptx.cuh); no load uses multicast.
#pragma once

#include "gemm.cuh"

namespace poetx {
namespace tc2 {

constexpr int BM = 256;          // rows per pair (128 per CTA)
constexpr int BN = 256;          // columns per pair (each CTA stages 128 of B)
constexpr int CH = 64;           // bf16 elements per 128-byte row = K per stage
constexpr int UMMA_K = 16;
constexpr int A_BYTES = 128 * 128;   // this CTA's 128 rows x 64 K
constexpr int B_BYTES = 128 * 128;   // this CTA's 128 columns x 64 K
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int STAGES = 6;
constexpr int TMEM_COLS = 2 * BN;    // two 256-column accumulators (128 lanes each CTA)
constexpr int EPI_BOX = 32 * 128;
constexpr int EPI_BYTES = 4 * 2 * EPI_BOX;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + 256;
constexpr int NUM_THREADS = 192;
struct Params {
  int M, N, K;
  int tiles_m, tiles_n;
  int group;             // raster: panels per group along the grouped dimension
  int group_n;           // 0: groups of M panels (A group held in L2, B streamed); 1: groups of N panels
  int b_mn;              // B operand MN-major (W~^T in the backward)
  uint32_t idesc;
  uint32_t b_lbo, b_kstep;
  float alpha;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void remote_arrive(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on the
// leader CTA's barrier (cluster address); no multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar_cluster, int32_t c0,
                                                 int32_t c1) {
  if (!copy_ok((c0 & 3) == 0 && (dst & 127u) == 0)) return;
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(tmap), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at this offset in both CTAs of the pair once the
// leader's MMAs issued so far have completed.
__device__ __forceinline__ void commit_pair(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void decode(const Params& p, int tile, int& mt, int& nt) {
  // Tiles of one group share a set of `group` panels of the grouped dimension,
  // which stay in L2 while the other dimension is swept (grouped dimension
  // fastest, so the pairs of one wave read the same streamed panel together).
  const int grouped = p.group_n ? p.tiles_n : p.tiles_m;
  const int other = p.group_n ? p.tiles_m : p.tiles_n;
  const int span = p.group * other;
  const int g = tile / span;
  const int first = g * p.group;
  const int gsize = min(grouped - first, p.group);
  const int r = tile - g * span;
  const int a = first + r % gsize, b = r / gsize;
  mt = p.group_n ? b : a;
  nt = p.group_n ? a : b;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + EPI_BYTES);
  // bars: full[STAGES] (leader), empty[STAGES], tfull[2], tempty[2] (leader), drain
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t sEpi = smem_base + STAGES * STAGE_BYTES;
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = STAGES, TFULL = 2 * STAGES, TEMPTY = 2 * STAGES + 2, DRAIN = 2 * STAGES + 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(FULL + s), 1);
      mbar_init(bar(EMPTY + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(TFULL + a), 1);
      mbar_init(bar(TEMPTY + a), 8);  // 4 epilogue warps x 2 CTAs
    }
    mbar_init(bar(DRAIN), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int total = p.tiles_m * p.tiles_n;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        int mt, nt;
        decode(p, tile, mt, nt);
        const int m0 = mt * BM + rank * 128;  // this CTA's rows of A
        const int n0 = nt * BN + rank * 128;  // this CTA's columns of B
        const int nkb = (p.K + CH - 1) / CH;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(bar(EMPTY + stage), phase ^ 1u, DERR_GEMM_WAIT)) { ok = false; break; }
          const uint32_t full_leader = map_to_rank(bar(FULL + stage), 0);
          if (leader) mbar_arrive_expect_tx(bar(FULL + stage), 2 * STAGE_BYTES);
          const uint32_t sa = smem_base + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          const int k = kb * CH;
          tma_load_2d_pair(sa, &tmA, full_leader, k, m0);
          if (!p.b_mn) {
            tma_load_2d_pair(sb, &tmB, full_leader, k, n0);
          } else {
            tma_load_2d_pair(sb, &tmB, full_leader, n0, k);
            tma_load_2d_pair(sb + CH * 128, &tmB, full_leader, n0 + CH, k);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // give copies already issued time to land before the block leaves
        const uint64_t t0 = global_ns();
        while (global_ns() - t0 < 100000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // ---------------- MMA issuer (leader CTA, for both)
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      const int nkb = (p.K + CH - 1) / CH;
      for (int tile = pair; tile < total && ok; tile += npairs, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(bar(TEMPTY + acc), acc_phase ^ 1u, DERR_GEMM_WAIT)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(bar(FULL + stage), phase, DERR_GEMM_WAIT)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < CH / UMMA_K; ++kk) {
            const uint64_t da = smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t db = smem_desc_sw128(sb + kk * p.b_kstep, p.b_lbo, 1024);
            mma_pair(d_tmem, da, db, p.idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          commit_pair(bar(EMPTY + stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        commit_pair(bar(TFULL + acc));
      }
      asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar(DRAIN))
                   : "memory");
      mbar_wait(bar(DRAIN), 0, DERR_GEMM_WAIT);
    }
  } else {
    // ---------------- epilogue (both CTAs): this CTA's 128 rows of each tile
    const int quarter = warp & 3;
    const uint32_t my_boxes = sEpi + (warp - 2) * 2 * EPI_BOX;
    const uint32_t tempty_leader = map_to_rank(bar(TEMPTY), 0);  // + 8 * acc
    int buf = 0;
    int local = 0;
    for (int tile = pair; tile < total; tile += npairs, ++local) {
      int mt, nt;
      decode(p, tile, mt, nt);
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      bool ok = mbar_wait(bar(TFULL + acc), acc_phase, DERR_GEMM_WAIT);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int row0 = mt * BM + rank * 128 + quarter * 32;
      const bool rows_in = row0 < p.M;
      const uint32_t tl = tmem_base + acc * BN + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 64) {
        uint32_t w[32];
        float v[32];
        tmem_ld_32cols(tl + c0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(p.alpha * v[2 * i], p.alpha * v[2 * i + 1]);
        tmem_ld_32cols(tl + c0 + 32, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) w[16 + i] = pack_bf16x2(p.alpha * v[2 * i], p.alpha * v[2 * i + 1]);
        if (!rows_in) continue;
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        const uint32_t box = my_boxes + buf * EPI_BOX;
        const uint32_t rowp = box + lane * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowp + ((k ^ (lane & 7)) << 4)),
                       "r"(w[4 * k]), "r"(w[4 * k + 1]), "r"(w[4 * k + 2]), "r"(w[4 * k + 3])
                       : "memory");
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmC, box, nt * BN + c0, row0);
          bulk_commit();
        }
        buf ^= 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) remote_arrive(tempty_leader + 8 * acc);
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // every MMA into either CTA's TMEM and every remote arrive is done
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
  cluster_sync();
}

}  // namespace tc2
}  // namespace poetx
