// Cayley-Neumann backward for b = 256 blocks on CTA pairs (POET-X write-up,
// section 3: the gradient of the packed triangle of G = (I+Q)(I+Q+Q^2+Q^3)),
// and the prep kernel it shares with the build (cnp2build.cuh).
//
// A grid-wide prep kernel first writes, for every block of the batch, Q in
// bf16 (Qb) and, for the backward, dG in bf16 (Gb) and the part of dq that
// needs no product, dq = 2 (dG[i][j] - dG[j][i]).  The fused kernel then
// takes one 256 x 256 block per pair of SMs at a time: the leader CTA issues every product of the block back to
// back as tcgen05 MMAs with cta_group::2 (bf16 operands, fp32 accumulation),
// each CTA keeping the accumulator rows of its half (rows 128*rank .. +127)
// in its own TMEM.  Operands are read with TMA from Qb, Gb and a per-pair
// slot (S, H^T, dS, written by the previous epilogue with TMA stores from
// swizzled 32-row boxes; one slot per pair, reused block after block, so it
// stays in L2).  A K-major tile of a matrix
// is its rows and an MN-major tile its columns, so Q^T = -Q and dG^T, dS^T
// need no copies.
//
// With S = Q^2 = -Q Q^T and H = 2Q + S (G = I + 2Q + 2S + H S^T):
// dS = 2dG + H^T dG + dG S, dA = 2dG + 2 dG S - dS Q - Q dS,
// dq_k = dA[i][j] - dA[j][i] for k = k(i, j):
//   P1: acc0 = Q Q^T                          E1: S = -acc0, H^T = S - 2Q
//   P2: acc0 = H^T dG,  acc1 = dG S^T         E2: dS = 2dG + acc0 + acc1;
//                                                 acc1 <- 2 acc1 (TMEM store)
//   P3: acc1 += dS Q^T + Q^T dS               E3: acc1 (= dA - 2dG) -> smem
//   F : dq += acc1[i][j] - acc1[j][i]  (the partner's rows through
//       distributed shared memory; dq staged in shared memory by bulk copies)
// The additive terms are added in fp32: S from the fp32 accumulator; the 2dG
// of dq exactly (prep).  2Q in H^T and 2dG in dS, which only feed bf16
// operands, use the bf16 copies the epilogue finds
// in the staged operand tiles (the last four chunks of a phase always sit in
// stages 0..3 when its epilogue runs).
//
//   warp 0: TMA producer (both CTAs; copies signal the leader's barrier) and
//           the bulk copies of this CTA's half of dq
//   warp 1: TMEM owner (both CTAs) and MMA issuer (leader only)
//   warps 2-5: epilogues; all six warps: fold
// All threads of both CTAs meet at a cluster barrier between phases.  Every
// mbarrier wait is bounded (ptx.cuh); after a timeout a thread skips the
// rest of its work but still takes every cluster barrier.  No load uses
// multicast.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "cnp.cuh"
#include "gemm2sm.cuh"

namespace poetx {
namespace cnp2 {

constexpr int BLK = 256;                 // block size this kernel handles
constexpr int HALF = 128;                // rows per CTA
constexpr int CH = 64;                   // K per stage (128 bytes of bf16)
constexpr int UMMA_K = 16;
constexpr int TILE_BYTES = HALF * 128;   // 128 rows x 64 bf16, or 64 rows x 2 x 64 (MN-major)
constexpr int STAGE_BYTES = 2 * TILE_BYTES;
constexpr int STAGES = 4;
constexpr int EPI_BOX = 32 * 128;        // 32 rows x 64 bf16: one TMA store of an epilogue warp
constexpr int RING_BYTES = STAGES * STAGE_BYTES;
constexpr int DA_LD = BLK + 1;           // padded fp32 row of acc1 in shared memory
constexpr int DA_SMEM = HALF * DA_LD * 4;
constexpr int REGION0 = ((RING_BYTES > DA_SMEM ? RING_BYTES : DA_SMEM) + 1023) & ~1023;
constexpr int64_t TRI = int64_t(BLK) * (BLK - 1) / 2;
constexpr int DQ_HALF = static_cast<int>(TRI / 2);      // dq entries per CTA
constexpr int DQ_BYTES = DQ_HALF * 4;                   // 65280, a multiple of 16
// The fold splits the triangle into eight bands of 32 rows; band I holds the
// entries of rows 32I .. 32I+31 (7664 - 1024 I of them, a contiguous run of
// dq).  CTA 0 folds bands 0, 3, 4, 7 and CTA 1 bands 1, 2, 5, 6: 16320
// entries and 18 tiles of 32 x 32 each.
constexpr int BANDS = BLK / 32;
__host__ __device__ constexpr int band_of(int rank, int b) {
  return rank == 0 ? (b == 0 ? 0 : b == 1 ? 3 : b == 2 ? 4 : 7) : (b == 0 ? 1 : b == 1 ? 2 : b == 2 ? 5 : 6);
}
__host__ __device__ constexpr int band_start(int I) { return I * (2 * BLK - 1 - 32 * I) * 16; }  // tri_index(32I, 32I+1)
__host__ __device__ constexpr int band_size(int I) { return band_start(I + 1) - band_start(I); }
static_assert(band_start(BANDS) == TRI, "bands cover the triangle");
static_assert(band_size(0) + band_size(3) + band_size(4) + band_size(7) == DQ_HALF &&
                  band_size(1) + band_size(2) + band_size(5) + band_size(6) == DQ_HALF,
              "each CTA folds half of dq");
constexpr int NUM_THREADS = 192;
constexpr int TT_LD = 33;                // padded row of a warp's 32 x 32 transpose tile
constexpr int TT_BYTES = (NUM_THREADS / 32) * 32 * TT_LD * 4;
constexpr int SMEM_BYTES = REGION0 + DQ_BYTES + 256 + TT_BYTES + 1024;
constexpr int SKINDS = 3;                // per-pair slot: S, H^T, dS
enum SlotKind : int { KS = 0, KH, KDS };
constexpr size_t MAT_BYTES = size_t(BLK) * BLK * 2;

// Operands of one K chunk: A and B are this CTA's rows (K-major) or, with a
// "C" suffix, this CTA's columns (MN-major) of the named matrices.
enum Chunk : int { C_QQ = 0, C_H_GC, C_G_S, C_DS_Q, C_QC_DSC };

struct PairSegs {
  int n;
  int start[kMaxSegs + 1];
  const float* q[kMaxSegs];   // packed triangles [blocks][TRI]
  const float* dG[kMaxSegs];  // backward: dL/dG [blocks][BLK][BLK]
  void* out[kMaxSegs];        // build: G (bf16); backward: dq (fp32)
};

struct Params {
  int nblk;
  uint32_t idesc_kk;       // A K-major, B K-major, M = N = 256
  uint32_t idesc_kmn;      // A K-major, B MN-major
  uint32_t idesc_mnmn;     // A MN-major, B MN-major
};
// The operand region the tensor maps cover: [Qb: nblk][Gb: nblk][slots: pairs x SKINDS], BLK x BLK bf16 each.

__device__ __forceinline__ int pair_seg_of(const PairSegs& sg, int blk) {
  int s = 0;
  while (s + 1 < sg.n && blk >= sg.start[s + 1]) ++s;
  return s;
}

// Chunks of phase ph (1-based): count and type of chunk c.
__device__ __forceinline__ int phase_chunks(int ph) { return ph >= 2 ? 8 : 4; }
__device__ __forceinline__ int chunk_type(int ph, int c) {
  if (ph == 1) return C_QQ;
  if (ph == 2) return c < 4 ? C_H_GC : C_G_S;
  return c < 4 ? C_DS_Q : C_QC_DSC;
}

// ---------------------------------------------------------------- prep
// Qb, and for the backward Gb and dq = 2 (dG[i][j] - dG[j][i]), of the
// 64 x 64 tile pair (I, J), I <= J, of block blockIdx.y; grid (PREP_PAIRS,
// nblk), PREP_THREADS threads.  Warp w handles rows w, w + 8, ... of a tile
// and lane l its columns 2l and 2l + 1, so each warp store is one 128-byte
// (bf16) or 256-byte (fp32) run, and a thread issues all of its loads
// (16 triangle entries, 8 + 8 float2 of dG) before its first store.
constexpr int PREP_T = 64;
constexpr int PREP_TILES = BLK / PREP_T;
constexpr int PREP_PAIRS = PREP_TILES * (PREP_TILES + 1) / 2;
constexpr int PREP_THREADS = 256;
constexpr int PREP_ROWS = PREP_T / (PREP_THREADS / 32);  // rows per warp

template <bool BWD>
__global__ void __launch_bounds__(PREP_THREADS) prep_kernel(const __grid_constant__ PairSegs sg,
                                                            __nv_bfloat16* __restrict__ Qb,
                                                            __nv_bfloat16* __restrict__ Gb) {
  __shared__ float tq[PREP_T][PREP_T + 1];                 // triangle entries of tile (I, J)
  __shared__ float gs[BWD ? PREP_T : 1][PREP_T + 1];       // dG tile (J, I), read transposed
  const int t = blockIdx.y;
  int I = 0, x = blockIdx.x;
  while (x >= PREP_TILES - I) {
    x -= PREP_TILES - I;
    ++I;
  }
  const int J = I + x;
  const int s = pair_seg_of(sg, t), lt = t - sg.start[s];
  const float* q = sg.q[s] + int64_t(lt) * TRI;
  __nv_bfloat16* Qt = Qb + size_t(t) * BLK * BLK;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = 2 * lane;

  // loads: the triangle's runs are not 8-byte aligned, so its entries come one
  // float at a time (columns lane and lane + 32); dG rows come as float2
  float v[PREP_ROWS][2];
#pragma unroll
  for (int k = 0; k < PREP_ROWS; ++k) {
    const int r = warp + 8 * k, i = PREP_T * I + r;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = PREP_T * J + lane + 32 * h;
      v[k][h] = j > i ? q[tri_index(i, j, BLK)] : 0.f;
    }
  }
  float2 g1[BWD ? PREP_ROWS : 1], g2[BWD ? PREP_ROWS : 1];
  const float* dG = BWD ? sg.dG[s] + int64_t(lt) * BLK * BLK : nullptr;
  if (BWD) {
#pragma unroll
    for (int k = 0; k < PREP_ROWS; ++k) {
      const int r = warp + 8 * k;
      g1[k] = *reinterpret_cast<const float2*>(dG + (PREP_T * I + r) * BLK + PREP_T * J + c0);
      g2[k] = I < J ? *reinterpret_cast<const float2*>(dG + (PREP_T * J + r) * BLK + PREP_T * I + c0) : g1[k];
    }
  }
#pragma unroll
  for (int k = 0; k < PREP_ROWS; ++k) {
    const int r = warp + 8 * k;
    tq[r][lane] = v[k][0];
    tq[r][lane + 32] = v[k][1];
    if (BWD) {
      gs[r][c0] = g2[k].x;
      gs[r][c0 + 1] = g2[k].y;
    }
  }
  __syncthreads();

  float* dq = BWD ? static_cast<float*>(sg.out[s]) + int64_t(lt) * TRI : nullptr;
#pragma unroll
  for (int k = 0; k < PREP_ROWS; ++k) {
    const int r = warp + 8 * k, i = PREP_T * I + r;
    float a[2], m[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int c = c0 + e, j = PREP_T * J + c;
      // tile (I, J); for I < J also its mirror (J, I), Q[j][i] = -Q[i][j]
      a[e] = I < J ? tq[r][c] : (j > i ? tq[r][c] : (j < i ? -tq[c][r] : 0.f));
      m[e] = -tq[c][r];
    }
    *reinterpret_cast<uint32_t*>(Qt + i * BLK + PREP_T * J + c0) = pack_bf16x2(a[0], a[1]);
    if (I < J) *reinterpret_cast<uint32_t*>(Qt + (PREP_T * J + r) * BLK + PREP_T * I + c0) = pack_bf16x2(m[0], m[1]);
    if (BWD) {
      __nv_bfloat16* Gt = Gb + size_t(t) * BLK * BLK;
      *reinterpret_cast<uint32_t*>(Gt + i * BLK + PREP_T * J + c0) = pack_bf16x2(g1[k].x, g1[k].y);
      if (I < J)
        *reinterpret_cast<uint32_t*>(Gt + (PREP_T * J + r) * BLK + PREP_T * I + c0) = pack_bf16x2(g2[k].x, g2[k].y);
      const float gij[2] = {g1[k].x, g1[k].y};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = c0 + e, j = PREP_T * J + c;
        // dG[j][i]: gs holds tile (J, I), the tile itself when I == J
        if (j > i) dq[tri_index(i, j, BLK)] = 2.f * (gij[e] - gs[c][r]);
      }
    }
  }
}

// ---------------------------------------------------------------- fused kernel
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  if (!copy_ok(((src | bytes) & 15u) == 0 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0)) return;
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns into TMEM (the inverse of
// tmem_ld_32cols).
__device__ __forceinline__ void tmem_st_32cols(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 bf16 of row r, columns c0 .. c0+31 (c0 % 32 == 0), of a K-major operand
// staged by TMA: the 128-row x 64-column tile with 128-byte swizzle of stage
// c0/64 (16-byte chunk u of a row sits at chunk u ^ (r % 8)).
__device__ __forceinline__ void tile_row_bf16x32(uint32_t tile, int r, int c0, float* v) {
  const uint32_t rowp = tile + r * 128;
  const int u0 = (c0 & 63) >> 3;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w[4];
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "r"(rowp + (((u0 + u) ^ (r & 7)) << 4)));
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&w[h]);
      v[8 * u + 2 * h] = __low2float(b2);
      v[8 * u + 2 * h + 1] = __high2float(b2);
    }
  }
}
// 32 values of row r (0..31), columns 32h .. 32h+31, of a 32-row x 64-column
// bf16 box with 128-byte swizzle (16-byte chunk u of a row at u ^ (r % 8)),
// the layout a TMA store of that box reads.
__device__ __forceinline__ void box_row_bf16x32(uint32_t box, int r, int h, const float* v) {
  const uint32_t rowp = box + r * 128;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t w0 = pack_bf16x2(v[8 * u], v[8 * u + 1]), w1 = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
    const uint32_t w2 = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), w3 = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowp + (((4 * h + u) ^ (r & 7)) << 4)), "r"(w0),
                 "r"(w1), "r"(w2), "r"(w3)
                 : "memory");
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    cnp_pair_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmMN,
                    const __grid_constant__ CUtensorMap tmS, const __grid_constant__ PairSegs sg, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* dAs = reinterpret_cast<float*>(smem);                // acc1 rows after P3 (over the ring)
  float* dqs = reinterpret_cast<float*>(smem + REGION0);      // this CTA's four bands of the block's dq
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + REGION0 + DQ_BYTES);
  // bars: full[STAGES] (leader), empty[STAGES], acc, dq
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 2);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* tt = reinterpret_cast<float*>(smem + REGION0 + DQ_BYTES + 256) + (threadIdx.x >> 5) * 32 * TT_LD;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = tc2::cluster_rank();
  const bool leader = rank == 0;
  const uint32_t smem_base = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = STAGES, ACC = 2 * STAGES, DQ = 2 * STAGES + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(FULL + s), 1);
      mbar_init(bar(EMPTY + s), 1);
    }
    mbar_init(bar(ACC), 1);
    mbar_init(bar(DQ), 1);
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
  const int nph = 3;
  const int slot0 = 2 * p.nblk + pair * SKINDS;  // matrix index of this pair's S
  // shared-memory addresses of acc1's rows in both CTAs of the pair
  const uint32_t dA_cl0 = tc2::map_to_rank(smem_base, 0), dA_cl1 = tc2::map_to_rank(smem_base, 1);

  // ring state (the producer and the MMA issuer each keep their own copy),
  // carried across phases and blocks; every block issues a multiple of
  // STAGES chunks, so each phase's last four chunks sit in stages 0..3
  int stage = 0;
  uint32_t ring_phase = 0;
  uint32_t acc_phase = 0, dq_phase = 0;

  auto phase_barrier = [&]() {
    fence_proxy_async_all();
    tc_fence_before();
    __syncwarp();
    tc2::cluster_sync();
    tc_fence_after();
  };

  const int quarter = warp & 3;
  const int lrow = quarter * 32 + lane;           // this thread's row of the CTA's half in the epilogues

  for (int blk = pair; blk < p.nblk; blk += npairs) {
    const int s = pair_seg_of(sg, blk);
    const int lt = blk - sg.start[s];
    const int mQ = blk, mG = p.nblk + blk;
    float* dq_g = static_cast<float*>(sg.out[s]) + int64_t(lt) * TRI;

    if (threadIdx.x == 0 && !*s_abort) {
      // this CTA's half of dq (2 (dG - dG^T) from the prep) into shared memory
      bulk_wait_read<0>();  // the previous block's store has read the staging buffer
      mbar_arrive_expect_tx(bar(DQ), DQ_BYTES);
      for (int b = 0, off = 0; b < 4; off += band_size(band_of(rank, b)), ++b)
        bulk_load(smem_u32(dqs + off), dq_g + band_start(band_of(rank, b)), band_size(band_of(rank, b)) * 4,
                  bar(DQ));
    }

    for (int ph = 1; ph <= nph; ++ph) {
      const int nch = phase_chunks(ph);
      if (warp == 0) {
        if (lane == 0 && !*s_abort) {
          // ---------------- TMA producer
          for (int c = 0; c < nch; ++c) {
            if (!mbar_wait(bar(EMPTY + stage), ring_phase ^ 1u, DERR_GEMM_WAIT)) {
              *s_abort = 1;
              break;
            }
            const int type = chunk_type(ph, c);
            const int k = (c & 3) * CH;
            const uint32_t full_leader = tc2::map_to_rank(bar(FULL + stage), 0);
            const uint32_t sa = smem_base + stage * STAGE_BYTES, sb = sa + TILE_BYTES;
            if (leader) mbar_arrive_expect_tx(bar(FULL + stage), type == C_QQ ? 2 * TILE_BYTES : 2 * STAGE_BYTES);
            // this CTA's rows (K-major) or columns (MN-major, rows k .. k+63) of matrix m
            auto rows = [&](uint32_t dst, int m) {
              tc2::tma_load_2d_pair(dst, &tmK, full_leader, k, m * BLK + int(rank) * HALF);
            };
            auto cols = [&](uint32_t dst, int m) {
              tc2::tma_load_2d_pair(dst, &tmMN, full_leader, int(rank) * HALF, m * BLK + k);
              tc2::tma_load_2d_pair(dst + CH * 128, &tmMN, full_leader, int(rank) * HALF + CH, m * BLK + k);
            };
            switch (type) {
              case C_QQ: rows(sa, mQ); break;
              case C_H_GC: rows(sa, slot0 + KH); cols(sb, mG); break;
              case C_G_S: rows(sa, mG); rows(sb, slot0 + KS); break;
              case C_DS_Q: rows(sa, slot0 + KDS); rows(sb, mQ); break;
              default: cols(sa, mQ); cols(sb, slot0 + KDS); break;  // C_QC_DSC
            }
            if (++stage == STAGES) { stage = 0; ring_phase ^= 1u; }
          }
        }
      } else if (warp == 1) {
        if (leader && lane == 0 && !*s_abort) {
          // ---------------- MMA issuer (leader, for both CTAs)
          const uint32_t acc0 = tmem_base, acc1 = tmem_base + BLK;
          bool ok = true;
          for (int c = 0; c < nch; ++c) {
            if (!mbar_wait(bar(FULL + stage), ring_phase, DERR_GEMM_WAIT)) {
              *s_abort = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const int type = chunk_type(ph, c);
            const uint32_t sa = smem_base + stage * STAGE_BYTES, sb = sa + TILE_BYTES;
            const bool a_mn = type == C_QC_DSC;
            const bool b_mn = type == C_H_GC || type == C_QC_DSC;
            const uint32_t id = a_mn ? p.idesc_mnmn : (b_mn ? p.idesc_kmn : p.idesc_kk);
#pragma unroll
            for (int kk = 0; kk < CH / UMMA_K; ++kk) {
              const uint64_t da = a_mn ? smem_desc_sw128(sa + kk * (UMMA_K * 128), CH * 128, 1024)
                                       : smem_desc_sw128(sa + kk * 32, 16, 1024);
              const uint64_t db = type == C_QQ ? da
                                  : b_mn       ? smem_desc_sw128(sb + kk * (UMMA_K * 128), CH * 128, 1024)
                                               : smem_desc_sw128(sb + kk * 32, 16, 1024);
              const uint32_t fresh = ((c & 3) == 0 && kk == 0) ? 0u : 1u;  // 0: overwrite
              switch (type) {
                case C_QQ:
                case C_H_GC: tc2::mma_pair(acc0, da, db, id, fresh); break;
                case C_G_S: tc2::mma_pair(acc1, da, db, id, fresh); break;
                default: tc2::mma_pair(acc1, da, db, id, 1u); break;  // P3 adds to 2 dG S^T
              }
            }
            tc2::commit_pair(bar(EMPTY + stage));
            if (++stage == STAGES) { stage = 0; ring_phase ^= 1u; }
          }
          if (ok) tc2::commit_pair(bar(ACC));
        }
      } else {
        // ---------------- epilogue of phase ph (this CTA's 128 rows)
        bool ok = !*s_abort && mbar_wait(bar(ACC), acc_phase, DERR_GEMM_WAIT);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          if (lane == 0) *s_abort = 1;
        } else {
          tc_fence_after();
          const uint32_t t0 = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
          // E1 and E2 stage their bf16 rows in 32-row x 64-column boxes and
          // write them with TMA stores: the B tile of ring stage `quarter` is
          // free then (P1 loads only A tiles; P2's last B tiles, S, are read)
          const uint32_t stg = smem_base + quarter * STAGE_BYTES + TILE_BYTES;
          const int grow = int(rank) * HALF + quarter * 32;  // this warp's first row of a slot matrix
          float v0[32], v1[32], w[32];
          // 64 columns per step: the TMEM loads of a step share one round trip
          for (int c0 = 0; c0 < BLK; c0 += 64) {
            const uint32_t tileA = smem_base + (c0 >> 6) * STAGE_BYTES;
            if (ph <= 2) {
              if (lane == 0) bulk_wait_read<1>();  // the boxes of two steps ago have been read
              __syncwarp();
            }
            if (ph == 1) {
              // S = -acc0;  H^T = S - 2Q; Q from P1's A tiles
              float a1[32];
              tmem_ld_32cols_x2(t0 + c0, t0 + c0 + 32, v0, a1);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int cc = c0 + 32 * h;
                float* a = h ? a1 : v0;
                tile_row_bf16x32(tileA, lrow, cc, w);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                  a[e] = -a[e];
                  v1[e] = a[e] - 2.f * w[e];
                }
                const uint32_t bS = stg + ((c0 >> 6) & 1) * 2 * EPI_BOX;
                box_row_bf16x32(bS, lane, h, a);
                box_row_bf16x32(bS + EPI_BOX, lane, h, v1);
              }
              fence_async_smem();
              __syncwarp();
              if (lane == 0) {
                const uint32_t bS = stg + ((c0 >> 6) & 1) * 2 * EPI_BOX;
                tma_store_2d(&tmS, bS, c0, (slot0 + KS) * BLK + grow);
                tma_store_2d(&tmS, bS + EPI_BOX, c0, (slot0 + KH) * BLK + grow);
                bulk_commit();
              }
            } else if (ph == 2) {
              // dS = 2dG + acc0 + acc1 (a bf16 operand; dG from P2's A tiles); acc1 <- 2 acc1
#pragma unroll 1
              for (int h = 0; h < 2; ++h) {
                const int cc = c0 + 32 * h;
                tmem_ld_32cols_x2(t0 + cc, t0 + BLK + cc, v0, v1);
                tile_row_bf16x32(tileA, lrow, cc, w);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                  v0[e] = (2.f * w[e] + v0[e]) + v1[e];
                  v1[e] = 2.f * v1[e];
                }
                box_row_bf16x32(stg + ((c0 >> 6) & 1) * EPI_BOX, lane, h, v0);
                tmem_st_32cols(t0 + BLK + cc, v1);
              }
              fence_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&tmS, stg + ((c0 >> 6) & 1) * EPI_BOX, c0, (slot0 + KDS) * BLK + grow);
                bulk_commit();
              }
            } else {
              // acc1 = dA - 2dG for the fold (padded rows: conflict-free transposed reads)
              tmem_ld_32cols_x2(t0 + BLK + c0, t0 + BLK + c0 + 32, v0, v1);
              float* d = dAs + lrow * DA_LD + c0;
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                d[e] = v0[e];
                d[32 + e] = v1[e];
              }
            }
          }
          // the slot rows are complete in global memory before the phase barrier
          if (lane == 0) bulk_wait_all();
          __syncwarp();
        }
      }
      acc_phase ^= 1u;
      phase_barrier();
    }

    {
      // ---------------- F: this CTA's four bands of dq
      bool ok = !*s_abort && mbar_wait(bar(DQ), dq_phase, DERR_GEMM_WAIT);
      dq_phase ^= 1u;
      if (!ok) *s_abort = 1;
      __syncwarp();
      if (!*s_abort) {
        // Warp w folds tiles w, w + 6, w + 12 of this CTA's 18 (band I, tile
        // column J >= I).  Lane l holds column j = 32J + l.  Every load reads
        // one row with the lanes on consecutive columns (one request per warp,
        // local or from the partner CTA): a[r] = acc1[32I + r][j] and u[r] =
        // acc1[32J + r][32I + l]; u is transposed through the warp's own
        // padded tile, so lane l gets acc1[j][32I + r].  All 64 loads are
        // issued before use.
        for (int tile = warp; tile < 18; tile += NUM_THREADS / 32) {
          int b = 0, rest = tile, off = 0;
          while (rest >= BANDS - band_of(rank, b)) {
            rest -= BANDS - band_of(rank, b);
            off += band_size(band_of(rank, b));
            ++b;
          }
          const int I = band_of(rank, b), J = I + rest;
          const int i0 = 32 * I, j = 32 * J + lane;
          const int j0 = 32 * J;
          const uint32_t rowI = (i0 < HALF ? dA_cl0 : dA_cl1) + uint32_t((i0 & (HALF - 1)) * DA_LD + j) * 4u;
          const uint32_t rowJ = (j0 < HALF ? dA_cl0 : dA_cl1) + uint32_t((j0 & (HALF - 1)) * DA_LD + i0 + lane) * 4u;
          float a[32], t[32];
#pragma unroll
          for (int r = 0; r < 32; ++r) a[r] = ld_cluster_f32(rowI + uint32_t(r * DA_LD) * 4u);
#pragma unroll
          for (int r = 0; r < 32; ++r) t[r] = ld_cluster_f32(rowJ + uint32_t(r * DA_LD) * 4u);
#pragma unroll
          for (int r = 0; r < 32; ++r) tt[r * TT_LD + lane] = t[r];
          __syncwarp();
#pragma unroll
          for (int r = 0; r < 32; ++r) t[r] = tt[lane * TT_LD + r];
          __syncwarp();
          const int base = off - band_start(I);  // dqs index of entry k is base + k
#pragma unroll
          for (int r = 0; r < 32; ++r) {
            const int i = i0 + r;
            if (j > i) dqs[base + static_cast<int>(tri_index(i, j, BLK))] += a[r] - t[r];
          }
        }
      }
      fence_proxy_async_all();
      __syncthreads();
      tc2::cluster_sync();  // both CTAs are done reading each other's rows; staging complete
      if (threadIdx.x == 0 && !*s_abort) {
        for (int b = 0, off = 0; b < 4; off += band_size(band_of(rank, b)), ++b)
          bulk_store(dq_g + band_start(band_of(rank, b)), smem_u32(dqs + off), band_size(band_of(rank, b)) * 4);
        bulk_commit();
      }
    }
  }

  if (threadIdx.x == 0) bulk_wait_all();
  if (*s_abort && threadIdx.x == 0) {
    // give copies already issued time to land before the block leaves
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < 100000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  tc2::cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512) : "memory");
  }
  tc2::cluster_sync();
}

}  // namespace cnp2
}  // namespace poetx
