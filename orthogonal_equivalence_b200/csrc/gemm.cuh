// Batched, split-K GEMM used by every contraction of the POET-X layer:
//   C[t][s] = alpha * A_t(K-range s) B_t(K-range s) + beta1 X1 + beta2 X2 + diag I
// where t runs over a batch (the b x b blocks of Diag(G_1..G_k)) and s over
// K-splits.  Two back ends consume the same description:
//   * tc_gemm  : tcgen05 tensor cores (kind::f16 with bf16 operands, or
//                kind::tf32 with fp32 operands), TMA-fed, fp32 accumulators in
//                TMEM, persistent and warp-specialised;
//   * simt_gemm: fp32 FFMA, for the all-fp32 layer (tcgen05 has no fp32 kind).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace poetx {

enum ElemType : int { ET_F32 = 0, ET_BF16 = 1 };

inline int elem_size(int et) { return et == ET_BF16 ? 2 : 4; }

// A 2-D row-major view of an operand (element units).  Element (mn, k) of
// batch t sits at view coordinate
//   K-major  (mn_major == false): row = mn + t*b_row, col = k + t*b_col
//   MN-major (mn_major == true) : row = k + t*b_row,  col = mn + t*b_col
// Coordinates outside [0,rows) x [0,cols) read as zero.
struct Operand2D {
  const void* ptr = nullptr;
  int et = ET_BF16;
  int64_t rows = 0, cols = 0, ld = 0;
  bool mn_major = false;
  int64_t b_row = 0, b_col = 0;
};

struct OutDesc {
  void* ptr = nullptr;
  int et = ET_BF16;
  int64_t ld = 0;            // row stride
  int64_t batch_stride = 0;  // element offset per batch index
  int64_t split_stride = 0;  // element offset per K-split (partial sums)
  void* ptr2 = nullptr;      // batches t >= split_batch go to ptr2 (as batch t - split_batch)
  int split_batch = 1 << 30;
  // 2-D view of the output for TMA tensor stores (view_rows == 0: plain
  // stores).  Element (r, n) of batch t, split s is at view row
  // r + t*b_row + s*s_row, column n + t*b_col.
  int64_t view_rows = 0, view_cols = 0;
  int b_row = 0, b_col = 0, s_row = 0;
};

struct AddDesc {
  const float* ptr = nullptr;  // fp32, indexed like the output
  int64_t ld = 0, batch_stride = 0;
  float beta = 0.f;
};

// Extra fp32 output written from the final value v of the main output:
//   out = cv * v + ca * add,  stored at (r, n) or, transposed, at (n, r).
struct ExtraOut {
  float* ptr = nullptr;
  int64_t ld = 0, batch_stride = 0;
  float cv = 1.f;
  const float* add = nullptr;
  int64_t add_ld = 0, add_bs = 0;
  float ca = 0.f;
  int transposed = 0;
};

struct GemmDesc {
  int M = 0, N = 0, K = 0;
  int batch = 1, splits = 1;
  Operand2D A, B;
  OutDesc C;
  float alpha = 1.f;
  AddDesc add1, add2;
  float diag = 0.f;
  ExtraOut ex[2];
};

// ------------------------------------------------------------------ epilogue
struct EpiParams {
  int M, N;
  void* c;
  void* c2;
  int c_split;
  int c_et;
  int64_t ldc, c_bs, c_ss;
  float alpha;
  const float* x1;
  int64_t x1_ld, x1_bs;
  float beta1;
  const float* x2;
  int64_t x2_ld, x2_bs;
  float beta2;
  float diag;
  ExtraOut ex[2];
};

inline EpiParams make_epi(const GemmDesc& g) {
  EpiParams e;
  e.M = g.M;
  e.N = g.N;
  e.c = g.C.ptr;
  e.c2 = g.C.ptr2;
  e.c_split = g.C.split_batch;
  e.c_et = g.C.et;
  e.ldc = g.C.ld;
  e.c_bs = g.C.batch_stride;
  e.c_ss = g.C.split_stride;
  e.alpha = g.alpha;
  e.x1 = g.add1.ptr;
  e.x1_ld = g.add1.ld;
  e.x1_bs = g.add1.batch_stride;
  e.beta1 = g.add1.beta;
  e.x2 = g.add2.ptr;
  e.x2_ld = g.add2.ld;
  e.x2_bs = g.add2.batch_stride;
  e.beta2 = g.add2.beta;
  e.diag = g.diag;
  e.ex[0] = g.ex[0];
  e.ex[1] = g.ex[1];
  return e;
}

// alpha * acc + beta1 X1 + beta2 X2 + diag I at (r, n) of batch t
__device__ __forceinline__ float epi_value(const EpiParams& e, float acc, int t, int64_t r, int64_t n) {
  float v = e.alpha * acc;
  if (e.x1) v += e.beta1 * e.x1[t * e.x1_bs + r * e.x1_ld + n];
  if (e.x2) v += e.beta2 * e.x2[t * e.x2_bs + r * e.x2_ld + n];
  if (r == n) v += e.diag;
  return v;
}

// Element offset of the main output for batch t / split sp (and the base
// pointer that batch goes to).
__device__ __forceinline__ int64_t epi_out_base(const EpiParams& e, int t, int sp, void*& base) {
  if (t >= e.c_split) {
    base = e.c2;
    t -= e.c_split;
  } else {
    base = e.c;
  }
  return t * e.c_bs + sp * e.c_ss;
}

// Extra outputs of one element with final value v.
__device__ __forceinline__ void epi_extra_scalar(const EpiParams& e, int t, int64_t r, int64_t n, float v) {
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const ExtraOut& x = e.ex[k];
    if (!x.ptr) continue;
    float o = x.cv * v;
    if (x.add) o += x.ca * x.add[t * x.add_bs + r * x.add_ld + n];
    x.ptr[t * x.batch_stride + (x.transposed ? n * x.ld + r : r * x.ld + n)] = o;
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ------------------------------------------------------------------ tcgen05 GEMM
namespace tc {

constexpr int BM = 128;
constexpr int NUM_THREADS = 192;  // warp 0: TMA, warp 1: MMA + TMEM owner, warps 2-5: epilogue
constexpr int GROUP_M = 16;       // M-tiles per raster group (L2 reuse of the B panel)

struct Params {
  int tma_store;  // 1: the epilogue writes C through shared memory with TMA stores
  int c_brow, c_bcol, c_srow;
  int M, N, K, batch, splits, k_per_split;
  int tiles_m, tiles_n;
  int a_mn, b_mn;
  int a_brow, a_bcol, b_brow, b_bcol;
  uint32_t idesc;
  uint32_t a_lbo, b_lbo, a_kstep, b_kstep;
  EpiParams epi;
};

// Two operand-feeding modes:
//  * streamed  (B_RES = false): every pipeline stage carries one K-block of A
//    and of B; tiles are dealt to the persistent CTAs round-robin, M-tiles
//    grouped GROUP_M at a time so a B panel is reused from L2;
//  * B-resident (B_RES = true): the whole K-range of the B tile (a b x b block
//    of Diag(G) for the block-diagonal products) is loaded once into shared
//    memory and kept while the CTA streams a contiguous run of M-tiles (token
//    tiles) of A through the stages; B is reloaded only when the block changes.
template <int BN, bool TF32, bool B_RES>
struct Cfg {
  static constexpr int ESZ = TF32 ? 4 : 2;
  static constexpr int CH = 128 / ESZ;  // elements per 128-byte swizzle row = K per stage
  static constexpr int UMMA_K = TF32 ? 8 : 16;
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = B_RES ? A_BYTES : A_BYTES + B_BYTES;
  static constexpr int STAGES = B_RES ? 4 : (BN == 256 ? 4 : (BN == 128 ? 6 : 8));
  static constexpr int MAX_KB_RES = B_RES ? (128 * 1024) / B_BYTES : 0;  // resident K-blocks of B
  static constexpr int TMEM_COLS = 2 * BN;  // double-buffered fp32 accumulator
  static constexpr int EPI_BOX = 32 * 128;       // one warp's 32-row x 128-byte output box
  static constexpr int EPI_BYTES = 4 * 2 * EPI_BOX;  // 4 epilogue warps, double-buffered
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + MAX_KB_RES * B_BYTES + EPI_BYTES + 1024 + 256;
};

// Streamed mode: round-robin tiles, GROUP_M-grouped raster inside each
// (batch, split).  B-resident mode: contiguous tiles, M fastest.
template <bool B_RES>
__device__ __forceinline__ void decode_tile(const Params& p, int tile, int& bt, int& sp, int& mt, int& nt) {
  const int per = p.tiles_m * p.tiles_n;
  const int bs = tile / per;
  int r = tile - bs * per;
  bt = bs / p.splits;
  sp = bs - bt * p.splits;
  if constexpr (B_RES) {
    nt = r / p.tiles_m;
    mt = r - nt * p.tiles_m;
  } else {
    const int group_span = GROUP_M * p.tiles_n;
    const int g = r / group_span;
    const int first_m = g * GROUP_M;
    const int gsize = min(p.tiles_m - first_m, GROUP_M);
    r -= g * group_span;
    mt = first_m + r % gsize;
    nt = r / gsize;
  }
}

// Tiles of this CTA: [t0, t1) with stride `step`.
template <bool B_RES>
__device__ __forceinline__ void tile_range(int total, int& t0, int& t1, int& step) {
  if constexpr (B_RES) {
    t0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * total / gridDim.x);
    t1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * total / gridDim.x);
    step = 1;
  } else {
    t0 = blockIdx.x;
    t1 = total;
    step = gridDim.x;
  }
}

template <int BN, bool TF32, bool B_RES>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, Params p) {
  using C = Cfg<BN, TF32, B_RES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::MAX_KB_RES * C::B_BYTES +
                                               C::EPI_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain, bfull, bempty
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 7);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t sB_res = smem_base + C::STAGES * C::STAGE_BYTES;  // resident B (B_RES only)
  const uint32_t sEpi = sB_res + C::MAX_KB_RES * C::B_BYTES;         // output staging boxes
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = C::STAGES, TFULL = 2 * C::STAGES, TEMPTY = 2 * C::STAGES + 2,
            DRAIN = 2 * C::STAGES + 4, BFULL = 2 * C::STAGES + 5, BEMPTY = 2 * C::STAGES + 6;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(FULL + s), 1);
      mbar_init(bar(EMPTY + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(TFULL + a), 1);
      mbar_init(bar(TEMPTY + a), 128);
    }
    mbar_init(bar(DRAIN), 1);
    mbar_init(bar(BFULL), 1);
    mbar_init(bar(BEMPTY), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int total = p.batch * p.splits * p.tiles_m * p.tiles_n;
  int t0, t1, tstep;
  tile_range<B_RES>(total, t0, t1, tstep);
  // key of the resident B tile: (batch, split, n-tile)
  auto b_key = [&](int bt, int sp, int nt) { return (bt * p.splits + sp) * p.tiles_n + nt; };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;  // per-stage bits for the abort drain
      int key_prev = -1;
      uint32_t bloads = 0;
      bool b_armed = false;
      bool ok = true;
      for (int tile = t0; tile < t1 && ok; tile += tstep) {
        int bt, sp, mt, nt;
        decode_tile<B_RES>(p, tile, bt, sp, mt, nt);
        const int kbeg = sp * p.k_per_split;
        const int kend = min(p.K, kbeg + p.k_per_split);
        const int nkb = (kend - kbeg + C::CH - 1) / C::CH;
        const int m0 = mt * BM, n0 = nt * BN;
        if constexpr (B_RES) {
          const int key = b_key(bt, sp, nt);
          if (key != key_prev) {
            // the previous resident B is free once the MMAs that read it are done
            if (bloads > 0 && !mbar_wait(bar(BEMPTY), (bloads - 1) & 1u, DERR_GEMM_WAIT)) { ok = false; break; }
            const uint32_t fb = bar(BFULL);
            mbar_arrive_expect_tx(fb, nkb * C::B_BYTES);
            b_armed = true;
            for (int kb = 0; kb < nkb; ++kb) {
              const int k = kbeg + kb * C::CH;
              const uint32_t sb = sB_res + kb * C::B_BYTES;
              if (!p.b_mn) {
                tma_load_2d(sb, &tmB, fb, k + bt * p.b_bcol, n0 + bt * p.b_brow);
              } else {
#pragma unroll
                for (int c = 0; c < BN / C::CH; ++c)
                  tma_load_2d(sb + c * (C::CH * 128), &tmB, fb, n0 + c * C::CH + bt * p.b_bcol, k + bt * p.b_brow);
              }
            }
            ++bloads;
            key_prev = key;
          }
        }
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(bar(EMPTY + stage), phase ^ 1u, DERR_GEMM_WAIT)) { ok = false; break; }
          const uint32_t fb = bar(FULL + stage);
          mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          const uint32_t sa = smem_base + stage * C::STAGE_BYTES;
          const int k = kbeg + kb * C::CH;
          if (!p.a_mn) {
            tma_load_2d(sa, &tmA, fb, k + bt * p.a_bcol, m0 + bt * p.a_brow);
          } else {
#pragma unroll
            for (int c = 0; c < BM / C::CH; ++c)
              tma_load_2d(sa + c * (C::CH * 128), &tmA, fb, m0 + c * C::CH + bt * p.a_bcol, k + bt * p.a_brow);
          }
          if constexpr (!B_RES) {
            const uint32_t sb = sa + C::A_BYTES;
            if (!p.b_mn) {
              tma_load_2d(sb, &tmB, fb, k + bt * p.b_bcol, n0 + bt * p.b_brow);
            } else {
#pragma unroll
              for (int c = 0; c < BN / C::CH; ++c)
                tma_load_2d(sb + c * (C::CH * 128), &tmB, fb, n0 + c * C::CH + bt * p.b_bcol, k + bt * p.b_brow);
            }
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the block exits.
        for (int s = 0; s < C::STAGES; ++s)
          if (armed & (1u << s)) mbar_wait(bar(FULL + s), (armed_phase >> s) & 1u, DERR_GEMM_WAIT);
        if (b_armed) mbar_wait(bar(BFULL), (bloads - 1) & 1u, DERR_GEMM_WAIT);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      int key_prev = -1;
      uint32_t bwaits = 0;
      bool ok = true;
      for (int tile = t0; tile < t1 && ok; tile += tstep, ++local) {
        int bt, sp, mt, nt;
        decode_tile<B_RES>(p, tile, bt, sp, mt, nt);
        const int kbeg = sp * p.k_per_split;
        const int kend = min(p.K, kbeg + p.k_per_split);
        const int nkb = (kend - kbeg + C::CH - 1) / C::CH;
        bool last_of_key = false;
        if constexpr (B_RES) {
          const int key = b_key(bt, sp, nt);
          if (key != key_prev) {
            if (!mbar_wait(bar(BFULL), bwaits & 1u, DERR_GEMM_WAIT)) { ok = false; break; }
            ++bwaits;
            key_prev = key;
          }
          if (tile + tstep >= t1) {
            last_of_key = true;
          } else {
            int bt2, sp2, mt2, nt2;
            decode_tile<B_RES>(p, tile + tstep, bt2, sp2, mt2, nt2);
            last_of_key = b_key(bt2, sp2, nt2) != key;
          }
        }
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(bar(TEMPTY + acc), acc_phase ^ 1u, DERR_GEMM_WAIT)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(bar(FULL + stage), phase, DERR_GEMM_WAIT)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * C::STAGE_BYTES;
          const uint32_t sb = B_RES ? sB_res + kb * C::B_BYTES : sa + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::CH / C::UMMA_K; ++kk) {
            const uint64_t da = smem_desc_sw128(sa + kk * p.a_kstep, p.a_lbo, 1024);
            const uint64_t db = smem_desc_sw128(sb + kk * p.b_kstep, p.b_lbo, 1024);
            tc_mma<TF32>(d_tmem, da, db, p.idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(bar(EMPTY + stage));
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(bar(TFULL + acc));
        if (B_RES && last_of_key) tc_commit(bar(BEMPTY));
      }
      // All MMAs issued by this thread have completed once DRAIN fires.
      tc_commit(bar(DRAIN));
      mbar_wait(bar(DRAIN), 0, DERR_GEMM_WAIT);
    }
  } else if (p.tma_store) {
    // ---------------- epilogue: TMEM -> registers -> swizzled smem box -> TMA store
    // Each warp owns TMEM lanes [32*quarter, +32) = 32 output rows; one box is
    // 32 rows x 128 bytes (64 bf16 or 32 fp32 columns), 128-byte swizzled:
    // the 16-byte chunk k of row i sits at slot k ^ (i & 7).
    const int quarter = warp & 3;
    const EpiParams& e = p.epi;
    const uint32_t my_boxes = sEpi + (warp - 2) * 2 * C::EPI_BOX;
    constexpr int CHO_BF16 = 64, CHO_F32 = 32;
    int buf = 0;
    int local = 0;
    for (int tile = t0; tile < t1; tile += tstep, ++local) {
      int bt, sp, mt, nt;
      decode_tile<B_RES>(p, tile, bt, sp, mt, nt);
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      bool ok = mbar_wait(bar(TFULL + acc), acc_phase, DERR_GEMM_WAIT);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int row0 = mt * BM + quarter * 32;
      const bool warp_rows = row0 < e.M;  // boxes past M (a b x b block smaller than the tile) are skipped
      const int vrow = row0 + bt * p.c_brow + sp * p.c_srow;
      const int cho = e.c_et == ET_BF16 ? CHO_BF16 : CHO_F32;
      const uint32_t tl = tmem_base + acc * BN + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += cho) {
        uint32_t w[32];  // one 128-byte output row of this lane
        if (e.c_et == ET_BF16) {
          float v[32], u[32];
          tmem_ld_32cols_x2(tl + c0, tl + c0 + 32, v, u);
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(e.alpha * v[2 * i], e.alpha * v[2 * i + 1]);
#pragma unroll
          for (int i = 0; i < 16; ++i) w[16 + i] = pack_bf16x2(e.alpha * u[2 * i], e.alpha * u[2 * i + 1]);
        } else {
          float v[32];
          tmem_ld_32cols(tl + c0, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(e.alpha * v[i]);
        }
        if (!warp_rows) continue;
        if (lane == 0) bulk_wait_read<1>();  // the store that last used this box has read it
        __syncwarp();
        const uint32_t box = my_boxes + buf * C::EPI_BOX;
        const uint32_t rowp = box + lane * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowp + ((k ^ (lane & 7)) << 4)),
                       "r"(w[4 * k]), "r"(w[4 * k + 1]), "r"(w[4 * k + 2]), "r"(w[4 * k + 3])
                       : "memory");
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmC, box, nt * BN + c0 + bt * p.c_bcol, vrow);
          bulk_commit();
        }
        buf ^= 1;
      }
      tc_fence_before();
      mbar_arrive(bar(TEMPTY + acc));
    }
    if (lane == 0) bulk_wait_all();
  } else {
    // ---------------- epilogue: TMEM -> registers -> global
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    const EpiParams& e = p.epi;
    int local = 0;
    for (int tile = t0; tile < t1; tile += tstep, ++local) {
      int bt, sp, mt, nt;
      decode_tile<B_RES>(p, tile, bt, sp, mt, nt);
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      bool ok = mbar_wait(bar(TFULL + acc), acc_phase, DERR_GEMM_WAIT);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int64_t r = static_cast<int64_t>(mt) * BM + quarter * 32 + lane;
      const bool row_ok = r < e.M;
      void* cbase;
      const int64_t obase = epi_out_base(e, bt, sp, cbase) + r * e.ldc;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float v[32];
        tmem_ld_32cols(tmem_base + acc * BN + c0 + (static_cast<uint32_t>(quarter * 32) << 16), v);
        const int64_t n0 = static_cast<int64_t>(nt) * BN + c0;
        if (!row_ok) continue;
        if (n0 + 32 <= e.N) {
          // alpha * acc + beta1 X1 + beta2 X2 + diag I; the addends are read
          // as 16-byte vectors (host guarantees 16-byte alignment)
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= e.alpha;
          if (e.x1) {
            const float4* xp = reinterpret_cast<const float4*>(e.x1 + bt * e.x1_bs + r * e.x1_ld + n0);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 a = __ldg(xp + q);
              v[4 * q] += e.beta1 * a.x;
              v[4 * q + 1] += e.beta1 * a.y;
              v[4 * q + 2] += e.beta1 * a.z;
              v[4 * q + 3] += e.beta1 * a.w;
            }
          }
          if (e.x2) {
            const float4* xp = reinterpret_cast<const float4*>(e.x2 + bt * e.x2_bs + r * e.x2_ld + n0);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 a = __ldg(xp + q);
              v[4 * q] += e.beta2 * a.x;
              v[4 * q + 1] += e.beta2 * a.y;
              v[4 * q + 2] += e.beta2 * a.z;
              v[4 * q + 3] += e.beta2 * a.w;
            }
          }
          if (e.diag != 0.f && r >= n0 && r < n0 + 32) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (r == n0 + i) v[i] += e.diag;
          }
          if (e.c_et == ET_BF16) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(cbase) + obase + n0);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(pack_bf16x2(v[8 * q + 0], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                  pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(cbase) + obase + n0);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const ExtraOut& x = e.ex[k];
            if (!x.ptr) continue;
            float o[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = x.cv * v[i];
            if (x.add) {
              const float4* ap = reinterpret_cast<const float4*>(x.add + bt * x.add_bs + r * x.add_ld + n0);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 a = __ldg(ap + q);
                o[4 * q] += x.ca * a.x;
                o[4 * q + 1] += x.ca * a.y;
                o[4 * q + 2] += x.ca * a.z;
                o[4 * q + 3] += x.ca * a.w;
              }
            }
            if (x.transposed) {
              // lanes hold consecutive rows r: each column n is one coalesced 128-byte row segment
              float* dst = x.ptr + bt * x.batch_stride + n0 * x.ld + r;
#pragma unroll
              for (int i = 0; i < 32; ++i) dst[i * x.ld] = o[i];
            } else {
              float4* dst = reinterpret_cast<float4*>(x.ptr + bt * x.batch_stride + r * x.ld + n0);
#pragma unroll
              for (int q = 0; q < 8; ++q) dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
            }
          }
        } else {
          // ragged last chunk: element by element (fully unrolled so v stays in registers)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (n0 + i < e.N) {
              const float o = epi_value(e, v[i], bt, r, n0 + i);
              if (e.c_et == ET_BF16)
                reinterpret_cast<__nv_bfloat16*>(cbase)[obase + n0 + i] = __float2bfloat16_rn(o);
              else
                reinterpret_cast<float*>(cbase)[obase + n0 + i] = o;
              epi_extra_scalar(e, bt, r, n0 + i, o);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(TEMPTY + acc));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace tc

// ------------------------------------------------------------------ SIMT fp32 GEMM
namespace simt {

constexpr int TM = 64, TN = 64, TK = 16, THREADS = 256;

struct Params {
  int M, N, K, splits, k_per_split;
  const float* a;
  int64_t a_rows, a_cols, a_ld, a_brow, a_bcol;
  int a_mn;
  const float* b;
  int64_t b_rows, b_cols, b_ld, b_brow, b_bcol;
  int b_mn;
  EpiParams epi;
};

__device__ __forceinline__ float load_op(const float* base, int64_t rows, int64_t cols, int64_t ld, int64_t brow,
                                         int64_t bcol, int mn_major, int t, int64_t mn, int64_t k) {
  int64_t row, col;
  if (mn_major) {
    row = k + t * brow;
    col = mn + t * bcol;
  } else {
    row = mn + t * brow;
    col = k + t * bcol;
  }
  if (row < 0 || row >= rows || col < 0 || col >= cols) return 0.f;
  return base[row * ld + col];
}

__global__ void __launch_bounds__(THREADS) gemm_kernel(Params p) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int bz = blockIdx.z;
  const int t = bz / p.splits;
  const int sp = bz - t * p.splits;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int kbeg = sp * p.k_per_split;
  const int kend = min(p.K, kbeg + p.k_per_split);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = kbeg; k0 < kend; k0 += TK) {
    for (int i = threadIdx.x; i < TK * TM; i += THREADS) {
      const int kk = i / TM, mm = i % TM;
      const int64_t mg = m0 + mm, kg = k0 + kk;
      As[kk][mm] = (mg < p.M && kg < kend)
                       ? load_op(p.a, p.a_rows, p.a_cols, p.a_ld, p.a_brow, p.a_bcol, p.a_mn, t, mg, kg)
                       : 0.f;
    }
    for (int i = threadIdx.x; i < TK * TN; i += THREADS) {
      const int kk = i / TN, nn = i % TN;
      const int64_t ng = n0 + nn, kg = k0 + kk;
      Bs[kk][nn] = (ng < p.N && kg < kend)
                       ? load_op(p.b, p.b_rows, p.b_cols, p.b_ld, p.b_brow, p.b_bcol, p.b_mn, t, ng, kg)
                       : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  const EpiParams& e = p.epi;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = m0 + ty * 4 + i;
    if (r >= e.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n >= e.N) continue;
      const float v = epi_value(e, acc[i][j], t, r, n);
      void* cbase;
      const int64_t o = epi_out_base(e, t, sp, cbase) + r * e.ldc + n;
      if (e.c_et == ET_BF16)
        reinterpret_cast<__nv_bfloat16*>(cbase)[o] = __float2bfloat16_rn(v);
      else
        reinterpret_cast<float*>(cbase)[o] = v;
      epi_extra_scalar(e, t, r, n, v);
    }
  }
}

}  // namespace simt
}  // namespace poetx
