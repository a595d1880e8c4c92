// Host side of the batched GEMM: tensor-map encoding, tile-shape choice,
// split-K sizing and launch of the tcgen05 or SIMT back end.
#pragma once

#include <cudaTypedefs.h>

#include <mutex>

#include "gemm.cuh"
#include "gemm2sm.cuh"

namespace poetx {

// cuTensorMapEncodeTiled from the driver, fetched through the runtime so the
// library links against cudart only.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

inline int sm_count(int device) {
  static int counts[64] = {0};
  if (device < 0 || device >= 64) return 148;
  if (counts[device] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || v <= 0) v = 148;
    counts[device] = v;
  }
  return counts[device];
}

// 2-D tensor map over a row-major view with a 128-byte swizzled box of
// (box_inner elements = 128 bytes) x box_outer rows.
inline bool encode_map(CUtensorMap* map, const Operand2D& op, int box_outer) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const int esz = elem_size(op.et);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(op.cols), static_cast<cuuint64_t>(op.rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(op.ld) * esz};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, op.et == ET_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                   const_cast<void*>(op.ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, bool TF32, bool B_RES>
cudaError_t launch_tc_typed(const GemmDesc& g, cudaStream_t st, int device) {
  using C = tc::Cfg<BN, TF32, B_RES>;
  // tf32 operands are read as K-major tiles only (see nt_desc in poetx.cu).
  if (TF32 && (g.A.mn_major || g.B.mn_major)) return cudaErrorNotSupported;
  if (g.A.et != g.B.et) return cudaErrorInvalidValue;
  // the epilogue reads addends and writes full 32-column chunks as 16-byte vectors
  auto vec_ok = [](const AddDesc& a) {
    return !a.ptr || ((reinterpret_cast<uintptr_t>(a.ptr) & 15u) == 0 && a.ld % 4 == 0 && a.batch_stride % 4 == 0);
  };
  if (!vec_ok(g.add1) || !vec_ok(g.add2)) return cudaErrorInvalidValue;
  {
    const int v = g.C.et == ET_BF16 ? 8 : 4;
    if ((reinterpret_cast<uintptr_t>(g.C.ptr) & 15u) != 0 || (reinterpret_cast<uintptr_t>(g.C.ptr2) & 15u) != 0 ||
        g.C.ld % v != 0 || g.C.batch_stride % v != 0 || g.C.split_stride % v != 0)
      return cudaErrorInvalidValue;
    for (const ExtraOut& x : g.ex) {
      if (!x.ptr) continue;
      if ((reinterpret_cast<uintptr_t>(x.ptr) & 15u) != 0 || x.ld % 4 != 0 || x.batch_stride % 4 != 0)
        return cudaErrorInvalidValue;
      if (x.add && ((reinterpret_cast<uintptr_t>(x.add) & 15u) != 0 || x.add_ld % 4 != 0 || x.add_bs % 4 != 0))
        return cudaErrorInvalidValue;
    }
  }
  static bool attr_set[64] = {false};
  if (device >= 0 && device < 64 && !attr_set[device]) {
    cudaError_t e =
        cudaFuncSetAttribute(tc::gemm_kernel<BN, TF32, B_RES>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[device] = true;
  }
  CUtensorMap ma, mb, mc;
  if (!encode_map(&ma, g.A, g.A.mn_major ? C::CH : tc::BM)) return cudaErrorInvalidValue;
  if (!encode_map(&mb, g.B, g.B.mn_major ? C::CH : BN)) return cudaErrorInvalidValue;
  tc::Params p;
  // TMA-store epilogue: plain output (no addends, extra outputs, split pointer
  // or diagonal) described by a 2-D view; boxes of 32 rows x 128 bytes.
  const int c_esz = elem_size(g.C.et);
  const bool plain_out = g.C.view_rows > 0 && !g.add1.ptr && !g.add2.ptr && !g.ex[0].ptr && !g.ex[1].ptr &&
                         !g.C.ptr2 && g.diag == 0.f;
  // rows past M inside a 32-row box must fall outside the view (TMA clips
  // them) unless M is a whole number of boxes
  const bool rows_ok = g.M % 32 == 0 || (g.C.b_row == 0 && g.C.s_row == 0 && g.M == g.C.view_rows);
  p.tma_store = plain_out && rows_ok && (reinterpret_cast<uintptr_t>(g.C.ptr) & 15u) == 0 &&
                (g.C.ld * c_esz) % 16 == 0;
  p.c_brow = g.C.b_row;
  p.c_bcol = g.C.b_col;
  p.c_srow = g.C.s_row;
  if (p.tma_store) {
    Operand2D cv;
    cv.ptr = g.C.ptr;
    cv.et = g.C.et;
    cv.rows = g.C.view_rows;
    cv.cols = g.C.view_cols;
    cv.ld = g.C.ld;
    if (!encode_map(&mc, cv, 32)) return cudaErrorInvalidValue;
  } else {
    mc = ma;  // unused
  }
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.batch = g.batch;
  p.splits = g.splits;
  const int nkb = (g.K + C::CH - 1) / C::CH;
  const int kb_per = (nkb + g.splits - 1) / g.splits;
  p.k_per_split = kb_per * C::CH;
  p.tiles_m = (g.M + tc::BM - 1) / tc::BM;
  p.tiles_n = (g.N + BN - 1) / BN;
  p.a_mn = g.A.mn_major;
  p.b_mn = g.B.mn_major;
  p.a_brow = static_cast<int>(g.A.b_row);
  p.a_bcol = static_cast<int>(g.A.b_col);
  p.b_brow = static_cast<int>(g.B.b_row);
  p.b_bcol = static_cast<int>(g.B.b_col);
  const uint32_t fmt = TF32 ? 2u : 1u;
  p.idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | (static_cast<uint32_t>(g.A.mn_major) << 15) |
            (static_cast<uint32_t>(g.B.mn_major) << 16) | (static_cast<uint32_t>(BN >> 3) << 17) |
            (static_cast<uint32_t>(tc::BM >> 4) << 24);
  // K-major: the K step of one MMA is 32 bytes inside the 128-byte row; the
  // leading offset is unused.  MN-major: one MMA spans UMMA_K rows of 128
  // bytes; 128-byte MN chunks sit one box (CH rows x 128 B) apart.
  p.a_kstep = g.A.mn_major ? C::UMMA_K * 128 : 32;
  p.b_kstep = g.B.mn_major ? C::UMMA_K * 128 : 32;
  p.a_lbo = g.A.mn_major ? C::CH * 128 : 16;
  p.b_lbo = g.B.mn_major ? C::CH * 128 : 16;
  p.epi = make_epi(g);
  const int total = g.batch * g.splits * p.tiles_m * p.tiles_n;
  const int grid = total < sm_count(device) ? total : sm_count(device);
  if (grid <= 0) return cudaSuccess;
  if (B_RES && p.k_per_split > C::MAX_KB_RES * C::CH) return cudaErrorInvalidValue;
  tc::gemm_kernel<BN, TF32, B_RES><<<grid, tc::NUM_THREADS, C::SMEM_BYTES, st>>>(ma, mb, mc, p);
  return cudaGetLastError();
}

// The N tile: the widest of 256/128/64 that divides N (N is a multiple of 64
// on the tensor-core path).
inline int choose_bn(int N) {
  if (N % 256 == 0) return 256;
  if (N % 128 == 0) return 128;
  return 64;
}

// B stays resident when its whole K-range fits the resident area and enough
// M-tiles share it (block-diagonal products: K = N = b, M = tokens).
template <int BN, bool TF32>
cudaError_t launch_tc_bn(const GemmDesc& g, cudaStream_t st, int device) {
  using CR = tc::Cfg<BN, TF32, true>;
  const int tiles_m = (g.M + tc::BM - 1) / tc::BM;
  const int nkb = (g.K + CR::CH - 1) / CR::CH;
  const bool resident = g.splits == 1 && nkb <= CR::MAX_KB_RES && tiles_m >= 4;
  return resident ? launch_tc_typed<BN, TF32, true>(g, st, device) : launch_tc_typed<BN, TF32, false>(g, st, device);
}

inline cudaError_t launch_tc(const GemmDesc& g, cudaStream_t st, int device) {
  const bool tf32 = g.A.et == ET_F32;
  int bn = choose_bn(g.N);
  // Small batched products (the CNP blocks) fill few SMs with 256-wide tiles:
  // halve the tile width when that leaves more than a quarter of the SMs idle.
  if (bn == 256) {
    const int64_t tiles = int64_t(g.batch) * g.splits * ((g.M + tc::BM - 1) / tc::BM) * (g.N / 256);
    if (4 * tiles < 3 * int64_t(sm_count(device))) bn = 128;
  }
  switch (bn) {
    case 256: return tf32 ? launch_tc_bn<256, true>(g, st, device) : launch_tc_bn<256, false>(g, st, device);
    case 128: return tf32 ? launch_tc_bn<128, true>(g, st, device) : launch_tc_bn<128, false>(g, st, device);
    default: return tf32 ? launch_tc_bn<64, true>(g, st, device) : launch_tc_bn<64, false>(g, st, device);
  }
}

inline cudaError_t launch_simt(const GemmDesc& g, cudaStream_t st) {
  simt::Params p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.splits = g.splits;
  const int nkb = (g.K + simt::TK - 1) / simt::TK;
  p.k_per_split = ((nkb + g.splits - 1) / g.splits) * simt::TK;
  p.a = static_cast<const float*>(g.A.ptr);
  p.a_rows = g.A.rows;
  p.a_cols = g.A.cols;
  p.a_ld = g.A.ld;
  p.a_brow = g.A.b_row;
  p.a_bcol = g.A.b_col;
  p.a_mn = g.A.mn_major;
  p.b = static_cast<const float*>(g.B.ptr);
  p.b_rows = g.B.rows;
  p.b_cols = g.B.cols;
  p.b_ld = g.B.ld;
  p.b_brow = g.B.b_row;
  p.b_bcol = g.B.b_col;
  p.b_mn = g.B.mn_major;
  p.epi = make_epi(g);
  dim3 grid((g.N + simt::TN - 1) / simt::TN, (g.M + simt::TM - 1) / simt::TM, g.batch * g.splits);
  if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
  simt::gemm_kernel<<<grid, simt::THREADS, 0, st>>>(p);
  return cudaGetLastError();
}

// The CTA-pair kernel takes plain bf16 products with one batch, no split,
// K-major A, N a multiple of 256 and a TMA-store output view (the W0 GEMMs).
inline bool pair_eligible(const GemmDesc& g) {
  return g.A.et == ET_BF16 && g.B.et == ET_BF16 && !g.A.mn_major && g.batch == 1 && g.splits == 1 &&
         g.N % tc2::BN == 0 && g.K % tc2::CH == 0 && g.M >= 2 * tc::BM && g.C.et == ET_BF16 &&
         g.C.view_rows > 0 && g.C.b_row == 0 && g.C.b_col == 0 && !g.add1.ptr && !g.add2.ptr && !g.ex[0].ptr &&
         !g.ex[1].ptr && !g.C.ptr2 && g.diag == 0.f && (reinterpret_cast<uintptr_t>(g.C.ptr) & 15u) == 0 &&
         (g.C.ld * 2) % 16 == 0 && g.A.b_row == 0 && g.A.b_col == 0 && g.B.b_row == 0 && g.B.b_col == 0;
}

// Raster of the pair GEMM: groups of 16 N panels (256 columns of B, i.e. of
// the weight, each), N fastest inside a group, so the pairs of a wave share
// the token panel they stream while the group's weight panels are re-read
// from L2 for every token panel.  Measured in the 8B block step against
// groups of 4-64 panels along either dimension: 16 weight panels took the
// least time (W0 GEMM stage -1.1 to -2.7% against 8 token panels) and cut
// the DRAM reads of the [16384 x 4096] x [4096 x 14336] product from 1.23
// to 1.01 GB and of its dU product from 2.88 to 2.25 GB.
inline void choose_raster(tc2::Params& p) {
  p.group_n = 1;
  p.group = p.tiles_n < 16 ? p.tiles_n : 16;
}

inline cudaError_t launch_tc_pair(const GemmDesc& g, cudaStream_t st, int device) {
  static bool attr_set[64] = {false};
  if (device >= 0 && device < 64 && !attr_set[device]) {
    cudaError_t e =
        cudaFuncSetAttribute(tc2::gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc2::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[device] = true;
  }
  CUtensorMap ma, mb, mc;
  if (!encode_map(&ma, g.A, 128)) return cudaErrorInvalidValue;
  if (!encode_map(&mb, g.B, g.B.mn_major ? tc2::CH : 128)) return cudaErrorInvalidValue;
  Operand2D cv;
  cv.ptr = g.C.ptr;
  cv.et = ET_BF16;
  cv.rows = g.C.view_rows;
  cv.cols = g.C.view_cols;
  cv.ld = g.C.ld;
  if (!encode_map(&mc, cv, 32)) return cudaErrorInvalidValue;
  tc2::Params p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.tiles_m = (g.M + tc2::BM - 1) / tc2::BM;
  p.tiles_n = g.N / tc2::BN;
  p.b_mn = g.B.mn_major;
  p.idesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(g.B.mn_major) << 16) |
            (static_cast<uint32_t>(tc2::BN >> 3) << 17) | (static_cast<uint32_t>(tc2::BM >> 4) << 24);
  p.b_kstep = g.B.mn_major ? tc2::UMMA_K * 128 : 32;
  p.b_lbo = g.B.mn_major ? tc2::CH * 128 : 16;
  p.alpha = g.alpha;
  choose_raster(p);
  const int tiles = p.tiles_m * p.tiles_n;
  const int pairs = sm_count(device) / 2;
  const int grid = 2 * (tiles < pairs ? tiles : pairs);
  if (grid <= 0) return cudaSuccess;
  tc2::gemm_pair_kernel<<<grid, tc2::NUM_THREADS, tc2::SMEM_BYTES, st>>>(ma, mb, mc, p);
  return cudaGetLastError();
}

// Tensor cores for bf16 and tf32 operands, FFMA for an all-fp32 layer.
inline cudaError_t launch_gemm(const GemmDesc& g, bool tensor_cores, cudaStream_t st, int device) {
  if (!tensor_cores) return launch_simt(g, st);
  return pair_eligible(g) ? launch_tc_pair(g, st, device) : launch_tc(g, st, device);
}

}  // namespace poetx
