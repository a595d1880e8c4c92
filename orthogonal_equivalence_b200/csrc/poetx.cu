// C ABI of the POET-X layer (declared in include/poetx.h): argument
// validation, workspace carving and the launch sequence of each call on the
// caller's stream.  The arithmetic lives in the kernels of gemm.cuh, perm.cuh
// and cnp.cuh.
//
// Source of the method: POET-X write-up (zhichai.net), sections 1 (input-
// centric layer), 2 (block-stochastic R, P), 3 (Cayley-Neumann blocks,
// packed triangle) and the merge_if_needed step of its API snippet.
#include <cstdint>
#include <cmath>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "poetx.h"
#include "cnp.cuh"
#include "gemm_host.cuh"
#include "perm.cuh"
#include "quant.cuh"
#include "adamw.cuh"
#include "cnp2sm.cuh"
#include "cnp2build.cuh"
#include "bdg2sm.cuh"

using namespace poetx;

namespace {

constexpr size_t kAlign = 256;
constexpr int kSplitSMs = 148;  // fixed split-K target (B200 SM count): sums do not depend on the device

inline size_t al(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int dtype_size(int32_t dt) { return dt == POETX_BF16 ? 2 : 4; }
inline int elem_type(int32_t dt) { return dt == POETX_BF16 ? ET_BF16 : ET_F32; }
// Widest rows the row-staging kernels take (one row of at most 200 KB in
// shared memory): n for the activation permutations (rows of the layer dtype),
// m also for the merge, whose reframing gather reads fp32 rows of length m.
constexpr int32_t kMaxM = 51200;
inline int32_t max_n(int32_t dt) { return dt == POETX_BF16 ? 102400 : 51200; }
// Token rows: GEMM row counts and TMA row coordinates are 32-bit.
constexpr int64_t kMaxT = 2147483647 - 256;

struct Carver {
  uint8_t* base;
  size_t cap, used = 0;
  Carver(void* b, size_t c) : base(static_cast<uint8_t*>(b)), cap(c) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(base);
    const uintptr_t r = (a + kAlign - 1) & ~uintptr_t(kAlign - 1);
    used = r - a;
  }
  template <typename T>
  T* take(size_t bytes) {
    T* p = reinterpret_cast<T*>(base + used);
    used += al(bytes);
    return p;
  }
  bool fits(size_t bytes) const { return used + al(bytes) <= cap; }
};

#define POETX_TRY(expr)                         \
  do {                                          \
    const poetx_status _s = (expr);             \
    if (_s != POETX_OK) return _s;              \
  } while (0)
#define POETX_CUDA_ERR(expr)                    \
  do {                                          \
    const cudaError_t _e = (expr);              \
    if (_e != cudaSuccess) return _e;           \
  } while (0)
#define POETX_CUDA(expr)                        \
  do {                                          \
    if ((expr) != cudaSuccess) {                \
      (void)cudaGetLastError();                 \
      return POETX_E_CUDA;                      \
    }                                           \
  } while (0)

poetx_status current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return POETX_E_CUDA;
  }
  static int cc[64] = {0};
  if (*dev < 0 || *dev >= 64) return POETX_E_ARCH;
  if (cc[*dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess) {
      (void)cudaGetLastError();
      return POETX_E_CUDA;
    }
    cc[*dev] = major * 10 + minor;
  }
  return cc[*dev] == 100 ? POETX_OK : POETX_E_ARCH;
}

poetx_status check_dtype_b(int32_t dtype, int32_t b) {
  if (dtype != POETX_FP32 && dtype != POETX_BF16) return POETX_E_DTYPE;
  if (b < 2) return POETX_E_SHAPE;
  if (dtype == POETX_BF16 && b % 64 != 0) return POETX_E_SHAPE;
  return POETX_OK;
}

poetx_status check_layer(const poetx_layer* L) {
  if (!L) return POETX_E_ARG;
  POETX_TRY(check_dtype_b(L->dtype, L->b));
  if (L->m <= 0 || L->n <= 0 || L->m % L->b != 0 || L->n % L->b != 0) return POETX_E_SHAPE;
  if (L->m > kMaxM || L->n > max_n(L->dtype)) return POETX_E_SHAPE;
  if (L->fold & ~POETX_FOLD_ALL) return POETX_E_ARG;
  const void* ptrs[] = {L->W, L->permR, L->permP, L->qR, L->qP, L->GR, L->GP};
  for (const void* p : ptrs) {
    if (!p) return POETX_E_ARG;
    if (!aligned16(p)) return POETX_E_ALIGN;
  }
  return POETX_OK;
}

poetx_status check_ptr(const void* p) {
  if (!p) return POETX_E_ARG;
  return aligned16(p) ? POETX_OK : POETX_E_ALIGN;
}


// ---------------------------------------------------------------- stage profiler
// When enabled (poetx_profile_begin), every kernel launch is bracketed by a
// pair of CUDA events on its stream, tagged with the stage it belongs to;
// poetx_profile_end sums the elapsed times per stage.
enum Stage : int {
  ST_PERMUTE = 0,
  ST_BLOCKDIAG,
  ST_W0,
  ST_DG,
  ST_CNP_GEMM,
  ST_CNP_ELEM,
  ST_REDUCE,
  ST_MERGE,
  ST_DEQUANT,
  ST_OPTIM,
  ST_BDG,
  ST_COUNT
};
const char* const kStageNames[ST_COUNT] = {"permute",  "blockdiag_gemm",  "w0_gemm",   "dg_gemm", "cnp_gemm",
                                           "cnp_elementwise", "dg_reduce", "merge", "dequant", "optimizer",
                                            "blockdiag_dg"};

struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  std::vector<std::pair<int, size_t>> recs;  // (stage, index of the start event)
  std::vector<std::pair<int, float>> done;   // (stage, ms) of the last finished session
};

Profiler& profiler() {
  static Profiler p;
  return p;
}

struct Prof {
  int stage;
  cudaStream_t st;
  size_t idx = SIZE_MAX;
  Prof(int s, cudaStream_t stream) : stage(s), st(stream) {
    Profiler& P = profiler();
    std::lock_guard<std::mutex> g(P.mu);
    if (!P.on) return;
    while (P.used + 2 > P.pool.size()) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) {
        (void)cudaGetLastError();
        return;
      }
      P.pool.push_back(e);
    }
    idx = P.used;
    P.used += 2;
    cudaEventRecord(P.pool[idx], st);
  }
  ~Prof() {
    if (idx == SIZE_MAX) return;
    Profiler& P = profiler();
    std::lock_guard<std::mutex> g(P.mu);
    cudaEventRecord(P.pool[idx + 1], st);
    P.recs.emplace_back(stage, idx);
  }
};

#define PROFILED(stage, st, ...)  \
  do {                            \
    Prof _prof((stage), (st));    \
    __VA_ARGS__;                  \
  } while (0)

// ---------------------------------------------------------------- sizing
inline bool use_tc(int32_t dtype) { return dtype == POETX_BF16; }

// K-splits of the dG = Y_j^T dV_j contractions (K = T tokens): enough
// (blocks x tiles x splits) to fill one wave, at least 4 K-blocks per split.
int dg_splits(int nblk, int b, int64_t T, int32_t dtype) {
  int tiles, kblock;
  if (use_tc(dtype)) {
    tiles = nblk * ((b + tc::BM - 1) / tc::BM) * ((b + choose_bn(b) - 1) / choose_bn(b));
    kblock = 64;
  } else {
    tiles = nblk * ((b + simt::TM - 1) / simt::TM) * ((b + simt::TN - 1) / simt::TN);
    kblock = simt::TK;
  }
  const int64_t nkb = (T + kblock - 1) / kblock;
  int64_t s = kSplitSMs / (tiles > 0 ? tiles : 1);
  if (s > nkb / 4) s = nkb / 4;
  if (s > 32) s = 32;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

// Scratch of the CNP build (3 b x b arrays per block) and backward (11).
size_t cnp_bwd_ws(int32_t nblk, int32_t b) {
  const size_t u = sizeof(float) * size_t(nblk) * b * b;
  return al(2 * u) + al(2 * u) + al(3 * u) + al(3 * u) + al(u);
}

size_t fwd_ws(const poetx_layer* L, int64_t T) {
  const size_t es = dtype_size(L->dtype);
  return kAlign + 2 * al(es * T * L->m) + 2 * al(es * T * L->n);
}

size_t bwd_ws(const poetx_layer* L, int64_t T) {
  const size_t es = dtype_size(L->dtype);
  const int64_t mx = L->m > L->n ? L->m : L->n;
  const int nR = L->m / L->b, nP = L->n / L->b;
  const size_t bb = size_t(L->b) * L->b;
  return kAlign + 2 * al(es * T * mx) + al(es * T * L->m) +
         al(sizeof(float) * dg_splits(nP, L->b, T, L->dtype) * nP * bb) +
         al(sizeof(float) * dg_splits(nR, L->b, T, L->dtype) * nR * bb) + cnp_bwd_ws(nR + nP, L->b);
}

// The backward that recomputes Y (y_save == NULL) also needs Y [T][n] and Xg [T][m].
size_t bwd_recompute_ws(const poetx_layer* L, int64_t T) {
  const size_t es = dtype_size(L->dtype);
  return bwd_ws(L, T) + al(es * T * L->n) + al(es * T * L->m);
}

size_t merge_ws(const poetx_layer* L) {
  const size_t nm = size_t(L->n) * L->m;
  const int nP = L->n / L->b;
  return kAlign + 2 * al(sizeof(float) * nm) + al(sizeof(float) * size_t(nP) * L->b * L->b) +
         2 * al(sizeof(int32_t) * L->m) + 2 * al(sizeof(int32_t) * L->n);
}

// ---------------------------------------------------------------- launch helpers
int grid_for(int64_t n, int threads, int device) {
  int64_t g = (n + threads - 1) / threads;
  const int64_t cap = int64_t(sm_count(device)) * 16;
  if (g > cap) g = cap;
  return g < 1 ? 1 : static_cast<int>(g);
}

template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes, bool* done) {
  if (bytes + 1024 <= 48 * 1024 || *done) return cudaSuccess;  // (static shared memory counts too)
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  if (e == cudaSuccess) *done = true;
  return e;
}

int rows_per_iter(int cols, size_t esz) {
  const size_t row = cols * esz;
  int r = static_cast<int>((40 * 1024) / (row ? row : 1));
  if (r > 8) r = 8;
  return r < 1 ? 1 : r;
}

template <typename Tin, typename Tout>
cudaError_t gather(const Tin* in, int64_t ld_in, int64_t in_rows, Tout* out, int64_t ld_out, int64_t rows, int cols,
                   const int32_t* colmap, const int32_t* rowmap, cudaStream_t st, int device) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  static bool attr[64] = {false};
  const int rpi = rows_per_iter(cols, sizeof(Tin));
  const size_t smem = size_t(rpi) * cols * sizeof(Tin);
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = allow_smem(gather_kernel<Tin, Tout>, smem, &attr[device & 63]);
  if (e != cudaSuccess) return e;
  int64_t g = (rows + rpi - 1) / rpi;
  const int64_t cap = int64_t(sm_count(device)) * 8;
  if (g > cap) g = cap;
  gather_kernel<Tin, Tout><<<static_cast<int>(g), 256, smem, st>>>(in, ld_in, in_rows, out, ld_out, rows, cols,
                                                                    colmap, rowmap, rpi);
  return cudaGetLastError();
}

template <typename T>
cudaError_t scatter(const T* in, int64_t ld_in, T* out, int64_t ld_out, int64_t out_rows, int64_t rows, int cols,
                    const int32_t* colmap, const int32_t* rowmap, cudaStream_t st, int device) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  static bool attr[64] = {false};
  const int rpi = rows_per_iter(cols, sizeof(T));
  const size_t smem = size_t(rpi) * cols * sizeof(T);
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = allow_smem(scatter_kernel<T>, smem, &attr[device & 63]);
  if (e != cudaSuccess) return e;
  int64_t g = (rows + rpi - 1) / rpi;
  const int64_t cap = int64_t(sm_count(device)) * 8;
  if (g > cap) g = cap;
  scatter_kernel<T><<<static_cast<int>(g), 256, smem, st>>>(in, ld_in, out, ld_out, out_rows, rows, cols, colmap,
                                                             rowmap, rpi);
  return cudaGetLastError();
}

// Hot-path column permutation of contiguous [rows][cols] activations:
// out = in[:, map] (inverse == 0) or out[:, map] = in (inverse == 1).
template <typename T>
cudaError_t permute_cols(const T* in, T* out, int64_t rows, int cols, const int32_t* map, int inverse,
                         cudaStream_t st, int device) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  constexpr int V = 16 / sizeof(T);
  const bool fast = cols < 65536 && cols % V == 0 && aligned16(in) && aligned16(out);
  if (!fast) {
    return inverse ? scatter(in, cols, out, cols, rows, rows, cols, map, nullptr, st, device)
                   : gather(in, cols, rows, out, cols, rows, cols, map, nullptr, st, device);
  }
  static bool attr[64] = {false};
  const size_t row_bytes = size_t(cols) * sizeof(T);
  int rps = static_cast<int>((24 * 1024) / row_bytes);
  if (rps < 1) rps = 1;
  if (rps > 64) rps = 64;
  const size_t idx_bytes = (size_t(cols) * 2 + 127) & ~size_t(127);
  size_t smem = idx_bytes + 2 * size_t(rps) * row_bytes;
  if (smem > 200 * 1024) {
    // rows too wide for two staged rows and the index table: one row at a time
    return inverse ? scatter(in, cols, out, cols, rows, rows, cols, map, nullptr, st, device)
                   : gather(in, cols, rows, out, cols, rows, cols, map, nullptr, st, device);
  }
  // each thread's index entries in registers when it owns at most kRegVecs
  // 16-byte output vectors per row
  constexpr int kRegVecs = 8;
  const int vpr = cols / V;
  const bool reg_idx = (vpr + 255) / 256 <= kRegVecs;
  // the register-index kernel keeps its table in stage 1 when it fits there
  // (more blocks per SM for wide rows)
  const int idx_in_stage = reg_idx && idx_bytes <= size_t(rps) * row_bytes ? 1 : 0;
  if (idx_in_stage) smem = 2 * size_t(rps) * row_bytes;
  static bool attr_reg[64] = {false};
  cudaError_t e = reg_idx ? allow_smem(permute_rows_reg_kernel<T, kRegVecs>, smem, &attr_reg[device & 63])
                          : allow_smem(permute_rows_kernel<T>, smem, &attr[device & 63]);
  if (e != cudaSuccess) return e;
  int per_sm = static_cast<int>((220 * 1024) / (smem + 1024));
  if (reg_idx && per_sm > 3) per_sm = 3;  // its registers (76 per thread) fit three 256-thread blocks per SM
  const int64_t chunks = (rows + rps - 1) / rps;
  int64_t g = int64_t(sm_count(device)) * (per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm));
  if (g > chunks) g = chunks;
  if (reg_idx)
    permute_rows_reg_kernel<T, kRegVecs><<<static_cast<int>(g), 256, smem, st>>>(in, out, rows, cols, map, inverse,
                                                                                 rps, idx_in_stage);
  else
    permute_rows_kernel<T><<<static_cast<int>(g), 256, smem, st>>>(in, out, rows, cols, map, inverse, rps);
  return cudaGetLastError();
}

cudaError_t permute_dt(int32_t dt, const void* in, void* out, int64_t rows, int cols, const int32_t* map, int inverse,
                       cudaStream_t st, int device) {
  if (dt == POETX_BF16)
    return permute_cols(static_cast<const __nv_bfloat16*>(in), static_cast<__nv_bfloat16*>(out), rows, cols, map,
                        inverse, st, device);
  return permute_cols(static_cast<const float*>(in), static_cast<float*>(out), rows, cols, map, inverse, st, device);
}

cudaError_t gather_dt(int32_t dt, const void* in, int64_t ld_in, int64_t in_rows, void* out, int64_t ld_out,
                      int64_t rows, int cols, const int32_t* colmap, const int32_t* rowmap, cudaStream_t st,
                      int device) {
  if (dt == POETX_BF16)
    return gather(static_cast<const __nv_bfloat16*>(in), ld_in, in_rows, static_cast<__nv_bfloat16*>(out), ld_out,
                  rows, cols, colmap, rowmap, st, device);
  return gather(static_cast<const float*>(in), ld_in, in_rows, static_cast<float*>(out), ld_out, rows, cols, colmap,
                rowmap, st, device);
}

cudaError_t scatter_dt(int32_t dt, const void* in, int64_t ld_in, void* out, int64_t ld_out, int64_t out_rows,
                       int64_t rows, int cols, const int32_t* colmap, const int32_t* rowmap, cudaStream_t st,
                       int device) {
  if (dt == POETX_BF16)
    return scatter(static_cast<const __nv_bfloat16*>(in), ld_in, static_cast<__nv_bfloat16*>(out), ld_out, out_rows,
                   rows, cols, colmap, rowmap, st, device);
  return scatter(static_cast<const float*>(in), ld_in, static_cast<float*>(out), ld_out, out_rows, rows, cols, colmap,
                 rowmap, st, device);
}

// ---------------------------------------------------------------- GEMM descriptions
// View of a [nblk][b][b] block array as a 2-D [nblk*b][b] matrix.
Operand2D blocks_view(const void* p, int et, int nblk, int b, bool transposed) {
  // transposed == false: element (mn, k) of block t is blk[t][k][mn] (MN-major)
  // transposed == true : element (mn, k) of block t is blk[t][mn][k] (K-major)
  Operand2D o;
  o.ptr = p;
  o.et = et;
  o.rows = int64_t(nblk) * b;
  o.cols = b;
  o.ld = b;
  o.mn_major = !transposed;
  o.b_row = b;
  o.b_col = 0;
  return o;
}

// Row-major [rows][cols] activation whose column blocks of width b are the
// batch (A operand of a block-diagonal product, K-major).
Operand2D colblocks_view(const void* p, int et, int64_t rows, int64_t cols, int b) {
  Operand2D o;
  o.ptr = p;
  o.et = et;
  o.rows = rows;
  o.cols = cols;
  o.ld = cols;
  o.mn_major = false;
  o.b_row = 0;
  o.b_col = b;
  return o;
}

// out[:, jb:(j+1)b] = in[:, jb:(j+1)b] . op(G_j) for every block j.
GemmDesc blockdiag_desc(const void* in, int et_in, int64_t T, int d, int b, const void* G, bool transpose_g,
                        void* out, int et_out) {
  GemmDesc g;
  g.M = static_cast<int>(T);
  g.N = b;
  g.K = b;
  g.batch = d / b;
  g.A = colblocks_view(in, et_in, T, d, b);
  // B(k, n) = G_j[k][n] (MN-major) or G_j[n][k] (K-major) for G_j^T.
  g.B = blocks_view(G, et_in, d / b, b, transpose_g);
  g.C.ptr = out;
  g.C.et = et_out;
  g.C.ld = d;
  g.C.batch_stride = b;
  g.C.view_rows = T;
  g.C.view_cols = d;
  g.C.b_col = b;
  return g;
}

// part[s][j] = (in1[:, jb:(j+1)b])^T in2[:, jb:(j+1)b] over token range s.
GemmDesc blockgrad_desc(const void* in1, const void* in2, int et, int64_t T, int d, int b, int splits,
                        float* part) {
  GemmDesc g;
  g.M = b;
  g.N = b;
  g.K = static_cast<int>(T);
  g.batch = d / b;
  g.splits = splits;
  Operand2D a;
  a.ptr = in1;
  a.et = et;
  a.rows = T;
  a.cols = d;
  a.ld = d;
  a.mn_major = true;
  a.b_row = 0;
  a.b_col = b;
  g.A = a;
  Operand2D bo = a;
  bo.ptr = in2;
  g.B = bo;
  g.C.ptr = part;
  g.C.et = ET_F32;
  g.C.ld = b;
  g.C.batch_stride = int64_t(b) * b;
  g.C.split_stride = int64_t(d / b) * b * b;
  g.C.view_rows = int64_t(splits) * (d / b) * b;
  g.C.view_cols = b;
  g.C.b_row = b;
  g.C.s_row = (d / b) * b;
  return g;
}

// ---------------------------------------------------------------- CNP
// With Q skew (Q^T = -Q) and S = Q^2 symmetric, every product the
// Cayley-Neumann block and its backward need is an X Y^T product:
//   S   = Q Q    = -(Q Q^T)
//   H S = H S^T                       (H = 2Q + S)
//   G   = I + 2Q + 2S + H S           (= (I+Q)(I+Q+Q^2+Q^3))
// Both sides of a layer (the G_R and G_P blocks) run as one batch of
// n0 + n1 blocks.

// View of a block array whose block t starts at p + t*b*ld (b rows, ld apart),
// using its first kcols columns as the K dimension (K-major).
Operand2D cat_view(const float* p, int nblk, int b, int64_t ld, int kcols) {
  Operand2D o;
  o.ptr = p;
  o.et = ET_F32;
  o.rows = int64_t(nblk) * b;
  o.cols = kcols;
  o.ld = ld;
  o.mn_major = false;
  o.b_row = b;
  o.b_col = 0;
  return o;
}

GemmDesc cat_nt_desc(const float* X, const float* Y, int nblk, int b, int64_t ld, int kcols, float alpha) {
  GemmDesc g;
  g.M = b;
  g.N = b;
  g.K = kcols;
  g.batch = nblk;
  g.A = cat_view(X, nblk, b, ld, kcols);
  g.B = cat_view(Y, nblk, b, ld, kcols);
  g.alpha = alpha;
  return g;
}

OutDesc out_blocks(void* p, int et, int b, int64_t ld) {
  OutDesc o;
  o.ptr = p;
  o.et = et;
  o.ld = ld;
  o.batch_stride = int64_t(b) * ld;
  return o;
}

AddDesc add_view(const float* p, int b, int64_t ld, float beta) {
  AddDesc a;
  a.ptr = p;
  a.ld = ld;
  a.batch_stride = int64_t(b) * ld;
  a.beta = beta;
  return a;
}

ExtraOut extra_out(float* p, int b, int64_t ld, float cv, bool transposed) {
  ExtraOut x;
  x.ptr = p;
  x.ld = ld;
  x.batch_stride = int64_t(b) * ld;
  x.cv = cv;
  x.transposed = transposed ? 1 : 0;
  return x;
}

size_t cnp_units(int32_t nblk, int32_t b) { return al(sizeof(float) * size_t(nblk) * b * b); }

Segs two_segs(const float* q0, int n0, void* G0, const float* q1, int n1, void* G1) {
  Segs sg{};
  sg.n = n1 > 0 ? 2 : 1;
  sg.start[0] = 0;
  sg.start[1] = n0;
  sg.start[2] = n0 + n1;
  sg.q[0] = q0;
  sg.q[1] = q1;
  sg.G[0] = G0;
  sg.G[1] = G1;
  return sg;
}

// G of every segment from its packed triangles, all blocks in one batch.
// Up to two segments write G straight from the GEMM epilogue; more go
// through a contiguous scratch copy (`gall`, nblk*b*b elements of dtype).
// ---- fused CNP on CTA pairs (b = 256, bf16 layers): one kernel per batch,
// every product of a block on tcgen05; the build keeps its operands in shared
// memory (cnp2build.cuh), the backward passes them through an L2-resident
// per-pair slot (cnp2sm.cuh).
bool use_pair_cnp(int32_t b, int32_t dtype) { return b == cnp2::BLK && dtype == POETX_BF16; }

int cnp_pair_count(int nblk, int device) {
  const int pairs = sm_count(device) / 2;
  return nblk < pairs ? nblk : pairs;
}

// bf16 operand region: the build's Q (nblk matrices); the backward's Q, dG
// and the per-pair slots (plus an fp32 dq scratch when it accumulates)
size_t cnp_pair_bytes(int nblk, bool backward, bool accumulate, int device) {
  if (!backward) return al(size_t(nblk) * cnp2::MAT_BYTES);
  const int pairs = cnp_pair_count(nblk, device);
  return al((size_t(nblk) * 2 + size_t(pairs) * cnp2::SKINDS) * cnp2::MAT_BYTES) +
         (accumulate ? al(sizeof(float) * size_t(nblk) * cnp2::TRI) : 0);
}

// Prep (bf16 Q, and for the backward bf16 dG and dq = 2 (dG - dG^T)) and the
// fused kernel.  With `accumulate` the backward writes its dq into a scratch
// copy and adds that to the caller's dq at the end, so the sum is exactly
// dq + (the dq a plain call gives).
cudaError_t launch_cnp_pair(const cnp2::PairSegs& sg_in, int nblk, bool backward, int accumulate, Carver& ws,
                            cudaStream_t st, int device) {
  static bool attr_set[64] = {false};
  if (device >= 0 && device < 64 && !attr_set[device]) {
    const cudaError_t e = cudaFuncSetAttribute(cnp2::cnp_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               cnp2::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[device] = true;
  }
  const int pairs = cnp_pair_count(nblk, device);
  if (pairs <= 0) return cudaSuccess;
  const int nmat = backward ? 2 * nblk + pairs * cnp2::SKINDS : nblk;
  __nv_bfloat16* region = ws.take<__nv_bfloat16>(size_t(nmat) * cnp2::MAT_BYTES);
  cnp2::PairSegs sg = sg_in;
  float* dq_tmp = nullptr;
  if (backward && accumulate) {
    dq_tmp = ws.take<float>(sizeof(float) * size_t(nblk) * cnp2::TRI);
    for (int i = 0; i < sg.n; ++i) sg.out[i] = dq_tmp + size_t(sg.start[i]) * cnp2::TRI;
  }
  Operand2D v;
  v.ptr = region;
  v.et = ET_BF16;
  v.rows = int64_t(nmat) * cnp2::BLK;
  v.cols = cnp2::BLK;
  v.ld = cnp2::BLK;
  CUtensorMap mk, mm, ms;
  if (!encode_map(&mk, v, cnp2::HALF) || !encode_map(&mm, v, cnp2::CH) || !encode_map(&ms, v, 32))
    return cudaErrorInvalidValue;
  const dim3 pgrid(cnp2::PREP_PAIRS, nblk), pblock(cnp2::PREP_THREADS);
  if (backward)
    PROFILED(ST_CNP_ELEM, st,
             cnp2::prep_kernel<true><<<pgrid, pblock, 0, st>>>(sg, region,
                                                               region + size_t(nblk) * cnp2::BLK * cnp2::BLK));
  else
    PROFILED(ST_CNP_ELEM, st, cnp2::prep_kernel<false><<<pgrid, pblock, 0, st>>>(sg, region, nullptr));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const uint32_t idesc_kk = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(cnp2::BLK >> 3) << 17) |
                            (static_cast<uint32_t>(cnp2::BLK >> 4) << 24);
  if (!backward) {
    // the build keeps S and H in shared memory (cnp2build.cuh)
    static bool battr[64] = {false};
    if (device >= 0 && device < 64 && !battr[device]) {
      e = cudaFuncSetAttribute(cnp2b::cnp_build_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               cnp2b::SMEM_BYTES);
      if (e != cudaSuccess) return e;
      battr[device] = true;
    }
    cnp2b::Params bp;
    bp.nblk = nblk;
    bp.idesc = idesc_kk;
    cnp2b::GMaps gm;
    for (int i = 0; i < sg.n; ++i) {
      Operand2D g;
      g.ptr = sg.out[i];
      g.et = ET_BF16;
      g.rows = int64_t(sg.start[i + 1] - sg.start[i]) * cnp2::BLK;
      g.cols = cnp2::BLK;
      g.ld = cnp2::BLK;
      if (g.rows > 0 && !encode_map(&gm.m[i], g, 32)) return cudaErrorInvalidValue;
    }
    PROFILED(ST_CNP_GEMM, st,
             cnp2b::cnp_build_pair_kernel<<<2 * pairs, cnp2b::NUM_THREADS, cnp2b::SMEM_BYTES, st>>>(mk, sg, gm, bp));
    return cudaGetLastError();
  }
  cnp2::Params p;
  p.nblk = nblk;
  // D fp32, A and B bf16, N = 256 (bits 17-22: N >> 3), M = 256 (bits 24-28: M >> 4);
  // bit 15: A MN-major, bit 16: B MN-major
  p.idesc_kk = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(cnp2::BLK >> 3) << 17) |
               (static_cast<uint32_t>(cnp2::BLK >> 4) << 24);
  p.idesc_kmn = p.idesc_kk | (1u << 16);
  p.idesc_mnmn = p.idesc_kk | (1u << 15) | (1u << 16);
  PROFILED(ST_CNP_GEMM, st,
           cnp2::cnp_pair_kernel<<<2 * pairs, cnp2::NUM_THREADS, cnp2::SMEM_BYTES, st>>>(mk, mm, ms, sg, p));
  e = cudaGetLastError();
  if (e != cudaSuccess || !dq_tmp) return e;
  for (int i = 0; i < sg.n; ++i) {
    const int64_t n4 = int64_t(sg.start[i + 1] - sg.start[i]) * cnp2::TRI / 4;
    if (n4 <= 0) continue;
    PROFILED(ST_CNP_ELEM, st,
             add_f32x4_kernel<<<grid_for(n4, 256, device), 256, 0, st>>>(
                 static_cast<float4*>(sg_in.out[i]), reinterpret_cast<const float4*>(sg.out[i]), n4));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ---- fused backward of one side for b = 256 bf16 layers (bdg2sm.cuh):
// O = D G^T blockwise (skipped when O is NULL) and the split-K partials of
// dG = X^T D, reading D once.
bool use_pair_bdg(const poetx_layer& L) { return L.b == bdg2::BLK && L.dtype == POETX_BF16; }

cudaError_t launch_bdg(const void* D, const void* X, const void* G, void* O, float* part, int64_t T, int d, int splits,
                       cudaStream_t st, int device) {
  static bool attr_set[64] = {false};
  if (device >= 0 && device < 64 && !attr_set[device]) {
    const cudaError_t e =
        cudaFuncSetAttribute(bdg2::bdg_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bdg2::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[device] = true;
  }
  const int nblk = d / bdg2::BLK;
  const int ntiles = static_cast<int>((T + bdg2::BLK - 1) / bdg2::BLK);
  if (splits < 1 || splits > ntiles) return cudaErrorInvalidValue;
  auto view = [](const void* ptr, int64_t rows, int64_t cols) {
    Operand2D v;
    v.ptr = ptr;
    v.et = ET_BF16;
    v.rows = rows;
    v.cols = cols;
    v.ld = cols;
    return v;
  };
  CUtensorMap mDk, mDmn, mXmn, mG, mO;
  if (!encode_map(&mDk, view(D, T, d), bdg2::HALF) || !encode_map(&mDmn, view(D, T, d), bdg2::CH) ||
      !encode_map(&mXmn, view(X, T, d), bdg2::CH) ||
      !encode_map(&mG, view(G, int64_t(nblk) * bdg2::BLK, bdg2::BLK), bdg2::HALF) ||
      !encode_map(&mO, view(O ? O : D, T, d), 32))
    return cudaErrorInvalidValue;
  bdg2::Params p;
  p.T = static_cast<int>(T);
  p.nblk = nblk;
  p.splits = splits;
  p.ntiles = ntiles;
  p.want_o = O ? 1 : 0;
  // D fp32, A and B bf16, N = 256 (bits 17-22: N >> 3), M = 256 (bits 24-28: M >> 4);
  // bit 15: A MN-major, bit 16: B MN-major
  p.idesc_kk = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(bdg2::BLK >> 3) << 17) |
               (static_cast<uint32_t>(bdg2::BLK >> 4) << 24);
  p.idesc_mnmn = p.idesc_kk | (1u << 15) | (1u << 16);
  p.part = part;
  const int items = nblk * splits;
  const int pairs = sm_count(device) / 2 < items ? sm_count(device) / 2 : items;
  bdg2::bdg_pair_kernel<<<2 * pairs, bdg2::NUM_THREADS, bdg2::SMEM_BYTES, st>>>(mDk, mDmn, mXmn, mG, mO, p);
  return cudaGetLastError();
}

// Y = (Xg Diag(G_R)) W~^T for T token rows.  With POETX_FOLD_R and T > n
// the R-side block product is applied to the n rows of the weight instead of
// the T rows of activations: W_R = W~ Diag(G_R)^T ([n][m], one weight-sized
// pass), then Y = Xg W_R^T, which skips the [T][m] intermediate U.
// `scratch` holds U ([T][m]) or W_R ([n][m], smaller when T > n).  The choice
// depends only on (layer, T), so a recomputing backward gets the forward's Y
// bit for bit.  Without the flag (the default) the layer stays input-centric.
bool fold_r_into_weight(const poetx_layer& L, int64_t T) {
  return (L.fold & POETX_FOLD_R) && L.dtype == POETX_BF16 && T > L.n;
}

// Backward P side, with POETX_FOLD_P: dU = dV (Diag(G_P)^T W~) instead of
// (dV Diag(G_P)^T) W~ when T > m (the [n][m] folded weight is smaller than
// the [T][n] dY it replaces, and fits in the dY buffer).
bool fold_p_into_weight(const poetx_layer& L, int64_t T) {
  return (L.fold & POETX_FOLD_P) && L.dtype == POETX_BF16 && T > L.m;
}

// Wout = Diag(G_P)^T Win over the n/b row blocks of an [n][m] weight:
// Wout[bj + c][i'] = sum_j' G_Pj[j'][c] Win[bj + j'][i'] (one batched GEMM).
cudaError_t fold_p_rows(const poetx_layer& L, const void* Win, void* Wout, cudaStream_t st, int dev) {
  const int et = elem_type(L.dtype);
  GemmDesc g;
  g.M = L.b;
  g.N = L.m;
  g.K = L.b;
  g.batch = L.n / L.b;
  Operand2D a;
  a.ptr = L.GP;
  a.et = et;
  a.rows = L.n;
  a.cols = L.b;
  a.ld = L.b;
  a.mn_major = true;  // A[c][j'] = G_Pj[j'][c]
  a.b_row = L.b;
  g.A = a;
  Operand2D w;
  w.ptr = Win;
  w.et = et;
  w.rows = L.n;
  w.cols = L.m;
  w.ld = L.m;
  w.mn_major = true;  // B(k = j', n = i') = Win[bj + j'][i']
  w.b_row = L.b;
  g.B = w;
  g.C.ptr = Wout;
  g.C.et = et;
  g.C.ld = L.m;
  g.C.batch_stride = int64_t(L.b) * L.m;
  g.C.view_rows = L.n;
  g.C.view_cols = L.m;
  g.C.b_row = L.b;
  PROFILED(ST_BLOCKDIAG, st, POETX_CUDA_ERR(launch_gemm(g, use_tc(L.dtype), st, dev)));
  return cudaSuccess;
}

// With nothing saved (inference, or a backward that recomputes) and
// POETX_FOLD_WEIGHT_CENTRIC, a forward of T > 6nm / (2m + 4n) rows is cheaper
// as one GEMM with the whole layer
// folded into the weight in the natural frames,
//   z = x W_eff^T,  W_eff = Psi_P^T Diag(G_P)^T W~ Diag(G_R)^T Psi_R,
// than as gather, block products and scatter over the token rows (three
// weight-sized passes instead of 2m + 4n activation columns).
bool weight_centric_forward(const poetx_layer& L, int64_t T) {
  return (L.fold & POETX_FOLD_WEIGHT_CENTRIC) && L.dtype == POETX_BF16 &&
         T * (2 * int64_t(L.m) + 4 * int64_t(L.n)) > 6 * int64_t(L.n) * L.m;
}

cudaError_t y_from_xg(const poetx_layer& L, int64_t T, const void* Xg, void* Y, void* scratch, cudaStream_t st,
                      int dev) {
  const int et = elem_type(L.dtype);
  const bool tc_path = use_tc(L.dtype);
  const void* A;
  const void* Wb;
  if (fold_r_into_weight(L, T)) {
    PROFILED(ST_BLOCKDIAG, st,
             POETX_CUDA_ERR(launch_gemm(blockdiag_desc(L.W, et, L.n, L.m, L.b, L.GR, true, scratch, et), tc_path, st,
                                        dev)));
    A = Xg;
    Wb = scratch;
  } else {
    PROFILED(ST_BLOCKDIAG, st,
             POETX_CUDA_ERR(launch_gemm(blockdiag_desc(Xg, et, T, L.m, L.b, L.GR, false, scratch, et), tc_path, st,
                                        dev)));
    A = scratch;
    Wb = L.W;
  }
  // B(k=i', n=j') = W[j'][i'], K-major
  GemmDesc g;
  g.M = static_cast<int>(T);
  g.N = L.n;
  g.K = L.m;
  g.A = colblocks_view(A, et, T, L.m, 0);
  Operand2D b;
  b.ptr = Wb;
  b.et = et;
  b.rows = L.n;
  b.cols = L.m;
  b.ld = L.m;
  b.mn_major = false;
  g.B = b;
  g.C.ptr = Y;
  g.C.et = et;
  g.C.ld = L.n;
  g.C.view_rows = T;
  g.C.view_cols = L.n;
  PROFILED(ST_W0, st, POETX_CUDA_ERR(launch_gemm(g, tc_path, st, dev)));
  return cudaSuccess;
}

poetx_status cnp_build_segs(int32_t b, int32_t dtype, const Segs& sg, Carver& ws, cudaStream_t st, int device) {
  const int nblk = sg.start[sg.n];
  if (use_pair_cnp(b, dtype) && ws.fits(cnp_pair_bytes(nblk, false, false, device))) {
    if (nblk == 0) return POETX_OK;
    cnp2::PairSegs ps{};
    ps.n = sg.n;
    for (int i = 0; i <= sg.n; ++i) ps.start[i] = sg.start[i];
    for (int i = 0; i < sg.n; ++i) {
      ps.q[i] = sg.q[i];
      ps.out[i] = sg.G[i];
    }
    POETX_CUDA(launch_cnp_pair(ps, nblk, false, 0, ws, st, device));
    return POETX_OK;
  }
  const size_t nbb = size_t(nblk) * b * b;
  float* Q = ws.take<float>(sizeof(float) * nbb);
  float* S = ws.take<float>(sizeof(float) * nbb);
  float* H = ws.take<float>(sizeof(float) * nbb);
  void* gall = sg.n > 2 ? ws.take<uint8_t>(dtype_size(dtype) * nbb) : nullptr;
  const bool tc_path = use_tc(dtype);
  const int64_t bb = int64_t(b) * b;
  const dim3 ugrid((b + 31) / 32, (b + 31) / 32, nblk), ublock(32, 8);
  PROFILED(ST_CNP_ELEM, st, unpack_skew_kernel<<<ugrid, ublock, 0, st>>>(sg, nblk, b, Q, b, bb, nullptr, 0, 0));
  POETX_CUDA(cudaGetLastError());
  // S = -(Q Q^T); H = S + 2Q as a second output
  {
    GemmDesc g = cat_nt_desc(Q, Q, nblk, b, b, b, -1.f);
    g.C = out_blocks(S, ET_F32, b, b);
    g.ex[0] = extra_out(H, b, b, 1.f, false);
    g.ex[0].add = Q;
    g.ex[0].add_ld = b;
    g.ex[0].add_bs = bb;
    g.ex[0].ca = 2.f;
    PROFILED(ST_CNP_GEMM, st, POETX_CUDA(launch_gemm(g, tc_path, st, device)));
  }
  // G = H S^T + 2Q + 2S + I  (S^T = S)
  {
    GemmDesc g = cat_nt_desc(H, S, nblk, b, b, b, 1.f);
    if (gall) {
      g.C = out_blocks(gall, elem_type(dtype), b, b);
    } else {
      g.C = out_blocks(sg.G[0], elem_type(dtype), b, b);
      g.C.ptr2 = sg.G[1];
      g.C.split_batch = sg.start[1];
    }
    g.add1 = add_view(Q, b, b, 2.f);
    g.add2 = add_view(S, b, b, 2.f);
    g.diag = 1.f;
    PROFILED(ST_CNP_GEMM, st, POETX_CUDA(launch_gemm(g, tc_path, st, device)));
  }
  if (gall) {
    const int64_t block_bytes = int64_t(dtype_size(dtype)) * bb;
    const dim3 grid(static_cast<unsigned>((block_bytes / 16 + 255) / 256), nblk);
    PROFILED(ST_CNP_ELEM, st,
             split_blocks_kernel<<<grid, 256, 0, st>>>(sg, static_cast<const uint8_t*>(gall), nblk, block_bytes));
    POETX_CUDA(cudaGetLastError());
  }
  return POETX_OK;
}

poetx_status cnp_build2(int32_t b, int32_t dtype, const float* q0, int n0, void* G0, const float* q1, int n1,
                        void* G1, Carver& ws, cudaStream_t st, int device) {
  return cnp_build_segs(b, dtype, two_segs(q0, n0, G0, q1, n1, G1), ws, st, device);
}

// dq from dG for G = I + 2A + 2S + H S with S = A A, H = 2A + S:
//   dH = dG S^T;  dS = 2 dG + H^T dG + dH;  dA = 2 dG + 2 dH + dS A^T + A^T dS;
//   dq_k = dA[i][j] - dA[j][i].
// Written as three X Y^T products over concatenated K (A^T = -A):
//   S  = -(A A^T)
//   dS = 2 dG + [H^T | dG] [dG^T | S]^T
//   dA = 2 dG + [dS | A | dG] [A | -dS^T | 2S]^T
// The concatenated operands X1 = [H^T | dG], Y1 = [dG^T | S] (b x 2b blocks)
// and X2 = [dS | A | dG], Y2 = [A | -dS^T | 2S] (b x 3b blocks) are filled
// in place by the unpack, the split reduction and the GEMM epilogues.
// dG of side k is the sum of splits_k partial arrays part_k.
poetx_status cnp_backward2(int32_t b, int32_t dtype, const float* q0, int n0, const float* part0, int splits0,
                           float* dq0, const float* q1, int n1, const float* part1, int splits1, float* dq1,
                           int32_t accumulate, Carver& ws, cudaStream_t st, int device) {
  const int nblk = n0 + n1;
  const size_t nbb = size_t(nblk) * b * b;
  if (use_pair_cnp(b, dtype) &&
      ws.fits(((splits0 > 1 || splits1 > 1) ? al(sizeof(float) * nbb) : 0) +
              cnp_pair_bytes(nblk, true, accumulate != 0, device))) {
    if (nblk == 0) return POETX_OK;
    const float* dG0 = part0;
    const float* dG1 = part1;
    if (splits0 > 1 || splits1 > 1) {
      // dG = fixed-order sum of the token splits, both sides into one scratch
      float* sum = ws.take<float>(sizeof(float) * nbb);
      const int64_t n40 = int64_t(n0) * b * b / 4, n41 = int64_t(n1) * b * b / 4;
      PROFILED(ST_REDUCE, st,
               sum_splits2_kernel<<<grid_for(n40 + n41, 256, device), 256, 0, st>>>(
                   reinterpret_cast<const float4*>(part0), splits0, n40, reinterpret_cast<float4*>(sum),
                   reinterpret_cast<const float4*>(part1), splits1, n41, reinterpret_cast<float4*>(sum + n40 * 4), 0));
      POETX_CUDA(cudaGetLastError());
      dG0 = sum;
      dG1 = sum + n40 * 4;
    }
    cnp2::PairSegs ps{};
    ps.n = n1 > 0 ? 2 : 1;
    ps.start[0] = 0;
    ps.start[1] = n0;
    ps.start[2] = n0 + n1;
    ps.q[0] = q0;
    ps.dG[0] = dG0;
    ps.out[0] = dq0;
    ps.q[1] = q1;
    ps.dG[1] = dG1;
    ps.out[1] = dq1;
    POETX_CUDA(launch_cnp_pair(ps, nblk, true, accumulate, ws, st, device));
    return POETX_OK;
  }
  const int64_t b2 = 2 * int64_t(b), b3 = 3 * int64_t(b);
  float* X1 = ws.take<float>(sizeof(float) * 2 * nbb);
  float* Y1 = ws.take<float>(sizeof(float) * 2 * nbb);
  float* X2 = ws.take<float>(sizeof(float) * 3 * nbb);
  float* Y2 = ws.take<float>(sizeof(float) * 3 * nbb);
  float* dA = ws.take<float>(sizeof(float) * nbb);
  const bool tc_path = use_tc(dtype);
  // A -> X2[:, b:2b] and Y2[:, 0:b]
  const dim3 ugrid((b + 31) / 32, (b + 31) / 32, nblk), ublock(32, 8);
  PROFILED(ST_CNP_ELEM, st,
           unpack_skew_kernel<<<ugrid, ublock, 0, st>>>(two_segs(q0, n0, nullptr, q1, n1, nullptr), nblk, b, X2 + b,
                                                        b3, b * b3, Y2, b3, b * b3));
  // dG -> X1[:, b:2b], X2[:, 2b:3b];  dG^T -> Y1[:, 0:b]
  {
    if (b % 32 == 0) {
      const dim3 grid(b / 32, b / 32, nblk), block(8, 32);
      PROFILED(ST_CNP_ELEM, st,
               reduce_transpose_kernel<<<grid, block, 0, st>>>(part0, splits0, n0, part1, splits1, n1, b, X1 + b,
                                                               b2, b * b2, X2 + 2 * b, b3, b * b3, Y1, b2, b * b2));
    } else {
      const dim3 grid((b + 31) / 32, (b + 31) / 32, nblk), block(32, 8);
      PROFILED(ST_CNP_ELEM, st,
               reduce_transpose_any_kernel<<<grid, block, 0, st>>>(part0, splits0, n0, part1, splits1, n1, b,
                                                                   X1 + b, b2, b * b2, X2 + 2 * b, b3, b * b3, Y1, b2,
                                                                   b * b2));
    }
  }
  POETX_CUDA(cudaGetLastError());
  // S = -(A A^T) -> Y1[:, b:2b];  H^T = (S + 2A)^T -> X1[:, 0:b];  2S -> Y2[:, 2b:3b]
  {
    GemmDesc g = cat_nt_desc(X2 + b, X2 + b, nblk, b, b3, b, -1.f);
    g.C = out_blocks(Y1 + b, ET_F32, b, b2);
    g.ex[0] = extra_out(X1, b, b2, 1.f, true);
    g.ex[0].add = X2 + b;
    g.ex[0].add_ld = b3;
    g.ex[0].add_bs = b * b3;
    g.ex[0].ca = 2.f;
    g.ex[1] = extra_out(Y2 + 2 * b, b, b3, 2.f, false);
    PROFILED(ST_CNP_GEMM, st, POETX_CUDA(launch_gemm(g, tc_path, st, device)));
  }
  // dS = 2 dG + X1 Y1^T -> X2[:, 0:b];  -dS^T -> Y2[:, b:2b]
  {
    GemmDesc g = cat_nt_desc(X1, Y1, nblk, b, b2, 2 * b, 1.f);
    g.C = out_blocks(X2, ET_F32, b, b3);
    g.add1 = add_view(X1 + b, b, b2, 2.f);
    g.ex[0] = extra_out(Y2 + b, b, b3, -1.f, true);
    PROFILED(ST_CNP_GEMM, st, POETX_CUDA(launch_gemm(g, tc_path, st, device)));
  }
  // dA = 2 dG + X2 Y2^T
  {
    GemmDesc g = cat_nt_desc(X2, Y2, nblk, b, b3, 3 * b, 1.f);
    g.C = out_blocks(dA, ET_F32, b, b);
    g.add1 = add_view(X2 + 2 * b, b, b3, 2.f);
    PROFILED(ST_CNP_GEMM, st, POETX_CUDA(launch_gemm(g, tc_path, st, device)));
  }
  PROFILED(ST_CNP_ELEM, st,
           fold_skew2_kernel<<<static_cast<int>(int64_t(nblk) * b), 128, 0, st>>>(dA, b, int64_t(b) * b, n0, b, dq0,
                                                                                   dq1, accumulate));
  POETX_CUDA(cudaGetLastError());
  return POETX_OK;
}

}  // namespace

// ======================================================================== ABI

extern "C" {

const char* poetx_status_string(int status) {
  switch (status) {
    case POETX_OK: return "POETX_OK";
    case POETX_E_ARG: return "POETX_E_ARG: null pointer, negative size or bad flag";
    case POETX_E_SHAPE: return "POETX_E_SHAPE: b must divide m and n (and be a multiple of 64 for bf16)";
    case POETX_E_DTYPE: return "POETX_E_DTYPE: unknown dtype";
    case POETX_E_ALIGN: return "POETX_E_ALIGN: pointer not 16-byte aligned";
    case POETX_E_WORKSPACE: return "POETX_E_WORKSPACE: workspace missing or too small";
    case POETX_E_ARCH: return "POETX_E_ARCH: current device is not compute capability 10.0 (B200)";
    case POETX_E_CUDA: return "POETX_E_CUDA: CUDA runtime error while queueing work";
    default: return "POETX: unknown status";
  }
}

int32_t poetx_version(void) { return 10100; }

poetx_status poetx_device_error(uint32_t* code) {
  if (!code) return POETX_E_ARG;
  int dev;
  POETX_TRY(current_device(&dev));
  unsigned int v = 0, zero = 0;
  POETX_CUDA(cudaDeviceSynchronize());
  POETX_CUDA(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)));
  POETX_CUDA(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)));
  *code = v;
  return POETX_OK;
}

size_t poetx_cnp_workspace_bytes(int32_t nblk, int32_t b, int32_t dtype) {
  (void)dtype;
  if (nblk <= 0 || b < 2) return 0;
  return kAlign + cnp_bwd_ws(nblk, b);
}

size_t poetx_layers_cnp_workspace_bytes(int32_t nlayers, const poetx_layer* layers) {
  if (nlayers < 1 || 2 * nlayers > kMaxSegs || !layers) return 0;
  int64_t nblk = 0;
  for (int i = 0; i < nlayers; ++i) {
    if (check_layer(&layers[i]) != POETX_OK || layers[i].b != layers[0].b || layers[i].dtype != layers[0].dtype)
      return 0;
    nblk += layers[i].m / layers[i].b + layers[i].n / layers[i].b;
  }
  const int b = layers[0].b;
  return kAlign + 3 * cnp_units(static_cast<int32_t>(nblk), b) +
         al(size_t(dtype_size(layers[0].dtype)) * size_t(nblk) * b * b);
}

poetx_status poetx_layers_cnp_build(int32_t nlayers, const poetx_layer* layers, void* ws, size_t ws_bytes,
                                    void* stream) {
  if (nlayers < 1 || 2 * nlayers > kMaxSegs || !layers) return POETX_E_ARG;
  for (int i = 0; i < nlayers; ++i) {
    POETX_TRY(check_layer(&layers[i]));
    if (layers[i].b != layers[0].b) return POETX_E_SHAPE;
    if (layers[i].dtype != layers[0].dtype) return POETX_E_DTYPE;
  }
  if (!ws || ws_bytes < poetx_layers_cnp_workspace_bytes(nlayers, layers)) return POETX_E_WORKSPACE;
  int dev;
  POETX_TRY(current_device(&dev));
  Segs sg{};
  sg.n = 2 * nlayers;
  int blk = 0;
  for (int i = 0; i < nlayers; ++i) {
    const poetx_layer& L = layers[i];
    sg.start[2 * i] = blk;
    sg.q[2 * i] = L.qR;
    sg.G[2 * i] = L.GR;
    blk += L.m / L.b;
    sg.start[2 * i + 1] = blk;
    sg.q[2 * i + 1] = L.qP;
    sg.G[2 * i + 1] = L.GP;
    blk += L.n / L.b;
  }
  sg.start[sg.n] = blk;
  Carver c(ws, ws_bytes);
  return cnp_build_segs(layers[0].b, layers[0].dtype, sg, c, static_cast<cudaStream_t>(stream), dev);
}

size_t poetx_layer_cnp_workspace_bytes(const poetx_layer* layer) {
  if (check_layer(layer) != POETX_OK) return 0;
  return kAlign + cnp_bwd_ws(layer->m / layer->b + layer->n / layer->b, layer->b);
}

poetx_status poetx_layer_cnp_build(const poetx_layer* layer, void* ws, size_t ws_bytes, void* stream) {
  POETX_TRY(check_layer(layer));
  if (!ws || ws_bytes < poetx_layer_cnp_workspace_bytes(layer)) return POETX_E_WORKSPACE;
  int dev;
  POETX_TRY(current_device(&dev));
  const poetx_layer& L = *layer;
  Carver c(ws, ws_bytes);
  return cnp_build2(L.b, L.dtype, L.qR, L.m / L.b, L.GR, L.qP, L.n / L.b, L.GP, c, static_cast<cudaStream_t>(stream),
                    dev);
}

size_t poetx_forward_workspace_bytes(const poetx_layer* layer, int64_t T) {
  if (check_layer(layer) != POETX_OK || T < 0 || T > kMaxT) return 0;
  return fwd_ws(layer, T);
}

size_t poetx_backward_workspace_bytes(const poetx_layer* layer, int64_t T) {
  if (check_layer(layer) != POETX_OK || T < 0 || T > kMaxT) return 0;
  return bwd_ws(layer, T);
}

size_t poetx_backward_recompute_workspace_bytes(const poetx_layer* layer, int64_t T) {
  if (check_layer(layer) != POETX_OK || T < 0 || T > kMaxT) return 0;
  return bwd_recompute_ws(layer, T);
}

size_t poetx_merge_workspace_bytes(const poetx_layer* layer) {
  if (check_layer(layer) != POETX_OK) return 0;
  return merge_ws(layer);
}

size_t poetx_check_perm_workspace_bytes(int32_t len) {
  if (len <= 0) return 0;
  return kAlign + al(sizeof(int32_t) * size_t(len));
}

poetx_status poetx_frame_import(const poetx_layer* layer, const void* W0lin, void* stream) {
  POETX_TRY(check_layer(layer));
  POETX_TRY(check_ptr(W0lin));
  int dev;
  POETX_TRY(current_device(&dev));
  const poetx_layer& L = *layer;
  // W[j'][i'] = W0lin[permP[j']][permR[i']]
  POETX_CUDA(gather_dt(L.dtype, W0lin, L.m, L.n, L.W, L.m, L.n, L.m, L.permR, L.permP,
                       static_cast<cudaStream_t>(stream), dev));
  return POETX_OK;
}

poetx_status poetx_frame_export(const poetx_layer* layer, void* W0lin, void* stream) {
  POETX_TRY(check_layer(layer));
  POETX_TRY(check_ptr(W0lin));
  int dev;
  POETX_TRY(current_device(&dev));
  const poetx_layer& L = *layer;
  // W0lin[permP[j']][permR[i']] = W[j'][i']
  POETX_CUDA(scatter_dt(L.dtype, L.W, L.m, W0lin, L.m, L.n, L.n, L.m, L.permR, L.permP,
                        static_cast<cudaStream_t>(stream), dev));
  return POETX_OK;
}

poetx_status poetx_cnp_build(int32_t nblk, int32_t b, const float* q, int32_t dtype, void* G, void* ws,
                             size_t ws_bytes, void* stream) {
  POETX_TRY(check_dtype_b(dtype, b));
  if (nblk < 0) return POETX_E_ARG;
  if (nblk == 0) return POETX_OK;
  POETX_TRY(check_ptr(q));
  POETX_TRY(check_ptr(G));
  if (!ws || ws_bytes < poetx_cnp_workspace_bytes(nblk, b, dtype)) return POETX_E_WORKSPACE;
  int dev;
  POETX_TRY(current_device(&dev));
  Carver c(ws, ws_bytes);
  return cnp_build2(b, dtype, q, nblk, G, nullptr, 0, nullptr, c, static_cast<cudaStream_t>(stream), dev);
}

poetx_status poetx_cnp_backward(int32_t nblk, int32_t b, const float* q, const float* dG, float* dq,
                                int32_t accumulate, int32_t dtype, void* ws, size_t ws_bytes, void* stream) {
  POETX_TRY(check_dtype_b(dtype, b));
  if (nblk < 0) return POETX_E_ARG;
  if (nblk == 0) return POETX_OK;
  POETX_TRY(check_ptr(q));
  POETX_TRY(check_ptr(dG));
  POETX_TRY(check_ptr(dq));
  if (!ws || ws_bytes < poetx_cnp_workspace_bytes(nblk, b, dtype)) return POETX_E_WORKSPACE;
  int dev;
  POETX_TRY(current_device(&dev));
  Carver c(ws, ws_bytes);
  return cnp_backward2(b, dtype, q, nblk, dG, 1, dq, nullptr, 0, nullptr, 1, nullptr, accumulate, c,
                       static_cast<cudaStream_t>(stream), dev);
}

poetx_status poetx_forward(const poetx_layer* layer, int64_t T, const void* x, void* z, void* y_save,
                           void* xg_save, void* ws, size_t ws_bytes, void* stream) {
  POETX_TRY(check_layer(layer));
  if (T < 0) return POETX_E_ARG;
  if (T > kMaxT) return POETX_E_SHAPE;
  if (T == 0) return POETX_OK;
  POETX_TRY(check_ptr(x));
  POETX_TRY(check_ptr(z));
  if (y_save && !aligned16(y_save)) return POETX_E_ALIGN;
  if (xg_save && !aligned16(xg_save)) return POETX_E_ALIGN;
  if (!ws || ws_bytes < fwd_ws(layer, T)) return POETX_E_WORKSPACE;
  int dev;
  POETX_TRY(current_device(&dev));
  const poetx_layer& L = *layer;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int et = elem_type(L.dtype);
  const size_t es = dtype_size(L.dtype);
  const bool tc_path = use_tc(L.dtype);
  if (!y_save && !xg_save && weight_centric_forward(L, T)) {
    // two [n][m] weights fit in the workspace whenever this path is chosen
    Carver cw(ws, ws_bytes);
    if (cw.fits(2 * al(es * size_t(L.n) * L.m))) {
      void* W1 = cw.take<uint8_t>(es * size_t(L.n) * L.m);
      void* W2 = cw.take<uint8_t>(es * size_t(L.n) * L.m);
      // W1 = W~ Diag(G_R)^T, W2 = Diag(G_P)^T W1, W1 = W2 in natural order
      PROFILED(ST_BLOCKDIAG, st,
               POETX_CUDA(launch_gemm(blockdiag_desc(L.W, et, L.n, L.m, L.b, L.GR, true, W1, et), tc_path, st, dev)));
      POETX_CUDA(fold_p_rows(L, W1, W2, st, dev));
      PROFILED(ST_PERMUTE, st,
               POETX_CUDA(scatter_dt(L.dtype, W2, L.m, W1, L.m, L.n, L.n, L.m, L.permR, L.permP, st, dev)));
      // z = x W1^T
      GemmDesc g;
      g.M = static_cast<int>(T);
      g.N = L.n;
      g.K = L.m;
      g.A = colblocks_view(x, et, T, L.m, 0);
      Operand2D b;
      b.ptr = W1;
      b.et = et;
      b.rows = L.n;
      b.cols = L.m;
      b.ld = L.m;
      b.mn_major = false;
      g.B = b;
      g.C.ptr = z;
      g.C.et = et;
      g.C.ld = L.n;
      g.C.view_rows = T;
      g.C.view_cols = L.n;
      PROFILED(ST_W0, st, POETX_CUDA(launch_gemm(g, tc_path, st, dev)));
      return POETX_OK;
    }
  }
  Carver c(ws, ws_bytes);
  void* Xw = c.take<uint8_t>(es * T * L.m);
  void* Xg = xg_save ? xg_save : Xw;
  void* U = c.take<uint8_t>(es * T * L.m);
  void* V = c.take<uint8_t>(es * T * L.n);
  void* Yw = c.take<uint8_t>(es * T * L.n);
  void* Y = y_save ? y_save : Yw;
  // Xg = x Psi_R^T  (columns gathered into the Psi_R frame)
  PROFILED(ST_PERMUTE, st, POETX_CUDA(permute_dt(L.dtype, x, Xg, T, L.m, L.permR, 0, st, dev)));
  // Y = (Xg Diag(G_R)) W~^T  (W~ = Psi_R W0 Psi_P^T stored [n][m]); U in `U`, or,
  // with POETX_FOLD_R and T > n, the weight with G_R folded in
  POETX_CUDA(y_from_xg(L, T, Xg, Y, U, st, dev));
  // V_j = Y_j G_Pj
  PROFILED(ST_BLOCKDIAG, st, POETX_CUDA(launch_gemm(blockdiag_desc(Y, et, T, L.n, L.b, L.GP, false, V, et), tc_path, st, dev)));
  // z = V Psi_P  (columns scattered back to natural order)
  PROFILED(ST_PERMUTE, st, POETX_CUDA(permute_dt(L.dtype, V, z, T, L.n, L.permP, 1, st, dev)));
  return POETX_OK;
}

// Backward of one layer.  Gradient mode "dq" (dGR == dGP == NULL): the
// packed dq of both sides through the CNP backward.  Mode "dG" (dqR == dqP
// == NULL): the token sums dG of both sides, CNP backward left to the caller.
static poetx_status backward_impl(const poetx_layer* layer, int64_t T, const void* x, const void* y_save,
                           const void* xg_save, const void* dz, void* dx, float* dqR, float* dqP, float* dGR,
                           float* dGP, int32_t accumulate, void* ws, size_t ws_bytes, void* stream) {
  POETX_TRY(check_layer(layer));
  if (T < 0) return POETX_E_ARG;
  if (T > kMaxT) return POETX_E_SHAPE;
  const bool dg_mode = dGR != nullptr;
  const poetx_layer& L = *layer;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nR = L.m / L.b, nP = L.n / L.b;
  const size_t outR = dg_mode ? size_t(nR) * L.b * L.b : size_t(nR) * L.b * (L.b - 1) / 2;
  const size_t outP = dg_mode ? size_t(nP) * L.b * L.b : size_t(nP) * L.b * (L.b - 1) / 2;
  float* oR = dg_mode ? dGR : dqR;
  float* oP = dg_mode ? dGP : dqP;
  if (T == 0) {
    if (!accumulate) {
      POETX_CUDA(cudaMemsetAsync(oR, 0, sizeof(float) * outR, st));
      POETX_CUDA(cudaMemsetAsync(oP, 0, sizeof(float) * outP, st));
    }
    return POETX_OK;
  }
  if (!xg_save) POETX_TRY(check_ptr(x));
  if (y_save && !aligned16(y_save)) return POETX_E_ALIGN;
  POETX_TRY(check_ptr(dz));
  if (xg_save && !aligned16(xg_save)) return POETX_E_ALIGN;
  if (dx && !aligned16(dx)) return POETX_E_ALIGN;
  const bool recompute = y_save == nullptr;
  if (!ws || ws_bytes < (recompute ? bwd_recompute_ws(layer, T) : bwd_ws(layer, T))) return POETX_E_WORKSPACE;
  int dev;
  POETX_TRY(current_device(&dev));
  const int et = elem_type(L.dtype);
  const size_t es = dtype_size(L.dtype);
  const bool tc_path = use_tc(L.dtype);
  const int64_t mx = L.m > L.n ? L.m : L.n;
  const size_t bb = size_t(L.b) * L.b;
  const int sP = dg_splits(nP, L.b, T, L.dtype), sR = dg_splits(nR, L.b, T, L.dtype);
  Carver c(ws, ws_bytes);
  void* bufA = c.take<uint8_t>(es * T * mx);
  void* bufB = c.take<uint8_t>(es * T * mx);
  void* dU = c.take<uint8_t>(es * T * L.m);
  float* partP = c.take<float>(sizeof(float) * sP * nP * bb);
  float* partR = c.take<float>(sizeof(float) * sR * nR * bb);
  // dG mode: a single split without accumulation goes straight to dG
  if (dg_mode && !accumulate && sP == 1) partP = dGP;
  if (dg_mode && !accumulate && sR == 1) partR = dGR;

  if (recompute) {
    // "mem" variant: Y was not kept; recompute it from x (Xg, then Y as in the forward)
    void* Ybuf = c.take<uint8_t>(es * T * L.n);
    void* Xbuf = c.take<uint8_t>(es * T * L.m);
    if (!xg_save) {
      PROFILED(ST_PERMUTE, st, POETX_CUDA(permute_dt(L.dtype, x, Xbuf, T, L.m, L.permR, 0, st, dev)));
      xg_save = Xbuf;
    }
    // the forward's Y, by the same arithmetic (dU, written only later, holds U or the folded weight)
    POETX_CUDA(y_from_xg(L, T, xg_save, Ybuf, dU, st, dev));
    y_save = Ybuf;
  }

  // dV = dz Psi_P^T
  void* dV = bufA;
  PROFILED(ST_PERMUTE, st, POETX_CUDA(permute_dt(L.dtype, dz, dV, T, L.n, L.permP, 0, st, dev)));
  // dY_j = dV_j G_Pj^T and dG_Pj = Y_j^T dV_j (split over tokens): one kernel
  // reading dV once (b = 256 bf16), else two GEMMs.  With POETX_FOLD_P and
  // T > m (bf16) dY is not formed at all: G_P is folded into the weight (W_P = Diag(G_P)^T W~,
  // [n][m], one weight-sized pass) and dU = dV W_P below, so only the dG
  // product reads dV here.
  void* dY = bufB;
  const bool fold_p = fold_p_into_weight(L, T);
  if (fold_p) {
    POETX_CUDA(fold_p_rows(L, L.W, bufB, st, dev));
    PROFILED(ST_DG, st, POETX_CUDA(launch_gemm(blockgrad_desc(y_save, dV, et, T, L.n, L.b, sP, partP), tc_path, st, dev)));
  } else if (use_pair_bdg(L)) {
    PROFILED(ST_BDG, st, POETX_CUDA(launch_bdg(dV, y_save, L.GP, dY, partP, T, L.n, sP, st, dev)));
  } else {
    PROFILED(ST_BLOCKDIAG, st, POETX_CUDA(launch_gemm(blockdiag_desc(dV, et, T, L.n, L.b, L.GP, true, dY, et), tc_path, st, dev)));
    PROFILED(ST_DG, st, POETX_CUDA(launch_gemm(blockgrad_desc(y_save, dV, et, T, L.n, L.b, sP, partP), tc_path, st, dev)));
  }
  // dU = dY W~^T  (B(k=j', n=i') = W[j'][i'], MN-major), or dU = dV W_P
  {
    GemmDesc g;
    g.M = static_cast<int>(T);
    g.N = L.m;
    g.K = L.n;
    g.A = colblocks_view(fold_p ? dV : dY, et, T, L.n, 0);
    Operand2D b;
    b.ptr = fold_p ? bufB : L.W;
    b.et = et;
    b.rows = L.n;
    b.cols = L.m;
    b.ld = L.m;
    b.mn_major = true;
    g.B = b;
    g.C.ptr = dU;
    g.C.et = et;
    g.C.ld = L.m;
    g.C.view_rows = T;
    g.C.view_cols = L.m;
    PROFILED(ST_W0, st, POETX_CUDA(launch_gemm(g, tc_path, st, dev)));
  }
  // Xg = x Psi_R^T: the forward's copy when it saved one, else re-gathered (dV is dead)
  const void* Xg = xg_save;
  if (!Xg) {
    Xg = bufA;
    PROFILED(ST_PERMUTE, st, POETX_CUDA(permute_dt(L.dtype, x, bufA, T, L.m, L.permR, 0, st, dev)));
  }
  // dXg_j = dU_j G_Rj^T (dY is dead; only with dx) and dG_Rj = Xg_j^T dU_j
  void* dXg = bufB;
  if (use_pair_bdg(L)) {
    PROFILED(ST_BDG, st, POETX_CUDA(launch_bdg(dU, Xg, L.GR, dx ? dXg : nullptr, partR, T, L.m, sR, st, dev)));
  } else {
    if (dx) PROFILED(ST_BLOCKDIAG, st, POETX_CUDA(launch_gemm(blockdiag_desc(dU, et, T, L.m, L.b, L.GR, true, dXg, et), tc_path, st, dev)));
    PROFILED(ST_DG, st, POETX_CUDA(launch_gemm(blockgrad_desc(Xg, dU, et, T, L.m, L.b, sR, partR), tc_path, st, dev)));
  }
  // dx = dXg Psi_R
  if (dx) PROFILED(ST_PERMUTE, st, POETX_CUDA(permute_dt(L.dtype, dXg, dx, T, L.m, L.permR, 1, st, dev)));
  if (dg_mode) {
    // dG = fixed-order sum of the token splits (skipped when the GEMM wrote dG)
    const bool sumP = partP != dGP, sumR = partR != dGR;
    if (sumP || sumR) {
      const int64_t n4P = sumP ? int64_t(nP) * int64_t(bb) / 4 : 0;
      const int64_t n4R = sumR ? int64_t(nR) * int64_t(bb) / 4 : 0;
      PROFILED(ST_REDUCE, st,
               sum_splits2_kernel<<<grid_for(n4P + n4R, 256, dev), 256, 0, st>>>(
                   reinterpret_cast<const float4*>(partP), sP, n4P, reinterpret_cast<float4*>(dGP),
                   reinterpret_cast<const float4*>(partR), sR, n4R, reinterpret_cast<float4*>(dGR), accumulate));
      POETX_CUDA(cudaGetLastError());
    }
    return POETX_OK;
  }
  // dq from the dG partial sums of both sides (fixed-order reduction of the
  // token splits inside the CNP backward)
  POETX_TRY(cnp_backward2(L.b, L.dtype, L.qP, nP, partP, sP, dqP, L.qR, nR, partR, sR, dqR, accumulate, c, st, dev));
  return POETX_OK;
}

poetx_status poetx_backward(const poetx_layer* layer, int64_t T, const void* x, const void* y_save,
                            const void* xg_save, const void* dz, void* dx, float* dqR, float* dqP,
                            int32_t accumulate, void* ws, size_t ws_bytes, void* stream) {
  POETX_TRY(check_ptr(dqR));
  POETX_TRY(check_ptr(dqP));
  return backward_impl(layer, T, x, y_save, xg_save, dz, dx, dqR, dqP, nullptr, nullptr, accumulate, ws, ws_bytes,
                       stream);
}

poetx_status poetx_backward_dG(const poetx_layer* layer, int64_t T, const void* x, const void* y_save,
                               const void* xg_save, const void* dz, void* dx, float* dGR, float* dGP,
                               int32_t accumulate, void* ws, size_t ws_bytes, void* stream) {
  POETX_TRY(check_ptr(dGR));
  POETX_TRY(check_ptr(dGP));
  return backward_impl(layer, T, x, y_save, xg_save, dz, dx, nullptr, nullptr, dGR, dGP, accumulate, ws, ws_bytes,
                       stream);
}

poetx_status poetx_merge(const poetx_layer* layer, const int32_t* new_permR, const int32_t* new_permP,
                         void* W_out, void* ws, size_t ws_bytes, void* stream) {
  POETX_TRY(check_layer(layer));
  POETX_TRY(check_ptr(new_permR));
  POETX_TRY(check_ptr(new_permP));
  POETX_TRY(check_ptr(W_out));
  const poetx_layer& L = *layer;
  const size_t es = dtype_size(L.dtype);
  const size_t wbytes = es * size_t(L.n) * L.m;
  {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(L.W), b0 = reinterpret_cast<uintptr_t>(W_out);
    if (a0 < b0 + wbytes && b0 < a0 + wbytes) return POETX_E_ARG;
  }
  if (!ws || ws_bytes < merge_ws(layer)) return POETX_E_WORKSPACE;
  int dev;
  POETX_TRY(current_device(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int et = elem_type(L.dtype);
  const bool tc_path = use_tc(L.dtype);
  const int nR = L.m / L.b, nP = L.n / L.b;
  const size_t nm = size_t(L.n) * L.m;
  Carver c(ws, ws_bytes);
  float* B1t = c.take<float>(sizeof(float) * nm);
  float* At = c.take<float>(sizeof(float) * nm);
  float* GPt = c.take<float>(sizeof(float) * size_t(nP) * L.b * L.b);
  int32_t* invR = c.take<int32_t>(sizeof(int32_t) * L.m);
  int32_t* invP = c.take<int32_t>(sizeof(int32_t) * L.n);
  int32_t* sigR = c.take<int32_t>(sizeof(int32_t) * L.m);
  int32_t* sigP = c.take<int32_t>(sizeof(int32_t) * L.n);

  // Stored W~ = (Psi_R W0 Psi_P^T)^T.  New weight R W0 P in the old frame is
  // A' = Diag(G_R) W~ Diag(G_P), stored transposed:
  //   At = Diag(G_P)^T . W . Diag(G_R)^T     ([n][m])
  // pass 1: B1t = Diag(G_R) . W^T ([m][n]); block i: B1t[ib + r][c] = sum_k G_Ri[r][k] W[c][ib + k]
  {
    GemmDesc g;
    g.M = L.b;
    g.N = L.n;
    g.K = L.b;
    g.batch = nR;
    g.A = blocks_view(L.GR, et, nR, L.b, true);          // A(r, k) = G_Ri[r][k]
    g.B = colblocks_view(L.W, et, L.n, L.m, L.b);        // B(k, c) = W[c][ib + k]
    g.C.ptr = B1t;
    g.C.et = ET_F32;
    g.C.ld = L.n;
    g.C.batch_stride = int64_t(L.b) * L.n;
    g.C.view_rows = L.m;
    g.C.view_cols = L.n;
    g.C.b_row = L.b;
    PROFILED(ST_MERGE, st, POETX_CUDA(launch_gemm(g, tc_path, st, dev)));
  }
  // pass 2: At[jb + r][c] = sum_k G_Pj[k][r] B1t[c][jb + k]  (G_Pj^T, fp32, K-major)
  {
    const dim3 tgrid((L.b + 31) / 32, (L.b + 31) / 32, nP), tblock(32, 8);
    if (L.dtype == POETX_BF16)
      PROFILED(ST_MERGE, st, transpose_blocks_kernel<<<tgrid, tblock, 0, st>>>(
                                 static_cast<const __nv_bfloat16*>(L.GP), GPt, L.b));
    else
      PROFILED(ST_MERGE, st,
               transpose_blocks_kernel<<<tgrid, tblock, 0, st>>>(static_cast<const float*>(L.GP), GPt, L.b));
    POETX_CUDA(cudaGetLastError());
    GemmDesc g;
    g.M = L.b;
    g.N = L.m;
    g.K = L.b;
    g.batch = nP;
    g.A = blocks_view(GPt, ET_F32, nP, L.b, true);       // A(r, k) = G_Pj[k][r]
    g.B = colblocks_view(B1t, ET_F32, L.m, L.n, L.b);    // B(k, c) = B1t[c][jb + k]
    g.C.ptr = At;
    g.C.et = ET_F32;
    g.C.ld = L.m;
    g.C.batch_stride = int64_t(L.b) * L.m;
    g.C.view_rows = L.n;
    g.C.view_cols = L.m;
    g.C.b_row = L.b;
    PROFILED(ST_MERGE, st, POETX_CUDA(launch_gemm(g, tc_path, st, dev)));
  }
  // New frame: W'[j'][i'] = At[sigP[j']][sigR[i']], sig = perm_old^-1 o perm_new.
  invert_perm_kernel<<<(L.m + 255) / 256, 256, 0, st>>>(L.permR, invR, L.m);
  invert_perm_kernel<<<(L.n + 255) / 256, 256, 0, st>>>(L.permP, invP, L.n);
  compose_perm_kernel<<<(L.m + 255) / 256, 256, 0, st>>>(invR, new_permR, sigR, L.m);
  compose_perm_kernel<<<(L.n + 255) / 256, 256, 0, st>>>(invP, new_permP, sigP, L.n);
  POETX_CUDA(cudaGetLastError());
  if (L.dtype == POETX_BF16)
    POETX_CUDA(gather(static_cast<const float*>(At), L.m, L.n, static_cast<__nv_bfloat16*>(W_out), L.m, L.n, L.m,
                      sigR, sigP, st, dev));
  else
    POETX_CUDA(gather(static_cast<const float*>(At), L.m, L.n, static_cast<float*>(W_out), L.m, L.n, L.m, sigR, sigP,
                      st, dev));
  // Reset: Q = 0, G = I.
  POETX_CUDA(cudaMemsetAsync(L.qR, 0, sizeof(float) * size_t(nR) * L.b * (L.b - 1) / 2, st));
  POETX_CUDA(cudaMemsetAsync(L.qP, 0, sizeof(float) * size_t(nP) * L.b * (L.b - 1) / 2, st));
  const int64_t cR = int64_t(nR) * L.b * L.b, cP = int64_t(nP) * L.b * L.b;
  if (L.dtype == POETX_BF16) {
    identity_blocks_kernel<__nv_bfloat16>
        <<<grid_for(cR, 256, dev), 256, 0, st>>>(static_cast<__nv_bfloat16*>(L.GR), nR, L.b);
    identity_blocks_kernel<__nv_bfloat16>
        <<<grid_for(cP, 256, dev), 256, 0, st>>>(static_cast<__nv_bfloat16*>(L.GP), nP, L.b);
  } else {
    identity_blocks_kernel<float><<<grid_for(cR, 256, dev), 256, 0, st>>>(static_cast<float*>(L.GR), nR, L.b);
    identity_blocks_kernel<float><<<grid_for(cP, 256, dev), 256, 0, st>>>(static_cast<float*>(L.GP), nP, L.b);
  }
  POETX_CUDA(cudaGetLastError());
  return POETX_OK;
}

poetx_status poetx_check_perm(const int32_t* perm, int32_t len, int32_t* d_ok, void* ws, size_t ws_bytes,
                              void* stream) {
  if (len <= 0) return POETX_E_ARG;
  POETX_TRY(check_ptr(perm));
  if (!d_ok) return POETX_E_ARG;
  if (!ws || ws_bytes < poetx_check_perm_workspace_bytes(len)) return POETX_E_WORKSPACE;
  int dev;
  POETX_TRY(current_device(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c(ws, ws_bytes);
  int32_t* hist = c.take<int32_t>(sizeof(int32_t) * len);
  POETX_CUDA(cudaMemsetAsync(hist, 0, sizeof(int32_t) * len, st));
  set_int_kernel<<<1, 1, 0, st>>>(d_ok, 1);
  perm_histogram_kernel<<<(len + 255) / 256, 256, 0, st>>>(perm, hist, len, d_ok);
  perm_check_kernel<<<(len + 255) / 256, 256, 0, st>>>(hist, len, d_ok);
  POETX_CUDA(cudaGetLastError());
  return POETX_OK;
}

int32_t poetx_profile_stage_count(void) { return ST_COUNT; }

const char* poetx_profile_stage_name(int32_t stage) {
  if (stage < 0 || stage >= ST_COUNT) return "unknown";
  return kStageNames[stage];
}

poetx_status poetx_profile_begin(void) {
  Profiler& P = profiler();
  std::lock_guard<std::mutex> g(P.mu);
  P.on = true;
  P.used = 0;
  P.recs.clear();
  P.done.clear();
  return POETX_OK;
}

poetx_status poetx_profile_end(double* ms_per_stage, int64_t* launches_per_stage, int32_t nstages) {
  if (!ms_per_stage || !launches_per_stage || nstages < 0) return POETX_E_ARG;
  Profiler& P = profiler();
  std::lock_guard<std::mutex> g(P.mu);
  for (int i = 0; i < nstages; ++i) {
    ms_per_stage[i] = 0.0;
    launches_per_stage[i] = 0;
  }
  poetx_status st = POETX_OK;
  for (const auto& r : P.recs) {
    if (cudaEventSynchronize(P.pool[r.second + 1]) != cudaSuccess) {
      (void)cudaGetLastError();
      st = POETX_E_CUDA;
      break;
    }
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, P.pool[r.second], P.pool[r.second + 1]) != cudaSuccess) {
      (void)cudaGetLastError();
      st = POETX_E_CUDA;
      break;
    }
    if (r.first < nstages) {
      ms_per_stage[r.first] += ms;
      launches_per_stage[r.first] += 1;
    }
    P.done.emplace_back(r.first, ms);
  }
  P.on = false;
  P.used = 0;
  P.recs.clear();
  return st;
}

int32_t poetx_profile_records(int32_t* stages, float* ms, int32_t max_records) {
  Profiler& P = profiler();
  std::lock_guard<std::mutex> g(P.mu);
  const int32_t n = static_cast<int32_t>(P.done.size());
  if (!stages || !ms || max_records <= 0) return n;
  const int32_t k = n < max_records ? n : max_records;
  for (int32_t i = 0; i < k; ++i) {
    stages[i] = P.done[i].first;
    ms[i] = P.done[i].second;
  }
  return n;
}

}  // extern "C"

// ---------------------------------------------------------------- fixed-scratch CNP build
// Some callers cannot allocate device memory when they build G: a host
// program that links only this C library and has no device allocator of its
// own, or a serving process that reserves its whole memory budget at start-up
// and forbids allocations afterwards.  For them poetx_cnp_build_fixed takes
// its scratch (Q, S and H for every block) from this file-scope device array
// instead of a caller workspace.  The array is kFixedScratchBytes on every
// GPU that loads the library, for the life of the process: b = 256 bf16
// builds of up to 47 blocks (the pair kernel takes 128 KiB per block plus
// three per pair of SMs), other builds of up to ~2.09e6 fp32 elements of Q
// (b = 512: 7 blocks).  Host code must
// not hand the symbol itself to a kernel (on the host it only names the
// array); the device address comes from cudaGetSymbolAddress, looked up once
// per device on that device's first call.
constexpr size_t kFixedScratchBytes = size_t(24) << 20;
static __device__ __align__(256) unsigned char g_cnp_fixed_scratch[kFixedScratchBytes];

namespace {
std::mutex g_fixed_mu;
void* g_fixed_scratch_ptr[64] = {nullptr};

// Device address of the fixed scratch on the current device `dev`.
poetx_status fixed_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> g(g_fixed_mu);
  if (!g_fixed_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_cnp_fixed_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return POETX_E_CUDA;
    }
    g_fixed_scratch_ptr[dev] = p;
  }
  *out = g_fixed_scratch_ptr[dev];
  return POETX_OK;
}
}  // namespace

extern "C" poetx_status poetx_cnp_build_fixed(int32_t nblk, int32_t b, const float* q, int32_t dtype, void* G,
                                              void* stream) {
  POETX_TRY(check_dtype_b(dtype, b));
  if (nblk < 0) return POETX_E_ARG;
  if (nblk == 0) return POETX_OK;
  POETX_TRY(check_ptr(q));
  POETX_TRY(check_ptr(G));
  int dev;
  POETX_TRY(current_device(&dev));
  // the scratch the build will carve: the fused pair kernel's bf16 operand
  // region (b = 256 bf16), else Q, S and H in fp32 for every block; requests
  // that do not fit are refused before anything is queued
  const size_t need = kAlign + (use_pair_cnp(b, dtype) ? cnp_pair_bytes(nblk, false, false, dev)
                                                       : 3 * cnp_units(nblk, b));
  if (need > kFixedScratchBytes) return POETX_E_WORKSPACE;  // too many blocks for the fixed scratch
  void* scratch = nullptr;
  POETX_TRY(fixed_scratch(dev, &scratch));
  // Every scratch matrix (Q, S, H, or the pair kernel's bf16 operands) is
  // written in full before it is read: nothing to clear.
  Carver c(scratch, kFixedScratchBytes);
  return cnp_build2(b, dtype, q, nblk, G, nullptr, 0, nullptr, c, static_cast<cudaStream_t>(stream), dev);
}

// ---------------------------------------------------------------- failure-path self-test
// One warp waits on an mbarrier that no thread ever arrives on, through the
// same bounded wait the GEMM and copy kernels use, with a short limit: the
// wait gives up, records DERR_GEMM_WAIT in the sticky error word and the
// kernel returns normally.  No copy, MMA or TMEM allocation is involved, so
// nothing is left in flight.  out[0] = 1 if the wait ended by an arrival
// (never expected), out[1] = nanoseconds waited.
namespace {
__global__ void stalled_wait_kernel(uint64_t limit_ns, unsigned long long* out) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = global_ns();
    const bool arrived = mbar_wait_for(smem_u32(&bar), 0, DERR_GEMM_WAIT, limit_ns);
    out[0] = arrived ? 1ull : 0ull;
    out[1] = global_ns() - t0;
  }
}
}  // namespace

extern "C" poetx_status poetx_selftest_wait_timeout(uint32_t limit_us, unsigned long long* d_out, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return POETX_E_ARG;
  if (!d_out) return POETX_E_ARG;
  if (reinterpret_cast<uintptr_t>(d_out) & 7u) return POETX_E_ALIGN;
  int dev;
  POETX_TRY(current_device(&dev));
  stalled_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(uint64_t(limit_us) * 1000ull, d_out);
  POETX_CUDA(cudaGetLastError());
  return POETX_OK;
}

// ---------------------------------------------------------------- POET-XQ weight storage
extern "C" poetx_status poetx_weight_quantize(int32_t n, int32_t m, const void* W, int32_t dtype, int8_t* Wq,
                                              float* scale, void* stream) {
  if (dtype != POETX_FP32 && dtype != POETX_BF16) return POETX_E_DTYPE;
  if (n < 0 || m <= 0) return POETX_E_ARG;
  if (n == 0) return POETX_OK;
  POETX_TRY(check_ptr(W));
  POETX_TRY(check_ptr(Wq));
  POETX_TRY(check_ptr(scale));
  int dev;
  POETX_TRY(current_device(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int grid = n < sm_count(dev) * 8 ? n : sm_count(dev) * 8;
  if (dtype == POETX_BF16)
    quantize_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), n, m, Wq, scale);
  else
    quantize_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const float*>(W), n, m, Wq, scale);
  POETX_CUDA(cudaGetLastError());
  return POETX_OK;
}

extern "C" poetx_status poetx_weight_dequantize(int32_t n, int32_t m, const int8_t* Wq, const float* scale,
                                                int32_t dtype, void* W, void* stream) {
  if (dtype != POETX_FP32 && dtype != POETX_BF16) return POETX_E_DTYPE;
  if (n < 0 || m <= 0) return POETX_E_ARG;
  if (n == 0) return POETX_OK;
  POETX_TRY(check_ptr(W));
  POETX_TRY(check_ptr(Wq));
  POETX_TRY(check_ptr(scale));
  int dev;
  POETX_TRY(current_device(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t total = int64_t(n) * m;
  if (dtype == POETX_BF16 && m % 16 == 0) {
    PROFILED(ST_DEQUANT, st,
             dequantize_rows_bf16x16_kernel<<<grid_for(total / 16, 256, dev), 256, 0, st>>>(
                 Wq, scale, n, m, static_cast<__nv_bfloat16*>(W)));
  } else if (dtype == POETX_BF16) {
    PROFILED(ST_DEQUANT, st,
             dequantize_rows_kernel<<<grid_for(total, 256, dev), 256, 0, st>>>(Wq, scale, n, m,
                                                                              static_cast<__nv_bfloat16*>(W)));
  } else {
    PROFILED(ST_DEQUANT, st,
             dequantize_rows_kernel<<<grid_for(total, 256, dev), 256, 0, st>>>(Wq, scale, n, m, static_cast<float*>(W)));
  }
  POETX_CUDA(cudaGetLastError());
  return POETX_OK;
}

// ---------------------------------------------------------------- optimizer step on packed q
extern "C" poetx_status poetx_adamw_step(int64_t n, float* q, const float* grad, float* m1, float* m2, float lr,
                                         float beta1, float beta2, float eps, float weight_decay, int32_t step,
                                         void* stream) {
  if (n < 0 || step < 1) return POETX_E_ARG;
  if (n == 0) return POETX_OK;
  POETX_TRY(check_ptr(q));
  POETX_TRY(check_ptr(grad));
  POETX_TRY(check_ptr(m1));
  POETX_TRY(check_ptr(m2));
  int dev;
  POETX_TRY(current_device(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(beta1), step));
  const float bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(beta2), step));
  PROFILED(ST_OPTIM, st,
           adamw_kernel<<<grid_for((n + 3) / 4, 256, dev), 256, 0, st>>>(n, q, grad, m1, m2, lr, beta1, beta2, eps,
                                                                         weight_decay, bc1, bc2));
  POETX_CUDA(cudaGetLastError());
  return POETX_OK;
}
