// Element-wise kernels of the Cayley-Neumann parameterisation (POET-X
// write-up, section 3): unpacking the stored strict upper triangle of the
// skew-symmetric Q, folding a full-matrix gradient back onto the triangle,
// deterministic reduction of split-K partial sums, and small helpers.
//
// Packing order: row-major over i < j, k(i,j) = i(b-1) - i(i-1)/2 + (j-i-1),
// Q[i][j] = +q[k], Q[j][i] = -q[k].
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace poetx {

__device__ __forceinline__ int64_t tri_index(int64_t i, int64_t j, int64_t b) {
  return i * (b - 1) - i * (i - 1) / 2 + (j - i - 1);
}

// G blocks := I (the state right after a merge), in the layer's dtype.
template <typename T>
__global__ void identity_blocks_kernel(T* __restrict__ G, int nblk, int b) {
  const int64_t n = static_cast<int64_t>(nblk) * b * b;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t w = e % (static_cast<int64_t>(b) * b);
    const bool d = (w / b) == (w % b);
    if constexpr (std::is_same<T, float>::value) G[e] = d ? 1.f : 0.f;
    else G[e] = __float2bfloat16_rn(d ? 1.f : 0.f);
  }
}

__global__ void set_int_kernel(int32_t* p, int32_t v) { *p = v; }

// out[t][c][r] = in[t][r][c] for b x b blocks (fp32 out; bf16 in is widened
// exactly).  32 x 32 tiles through shared memory; grid (b/32, b/32, nblk),
// block (32, 8).
template <typename T>
__global__ void transpose_blocks_kernel(const T* __restrict__ in, float* __restrict__ out, int b) {
  __shared__ float tile[32][33];
  const int64_t base = static_cast<int64_t>(blockIdx.z) * b * b;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < b && c < b) {
      if constexpr (std::is_same<T, float>::value) tile[i][threadIdx.x] = in[base + static_cast<int64_t>(r) * b + c];
      else tile[i][threadIdx.x] = __bfloat162float(in[base + static_cast<int64_t>(r) * b + c]);
    }
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = c0 + i, c = r0 + threadIdx.x;
    if (r < b && c < b) out[base + static_cast<int64_t>(r) * b + c] = tile[threadIdx.x][i];
  }
}


// ---------------------------------------------------------------------------
// Two-sided variants: the blocks of G_R and G_P (or of any two block sets
// with the same b) are processed as one batch [0, n0) + [n0, nblk).
// Matrices live in row-strided block arrays: block t starts at t * bs, rows
// ld apart (so a block can sit inside a wider concatenated row).

// Block ranges of up to kMaxSegs sources batched into one launch (the R and
// P sides of one layer, or of several layers): blocks [start[s], start[s+1])
// take their packed triangles from q[s] and (for the build) write G to G[s].
constexpr int kMaxSegs = 32;
struct Segs {
  int n;
  int start[kMaxSegs + 1];
  const float* q[kMaxSegs];
  void* G[kMaxSegs];
};

__device__ __forceinline__ int seg_of(const Segs& sg, int blk) {
  int s = 0;
  while (s + 1 < sg.n && blk >= sg.start[s + 1]) ++s;
  return s;
}

// Unpack packed triangles into Q (and optionally a second copy).  One block
// per 32 x 32 tile (ti, tj) with ti <= tj of one b x b block: row i of the
// tile reads its run of q (contiguous for i < j), writes Q[i][j] = q and,
// through a shared-memory transpose, the mirrored tile Q[j][i] = -q, so both
// the reads and the writes are coalesced.  grid (b/32, b/32, nblk), block
// (32, 8); tiles below the diagonal exit at once.
__global__ void unpack_skew_kernel(const Segs sg, int nblk, int b, float* __restrict__ o1, int64_t ld1, int64_t bs1,
                                   float* __restrict__ o2, int64_t ld2, int64_t bs2) {
  __shared__ float tile[32][33];
  const int ti = blockIdx.y, tj = blockIdx.x, blk = blockIdx.z;
  if (ti > tj || blk >= nblk) return;
  const int64_t L = static_cast<int64_t>(b) * (b - 1) / 2;
  const int sgi = seg_of(sg, blk);
  const float* qb = sg.q[sgi] + (blk - sg.start[sgi]) * L;
  float* A1 = o1 + blk * bs1;
  float* A2 = o2 ? o2 + blk * bs2 : nullptr;
  const int r0 = ti * 32, c0 = tj * 32;
  for (int ii = threadIdx.y; ii < 32; ii += 8) {
    const int i = r0 + ii, j = c0 + threadIdx.x;
    float v = 0.f;
    if (i < b && j < b) {
      if (i < j) v = qb[tri_index(i, j, b)];
      else if (i > j) v = -qb[tri_index(j, i, b)];  // diagonal tile, lower half
      A1[i * ld1 + j] = v;
      if (A2) A2[i * ld2 + j] = v;
    }
    tile[ii][threadIdx.x] = v;
  }
  if (ti == tj) return;  // a diagonal tile is its own mirror
  __syncthreads();
  for (int jj = threadIdx.y; jj < 32; jj += 8) {
    const int j = c0 + jj, i = r0 + threadIdx.x;
    if (i < b && j < b) {
      const float v = -tile[threadIdx.x][jj];
      A1[j * ld1 + i] = v;
      if (A2) A2[j * ld2 + i] = v;
    }
  }
}

// Copy contiguous G blocks [nblk][b][b] (elem_bytes each element) to each
// segment's own G array, 16 bytes per thread.  grid (chunks, nblk).
__global__ void split_blocks_kernel(const Segs sg, const uint8_t* __restrict__ all, int nblk, int64_t block_bytes) {
  const int blk = blockIdx.y;
  if (blk >= nblk) return;
  const int sgi = seg_of(sg, blk);
  const uint4* src = reinterpret_cast<const uint4*>(all + blk * block_bytes);
  uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(sg.G[sgi]) + (blk - sg.start[sgi]) * block_bytes);
  const int64_t n16 = block_bytes / 16;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = src[i];
}

// dG = sum over token splits of the partial products, in split order, for
// both sides; writes dG to o1 (and o2 if given) and dG^T to ot.  One block
// per 32 x 32 tile: thread (x, y) of the (8, 32) block owns row y, columns
// 4x..4x+3 (16-byte loads and stores); the transpose goes through shared
// memory with a padded row, conflict-free.  grid (b/32, b/32, nblk).
// Requires b % 32 == 0 and 16-byte aligned rows.
__global__ void reduce_transpose_kernel(const float* __restrict__ part0, int splits0, int n0,
                                        const float* __restrict__ part1, int splits1, int n1, int b,
                                        float* __restrict__ o1, int64_t ld1, int64_t bs1, float* __restrict__ o2,
                                        int64_t ld2, int64_t bs2, float* __restrict__ ot, int64_t ldt, int64_t bst) {
  __shared__ float tile[32][33];
  const int t = blockIdx.z;
  const float* part;
  int splits;
  int64_t sstride, off;
  const int64_t bb = static_cast<int64_t>(b) * b;
  if (t < n0) {
    part = part0;
    splits = splits0;
    sstride = static_cast<int64_t>(n0) * bb;
    off = t * bb;
  } else {
    part = part1;
    splits = splits1;
    sstride = static_cast<int64_t>(n1) * bb;
    off = (t - n0) * bb;
  }
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const int x = threadIdx.x, y = threadIdx.y;
  const int r = r0 + y, c = c0 + 4 * x;
  const int64_t e = off + static_cast<int64_t>(r) * b + c;
  float4 acc = *reinterpret_cast<const float4*>(part + e);
  for (int s = 1; s < splits; ++s) {
    const float4 v = *reinterpret_cast<const float4*>(part + s * sstride + e);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  *reinterpret_cast<float4*>(o1 + t * bs1 + r * ld1 + c) = acc;
  if (o2) *reinterpret_cast<float4*>(o2 + t * bs2 + r * ld2 + c) = acc;
  tile[y][4 * x] = acc.x;
  tile[y][4 * x + 1] = acc.y;
  tile[y][4 * x + 2] = acc.z;
  tile[y][4 * x + 3] = acc.w;
  __syncthreads();
  // transposed tile: row c0 + y of dG^T holds column c0 + y of dG
  const float4 tv = make_float4(tile[4 * x][y], tile[4 * x + 1][y], tile[4 * x + 2][y], tile[4 * x + 3][y]);
  *reinterpret_cast<float4*>(ot + t * bst + static_cast<int64_t>(c0 + y) * ldt + r0 + 4 * x) = tv;
}

// Same result for any b (scalar, bounds-checked): grid (ceil(b/32),
// ceil(b/32), nblk), block (32, 8).
__global__ void reduce_transpose_any_kernel(const float* __restrict__ part0, int splits0, int n0,
                                            const float* __restrict__ part1, int splits1, int n1, int b,
                                            float* __restrict__ o1, int64_t ld1, int64_t bs1, float* __restrict__ o2,
                                            int64_t ld2, int64_t bs2, float* __restrict__ ot, int64_t ldt,
                                            int64_t bst) {
  __shared__ float tile[32][33];
  const int t = blockIdx.z;
  const int64_t bb = static_cast<int64_t>(b) * b;
  const float* part = t < n0 ? part0 : part1;
  const int splits = t < n0 ? splits0 : splits1;
  const int64_t sstride = static_cast<int64_t>(t < n0 ? n0 : n1) * bb;
  const int64_t off = (t < n0 ? t : t - n0) * bb;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < b && c < b) {
      const int64_t e = off + static_cast<int64_t>(r) * b + c;
      float acc = part[e];
      for (int s = 1; s < splits; ++s) acc += part[s * sstride + e];
      o1[t * bs1 + r * ld1 + c] = acc;
      if (o2) o2[t * bs2 + r * ld2 + c] = acc;
      tile[i][threadIdx.x] = acc;
    }
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = c0 + i, c = r0 + threadIdx.x;
    if (r < b && c < b) ot[t * bst + r * ldt + c] = tile[threadIdx.x][i];
  }
}

// dG (+)= sum over token splits of the partial products, in split order,
// for two independent arrays (the two sides of a layer): part_k holds
// splits_k slices of n4_k float4 each, one slice after the other.  16-byte
// loads and stores, grid-stride over both arrays.
__global__ void sum_splits2_kernel(const float4* __restrict__ part0, int splits0, int64_t n40,
                                   float4* __restrict__ out0, const float4* __restrict__ part1, int splits1,
                                   int64_t n41, float4* __restrict__ out1, int accumulate) {
  const int64_t total = n40 + n41;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const bool first = i < n40;
    const float4* part = first ? part0 : part1;
    float4* out = first ? out0 : out1;
    const int splits = first ? splits0 : splits1;
    const int64_t n4 = first ? n40 : n41;
    const int64_t e = first ? i : i - n40;
    float4 acc = part[e];
    for (int s = 1; s < splits; ++s) {
      const float4 v = part[s * n4 + e];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if (accumulate) {
      const float4 o = out[e];
      acc.x = o.x + acc.x;
      acc.y = o.y + acc.y;
      acc.z = o.z + acc.z;
      acc.w = o.w + acc.w;
    }
    out[e] = acc;
  }
}

// dst += src, 16-byte elements, grid-stride.
__global__ void add_f32x4_kernel(float4* __restrict__ dst, const float4* __restrict__ src, int64_t n4) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = dst[i], b = src[i];
    dst[i] = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
  }
}

// dq[k(i,j)] (+)= dA[i][j] - dA[j][i] for both sides; one block row per
// (blk, i).
__global__ void fold_skew2_kernel(const float* __restrict__ dA, int64_t ld, int64_t bs, int n0, int b,
                                  float* __restrict__ dq0, float* __restrict__ dq1, int accumulate) {
  const int64_t row_global = blockIdx.x;
  const int blk = static_cast<int>(row_global / b);
  const int i = static_cast<int>(row_global - static_cast<int64_t>(blk) * b);
  const int64_t L = static_cast<int64_t>(b) * (b - 1) / 2;
  const float* Ab = dA + blk * bs;
  float* qb = blk < n0 ? dq0 + blk * L : dq1 + (blk - n0) * L;
  const int64_t k0 = tri_index(i, i + 1, b);
  for (int j = i + 1 + threadIdx.x; j < b; j += blockDim.x) {
    const float g = Ab[static_cast<int64_t>(i) * ld + j] - Ab[static_cast<int64_t>(j) * ld + i];
    const int64_t k = k0 + (j - i - 1);
    qb[k] = accumulate ? qb[k] + g : g;
  }
}

}  // namespace poetx
