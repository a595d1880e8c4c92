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

// One warp per row of the triangle: lanes read the row's contiguous run of
// q and write Q[i][j] = q (coalesced) and Q[j][i] = -q; lane 0 writes the
// zero diagonal entry.  grid.x covers nblk*b rows, 8 warps per block.
__global__ void unpack_skew_kernel(const float* __restrict__ q, int nblk, int b, float* __restrict__ Q) {
  const int64_t row_global = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row_global >= static_cast<int64_t>(nblk) * b) return;
  const int64_t blk = row_global / b;
  const int i = static_cast<int>(row_global - blk * b);
  const int64_t L = static_cast<int64_t>(b) * (b - 1) / 2;
  const float* qb = q + blk * L;
  float* Qb = Q + blk * b * b;
  const int64_t k0 = tri_index(i, i + 1, b);
  for (int j = i + 1 + lane; j < b; j += 32) {
    const float v = qb[k0 + (j - i - 1)];
    Qb[static_cast<int64_t>(i) * b + j] = v;
    Qb[static_cast<int64_t>(j) * b + i] = -v;
  }
  if (lane == 0) Qb[static_cast<int64_t>(i) * b + i] = 0.f;
}

// out = a*X + c*Y (fp32, n elements)
__global__ void axpby_kernel(const float* __restrict__ X, float a, const float* __restrict__ Y, float c,
                             float* __restrict__ out, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = a * X[i] + c * Y[i];
}

// dq[k(i,j)] (+)= dA[i][j] - dA[j][i]; one block row per (blk, i).
__global__ void fold_skew_kernel(const float* __restrict__ dA, int nblk, int b, float* __restrict__ dq,
                                 int accumulate) {
  const int64_t row_global = blockIdx.x;
  const int64_t blk = row_global / b;
  const int i = static_cast<int>(row_global - blk * b);
  const int64_t L = static_cast<int64_t>(b) * (b - 1) / 2;
  const float* Ab = dA + blk * b * b;
  float* qb = dq + blk * L;
  const int64_t k0 = tri_index(i, i + 1, b);
  for (int j = i + 1 + threadIdx.x; j < b; j += blockDim.x) {
    const float g = Ab[static_cast<int64_t>(i) * b + j] - Ab[static_cast<int64_t>(j) * b + i];
    const int64_t k = k0 + (j - i - 1);
    qb[k] = accumulate ? qb[k] + g : g;
  }
}

// out[e] = sum_{s < splits} part[s*count + e], summed in split order (the
// result does not depend on the launch shape).
__global__ void reduce_splits_kernel(const float* __restrict__ part, int splits, int64_t count,
                                     float* __restrict__ out) {
  const int64_t n4 = count / 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 acc = reinterpret_cast<const float4*>(part)[i];
    for (int s = 1; s < splits; ++s) {
      const float4 v = reinterpret_cast<const float4*>(part + s * count)[i];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    reinterpret_cast<float4*>(out)[i] = acc;
  }
  for (int64_t i = n4 * 4 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float acc = part[i];
    for (int s = 1; s < splits; ++s) acc += part[s * count + i];
    out[i] = acc;
  }
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

}  // namespace poetx
