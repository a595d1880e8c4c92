// Permutation traffic of the layer (POET-X write-up, section 2: R = Psi^T
// Diag(G) Psi).  With perm[i'] the natural index at Psi-frame position i':
//   gather : out[r][c]            = in[rowmap? rowmap[r] : r][colmap[c]]
//   scatter: out[rowmap? rowmap[r] : r][colmap[c]] = in[r][c]
// A block stages whole rows in shared memory, so global reads and writes are
// contiguous 16-byte vectors and only the shared-memory side is permuted.
// Out-of-range indices are skipped (zero written) and flagged in the device
// error word.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace poetx {

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

template <typename Tin, typename Tout>
__device__ __forceinline__ Tout convert(Tin v) {
  if constexpr (std::is_same<Tin, Tout>::value) return v;
  else return from_f32<Tout>(to_f32<Tin>(v));
}

// Copy `count` elements of a row into shared memory (16-byte vectors when the
// row is 16-byte aligned and a whole number of vectors).
template <typename T>
__device__ __forceinline__ void row_to_smem(const T* __restrict__ src, T* dst, int count) {
  constexpr int V = 16 / sizeof(T);
  if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0 && count % V == 0) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    for (int i = threadIdx.x; i < count / V; i += blockDim.x) d4[i] = __ldg(s4 + i);
  } else {
    for (int i = threadIdx.x; i < count; i += blockDim.x) dst[i] = src[i];
  }
}

template <typename T>
__device__ __forceinline__ void smem_to_row(const T* src, T* __restrict__ dst, int count) {
  constexpr int V = 16 / sizeof(T);
  if ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0 && count % V == 0) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    for (int i = threadIdx.x; i < count / V; i += blockDim.x) d4[i] = s4[i];
  } else {
    for (int i = threadIdx.x; i < count; i += blockDim.x) dst[i] = src[i];
  }
}

// rows_per_iter rows are staged per pass (shared memory = rows_per_iter *
// cols * sizeof(Tin)).
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) gather_kernel(const Tin* __restrict__ in, int64_t ld_in, int64_t in_rows,
                                                     Tout* __restrict__ out, int64_t ld_out, int64_t rows, int cols,
                                                     const int32_t* __restrict__ colmap,
                                                     const int32_t* __restrict__ rowmap, int rows_per_iter) {
  extern __shared__ __align__(128) uint8_t sm_raw[];
  Tin* sm = reinterpret_cast<Tin*>(sm_raw);
  constexpr int VO = 16 / sizeof(Tout);
  const bool vec_out = (cols % VO == 0) && (ld_out % VO == 0) && ((reinterpret_cast<uintptr_t>(out) & 15u) == 0);
  for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_iter; r0 < rows;
       r0 += static_cast<int64_t>(gridDim.x) * rows_per_iter) {
    const int nr = static_cast<int>(rows - r0 < rows_per_iter ? rows - r0 : rows_per_iter);
    for (int q = 0; q < nr; ++q) {
      int64_t sr = r0 + q;
      if (rowmap) sr = rowmap[sr];
      if (sr < 0 || sr >= in_rows) {
        if (threadIdx.x == 0) record_error(DERR_BAD_INDEX);
        for (int i = threadIdx.x; i < cols; i += blockDim.x) sm[q * cols + i] = Tin(0.f);
      } else {
        row_to_smem(in + sr * ld_in, sm + q * cols, cols);
      }
    }
    __syncthreads();
    for (int q = 0; q < nr; ++q) {
      const Tin* srow = sm + q * cols;
      Tout* orow = out + (r0 + q) * ld_out;
      if (vec_out) {
        for (int v = threadIdx.x; v < cols / VO; v += blockDim.x) {
          union {
            uint4 u;
            Tout e[VO];
          } pk;
#pragma unroll
          for (int i = 0; i < VO; ++i) {
            const int s = colmap[v * VO + i];
            if (s < 0 || s >= cols) {
              record_error(DERR_BAD_INDEX);
              pk.e[i] = from_f32<Tout>(0.f);
            } else {
              pk.e[i] = convert<Tin, Tout>(srow[s]);
            }
          }
          reinterpret_cast<uint4*>(orow)[v] = pk.u;
        }
      } else {
        for (int c = threadIdx.x; c < cols; c += blockDim.x) {
          const int s = colmap[c];
          if (s < 0 || s >= cols) {
            record_error(DERR_BAD_INDEX);
            orow[c] = from_f32<Tout>(0.f);
          } else {
            orow[c] = convert<Tin, Tout>(srow[s]);
          }
        }
      }
    }
    __syncthreads();
  }
}

template <typename T>
__global__ void __launch_bounds__(256) scatter_kernel(const T* __restrict__ in, int64_t ld_in, T* __restrict__ out,
                                                      int64_t ld_out, int64_t out_rows, int64_t rows, int cols,
                                                      const int32_t* __restrict__ colmap,
                                                      const int32_t* __restrict__ rowmap, int rows_per_iter) {
  extern __shared__ __align__(128) uint8_t sm_raw[];
  T* sm = reinterpret_cast<T*>(sm_raw);
  constexpr int V = 16 / sizeof(T);
  const bool vec_in = (cols % V == 0) && (ld_in % V == 0) && ((reinterpret_cast<uintptr_t>(in) & 15u) == 0);
  for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_iter; r0 < rows;
       r0 += static_cast<int64_t>(gridDim.x) * rows_per_iter) {
    const int nr = static_cast<int>(rows - r0 < rows_per_iter ? rows - r0 : rows_per_iter);
    for (int q = 0; q < nr; ++q) {
      const T* irow = in + (r0 + q) * ld_in;
      T* srow = sm + q * cols;
      if (vec_in) {
        for (int v = threadIdx.x; v < cols / V; v += blockDim.x) {
          union {
            uint4 u;
            T e[V];
          } pk;
          pk.u = __ldg(reinterpret_cast<const uint4*>(irow) + v);
#pragma unroll
          for (int i = 0; i < V; ++i) {
            const int d = colmap[v * V + i];
            if (d < 0 || d >= cols) record_error(DERR_BAD_INDEX);
            else srow[d] = pk.e[i];
          }
        }
      } else {
        for (int c = threadIdx.x; c < cols; c += blockDim.x) {
          const int d = colmap[c];
          if (d < 0 || d >= cols) record_error(DERR_BAD_INDEX);
          else srow[d] = irow[c];
        }
      }
    }
    __syncthreads();
    for (int q = 0; q < nr; ++q) {
      int64_t dr = r0 + q;
      if (rowmap) dr = rowmap[dr];
      if (dr < 0 || dr >= out_rows) {
        if (threadIdx.x == 0) record_error(DERR_BAD_INDEX);
        continue;
      }
      smem_to_row(sm + q * cols, out + dr * ld_out, cols);
    }
    __syncthreads();
  }
}

// Column permutation of row-major activations on the hot path, fed by bulk
// copies.  out[r][c] = in[r][map[c]] (gather), or with `inverse` set
// out[r][map[c]] = in[r][c] (scatter, done as a gather through the inverse
// map, which every block first builds in shared memory).  Rows are contiguous
// (leading dimension == cols), so a chunk of rows_per_stage rows is one
// contiguous bulk copy; two stages are double-buffered: while the block
// permutes one chunk out of shared memory, the next one is in flight.  Each
// thread writes whole 16-byte vectors, so the global stores are coalesced.
// Shared memory: cols 16-bit indices + 2 * rows_per_stage * cols * sizeof(T).
template <typename T>
__global__ void __launch_bounds__(256) permute_rows_kernel(const T* __restrict__ in, T* __restrict__ out, int64_t rows,
                                                           int cols, const int32_t* __restrict__ map, int inverse,
                                                           int rows_per_stage) {
  extern __shared__ __align__(128) uint8_t sm_raw[];
  __shared__ __align__(8) uint64_t full_bar[2];
  constexpr int V = 16 / sizeof(T);
  uint16_t* idx = reinterpret_cast<uint16_t*>(sm_raw);
  const size_t idx_bytes = (static_cast<size_t>(cols) * 2 + 127) & ~size_t(127);
  T* stage_base = reinterpret_cast<T*>(sm_raw + idx_bytes);
  const int64_t stage_elems = static_cast<int64_t>(rows_per_stage) * cols;
  const int64_t nchunks = (rows + rows_per_stage - 1) / rows_per_stage;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&full_bar[0]), 1);
    mbar_init(smem_u32(&full_bar[1]), 1);
    fence_barrier_init();
  }
  if (inverse) {
    // entries a non-bijective map never reaches stay 0 (in range)
    for (int c = threadIdx.x; c < cols; c += blockDim.x) idx[c] = 0;
    __syncthreads();
  }
  for (int c = threadIdx.x; c < cols; c += blockDim.x) {
    const int m = map[c];
    if (m < 0 || m >= cols) {
      record_error(DERR_BAD_INDEX);
      if (!inverse) idx[c] = 0;
      continue;
    }
    if (inverse) idx[m] = static_cast<uint16_t>(c);
    else idx[c] = static_cast<uint16_t>(m);
  }
  __syncthreads();

  uint32_t pending = 0;  // stages with a copy in flight (thread 0's view)
  auto issue = [&](int64_t chunk, int s) {
    const int64_t r0 = chunk * rows_per_stage;
    const int64_t nr = rows - r0 < rows_per_stage ? rows - r0 : rows_per_stage;
    const uint32_t bytes = static_cast<uint32_t>(nr * cols * sizeof(T));
    const uint32_t bar = smem_u32(&full_bar[s]);
    // earlier generic-proxy reads of this stage (ordered by the block barrier)
    // come before the async-proxy write
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(smem_u32(stage_base + s * stage_elems), in + r0 * cols, bytes, bar);
    pending |= 1u << s;
  };

  int64_t chunk = blockIdx.x;
  if (threadIdx.x == 0 && chunk < nchunks) issue(chunk, 0);
  uint32_t phase[2] = {0u, 0u};
  bool ok = true;
  for (int it = 0; chunk < nchunks; chunk += gridDim.x, ++it) {
    const int s = it & 1;
    const int64_t next = chunk + gridDim.x;
    if (threadIdx.x == 0 && next < nchunks) issue(next, s ^ 1);
    ok = mbar_wait(smem_u32(&full_bar[s]), phase[s], DERR_PERM_WAIT);
    if (ok) {
      phase[s] ^= 1u;
      pending &= ~(1u << s);
    }
    if (!__syncthreads_and(ok)) break;
    const int64_t r0 = chunk * rows_per_stage;
    const int nr = static_cast<int>(rows - r0 < rows_per_stage ? rows - r0 : rows_per_stage);
    const T* st = stage_base + s * stage_elems;
    const int vpr = cols / V;  // vectors per row
    for (int v = threadIdx.x; v < nr * vpr; v += blockDim.x) {
      const int rr = v / vpr;
      const int c0 = (v - rr * vpr) * V;
      const T* srow = st + static_cast<int64_t>(rr) * cols;
      union {
        uint4 u;
        T e[V];
      } pk;
      if constexpr (V == 8) {
        const uint4 ii = *reinterpret_cast<const uint4*>(idx + c0);
        const uint16_t* iv = reinterpret_cast<const uint16_t*>(&ii);
#pragma unroll
        for (int k = 0; k < 8; ++k) pk.e[k] = srow[iv[k]];
      } else {
        const uint2 ii = *reinterpret_cast<const uint2*>(idx + c0);
        const uint16_t* iv = reinterpret_cast<const uint16_t*>(&ii);
#pragma unroll
        for (int k = 0; k < V; ++k) pk.e[k] = srow[iv[k]];
      }
      reinterpret_cast<uint4*>(out + (r0 + rr) * cols + c0)[0] = pk.u;
    }
    __syncthreads();  // stage s may be refilled next iteration
  }
  if (!ok && threadIdx.x == 0) {
    // let a copy still in flight land before the block exits
    for (int s = 0; s < 2; ++s)
      if (pending & (1u << s)) mbar_wait(smem_u32(&full_bar[s]), phase[s], DERR_PERM_WAIT);
  }
}

// permute_rows_kernel with every thread's index entries held in registers.
// The block gives each thread a fixed set of output vectors: with vpr =
// cols / V vectors per row, thread t owns vectors t, t + 256, ... of every
// row (vpr >= 256), or, when vpr < 256, vector t % vpr of rows t / vpr,
// t / vpr + 256 / vpr, ... of each stage.  So a thread reads its (at most
// MAXV) vectors of indices out of the shared table once, before the first
// stage, instead of once per row: the random 2-byte reads of the staged rows
// are the only shared-memory loads left in the loop.
template <typename T, int MAXV>
__global__ void __launch_bounds__(256) permute_rows_reg_kernel(const T* __restrict__ in, T* __restrict__ out,
                                                               int64_t rows, int cols,
                                                               const int32_t* __restrict__ map, int inverse,
                                                               int rows_per_stage, int idx_in_stage) {
  extern __shared__ __align__(128) uint8_t sm_raw[];
  __shared__ __align__(8) uint64_t full_bar[2];
  constexpr int V = 16 / sizeof(T);
  using IdxVec = typename std::conditional<V == 8, uint4, uint2>::type;  // V 16-bit indices
  const size_t idx_bytes = (static_cast<size_t>(cols) * 2 + 127) & ~size_t(127);
  // the index table is only read before the first stage lands: with
  // idx_in_stage it lives in stage 1, which is first filled after that
  T* stage_base = reinterpret_cast<T*>(sm_raw + (idx_in_stage ? 0 : idx_bytes));
  const int64_t stage_elems = static_cast<int64_t>(rows_per_stage) * cols;
  uint16_t* idx = idx_in_stage ? reinterpret_cast<uint16_t*>(stage_base + stage_elems)
                               : reinterpret_cast<uint16_t*>(sm_raw);
  const int64_t nchunks = (rows + rows_per_stage - 1) / rows_per_stage;
  const int vpr = cols / V;
  const int nthr = static_cast<int>(blockDim.x);
  // this thread's vectors: columns (vec0 + k * nthr) * V for k < nvec, in rows
  // row0, row0 + rstep, ... of each stage
  const bool wide = vpr >= nthr;
  const int rstep = wide ? 1 : nthr / vpr;
  const int vec0 = wide ? static_cast<int>(threadIdx.x) : static_cast<int>(threadIdx.x) % vpr;
  const int row0 = wide ? 0 : static_cast<int>(threadIdx.x) / vpr;
  const bool active = wide || static_cast<int>(threadIdx.x) < rstep * vpr;
  const int nvec = wide ? (vpr - vec0 + nthr - 1) / nthr : 1;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&full_bar[0]), 1);
    mbar_init(smem_u32(&full_bar[1]), 1);
    fence_barrier_init();
  }
  if (inverse) {
    // entries a non-bijective map never reaches stay 0 (in range)
    for (int c = threadIdx.x; c < cols; c += blockDim.x) idx[c] = 0;
    __syncthreads();
  }
  for (int c = threadIdx.x; c < cols; c += blockDim.x) {
    const int m = map[c];
    if (m < 0 || m >= cols) {
      record_error(DERR_BAD_INDEX);
      if (!inverse) idx[c] = 0;
      continue;
    }
    if (inverse) idx[m] = static_cast<uint16_t>(c);
    else idx[c] = static_cast<uint16_t>(m);
  }
  __syncthreads();
  IdxVec myidx[MAXV];
#pragma unroll
  for (int k = 0; k < MAXV; ++k)
    if (active && k < nvec) myidx[k] = *reinterpret_cast<const IdxVec*>(idx + (vec0 + k * nthr) * V);
  __syncthreads();  // every thread has its indices before stage 1 may be overwritten

  uint32_t pending = 0;  // stages with a copy in flight (thread 0's view)
  auto issue = [&](int64_t chunk, int s) {
    const int64_t r0 = chunk * rows_per_stage;
    const int64_t nr = rows - r0 < rows_per_stage ? rows - r0 : rows_per_stage;
    const uint32_t bytes = static_cast<uint32_t>(nr * cols * sizeof(T));
    const uint32_t bar = smem_u32(&full_bar[s]);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(smem_u32(stage_base + s * stage_elems), in + r0 * cols, bytes, bar);
    pending |= 1u << s;
  };

  int64_t chunk = blockIdx.x;
  if (threadIdx.x == 0 && chunk < nchunks) issue(chunk, 0);
  uint32_t phase[2] = {0u, 0u};
  bool ok = true;
  for (int it = 0; chunk < nchunks; chunk += gridDim.x, ++it) {
    const int s = it & 1;
    const int64_t next = chunk + gridDim.x;
    if (threadIdx.x == 0 && next < nchunks) issue(next, s ^ 1);
    ok = mbar_wait(smem_u32(&full_bar[s]), phase[s], DERR_PERM_WAIT);
    if (ok) {
      phase[s] ^= 1u;
      pending &= ~(1u << s);
    }
    if (!__syncthreads_and(ok)) break;
    const int64_t r0 = chunk * rows_per_stage;
    const int nr = static_cast<int>(rows - r0 < rows_per_stage ? rows - r0 : rows_per_stage);
    const T* st = stage_base + s * stage_elems;
    if (active) {
      for (int rr = row0; rr < nr; rr += rstep) {
        const T* srow = st + static_cast<int64_t>(rr) * cols;
        T* orow = out + (r0 + rr) * cols;
#pragma unroll
        for (int k = 0; k < MAXV; ++k) {
          if (k < nvec) {
            const uint16_t* iv = reinterpret_cast<const uint16_t*>(&myidx[k]);
            union {
              uint4 u;
              T e[V];
            } pk;
#pragma unroll
            for (int e = 0; e < V; ++e) pk.e[e] = srow[iv[e]];
            reinterpret_cast<uint4*>(orow + (vec0 + k * nthr) * V)[0] = pk.u;
          }
        }
      }
    }
    __syncthreads();  // stage s may be refilled next iteration
  }
  if (!ok && threadIdx.x == 0) {
    // let a copy still in flight land before the block exits
    for (int s = 0; s < 2; ++s)
      if (pending & (1u << s)) mbar_wait(smem_u32(&full_bar[s]), phase[s], DERR_PERM_WAIT);
  }
}

// inv[perm[i]] = i
__global__ void invert_perm_kernel(const int32_t* __restrict__ perm, int32_t* __restrict__ inv, int len) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= len) return;
  const int p = perm[i];
  if (p < 0 || p >= len) {
    record_error(DERR_BAD_INDEX);
    return;
  }
  inv[p] = i;
}

// out[i] = a[b[i]]
__global__ void compose_perm_kernel(const int32_t* __restrict__ a, const int32_t* __restrict__ b,
                                    int32_t* __restrict__ out, int len) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= len) return;
  const int j = b[i];
  if (j < 0 || j >= len) {
    record_error(DERR_BAD_INDEX);
    out[i] = 0;
    return;
  }
  out[i] = a[j];
}

__global__ void perm_histogram_kernel(const int32_t* __restrict__ perm, int32_t* hist, int len, int32_t* ok) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= len) return;
  const int p = perm[i];
  if (p < 0 || p >= len) {
    *ok = 0;
    return;
  }
  atomicAdd(hist + p, 1);
}

__global__ void perm_check_kernel(const int32_t* __restrict__ hist, int len, int32_t* ok) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < len && hist[i] != 1) *ok = 0;
}

}  // namespace poetx
