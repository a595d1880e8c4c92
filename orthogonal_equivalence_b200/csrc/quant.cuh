// POET-XQ (POET-X write-up, section "POET-XQ：量化训练的额外红利"): the frozen
// base weight is stored quantized and only dequantized at run time, with no
// quantization-aware training.  The write-up fixes neither the format nor
// the granularity; the reading taken here is the plain 8-bit one it compares
// against: int8 codes, symmetric, one fp32 scale per row of the stored
// [n][m] weight (one per output feature), scale = max|row| / 127,
// code = round-half-even(w / scale) clamped to [-127, 127], w ~= code * scale.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace poetx {

template <typename T>
__device__ __forceinline__ float load_f32(const T* p, int64_t i);
template <>
__device__ __forceinline__ float load_f32<float>(const float* p, int64_t i) { return p[i]; }
template <>
__device__ __forceinline__ float load_f32<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

// One block per row: absmax by a block reduction, then the codes.
template <typename T>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const T* __restrict__ W, int64_t rows, int cols,
                                                            int8_t* __restrict__ Wq, float* __restrict__ scale) {
  __shared__ float red[8];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const T* w = W + r * cols;
    float amax = 0.f;
    for (int c = threadIdx.x; c < cols; c += blockDim.x) amax = fmaxf(amax, fabsf(load_f32(w, c)));
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x < 32) {
      float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
      for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    const float s = red[0] / 127.f;
    if (threadIdx.x == 0) scale[r] = s;
    for (int c = threadIdx.x; c < cols; c += blockDim.x) {
      float q = 0.f;
      if (s > 0.f) q = fminf(fmaxf(rintf(load_f32(w, c) / s), -127.f), 127.f);
      Wq[r * cols + c] = static_cast<int8_t>(q);
    }
    __syncthreads();  // red[] is reused by the next row
  }
}

// w = code * scale (fp32 product), rounded once to the weight dtype.
template <typename T>
__global__ void dequantize_rows_kernel(const int8_t* __restrict__ Wq, const float* __restrict__ scale, int64_t rows,
                                       int cols, T* __restrict__ W) {
  const int64_t n = rows * cols;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = static_cast<float>(Wq[i]) * scale[i / cols];
    if constexpr (std::is_same<T, float>::value) W[i] = v;
    else W[i] = __float2bfloat16_rn(v);
  }
}

// 16 codes per thread (one 16-byte load, two 16-byte bf16 stores); cols % 16 == 0.
__global__ void dequantize_rows_bf16x16_kernel(const int8_t* __restrict__ Wq, const float* __restrict__ scale,
                                               int64_t rows, int cols, __nv_bfloat16* __restrict__ W) {
  const int64_t n16 = rows * cols / 16;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float s = scale[(i * 16) / cols];
    const int4 codes = reinterpret_cast<const int4*>(Wq)[i];
    const int8_t* c = reinterpret_cast<const int8_t*>(&codes);
    uint4 out[2];
    uint32_t* o = reinterpret_cast<uint32_t*>(out);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      __nv_bfloat162 h = __floats2bfloat162_rn(static_cast<float>(c[2 * k]) * s, static_cast<float>(c[2 * k + 1]) * s);
      o[k] = *reinterpret_cast<uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(W)[2 * i] = out[0];
    reinterpret_cast<uint4*>(W)[2 * i + 1] = out[1];
  }
}

}  // namespace poetx
