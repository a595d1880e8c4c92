// Optimizer step on the packed triangles q (the trainable parameters of a
// POET-X layer).  The write-up's get_poet_optimizer is not described; the
// reading taken is AdamW (decoupled weight decay) applied to the packed
// triangles, the plain optimizer of its comparison runs:
//   m <- b1 m + (1-b1) g,  v <- b2 v + (1-b2) g^2,
//   q <- q (1 - lr wd) - lr (m / (1-b1^t)) / (sqrt(v / (1-b2^t)) + eps).
#pragma once

#include <cstdint>

namespace poetx {

__device__ __forceinline__ void adamw_one(float& q, float g, float& m, float& v, float lr, float b1, float b2,
                                          float eps, float wd, float bc1, float bc2) {
  m = b1 * m + (1.f - b1) * g;
  v = b2 * v + (1.f - b2) * g * g;
  q = q * (1.f - lr * wd) - lr * (m / bc1) / (sqrtf(v / bc2) + eps);
}

__global__ void adamw_kernel(int64_t n, float* __restrict__ q, const float* __restrict__ g, float* __restrict__ m,
                             float* __restrict__ v, float lr, float b1, float b2, float eps, float wd, float bc1,
                             float bc2) {
  const int64_t n4 = n / 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 qq = reinterpret_cast<float4*>(q)[i];
    const float4 gg = reinterpret_cast<const float4*>(g)[i];
    float4 mm = reinterpret_cast<float4*>(m)[i];
    float4 vv = reinterpret_cast<float4*>(v)[i];
    adamw_one(qq.x, gg.x, mm.x, vv.x, lr, b1, b2, eps, wd, bc1, bc2);
    adamw_one(qq.y, gg.y, mm.y, vv.y, lr, b1, b2, eps, wd, bc1, bc2);
    adamw_one(qq.z, gg.z, mm.z, vv.z, lr, b1, b2, eps, wd, bc1, bc2);
    adamw_one(qq.w, gg.w, mm.w, vv.w, lr, b1, b2, eps, wd, bc1, bc2);
    reinterpret_cast<float4*>(q)[i] = qq;
    reinterpret_cast<float4*>(m)[i] = mm;
    reinterpret_cast<float4*>(v)[i] = vv;
  }
  for (int64_t i = n4 * 4 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float qq = q[i], mm = m[i], vv = v[i];
    adamw_one(qq, g[i], mm, vv, lr, b1, b2, eps, wd, bc1, bc2);
    q[i] = qq;
    m[i] = mm;
    v[i] = vv;
  }
}

}  // namespace poetx
