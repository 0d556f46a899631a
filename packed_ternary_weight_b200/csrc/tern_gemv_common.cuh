// Device helpers shared by the GEMV kernels of the 2-bit and base-3 formats.
#pragma once
#include <cuda_runtime.h>

#include "tern_ptx.cuh"

namespace tern {
namespace gemv_common {

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

template <int I>
__device__ __forceinline__ uint32_t u4_get(const uint4& v) {
  if constexpr (I == 0) return v.x;
  if constexpr (I == 1) return v.y;
  if constexpr (I == 2) return v.z;
  return v.w;
}


// Stages a bf16 activation range [k0, k0 + kr) as a 24-bit fixed-point image
// per group of `g` (q = x * 2^(22-E), E the exponent of the group's largest
// |x|): signed high byte at xh, middle and low bytes at xm and xl, the exact
// integer sum of q per group at gs and 2^(E-22) per group at gm.
__device__ inline void stage_x_bf16_image(const uint16_t* x, int K, int g, int k0, int kr, int8_t* xh, uint8_t* xm,
                                          uint8_t* xl, long long* gs, float* gm) {
  const int gr = kr / g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int grp = warp; grp < gr; grp += nw) {
    const int kb = grp * g;
    float amax = 0.f;
    for (int kk = kb + lane; kk < kb + g; kk += 32) {
      const int k = k0 + kk;
      const float v = k < K ? __uint_as_float((uint32_t)x[k] << 16) : 0.f;
      amax = fmaxf(amax, fabsf(v));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int e = amax > 0.f ? ilogbf(amax) : 0;
    // multiply by 2^(22-e) in at most two exact power-of-two steps
    const int sh = 22 - e;
    const float up1 = ldexpf(1.0f, sh > 100 ? 100 : sh), up2 = ldexpf(1.0f, sh > 100 ? sh - 100 : 0);
    long long s = 0;
    for (int kk = kb + lane; kk < kb + g; kk += 32) {
      const int k = k0 + kk;
      const float v = k < K ? __uint_as_float((uint32_t)x[k] << 16) : 0.f;
      const int q = __float2int_rn(__fmul_rn(__fmul_rn(v, up1), up2));  // |q| < 2^23
      s += q;
      xh[kk] = (int8_t)(q >> 16);
      xm[kk] = (uint8_t)((q >> 8) & 0xFF);
      xl[kk] = (uint8_t)(q & 0xFF);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
      gs[grp] = s;
      gm[grp] = amax > 0.f ? ldexpf(1.0f, e - 22) : 0.f;
    }
  }
}

}  // namespace gemv_common
}  // namespace tern
