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

// As stage_x_bf16_image, but instead of the exact sum of q per group it writes
// one 16-byte record per group: the sums of the high (signed), middle and low
// byte chains, {sum h, sum m, sum l, bits of 2^(E-22)}, so that a group's
// sum of w * q can be formed as 65536 * (H - c sum h) + 256 * (M - c sum m) +
// (L - c sum l) from small integers (q = 65536 h + 256 m + l exactly).
__device__ inline void stage_x_bf16_chains(const uint16_t* x, int K, int g, int k0, int kr, int8_t* xh, uint8_t* xm,
                                           uint8_t* xl, int4* rec) {
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
    const int sh = 22 - e;
    const float up1 = ldexpf(1.0f, sh > 100 ? 100 : sh), up2 = ldexpf(1.0f, sh > 100 ? sh - 100 : 0);
    int sh_ = 0, sm = 0, sl = 0;
    for (int kk = kb + lane; kk < kb + g; kk += 32) {
      const int k = k0 + kk;
      const float v = k < K ? __uint_as_float((uint32_t)x[k] << 16) : 0.f;
      const int q = __float2int_rn(__fmul_rn(__fmul_rn(v, up1), up2));  // |q| < 2^23
      const int h = q >> 16, m = (q >> 8) & 0xFF, l = q & 0xFF;
      sh_ += h;
      sm += m;
      sl += l;
      xh[kk] = (int8_t)h;
      xm[kk] = (uint8_t)m;
      xl[kk] = (uint8_t)l;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      sh_ += __shfl_xor_sync(0xffffffffu, sh_, o);
      sm += __shfl_xor_sync(0xffffffffu, sm, o);
      sl += __shfl_xor_sync(0xffffffffu, sl, o);
    }
    if (lane == 0) rec[grp] = make_int4(sh_, sm, sl, __float_as_int(amax > 0.f ? ldexpf(1.0f, e - 22) : 0.f));
  }
}

// 65536 a + 256 b + c as fp32, rounded once when |256 b + c| < 2^24 and |a| < 2^24.
__device__ __forceinline__ float chains_to_float(int a, int b, int c) {
  return fmaf(__int2float_rn(a), 65536.0f, fmaf(__int2float_rn(b), 256.0f, __int2float_rn(c)));
}

// Five base-3 digits of the two values (each <= 242) held in the 16-bit lanes of v.
__device__ __forceinline__ void digits5(uint32_t v, uint32_t (&d)[5]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t q = ((v * 171u) >> 9) & 0x007F007Fu;  // floor(v / 3) in both lanes
    d[j] = v - 3u * q;
    v = q;
  }
  d[4] = v;
}

// The five levels of the triples held in the 16-bit lanes of b0, b1, b2 (the
// triples' bytes 0, 1, 2; every byte <= 242). Exact in both lanes:
// floor(v / 27) = (19 v) >> 9 (v <= 242), floor(v / 3) = (171 v) >> 9,
// floor(v / 9) = (57 v) >> 9; no lane carries into the other (products < 2^16,
// differences >= 0).
__device__ __forceinline__ void triple_levels(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t (&U)[5]) {
  constexpr uint32_t kM = 0x007F007Fu;
  const uint32_t h1 = ((b0 * 19u) >> 9) & kM;  // u0 + 3 u1 of weight 1
  U[0] = b0 - 27u * h1;
  const uint32_t r = ((b1 * 171u) >> 9) & kM;  // b1 / 3
  const uint32_t l1 = b1 - 3u * r;             // u2 of weight 1
  const uint32_t h3 = ((r * 19u) >> 9) & kM;   // u0 of weight 3
  U[2] = r - 27u * h3;
  U[4] = ((b2 * 57u) >> 9) & kM;
  const uint32_t l3 = b2 - 9u * U[4];          // u1 + 3 u2 of weight 3
  U[1] = h1 + 9u * l1;
  U[3] = h3 + 3u * l3;
}

}  // namespace gemv_common
}  // namespace tern
