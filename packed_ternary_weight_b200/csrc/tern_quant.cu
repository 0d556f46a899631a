// Per-token absmax int8 quantisation of bf16 activations (the single-GEMV
// workload's "int8 from per-token absmax quantisation"). The pages give no
// rounding rule; the rule used is
//   a = max|x|, inv = fl32(127 / a), xq = clamp(rint(fl32(x * inv)), -127, 127)
// with IEEE division, round-half-to-even and no fused multiply-add, and
// sx = fl32(a / 127); an all-zero token gives xq = 0 and sx = 0.
#include <cuda_runtime.h>

#include "tern_internal.h"

namespace tern {

__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t* __restrict__ x, int k,
                                                      int8_t* __restrict__ xq, float* __restrict__ xs) {
  __shared__ float red[8];
  const int row = blockIdx.x;
  const uint16_t* xr = x + (size_t)row * k;
  float amax = 0.f;
  for (int i = threadIdx.x; i < k; i += blockDim.x) amax = fmaxf(amax, fabsf(__uint_as_float((uint32_t)xr[i] << 16)));
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float a = red[0];
  const float inv = a > 0.f ? __fdiv_rn(127.0f, a) : 0.f;
  int8_t* qr = xq + (size_t)row * k;
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    const float v = __fmul_rn(__uint_as_float((uint32_t)xr[i] << 16), inv);
    int q = __float2int_rn(v);
    q = max(-127, min(127, q));
    qr[i] = (int8_t)q;
  }
  if (threadIdx.x == 0) xs[row] = a > 0.f ? __fdiv_rn(a, 127.0f) : 0.f;
}

int launch_quantize(const uint16_t* x, int m, int k, int8_t* xq, float* xs, void* stream) {
  if (m == 0) return 0;
  quantize_kernel<<<m, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, k, xq, xs);
  return (int)cudaGetLastError();
}

}  // namespace tern
