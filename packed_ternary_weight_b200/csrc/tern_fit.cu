// Dense -> ternary fits on the GPU: the inputs of tern_pack from fp32 weights.
//
// The pages describe the fits without an algorithm: a per-matrix, weight-only
// fit into K per-group-scaled trit planes, no calibration (sasori README, "How
// it works & paper"; "K and g"), and "Uniform PTQ" at depth 3 with group 16 and
// a 27-entry log-spaced scale codebook (Entrit card, "Quantization details").
// The readings implemented here:
//
//   TQ{K}P   greedy residual planes. R_0 = W; per (row, group) and plane p:
//            gamma = mean |R_p|, t = sign(R_p) where |R_p| > gamma / 2 (else
//            0), s = fp16_rn(sum_{t != 0} |R_p| / #{t != 0}) (0 without
//            trits), R_{p+1} = R_p - s t.
//   depth d  per group of 16: for each codebook entry c, L = clamp(rint(w / c),
//            -(3^d - 1)/2, (3^d - 1)/2); the entry with the least sum of
//            squared errors (lowest index on a tie); trits = the balanced
//            ternary digits of L.
//
// One thread per (row, group) walks the group in index order in fp64 with
// every product and sum rounded on its own (no contraction), so its decisions
// and its fp16 scales are those of the definition. The residual of plane p is
// recomputed from w and the trits already written, by the same chain of
// subtractions.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tern_internal.h"

namespace tern {
namespace {

__global__ void fit_tq_kernel(const float* __restrict__ w, int n, int k, int planes, int g, int8_t* __restrict__ trits,
                              uint16_t* __restrict__ scales) {
  const int G = k / g;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)n * G) return;
  const int row = (int)(gid / G), grp = (int)(gid - (long long)row * G);
  const float* wr = w + (size_t)row * k + (size_t)grp * g;
  const size_t plane_stride = (size_t)n * k;
  int8_t* tr = trits + (size_t)row * k + (size_t)grp * g;
  double s[4] = {0.0, 0.0, 0.0, 0.0};
  auto resid = [&](int i, int p) -> double {
    double r = (double)wr[i];
    for (int q = 0; q < p; ++q) r = __dsub_rn(r, s[q] * (double)tr[q * plane_stride + i]);
    return r;
  };
  for (int p = 0; p < planes; ++p) {
    double a = 0.0;
    for (int i = 0; i < g; ++i) a = __dadd_rn(a, fabs(resid(i, p)));
    const double gamma = __ddiv_rn(a, (double)g);
    const double half = gamma * 0.5;
    double num = 0.0;
    int cnt = 0;
    for (int i = 0; i < g; ++i) {
      const double r = resid(i, p);
      int t = 0;
      if (gamma != 0.0) t = r > half ? 1 : (r < -half ? -1 : 0);
      tr[p * plane_stride + i] = (int8_t)t;
      if (t != 0) {
        num = __dadd_rn(num, fabs(r));
        ++cnt;
      }
    }
    const double sstar = cnt > 0 ? __ddiv_rn(num, (double)cnt) : 0.0;
    const __half hs = __double2half(sstar);
    scales[((size_t)p * n + row) * G + grp] = __half_as_ushort(hs);
    s[p] = (double)__half2float(hs);
  }
}

__global__ void fit_bt_kernel(const float* __restrict__ w, int n, int k, int depth, const float* __restrict__ cb,
                              int8_t* __restrict__ trits, uint8_t* __restrict__ idx) {
  const int G = k / 16;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)n * G) return;
  const int row = (int)(gid / G), grp = (int)(gid - (long long)row * G);
  const float* wr = w + (size_t)row * k + (size_t)grp * 16;
  double x[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = (double)wr[i];
  const double lmax = depth == 2 ? 4.0 : (depth == 3 ? 13.0 : 40.0);
  auto level = [&](double xi, double c) -> double { return fmin(lmax, fmax(-lmax, rint(__ddiv_rn(xi, c)))); };
  double best_err = INFINITY;
  int best = 0;
  for (int ci = 0; ci < 27; ++ci) {
    const double c = (double)cb[ci];
    double err = 0.0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const double d = __dsub_rn(x[i], __dmul_rn(c, level(x[i], c)));
      err = __dadd_rn(err, __dmul_rn(d, d));
    }
    if (err < best_err) {
      best_err = err;
      best = ci;
    }
  }
  idx[(size_t)row * G + grp] = (uint8_t)best;
  const double c = (double)cb[best];
  const size_t plane_stride = (size_t)n * k;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    int L = (int)level(x[i], c);
    for (int j = 0; j < depth; ++j) {
      const int r = ((L + 1) % 3 + 3) % 3 - 1;  // the digit in {-1, 0, 1} with L = r (mod 3)
      trits[j * plane_stride + (size_t)row * k + (size_t)grp * 16 + i] = (int8_t)r;
      L = (L - r) / 3;
    }
  }
}

}  // namespace
}  // namespace tern

extern "C" tern_status tern_fit_tq(const float* d_w, int32_t n, int32_t k, int32_t planes, int32_t group,
                                   int8_t* d_trits, uint16_t* d_scales, void* stream) {
  if (!d_w || !d_trits || !d_scales || n < 1 || k < 1 || planes < 1 || planes > 4) return TERN_EINVAL;
  if (group < 16 || group > 256 || (group & (group - 1)) || k % group) return TERN_EINVAL;
  const long long groups = (long long)n * (k / group);
  const int threads = 128;
  const long long blocks = (groups + threads - 1) / threads;
  if (blocks > 0x7FFFFFFF) return TERN_EINVAL;
  tern::fit_tq_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(d_w, n, k, planes, group,
                                                                                          d_trits, d_scales);
  return cudaGetLastError() == cudaSuccess ? TERN_OK : TERN_ECUDA;
}

extern "C" tern_status tern_fit_bt(const float* d_w, int32_t n, int32_t k, int32_t depth, const float* d_codebook,
                                   int8_t* d_trits, uint8_t* d_idx, void* stream) {
  if (!d_w || !d_codebook || !d_trits || !d_idx || n < 1 || k < 16 || k % 16 || depth < 2 || depth > 4)
    return TERN_EINVAL;
  const long long groups = (long long)n * (k / 16);
  const int threads = 128;
  const long long blocks = (groups + threads - 1) / threads;
  if (blocks > 0x7FFFFFFF) return TERN_EINVAL;
  tern::fit_bt_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(d_w, n, k, depth,
                                                                                          d_codebook, d_trits, d_idx);
  return cudaGetLastError() == cudaSuccess ? TERN_OK : TERN_ECUDA;
}
