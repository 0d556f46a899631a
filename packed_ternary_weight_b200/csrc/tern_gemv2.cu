// Decode GEMV over 2-bit ternary planes (BitNet b1.58 single plane with a
// per-tensor scale; sasori-style additive TQ{K}P planes with fp16 group scales).
//
// Work split. One warp owns one row tile (32 rows, one per lane) over one
// K-split; a CTA holds `wpc` such warps for consecutive row tiles of one
// problem and the same K-split, and they share the staged activations. A
// launch may carry several independent problems of the same K and format
// (q/k/v, or gate/up), laid out one after another along blockIdx.x.
//
// Weight stream. Each warp streams its rows' packed columns (512*P bytes per
// 64 k, contiguous in the packed layout) into a private ring of shared-memory
// stages with 1-D bulk async copies (the TMA bulk engine) completing on
// mbarriers, so weights move HBM -> SMEM without passing through registers and
// several stages stay in flight per warp. With programmatic dependent launch
// the first stages are requested before the kernel waits for its predecessor.
//
// K-splits. When K is split across blockIdx.y, the splits of one row group
// form a thread-block cluster: partial row sums are written into the shared
// memory of the cluster's first CTA (distributed shared memory) and reduced
// there in a fixed order after one cluster barrier. When a cluster cannot be
// used (more than 16 splits), the partials go through a global workspace and
// the last CTA to arrive reduces them.
//
// Inner loop (per lane, per 16 k of one plane = one u32 word). Each 2-bit code
// c (00 -> 0, 01 -> +1, 10 -> -1) is mapped by one LOP3 to the digit
// F = 1 - t in {1, 0, 2}; masking one field per byte gives four digits that
// line up with four consecutive activations, and a byte dot-product
// accumulates sum F*x. Then sum t*x = sum x - sum F*x, where sum x is computed
// once per group (or per K-split) for all rows. Digits are 0, 1 or 2, so no
// weight value multiplies an activation: the dot-product unit only adds x or
// 2x ("additions instead of weight multiplies", sasori README;
// "zero-multiplication inner loop", QORA-LLM-2B page).
//
// Activations:
//  * int8 (per-token absmax quantised, given or done here): the sums are exact
//    integers. BitNet applies the layer scale once per row at the end
//    (QORA-LLM-2B, "Ternary GEMV (No Multiplication)"); TQ folds each fp16
//    group scale into an exact int64 count of 2^-24 (every fp16 value is an
//    integer multiple of 2^-24), so the result is the exactly rounded
//    group-scaled sum in any order.
//  * bf16: each group of x is written as q * 2^(E-22) with q a 24-bit integer
//    (E = exponent of the group's largest |x|; bf16 carries 8 significant
//    bits, so every element within 2^15 of the group maximum is exact and
//    smaller ones round by at most 2^(E-23)), split into a signed high byte and
//    unsigned middle and low bytes; integer group sums are exact, and each is
//    rounded once to fp32, scaled and accumulated once per group in fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tern_ptx.cuh"

namespace tern {

int read_clear_dev_error_gemv2(void* stream, unsigned* out) { return read_clear_dev_error_tu(stream, out); }

namespace {

constexpr uint32_t kM03 = 0x03030303u;
constexpr uint32_t kM30 = 0x30303030u;

struct SmemPlan {
  size_t bars, ring, xa, xb, xc, xraw, gsum, gmult, red, amx, misc, total;
  int stage_bytes;
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline int red_elem(int xmode, bool tq) { return (xmode != kXBf16 && tq) ? 8 : 4; }

__host__ __device__ inline SmemPlan smem_plan(const Gemv2Params& p, int xmode, int mt) {
  SmemPlan s{};
  const bool tq = p.tq != 0;
  const int kr = p.cols_per_split * kColK2;                                // k per split
  const int gr = tq ? (kr + p.group - 1) / p.group : 1;                      // groups per split
  const int gps = tq ? (p.stage_cols * kColK2 + p.group - 1) / p.group : 0;  // groups per stage
  s.stage_bytes = (int)align_up((size_t)p.stage_cols * p.planes * kPlaneColBytes + (size_t)gps * p.planes * 64, 128);
  const bool bf = xmode == kXBf16;
  size_t off = 0;
  s.bars = off;
  off = align_up(off + (size_t)p.wpc * p.nstage * 8, 128);
  s.ring = off;
  off += (size_t)p.wpc * p.nstage * s.stage_bytes;
  s.xa = off;  // int8 x [mt][kr], or the signed high byte of the bf16 image [kr]
  off = align_up(off + (size_t)(bf ? 1 : mt) * kr, 128);
  s.xb = off;  // bf16 image: middle byte [kr]
  off = align_up(off + (bf ? (size_t)kr : 0), 128);
  s.xc = off;  // bf16 image: low byte [kr]
  off = align_up(off + (bf ? (size_t)kr : 0), 128);
  s.xraw = off;  // in-kernel quantisation: raw bf16 [mt][kr]
  off = align_up(off + (xmode == kXBf16Q8 ? (size_t)mt * kr * 2 : 0), 128);
  s.gsum = off;  // int32 [mt][gr]: sum x (int8); int64 [gr]: sum q (bf16)
  off = align_up(off + (size_t)mt * gr * (bf ? 8 : 4), 16);
  s.gmult = off;  // float [gr]: 2^(E-22) (bf16)
  off = align_up(off + (bf ? (size_t)gr * 4 : 0), 16);
  s.red = off;  // cluster reduction in the first CTA: [ks][mt][wpc*32]
  off = align_up(off + ((p.cluster && p.ks > 1) ? (size_t)p.ks * mt * p.wpc * 32 * red_elem(xmode, tq) : 0), 16);
  s.amx = off;  // per-split token maxima [kMaxCluster][mt] (in-kernel quantisation)
  off = align_up(off + (xmode == kXBf16Q8 ? (size_t)kMaxCluster * mt * 4 : 0), 16);
  s.misc = off;  // [0..mt): token max (bits); [mt..2mt): sx; then a flag
  off += align_up((size_t)mt * 8 + 16, 16);
  s.total = off;
  return s;
}

// ------------------------------------------------------------ activations
// Per-(token, group) sums of the staged int8 activations.
template <int MT>
__device__ void int8_group_sums(const SmemPlan& sp, uint8_t* smem, int kr, int gsz) {
  const int8_t* xs = reinterpret_cast<const int8_t*>(smem + sp.xa);
  int* gs = reinterpret_cast<int*>(smem + sp.gsum);
  const int gr = (kr + gsz - 1) / gsz;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int t = warp; t < MT * gr; t += nw) {
    const int mm = t / gr, g = t - mm * gr;
    const int* w = reinterpret_cast<const int*>(xs + mm * kr + g * gsz);  // gsz, kr multiples of 16
    int s = 0;
    for (int i = lane; i < min(gsz, kr - g * gsz) / 4; i += 32) s = __dp4a(w[i], 0x01010101, s);
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) gs[mm * gr + g] = s;
  }
}

template <int MT>
__device__ void stage_x_int8(const Gemv2Params& p, const Gemv2Problem& pr, const SmemPlan& sp, uint8_t* smem, int k0,
                             int kr) {
  int8_t* xs = reinterpret_cast<int8_t*>(smem + sp.xa);
  const int8_t* x = static_cast<const int8_t*>(pr.x);
  const int m = p.m, K = p.k, nch = kr / 16;
  for (int i = threadIdx.x; i < MT * nch; i += blockDim.x) {
    const int t = i / nch, c = i - t * nch, k = k0 + 16 * c;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (t < m) {
      const int8_t* src = x + (size_t)t * K + k;
      if (p.x_vec && k + 16 <= K) {
        v = __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (k + j < K) w[j >> 2] |= (uint32_t)(uint8_t)src[j] << (8 * (j & 3));
        v = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    *reinterpret_cast<uint4*>(xs + t * kr + 16 * c) = v;
  }
}

__device__ __forceinline__ float bf16_abs_max8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t mx = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    mx = max(mx, (w[j] & 0x7FFFu) << 16);
    mx = max(mx, w[j] & 0x7FFF0000u);
  }
  return __uint_as_float(mx);  // non-negative floats order like their bits
}

// In-kernel per-token absmax quantisation (same rule as tern_quantize_act):
// the token maxima of all K-splits are exchanged through the cluster.
template <int MT>
__device__ void stage_x_q8(const Gemv2Params& p, const Gemv2Problem& pr, const SmemPlan& sp, uint8_t* smem, int k0,
                           int kr, bool clus, int split) {
  uint16_t* raw = reinterpret_cast<uint16_t*>(smem + sp.xraw);
  int8_t* xs = reinterpret_cast<int8_t*>(smem + sp.xa);
  unsigned* tmax = reinterpret_cast<unsigned*>(smem + sp.misc);     // [MT], zeroed in the prologue
  float* sxs = reinterpret_cast<float*>(smem + sp.misc) + MT;        // [MT]
  float* amx = reinterpret_cast<float*>(smem + sp.amx);             // [ks][MT]
  const uint16_t* x = static_cast<const uint16_t*>(pr.x);
  const int m = p.m, K = p.k, nch = kr / 8;
  for (int i = threadIdx.x; i < MT * nch; i += blockDim.x) {
    const int t = i / nch, c = i - t * nch, k = k0 + 8 * c;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (t < m) {
      const uint16_t* src = x + (size_t)t * K + k;
      if (p.x_vec && k + 8 <= K) {
        v = __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (k + j < K) w[j >> 1] |= (uint32_t)src[j] << (16 * (j & 1));
        v = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    *reinterpret_cast<uint4*>(raw + t * kr + 8 * c) = v;
    const float mx = bf16_abs_max8(v);
    if (mx > 0.f) atomicMax(&tmax[t], __float_as_uint(mx));
  }
  __syncthreads();
  if (clus) {
    for (int i = threadIdx.x; i < p.ks * MT; i += blockDim.x) {
      const int r = i / MT, t = i - r * MT;
      st_cluster_u32(map_cluster_rank(smem_u32(&amx[split * MT + t]), (uint32_t)r), tmax[t]);
    }
    cluster_sync();
  } else {
    if (threadIdx.x < MT) amx[threadIdx.x] = __uint_as_float(tmax[threadIdx.x]);
    __syncthreads();
  }
  const int nsp = clus ? p.ks : 1;
  float inv[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    float a = 0.f;
    for (int r = 0; r < nsp; ++r) a = fmaxf(a, amx[r * MT + t]);
    inv[t] = a > 0.f ? __fdiv_rn(127.0f, a) : 0.f;
    if (threadIdx.x == 0) sxs[t] = a > 0.f ? __fdiv_rn(a, 127.0f) : 0.f;
  }
  const int n4 = kr / 4;
  for (int i = threadIdx.x; i < MT * n4; i += blockDim.x) {
    const int t = i / n4, c = i - t * n4;
    float it = inv[0];
#pragma unroll
    for (int u = 1; u < MT; ++u)
      if (t == u) it = inv[u];
    const uint2 v = *reinterpret_cast<const uint2*>(raw + t * kr + 4 * c);
    const uint32_t h[4] = {v.x & 0xFFFFu, v.x >> 16, v.y & 0xFFFFu, v.y >> 16};
    uint32_t packed = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int q = __float2int_rn(__fmul_rn(__uint_as_float(h[j] << 16), it));
      q = max(-127, min(127, q));
      packed |= ((uint32_t)q & 0xFFu) << (8 * j);
    }
    *reinterpret_cast<uint32_t*>(xs + t * kr + 4 * c) = packed;
  }
}

__device__ void stage_x_bf16(const Gemv2Params& p, const Gemv2Problem& pr, const SmemPlan& sp, uint8_t* smem, int k0,
                             int kr) {
  int8_t* xh = reinterpret_cast<int8_t*>(smem + sp.xa);
  uint8_t* xm = smem + sp.xb;
  uint8_t* xl = smem + sp.xc;
  long long* gs = reinterpret_cast<long long*>(smem + sp.gsum);
  float* gm = reinterpret_cast<float*>(smem + sp.gmult);
  const uint16_t* x = static_cast<const uint16_t*>(pr.x);
  const int g = p.group, gr = kr / g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int grp = warp; grp < gr; grp += nw) {
    const int kb = grp * g;
    float amax = 0.f;
    for (int kk = kb + lane; kk < kb + g; kk += 32) {
      const int k = k0 + kk;
      const float v = k < p.k ? __uint_as_float((uint32_t)x[k] << 16) : 0.f;
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
      const float v = k < p.k ? __uint_as_float((uint32_t)x[k] << 16) : 0.f;
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

// Exact fold of an fp16 scale times an integer group sum into a count of 2^-24.
__device__ __forceinline__ long long fold_fp16_exact(uint16_t h, int S) {
  const int ex = (h >> 10) & 0x1F, man = h & 0x3FF;
  int mm = ex ? man + 1024 : man;
  const int sh = ex ? ex - 1 : 0;
  if (h & 0x8000) mm = -mm;
  return (long long)(mm * S) * (1ll << sh);
}

}  // namespace

// XM: activation mode; P: planes; WG: words (16 k) per scale group, 0 = one
// per-tensor scale (BitNet); MT: maximum tokens handled by one pass.
template <int XM, int P, int WG, int MT>
__global__ void __launch_bounds__(256) gemv2_kernel(const __grid_constant__ Gemv2Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr bool kTQ = WG > 0;
  constexpr bool kIntX = XM != kXBf16;
  const SmemPlan sp = smem_plan(p, XM, MT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int pi = 0;
  while (pi + 1 < p.nprob && (int)blockIdx.x >= p.prob[pi + 1].cta_begin) ++pi;
  const Gemv2Problem& pr = p.prob[pi];
  const int T = ((int)blockIdx.x - pr.cta_begin) * p.wpc + warp;
  const bool active = T < pr.row_tiles;
  const int split = blockIdx.y;
  const bool clus = p.cluster && p.ks > 1;
  const int c0 = split * p.cols_per_split;
  const int c1 = min(p.cols, c0 + p.cols_per_split);
  const int ncols = c1 - c0;
  const int sc = p.stage_cols, nst = p.nstage;
  const int nstages = (ncols + sc - 1) / sc;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sp.bars) + warp * nst;
  uint8_t* ring = smem + sp.ring + (size_t)warp * nst * sp.stage_bytes;

  // ---- prologue (independent of the preceding kernel): barriers, first weight stages
  if (clus) cluster_arrive_relaxed();  // DSMEM is used only after every CTA of the cluster runs
  if (active && lane == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  if (XM == kXBf16Q8 && threadIdx.x < MT) reinterpret_cast<unsigned*>(smem + sp.misc)[threadIdx.x] = 0u;
  __syncwarp();
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int i) {
    const int slot = i % nst;
    const int cs = c0 + i * sc, ce = min(c1, cs + sc);
    const uint32_t tb = (uint32_t)(ce - cs) * P * kPlaneColBytes;
    const uint8_t* src = pr.trit + ((size_t)T * p.cols + cs) * P * kPlaneColBytes;
    uint8_t* dst = ring + (size_t)slot * sp.stage_bytes;
    uint32_t sb = 0;
    int ga = 0;
    if (kTQ) {
      ga = cs * kColK2 / p.group;
      const int gb = min(p.groups, (ce * kColK2 + p.group - 1) / p.group);
      sb = (uint32_t)(gb - ga) * P * 64;
    }
    mbar_arrive_expect_tx(&bars[slot], tb + sb);
    bulk_g2s(dst, src, tb, &bars[slot], pol);
    if (kTQ)
      bulk_g2s(dst + (size_t)sc * P * kPlaneColBytes,
               reinterpret_cast<const uint8_t*>(pr.scale) + ((size_t)T * p.groups + ga) * P * 64, sb, &bars[slot],
               pol);
  };
  if (active && lane == 0)
    for (int i = 0; i < min(nst, nstages); ++i) issue(i);
  pdl_launch_dependents();

  // ---- wait for the producer of x, then stage x for this K-split
  pdl_wait();
  if (clus) cluster_wait_acquire();
  __syncthreads();
  const int k0 = c0 * kColK2, kr = ncols * kColK2;
  if (XM == kXInt8) {
    stage_x_int8<MT>(p, pr, sp, smem, k0, kr);
    __syncthreads();
    int8_group_sums<MT>(sp, smem, kr, kTQ ? p.group : kr);
  } else if (XM == kXBf16Q8) {
    stage_x_q8<MT>(p, pr, sp, smem, k0, kr, clus, split);
    __syncthreads();
    int8_group_sums<MT>(sp, smem, kr, kTQ ? p.group : kr);
  } else {
    stage_x_bf16(p, pr, sp, smem, k0, kr);
  }
  __syncthreads();

  const int8_t* xs = reinterpret_cast<const int8_t*>(smem + sp.xa);
  const uint8_t* xmid = smem + sp.xb;
  const uint8_t* xl = smem + sp.xc;
  const int* gsum = reinterpret_cast<const int*>(smem + sp.gsum);
  const long long* gsum64 = reinterpret_cast<const long long*>(smem + sp.gsum);
  const float* gmul = reinterpret_cast<const float*>(smem + sp.gmult);
  const int gr = kTQ ? kr / p.group : 1;
  const int m = p.m;

  // accumulators: a = fields 0,1 (weight 1), b = fields 2,3 (weight 16)
  int a[P][MT], b[P][MT];     // int8 x   (or high bytes for bf16)
  unsigned ma[P], mb[P];      // bf16 middle bytes
  unsigned la[P], lb[P];      // bf16 low bytes
  long long acc64[MT];        // TQ int8
  float yacc = 0.f;           // bf16
#pragma unroll
  for (int q = 0; q < P; ++q) {
#pragma unroll
    for (int t = 0; t < MT; ++t) a[q][t] = b[q][t] = 0;
    la[q] = lb[q] = ma[q] = mb[q] = 0;
  }
#pragma unroll
  for (int t = 0; t < MT; ++t) acc64[t] = 0;

  int ifail = -1;
  if (active) {
    for (int i = 0; i < nstages; ++i) {
      const int slot = i % nst;
      // warp-uniform outcome, so that no lane is left behind at __syncwarp
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars[slot], (uint32_t)(i / nst) & 1u))) {
        ifail = i;
        break;
      }
      const uint8_t* st = ring + (size_t)slot * sp.stage_bytes;
      const uint16_t* sst = reinterpret_cast<const uint16_t*>(st + (size_t)sc * P * kPlaneColBytes);
      const int cs = c0 + i * sc;
      const int ncs = min(sc, c1 - cs);
      const int ga_stage = kTQ ? cs * kColK2 / p.group : 0;
      for (int cc = 0; cc < ncs; ++cc) {
        const int kx = (cs + cc - c0) * kColK2;
        uint4 wv[P];
#pragma unroll
        for (int q = 0; q < P; ++q)
          wv[q] = *reinterpret_cast<const uint4*>(st + ((size_t)cc * P + q) * kPlaneColBytes + lane * 16);
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          uint32_t F[P], F2[P];
#pragma unroll
          for (int q = 0; q < P; ++q) {
            const uint32_t w = wi == 0 ? wv[q].x : wi == 1 ? wv[q].y : wi == 2 ? wv[q].z : wv[q].w;
            F[q] = lop3_ternary_digit(w);
            F2[q] = F[q] >> 2;
          }
          if (kIntX) {
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              if (t < m) {
                const int4 xv = *reinterpret_cast<const int4*>(xs + t * kr + kx + wi * 16);
#pragma unroll
                for (int q = 0; q < P; ++q) {
                  a[q][t] = dp4a_ss((int)(F[q] & kM03), xv.x, a[q][t]);
                  a[q][t] = dp4a_ss((int)(F2[q] & kM03), xv.y, a[q][t]);
                  b[q][t] = dp4a_ss((int)(F[q] & kM30), xv.z, b[q][t]);
                  b[q][t] = dp4a_ss((int)(F2[q] & kM30), xv.w, b[q][t]);
                }
              }
            }
          } else {
            const int4 hv = *reinterpret_cast<const int4*>(xs + kx + wi * 16);
            const uint4 mv = *reinterpret_cast<const uint4*>(xmid + kx + wi * 16);
            const uint4 lv = *reinterpret_cast<const uint4*>(xl + kx + wi * 16);
#pragma unroll
            for (int q = 0; q < P; ++q) {
              a[q][0] = dp4a_ss((int)(F[q] & kM03), hv.x, a[q][0]);
              a[q][0] = dp4a_ss((int)(F2[q] & kM03), hv.y, a[q][0]);
              b[q][0] = dp4a_ss((int)(F[q] & kM30), hv.z, b[q][0]);
              b[q][0] = dp4a_ss((int)(F2[q] & kM30), hv.w, b[q][0]);
              ma[q] = dp4a_uu(F[q] & kM03, mv.x, ma[q]);
              ma[q] = dp4a_uu(F2[q] & kM03, mv.y, ma[q]);
              mb[q] = dp4a_uu(F[q] & kM30, mv.z, mb[q]);
              mb[q] = dp4a_uu(F2[q] & kM30, mv.w, mb[q]);
              la[q] = dp4a_uu(F[q] & kM03, lv.x, la[q]);
              la[q] = dp4a_uu(F2[q] & kM03, lv.y, la[q]);
              lb[q] = dp4a_uu(F[q] & kM30, lv.z, lb[q]);
              lb[q] = dp4a_uu(F2[q] & kM30, lv.w, lb[q]);
            }
          }
          // ---- group fold (TQ): after the last word of each group
          if constexpr (kTQ) {
            const int wglob = (cs + cc - c0) * 4 + wi;  // word index within the split
            if ((wglob + 1) % WG == 0) {
              const int gl = wglob / WG;                                                  // within split
              const int gst = (cs * kColK2 + ((cc * 4 + wi) * 16)) / p.group - ga_stage;  // within stage
#pragma unroll
              for (int q = 0; q < P; ++q) {
                const uint16_t h = sst[((size_t)gst * P + q) * kTileRows + lane];
                if (kIntX) {
#pragma unroll
                  for (int t = 0; t < MT; ++t) {
                    if (t < m) {
                      const int S = gsum[t * gr + gl] - (a[q][t] + (b[q][t] >> 4));
                      acc64[t] += fold_fp16_exact(h, S);
                    }
                    a[q][t] = b[q][t] = 0;
                  }
                } else {
                  const int H = a[q][0] + (b[q][0] >> 4);
                  const int Mi = (int)(ma[q] + (mb[q] >> 4));
                  const int L = (int)(la[q] + (lb[q] >> 4));
                  const long long S = gsum64[gl] - ((long long)H * 65536 + (long long)Mi * 256 + L);
                  yacc = fmaf(__half2float(__ushort_as_half(h)) * gmul[gl], __ll2float_rn(S), yacc);
                  a[q][0] = b[q][0] = 0;
                  la[q] = lb[q] = ma[q] = mb[q] = 0;
                }
              }
            }
          }
        }
      }
      // release the slot: reads of this stage are complete before the refill
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && i + nst < nstages) issue(i + nst);
    }
  }
  if (active && ifail >= 0) {
    // a wait expired: give the copies still in flight a bounded chance to land
    for (int j = ifail; j < min(nstages, ifail + nst); ++j) mbar_wait_bounded(&bars[j % nst], (uint32_t)(j / nst) & 1u);
  }

  // ---- epilogue: per-lane row results (int32 BitNet / int64 TQ-int8 / fp32 bf16)
  const int npad = pr.row_tiles * kTileRows;
  const int row = T * kTileRows + lane;
  int accb[MT];
  if (!kTQ) {
#pragma unroll
    for (int t = 0; t < MT; ++t) accb[t] = (t < m) ? gsum[t] - (a[0][t] + (b[0][t] >> 4)) : 0;
  }
  const float* sxs = reinterpret_cast<const float*>(smem + sp.misc) + MT;

  auto write_out = [&](int t, float v) {
    if (p.out_bf16)
      reinterpret_cast<__nv_bfloat16*>(pr.y)[(size_t)t * pr.n + row] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<float*>(pr.y)[(size_t)t * pr.n + row] = v;
  };
  auto finish = [&](int t, long long v64, int v32, float vf) {
    if (row >= pr.n) return;
    const float sx = XM == kXBf16Q8 ? sxs[t] : (XM == kXInt8 ? pr.xscale[t] : 0.f);
    if (XM == kXBf16) {
      write_out(t, vf);
    } else if (kTQ) {
      const float s = __fmul_rn(__ll2float_rn(v64), 0x1p-24f);
      write_out(t, __fmul_rn(s, sx));
    } else {
      write_out(t, __fmul_rn(__fmul_rn(__int2float_rn(v32), pr.tensor_scale), sx));
    }
  };

  if (p.ks == 1) {
    if (active) {
#pragma unroll
      for (int t = 0; t < MT; ++t)
        if (t < m) finish(t, acc64[t], kTQ ? 0 : accb[t], yacc);
    }
    return;
  }

  if (clus) {
    // ---- K-splits of this row group form the cluster: reduce in CTA rank 0
    const int rows_cta = p.wpc * kTileRows;
    const int esz = red_elem(XM, kTQ);
    if (active) {
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t >= m) continue;
        const size_t idx = ((size_t)split * MT + t) * rows_cta + warp * kTileRows + lane;
        const uint32_t dst = map_cluster_rank(smem_u32(smem + sp.red + idx * esz), 0);
        if (XM == kXBf16)
          st_cluster_u32(dst, __float_as_uint(yacc));
        else if (kTQ)
          st_cluster_u64(dst, (unsigned long long)acc64[t]);
        else
          st_cluster_u32(dst, (uint32_t)accb[t]);
      }
    }
    cluster_sync();
    if (split == 0 && active) {
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t >= m) continue;
        long long s64 = 0;
        int s32 = 0;
        float sf = 0.f;
        for (int s = 0; s < p.ks; ++s) {
          const size_t idx = ((size_t)s * MT + t) * rows_cta + warp * kTileRows + lane;
          if (XM == kXBf16)
            sf += reinterpret_cast<const float*>(smem + sp.red)[idx];
          else if (kTQ)
            s64 += reinterpret_cast<const long long*>(smem + sp.red)[idx];
          else
            s32 += reinterpret_cast<const int*>(smem + sp.red)[idx];
        }
        finish(t, s64, s32, sf);
      }
    }
    return;
  }

  // ---- more splits than a cluster holds: partials through the global workspace,
  // reduced by the last CTA of this row group to arrive
  if (active && row < npad) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t >= m) continue;
      const size_t idx = ((size_t)split * m + t) * npad + row;
      if (XM == kXBf16)
        reinterpret_cast<float*>(p.ws_part)[idx] = yacc;
      else if (kTQ)
        reinterpret_cast<long long*>(p.ws_part)[idx] = acc64[t];
      else
        reinterpret_cast<int*>(p.ws_part)[idx] = accb[t];
    }
  }
  __threadfence();
  __syncthreads();
  int* flag = reinterpret_cast<int*>(smem + sp.misc) + 2 * MT;
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&p.ws_cnt[blockIdx.x], 1u);
    *flag = (prev == (unsigned)(p.ks - 1));
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  if (active) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t >= m) continue;
      long long s64 = 0;
      int s32 = 0;
      float sf = 0.f;
      for (int s = 0; s < p.ks; ++s) {
        const size_t idx = ((size_t)s * m + t) * npad + row;
        if (XM == kXBf16)
          sf += __ldcg(reinterpret_cast<const float*>(p.ws_part) + idx);
        else if (kTQ)
          s64 += __ldcg(reinterpret_cast<const long long*>(p.ws_part) + idx);
        else
          s32 += __ldcg(reinterpret_cast<const int*>(p.ws_part) + idx);
      }
      finish(t, s64, s32, sf);
    }
  }
  if (threadIdx.x == 0) p.ws_cnt[blockIdx.x] = 0u;  // leave the counters at zero
}

// ------------------------------------------------------------------ launch
int gemv2_mt(int xmode, int m) {
  if (xmode == kXBf16) return 1;
  if (xmode == kXBf16Q8) return m <= 1 ? 1 : 4;
  return m <= 1 ? 1 : m <= 4 ? 4 : 16;
}

size_t gemv2_smem_bytes(const Gemv2Params& p, int xmode) { return smem_plan(p, xmode, gemv2_mt(xmode, p.m)).total; }

template <int XM, int P, int WG, int MT>
static int launch_one(const Gemv2Params& p, bool pdl, void* stream) {
  const SmemPlan sp = smem_plan(p, XM, MT);
  auto kern = gemv2_kernel<XM, P, WG, MT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
  if (e != cudaSuccess) return (int)e;
  const bool clus = p.cluster && p.ks > 1;
  if (clus && p.ks > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return (int)e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid_x, p.ks, 1);
  cfg.blockDim = dim3(32 * p.wpc, 1, 1);
  cfg.dynamicSmemBytes = sp.total;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (clus) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = p.ks;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  return (int)e;
}

// Instantiated combinations; anything else reports "unsupported" (-1).
int launch_gemv2(const Gemv2Params& p, int xmode, bool pdl, void* stream) {
  const bool tq = p.tq != 0;
  const int wg = tq ? p.group / 16 : 0;
  const int mt = gemv2_mt(xmode, p.m);
  if (xmode == kXInt8) {
    if (!tq && p.planes == 1) {
      if (mt == 1) return launch_one<kXInt8, 1, 0, 1>(p, pdl, stream);
      if (mt == 4) return launch_one<kXInt8, 1, 0, 4>(p, pdl, stream);
      return launch_one<kXInt8, 1, 0, 16>(p, pdl, stream);
    }
    if (tq && p.planes == 2 && wg == 2) {
      if (mt == 1) return launch_one<kXInt8, 2, 2, 1>(p, pdl, stream);
      if (mt == 4) return launch_one<kXInt8, 2, 2, 4>(p, pdl, stream);
      return launch_one<kXInt8, 2, 2, 16>(p, pdl, stream);
    }
    if (tq && p.planes == 3 && wg == 16 && mt == 1) return launch_one<kXInt8, 3, 16, 1>(p, pdl, stream);
    return -1;
  }
  if (xmode == kXBf16Q8) {
    if (!tq && p.planes == 1) {
      if (mt == 1) return launch_one<kXBf16Q8, 1, 0, 1>(p, pdl, stream);
      return launch_one<kXBf16Q8, 1, 0, 4>(p, pdl, stream);
    }
    if (tq && p.planes == 2 && wg == 2) {
      if (mt == 1) return launch_one<kXBf16Q8, 2, 2, 1>(p, pdl, stream);
      return launch_one<kXBf16Q8, 2, 2, 4>(p, pdl, stream);
    }
    return -1;
  }
  if (!tq || p.m != 1) return -1;
  switch (p.planes * 100 + wg) {
    case 116: return launch_one<kXBf16, 1, 16, 1>(p, pdl, stream);
    case 216: return launch_one<kXBf16, 2, 16, 1>(p, pdl, stream);
    case 316: return launch_one<kXBf16, 3, 16, 1>(p, pdl, stream);
    case 416: return launch_one<kXBf16, 4, 16, 1>(p, pdl, stream);
    case 202: return launch_one<kXBf16, 2, 2, 1>(p, pdl, stream);
    case 304: return launch_one<kXBf16, 3, 4, 1>(p, pdl, stream);
    default: return -1;
  }
}

}  // namespace tern
