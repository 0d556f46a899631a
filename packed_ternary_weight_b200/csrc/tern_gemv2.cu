// Decode GEMV over 2-bit ternary planes (BitNet b1.58 single plane with a
// per-tensor scale; sasori-style additive TQ{K}P planes with fp16 group scales).
//
// Work split. One warp owns one row tile (32 rows, one per lane) over one
// K-split; a CTA holds `wpc` such warps for consecutive row tiles and the same
// K-split, and they share the staged activations. Each warp streams its rows'
// packed columns (512*P bytes per 64 k, contiguous in the packed layout) into a
// private ring of shared-memory stages with 1-D bulk async copies (the TMA bulk
// engine) completing on mbarriers, so weights move HBM -> SMEM without passing
// through registers, and the ring keeps several stages in flight per warp.
// With programmatic dependent launch the first stages are requested before the
// kernel waits for its predecessor.
//
// Inner loop (per lane, per 16 k of one plane = one u32 word). Each 2-bit code
// c (00 -> 0, 01 -> +1, 10 -> -1) is mapped by one LOP3 to the digit
// F = 1 - t in {1, 0, 2}; masking one field per byte gives four digits that line
// up with four consecutive activations, and a byte dot-product accumulates
// sum F*x. Then sum t*x = sum x - sum F*x, where sum x is computed once per
// group (or per K-split) for all rows. Digits are 0, 1 or 2, so no weight value
// multiplies an activation: the dot-product unit only adds x or 2x ("additions
// instead of weight multiplies", sasori README; "zero-multiplication inner
// loop", QORA-LLM-2B page).
//
// Activations:
//  * int8 (per-token absmax quantised): the sums are exact integers. BitNet
//    applies the layer scale once per row at the end (QORA-LLM-2B, "Ternary
//    GEMV (No Multiplication)"); TQ folds each fp16 group scale into an exact
//    int64 count of 2^-24 (every fp16 value is an integer multiple of 2^-24),
//    so the result is the exactly rounded group-scaled sum in any order.
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
  size_t bars, ring, xa, xb, xc, gsum, gmult, flag, total;
  int stage_bytes;
};

__host__ __device__ inline int group_cols(int group, bool tq) { return tq ? (group >= 64 ? group / 64 : 1) : 1; }

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemPlan smem_plan(const Gemv2Params& p, int xmode, int mt) {
  SmemPlan s{};
  const bool tq = p.scale != nullptr;
  const int kr = p.cols_per_split * kColK2;                       // k per split
  const int gr = tq ? (kr + p.group - 1) / p.group : 1;             // groups per split
  const int gps = tq ? (p.stage_cols * kColK2 + p.group - 1) / p.group : 0;  // groups per stage
  s.stage_bytes = (int)align_up((size_t)p.stage_cols * p.planes * kPlaneColBytes + (size_t)gps * p.planes * 64, 128);
  size_t off = 0;
  s.bars = off;
  off = align_up(off + (size_t)p.wpc * p.nstage * 8, 128);
  s.ring = off;
  off += (size_t)p.wpc * p.nstage * s.stage_bytes;
  s.xa = off;  // int8 x [mt][kr], or the signed high byte of the bf16 image [kr]
  off = align_up(off + (size_t)(xmode == kXInt8 ? mt : 1) * kr, 128);
  s.xb = off;  // bf16 image: middle byte [kr]
  off = align_up(off + (xmode == kXBf16 ? (size_t)kr : 0), 128);
  s.xc = off;  // bf16 image: low byte [kr]
  off = align_up(off + (xmode == kXBf16 ? (size_t)kr : 0), 128);
  s.gsum = off;  // int32 [mt][gr]: sum x (int8); int64 [gr]: sum q (bf16)
  off = align_up(off + (size_t)mt * gr * (xmode == kXBf16 ? 8 : 4), 16);
  s.gmult = off;  // float [gr]: 2^(E-22) (bf16)
  off = align_up(off + (xmode == kXBf16 ? (size_t)gr * 4 : 0), 16);
  s.flag = off;
  off += 16;
  s.total = off;
  return s;
}

// ------------------------------------------------------------ activations
template <int MT>
__device__ void stage_x_int8(const Gemv2Params& p, const SmemPlan& sp, uint8_t* smem, int k0, int kr, int gsz) {
  int8_t* xs = reinterpret_cast<int8_t*>(smem + sp.xa);
  int* gs = reinterpret_cast<int*>(smem + sp.gsum);
  const int8_t* x = static_cast<const int8_t*>(p.x);
  const int m = p.m;
  for (int i = threadIdx.x; i < MT * kr; i += blockDim.x) {
    const int mm = i / kr, kk = i - mm * kr;
    const int k = k0 + kk;
    xs[i] = (mm < m && k < p.k) ? x[(size_t)mm * p.k + k] : 0;
  }
  __syncthreads();
  const int gr = (kr + gsz - 1) / gsz;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int t = warp; t < MT * gr; t += nw) {
    const int mm = t / gr, g = t - mm * gr;
    int s = 0;
    for (int kk = g * gsz + lane; kk < min(kr, (g + 1) * gsz); kk += 32) s += xs[mm * kr + kk];
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) gs[mm * gr + g] = s;
  }
}

__device__ void stage_x_bf16(const Gemv2Params& p, const SmemPlan& sp, uint8_t* smem, int k0, int kr) {
  int8_t* xh = reinterpret_cast<int8_t*>(smem + sp.xa);
  uint8_t* xm = smem + sp.xb;
  uint8_t* xl = smem + sp.xc;
  long long* gs = reinterpret_cast<long long*>(smem + sp.gsum);
  float* gm = reinterpret_cast<float*>(smem + sp.gmult);
  const uint16_t* x = static_cast<const uint16_t*>(p.x);
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
__global__ void __launch_bounds__(256) gemv2_kernel(const Gemv2Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr bool kTQ = WG > 0;
  const SmemPlan sp = smem_plan(p, XM, MT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = blockIdx.x * p.wpc + warp;
  const bool active = T < p.row_tiles;
  const int split = blockIdx.y;
  const int c0 = split * p.cols_per_split;
  const int c1 = min(p.cols, c0 + p.cols_per_split);
  const int ncols = c1 - c0;
  const int sc = p.stage_cols, nst = p.nstage;
  const int nstages = (ncols + sc - 1) / sc;
  const int gpc = kTQ ? (p.group >= 64 ? 0 : 64 / p.group) : 0;  // groups per column when g < 64
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sp.bars) + warp * nst;
  uint8_t* ring = smem + sp.ring + (size_t)warp * nst * sp.stage_bytes;

  // ---- prologue: barriers and the first weight stages (independent of x)
  if (active && lane == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int i) {
    const int slot = i % nst;
    const int cs = c0 + i * sc, ce = min(c1, cs + sc);
    const uint32_t tb = (uint32_t)(ce - cs) * P * kPlaneColBytes;
    const uint8_t* src = p.trit + ((size_t)T * p.cols + cs) * P * kPlaneColBytes;
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
               reinterpret_cast<const uint8_t*>(p.scale) + ((size_t)T * p.groups + ga) * P * 64, sb, &bars[slot],
               pol);
  };
  if (active && lane == 0)
    for (int i = 0; i < min(nst, nstages); ++i) issue(i);
  pdl_launch_dependents();

  // ---- wait for the producer of x, then stage x for this K-split
  pdl_wait();
  const int k0 = c0 * kColK2, kr = ncols * kColK2;
  if (XM == kXInt8)
    stage_x_int8<MT>(p, sp, smem, k0, kr, kTQ ? p.group : kr);
  else
    stage_x_bf16(p, sp, smem, k0, kr);
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
          if (XM == kXInt8) {
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
          if (kTQ) {
            const int wglob = (cs + cc - c0) * 4 + wi;  // word index within the split
            if ((wglob + 1) % WG == 0) {
              const int gl = wglob / WG;                   // group within the split
              const int gst = (cs * kColK2 + ((cc * 4 + wi) * 16)) / p.group - ga_stage;  // within stage
#pragma unroll
              for (int q = 0; q < P; ++q) {
                const uint16_t h = sst[((size_t)gst * P + q) * kTileRows + lane];
                if (XM == kXInt8) {
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
  (void)gpc;
  if (active && ifail >= 0) {
    // a wait expired: give the copies still in flight a bounded chance to land
    for (int j = ifail; j < min(nstages, ifail + nst); ++j) mbar_wait_bounded(&bars[j % nst], (uint32_t)(j / nst) & 1u);
  }

  // ---- epilogue: per-lane row results (int32 BitNet / int64 TQ-int8 / fp32 bf16)
  const int npad = p.row_tiles * kTileRows;
  const int row = T * kTileRows + lane;
  int accb[MT];
  if (!kTQ) {
#pragma unroll
    for (int t = 0; t < MT; ++t) accb[t] = (t < m) ? gsum[t] - (a[0][t] + (b[0][t] >> 4)) : 0;
  }

  auto write_out = [&](int t, float v) {
    if (p.out_bf16)
      reinterpret_cast<__nv_bfloat16*>(p.y)[(size_t)t * p.n + row] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<float*>(p.y)[(size_t)t * p.n + row] = v;
  };
  auto finish = [&](int t, long long v64, int v32, float vf) {
    if (row >= p.n) return;
    if (XM == kXBf16) {
      write_out(t, vf);
    } else if (kTQ) {
      const float s = __fmul_rn(__ll2float_rn(v64), 0x1p-24f);
      write_out(t, __fmul_rn(s, p.xscale[t]));
    } else {
      write_out(t, __fmul_rn(__fmul_rn(__int2float_rn(v32), p.tensor_scale), p.xscale[t]));
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

  // ---- split-K: publish partials; the last CTA of this row group reduces
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
  int* flag = reinterpret_cast<int*>(smem + sp.flag);
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
  if (threadIdx.x == 0) p.ws_cnt[blockIdx.x] = 0u;  // leave the workspace zeroed
}

// ------------------------------------------------------------------ launch
size_t gemv2_smem_bytes(const Gemv2Params& p, int xmode) {
  const int mt = xmode == kXBf16 ? 1 : (p.m <= 1 ? 1 : p.m <= 4 ? 4 : 16);
  return smem_plan(p, xmode, mt).total;
}

template <int XM, int P, int WG, int MT>
static int launch_one(const Gemv2Params& p, bool pdl, void* stream) {
  const SmemPlan sp = smem_plan(p, XM, MT);
  auto kern = gemv2_kernel<XM, P, WG, MT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
  if (e != cudaSuccess) return (int)e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.row_tiles + p.wpc - 1) / p.wpc, p.ks, 1);
  cfg.blockDim = dim3(32 * p.wpc, 1, 1);
  cfg.dynamicSmemBytes = sp.total;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  return (int)e;
}

// Instantiated combinations; anything else reports "unsupported" (-1).
int launch_gemv2(const Gemv2Params& p, int xmode, bool pdl, void* stream) {
  const bool tq = p.scale != nullptr;
  const int wg = tq ? p.group / 16 : 0;
  if (xmode == kXInt8) {
    const int mt = p.m <= 1 ? 1 : p.m <= 4 ? 4 : 16;
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
