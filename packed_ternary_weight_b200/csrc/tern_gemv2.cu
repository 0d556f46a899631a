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

#include <type_traits>

#include "tern_gemv_common.cuh"
#include "tern_ptx.cuh"

namespace tern {

int read_clear_dev_error_gemv2(void* stream, unsigned* out) { return read_clear_dev_error_tu(stream, out); }

namespace {

constexpr uint32_t kM03 = 0x03030303u;
constexpr uint32_t kM30 = 0x30303030u;

struct SmemPlan {
  size_t bars, cbar, ring, xa, xb, xc, xraw, gsum, gmult, red, amx, misc, total;
  int stage_bytes;
};

using gemv_common::align_up;
using gemv_common::u4_get;

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
  off += (size_t)p.wpc * p.nstage * 8;
  s.cbar = off;  // K split over a cluster: [0] the splits' token maxima arrived, [1] their partial sums
  off = align_up(off + 16, 128);
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
// Sum of the 16 signed bytes of v.
__device__ __forceinline__ int sum16_s8(uint4 v) {
  int s = __dp4a((int)v.x, 0x01010101, 0);
  s = __dp4a((int)v.y, 0x01010101, s);
  s = __dp4a((int)v.z, 0x01010101, s);
  return __dp4a((int)v.w, 0x01010101, s);
}

// Adds chunk sums to the per-(token, group) sums in shared memory with one
// atomic per change of group (a thread's chunks of one BitNet token all fall
// in the same group).
struct GroupSumAcc {
  int* gs;
  int key = -1, val = 0;
  __device__ void add(int k, int v) {
    if (k != key) {
      if (key >= 0) atomicAdd(&gs[key], val);
      key = k;
      val = 0;
    }
    val += v;
  }
  __device__ void flush() {
    if (key >= 0) atomicAdd(&gs[key], val);
  }
};

template <int MT>
__device__ void stage_x_int8(const Gemv2Params& p, const Gemv2Problem& pr, const SmemPlan& sp, uint8_t* smem, int k0,
                             int kr, int gsz) {
  int8_t* xs = reinterpret_cast<int8_t*>(smem + sp.xa);
  const int8_t* x = static_cast<const int8_t*>(pr.x);
  const int m = p.m, K = p.k, nch = kr / 16, gr = (kr + gsz - 1) / gsz;
  GroupSumAcc acc{reinterpret_cast<int*>(smem + sp.gsum)};
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
    acc.add(t * gr + (16 * c) / gsz, sum16_s8(v));
  }
  acc.flush();
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
// every split sends its token maxima to every CTA of the cluster with
// st.async, and each CTA waits for them on its own barrier.
template <int MT>
__device__ void stage_x_q8(const Gemv2Params& p, const Gemv2Problem& pr, const SmemPlan& sp, uint8_t* smem, int k0,
                           int kr, int gsz, bool clus, int split) {
  uint16_t* raw = reinterpret_cast<uint16_t*>(smem + sp.xraw);
  int8_t* xs = reinterpret_cast<int8_t*>(smem + sp.xa);
  unsigned* tmax = reinterpret_cast<unsigned*>(smem + sp.misc);     // [MT], zeroed in the prologue
  float* sxs = reinterpret_cast<float*>(smem + sp.misc) + MT;        // [MT]
  float* amx = reinterpret_cast<float*>(smem + sp.amx);             // [ks][MT]
  const uint16_t* x = static_cast<const uint16_t*>(pr.x);
  const int m = p.m, K = p.k, nch = kr / 8;
  float lmax[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) lmax[t] = 0.f;
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
    const float mx8 = bf16_abs_max8(v);
#pragma unroll
    for (int u = 0; u < MT; ++u)
      if (t == u) lmax[u] = fmaxf(lmax[u], mx8);
  }
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    float mx = lmax[t];
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0 && mx > 0.f) atomicMax(&tmax[t], __float_as_uint(mx));
  }
  __syncthreads();
  if (clus) {
    uint64_t* xbar = reinterpret_cast<uint64_t*>(smem + sp.cbar);
    if (threadIdx.x == 0) mbar_arrive_expect_tx(xbar, (uint32_t)(p.ks * MT * 4));
    for (int i = threadIdx.x; i < p.ks * MT; i += blockDim.x) {
      const int r = i / MT, t = i - r * MT;
      st_async_u32(map_cluster_rank(smem_u32(&amx[split * MT + t]), (uint32_t)r), tmax[t],
                   map_cluster_rank(smem_u32(xbar), (uint32_t)r));
    }
    (void)mbar_wait_bounded<true>(xbar, 0);  // on expiry the error word records a timeout
  }
  float inv[MT];
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    // maxima are non-negative floats: their bit patterns order like the values
    unsigned ab = tmax[t];
    if (clus) ab = __reduce_max_sync(0xffffffffu, lane < p.ks ? __float_as_uint(amx[lane * MT + t]) : 0u);
    const float a = __uint_as_float(ab);
    inv[t] = a > 0.f ? __fdiv_rn(127.0f, a) : 0.f;
    if (threadIdx.x == 0) sxs[t] = a > 0.f ? __fdiv_rn(a, 127.0f) : 0.f;
  }
  const int n16 = kr / 16, gr = (kr + gsz - 1) / gsz;
  GroupSumAcc acc{reinterpret_cast<int*>(smem + sp.gsum)};
  for (int i = threadIdx.x; i < MT * n16; i += blockDim.x) {
    const int t = i / n16, c = i - t * n16;
    float it = inv[0];
#pragma unroll
    for (int u = 1; u < MT; ++u)
      if (t == u) it = inv[u];
    const uint4 v0 = *reinterpret_cast<const uint4*>(raw + t * kr + 16 * c);
    const uint4 v1 = *reinterpret_cast<const uint4*>(raw + t * kr + 16 * c + 8);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t packed[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t h = (j & 1) ? (w[j >> 1] >> 16) : (w[j >> 1] & 0xFFFFu);
      int q = __float2int_rn(__fmul_rn(__uint_as_float(h << 16), it));
      q = max(-127, min(127, q));
      packed[j >> 2] |= ((uint32_t)q & 0xFFu) << (8 * (j & 3));
    }
    const uint4 pv = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    *reinterpret_cast<uint4*>(xs + t * kr + 16 * c) = pv;
    acc.add(t * gr + (16 * c) / gsz, sum16_s8(pv));
  }
  acc.flush();
}

__device__ void stage_x_bf16(const Gemv2Params& p, const Gemv2Problem& pr, const SmemPlan& sp, uint8_t* smem, int k0,
                             int kr) {
  gemv_common::stage_x_bf16_image(static_cast<const uint16_t*>(pr.x), p.k, p.group, k0, kr,
                                  reinterpret_cast<int8_t*>(smem + sp.xa), smem + sp.xb, smem + sp.xc,
                                  reinterpret_cast<long long*>(smem + sp.gsum), reinterpret_cast<float*>(smem + sp.gmult));
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
  const int split = blockIdx.y;
  const bool clus = p.cluster && p.ks > 1;
  const int c0 = split * p.cols_per_split;
  const int c1 = min(p.cols, c0 + p.cols_per_split);
  const int ncols = c1 - c0;
  const int sc = p.stage_cols, nst = p.nstage;
  const int spt = (ncols + sc - 1) / sc;  // stages per row tile
  const int m = p.m;
  const int k0 = c0 * kColK2, kr = ncols * kColK2;
  const int gr = kTQ ? kr / p.group : 1;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sp.bars) + warp * nst;
  uint8_t* ring = smem + sp.ring + (size_t)warp * nst * sp.stage_bytes;

  // Row groups (wpc consecutive row tiles of one problem) handled by this CTA:
  // one, or, in a persistent launch (no K split), a contiguous range of them,
  // so that each warp's weight stream runs on across tile boundaries and the
  // activations are staged once per problem.
  int gbeg = blockIdx.x, gend = blockIdx.x + 1;
  if (p.persistent) {
    gbeg = (int)((long long)p.groups_total * blockIdx.x / gridDim.x);
    gend = (int)((long long)p.groups_total * (blockIdx.x + 1) / gridDim.x);
  }
  auto prob_of = [&](int gi) {
    int q = 0;
    while (q + 1 < p.nprob && gi >= p.prob[q + 1].cta_begin) ++q;
    return q;
  };
  auto tile_of = [&](int gi, int q) { return (gi - p.prob[q].cta_begin) * p.wpc + warp; };

  // ---- prologue (independent of the preceding kernel): barriers, first weight stages
  if (clus && threadIdx.x == 0) {
    uint64_t* cbar = reinterpret_cast<uint64_t*>(smem + sp.cbar);
    mbar_init(cbar, 1);      // the token maxima (in-kernel quantisation)
    mbar_init(cbar + 1, 1);  // the splits' partial sums (rank 0)
    fence_mbar_init();
  }
  // other CTAs store into this one's shared memory only after every CTA of the
  // cluster runs and has initialised its barriers
  if (clus) cluster_arrive_relaxed();
  if (lane == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = policy_evict_first();
  // issue cursor of this warp (used by lane 0): next (row group, stage) to
  // request, with the problem of that row group tracked incrementally
  int ig = gbeg, iq = prob_of(gbeg), is_ = 0, nissued = 0, islot = 0;
  auto cursor_skip_inactive = [&]() {
    while (ig < gend) {
      while (iq + 1 < p.nprob && ig >= p.prob[iq + 1].cta_begin) ++iq;
      if (tile_of(ig, iq) < p.prob[iq].row_tiles) break;
      ++ig;
    }
  };
  cursor_skip_inactive();
  auto issue_next = [&]() {
    if (ig >= gend) return;
    const Gemv2Problem& pq = p.prob[iq];
    const int T = tile_of(ig, iq);
    const int slot = islot;
    islot = islot + 1 == nst ? 0 : islot + 1;
    const int cs = c0 + is_ * sc, ce = min(c1, cs + sc);
    const uint32_t tb = (uint32_t)(ce - cs) * P * kPlaneColBytes;
    const uint8_t* src = pq.trit + ((size_t)T * p.cols + cs) * P * kPlaneColBytes;
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
               reinterpret_cast<const uint8_t*>(pq.scale) + ((size_t)T * p.groups + ga) * P * 64, sb, &bars[slot],
               pol);
    ++nissued;
    if (++is_ == spt) {
      is_ = 0;
      ++ig;
      cursor_skip_inactive();
    }
  };
  if (lane == 0)
    for (int i = 0; i < nst; ++i) issue_next();
  pdl_launch_dependents();

  // ---- wait for the producer of x
  pdl_wait();
  if (clus) cluster_wait_acquire();

  const int* gsum = reinterpret_cast<const int*>(smem + sp.gsum);
  const long long* gsum64 = reinterpret_cast<const long long*>(smem + sp.gsum);
  const float* gmul = reinterpret_cast<const float*>(smem + sp.gmult);
  const float* sxs = reinterpret_cast<const float*>(smem + sp.misc) + MT;

  // Accumulators. After the digit transform a word holds 16 digits F = 1 - t,
  // four 2-bit fields per byte; field f of every byte lines up with the four
  // activations x[4f .. 4f+3]. With one token each field is masked in place
  // (value 4^f * F) and keeps its own accumulator, combined exactly at the end
  // (acc_f is a multiple of 4^f); with several tokens, fields 1 and 3 are
  // shifted down first and two accumulators (weights 1 and 16) are kept.
  constexpr int NF = MT == 1 ? 4 : 2;
  int acc[P][MT][NF];          // int8 x, or the high bytes of the bf16 image
  unsigned accm[P][NF];        // bf16 image: middle bytes
  unsigned accl[P][NF];        // bf16 image: low bytes
  long long acc64[MT];         // TQ int8: exact sum in units of 2^-24
  float yacc;                  // bf16
  auto reset = [&]() {
#pragma unroll
    for (int q = 0; q < P; ++q)
#pragma unroll
      for (int f = 0; f < NF; ++f) {
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[q][t][f] = 0;
        accm[q][f] = accl[q][f] = 0;
      }
#pragma unroll
    for (int t = 0; t < MT; ++t) acc64[t] = 0;
    yacc = 0.f;
  };
  // sum F*x over the chains
  auto fold_int = [&](const int* c) -> int {
    if (NF == 4) return c[0] + (c[1] >> 2) + (c[2] >> 4) + (c[3] >> 6);
    return c[0] + (c[NF - 1] >> 4);
  };
  auto fold_u = [&](const unsigned* c) -> int {
    if (NF == 4) return (int)(c[0] + (c[1] >> 2) + (c[2] >> 4) + (c[3] >> 6));
    return (int)(c[0] + (c[NF - 1] >> 4));
  };
  // one 16-k word of plane q against the int8 activations of token t
  auto word_int = [&](int q, int t, uint32_t F, int4 xv) {
    if (NF == 4) {
      acc[q][t][0] = dp4a_ss((int)(F & 0x03030303u), xv.x, acc[q][t][0]);
      acc[q][t][1] = dp4a_ss((int)(F & 0x0C0C0C0Cu), xv.y, acc[q][t][1]);
      acc[q][t][2] = dp4a_ss((int)(F & 0x30303030u), xv.z, acc[q][t][2]);
      acc[q][t][NF - 1] = dp4a_us(F & 0xC0C0C0C0u, xv.w, acc[q][t][NF - 1]);
    } else {
      const uint32_t F2 = F >> 2;
      acc[q][t][0] = dp4a_ss((int)(F & kM03), xv.x, acc[q][t][0]);
      acc[q][t][0] = dp4a_ss((int)(F2 & kM03), xv.y, acc[q][t][0]);
      acc[q][t][NF - 1] = dp4a_ss((int)(F & kM30), xv.z, acc[q][t][NF - 1]);
      acc[q][t][NF - 1] = dp4a_ss((int)(F2 & kM30), xv.w, acc[q][t][NF - 1]);
    }
  };
  // one word of plane q against the three bytes of the bf16 image (one token)
  auto word_bf = [&](int q, uint32_t F, int4 hv, uint4 mv, uint4 lv) {
    const uint32_t d0 = F & 0x03030303u, d1 = F & 0x0C0C0C0Cu, d2 = F & 0x30303030u, d3 = F & 0xC0C0C0C0u;
    acc[q][0][0] = dp4a_ss((int)d0, hv.x, acc[q][0][0]);
    acc[q][0][1] = dp4a_ss((int)d1, hv.y, acc[q][0][1]);
    acc[q][0][2] = dp4a_ss((int)d2, hv.z, acc[q][0][2]);
    acc[q][0][NF - 1] = dp4a_us(d3, hv.w, acc[q][0][NF - 1]);
    accm[q][0] = dp4a_uu(d0, mv.x, accm[q][0]);
    accm[q][1] = dp4a_uu(d1, mv.y, accm[q][1]);
    accm[q][2] = dp4a_uu(d2, mv.z, accm[q][2]);
    accm[q][NF - 1] = dp4a_uu(d3, mv.w, accm[q][NF - 1]);
    accl[q][0] = dp4a_uu(d0, lv.x, accl[q][0]);
    accl[q][1] = dp4a_uu(d1, lv.y, accl[q][1]);
    accl[q][2] = dp4a_uu(d2, lv.z, accl[q][2]);
    accl[q][NF - 1] = dp4a_uu(d3, lv.w, accl[q][NF - 1]);
  };

  int cur_prob = -1, nconsumed = 0, ifail = -1, pi = prob_of(gbeg);
  int cslot = 0;
  uint32_t cphase = 0;
  const uint32_t x32 = smem_u32(smem + sp.xa), xm32 = smem_u32(smem + sp.xb), xl32 = smem_u32(smem + sp.xc);
  const uint32_t ring32 = smem_u32(ring) + lane * 16;
  for (int gi = gbeg; gi < gend; ++gi) {
    while (pi + 1 < p.nprob && gi >= p.prob[pi + 1].cta_begin) ++pi;
    const Gemv2Problem& pr = p.prob[pi];
    if (pi != cur_prob) {
      // ---- stage x of this problem for this K-split (once per problem)
      __syncthreads();
      if (kIntX)
        for (int i = threadIdx.x; i < MT * gr; i += blockDim.x) reinterpret_cast<int*>(smem + sp.gsum)[i] = 0;
      if (XM == kXBf16Q8 && threadIdx.x < MT) reinterpret_cast<unsigned*>(smem + sp.misc)[threadIdx.x] = 0u;
      __syncthreads();
      if (XM == kXInt8)
        stage_x_int8<MT>(p, pr, sp, smem, k0, kr, kTQ ? p.group : kr);
      else if (XM == kXBf16Q8)
        stage_x_q8<MT>(p, pr, sp, smem, k0, kr, kTQ ? p.group : kr, clus, split);
      else
        stage_x_bf16(p, pr, sp, smem, k0, kr);
      __syncthreads();
      cur_prob = pi;
    }
    const int T = tile_of(gi, pi);
    const bool active = T < pr.row_tiles;
    reset();
    if (active && ifail < 0) {
      for (int s = 0; s < spt; ++s, ++nconsumed) {
        const int slot = cslot;
        const uint32_t phase = cphase;
        if (++cslot == nst) {
          cslot = 0;
          cphase ^= 1u;
        }
        // warp-uniform outcome, so that no lane is left behind at __syncwarp
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars[slot], phase))) {
          ifail = nconsumed;
          break;
        }
        const uint8_t* st = ring + (size_t)slot * sp.stage_bytes;
        const uint32_t st32 = ring32 + (uint32_t)slot * sp.stage_bytes;
        const uint16_t* sst = reinterpret_cast<const uint16_t*>(st + (size_t)sc * P * kPlaneColBytes);
        const int cs = c0 + s * sc;
        const int ncs = min(sc, c1 - cs);
        const int ga_stage = kTQ ? cs * kColK2 / p.group : 0;
        // one 16-k word (index WI of the column) of every plane
        auto word_step = [&](auto wi_c, const uint4* wv, int cc, int kx) {
          constexpr int wi = decltype(wi_c)::value;
          const uint32_t xo = (uint32_t)kx;
          uint32_t F[P];
#pragma unroll
          for (int q = 0; q < P; ++q) F[q] = lop3_ternary_digit(u4_get<wi>(wv[q]));
          if (kIntX) {
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              if (MT == 1 || t < m) {
                const int4 xv = u4_as_i4(lds128<wi * 16>(x32 + (uint32_t)(t * kr) + xo));
#pragma unroll
                for (int q = 0; q < P; ++q) word_int(q, t, F[q], xv);
              }
            }
          } else {
            const int4 hv = u4_as_i4(lds128<wi * 16>(x32 + xo));
            const uint4 mv = lds128<wi * 16>(xm32 + xo);
            const uint4 lv = lds128<wi * 16>(xl32 + xo);
#pragma unroll
            for (int q = 0; q < P; ++q) word_bf(q, F[q], hv, mv, lv);
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
                    if (MT == 1 || t < m) {
                      const int S = gsum[t * gr + gl] - fold_int(acc[q][t]);
                      acc64[t] += fold_fp16_exact(h, S);
                    }
#pragma unroll
                    for (int f = 0; f < NF; ++f) acc[q][t][f] = 0;
                  }
                } else {
                  const int H = fold_int(acc[q][0]);
                  const int Mi = fold_u(accm[q]);
                  const int L = fold_u(accl[q]);
                  const long long S = gsum64[gl] - ((long long)H * 65536 + (long long)Mi * 256 + L);
                  yacc = fmaf(__half2float(__ushort_as_half(h)) * gmul[gl], __ll2float_rn(S), yacc);
#pragma unroll
                  for (int f = 0; f < NF; ++f) acc[q][0][f] = accm[q][f] = accl[q][f] = 0;
                }
              }
            }
          }
        };
        for (int cc = 0; cc < ncs; ++cc) {
          const int kx = (cs + cc - c0) * kColK2;
          uint4 wv[P];
          const uint32_t wc = st32 + (uint32_t)(cc * P * kPlaneColBytes);
          wv[0] = lds128<0>(wc);
          if constexpr (P > 1) wv[1] = lds128<kPlaneColBytes>(wc);
          if constexpr (P > 2) wv[2] = lds128<2 * kPlaneColBytes>(wc);
          if constexpr (P > 3) wv[3] = lds128<3 * kPlaneColBytes>(wc);
          word_step(std::integral_constant<int, 0>{}, wv, cc, kx);
          word_step(std::integral_constant<int, 1>{}, wv, cc, kx);
          word_step(std::integral_constant<int, 2>{}, wv, cc, kx);
          word_step(std::integral_constant<int, 3>{}, wv, cc, kx);
        }
        // release the slot: reads of this stage are complete before the refill
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) issue_next();
      }
    }

    // ---- epilogue of this row tile: per-lane results (int32 BitNet / int64 TQ-int8 / fp32 bf16)
    const int npad = pr.row_tiles * kTileRows;
    const int row = T * kTileRows + lane;
    int accb[MT];
    if (!kTQ) {
#pragma unroll
      for (int t = 0; t < MT; ++t) accb[t] = (MT == 1 || t < m) ? gsum[t] - fold_int(acc[0][t]) : 0;
    }
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
        const float sv = __fmul_rn(__ll2float_rn(v64), 0x1p-24f);
        write_out(t, __fmul_rn(sv, sx));
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
      continue;
    }

    // ---- K is split (one row group per CTA): combine the splits' partial sums
    if (active && ifail >= 0) {
      // a wait expired: give the copies still in flight a bounded chance to land
      for (int j = ifail; j < min(nissued, ifail + nst); ++j)
        mbar_wait_bounded(&bars[j % nst], (uint32_t)(j / nst) & 1u);  // error path only
    }
    if (clus) {
      // the splits of this row group form the cluster: each sends its partial
      // sums to CTA rank 0 with st.async, which waits for them on its own
      // barrier, sums them in split order and writes the outputs; the other
      // CTAs are then done
      const int rows_cta = p.wpc * kTileRows;
      const int esz = red_elem(XM, kTQ);
      uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + sp.cbar) + 1;
      if (split == 0 && threadIdx.x == 0) {
        // every split's partials of the active warps (the same warps in every split)
        const int nact = max(0, min(p.wpc, pr.row_tiles - (T - warp)));
        mbar_arrive_expect_tx(rbar, (uint32_t)(p.ks * m * nact * kTileRows * esz));
      }
      if (active) {
        const uint32_t rbar0 = map_cluster_rank(smem_u32(rbar), 0);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          if (t >= m) continue;
          const size_t idx = ((size_t)split * MT + t) * rows_cta + warp * kTileRows + lane;
          const uint32_t dst = map_cluster_rank(smem_u32(smem + sp.red + idx * esz), 0);
          if (XM == kXBf16)
            st_async_u32(dst, __float_as_uint(yacc), rbar0);
          else if (kTQ)
            st_async_u64(dst, (unsigned long long)acc64[t], rbar0);
          else
            st_async_u32(dst, (uint32_t)accb[t], rbar0);
        }
      }
      if (split == 0) {
        (void)mbar_wait_bounded<true>(rbar, 0);  // on expiry the error word records a timeout
        if (active) {
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
      }
      return;
    }

    // more splits than a cluster holds: partials through the global workspace,
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
    return;
  }
  if (ifail >= 0) {
    // a wait expired: give the copies still in flight a bounded chance to land
    for (int j = ifail; j < min(nissued, ifail + nst); ++j) mbar_wait_bounded(&bars[j % nst], (uint32_t)(j / nst) & 1u);
  }
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
  // without a K split, run at most as many CTAs as fit at once; each then
  // walks a contiguous range of row groups
  Gemv2Params q = p;
  q.groups_total = p.grid_x;
  q.persistent = 0;
  int gx = p.grid_x;
  if (p.ks == 1) {
    int dev = 0, sms = 0, occ = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 32 * p.wpc, sp.total);
    if (e != cudaSuccess) return (int)e;
    if (occ > 0 && gx > sms * occ) {
      gx = sms * occ;
      q.persistent = 1;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gx, p.ks, 1);
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
  e = cudaLaunchKernelEx(&cfg, kern, q);
  return (int)e;
}

// Instantiated combinations; anything else reports "unsupported" (-1).
// Planes x group: TQ with 1-4 planes at g = 32, 64, 128 or 256 (sasori
// README, "K and g"); BitNet one plane.
#define TERN_TQ_CASES(XM, MT) \
  switch (p.planes * 100 + wg) { \
    case 102: return launch_one<XM, 1, 2, MT>(p, pdl, stream); \
    case 104: return launch_one<XM, 1, 4, MT>(p, pdl, stream); \
    case 108: return launch_one<XM, 1, 8, MT>(p, pdl, stream); \
    case 116: return launch_one<XM, 1, 16, MT>(p, pdl, stream); \
    case 202: return launch_one<XM, 2, 2, MT>(p, pdl, stream); \
    case 204: return launch_one<XM, 2, 4, MT>(p, pdl, stream); \
    case 208: return launch_one<XM, 2, 8, MT>(p, pdl, stream); \
    case 216: return launch_one<XM, 2, 16, MT>(p, pdl, stream); \
    case 302: return launch_one<XM, 3, 2, MT>(p, pdl, stream); \
    case 304: return launch_one<XM, 3, 4, MT>(p, pdl, stream); \
    case 308: return launch_one<XM, 3, 8, MT>(p, pdl, stream); \
    case 316: return launch_one<XM, 3, 16, MT>(p, pdl, stream); \
    case 402: return launch_one<XM, 4, 2, MT>(p, pdl, stream); \
    case 404: return launch_one<XM, 4, 4, MT>(p, pdl, stream); \
    case 408: return launch_one<XM, 4, 8, MT>(p, pdl, stream); \
    case 416: return launch_one<XM, 4, 16, MT>(p, pdl, stream); \
    default: return -1; \
  }

int launch_gemv2(const Gemv2Params& p, int xmode, bool pdl, void* stream) {
  const bool tq = p.tq != 0;
  const int wg = tq ? p.group / 16 : 0;
  const int mt = gemv2_mt(xmode, p.m);
  if (!tq) {
    if (p.planes != 1) return -1;
    if (xmode == kXInt8) {
      if (mt == 1) return launch_one<kXInt8, 1, 0, 1>(p, pdl, stream);
      if (mt == 4) return launch_one<kXInt8, 1, 0, 4>(p, pdl, stream);
      return launch_one<kXInt8, 1, 0, 16>(p, pdl, stream);
    }
    if (xmode == kXBf16Q8) {
      if (mt == 1) return launch_one<kXBf16Q8, 1, 0, 1>(p, pdl, stream);
      return launch_one<kXBf16Q8, 1, 0, 4>(p, pdl, stream);
    }
    return -1;
  }
  if (xmode == kXInt8) {
    if (mt == 1) TERN_TQ_CASES(kXInt8, 1)
    if (p.planes == 2 && wg == 2) {
      if (mt == 4) return launch_one<kXInt8, 2, 2, 4>(p, pdl, stream);
      return launch_one<kXInt8, 2, 2, 16>(p, pdl, stream);
    }
    return -1;
  }
  if (xmode == kXBf16Q8) {
    if (mt == 1) TERN_TQ_CASES(kXBf16Q8, 1)
    if (p.planes == 2 && wg == 2) return launch_one<kXBf16Q8, 2, 2, 4>(p, pdl, stream);
    return -1;
  }
  if (p.m != 1) return -1;
  TERN_TQ_CASES(kXBf16, 1)
}
#undef TERN_TQ_CASES

}  // namespace tern
