// Kernel template of the one-CTA-per-SM decode GEMV (gemv2w), shared by the
// translation units that instantiate it: tern_gemv2w.cu (one token per
// problem) and tern_gemv2w_mt.cu (several tokens sharing one weight stream).
//
// Single-token decode GEMV over 2-bit ternary planes with one CTA per SM
// (BitNet b1.58 single plane with a per-tensor scale; sasori-style additive
// TQ{K}P planes with fp16 group scales).
//
// Work split. The row tiles (32 rows) of all problems of the launch form one
// list; CTA c takes a contiguous range of it that starts at the first tile
// whose first column is at or after the c-th equal share of all columns
// (gemv2w_cta_tile), so that every SM gets the same number of columns to
// within one tile when problems differ in K. Inside the CTA the columns of
// that range (tiles x columns, in memory order; a tile has its own problem's
// column count) are split into equal contiguous ranges, one per warp, in units
// of whole scale groups. A warp
// therefore streams one contiguous stretch of each problem's packed bytes and
// the warps of a CTA finish together to within one column. A tile that lies
// inside one warp's range is finished by that warp; a tile cut by one or more
// warp boundaries is finished by the last of its warps to arrive, which adds
// the partial row sums in warp order (fixed order, so results do not depend on
// timing).
//
// Activations. Every problem a CTA touches has its activation image resident
// in shared memory for the whole launch (int8 with column or group sums for
// the integer paths; the 24-bit fixed-point image for bf16). The activations
// are read before most weight copies are requested, so that their loads do
// not queue behind megabytes of weight traffic.
//
// Weight stream and inner loop: per-warp rings of bulk async copies on
// mbarriers (bounded waits), and the digit transform F = 1 - t with byte
// dot-products, as in the row-group kernel (tern_gemv2.cu).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <type_traits>

#include "tern_gemv_common.cuh"
#include "tern_ptx.cuh"

namespace tern {

namespace {

using gemv_common::align_up;
using gemv_common::u4_get;

constexpr int kXR = 4;  // 16-byte activation chunks a thread holds in registers while staging

struct Plan2w {
  size_t bars, ring, xs, red, cnt, misc, total;
  size_t slot_bytes, sum_off, sx_off;  // per activation slot: sums and scale offsets
  int stage_bytes, kx;
};

// Shared-memory layout (host and device agree on it).
//   bars  [nw][nstage] mbarriers
//   ring  [nw][nstage] stages: stage_cols columns of P planes, then the stage's fp16 scales
//   xs    [xslots] activation slots:
//           integer paths: int8 x [kx] | int32 sums (BitNet: prefix sums per column [cols+1];
//                          TQ: per group [groups]) | fp32 token scale
//           bf16 path:     high, middle, low bytes [kx] each | per group {sum h, sum m, sum l,
//                          2^(E-22)} (16 bytes) (| fp32 codebook [27] for balanced ternary d = 3)
//   red   [nw][2][32] partial row sums of shared tiles (8 bytes each); with
//         several tokens [nw][mt][32] int64 sums of shared tiles, indexed by
//         the tile's first warp and added to atomically
//   cnt   [nw] arrival counters of shared tiles
//   misc  per-warp maxima [images][nw] for the in-kernel quantisation
// Activation images: one per problem (xslots), or one per token (mt > 1, a
// single problem per launch).
__host__ __device__ inline Plan2w plan2w(const Gemv2wParams& p, int xmode) {
  Plan2w s{};
  const bool tq = p.tq != 0;
  const bool bf = xmode == kXBf16;
  s.kx = p.cols * (p.bt3 ? kColK3 : kColK2);
  const int gps = tq ? (p.stage_cols * kColK2 + p.group - 1) / p.group : 0;
  const size_t colb = p.bt3 ? (size_t)kBt3ColBytes : (size_t)p.planes * kPlaneColBytes;
  s.stage_bytes = (int)align_up((size_t)p.stage_cols * colb + (size_t)gps * p.planes * 64, 128);
  if (bf) {
    // the image covers whole columns: d = 3 pads K to a multiple of 80, so it
    // holds kx / 16 groups (TQ: K is a multiple of 64, kx = K)
    const size_t gimg = p.bt3 ? (size_t)s.kx / 16 : (size_t)p.groups;
    s.sum_off = 3 * (size_t)s.kx;       // 16-byte group records {sum h, sum m, sum l, 2^(E-22)}
    s.sx_off = s.sum_off + 16 * gimg;   // d = 3: the 27-entry codebook
    s.slot_bytes = align_up(s.sx_off + (p.bt3 ? 27 * 4 : 0), 128);
  } else {
    s.sum_off = s.kx;
    s.sx_off = align_up(s.sum_off + 4 * (size_t)(tq ? p.groups : p.cols + 1), 16);
    s.slot_bytes = align_up(s.sx_off + 16, 128);
  }
  const size_t nimg = p.mt > 1 ? (size_t)gemv2w_mt_pad(p.mt) : (size_t)p.xslots;
  size_t off = 0;
  s.bars = off;
  off = align_up(off + (size_t)p.nw * p.nstage * 8, 128);
  s.ring = off;
  off += (size_t)p.nw * p.nstage * s.stage_bytes;
  s.xs = off;
  off += nimg * s.slot_bytes;
  s.red = off;
  off = align_up(off + (size_t)p.nw * (p.mt > 1 ? p.mt : 2) * 32 * 8, 16);
  s.cnt = off;
  off = align_up(off + (size_t)p.nw * 4, 16);
  s.misc = off;
  off = align_up(off + nimg * p.nw * 4 + 16, 16);
  s.total = off;
  return s;
}

__device__ __forceinline__ int sum16_s8(uint4 v) {
  int s = __dp4a((int)v.x, 0x01010101, 0);
  s = __dp4a((int)v.y, 0x01010101, s);
  s = __dp4a((int)v.z, 0x01010101, s);
  return __dp4a((int)v.w, 0x01010101, s);
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

// Eight bf16 values x[k .. k+8) (zero beyond K) as one 16-byte vector.
__device__ __forceinline__ uint4 load_bf16x8(const uint16_t* x, int K, int k, bool vec) {
  if (vec && k + 8 <= K) return __ldg(reinterpret_cast<const uint4*>(x + k));
  uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (k + j < K) w[j >> 1] |= (uint32_t)x[k + j] << (16 * (j & 1));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Sixteen int8 values x[k .. k+16) (zero beyond K).
__device__ __forceinline__ uint4 load_s8x16(const int8_t* x, int K, int k, bool vec) {
  if (vec && k + 16 <= K) return __ldg(reinterpret_cast<const uint4*>(x + k));
  uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (k + j < K) w[j >> 2] |= (uint32_t)(uint8_t)x[k + j] << (8 * (j & 3));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// In place: column sums -> prefix sums over columns (sums[0] = 0), one warp.
__device__ void prefix_columns(int* sums, int cols) {
  const int lane = threadIdx.x & 31;
  int carry = 0;
  for (int base = 1; base <= cols; base += 32) {
    const int i = base + lane;
    int v = i <= cols ? sums[i] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (i <= cols) sums[i] = v + carry;
    carry += __shfl_sync(0xffffffffu, v, 31);
  }
}

__device__ __forceinline__ uint32_t lds_u8w(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ long long fold_fp16_exact(uint16_t h, int S) {
  const int ex = (h >> 10) & 0x1F, man = h & 0x3FF;
  int mm = ex ? man + 1024 : man;
  const int sh = ex ? ex - 1 : 0;
  if (h & 0x8000) mm = -mm;
  return (long long)(mm * S) * (1ll << sh);
}

// XM: activation mode; P: planes; WG: words (16 k) per scale group, 0 = one
// per-tensor scale (BitNet), -1 = balanced ternary d = 3 (base-3 columns of
// 80 k with the group indices inside, group 16, bf16 activations, P = 3).
// MT: tokens per launch (1: one token per problem, several problems; more:
// up to MT tokens of one problem share the weight stream, integer paths).
// With several tokens every 16-weight word is decoded once and feeds MT
// tokens' byte dot-products; its four digit fields are shifted down to bit 0
// so that each (token, plane) keeps a single accumulator.
template <int XM, int P, int WG, int MT>
__global__ void __launch_bounds__(512, 1) gemv2w_kernel(const __grid_constant__ Gemv2wParams pg) {
  extern __shared__ __align__(128) uint8_t smem[];
  // The parameter block is copied to shared memory in two parallel rounds of
  // parameter reads (scalars and problem boundaries, then this CTA's problems):
  // each dependent round of parameter reads costs on the order of a
  // microsecond at launch (every SM misses at once), so nothing below reads
  // the parameter space again. Only the members before `prob` are valid in
  // the shared copy; the problems live in `sprob`.
  constexpr int kHeadBytes = (int)offsetof(Gemv2wParams, prob);
  // copied as 64-bit words: one word per thread covers the head in one round
  static_assert(kHeadBytes % 8 == 0 && sizeof(Gemv2wProblem) % 8 == 0 && kHeadBytes <= 512 * 8,
                "copied as 64-bit words, one round");
  __shared__ __align__(16) unsigned char shead[kHeadBytes];
  __shared__ __align__(16) Gemv2wProblem sprob[kMaxSlotsW];
  {
    const long long* src = reinterpret_cast<const long long*>(&pg);
    long long* dst = reinterpret_cast<long long*>(shead);
    for (int i = threadIdx.x; i < kHeadBytes / 8; i += blockDim.x) dst[i] = src[i];
  }
  __syncthreads();
  const Gemv2wParams& p = *reinterpret_cast<const Gemv2wParams*>(shead);
  constexpr bool kTQ = WG > 0;
  constexpr bool kB3 = WG < 0;
  constexpr bool kBf = XM == kXBf16;
  static_assert(!kB3 || (kBf && P == 3), "balanced ternary: bf16 activations, three digit planes");
  static_assert(MT == 1 || (!kBf && !kB3), "several tokens: integer paths over 2-bit planes");
  constexpr int kColB = kB3 ? kBt3ColBytes : P * kPlaneColBytes;  // bytes per tile column
  const Plan2w sp = plan2w(p, XM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = p.nw, nst = p.nstage, sc = p.stage_cols;

  // ---- this CTA's tiles, and this warp's columns of them (32-bit arithmetic:
  // the planner keeps tiles x CTAs and columns x warps below 2^31). The tiles'
  // problem boundaries are searched in shared memory, and only the problems
  // of this CTA's tiles are copied there (slot s = problem qa + s).
  const int* stb = p.tile_begin;
  const int t0 = gemv2w_cta_tile(stb, p.col_begin, p.nprob, blockIdx.x, gridDim.x);
  const int t1 = gemv2w_cta_tile(stb, p.col_begin, p.nprob, blockIdx.x + 1, gridDim.x);
  auto prob_of = [&](int t) {  // the last problem whose first tile is <= t
    int lo = 0, hi = p.nprob - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (stb[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  const int qa = prob_of(t0), nslots = min(kMaxSlotsW, prob_of(t1 - 1) - qa + 1);  // the host keeps it <= 16
  // activation images: one per problem, or one per token of the single
  // problem, padded to MT with zero images
  const int mt = MT > 1 ? p.mt : 1;
  const int nimg = MT > 1 ? MT : nslots;
  {  // slot s = problem qa + s
    constexpr int kPw = (int)(sizeof(Gemv2wProblem) / 8);
    const long long* src = reinterpret_cast<const long long*>(&pg.prob[qa]);
    long long* dst = reinterpret_cast<long long*>(sprob);
    for (int i = threadIdx.x; i < nslots * kPw; i += blockDim.x) dst[i] = src[i];
  }
  // the CTA's column space: slot s's tiles start at CTA tile stile[s] and CTA
  // column scol[s]; every tile of a problem has that problem's column count
  __shared__ int stile[kMaxSlotsW + 1], scol[kMaxSlotsW + 1];
  if (threadIdx.x == 0) {
    int c = 0;
    for (int s = 0; s < nslots; ++s) {
      const int ta = max(t0, stb[qa + s]), tb = min(t1, stb[qa + s + 1]);
      stile[s] = ta - t0;
      scol[s] = c;
      c += (tb - ta) * sprob[s].cols;
    }
    stile[nslots] = t1 - t0;
    scol[nslots] = c;
  }
  __syncthreads();
  const int gcols = p.gcols;
  const int cg = scol[nslots] / gcols;  // granules in this CTA
  auto bound = [&](int w) { return gcols * (cg * w / nw); };
  // the warp whose range holds column c (never an empty range)
  auto warp_of = [&](int c) {
    const int g = c / gcols;
    return min(nw - 1, ((g + 1) * nw + cg - 1) / cg - 1);
  };
  // slot, CTA tile and column within the tile of CTA column c
  auto locate = [&](int c, int& sl, int& r, int& cc) {
    sl = 0;
    while (sl + 1 < nslots && scol[sl + 1] <= c) ++sl;
    const int ncol = sprob[sl].cols, d = c - scol[sl];
    r = stile[sl] + d / ncol;
    cc = d - (d / ncol) * ncol;
  };
  // first CTA column of CTA tile r of slot sl
  auto tile_col = [&](int sl, int r) { return scol[sl] + (r - stile[sl]) * sprob[sl].cols; };
  const int ca = bound(warp), cb = bound(warp + 1);
  int s_ca, r_ca, c_ca;
  locate(ca, s_ca, r_ca, c_ca);
  const int q_ca = qa + s_ca;  // problem of this warp's first column

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sp.bars) + warp * nst;
  uint8_t* ring = smem + sp.ring + (size_t)warp * nst * sp.stage_bytes;
  int* cnt = reinterpret_cast<int*>(smem + sp.cnt);
  float* mx = reinterpret_cast<float*>(smem + sp.misc);
  auto slot_ptr = [&](int s) { return smem + sp.xs + (size_t)s * sp.slot_bytes; };

  if (lane == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  if (threadIdx.x < nw) cnt[threadIdx.x] = 0;
  unsigned long long* tacc = reinterpret_cast<unsigned long long*>(smem + sp.red);  // several tokens
  if constexpr (MT > 1)
    for (int i = threadIdx.x; i < nw * mt * 32; i += blockDim.x) tacc[i] = 0ull;  // ordered by the staging barriers
  __syncwarp();
  const uint64_t pol = policy_evict_first();

  // ---- producer cursor (lane 0): next column of this warp's range to request
  int pp = ca, rp = r_ca, ccp = c_ca, qp = q_ca, islot = 0, nissued = 0;
  auto issue_next = [&]() {
    if (pp >= cb) return;
    const Gemv2wProblem& pq = sprob[qp - qa];
    const int ncols = min(sc, min(pq.cols - ccp, cb - pp));
    const int T = t0 + rp - stb[qp];
    const int slot = islot;
    islot = islot + 1 == nst ? 0 : islot + 1;
    const uint32_t tb = (uint32_t)ncols * kColB;
    uint8_t* dst = ring + (size_t)slot * sp.stage_bytes;
    uint32_t sb = 0;
    int ga = 0;
    if constexpr (kTQ) {
      ga = ccp * kColK2 / p.group;
      const int gb = min(pq.groups, ((ccp + ncols) * kColK2 + p.group - 1) / p.group);
      sb = (uint32_t)(gb - ga) * P * 64;
    }
    mbar_arrive_expect_tx(&bars[slot], tb + sb);
    bulk_g2s(dst, pq.trit + ((size_t)T * pq.cols + ccp) * kColB, tb, &bars[slot], pol);
    if constexpr (kTQ)
      bulk_g2s(dst + (size_t)sc * P * kPlaneColBytes,
               reinterpret_cast<const uint8_t*>(pq.scale) + ((size_t)T * pq.groups + ga) * P * 64, sb, &bars[slot],
               pol);
    ++nissued;
    pp += ncols;
    ccp += ncols;
    if (ccp == pq.cols) {
      ccp = 0;
      ++rp;
      while (qp + 1 < p.nprob && t0 + rp >= stb[qp + 1]) ++qp;
    }
  };
  pdl_launch_dependents();
  // weights depend on no preceding kernel: with a programmatic dependent
  // launch the first stages are requested before the dependency wait
  if (p.early_w && lane == 0)
    for (int i = 0; i < nst; ++i) issue_next();

  // ---- activations of every problem this CTA touches (after the producer of
  // x). Each warp requests its first weight stages only once its activation
  // loads have returned: behind megabytes of outstanding bulk copies, a small
  // load waits for microseconds.
  pdl_wait();
  // the widest image of this CTA's problems (images of narrower problems are
  // staged to this width with zeros beyond their K)
  int cmax = 0, gmax = 0;
  for (int s = 0; s < nslots; ++s) {
    cmax = max(cmax, sprob[s].cols);
    gmax = max(gmax, sprob[s].groups);
  }
  if constexpr (!kBf) {
    constexpr bool kQ8 = XM == kXBf16Q8;
    constexpr int kCk = kQ8 ? 8 : 16;  // activations per 16-byte chunk
    const int nch = cmax * kColK2 / kCk;  // chunks per image
    const int nflat = nimg * nch;
    const int nthr = blockDim.x;
    auto chunk_load = [&](int f) -> uint4 {
      const int s = f / nch, c = f - s * nch;
      if (MT > 1 && s >= mt) return make_uint4(0u, 0u, 0u, 0u);  // padding token
      const int kq = sprob[MT > 1 ? 0 : s].k;
      const void* xp = MT > 1 ? static_cast<const void*>(static_cast<const int8_t*>(sprob[0].x) +
                                                         (size_t)s * kq * (kQ8 ? 2 : 1))
                              : sprob[s].x;
      if constexpr (kQ8)
        return load_bf16x8(static_cast<const uint16_t*>(xp), kq, c * 8, p.x_vec);
      else
        return load_s8x16(static_cast<const int8_t*>(xp), kq, c * 16, p.x_vec);
    };
    uint4 xr[kXR];
#pragma unroll
    for (int i = 0; i < kXR; ++i) {
      const int f = threadIdx.x + i * nthr;
      xr[i] = f < nflat ? chunk_load(f) : make_uint4(0, 0, 0, 0);
    }
    // the activation loads are on their way: request the first weight stages
    // now, so that the ring fills while the activations are staged
    if (!p.early_w && lane == 0)
      for (int i = 0; i < nst; ++i) issue_next();
    unsigned* amax = reinterpret_cast<unsigned*>(mx);  // token maxima (bits of non-negative floats)
    if (threadIdx.x < nimg) amax[threadIdx.x] = 0u;
    __syncthreads();
    if constexpr (kQ8) {
      // token maxima: per warp and token, then one shared atomic
      auto chunk_max = [&](int f, uint4 v) {
        const int s_lo = __shfl_sync(0xffffffffu, f, 0) / nch;
        const int s_hi = min(nimg - 1, __shfl_sync(0xffffffffu, f, 31) / nch);
        const uint32_t m = f < nflat ? __float_as_uint(bf16_abs_max8(v)) : 0u;
        for (int s = s_lo; s <= s_hi; ++s) {
          const uint32_t ms = __reduce_max_sync(0xffffffffu, (f < nflat && f / nch == s) ? m : 0u);
          if (lane == 0 && ms) atomicMax(&amax[s], ms);
        }
      };
#pragma unroll
      for (int i = 0; i < kXR; ++i) {
        const int f0 = warp * 32 + i * nthr;  // warp-uniform: skip registers no lane of this warp holds
        if (f0 < nflat) chunk_max(threadIdx.x + i * nthr, xr[i]);
      }
      for (int f0 = warp * 32 + kXR * nthr; f0 < nflat; f0 += nthr) {
        const int f = f0 + lane;
        chunk_max(f, f < nflat ? chunk_load(f) : make_uint4(0, 0, 0, 0));
      }
      __syncthreads();
    }
    // int8 image (per-token quantisation with the rule of tern_quantize_act:
    // inv = 127 / a, q = clamp(rint(x * inv), -127, 127))
    auto put = [&](int f, uint4 v) {
      const int s = f / nch, c = f - s * nch;
      uint8_t* sl = slot_ptr(s);
      if constexpr (kQ8) {
        const float a = __uint_as_float(amax[s]);
        const float inv = a > 0.f ? __fdiv_rn(127.0f, a) : 0.f;
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t pk[2] = {0, 0};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t h = (j & 1) ? (w[j >> 1] >> 16) : (w[j >> 1] & 0xFFFFu);
          int q = __float2int_rn(__fmul_rn(__uint_as_float(h << 16), inv));
          q = max(-127, min(127, q));
          pk[j >> 2] |= ((uint32_t)q & 0xFFu) << (8 * (j & 3));
        }
        *reinterpret_cast<uint2*>(sl + 8 * c) = make_uint2(pk[0], pk[1]);
      } else {
        *reinterpret_cast<uint4*>(sl + 16 * c) = v;
      }
    };
#pragma unroll
    for (int i = 0; i < kXR; ++i) {
      const int f = threadIdx.x + i * nthr;
      if (f < nflat) put(f, xr[i]);
    }
    for (int f = threadIdx.x + kXR * nthr; f < nflat; f += nthr) put(f, chunk_load(f));
    if (threadIdx.x < nimg) {
      float sx;
      if constexpr (kQ8) {
        const float a = __uint_as_float(amax[threadIdx.x]);
        sx = a > 0.f ? __fdiv_rn(a, 127.0f) : 0.f;
      } else {
        sx = MT > 1 ? (threadIdx.x < mt ? sprob[0].xscale[threadIdx.x] : 0.f) : sprob[threadIdx.x].xscale[0];
      }
      *reinterpret_cast<float*>(slot_ptr(threadIdx.x) + sp.sx_off) = sx;
    }
    __syncthreads();
    // sums of the image: per column (BitNet, then prefix sums) or per scale group (TQ)
    {
      const int span = kTQ ? p.group : kColK2;  // bytes summed per entry
      const int nent = kTQ ? gmax : cmax;
      for (int e = threadIdx.x; e < nimg * nent; e += nthr) {
        const int s = e / nent, i = e - s * nent;
        uint8_t* sl = slot_ptr(s);
        const uint32_t a0 = smem_u32(sl + (size_t)i * span);
        int sum = 0;
        for (int o = 0; o < span; o += 16) sum += sum16_s8(lds128<0>(a0 + o));
        reinterpret_cast<int*>(sl + sp.sum_off)[kTQ ? i : i + 1] = sum;
      }
      if constexpr (!kTQ)
        if (threadIdx.x < nimg) reinterpret_cast<int*>(slot_ptr(threadIdx.x) + sp.sum_off)[0] = 0;
    }
    __syncthreads();
  } else {
    if (!p.early_w && lane == 0)
      for (int i = 0; i < nst; ++i) issue_next();
    for (int s = 0; s < nslots; ++s) {
      uint8_t* sl = slot_ptr(s);
      if constexpr (kB3) {
        // the codebook from the packed header (the trit stream starts right after it)
        if (threadIdx.x < 27)
          reinterpret_cast<float*>(sl + sp.sx_off)[threadIdx.x] =
              reinterpret_cast<const float*>(sprob[s].trit - kHeaderBytes + kCodebookOffset)[threadIdx.x];
      }
      gemv_common::stage_x_bf16_chains(static_cast<const uint16_t*>(sprob[s].x), sprob[s].k, p.group, 0,
                                       sprob[s].cols * (kB3 ? kColK3 : kColK2),
                                       reinterpret_cast<int8_t*>(sl), sl + sp.kx, sl + 2 * (size_t)sp.kx,
                                       reinterpret_cast<int4*>(sl + sp.sum_off));
    }
    __syncthreads();
  }
  if constexpr (!kTQ && !kB3) {  // single plane: column sums -> prefix sums
    for (int s = warp; s < nimg; s += nw) prefix_columns(reinterpret_cast<int*>(slot_ptr(s) + sp.sum_off), cmax);
    __syncthreads();
  }

  // ---- accumulators of the current tile segment (see tern_gemv2.cu for the
  // four field chains per plane)
  int acc[P][4];
  unsigned accm[P][4], accl[P][4];
  long long acc64 = 0;
  float yacc = 0.f;
  int acct[MT][P];        // several tokens: sum of F x per (token, plane) of the current group
  long long acc64t[MT];   // several tokens: group-folded sums (TQ, units of 2^-24)
  auto reset = [&]() {
#pragma unroll
    for (int q = 0; q < P; ++q)
#pragma unroll
      for (int f = 0; f < 4; ++f) acc[q][f] = 0, accm[q][f] = accl[q][f] = 0;
    acc64 = 0;
    yacc = 0.f;
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      acc64t[t] = 0;
#pragma unroll
      for (int q = 0; q < P; ++q) acct[t][q] = 0;
    }
  };
  auto fold_int = [](const int* c) -> int { return c[0] + (c[1] >> 2) + (c[2] >> 4) + (c[3] >> 6); };
  auto fold_u = [](const unsigned* c) -> int { return (int)(c[0] + (c[1] >> 2) + (c[2] >> 4) + (c[3] >> 6)); };

  // one output row (lane) of tile T of problem pr: the finished sum
  auto finish = [&](const Gemv2wProblem& pr, int T, long long v, float vf, const uint8_t* sl) {
    const int row = T * kTileRows + lane;
    if (row >= pr.n) return;
    float out;
    if constexpr (kBf) {
      out = vf;
    } else {
      const float sx = *reinterpret_cast<const float*>(sl + sp.sx_off);
      if constexpr (kTQ)
        out = __fmul_rn(__fmul_rn(__ll2float_rn(v), 0x1p-24f), sx);
      else
        out = __fmul_rn(__fmul_rn(__int2float_rn((int)v), pr.tensor_scale), sx);
    }
    if (p.out_bf16)
      reinterpret_cast<__nv_bfloat16*>(pr.y)[row] = __float2bfloat16_rn(out);
    else
      reinterpret_cast<float*>(pr.y)[row] = out;
  };

  // several tokens: row (lane) of tile T for token t
  auto finish_t = [&](const Gemv2wProblem& pr, int T, int t, long long v) {
    const int row = T * kTileRows + lane;
    if (row >= pr.n) return;
    const float sx = *reinterpret_cast<const float*>(slot_ptr(t) + sp.sx_off);
    float out;
    if constexpr (kTQ)
      out = __fmul_rn(__fmul_rn(__ll2float_rn(v), 0x1p-24f), sx);
    else
      out = __fmul_rn(__fmul_rn(__int2float_rn((int)v), pr.tensor_scale), sx);
    const size_t o = (size_t)t * pr.n + row;
    if (p.out_bf16)
      reinterpret_cast<__nv_bfloat16*>(pr.y)[o] = __float2bfloat16_rn(out);
    else
      reinterpret_cast<float*>(pr.y)[o] = out;
  };

  // several tokens: end of this warp's segment [lo, hi) of CTA tile r. A tile
  // shared with other warps is summed with shared-memory int64 atomics (exact
  // integers: the order of arrival does not matter) and finished by the last
  // warp to arrive.
  auto segment_done_mt = [&](int r, int lo, int hi) {
    const Gemv2wProblem& pr = sprob[0];
    const int T = t0 + r - stb[0];
    long long v[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if constexpr (kTQ) {
        v[t] = acc64t[t];
      } else {
        const int* pre = reinterpret_cast<const int*>(slot_ptr(t) + sp.sum_off);
        v[t] = (long long)(pre[hi] - pre[lo] - acct[t][0]);
      }
    }
    const int cols = pr.cols;
    if (lo == 0 && hi == cols) {
#pragma unroll
      for (int t = 0; t < MT; ++t)
        if (t < mt) finish_t(pr, T, t, v[t]);
      return;
    }
    const int base = tile_col(0, r);
    const int wlo = warp_of(base), whi = warp_of(base + cols - 1);
    int ncontrib = 0;
    for (int w = wlo; w <= whi; ++w) ncontrib += bound(w + 1) > bound(w);
    unsigned long long* ta = tacc + (size_t)wlo * mt * 32 + lane;
#pragma unroll
    for (int t = 0; t < MT; ++t)
      if (t < mt) atomicAdd(ta + t * 32, (unsigned long long)v[t]);
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&cnt[wlo], 1) == ncontrib - 1;
    }
    if (!__shfl_sync(0xffffffffu, last, 0)) return;
    __threadfence_block();
#pragma unroll
    for (int t = 0; t < MT; ++t)
      if (t < mt) finish_t(pr, T, t, (long long)*reinterpret_cast<volatile unsigned long long*>(ta + t * 32));
  };

  // end of this warp's segment [lo, hi) of CTA tile r (problem q)
  long long* red = reinterpret_cast<long long*>(smem + sp.red);
  auto segment_done = [&](int r, int q, int lo, int hi) {
    const Gemv2wProblem& pr = sprob[q - qa];
    const int T = t0 + r - stb[q];
    const uint8_t* sl = slot_ptr(q - qa);
    long long v = 0;
    float vf = 0.f;
    if constexpr (kBf) {
      vf = yacc;
    } else if constexpr (kTQ) {
      v = acc64;
    } else {
      const int* pre = reinterpret_cast<const int*>(sl + sp.sum_off);
      v = (long long)(pre[hi] - pre[lo] - fold_int(acc[0]));
    }
    const int cols = pr.cols;
    if (lo == 0 && hi == cols) {
      finish(pr, T, v, vf, sl);
      return;
    }
    // a tile shared with other warps: partial row sums in warp order, added by the last to arrive
    const int base = tile_col(q - qa, r);
    const int wlo = warp_of(base), whi = warp_of(base + cols - 1);
    int ncontrib = 0;
    for (int w = wlo; w <= whi; ++w) ncontrib += bound(w + 1) > bound(w);
    const int mine = ca >= base ? 0 : 1;  // 0: the tile holds the start of this warp's range
    red[(warp * 2 + mine) * 32 + lane] = kBf ? (long long)__float_as_uint(vf) : v;
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&cnt[wlo], 1) == ncontrib - 1;
    }
    if (!__shfl_sync(0xffffffffu, last, 0)) return;
    __threadfence_block();
    long long s64 = 0;
    float sf = 0.f;
    for (int w = wlo; w <= whi; ++w) {
      const int bw = bound(w);
      if (bound(w + 1) <= bw) continue;
      const long long e = red[(w * 2 + (bw >= base ? 0 : 1)) * 32 + lane];
      if constexpr (kBf)
        sf += __uint_as_float((uint32_t)e);
      else
        s64 += e;
    }
    finish(pr, T, s64, sf, sl);
  };

  // ---- consumer: this warp's columns, stage by stage
  int pc = ca, rc = r_ca, ccc = c_ca, qc = q_ca, cslot = 0;
  int ccols = sprob[qc - qa].cols;  // columns of the current tile
  int seg_lo = ccc, ifail = -1, nconsumed = 0;
  uint32_t cphase = 0;
  reset();
  const uint32_t ring32 = smem_u32(ring) + lane * 16;
  while (pc < cb) {
    const int ncols = min(sc, min(ccols - ccc, cb - pc));
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
    const uint8_t* sl = slot_ptr(qc - qa);
    const uint32_t x32 = smem_u32(sl);
    const uint32_t st32 = ring32 + (uint32_t)slot * sp.stage_bytes;
    const uint16_t* sst =
        reinterpret_cast<const uint16_t*>(ring + (size_t)slot * sp.stage_bytes + (size_t)sc * P * kPlaneColBytes);
    const int ga_stage = kTQ ? ccc * kColK2 / p.group : 0;
    const int* gsum = reinterpret_cast<const int*>(sl + sp.sum_off);
    const int4* grec = reinterpret_cast<const int4*>(sl + sp.sum_off);  // bf16: per-group chain sums
    const float* cbk = reinterpret_cast<const float*>(sl + sp.sx_off);   // d = 3: codebook
    // one 16-k word (index WI of the column) of every plane
    // xw: the column's four activation words (integer paths, loaded ahead)
    auto word_step = [&](auto wi_c, const uint4* wv, const uint4* xw, int cc) {
      constexpr int wi = decltype(wi_c)::value;
      if constexpr (MT > 1) {
        // the word's digit fields, each at bit 0 of its byte, shared by the tokens
        uint32_t dg[P][4];
#pragma unroll
        for (int q = 0; q < P; ++q) {
          const uint32_t F = lop3_ternary_digit(u4_get<wi>(wv[q]));
          dg[q][0] = F & 0x03030303u;
          dg[q][1] = (F >> 2) & 0x03030303u;
          dg[q][2] = (F >> 4) & 0x03030303u;
          dg[q][3] = (F >> 6) & 0x03030303u;
        }
        const uint32_t xo = (uint32_t)(cc * kColK2 + wi * 16);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          const int4 xv = u4_as_i4(lds128<0>(x32 + (uint32_t)t * (uint32_t)sp.slot_bytes + xo));
#pragma unroll
          for (int q = 0; q < P; ++q) {
            int a = acct[t][q];
            a = dp4a_ss((int)dg[q][0], xv.x, a);
            a = dp4a_ss((int)dg[q][1], xv.y, a);
            a = dp4a_ss((int)dg[q][2], xv.z, a);
            a = dp4a_ss((int)dg[q][3], xv.w, a);
            acct[t][q] = a;
          }
        }
        if constexpr (kTQ) {
          // group fold: sum t x = sum x - sum F x, times the scale's integer
          // mantissa (exact in 32 bits), shifted to units of 2^-24
          const int wt = cc * 4 + wi;
          if ((wt + 1) % WG == 0) {
            const int gl = wt / WG;
            const int gst = gl - ga_stage;
            int gsx[MT];  // each token's sum of x over the group
#pragma unroll
            for (int t = 0; t < MT; ++t) gsx[t] = reinterpret_cast<const int*>(slot_ptr(t) + sp.sum_off)[gl];
#pragma unroll
            for (int q = 0; q < P; ++q) {
              const uint32_t h = sst[(gst * P + q) * kTileRows + lane];
              const int ex = (int)((h >> 10) & 0x1Fu), man = (int)(h & 0x3FFu);
              int mm = ex ? man + 1024 : man;
              if (h & 0x8000u) mm = -mm;
              const int sh = ex ? ex - 1 : 0;
#pragma unroll
              for (int t = 0; t < MT; ++t) {
                // the integer product (exact in 32 bits) shifted to units of 2^-24
                acc64t[t] += (long long)((unsigned long long)(long long)(mm * (gsx[t] - acct[t][q])) << sh);
                acct[t][q] = 0;
              }
            }
          }
        }
        return;
      }
      uint32_t F[P];
#pragma unroll
      for (int q = 0; q < P; ++q) F[q] = lop3_ternary_digit(u4_get<wi>(wv[q]));
      if constexpr (!kBf) {
        const int4 xv = u4_as_i4(xw[wi]);
#pragma unroll
        for (int q = 0; q < P; ++q) {
          acc[q][0] = dp4a_ss((int)(F[q] & 0x03030303u), xv.x, acc[q][0]);
          acc[q][1] = dp4a_ss((int)(F[q] & 0x0C0C0C0Cu), xv.y, acc[q][1]);
          acc[q][2] = dp4a_ss((int)(F[q] & 0x30303030u), xv.z, acc[q][2]);
          acc[q][3] = dp4a_us(F[q] & 0xC0C0C0C0u, xv.w, acc[q][3]);
        }
      } else {
        const uint32_t xo = (uint32_t)(cc * kColK2);
        const int4 hv = u4_as_i4(lds128<wi * 16>(x32 + xo));
        const uint4 mv = lds128<wi * 16>(x32 + (uint32_t)sp.kx + xo);
        const uint4 lv = lds128<wi * 16>(x32 + 2u * (uint32_t)sp.kx + xo);
#pragma unroll
        for (int q = 0; q < P; ++q) {
          const uint32_t d0 = F[q] & 0x03030303u, d1 = F[q] & 0x0C0C0C0Cu, d2 = F[q] & 0x30303030u,
                         d3 = F[q] & 0xC0C0C0C0u;
          acc[q][0] = dp4a_ss((int)d0, hv.x, acc[q][0]);
          acc[q][1] = dp4a_ss((int)d1, hv.y, acc[q][1]);
          acc[q][2] = dp4a_ss((int)d2, hv.z, acc[q][2]);
          acc[q][3] = dp4a_us(d3, hv.w, acc[q][3]);
          accm[q][0] = dp4a_uu(d0, mv.x, accm[q][0]);
          accm[q][1] = dp4a_uu(d1, mv.y, accm[q][1]);
          accm[q][2] = dp4a_uu(d2, mv.z, accm[q][2]);
          accm[q][3] = dp4a_uu(d3, mv.w, accm[q][3]);
          accl[q][0] = dp4a_uu(d0, lv.x, accl[q][0]);
          accl[q][1] = dp4a_uu(d1, lv.y, accl[q][1]);
          accl[q][2] = dp4a_uu(d2, lv.z, accl[q][2]);
          accl[q][3] = dp4a_uu(d3, lv.w, accl[q][3]);
        }
      }
      // ---- group fold (TQ): after the last word of each group
      if constexpr (kTQ) {
        const int wt = cc * 4 + wi;  // word index within the row
        if ((wt + 1) % WG == 0) {
          const int gl = wt / WG;
          const int gst = gl - ga_stage;
#pragma unroll
          for (int q = 0; q < P; ++q) {
            const uint16_t h = sst[(gst * P + q) * kTileRows + lane];
            if constexpr (!kBf) {
              acc64 += fold_fp16_exact(h, gsum[gl] - fold_int(acc[q]));
            } else {
              // sum t q = sum q - sum F q, chain by chain (small integers)
              const int4 r = grec[gl];
              const float S = gemv_common::chains_to_float(r.x - fold_int(acc[q]), r.y - fold_u(accm[q]),
                                                           r.z - fold_u(accl[q]));
              yacc = fmaf(__half2float(__ushort_as_half(h)) * __int_as_float(r.w), S, yacc);
            }
#pragma unroll
            for (int f = 0; f < 4; ++f) acc[q][f] = accm[q][f] = accl[q][f] = 0;
          }
        }
      }
    };
    auto load_w = [&](int j, uint4* wv) {
      const uint32_t wc = st32 + (uint32_t)(j * kColB);
      wv[0] = lds128<0>(wc);
      if constexpr (P > 1) wv[1] = lds128<kPlaneColBytes>(wc);
      if constexpr (P > 2) wv[2] = lds128<2 * kPlaneColBytes>(wc);
      if constexpr (P > 3) wv[3] = lds128<3 * kPlaneColBytes>(wc);
    };
    auto load_x = [&](int j, uint4* xw) {
      if constexpr (!kBf && MT == 1) {
        const uint32_t xc = x32 + (uint32_t)((ccc + j) * kColK2);
        xw[0] = lds128<0>(xc);
        xw[1] = lds128<16>(xc);
        xw[2] = lds128<32>(xc);
        xw[3] = lds128<48>(xc);
      }
    };
    // balanced ternary d = 3: one 80-k column of this lane's row (16 byte
    // triples in wv[0..2], the five group indices in three bytes after the
    // digit chunks), five groups of 16 folded with their codebook scales
    auto column3 = [&](const uint4* wv, int cc) {
      const uint32_t cbase = st32 - (uint32_t)(lane * 16) + (uint32_t)((cc - ccc) * kColB);
      // the five groups' codebook indices: one more triple, same order as the trits
      uint32_t ix[5];
      gemv_common::triple_levels(lds_u8w(cbase + 3 * kPlaneColBytes + lane),
                                 lds_u8w(cbase + 3 * kPlaneColBytes + 32 + lane),
                                 lds_u8w(cbase + 3 * kPlaneColBytes + 64 + lane), ix);
      uint32_t U[4][5];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t w0 = w == 0 ? wv[0].x : w == 1 ? wv[0].y : w == 2 ? wv[0].z : wv[0].w;
        const uint32_t w1 = w == 0 ? wv[1].x : w == 1 ? wv[1].y : w == 2 ? wv[1].z : wv[1].w;
        const uint32_t w2 = w == 0 ? wv[2].x : w == 1 ? wv[2].y : w == 2 ? wv[2].z : wv[2].w;
        uint32_t ue[5], uo[5];
        gemv_common::triple_levels(w0 & 0x00FF00FFu, w1 & 0x00FF00FFu, w2 & 0x00FF00FFu, ue);
        gemv_common::triple_levels((w0 >> 8) & 0x00FF00FFu, (w1 >> 8) & 0x00FF00FFu, (w2 >> 8) & 0x00FF00FFu, uo);
#pragma unroll
        for (int j = 0; j < 5; ++j) U[w][j] = ue[j] | (uo[j] << 8);
      }
#pragma unroll
      for (int j = 0; j < 5; ++j) {
        const uint32_t xo = (uint32_t)(cc * kColK3 + 16 * j);
        const uint4 hv = lds128<0>(x32 + xo), mv = lds128<0>(x32 + (uint32_t)sp.kx + xo),
                    lv = lds128<0>(x32 + 2u * (uint32_t)sp.kx + xo);
        int H = 0;
        unsigned M = 0, L = 0;
        H = dp4a_us(U[0][j], (int)hv.x, H);
        H = dp4a_us(U[1][j], (int)hv.y, H);
        H = dp4a_us(U[2][j], (int)hv.z, H);
        H = dp4a_us(U[3][j], (int)hv.w, H);
        M = dp4a_uu(U[0][j], mv.x, M);
        M = dp4a_uu(U[1][j], mv.y, M);
        M = dp4a_uu(U[2][j], mv.z, M);
        M = dp4a_uu(U[3][j], mv.w, M);
        L = dp4a_uu(U[0][j], lv.x, L);
        L = dp4a_uu(U[1][j], lv.y, L);
        L = dp4a_uu(U[2][j], lv.z, L);
        L = dp4a_uu(U[3][j], lv.w, L);
        const int g = cc * kBt3Groups + j;
        // sum (U - 13) q chain by chain: |H'| < 2^15, |256 M' + L'| < 2^24, so
        // the sum is rounded once, as an exact int64 conversion would be
        const int4 r = grec[g];
        const float S = gemv_common::chains_to_float(H - 13 * r.x, (int)M - 13 * r.y, (int)L - 13 * r.z);
        yacc = fmaf(cbk[ix[j]] * __int_as_float(r.w), S, yacc);
      }
    };
    auto column = [&](const uint4* wv, const uint4* xw, int cc) {
      if constexpr (kB3) {
        column3(wv, cc);
      } else {
        word_step(std::integral_constant<int, 0>{}, wv, xw, cc);
        word_step(std::integral_constant<int, 1>{}, wv, xw, cc);
        word_step(std::integral_constant<int, 2>{}, wv, xw, cc);
        word_step(std::integral_constant<int, 3>{}, wv, xw, cc);
      }
    };
    // two columns per trip, each one's shared loads issued a column ahead
    // (the load after the last column re-reads it and is not used)
    uint4 wa[P], wb[P], xa[4], xb[4];
    load_w(0, wa);
    load_x(0, xa);
#pragma unroll 1
    for (int j = 0; j < ncols; j += 2) {
      const int j1 = min(j + 1, ncols - 1), j2 = min(j + 2, ncols - 1);
      load_w(j1, wb);
      load_x(j1, xb);
      column(wa, xa, ccc + j);
      if (j + 1 < ncols) {
        load_w(j2, wa);
        load_x(j2, xa);
        column(wb, xb, ccc + j + 1);
      }
    }
    // release the slot: reads of this stage are complete before the refill
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) issue_next();
    ++nconsumed;
    pc += ncols;
    ccc += ncols;
    if (ccc == ccols || pc == cb) {
      if constexpr (MT > 1)
        segment_done_mt(rc, seg_lo, ccc);
      else
        segment_done(rc, qc, seg_lo, ccc);
      reset();
      seg_lo = 0;
    }
    if (ccc == ccols) {
      ccc = 0;
      ++rc;
      while (qc + 1 < p.nprob && t0 + rc >= stb[qc + 1]) ++qc;
      ccols = sprob[qc - qa].cols;
    }
  }
  if (ifail >= 0) {
    // a wait expired: give the copies still in flight a bounded chance to land
    for (int j = ifail; j < min(nissued, ifail + nst); ++j) mbar_wait_bounded(&bars[j % nst], (uint32_t)(j / nst) & 1u);
  }
}

// ------------------------------------------------------------------ launch
template <int XM, int P, int WG, int MT>
static int launch_w(const Gemv2wParams& p0, bool pdl, void* stream) {
  Gemv2wParams p = p0;
  p.early_w = pdl ? 1 : 0;
  const Plan2w sp = plan2w(p, XM);
  auto kern = gemv2w_kernel<XM, P, WG, MT>;
  // at least half of an SM's shared memory, so that CTAs never share an SM
  const size_t smem = sp.total > 120 * 1024 ? sp.total : 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid, 1, 1);
  cfg.blockDim = dim3(32 * p.nw, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return (int)cudaLaunchKernelEx(&cfg, kern, p);
}


}  // namespace
}  // namespace tern
