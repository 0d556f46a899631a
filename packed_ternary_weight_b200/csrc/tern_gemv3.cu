// Decode GEMV over balanced ternary of depth 3 (Entrit Llama-3.1-8B-trit-uniform-d3
// card, "Quantization details": 27 levels per weight, group 16, 27-entry
// log-spaced scale codebook; weight = cb[idx] * (9 t2 + 3 t1 + t0)), bf16
// activations.
//
// Layout of one 80-k column of a 32-row tile (the packer's): per row, 16 byte
// triples; triple i holds the digits u = t + 1 of the five weights
// k = 80c + 16j + i (j = 0..4), weight by weight (u0, u1, u2 of weight j are
// base-3 digits 3j .. 3j+2 of the triple, five digits per byte, first digit
// least significant), byte b of every triple in the b-th 16-byte chunk of the
// row; then one more triple per row holding the five groups' codebook indices
// in the same order. Weight j of the 16 triples of a row is group 5c + j.
//
// Work split, weight stream, K-splits and persistence follow the 2-bit kernel:
// one warp per 32-row tile and K-split, per-warp rings of shared-memory stages
// filled by 1-D bulk async copies on mbarriers, splits reduced in a
// thread-block cluster, persistent CTAs when K is not split.
//
// Decode (per lane = one row, per 4 triples): the 12 bytes are spread into
// 16-bit lanes (two triples per 32-bit register) and the five levels
// U = u0 + 3 u1 + 9 u2 = level + 13 in 0..26 read with exact multiply-shift
// divisions, both lanes at once (byte 0 = U0 + 27 h1; byte 1 = l1 + 3 U2 +
// 81 h3; byte 2 = l3 + 9 U4; U1 = h1 + 9 l1, U3 = h3 + 3 l3), about 0.8
// integer operations per trit. The levels, four per register in byte lanes,
// are dotted with the 24-bit fixed-point image of the activations (same as
// the 2-bit bf16 path) with byte dot-products, so the group sum is
// sum U q - 13 sum q, exact in integers; each group is then scaled once,
// cb[idx] * 2^(E-22), and accumulated in fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "tern_bt_levels.h"
#include "tern_gemv_common.cuh"
#include "tern_ptx.cuh"

namespace tern {

int read_clear_dev_error_gemv3(void* stream, unsigned* out) { return read_clear_dev_error_tu(stream, out); }

namespace {

using gemv_common::align_up;
using gemv_common::triple_levels;

struct Smem3 {
  size_t bars, cbar, ring, xa, xb, xc, gsum, gmult, cb, red, total;
  int stage_bytes;
};

__host__ __device__ inline Smem3 smem3_plan(const Gemv2Params& p) {
  Smem3 s{};
  const int kr = p.cols_per_split * kColK3;
  const int gr = kr / 16;
  const size_t mt = (size_t)gemv3_mt(p.m);  // activation images: one per token, padded to 1, 2, 4 or 8
  s.stage_bytes = (int)align_up((size_t)p.stage_cols * bt_col_bytes(p.planes), 128);
  size_t off = 0;
  s.bars = off;
  off += (size_t)p.wpc * p.nstage * 8;
  s.cbar = off;  // K split over a cluster: the splits' partial sums arrived (rank 0)
  off = align_up(off + 8, 128);
  s.ring = off;
  off += (size_t)p.wpc * p.nstage * s.stage_bytes;
  s.xa = off;  // [mt][kr] each
  off = align_up(off + mt * kr, 128);
  s.xb = off;
  off = align_up(off + mt * kr, 128);
  s.xc = off;
  off = align_up(off + mt * kr, 128);
  s.gsum = off;  // [mt][gr]
  off = align_up(off + mt * gr * 8, 16);
  s.gmult = off;
  off = align_up(off + mt * gr * 4, 16);
  s.cb = off;
  off = align_up(off + 27 * 4, 16);
  s.red = off;
  off = align_up(off + ((p.cluster && p.ks > 1) ? (size_t)p.ks * mt * p.wpc * 32 * 4 : 0), 16);
  s.total = off;
  return s;
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

}  // namespace

// D: the depth (2, 3 or 4); the tuple of a row holds D bytes, the level bias is (3^D - 1) / 2.
// MT: tokens per launch (1, 2, 4 or 8; p.m of them are real): each column's
// levels are decoded once and dotted with every token's activation image.
template <int D, int MT>
__global__ void __launch_bounds__(256) gemv3_kernel(const __grid_constant__ Gemv2Params p) {
  static_assert(D >= 2 && D <= 4, "depth 2..4");
  constexpr int kColB = bt_col_bytes(D);
  constexpr long long kBias = D == 2 ? 4 : (D == 3 ? 13 : 40);
  extern __shared__ __align__(128) uint8_t smem[];
  const Smem3 sp = smem3_plan(p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.y;
  const bool clus = p.cluster && p.ks > 1;
  const int c0 = split * p.cols_per_split;
  const int c1 = min(p.cols, c0 + p.cols_per_split);
  const int ncols = c1 - c0;
  const int sc = p.stage_cols, nst = p.nstage;
  const int spt = (ncols + sc - 1) / sc;
  const int k0 = c0 * kColK3, kr = ncols * kColK3;
  const int kr_img = p.cols_per_split * kColK3;  // per-token stride of the images
  const int gr_img = kr_img / 16;
  const int m = MT == 1 ? 1 : p.m;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sp.bars) + warp * nst;
  uint8_t* ring = smem + sp.ring + (size_t)warp * nst * sp.stage_bytes;

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

  // ---- prologue: barriers, first weight stages
  if (clus && threadIdx.x == 0) {
    mbar_init(reinterpret_cast<uint64_t*>(smem + sp.cbar), 1);
    fence_mbar_init();
  }
  // other CTAs store into this one's shared memory only after every CTA of the
  // cluster runs and has initialised its barrier
  if (clus) cluster_arrive_relaxed();
  if (lane == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = policy_evict_first();
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
    const uint32_t tb = (uint32_t)(ce - cs) * kColB;
    mbar_arrive_expect_tx(&bars[slot], tb);
    bulk_g2s(ring + (size_t)slot * sp.stage_bytes, pq.trit + ((size_t)T * p.cols + cs) * kColB, tb,
             &bars[slot], pol);
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
  pdl_wait();
  if (clus) cluster_wait_acquire();

  const long long* gsum = reinterpret_cast<const long long*>(smem + sp.gsum);
  const float* gmul = reinterpret_cast<const float*>(smem + sp.gmult);
  const uint32_t x32 = smem_u32(smem + sp.xa), xm32 = smem_u32(smem + sp.xb), xl32 = smem_u32(smem + sp.xc);
  const uint32_t cb32 = smem_u32(smem + sp.cb);
  const uint32_t ring32 = smem_u32(ring);

  int cur_prob = -1, nconsumed = 0, ifail = -1, pi = prob_of(gbeg);
  int cslot = 0;
  uint32_t cphase = 0;
  float yacc[MT];
  for (int gi = gbeg; gi < gend; ++gi) {
    while (pi + 1 < p.nprob && gi >= p.prob[pi + 1].cta_begin) ++pi;
    const Gemv2Problem& pr = p.prob[pi];
    if (pi != cur_prob) {
      __syncthreads();
      // codebook from the packed header (trit stream starts 256 bytes after the
      // header; the codebook sits at header byte 128)
      if (threadIdx.x < 27)
        reinterpret_cast<float*>(smem + sp.cb)[threadIdx.x] =
            reinterpret_cast<const float*>(pr.trit - kHeaderBytes + kCodebookOffset)[threadIdx.x];
      for (int t = 0; t < m; ++t)
        gemv_common::stage_x_bf16_image(static_cast<const uint16_t*>(pr.x) + (size_t)t * p.k, p.k, 16, k0, kr,
                                        reinterpret_cast<int8_t*>(smem + sp.xa) + (size_t)t * kr_img,
                                        smem + sp.xb + (size_t)t * kr_img, smem + sp.xc + (size_t)t * kr_img,
                                        reinterpret_cast<long long*>(smem + sp.gsum) + (size_t)t * gr_img,
                                        reinterpret_cast<float*>(smem + sp.gmult) + (size_t)t * gr_img);
      __syncthreads();
      cur_prob = pi;
    }
    const int T = tile_of(gi, pi);
    const bool active = T < pr.row_tiles;
#pragma unroll
    for (int t = 0; t < MT; ++t) yacc[t] = 0.f;
    if (active && ifail < 0) {
      for (int s = 0; s < spt; ++s, ++nconsumed) {
        const int slot = cslot;
        const uint32_t phase = cphase;
        if (++cslot == nst) {
          cslot = 0;
          cphase ^= 1u;
        }
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars[slot], phase))) {
          ifail = nconsumed;
          break;
        }
        const uint32_t st32 = ring32 + (uint32_t)slot * sp.stage_bytes;
        const int cs = c0 + s * sc;
        const int ncs = min(sc, c1 - cs);
        for (int cc = 0; cc < ncs; ++cc) {
          const uint32_t col = st32 + (uint32_t)(cc * kColB);
          const uint32_t kx = (uint32_t)((cs + cc - c0) * kColK3);
          // scale indices of the column's five groups: one more triple, same
          // order as the trits
          uint32_t ix[5];
          triple_levels(lds_u8(col + D * kPlaneColBytes + lane), lds_u8(col + D * kPlaneColBytes + 32 + lane),
                        lds_u8(col + D * kPlaneColBytes + 64 + lane), ix);
          // U = u0 + 3 u1 + 9 u2 in byte lanes, for the 4 words x 5 digit positions
          uint32_t U[4][5];
          const uint4 b0 = lds128<0>(col + lane * 16);
          const uint4 b1 = lds128<kPlaneColBytes>(col + lane * 16);
          uint4 b2 = make_uint4(0u, 0u, 0u, 0u), b3 = make_uint4(0u, 0u, 0u, 0u);
          if constexpr (D >= 3) b2 = lds128<2 * kPlaneColBytes>(col + lane * 16);
          if constexpr (D >= 4) b3 = lds128<3 * kPlaneColBytes>(col + lane * 16);
          // tuples 4w, 4w+2 in the 16-bit lanes of the even bytes, 4w+1, 4w+3 of the odd ones
          auto levels = [&](uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, uint32_t (&u)[5]) {
            if constexpr (D == 2)
              pair_levels(w0, w1, u);
            else if constexpr (D == 3)
              triple_levels(w0, w1, w2, u);
            else
              quad_levels(w0, w1, w2, w3, u);
          };
          auto word_u = [&](auto wi_c, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
            constexpr int w = decltype(wi_c)::value;
            constexpr uint32_t kE = 0x00FF00FFu;
            uint32_t ue[5], uo[5];
            levels(w0 & kE, w1 & kE, w2 & kE, w3 & kE, ue);
            levels((w0 >> 8) & kE, (w1 >> 8) & kE, (w2 >> 8) & kE, (w3 >> 8) & kE, uo);
#pragma unroll
            for (int j = 0; j < 5; ++j) U[w][j] = ue[j] | (uo[j] << 8);
          };
          word_u(std::integral_constant<int, 0>{}, b0.x, b1.x, b2.x, b3.x);
          word_u(std::integral_constant<int, 1>{}, b0.y, b1.y, b2.y, b3.y);
          word_u(std::integral_constant<int, 2>{}, b0.z, b1.z, b2.z, b3.z);
          word_u(std::integral_constant<int, 3>{}, b0.w, b1.w, b2.w, b3.w);
#pragma unroll
          for (int j = 0; j < 5; ++j) {
            const int g = (int)(kx >> 4) + j;  // group within the split
            const float cbv = lds_f32(cb32 + 4u * ix[j]);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              if (MT > 1 && t >= m) break;
              const uint32_t xo = kx + 16u * j + (uint32_t)(t * kr_img);
              const uint4 hv = lds128<0>(x32 + xo), mv = lds128<0>(xm32 + xo), lv = lds128<0>(xl32 + xo);
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
              const int gt = g + t * gr_img;
              const long long S = ((long long)H * 65536 + (long long)M * 256 + L) - kBias * gsum[gt];
              yacc[t] = fmaf(cbv * gmul[gt], __ll2float_rn(S), yacc[t]);
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) issue_next();
      }
    }

    const int row = T * kTileRows + lane;
    auto write_out = [&](int t, float v) {
      if (row >= pr.n) return;
      const size_t o = (size_t)t * pr.n + row;
      if (p.out_bf16)
        reinterpret_cast<__nv_bfloat16*>(pr.y)[o] = __float2bfloat16_rn(v);
      else
        reinterpret_cast<float*>(pr.y)[o] = v;
    };
    if (p.ks == 1) {
      if (active)
#pragma unroll
        for (int t = 0; t < MT; ++t)
          if (t < m) write_out(t, yacc[t]);
      continue;
    }
    if (active && ifail >= 0) {
      for (int j = ifail; j < min(nissued, ifail + nst); ++j)
        mbar_wait_bounded(&bars[j % nst], (uint32_t)(j / nst) & 1u);  // error path only
    }
    // K is split: the splits of this row group form the cluster. Each sends
    // its partial sums to CTA rank 0 with st.async; rank 0 waits for them on
    // its own barrier and sums them in split order, the others are done.
    const int rows_cta = p.wpc * kTileRows;
    uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + sp.cbar);
    if (split == 0 && threadIdx.x == 0) {
      // every split's partials of the active warps (the same warps in every split)
      const int nact = max(0, min(p.wpc, pr.row_tiles - (T - warp)));
      mbar_arrive_expect_tx(rbar, (uint32_t)(p.ks * m * nact * kTileRows * 4));
    }
    if (active) {
      const uint32_t rbar0 = map_cluster_rank(smem_u32(rbar), 0);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t >= m) break;
        const size_t idx = ((size_t)split * MT + t) * rows_cta + warp * kTileRows + lane;
        st_async_u32(map_cluster_rank(smem_u32(smem + sp.red + idx * 4), 0), __float_as_uint(yacc[t]), rbar0);
      }
    }
    if (split == 0) (void)mbar_wait_bounded<true>(rbar, 0);  // on expiry the error word records a timeout
    if (split == 0 && active) {
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t >= m) break;
        float sf = 0.f;
        for (int s = 0; s < p.ks; ++s)
          sf += reinterpret_cast<const float*>(smem + sp.red)[((size_t)s * MT + t) * rows_cta + warp * kTileRows + lane];
        write_out(t, sf);
      }
    }
    return;
  }
  if (ifail >= 0) {
    for (int j = ifail; j < min(nissued, ifail + nst); ++j) mbar_wait_bounded(&bars[j % nst], (uint32_t)(j / nst) & 1u);
  }
}

size_t gemv3_smem_bytes(const Gemv2Params& p) { return smem3_plan(p).total; }

int launch_gemv3(const Gemv2Params& p, bool pdl, void* stream) {
  if (p.m < 1 || p.m > 8 || (p.ks > 1 && !p.cluster) || p.planes < 2 || p.planes > 4) return -1;
  const Smem3 sp = smem3_plan(p);
  auto pick = [](int d, auto mt_c) {
    constexpr int T = decltype(mt_c)::value;
    return d == 2 ? gemv3_kernel<2, T> : (d == 3 ? gemv3_kernel<3, T> : gemv3_kernel<4, T>);
  };
  const int mt = gemv3_mt(p.m);
  auto kern = mt == 1   ? pick(p.planes, std::integral_constant<int, 1>{})
              : mt == 2 ? pick(p.planes, std::integral_constant<int, 2>{})
              : mt == 4 ? pick(p.planes, std::integral_constant<int, 4>{})
                        : pick(p.planes, std::integral_constant<int, 8>{});
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
  if (e != cudaSuccess) return (int)e;
  const bool clus = p.cluster && p.ks > 1;
  if (clus && p.ks > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return (int)e;
  }
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
  return (int)cudaLaunchKernelEx(&cfg, kern, q);
}

}  // namespace tern
