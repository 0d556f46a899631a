// Batched (prefill) packed ternary GEMM on the 5th-generation tensor cores:
// Y[m][n] = sum_p sum_groups s[p][n][grp] * sum_{k in grp} t[p][n][k] * xq[m][k]
// for int8 tokens (padded to a multiple of 16), bit-identical to the exact integer rule of the
// int8 path (every fp16 scale is an integer multiple of 2^-24, so the sum is an
// exact integer count of 2^-24, rounded once to fp32, then times the token's
// activation scale). Formats: sasori-style additive TQ{K}P planes with fp16
// group scales (sasori README, "How it works", "K and g"), and the BitNet
// b1.58 single plane with one per-tensor scale (QORA-LLM-2B, "Ternary GEMV").
//
// Group scales without per-group promotion. An int8 MMA of K = 32 produces
// one integer per row and token; applying a different fp16 scale to every 32
// columns would cost several CUDA-core instructions per accumulator element
// and K step. Instead the scale goes into the A operand: u = |s| / 2^-24 is an
// integer below 2^40, written in D' base-2^b digits u_d with b = 7 for one
// plane, 6 for two, 5 for three or four (D' = ceil(7 D / b), D the packed
// header's count of 7-bit digits of the largest scale). The A tile of digit d
// holds sum_p sign(s_p) * t_p * u_{p,d}: at most P (2^b - 1) <= 127 in
// magnitude, so the planes merge into one int8 operand. One tensor-memory
// int32 accumulator per digit then sums every group and plane of the K range,
// and the exact result is sum_d 2^(b d) * acc_d, formed in int64 once per
// output (|acc_d| <= 127 * 127 * K < 2^31 for the shapes the host admits).
// The tensor cores do D' times the algorithmic MACs of one plane; the CUDA
// cores only decode.
//
// Decode. A 2-bit code selects one of three bytes {beta, beta + a, beta - a}
// of a per-(plane, digit) lookup word by byte permutation (PRMT), four weights
// per instruction; the planes' bias bytes beta add up to 128, so the planes'
// words add without carries between bytes and one XOR with 0x80 per byte
// leaves the signed sum (one plane: beta = 0, no XOR). The selector nibbles
// come from masking the packed word, which yields the 16 weights of a word in
// the order 0,8,1,9,...,7,15; the activations are staged in the same order
// (tc_prep_x), so every dot product sees matching pairs.
//
// Pipeline (one CTA per SM, persistent). Work = (128-row tile, token pass) x
// 64-k columns; CTA c takes the contiguous range [W c / G, W (c+1) / G).
//   warp 0     bulk async copies into a ring of stages (mbarrier transaction
//              counts); a stage holds up to C consecutive columns of the four
//              row tiles' trits, their scale blocks and the activations, and
//              is fetched by ONE copy instruction with a lane per stream
//              (a bulk copy holds its warp for some hundreds of cycles
//              whatever its size, so fewer and larger copies);
//   warps 1-2  one thread each issues tcgen05.mma for half of the digit
//              accumulators and commits completion to mbarriers (two issuing
//              warps keep the tensor cores busier than one at small N);
//              warp 1 also owns the tensor-memory allocation;
//   warps 3-18 decode A tiles (the D' digit tiles of one column form a group
//              of the shared ring; one warp per 32 rows and 16-k chunk), then
//              drain the accumulators: a tile whose whole K range
//              lies in this CTA is written directly; a tile cut between CTAs is
//              summed exactly in an int64 workspace with atomic adds and
//              finished by the last CTA to arrive (integer sums, so the order
//              does not matter).
// Every wait is bounded (about 1 s); on expiry the device error word records a
// timeout and the CTA runs to completion without waiting further.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "tern_tc.cuh"

namespace tern {

int read_clear_dev_error_gemm_tc(void* stream, unsigned* out) { return read_clear_dev_error_tu(stream, out); }

namespace {

constexpr int kDecWarps = 16;
constexpr int kMmaWarps = 2;
constexpr int kDec0 = 1 + kMmaWarps;  // first decoder warp
constexpr int kThreads = 32 * (kDec0 + kDecWarps);
constexpr int kSlotBytes = kTcSlotBytes;  // one A tile: 128 rows x 64 k
constexpr int kTmemCols = 512;

using tc::kMiscAbort;
using tc::kMiscLast;
using tc::kMiscTmem;
using tc::bulk_g2s_plain;
using tc::mbar_arrive;
using tc::mbar_test;
using tc::tc_wait;
using tc::tc_wait_many;

__device__ __forceinline__ void named_sync_decoders() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kDecWarps) : "memory"); }

using tc::lds16;
using tc::lds32;
using tc::sts128;

// Digit width and per-plane bias of the merged A operand for P planes.
template <int P>
constexpr int kDigitBits = P == 1 ? 7 : (P == 2 ? 6 : 5);
template <int P>
__device__ __forceinline__ uint32_t plane_bias(int pl) {
  if constexpr (P == 1) return 0u;
  if constexpr (P == 2) return 64u;
  if constexpr (P == 3) return pl == 2 ? 42u : 43u;
  return 32u;
}

// u = |s| / 2^-24 of an fp16 scale (below 2^40) and the byte permutation that
// applies its sign (a negative scale swaps the +t and -t bytes).
__device__ __forceinline__ uint64_t scale_units(uint32_t h, uint32_t& sel) {
  const uint32_t ex = (h >> 10) & 31u, man = h & 1023u;
  sel = (h & 0x8000u) ? 0x3120u : 0x3210u;
  return ex ? (uint64_t)(1024u | man) << (ex - 1u) : (uint64_t)man;
}

// Lookup word of one plane and digit: byte 0 = beta (code 00, t = 0), byte 1 =
// beta + a (code 01, t = +1), byte 2 = beta - a (code 10, t = -1), a = sign(s)
// * ud; byte 3 is never selected (code 11 does not occur). ud * 0x00FF0100
// puts ud in byte 1 and -ud mod 256 in byte 2 (its borrow lands in byte 3).
__device__ __forceinline__ uint32_t digit_lut(uint32_t ud, uint32_t beta, uint32_t sel) {
  return __byte_perm(ud * 0x00FF0100u + beta * 0x00010101u, 0u, sel);
}

// y = fl32(fl32(acc * 2^-24) * s_x) for the group-scaled sum (acc counts 2^-24,
// converted to fp32 with one rounding), y = fl32(fl32(acc * s_w) * s_x) for the
// single plane (acc is an exact integer below 2^24).
__device__ __forceinline__ void store_y(const GemmTcParams& p, int t, int n, long long acc) {
  const float sx = __ldg(p.xscale + t);
  float v;
  if (p.tq) {
    v = __fmul_rn(__fmul_rn(__ll2float_rn(acc), 0x1p-24f), sx);
  } else {
    v = __fmul_rn(__fmul_rn(__int2float_rn((int)acc), p.tensor_scale), sx);
  }
  const size_t o = (size_t)t * p.n + n;
  if (p.out_bf16) {
    static_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(v);
  } else {
    static_cast<float*>(p.y)[o] = v;
  }
}

__device__ __forceinline__ long long to_ll(uint32_t v) { return (long long)(int)v; }

// The three roles of the kernel for P planes and D merged scale digits.
// A ring: groups of D tiles (the digits of one column); a tile is 128 rows x
// 64 k, 64 bytes per row, 64-byte swizzle. Stage boundaries: a stage starts
// at the CTA's first column and at every column that is a multiple of C (a new
// tile or pass starts at column 0), so every role finds them by itself.
template <int P, int D>
__device__ __forceinline__ void tc_roles(const GemmTcParams& p, uint8_t* smem, const TcLayout& L, uint32_t tmem,
                                         volatile uint32_t* misc, int passes, int tpass, int q0, int q1, int W) {
  const int NS = L.NS, NG = L.NG, C = L.C;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* full = bars;
  uint64_t* sfree = bars + kTcMaxStages;
  uint64_t* afull = bars + 2 * kTcMaxStages;
  uint64_t* afree = afull + kTcMaxSlots;
  uint64_t* accfull = afree + kTcMaxSlots;
  uint64_t* accfree = accfull + 1;
  uint64_t* fin = accfree + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cols = p.cols;
  const int G = p.grid;
  const int lg = p.tq ? 31 - __clz(p.group) : 0;  // groups are powers of two
  constexpr uint32_t kGroupBytes = (uint32_t)D * kSlotBytes;
  constexpr int kMw = D >= 2 ? 2 : 1;  // MMA-issuing warps with work

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    // lanes 0-3: the four row tiles' trits of the stage's columns, lanes 4-7
    // their scale blocks, lane 8 the activations: one copy instruction
    const int groups = p.tq ? p.k / p.group : 0;
    const size_t kchunks = (size_t)cols * 4;
    int col = q0 % cols, unit = q0 / cols;
    int tile = unit / passes, pass = unit % passes;
    int s = 0;
    uint32_t ph = 0;
    for (int q = q0, i = 0; q < q1; ++i) {
      const int n = min(min(C - (col & (C - 1)), cols - col), q1 - q);
      const int nrt = min(4, p.row_tiles - 4 * tile);
      const uint32_t st = smem_u32(smem + L.stages) + (uint32_t)s * L.stage_bytes;
      // scale blocks of the stage's columns; the last column may reach past
      // K, where the trits are zero and no block exists
      const int b0 = p.tq ? (col * 64) >> lg : 0;
      const int nb = p.tq ? min(((col + n) * 64 - 1) >> lg, groups - 1) - b0 + 1 : 0;
      uint32_t dst = 0, bytes = 0;
      const uint8_t* src = nullptr;
      if (lane < 4) {
        if (lane < nrt) {
          dst = st + (uint32_t)(lane * C * P * kPlaneColBytes);
          src = p.trit + ((size_t)(4 * tile + lane) * cols + col) * (P * kPlaneColBytes);
          bytes = (uint32_t)(n * P * kPlaneColBytes);
        }
      } else if (lane < 8) {
        const int r4 = lane - 4;
        if (p.tq && r4 < nrt) {
          dst = st + L.raw_bytes + (uint32_t)(r4 * L.sgroups * P * 64);
          src = reinterpret_cast<const uint8_t*>(p.scale + ((size_t)(4 * tile + r4) * groups + b0) * P * kTileRows);
          bytes = (uint32_t)(nb * P * 64);
        }
      } else if (lane == 8) {
        dst = st + L.raw_bytes + L.sc_bytes;
        src = p.xp + ((size_t)pass * kchunks + (size_t)col * 4) * (size_t)tpass * 16;
        bytes = (uint32_t)n * L.xcol_bytes;
      }
      uint32_t go = 1;
      if (lane == 0) {
        if (i >= NS && !tc_wait(&sfree[s], ph ^ 1u, misc)) go = 0;
        if (misc[kMiscAbort]) go = 0;
        const uint32_t total = (uint32_t)(nrt * n * P * kPlaneColBytes + nrt * nb * P * 64) + (uint32_t)n * L.xcol_bytes;
        if (go) mbar_arrive_expect_tx(&full[s], total);
      }
      go = __shfl_sync(0xffffffffu, go, 0);
      if (!go) break;
      if (bytes != 0u) bulk_g2s_plain(dst, src, bytes, &full[s]);
      q += n;
      col += n;
      if (col == cols) {
        col = 0;
        if (++pass == passes) {
          pass = 0;
          ++tile;
        }
      }
      if (++s == NS) {
        s = 0;
        ph ^= 1u;
      }
    }
    __syncwarp();
  } else if (warp < kDec0) {
    // ---------------------------------------------------------------- MMA
    // warp 1 issues digits [0, dh), warp 2 digits [dh, D)
    const int mw = warp - 1;
    constexpr int dh = kMw == 2 ? (D + 1) / 2 : D;
    if (lane == 0 && mw < kMw) {
      const int da = mw == 0 ? 0 : dh, db = mw == 0 ? dh : D;
      const uint32_t idesc = tc::idesc_i8_s32(tpass);
      const uint32_t slots = smem_u32(smem + L.slots);
      int col = q0 % cols, s = 0, j = 0, seg = 0, cc = 0;
      uint32_t ph = 0, aph = 0;
      for (int q = q0; q < q1; ++q) {
        if (misc[kMiscAbort]) break;
        const bool first = q == q0 || col == 0;
        const bool last = q == q1 - 1 || col == cols - 1;
        const bool sstart = q == q0 || (col & (C - 1)) == 0;
        const bool send = q + 1 == q1 || ((col + 1) & (C - 1)) == 0 || col + 1 == cols;
        if (first && seg > 0) {
          tc_wait(accfree, (uint32_t)(seg - 1) & 1u, misc);
          tc::fence_after_sync();
        }
        if (sstart) {
          tc_wait(&full[s], ph, misc);
          cc = 0;
        }
        const uint32_t xs = smem_u32(smem + L.stages) + (uint32_t)s * L.stage_bytes + L.raw_bytes + L.sc_bytes +
                            (uint32_t)cc * L.xcol_bytes;
        const uint64_t bd0 = tc::smem_desc(xs, tpass * 16, 128);
        const uint64_t bd1 = tc::smem_desc(xs + 2 * tpass * 16, tpass * 16, 128);
        tc_wait(&afull[j], aph, misc);
        tc::fence_after_sync();
        const uint32_t a0 = slots + (uint32_t)j * kGroupBytes;
        // this warp's accumulators are independent: interleave them so that
        // consecutive instructions do not wait on one another
#pragma unroll
        for (int d = 0; d < D; ++d)
          if (d >= da && d < db)
            tc::mma_i8(tmem + (uint32_t)(d * tpass), tc::smem_desc_sw64(a0 + (uint32_t)d * kSlotBytes, 512), bd0,
                       idesc, first ? 0u : 1u);
#pragma unroll
        for (int d = 0; d < D; ++d)
          if (d >= da && d < db)
            tc::mma_i8(tmem + (uint32_t)(d * tpass), tc::smem_desc_sw64(a0 + (uint32_t)d * kSlotBytes + 32, 512),
                       bd1, idesc, 1u);
        tc::commit(&afree[j]);
        if (++j == NG) {
          j = 0;
          aph ^= 1u;
        }
        if (send) {
          tc::commit(&sfree[s]);
          if (++s == NS) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (last) {
          tc::commit(accfull);
          ++seg;
        }
        ++cc;
        if (++col == cols) col = 0;
      }
      // every MMA issued has completed before tensor memory is released
      tc::commit(fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_test(fin, 0u)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          atomicOr(&g_dev_error, TERN_DEVERR_TIMEOUT);
          break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ decoders + epilogue
    // warp (q4, c): rows 32 q4 .. 32 q4 + 31 (tensor-memory lane quarter
    // warp % 4), chunk c (16 k) of every column, and a quarter of the tokens
    // in the epilogue
    const int ew = warp - kDec0, q4 = warp & 3, c = ew >> 2;
    const int r = 32 * q4 + lane;
    // A tiles in the 64-byte swizzled K-major layout: row r at 64 r, its
    // 16-byte chunk c at chunk position c ^ ((r >> 1) & 3)
    const uint32_t slots = smem_u32(smem + L.slots) + (uint32_t)r * 64u + (uint32_t)((c ^ ((r >> 1) & 3)) * 16);
    const uint32_t taddr = tmem + ((uint32_t)(32 * q4) << 16);
    int col = q0 % cols, unit = q0 / cols, s = 0, j = 0, seg = 0, gc = 0, cc = 0, b0 = 0;
    uint32_t ph = 0, aph = 0;
    for (int q = q0; q < q1; ++q) {
      const bool last = q == q1 - 1 || col == cols - 1;
      if (q == q0 || (col & (C - 1)) == 0) {
        tc_wait_many(&full[s], ph, misc);
        cc = 0;
        b0 = p.tq ? (col * 64) >> lg : 0;
      }
      const bool send = q + 1 == q1 || ((col + 1) & (C - 1)) == 0 || col + 1 == cols;
      const uint32_t st = smem_u32(smem + L.stages) + (uint32_t)s * L.stage_bytes;
      const uint32_t raw = st + (uint32_t)((q4 * C + cc) * P * kPlaneColBytes + lane * kChunkBytes + 4 * c);
      const int blk = p.tq ? ((col * 64 + 16 * c) >> lg) - b0 : 0;  // scale block of this chunk in the stage
      const uint32_t scs = st + L.raw_bytes + (uint32_t)((q4 * L.sgroups + blk) * P * 64 + lane * 2);
      ++cc;
      if (send && ++s == NS) {
        s = 0;
        ph ^= 1u;
      }
      // the column's word of every plane, its scale and selector nibbles
      uint32_t lo[P], lo2[P], hi[P], hi2[P], sel[P];
      uint64_t u[P];
#pragma unroll
      for (int pl = 0; pl < P; ++pl) {
        const uint32_t w = lds32(raw + pl * kPlaneColBytes);
        if (p.tq) {
          u[pl] = scale_units(lds16(scs + (uint32_t)(pl * 64)), sel[pl]);
        } else {
          u[pl] = 1u;
          sel[pl] = 0x3210u;
        }
        lo[pl] = w & 0x33333333u;
        hi[pl] = (w >> 2) & 0x33333333u;
        lo2[pl] = lo[pl] >> 16;
        hi2[pl] = hi[pl] >> 16;
      }
      if (gc >= NG) tc_wait_many(&afree[j], aph ^ 1u, misc);
      const uint32_t a = slots + (uint32_t)j * kGroupBytes;
      constexpr int kB = kDigitBits<P>;
      constexpr uint32_t kMask = (1u << kB) - 1u;
#pragma unroll
      for (int d = 0; d < D; ++d) {
        uint32_t o0 = 0, o1 = 0, o2 = 0, o3 = 0;
#pragma unroll
        for (int pl = 0; pl < P; ++pl) {
          const uint32_t ud = (uint32_t)(u[pl] >> (kB * d)) & kMask;
          const uint32_t lut = digit_lut(ud, plane_bias<P>(pl), sel[pl]);
          o0 += __byte_perm(lut, 0u, lo[pl]);
          o1 += __byte_perm(lut, 0u, lo2[pl]);
          o2 += __byte_perm(lut, 0u, hi[pl]);
          o3 += __byte_perm(lut, 0u, hi2[pl]);
        }
        if constexpr (P > 1) {  // remove the bias of 128 per byte
          o0 ^= 0x80808080u;
          o1 ^= 0x80808080u;
          o2 ^= 0x80808080u;
          o3 ^= 0x80808080u;
        }
        sts128(a + (uint32_t)d * kSlotBytes, o0, o1, o2, o3);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[j]);
      ++gc;
      if (++j == NG) {
        j = 0;
        aph ^= 1u;
      }
      const int ucur = unit;
      if (++col == cols) {
        col = 0;
        ++unit;
      }
      if (!last) continue;
      // ------------------------------------------------ segment epilogue
      const int tile = ucur / passes, pass = ucur % passes;
      // the tile's whole K range lies in this CTA's range
      const bool owned = col == 0 && q0 <= ucur * cols;
      tc_wait_many(accfull, (uint32_t)seg & 1u, misc);
      tc::fence_after_sync();
      const int n = tile * kTcRows + r;
      const int tq4 = tpass >> 2, tb = c * tq4, t0 = pass * tpass;
      for (int c4 = 0; c4 < tq4; c4 += 4) {
        long long acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int d = 0; d < D; ++d) {
          uint32_t v[4];
          tc::ld_x4_sync(taddr + (uint32_t)(d * tpass + tb + c4), v);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) acc[jj] += to_ll(v[jj]) << (kDigitBits<P> * d);
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int t = t0 + tb + c4 + jj;
          if (t < p.m && n < p.n) {
            if (owned) {
              store_y(p, t, n, acc[jj]);
            } else {
              atomicAdd(p.part + (size_t)t * p.n_pad + n, (unsigned long long)acc[jj]);
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(accfree);
      ++seg;
      if (!owned) {
        // the last CTA of this tile to arrive converts the exact sums
        __threadfence();
        named_sync_decoders();
        if (ew == 0 && lane == 0) {
          const long long qa = (long long)ucur * cols, qb = qa + cols - 1;
          const long long ca = ((qa + 1) * G - 1) / W, cb = ((qb + 1) * G - 1) / W;
          const unsigned old = atomicAdd(p.cnt + ucur, 1u);
          misc[kMiscLast] = (old + 1u == (unsigned)(cb - ca + 1)) ? 1u : 0u;
        }
        named_sync_decoders();
        if (misc[kMiscLast]) {
          __threadfence();
          for (int tt = tb; tt < tb + tq4; ++tt) {
            const int t = t0 + tt;
            if (t < p.m && n < p.n) {
              const unsigned long long v = atomicExch(p.part + (size_t)t * p.n_pad + n, 0ull);
              store_y(p, t, n, (long long)v);
            }
          }
          if (ew == 0 && lane == 0) atomicExch(p.cnt + ucur, 0u);
        }
      }
    }
  }
}

template <int P>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;

  int D7 = 1;
  if (p.tq) D7 = (int)__ldg(reinterpret_cast<const unsigned*>(p.header + kDigitsOffset));
  bool bad = D7 < 1 || D7 > kTcMaxDigits || (P > 1 && !p.tq);
  const int D = bad ? 1 : tc_merged_digits(P, D7);  // digits of the merged A operand
  int passes = 1, tpass = 16;
  tc_passes(D, p.m16, &passes, &tpass);
  TcLayout L;
  bad = !tc_layout(P, p.tq, p.group, D, tpass, &L) || bad || passes > p.passes_cap;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + L.misc);
  const uint32_t nmw = D >= 2 ? 2u : 1u;  // MMA warps that commit

  if (threadIdx.x == 0) {
    for (int i = 0; i < L.NS; ++i) {
      mbar_init(&bars[i], 1);                   // full
      mbar_init(&bars[kTcMaxStages + i], nmw);  // sfree
    }
    for (int j = 0; j < L.nslot; ++j) {
      mbar_init(&bars[2 * kTcMaxStages + j], kDecWarps);            // afull
      mbar_init(&bars[2 * kTcMaxStages + kTcMaxSlots + j], nmw);    // afree
    }
    uint64_t* acc = bars + 2 * kTcMaxStages + 2 * kTcMaxSlots;
    mbar_init(acc, nmw);            // accfull
    mbar_init(acc + 1, kDecWarps);  // accfree
    mbar_init(acc + 2, nmw);        // fin
    misc[kMiscAbort] = 0u;
    misc[kMiscLast] = 0u;
    if (bad && blockIdx.x == 0) atomicOr(&g_dev_error, TERN_DEVERR_FORMAT);
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32((const void*)&misc[kMiscTmem]), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = misc[kMiscTmem];

  // positions fit in 32 bits (the host checks tiles x 4 passes x columns)
  const int W = p.tiles * passes * p.cols;
  const int G = p.grid;
  const int q0 = (int)((long long)W * blockIdx.x / G);
  const int q1 = bad ? q0 : (int)((long long)W * (blockIdx.x + 1) / G);

  switch (D) {
    case 1: tc_roles<P, 1>(p, smem, L, tmem, misc, passes, tpass, q0, q1, W); break;
    case 2: tc_roles<P, 2>(p, smem, L, tmem, misc, passes, tpass, q0, q1, W); break;
    case 3: tc_roles<P, 3>(p, smem, L, tmem, misc, passes, tpass, q0, q1, W); break;
    case 4: tc_roles<P, 4>(p, smem, L, tmem, misc, passes, tpass, q0, q1, W); break;
    case 5: tc_roles<P, 5>(p, smem, L, tmem, misc, passes, tpass, q0, q1, W); break;
    case 6: tc_roles<P, 6>(p, smem, L, tmem, misc, passes, tpass, q0, q1, W); break;
    case 7: tc_roles<P, 7>(p, smem, L, tmem, misc, passes, tpass, q0, q1, W); break;
    case 8: tc_roles<P, 8>(p, smem, L, tmem, misc, passes, tpass, q0, q1, W); break;
    default: tc_roles<P, 9>(p, smem, L, tmem, misc, passes, tpass, q0, q1, W); break;
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// Activations in MMA order, pass-major so that the columns of one token pass
// are contiguous: xp[((pass * kchunks + kc) * tpass + t) * 16 + j] =
// xq[pass * tpass + t][16 kc + perm(j)] with perm = 0,8,1,9,...,7,15 (the
// decode order of a packed word); zero for tokens >= m and columns k >= K.
// The pass split follows the packed header's digit count, read here as in the
// GEMM kernel (an invalid count is flagged there; here it only keeps the
// writes inside the workspace).
__global__ void tc_prep_x_kernel(const int8_t* __restrict__ xq, int m, int k, int kchunks, long long total_max,
                                 int planes, int tq, const uint8_t* __restrict__ header, int m16, bool vec,
                                 uint8_t* __restrict__ xp) {
  int D7 = 1;
  if (tq) {
    D7 = (int)__ldg(reinterpret_cast<const unsigned*>(header + kDigitsOffset));
    if (D7 < 1 || D7 > kTcMaxDigits) D7 = 1;
  }
  int passes, tpass;
  tc_passes(tc_merged_digits(planes, D7), m16, &passes, &tpass);
  const long long total = (long long)passes * kchunks * tpass;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total || idx >= total_max) return;
  const int tl = (int)(idx % tpass);
  const long long rest = idx / tpass;
  const int kc = (int)(rest % kchunks), pass = (int)(rest / kchunks);
  const int t = pass * tpass + tl;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (t < m) {
    const int k0 = kc * 16;
    const int8_t* row = xq + (size_t)t * k;
    if (vec && k0 + 16 <= k) {
      v = *reinterpret_cast<const uint4*>(row + k0);
    } else {
      uint32_t wds[4] = {0u, 0u, 0u, 0u};
      for (int j = 0; j < 16 && k0 + j < k; ++j) wds[j >> 2] |= (uint32_t)(uint8_t)row[k0 + j] << (8 * (j & 3));
      v = make_uint4(wds[0], wds[1], wds[2], wds[3]);
    }
  }
  const uint4 o = make_uint4(__byte_perm(v.x, v.z, 0x5140), __byte_perm(v.x, v.z, 0x7362),
                             __byte_perm(v.y, v.w, 0x5140), __byte_perm(v.y, v.w, 0x7362));
  reinterpret_cast<uint4*>(xp)[idx] = o;
}

template <int P>
int launch_p(const GemmTcParams& p, void* stream) {
  auto kern = gemm_tc_kernel<P>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes);
  if (e != cudaSuccess) return (int)e;
  kern<<<p.grid, kThreads, kTcSmemBytes, static_cast<cudaStream_t>(stream)>>>(p);
  return (int)cudaGetLastError();
}

}  // namespace

int launch_gemm_tc(const GemmTcParams& p, void* stream) {
  switch (p.planes) {
    case 1: return launch_p<1>(p, stream);
    case 2: return launch_p<2>(p, stream);
    case 3: return launch_p<3>(p, stream);
    case 4: return launch_p<4>(p, stream);
    default: return -1;
  }
}

int launch_tc_prep_x(const int8_t* xq, int m, int k, int kchunks, int total_max, const GemmTcParams& p, uint8_t* xp,
                     void* stream) {
  if (total_max <= 0) return 0;
  const bool vec = (reinterpret_cast<uintptr_t>(xq) & 15u) == 0 && k % 16 == 0;
  const int threads = 256;
  const long long blocks = ((long long)total_max + threads - 1) / threads;
  tc_prep_x_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      xq, m, k, kchunks, total_max, p.planes, p.tq, p.header, p.m16, vec, xp);
  return (int)cudaGetLastError();
}

}  // namespace tern
