// Persistent decode step of a BitNet b1.58 transformer (QORA-LLM-2B page,
// "Architecture" and "SubLN Pattern (4 norms per layer)"): every layer of one
// token in one cooperative launch, one CTA per SM.
//
// Per layer, five stages separated by grid-wide barriers (and one more
// inside the attention):
//   S1  x = input_layernorm(h), int8 per token; q, k, v = ternary GEMVs
//   S2  RoPE (rotate_half) on q and k, the new k and v appended to the bf16
//       cache at `pos`, GQA attention over positions 0..pos
//   S3  a = attn_sub_norm(attn), int8; o = o_proj(a)
//   S4  h += o; x = post_attention_layernorm(h), int8; gate, up = GEMVs
//   S5  m = ffn_sub_norm(relu(gate)^2 * up), int8; d = down_proj(m)
//   (the next S1 starts with h += d)
//
// Every CTA holds the residual stream h in shared memory and computes each
// stage's normalisation and int8 quantisation itself, identically in every
// CTA (same data, same operation order), so no stage writes h or an
// activation vector to global memory; the stages exchange only the GEMVs'
// exact integer partial sums and the attention output.
//
// GEMV stages: the row tiles of the stage's projections, each cut into S
// column ranges ("parts"; S = 1 unless fewer than half the CTAs would get a
// tile), are dealt to the CTAs in contiguous runs. Inside a CTA every
// 64-k column is one warp's task (the CTA's column q to warp q mod 16). A
// part's exact int32 row sums go to its own slot of the workspace, and a
// consumer adds a row's S slots in order, so results do not depend on timing
// and nothing needs clearing between steps. Weights stream through a ring of
// 8 KB shared-memory slots filled by a producer warp with bulk async copies:
// the producer walks this CTA's chunks of every stage of every layer in order
// and runs ahead of the consumers across the grid barriers (weights depend on
// no stage), so the next stages' weights land while a barrier, a
// normalisation or the attention is in progress.
//
// A stage's input vector is gathered with every load in flight at once (four
// rows per 16-byte load of the partial sums), normalised and quantised in
// registers; the image's column sums come from shuffles of the same
// registers.
//
// Attention: the positions of each KV head are cut into NS ranges, one per
// CTA; each CTA computes its query heads' partial softmax state (running
// maximum, sum, weighted values) over its positions; after a grid barrier
// every CTA combines the NS states of a 1/G share of the outputs in a fixed
// order. The producer warp requests the cached keys and values of a CTA's
// range as soon as the previous layer's attention has released the buffer,
// so that they land long before they are used.
//
// Numerics follow the oracle's readings: RMSNorm with the factor
// 1/sqrt(mean(x^2) + eps) formed in double precision and rounded once to fp32;
// int8 absmax quantisation with the rule of tern_quantize_act; the ternary
// GEMV exact, y = fl(fl(float(acc) * s_w) * s_x); RoPE with every product and
// sum rounded; relu(g)^2 * up and the residual adds in fp32. Attention runs in
// fp32 (scores, softmax, weighted sum).
//
// Every wait is bounded (the mbarrier waits and the grid barrier give up
// after 1 s, raise an abort flag that the other CTAs see, and record a timeout
// in the device error word); on abort the producer waits, with a limit, for
// the copies it has in flight before its CTA exits.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "tern_internal.h"
#include "tern_ptx.cuh"

namespace tern {

int read_clear_dev_error_decode(void* stream, unsigned* out) { return read_clear_dev_error_tu(stream, out); }

namespace {

constexpr int kDW = 16;                  // consumer warps
constexpr int kDT = 32 * kDW;            // consumer threads
constexpr int kDBlock = kDT + 32;        // + the producer warp
constexpr int kChunkCols = 16;           // 64-k columns per ring slot
constexpr int kSlotBytes = kChunkCols * kPlaneColBytes;  // 8 KB
constexpr int kKvPass = 64;              // cached positions per attention pass (a whole range up to ~1,850 positions)
constexpr int kHD = kDecHeadDim;         // 128
constexpr int kBarNamed = 1;             // named barrier of the consumer threads

// ------------------------------------------------------------ shared plan
struct DecSmem {
  size_t params, tsc, tab, full, empty, kvbar, misc, h, img, csum, kv, scr, sacc, ring, total;  // kvbar: full, empty
  int nslot;
};

__host__ __device__ inline DecSmem dec_smem(const DecParams& p) {
  DecSmem s{};
  size_t off = 0;
  auto take = [&](size_t bytes, size_t align) {
    off = (off + align - 1) / align * align;
    const size_t at = off;
    off += bytes;
    return at;
  };
  s.params = take(sizeof(DecParams), 16);                   // the launch parameters
  s.tsc = take(4 * (size_t)kDecMaxLayers * 7, 16);          // every projection's tensor scale
  s.tab = take(4 * (4 + 5 * (size_t)kDecMaxPartsPerCta) * 4, 16);  // this CTA's share of the 4 GEMV stages
  s.full = take(8 * kDecMaxSlots, 8);
  s.empty = take(8 * kDecMaxSlots, 8);
  s.kvbar = take(16, 8);
  s.misc = take(1024, 16);                                  // reductions, flags, scales
  s.h = take(4 * (size_t)p.D, 16);                          // residual stream
  s.img = take((size_t)p.vmax, 16);                         // int8 image of a stage's input
  s.csum = take(4 * ((size_t)p.vmax / 64), 16);             // its column sums
  s.kv = take(2 * (size_t)kKvPass * kHD * 2, 128);          // cached keys then values of one pass
  s.scr = take(4 * ((size_t)(kDecMaxRep + 2) * kHD + (size_t)kDW * (kHD + 2)), 16);  // attention
  s.sacc = take(4 * 32 * (size_t)kDecMaxPartsPerCta, 16);   // a stage's part row sums
  s.ring = take(0, 128);
  const size_t avail = kDecSmemBytes > s.ring ? kDecSmemBytes - s.ring : 0;
  s.nslot = (int)(avail / kSlotBytes);
  if (s.nslot > kDecMaxSlots) s.nslot = kDecMaxSlots;
  s.total = s.ring + (size_t)s.nslot * kSlotBytes;
  return s;
}

// parts [a, b) of a GEMV stage for CTA c
__host__ __device__ inline void dec_parts(const DecStage& S, int c, int G, int* a, int* b) {
  *a = (int)((long long)S.parts * c / G);
  *b = (int)((long long)S.parts * (c + 1) / G);
}
__host__ __device__ inline void dec_part_cols(const DecStage& S, int part, int* tile, int* c0, int* c1) {
  *tile = part / S.splits;
  const int s = part - *tile * S.splits;
  *c0 = S.cols * s / S.splits;
  *c1 = S.cols * (s + 1) / S.splits;
}
__host__ __device__ inline int dec_problem_of(const DecStage& S, int tile) {
  int q = 0;
  while (q + 1 < S.nprob && S.tile0[q + 1] <= tile) ++q;
  return q;
}
// GEMV stage of stage index si (0: qkv, -1: attention, 1: o, 2: gate/up, 3: down)
__host__ __device__ inline int dec_gemv_of(int si) {
  const int s = si % 5;
  return s == 0 ? 0 : (s == 1 ? -1 : s - 1);
}

// This CTA's share of one GEMV stage, computed once per launch: its parts
// (tile, projection, columns [c0, c1) of the tile) in order, the chunk index
// of each part's first column within the stage, and the totals.
struct CtaStage {
  int pa, npart, ntot, nchunk;
  int tile[kDecMaxPartsPerCta], q[kDecMaxPartsPerCta], c0[kDecMaxPartsPerCta], c1[kDecMaxPartsPerCta];
  int cb[kDecMaxPartsPerCta];
};

static_assert(sizeof(CtaStage) == 4 * (4 + 5 * kDecMaxPartsPerCta), "shared-memory plan of the stage tables");

__device__ void cta_stage_table(const DecStage& S, int c, int G, CtaStage* T) {
  int pa, pb;
  dec_parts(S, c, G, &pa, &pb);
  T->pa = pa;
  T->npart = pb - pa;
  int ntot = 0, cb = 0;
  for (int i = 0; i < pb - pa; ++i) {
    int tile, c0, c1;
    dec_part_cols(S, pa + i, &tile, &c0, &c1);
    T->tile[i] = tile;
    T->q[i] = dec_problem_of(S, tile);
    T->c0[i] = c0;
    T->c1[i] = c1;
    T->cb[i] = cb;
    ntot += c1 - c0;
    cb += (c1 - c0 + kChunkCols - 1) / kChunkCols;
  }
  T->ntot = ntot;
  T->nchunk = cb;
}

// ------------------------------------------------------------ primitives
__device__ __forceinline__ void named_sync() { asm volatile("bar.sync %0, %1;" ::"n"(kBarNamed), "n"(kDT) : "memory"); }

// AND of a predicate over the consumer threads, with the named barrier: a
// stage's outcome becomes the same in every warp before anything that
// depends on it (warps that disagreed would reach different barriers)
__device__ __forceinline__ bool cta_and(bool v) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((unsigned)v), "n"(kBarNamed), "n"(kDT)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t cnt) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(cnt) : "memory");
}

__device__ __forceinline__ int4 ldcg_i4(const int* p) { return __ldcg(reinterpret_cast<const int4*>(p)); }

__device__ __forceinline__ float bf16_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ uint32_t f32_to_bf16_rn(float v) {
  const uint32_t b = __float_as_uint(v);
  return (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;
}

// `bar` counts barrier arrivals; its top bit is the abort flag, so that one
// load tells a waiting CTA both whether the barrier has opened and whether
// some CTA gave up.
struct DecCtl {
  unsigned bar, exitc, pad0, pad1;
};
constexpr unsigned kAbortBit = 0x80000000u;

__device__ __noinline__ void raise_abort(DecCtl* ctl) {
  atomicOr(&g_dev_error, TERN_DEVERR_TIMEOUT);
  atomicOr(&ctl->bar, kAbortBit);
}
__device__ __forceinline__ bool aborted(const DecCtl* ctl) { return (ld_acquire_u32(&ctl->bar) & kAbortBit) != 0u; }

// Grid barrier over the consumer threads of every CTA (bounded). Returns false
// if a CTA gave up (timeout here or elsewhere).
__device__ bool grid_sync(DecCtl* ctl, unsigned& epoch, volatile int* s_ok) {
  named_sync();
  if (threadIdx.x == 0) {
    bool ok = true;
    red_release_add(&ctl->bar, 1u);
    const unsigned target = (epoch + 1u) * gridDim.x;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
      const unsigned v = ld_acquire_u32(&ctl->bar);
      if (v & kAbortBit) {
        ok = false;
        break;
      }
      if (v >= target) break;
      if ((it & 63u) == 63u) {
        if (t0 == 0) t0 = global_timer_ns();
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          raise_abort(ctl);
          ok = false;
          break;
        }
      }
    }
    *s_ok = ok ? 1 : 0;
  }
  ++epoch;
  named_sync();
  return *s_ok != 0;
}

// Sum / maximum over the consumer threads in a fixed order (butterfly in the
// warp, then the warps' values in warp order): every CTA gets bit-identical
// results. `red` is read before the caller's next named barrier and written
// again only after it.
__device__ double block_sum_d(double v, double* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  named_sync();
  double s = 0.0;
#pragma unroll
  for (int w = 0; w < kDW; ++w) s += red[w];
  return s;
}

__device__ unsigned block_max_u(unsigned v, unsigned* red) {
  v = __reduce_max_sync(0xffffffffu, v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  named_sync();
  unsigned m = 0;
#pragma unroll
  for (int w = 0; w < kDW; ++w) m = max(m, red[w]);
  return m;
}

__device__ __forceinline__ float4 i4_to_f4_scaled(int4 a, float sw, float sx) {
  return make_float4(__fmul_rn(__fmul_rn(__int2float_rn(a.x), sw), sx), __fmul_rn(__fmul_rn(__int2float_rn(a.y), sw), sx),
                     __fmul_rn(__fmul_rn(__int2float_rn(a.z), sw), sx), __fmul_rn(__fmul_rn(__int2float_rn(a.w), sw), sx));
}
__device__ __forceinline__ int4 add_i4(int4 a, int4 b) { return make_int4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
__device__ __forceinline__ float4 add_f4(float4 a, float4 b) {
  return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z), __fadd_rn(a.w, b.w));
}
__device__ __forceinline__ float relu2_mul(float g, float u) {
  const float r = g > 0.f ? g : 0.f;
  return __fmul_rn(__fmul_rn(r, r), u);
}
__device__ __forceinline__ int quant1(float v, float inv) {
  return v != 0.f ? max(-127, min(127, __float2int_rn(__fmul_rn(v, inv)))) : 0;
}

// cached positions (before `pos`) of CTA c's attention range
__device__ __forceinline__ int kv_cached(const DecParams& p, int c) {
  if (c >= p.KVH * p.ns) return 0;
  const int j = c / p.ns, s = c - j * p.ns;
  const int npos = p.pos + 1;
  const int p0 = (int)((long long)npos * s / p.ns);
  const int pc1 = min((int)((long long)npos * (s + 1) / p.ns), p.pos);
  return max(0, pc1 - p0);
}

// copy `cnt` cached keys and values of CTA c's KV head, from position
// p0 + base, into the pass buffer (keys, then values at kKvPass rows)
__device__ __forceinline__ void kv_issue(const DecParams& p, uint64_t* bar, uint16_t* kvs, int layer, int c, int base,
                                         int cnt) {
  const int j = c / p.ns, s = c - j * p.ns;
  const int p0 = (int)((long long)(p.pos + 1) * s / p.ns);
  const size_t row = ((size_t)(layer * p.KVH + j) * p.max_pos + p0 + base) * kHD;
  const uint32_t bytes = (uint32_t)cnt * kHD * 2;
  mbar_arrive_expect_tx(bar, 2 * bytes);
  const uint64_t pol = policy_evict_first();
  bulk_g2s(kvs, p.kc + row, bytes, bar, pol);
  bulk_g2s(kvs + kKvPass * kHD, p.vc + row, bytes, bar, pol);
}

// ------------------------------------------------------------ the kernel
// NW: 4-element words of a stage's input vector per consumer thread.
template <int NW>
__global__ void __launch_bounds__(kDBlock, 1) decode_kernel(const __grid_constant__ DecParams pg) {
  extern __shared__ __align__(128) uint8_t smem[];
  const DecSmem sp = dec_smem(pg);
  // The parameter block goes to shared memory once: the stages index it with
  // run-time values (stage, layer, projection), and reads of the parameter
  // space that miss its cache cost on the order of a microsecond each. The
  // projections' tensor scales (in their packed headers) are read once too.
  {
    static_assert(sizeof(DecParams) % 8 == 0, "copied as 64-bit words");
    const long long* src = reinterpret_cast<const long long*>(&pg);
    long long* dst = reinterpret_cast<long long*>(smem + sp.params);
    for (int i = threadIdx.x; i < (int)(sizeof(DecParams) / 8); i += blockDim.x) dst[i] = src[i];
    float* tsc = reinterpret_cast<float*>(smem + sp.tsc);
    for (int i = threadIdx.x; i < pg.layers * 7; i += blockDim.x)
      tsc[i] = __ldg(reinterpret_cast<const float*>(pg.packed[i / 7][i % 7] + 28));
  }
  if (threadIdx.x < 4) cta_stage_table(pg.st[threadIdx.x], blockIdx.x, gridDim.x, reinterpret_cast<CtaStage*>(smem + sp.tab) + threadIdx.x);
  __syncthreads();
  const DecParams& p = *reinterpret_cast<const DecParams*>(smem + sp.params);
  const float* tsc = reinterpret_cast<const float*>(smem + sp.tsc);
  const CtaStage* tab = reinterpret_cast<const CtaStage*>(smem + sp.tab);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + sp.full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + sp.empty);
  uint64_t* kvbar = reinterpret_cast<uint64_t*>(smem + sp.kvbar);
  uint8_t* ring = smem + sp.ring;
  const int nslot = sp.nslot;
  DecCtl* ctl = reinterpret_cast<DecCtl*>(p.ws + p.off_ctl);

  if (threadIdx.x == 0) {
    for (int i = 0; i < nslot; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kChunkCols);  // one arrival per column (partial chunks make up the rest)
    }
    mbar_init(kvbar, 1);      // the cached keys and values of a pass have landed
    mbar_init(kvbar + 1, 1);  // the consumers are done with the buffer
    fence_mbar_init();
  }
  __syncthreads();

  // ================================================== producer warp
  if (warp == kDW) {
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    unsigned n = 0;  // chunks issued
    bool ok = true;
    unsigned nkv = 0;  // first passes of cached keys and values issued
    for (int si = p.first; si <= p.last && ok; ++si) {
      // once per stage: a CTA that gave up stops the copies (a wait below that
      // the consumers no longer answer ends at its own limit)
      if (aborted(ctl)) {
        ok = false;
        break;
      }
      const int gt = dec_gemv_of(si);
      if (gt < 0) {
        // this layer's cached keys and values, pass by pass, into the KV buffer
        // once the consumers have released the previous pass
        const int ncached = kv_cached(p, cta);
        for (int base = 0; base < ncached && ok; base += kKvPass) {
          if (nkv > 0 && !mbar_wait_bounded(kvbar + 1, (nkv - 1u) & 1u)) {
            ok = false;
            break;
          }
          kv_issue(p, kvbar, reinterpret_cast<uint16_t*>(smem + sp.kv), si / 5, cta, base,
                   min(kKvPass, ncached - base));
          ++nkv;
        }
        continue;
      }
      const DecStage& S = p.st[gt];
      const CtaStage& T = tab[gt];
      const int layer = si / 5;
      for (int i = 0; i < T.npart && ok; ++i) {
        const int q = T.q[i], c0 = T.c0[i], c1 = T.c1[i];
        const uint8_t* tr = p.packed[layer][S.proj[q]] + kHeaderBytes;
        const int tt = T.tile[i] - S.tile0[q];
        for (int c = c0; c < c1; c += kChunkCols) {
          const int nc = min(kChunkCols, c1 - c);
          const int slot = (int)(n % (unsigned)nslot);
          const unsigned round = n / (unsigned)nslot;
          if (round > 0 && !mbar_wait_bounded(&empty[slot], (round - 1u) & 1u)) {
            ok = false;
            break;
          }
          const uint32_t bytes = (uint32_t)nc * kPlaneColBytes;
          mbar_arrive_expect_tx(&full[slot], bytes);
          bulk_g2s(ring + (size_t)slot * kSlotBytes, tr + ((size_t)tt * S.cols + c) * kPlaneColBytes, bytes,
                   &full[slot], pol);
          ++n;
        }
      }
    }
    if (!ok) raise_abort(ctl);
    // every copy this warp issued has landed before the CTA can exit (bounded;
    // immediate on the normal path, where the consumers have used them all)
    const unsigned lo = n > (unsigned)nslot ? n - (unsigned)nslot : 0u;
    for (unsigned j = lo; j < n; ++j) (void)mbar_wait_bounded(&full[j % nslot], (j / nslot) & 1u);
    // and the last copy of cached keys and values
    if (nkv > 0) (void)mbar_wait_bounded(kvbar, (nkv - 1u) & 1u);
    return;
  }

  // ================================================== consumer threads
  const int tid = threadIdx.x;
  float* h = reinterpret_cast<float*>(smem + sp.h);
  uint32_t* img = reinterpret_cast<uint32_t*>(smem + sp.img);  // 4 int8 per word
  int* csum = reinterpret_cast<int*>(smem + sp.csum);
  float* scr = reinterpret_cast<float*>(smem + sp.scr);
  int* sacc = reinterpret_cast<int*>(smem + sp.sacc);
  uint16_t* kvs = reinterpret_cast<uint16_t*>(smem + sp.kv);
  double* red_d = reinterpret_cast<double*>(smem + sp.misc);           // [16]
  unsigned* red_u = reinterpret_cast<unsigned*>(smem + sp.misc + 128);  // [16]
  volatile int* s_flag = reinterpret_cast<volatile int*>(smem + sp.misc + 192);
  float* s_scale = reinterpret_cast<float*>(smem + sp.misc + 256);     // [4] the GEMV stages' s_x

  unsigned epoch = 0, nchunk = 0, kvphase = 0;
  bool ok = true;
  const int D = p.D, HQ = p.H * kHD, KVH = p.KVH, rep = p.H / p.KVH;
  const int ns = p.ns;

  for (int i = tid; i < D; i += kDT) h[i] = p.h_in[i];
  named_sync();

  auto tensor_scale = [&](int layer, int proj) -> float { return tsc[layer * 7 + proj]; };
  // partial-sum slot of rows n..n+3 (n % 4 == 0) of problem q of GEMV stage gt, split 0
  auto part_ptr = [&](int gt, int q, int n) -> const int* {
    const DecStage& S = p.st[gt];
    const int t = S.tile0[q] + (n >> 5);
    return reinterpret_cast<const int*>(p.ws + p.off_part[gt]) + (size_t)t * S.splits * 32 + (n & 31);
  };

  // ---- RMSNorm + int8 image of a GEMV stage's input (every CTA, identically)
  auto image_stage = [&](int si) {
    const int layer = si / 5, st = si % 5, gt = dec_gemv_of(si);
    const bool fresh = si == p.first;
    const float* gains = p.gains + (size_t)layer * p.gain_stride;
    int n, mode, sgt = 0;  // mode 0: h += linear; 1: h; 2: attention output; 3: relu^2(gate) * up
    const float* g;
    float sw0 = 0.f, sw1 = 0.f;
    if (st == 0) {
      n = D, g = gains, mode = fresh ? 1 : 0, sgt = 3;
      if (!fresh) sw0 = tensor_scale(layer - 1, 6);
    } else if (st == 2) {
      n = HQ, g = gains + D, mode = 2;
    } else if (st == 3) {
      n = D, g = gains + D + HQ, mode = fresh ? 1 : 0, sgt = 1;
      if (!fresh) sw0 = tensor_scale(layer, 3);
    } else {
      n = p.F, g = gains + 2 * D + HQ, mode = 3, sgt = 2;
      sw0 = tensor_scale(layer, 4), sw1 = tensor_scale(layer, 5);
    }
    const int nwords = n >> 2;
    // phase 1: every load of the stage's inputs (and the norm's gains) in flight at once
    int4 ra[NW], rb[NW];
    float4 fa[NW], gv[NW];
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      ra[j] = rb[j] = make_int4(0, 0, 0, 0);
      fa[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      const int w = tid + j * kDT;
      gv[j] = w < nwords ? __ldg(reinterpret_cast<const float4*>(g) + w) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (mode == 0 || mode == 3) {
      const int splits = p.st[sgt].splits;
      for (int s = 0; s < splits; ++s) {
#pragma unroll
        for (int j = 0; j < NW; ++j) {
          const int w = tid + j * kDT;
          if (w < nwords) {
            ra[j] = add_i4(ra[j], ldcg_i4(part_ptr(sgt, 0, 4 * w) + 32 * s));
            if (mode == 3) rb[j] = add_i4(rb[j], ldcg_i4(part_ptr(sgt, 1, 4 * w) + 32 * s));
          }
        }
      }
    } else if (mode == 2) {
      const float* src = fresh ? p.attn_in : reinterpret_cast<const float*>(p.ws + p.off_attn);
#pragma unroll
      for (int j = 0; j < NW; ++j) {
        const int w = tid + j * kDT;
        if (w < nwords)
          fa[j] = fresh ? __ldg(reinterpret_cast<const float4*>(src) + w) : __ldcg(reinterpret_cast<const float4*>(src) + w);
      }
    }
    // phase 2: the vector (residual adds into h) and its sum of squares
    const float sx = s_scale[sgt];
    float4 v[NW];
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      const int w = tid + j * kDT;
      v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (w < nwords) {
        float4 x;
        if (mode <= 1) {
          x = reinterpret_cast<const float4*>(h)[w];
          if (mode == 0) {
            x = add_f4(x, i4_to_f4_scaled(ra[j], sw0, sx));
            reinterpret_cast<float4*>(h)[w] = x;
          }
        } else if (mode == 2) {
          x = fa[j];
        } else {
          const float4 gg = i4_to_f4_scaled(ra[j], sw0, sx), uu = i4_to_f4_scaled(rb[j], sw1, sx);
          x = make_float4(relu2_mul(gg.x, uu.x), relu2_mul(gg.y, uu.y), relu2_mul(gg.z, uu.z), relu2_mul(gg.w, uu.w));
        }
        v[j] = x;
        ss += (double)x.x * x.x + (double)x.y * x.y + (double)x.z * x.z + (double)x.w * x.w;
      }
    }
    // phase 3: RMSNorm with the gain, absmax, int8 codes, column sums
    const double tot = block_sum_d(ss, red_d);
    const float r = (float)(1.0 / sqrt(tot / (double)n + (double)p.eps));
    unsigned am = 0;
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      const int w = tid + j * kDT;
      if (w < nwords) {
        v[j] = make_float4(__fmul_rn(__fmul_rn(v[j].x, r), gv[j].x), __fmul_rn(__fmul_rn(v[j].y, r), gv[j].y),
                           __fmul_rn(__fmul_rn(v[j].z, r), gv[j].z), __fmul_rn(__fmul_rn(v[j].w, r), gv[j].w));
        am = max(am, max(max(__float_as_uint(v[j].x) & 0x7FFFFFFFu, __float_as_uint(v[j].y) & 0x7FFFFFFFu),
                         max(__float_as_uint(v[j].z) & 0x7FFFFFFFu, __float_as_uint(v[j].w) & 0x7FFFFFFFu)));
      }
    }
    const float a = __uint_as_float(block_max_u(am, red_u));
    const float inv = a > 0.f ? __fdiv_rn(127.0f, a) : 0.f;
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      const int w = tid + j * kDT;  // the 16 words of a 64-k column sit in 16 consecutive lanes
      int bsum = 0;
      if (w < nwords) {
        const int q0 = quant1(v[j].x, inv), q1 = quant1(v[j].y, inv), q2 = quant1(v[j].z, inv),
                  q3 = quant1(v[j].w, inv);
        img[w] = (uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8) | ((uint32_t)(q2 & 0xFF) << 16) |
                 ((uint32_t)(q3 & 0xFF) << 24);
        bsum = q0 + q1 + q2 + q3;
      }
#pragma unroll
      for (int o = 8; o; o >>= 1) bsum += __shfl_xor_sync(0xffffffffu, bsum, o);
      if ((lane & 15) == 0 && w < nwords) csum[w >> 4] = bsum;
    }
    if (tid == 0) s_scale[gt] = a > 0.f ? __fdiv_rn(a, 127.0f) : 0.f;
    // the stage's part sums start at zero
    for (int i = tid; i < tab[gt].npart * 32; i += kDT) sacc[i] = 0;
    named_sync();
  };

  // ---- this CTA's parts of GEMV stage gt over the image: the CTA's columns
  // (its parts' 64-k columns in order) in 16 contiguous blocks, one per warp;
  // a warp waits for and releases each chunk it touches once; exact row sums
  // per part
  auto gemv_stage = [&](int gt) -> bool {
    const CtaStage& T = tab[gt];
    const int ntot = T.ntot;
    const int q0 = (ntot * warp) >> 4, q1 = (ntot * (warp + 1)) >> 4;  // this warp's columns (16 warps)
    const uint32_t ring32 = smem_u32(ring) + lane * 16;
    const uint32_t img32 = smem_u32(img);
    int qbase = 0;
    bool good = true;
    for (int part = 0; part < T.npart && good; ++part) {
      const int c0 = T.c0[part], len = T.c1[part] - c0, cb = T.cb[part];
      const int lo = max(q0, qbase) - qbase, hi = min(q1, qbase + len) - qbase;  // columns c0 + [lo, hi)
      qbase += len;
      if (hi <= lo) continue;
      int acc = 0;
      for (int a = lo; a < hi && good;) {
        const int ch = a >> 4, e = min(hi, (ch + 1) * kChunkCols);  // this chunk's columns [a, e)
        const unsigned nn = nchunk + (unsigned)(cb + ch);
        const int slot = (int)(nn % (unsigned)nslot);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[slot], (nn / (unsigned)nslot) & 1u))) {
          good = false;
          break;
        }
        const uint32_t sbase = ring32 + (uint32_t)(slot * kSlotBytes);
        for (int col = a; col < e; ++col) {
          const uint4 wv = lds128<0>(sbase + (uint32_t)((col - ch * kChunkCols) * kPlaneColBytes));
          const uint32_t xa = img32 + 64u * (uint32_t)(c0 + col);
          int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
          const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int4 xv = u4_as_i4(lds128<0>(xa + 16 * k));
            const uint32_t Fd = lop3_ternary_digit(wd[k]);
            a0 = dp4a_ss((int)(Fd & 0x03030303u), xv.x, a0);
            a1 = dp4a_ss((int)(Fd & 0x0C0C0C0Cu), xv.y, a1);
            a2 = dp4a_ss((int)(Fd & 0x30303030u), xv.z, a2);
            a3 = dp4a_us(Fd & 0xC0C0C0C0u, xv.w, a3);
          }
          acc += csum[c0 + col] - (a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6));  // sum t x = sum x - sum F x
        }
        // release: the arrival (release semantics) orders this warp's reads of
        // the slot before the producer's refill, which waits for it; one
        // arrival per column used, and the warp holding a short chunk's first
        // column arrives for the columns the chunk lacks
        __syncwarp();
        if (lane == 0) {
          const int nch = min(kChunkCols, len - ch * kChunkCols);
          uint32_t cnt = (uint32_t)(e - a);
          if (a == ch * kChunkCols) cnt += (uint32_t)(kChunkCols - nch);
          mbar_arrive_cnt(&empty[slot], cnt);
        }
        a = e;
      }
      atomicAdd(&sacc[part * 32 + lane], acc);
    }
    const int cb = T.nchunk;
    const int pa = T.pa, pb = T.pa + T.npart;
    nchunk += (unsigned)cb;
    if (!good) raise_abort(ctl);
    named_sync();
    int* P = reinterpret_cast<int*>(p.ws + p.off_part[gt]);
    for (int i2 = tid; i2 < (pb - pa) * 32; i2 += kDT) P[(size_t)pa * 32 + i2] = sacc[i2];
    return good;
  };

  // ---- attention of `layer` (stage S2): this CTA's KV head j and position
  // range [p0, p1): the partial softmax state of each of its query heads
  auto attention_stage = [&](int layer) -> bool {
    if (cta >= KVH * ns) return true;
    const int j = cta / ns, sp_ = cta - j * ns;
    const int npos = p.pos + 1;
    const int p0 = (int)((long long)npos * sp_ / ns);
    const int p1 = (int)((long long)npos * (sp_ + 1) / ns);
    float* qs = scr;                        // [rep][128] query heads, then the key, the value
    float* ks = scr + rep * kHD;
    float* vs = ks + kHD;
    {
      // q, k, v of this head group with RoPE (rotate_half, pair (f, f + 64)):
      // thread t < (rep + 1) * 16 takes pairs 4u .. 4u + 3 of one vector (two
      // 16-byte loads per split), threads above take 4 value rows
      const DecStage& S = p.st[0];
      const float sxq = s_scale[0];
      const int nrot = (rep + 1) * (kHD / 8);
      const float* cs = p.rope + (size_t)p.pos * kHD;  // [64][2] cos, sin
      float* tr = p.trace && sp_ == 0 ? p.trace + (size_t)layer * p.trace_stride : nullptr;
      if (tid < nrot) {
        const int vec = tid / (kHD / 8), u = tid - vec * (kHD / 8);  // vector, pairs 4u..4u+3
        const int q = vec < rep ? 0 : 1;
        const int row = (vec < rep ? j * rep + vec : j) * kHD + 4 * u;
        int4 ra = make_int4(0, 0, 0, 0), rb = ra;
        for (int s2 = 0; s2 < S.splits; ++s2) {
          ra = add_i4(ra, ldcg_i4(part_ptr(0, q, row) + 32 * s2));
          rb = add_i4(rb, ldcg_i4(part_ptr(0, q, row + kHD / 2) + 32 * s2));
        }
        const float sw = tensor_scale(layer, q);
        const float4 a = i4_to_f4_scaled(ra, sw, sxq), b = i4_to_f4_scaled(rb, sw, sxq);
        const float4 c0 = __ldg(reinterpret_cast<const float4*>(cs) + 2 * u);      // cos, sin of 4u, 4u+1
        const float4 c1 = __ldg(reinterpret_cast<const float4*>(cs) + 2 * u + 1);  // of 4u+2, 4u+3
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
        const float cv[4] = {c0.x, c0.z, c1.x, c1.z}, sv[4] = {c0.y, c0.w, c1.y, c1.w};
        float* v = scr + vec * kHD;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = __fsub_rn(__fmul_rn(av[e], cv[e]), __fmul_rn(bv[e], sv[e]));
          const float hi = __fadd_rn(__fmul_rn(bv[e], cv[e]), __fmul_rn(av[e], sv[e]));
          const int f = 4 * u + e;
          if (tr) {
            const size_t o = vec < rep ? (size_t)(j * rep + vec) * kHD : (size_t)HQ + (size_t)j * kHD;
            tr[o + f] = lo;
            tr[o + f + kHD / 2] = hi;
          }
          if (vec == rep) {  // the key: bf16 as stored in the cache
            const uint32_t kl = f32_to_bf16_rn(lo), kh = f32_to_bf16_rn(hi);
            if (sp_ == ns - 1) {
              const size_t at = ((size_t)(layer * KVH + j) * p.max_pos + p.pos) * kHD;
              p.kc[at + f] = (uint16_t)kl;
              p.kc[at + f + kHD / 2] = (uint16_t)kh;
            }
            v[f] = bf16_to_f32(kl);
            v[f + kHD / 2] = bf16_to_f32(kh);
          } else {
            v[f] = lo;
            v[f + kHD / 2] = hi;
          }
        }
      } else if (tid < nrot + kHD / 4) {
        const int u = tid - nrot;  // value rows 4u .. 4u + 3
        int4 ra = make_int4(0, 0, 0, 0);
        for (int s2 = 0; s2 < S.splits; ++s2) ra = add_i4(ra, ldcg_i4(part_ptr(0, 2, j * kHD + 4 * u) + 32 * s2));
        const float4 a = i4_to_f4_scaled(ra, tensor_scale(layer, 2), sxq);
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int f = 4 * u + e;
          if (tr) tr[(size_t)HQ + (size_t)KVH * kHD + (size_t)j * kHD + f] = av[e];
          const uint32_t vb = f32_to_bf16_rn(av[e]);
          if (sp_ == ns - 1) p.vc[((size_t)(layer * KVH + j) * p.max_pos + p.pos) * kHD + f] = (uint16_t)vb;
          vs[f] = bf16_to_f32(vb);
        }
      }
    }
    named_sync();
    // scores and running softmax: warp = (query head hh, position group pg);
    // scores are kept in units of log2(e) so that exp2 applies directly
    const int hh = warp >> 2, pg = warp & 3;
    const bool active = hh < rep;
    float qv[4] = {0.f, 0.f, 0.f, 0.f};
    if (active)
#pragma unroll
      for (int e = 0; e < 4; ++e) qv[e] = qs[hh * kHD + 4 * lane + e];
    float m = -INFINITY, l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    const float kScale = 0.08838834764831845f * 1.4426950408889634f;  // log2(e) / sqrt(128)
    auto visit = [&](const float* kv4, const float* vv4) {
      float part = qv[0] * kv4[0];
      part = fmaf(qv[1], kv4[1], part);
      part = fmaf(qv[2], kv4[2], part);
      part = fmaf(qv[3], kv4[3], part);
#pragma unroll
      for (int off = 16; off; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      const float sc = part * kScale;
      const float mn = fmaxf(m, sc);
      const float corr = exp2f(m - mn), pe = exp2f(sc - mn);
      l = fmaf(l, corr, pe);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = fmaf(o[e], corr, pe * vv4[e]);
      m = mn;
    };
    const int pc1 = min(p1, p.pos);  // cached positions of this range: [p0, pc1)
    bool good = true;
    for (int base = p0; base < pc1; base += kKvPass) {
      // every warp takes every pass (and its barrier), even after a failed wait
      const int cnt = min(kKvPass, pc1 - base);
      const bool landed = __all_sync(0xffffffffu, mbar_wait_bounded(kvbar, kvphase & 1u));
      good = good && landed;
      ++kvphase;
      if (active && landed) {
        for (int t = pg; t < cnt; t += 4) {
          const uint2 kr = *reinterpret_cast<const uint2*>(kvs + (size_t)t * kHD + 4 * lane);
          const uint2 vr = *reinterpret_cast<const uint2*>(kvs + (size_t)(kKvPass + t) * kHD + 4 * lane);
          const float k4[4] = {bf16_to_f32(kr.x & 0xFFFFu), bf16_to_f32(kr.x >> 16), bf16_to_f32(kr.y & 0xFFFFu),
                               bf16_to_f32(kr.y >> 16)};
          const float v4[4] = {bf16_to_f32(vr.x & 0xFFFFu), bf16_to_f32(vr.x >> 16), bf16_to_f32(vr.y & 0xFFFFu),
                               bf16_to_f32(vr.y >> 16)};
          visit(k4, v4);
        }
      }
      // the buffer is free for the producer's next pass
      named_sync();
      if (tid == 0) mbar_arrive_cnt(kvbar + 1, 1u);
    }
    if (!cta_and(good)) {  // the same decision in every warp: the merge below has a barrier
      raise_abort(ctl);
      return false;
    }
    // the current position (in the last range)
    if (active && p1 == npos && pg == ((npos - 1 - p0) & 3)) visit(ks + 4 * lane, vs + 4 * lane);
    // merge the four position groups of each query head into this range's state
    float* st = scr + (kDecMaxRep + 2) * kHD;  // [16 warps][130]
    if (lane == 0) {
      st[warp * (kHD + 2)] = m;
      st[warp * (kHD + 2) + 1] = l;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) st[warp * (kHD + 2) + 2 + 4 * lane + e] = o[e];
    named_sync();
    float* Pa = reinterpret_cast<float*>(p.ws + p.off_att);
    for (int i = tid; i < rep * kHD; i += kDT) {
      const int r = i / kHD, d = i - r * kHD;
      float M = -INFINITY;
      for (int g = 0; g < 4; ++g) M = fmaxf(M, st[(4 * r + g) * (kHD + 2)]);
      float L = 0.f, O = 0.f;
      for (int g = 0; g < 4; ++g) {
        const float* e = st + (4 * r + g) * (kHD + 2);
        if (e[1] == 0.f) continue;
        const float w = exp2f(e[0] - M);
        L = fmaf(e[1], w, L);
        O = fmaf(e[2 + d], w, O);
      }
      float* dst = Pa + ((size_t)(j * ns + sp_) * rep + r) * (kHD + 2);
      if (d == 0) {
        dst[0] = M;
        dst[1] = L;
      }
      dst[2 + d] = O;
    }
    return true;
  };

  // ---- combine the ranges' states (after the attention's grid barrier): CTA
  // c finishes outputs [c * HQ / G, (c + 1) * HQ / G) of the attention, a warp
  // per output and a lane per position range: each lane loads its ranges'
  // (maximum, sum, weighted value) in one round, folds them in order, and the
  // lanes' states merge by a fixed butterfly
  auto combine_stage = [&](int layer) {
    const int o0 = (int)((long long)HQ * cta / G), o1 = (int)((long long)HQ * (cta + 1) / G);
    const float* Pa = reinterpret_cast<const float*>(p.ws + p.off_att);
    float* outp = reinterpret_cast<float*>(p.ws + p.off_attn);
    const size_t stride = (size_t)rep * (kHD + 2);
    // two outputs per warp per trip, their loads issued together
    for (int out0 = o0 + warp; out0 < o1; out0 += 2 * kDW) {
      float M[2], L[2], O[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        M[u] = -INFINITY;
        L[u] = 0.f;
        O[u] = 0.f;
      }
      for (int s0 = 0; s0 < ns; s0 += 32) {
        const int s2 = s0 + lane;
        float ms[2], ls[2], os[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int out = out0 + u * kDW;
          ms[u] = -INFINITY;
          ls[u] = 0.f;
          os[u] = 0.f;
          if (s2 < ns && out < o1) {
            const int h = out / kHD, d = out - h * kHD;
            const int jj = h / rep, r = h - jj * rep;
            const float* e = Pa + ((size_t)jj * ns * rep + r) * (kHD + 2) + s2 * stride;
            ms[u] = __ldcg(e);
            ls[u] = __ldcg(e + 1);
            os[u] = __ldcg(e + 2 + d);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (ls[u] != 0.f) {
            const float mn = fmaxf(M[u], ms[u]);
            const float a = exp2f(M[u] - mn), b = exp2f(ms[u] - mn);
            L[u] = fmaf(L[u], a, ls[u] * b);
            O[u] = fmaf(O[u], a, os[u] * b);
            M[u] = mn;
          }
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float m2 = __shfl_xor_sync(0xffffffffu, M[u], o);
          const float l2 = __shfl_xor_sync(0xffffffffu, L[u], o);
          const float p2 = __shfl_xor_sync(0xffffffffu, O[u], o);
          const float mn = fmaxf(M[u], m2);
          const float a = L[u] != 0.f ? exp2f(M[u] - mn) : 0.f, b = l2 != 0.f ? exp2f(m2 - mn) : 0.f;
          L[u] = fmaf(L[u], a, l2 * b);
          O[u] = fmaf(O[u], a, p2 * b);
          M[u] = mn;
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int out = out0 + u * kDW;
          if (out >= o1) break;
          const float val = O[u] / L[u];
          outp[out] = val;
          if (p.trace) p.trace[(size_t)layer * p.trace_stride + HQ + 2 * KVH * kHD + out] = val;
        }
      }
    }
  };

  // ---- the stages: one call site per kind of work
  for (int si = p.first; si <= p.last && ok; ++si) {
    const int layer = si / 5, st = si % 5;
    if (st == 1) {
      ok = cta_and(attention_stage(layer)) && grid_sync(ctl, epoch, s_flag);
      if (ok) combine_stage(layer);
    } else {
      image_stage(si);
      ok = cta_and(gemv_stage(dec_gemv_of(si)));
    }
    ok = ok && grid_sync(ctl, epoch, s_flag);
  }

  // ---- the residual stream after the last stage run (CTA 0)
  if (ok && cta == 0) {
    const int layer = p.last / 5, st = p.last % 5;
    if (st == 2 || st == 4) {
      const int gt = st == 2 ? 1 : 3;
      const float sw = tensor_scale(layer, st == 2 ? 3 : 6), sx = s_scale[gt];
      for (int w = tid; w < D / 4; w += kDT) {
        int4 r = make_int4(0, 0, 0, 0);
        for (int s = 0; s < p.st[gt].splits; ++s) r = add_i4(r, ldcg_i4(part_ptr(gt, 0, 4 * w) + 32 * s));
        reinterpret_cast<float4*>(p.h_out)[w] = add_f4(reinterpret_cast<const float4*>(h)[w], i4_to_f4_scaled(r, sw, sx));
      }
    } else {
      for (int i = tid; i < D; i += kDT) p.h_out[i] = h[i];
    }
  }
  // ---- the last CTA out resets the barrier counters for the next launch
  named_sync();
  if (tid == 0 && ok) {
    __threadfence();
    if (atomicAdd(&ctl->exitc, 1u) == (unsigned)G - 1u) {
      ctl->bar = 0u;
      ctl->exitc = 0u;
    }
  }
}

}  // namespace

size_t decode_smem_bytes(const DecParams& p) { return dec_smem(p).total; }
int decode_ring_slots(const DecParams& p) { return dec_smem(p).nslot; }

int launch_decode(const DecParams& p, void* stream) {
  const DecSmem sp = dec_smem(p);
  // 4-element words of the widest stage input per consumer thread
  const int nw = (p.vmax / 4 + kDT - 1) / kDT;
  auto kern = nw <= 4 ? decode_kernel<4> : decode_kernel<7>;
  if (nw > 7) return -1;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
  if (e != cudaSuccess) return (int)e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kDBlock, sp.total);
  if (e != cudaSuccess) return (int)e;
  if (occ < 1) return -1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid, 1, 1);
  cfg.blockDim = dim3(kDBlock, 1, 1);
  cfg.dynamicSmemBytes = sp.total;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace tern

// ======================================================================== host
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// host-only checks of the model description
tern_status decode_check_model(const tern_decode_model* m) {
  using namespace tern;
  if (!m || !m->packed) return TERN_EINVAL;
  const int D = m->hidden, F = m->inter, H = m->heads, KVH = m->kv_heads;
  if (m->layers < 1 || m->layers > kDecMaxLayers || m->head_dim != kDecHeadDim) return TERN_EINVAL;
  if (D < 64 || F < 64 || D % 64 || F % 64 || H < 1 || KVH < 1 || KVH > kDecMaxKvHeads || H % KVH) return TERN_EINVAL;
  if (H / KVH > kDecMaxRep || D > kDecMaxVec || F > kDecMaxVec || H * kDecHeadDim > kDecMaxVec) return TERN_EINVAL;
  if (m->max_pos < 1 || !(m->eps >= 0.f) || !std::isfinite(m->eps)) return TERN_EINVAL;
  if (!m->d_gains || !m->d_kcache || !m->d_vcache || !m->d_rope) return TERN_EINVAL;
  return TERN_OK;
}

// the decode model's stages and workspace layout for `grid` CTAs
tern_status decode_plan(const tern_decode_model* m, int grid, tern::DecParams* p) {
  using namespace tern;
  if (!p) return TERN_EINVAL;
  const tern_status chk = decode_check_model(m);
  if (chk != TERN_OK) return chk;
  const int D = m->hidden, F = m->inter, H = m->heads, KVH = m->kv_heads;
  if (grid < KVH) return TERN_EUNSUPPORTED;
  std::memset(p, 0, sizeof(*p));
  const int HQ = H * kDecHeadDim, KQ = KVH * kDecHeadDim;
  p->layers = m->layers;
  p->D = D;
  p->F = F;
  p->H = H;
  p->KVH = KVH;
  p->max_pos = m->max_pos;
  p->eps = m->eps;
  p->grid = grid;
  p->ns = grid / KVH;
  p->gain_stride = 2 * D + HQ + F;
  p->trace_stride = 2 * HQ + 2 * KQ;
  p->vmax = D > F ? D : F;
  if (HQ > p->vmax) p->vmax = HQ;
  const int rows[4][3] = {{HQ, KQ, KQ}, {D, 0, 0}, {F, F, 0}, {D, 0, 0}};
  const int nprob[4] = {3, 1, 2, 1};
  const int proj[4][3] = {{0, 1, 2}, {3, 0, 0}, {4, 5, 0}, {6, 0, 0}};
  const int kin[4] = {D, HQ, D, F};
  size_t off = 256;  // control words
  p->off_ctl = 0;
  for (int s = 0; s < 4; ++s) {
    DecStage& S = p->st[s];
    S.nprob = nprob[s];
    int t = 0;
    for (int q = 0; q < S.nprob; ++q) {
      S.proj[q] = proj[s][q];
      S.tile0[q] = t;
      t += (rows[s][q] + kTileRows - 1) / kTileRows;
    }
    S.tile0[S.nprob] = t;
    S.cols = kin[s] / 64;
    // Tiles are cut into column ranges only when fewer than half the CTAs
    // would get a tile: each further range costs every consumer one more
    // round of L2 loads, more than the columns it takes off the busiest CTA.
    // Otherwise the fewest ranges that minimise the busiest CTA's columns.
    int best = 0;
    long long best_cols = 0;
    for (int sp = 1; sp <= kDecMaxSplits && sp <= S.cols && (sp == 1 || 2 * t < grid); ++sp) {
      const long long per = ((long long)t * sp + grid - 1) / grid;
      const long long mc = per * ((S.cols + sp - 1) / sp);
      if (per <= kDecMaxPartsPerCta && (best == 0 || mc < best_cols)) {
        best = sp;
        best_cols = mc;
      }
    }
    if (best == 0) return TERN_EUNSUPPORTED;
    S.splits = best;
    S.parts = t * best;
    p->off_part[s] = off;
    off += ((size_t)S.parts * 32 * 4 + 255) / 256 * 256;
  }
  p->off_att = off;
  off += ((size_t)KVH * p->ns * (H / KVH) * (kDecHeadDim + 2) * 4 + 255) / 256 * 256;
  p->off_attn = off;
  off += ((size_t)HQ * 4 + 255) / 256 * 256;
  p->ws_bytes = off;
  return TERN_OK;
}

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

}  // namespace

extern "C" tern_status tern_decode_rope_table(int32_t max_pos, int32_t head_dim, double theta, float* out) {
  if (max_pos < 1 || head_dim < 2 || head_dim % 2 || !out || !(theta > 1.0) || !std::isfinite(theta))
    return TERN_EINVAL;
  const int half = head_dim / 2;
  for (int p = 0; p < max_pos; ++p)
    for (int i = 0; i < half; ++i) {
      const double ang = (double)p * std::pow(theta, -2.0 * i / head_dim);
      out[((size_t)p * half + i) * 2] = (float)std::cos(ang);
      out[((size_t)p * half + i) * 2 + 1] = (float)std::sin(ang);
    }
  return TERN_OK;
}

extern "C" tern_status tern_decode_workspace_size(const tern_decode_model* model, size_t* bytes) {
  if (!bytes) return TERN_EINVAL;
  const tern_status chk = decode_check_model(model);
  if (chk != TERN_OK) return chk;
  const int sms = device_sms();
  if (sms <= 0) return TERN_ECUDA;
  tern::DecParams p;
  const tern_status st = decode_plan(model, sms, &p);
  if (st != TERN_OK) return st;
  *bytes = p.ws_bytes;
  return TERN_OK;
}

extern "C" tern_status tern_decode_step(const tern_decode_model* model, int32_t pos, const float* d_h_in,
                                        float* d_h_out, int32_t first, int32_t last, const float* d_attn_in,
                                        float* d_trace, void* d_ws, size_t ws_bytes, void* stream) {
  using namespace tern;
  if (!model || !d_h_in || !d_h_out || !d_ws) return TERN_EINVAL;
  const tern_status chk = decode_check_model(model);
  if (chk != TERN_OK) return chk;
  if (pos < 0 || pos >= model->max_pos || first < 0 || first > last || last >= 5 * model->layers) return TERN_EINVAL;
  if (first % 5 == 1 || first % 5 == 4 || (first % 5 == 2 && !d_attn_in)) return TERN_EINVAL;
  for (int l = 0; l < model->layers; ++l)
    for (int j = 0; j < 7; ++j)
      if (!model->packed[l * 7 + j]) return TERN_EINVAL;
  const int sms = device_sms();
  if (sms <= 0) return TERN_ECUDA;
  DecParams* p = new DecParams;
  tern_status st = decode_plan(model, sms, p);
  const size_t need = p->ws_bytes;
  if (st == TERN_OK && ws_bytes < need) st = TERN_ENOSPACE;
  if (st == TERN_OK && ((reinterpret_cast<uintptr_t>(d_ws) & 255u) || !aligned16(model->d_kcache) ||
                        !aligned16(model->d_vcache)))
    st = TERN_EALIGN;
  for (int l = 0; st == TERN_OK && l < model->layers; ++l)
    for (int j = 0; j < 7; ++j) {
      const void* q = model->packed[l * 7 + j];
      if (!aligned16(q)) st = TERN_EALIGN;
      else p->packed[l][j] = static_cast<const uint8_t*>(q);
    }
  if (st != TERN_OK) {
    delete p;
    return st;
  }
  p->gains = model->d_gains;
  p->kc = model->d_kcache;
  p->vc = model->d_vcache;
  p->rope = model->d_rope;
  p->h_in = d_h_in;
  p->h_out = d_h_out;
  p->attn_in = d_attn_in;
  p->trace = d_trace;
  p->ws = static_cast<uint8_t*>(d_ws);
  p->pos = pos;
  p->first = first;
  p->last = last;
  const int rc = launch_decode(*p, stream);
  delete p;
  if (rc < 0) return TERN_EUNSUPPORTED;
  return rc == 0 ? TERN_OK : TERN_ECUDA;
}
