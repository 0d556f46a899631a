// Persistent decode step of a BitNet b1.58 transformer (QORA-LLM-2B page,
// "Architecture" and "SubLN Pattern (4 norms per layer)"): every layer of one
// token in one cooperative launch, one CTA per SM.
//
// Per layer, five stages separated by grid-wide barriers:
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
// column ranges ("parts"; S chosen so that there are at least as many parts
// as CTAs), are dealt to the CTAs in contiguous runs. A part's exact int32 row
// sums go to its own slot of the workspace, and a consumer adds a row's S
// slots in order, so results do not depend on timing and nothing needs
// clearing between steps. Weights stream through a ring of 4 KB shared-memory
// slots filled by a producer warp with bulk async copies: the producer walks
// this CTA's chunks of every stage of every layer in order and runs ahead of
// the consumers across the grid barriers (weights depend on no stage), so
// the next stages' weights land while a barrier, a normalisation or the
// attention is in progress.
//
// Attention: the positions of each KV head are cut into NS ranges, one per
// CTA; each CTA computes its query heads' partial softmax state (running
// maximum, sum, weighted values) over its positions and the last CTA to
// finish a KV head combines the NS states in range order. The cached keys and
// values of a CTA's range are requested at the start of S1, so that they land
// during the QKV GEMV.
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
constexpr int kChunkCols = 8;            // 64-k columns per ring slot
constexpr int kSlotBytes = kChunkCols * kPlaneColBytes;  // 4096
constexpr int kNV = kDecMaxVec / kDT;    // vector elements per consumer thread
constexpr int kKvPass = 32;              // cached positions per attention pass
constexpr int kHD = kDecHeadDim;         // 128
constexpr int kBarNamed = 1;             // named barrier of the consumer threads

static_assert(kDecMaxVec % kDT == 0, "vector split");

// ------------------------------------------------------------ shared plan
struct DecSmem {
  size_t full, empty, kvbar, misc, h, img, pre, kv, scr, sacc, ring, total;
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
  s.full = take(8 * kDecMaxSlots, 8);
  s.empty = take(8 * kDecMaxSlots, 8);
  s.kvbar = take(8, 8);
  s.misc = take(512, 16);                                   // reductions, flags, scales
  s.h = take(4 * (size_t)p.D, 16);                          // residual stream
  s.img = take((size_t)p.vmax, 16);                         // int8 image of a stage's input
  s.pre = take(4 * ((size_t)p.vmax / 64 + 1), 16);          // column prefix sums of the image
  s.kv = take(2 * (size_t)kKvPass * kHD * 2, 128);          // cached keys then values of one pass
  s.scr = take(4 * ((size_t)(kDecMaxRep + 2) * kHD + (size_t)kDW * (kHD + 2)), 16);  // attention: q/k/v, states
  s.sacc = take(4 * 32 * (size_t)kDecMaxPartsPerCta, 16);   // a stage's part row sums
  s.ring = take(0, 128);
  const size_t avail = kDecSmemBytes > s.ring ? kDecSmemBytes - s.ring : 0;
  s.nslot = (int)(avail / kSlotBytes);
  if (s.nslot > kDecMaxSlots) s.nslot = kDecMaxSlots;
  s.total = s.ring + (size_t)s.nslot * kSlotBytes;
  return s;
}

// parts [a, b) of stage type st for CTA c
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
// stage type of stage index si (0: qkv, -1: attention, 1: o, 2: gate/up, 3: down)
__host__ __device__ inline int dec_gemv_of(int si) {
  const int s = si % 5;
  return s == 0 ? 0 : (s == 1 ? -1 : s - 1);
}

// ------------------------------------------------------------ primitives
__device__ __forceinline__ void named_sync() { asm volatile("bar.sync %0, %1;" ::"n"(kBarNamed), "n"(kDT) : "memory"); }

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ float bf16_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ uint32_t f32_to_bf16_rn(float v) {
  const uint32_t b = __float_as_uint(v);
  return (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;
}

struct DecCtl {
  unsigned bar, exitc, abort, pad;
  unsigned att[kDecMaxKvHeads];
};

// Grid barrier over the consumer threads of every CTA (bounded). Returns false
// if a CTA gave up (timeout here or elsewhere).
__device__ bool grid_sync(DecCtl* ctl, unsigned& epoch, volatile int* s_ok) {
  named_sync();
  if (threadIdx.x == 0) {
    bool ok = ld_acquire_u32(&ctl->abort) == 0u;
    if (ok) {
      __threadfence();
      atomicAdd(&ctl->bar, 1u);
      const unsigned target = (epoch + 1u) * gridDim.x;
      const uint64_t t0 = global_timer_ns();
      for (uint32_t it = 0;; ++it) {
        if (ld_acquire_u32(&ctl->bar) >= target) break;
        if ((it & 15u) == 15u) {
          if (ld_acquire_u32(&ctl->abort) != 0u) {
            ok = false;
            break;
          }
          if (global_timer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_dev_error, TERN_DEVERR_TIMEOUT);
            atomicExch(&ctl->abort, 1u);
            ok = false;
            break;
          }
        }
        __nanosleep(20);
      }
      __threadfence();
    }
    *s_ok = ok ? 1 : 0;
  }
  ++epoch;
  named_sync();
  return *s_ok != 0;
}

__device__ void raise_abort(DecCtl* ctl) {
  atomicOr(&g_dev_error, TERN_DEVERR_TIMEOUT);
  atomicExch(&ctl->abort, 1u);
}

// Sum over the consumer threads in a fixed order (butterfly in the warp, then
// the warps' values in warp order): every CTA gets bit-identical results.
__device__ double block_sum_d(double v, double* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  named_sync();
  double s = 0.0;
#pragma unroll
  for (int w = 0; w < kDW; ++w) s += red[w];
  named_sync();
  return s;
}

__device__ unsigned block_max_u(unsigned v, unsigned* red) {
  v = __reduce_max_sync(0xffffffffu, v);
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  named_sync();
  unsigned m = 0;
#pragma unroll
  for (int w = 0; w < kDW; ++w) m = max(m, red[w]);
  named_sync();
  return m;
}

// ------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(kDBlock, 1) decode_kernel(const __grid_constant__ DecParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const DecSmem sp = dec_smem(p);
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
      mbar_init(&empty[i], 1);
    }
    mbar_init(kvbar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // ================================================== producer warp
  if (warp == kDW) {
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    unsigned n = 0;  // chunks issued
    bool ok = true;
    for (int si = p.first; si <= p.last && ok; ++si) {
      const int gt = dec_gemv_of(si);
      if (gt < 0) continue;
      const DecStage& S = p.st[gt];
      const int layer = si / 5;
      int pa, pb;
      dec_parts(S, cta, G, &pa, &pb);
      for (int part = pa; part < pb && ok; ++part) {
        int tile, c0, c1;
        dec_part_cols(S, part, &tile, &c0, &c1);
        const int q = dec_problem_of(S, tile);
        const uint8_t* tr = p.packed[layer][S.proj[q]] + kHeaderBytes;
        const int tt = tile - S.tile0[q];
        for (int c = c0; c < c1; c += kChunkCols) {
          const int nc = min(kChunkCols, c1 - c);
          const int slot = (int)(n % (unsigned)nslot);
          const unsigned round = n / (unsigned)nslot;
          if (round > 0 && !mbar_wait_bounded(&empty[slot], (round - 1u) & 1u)) {
            ok = false;
            break;
          }
          if (ld_acquire_u32(&ctl->abort) != 0u) {
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
    if (!ok) atomicExch(&ctl->abort, 1u);
    // every copy this warp issued has landed before the CTA can exit (bounded;
    // immediate on the normal path, where the consumers have used them all)
    const unsigned lo = n > (unsigned)nslot ? n - (unsigned)nslot : 0u;
    for (unsigned j = lo; j < n; ++j) (void)mbar_wait_bounded(&full[j % nslot], (j / nslot) & 1u);
    return;
  }

  // ================================================== consumer threads
  const int tid = threadIdx.x;
  float* h = reinterpret_cast<float*>(smem + sp.h);
  int8_t* img = reinterpret_cast<int8_t*>(smem + sp.img);
  int* pre = reinterpret_cast<int*>(smem + sp.pre);
  float* scr = reinterpret_cast<float*>(smem + sp.scr);
  int* sacc = reinterpret_cast<int*>(smem + sp.sacc);
  uint16_t* kvs = reinterpret_cast<uint16_t*>(smem + sp.kv);
  double* red_d = reinterpret_cast<double*>(smem + sp.misc);          // [16]
  unsigned* red_u = reinterpret_cast<unsigned*>(smem + sp.misc + 128); // [16]
  volatile int* s_flag = reinterpret_cast<volatile int*>(smem + sp.misc + 192);
  float* s_scale = reinterpret_cast<float*>(smem + sp.misc + 256);    // [4] the GEMV stages' s_x

  unsigned epoch = 0, nchunk = 0, kvphase = 0;
  bool ok = true, kv_pending = false;  // kv_pending: a copy of cached keys/values is in flight (thread 0)
  const int D = p.D, F = p.F, HQ = p.H * kHD, KVH = p.KVH, rep = p.H / p.KVH;
  const int ns = p.ns;

  for (int i = tid; i < D; i += kDT) h[i] = p.h_in[i];
  named_sync();

  // exact row sum of row n of problem q of GEMV stage gt (after the stage's barrier)
  auto row_sum = [&](int gt, int q, int n) -> int {
    const DecStage& S = p.st[gt];
    const int t = S.tile0[q] + (n >> 5);
    const int* P = reinterpret_cast<const int*>(p.ws + p.off_part[gt]) + ((size_t)t * S.splits) * 32 + (n & 31);
    int s = 0;
#pragma unroll
    for (int j = 0; j < kDecMaxSplits; ++j)
      if (j < S.splits) s += __ldcg(P + 32 * j);
    return s;
  };
  auto tensor_scale = [&](int layer, int proj) -> float {
    return __ldg(reinterpret_cast<const float*>(p.packed[layer][proj] + 28));
  };
  auto linear_out = [&](int gt, int q, int n, float sw) -> float {
    return __fmul_rn(__fmul_rn(__int2float_rn(row_sum(gt, q, n)), sw), s_scale[gt]);
  };

  // RMSNorm (gain g) and int8 quantisation of the n values produced by val(i);
  // the image and its column prefix sums go to shared memory, the scale to
  // s_scale[gt]
  auto build_image = [&](int n, const float* g, int gt, auto&& val) {
    float v[kNV];
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < kNV; ++j) {
      const int i = tid + j * kDT;
      v[j] = 0.f;
      if (i < n) {
        v[j] = val(i);
        ss += (double)v[j] * (double)v[j];
      }
    }
    const double tot = block_sum_d(ss, red_d);
    const float r = (float)(1.0 / sqrt(tot / (double)n + (double)p.eps));
    unsigned am = 0;
#pragma unroll
    for (int j = 0; j < kNV; ++j) {
      const int i = tid + j * kDT;
      if (i < n) {
        v[j] = __fmul_rn(__fmul_rn(v[j], r), __ldg(g + i));
        am = max(am, __float_as_uint(v[j]) & 0x7FFFFFFFu);
      }
    }
    const float a = __uint_as_float(block_max_u(am, red_u));
    const float inv = a > 0.f ? __fdiv_rn(127.0f, a) : 0.f;
#pragma unroll
    for (int j = 0; j < kNV; ++j) {
      const int i = tid + j * kDT;
      if (i < n) {
        int qv = 0;
        if (v[j] != 0.f) qv = max(-127, min(127, __float2int_rn(__fmul_rn(v[j], inv))));
        img[i] = (int8_t)qv;
      }
    }
    if (tid == 0) s_scale[gt] = a > 0.f ? __fdiv_rn(a, 127.0f) : 0.f;
    named_sync();
    const int cols = n / 64;
    for (int c = tid; c < cols; c += kDT) {
      const uint32_t a0 = smem_u32(img + 64 * c);
      int s = 0;
#pragma unroll
      for (int o = 0; o < 64; o += 16) {
        const uint4 w = lds128<0>(a0 + o);
        s = __dp4a((int)w.x, 0x01010101, s);
        s = __dp4a((int)w.y, 0x01010101, s);
        s = __dp4a((int)w.z, 0x01010101, s);
        s = __dp4a((int)w.w, 0x01010101, s);
      }
      pre[c + 1] = s;
    }
    named_sync();
    if (warp == 0) {
      int carry = 0;
      for (int base = 1; base <= cols; base += 32) {
        const int i = base + lane;
        int x = i <= cols ? pre[i] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += u;
        }
        if (i <= cols) pre[i] = x + carry;
        carry += __shfl_sync(0xffffffffu, x, 31);
      }
      if (lane == 0) pre[0] = 0;
    }
    named_sync();
  };

  // this CTA's parts of GEMV stage gt over the image: chunks from the ring,
  // exact row sums per part written to the workspace
  auto gemv_stage = [&](int gt) -> bool {
    const DecStage& S = p.st[gt];
    int pa, pb;
    dec_parts(S, cta, G, &pa, &pb);
    for (int i = tid; i < (pb - pa) * 32; i += kDT) sacc[i] = 0;
    named_sync();
    // the stage's chunks in order: chunk ci goes to warp ci % 16
    int ci = 0;
    bool good = true;
    for (int part = pa; part < pb; ++part) {
      int tile, c0, c1;
      dec_part_cols(S, part, &tile, &c0, &c1);
      for (int c = c0; c < c1; c += kChunkCols, ++ci) {
        if (ci % kDW != warp) continue;
        const unsigned n = nchunk + (unsigned)ci;
        const int slot = (int)(n % (unsigned)nslot);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[slot], (n / (unsigned)nslot) & 1u))) {
          good = false;
          break;
        }
        const int nc = min(kChunkCols, c1 - c);
        const uint32_t wb = smem_u32(ring + (size_t)slot * kSlotBytes) + lane * 16;
        int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
        for (int cc = 0; cc < nc; ++cc) {
          const uint4 w = lds128<0>(wb + cc * kPlaneColBytes);
          const uint32_t xa = smem_u32(img + 64 * (c + cc));
          const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int4 xv = u4_as_i4(lds128<0>(xa + 16 * k));
            const uint32_t Fd = lop3_ternary_digit(wd[k]);
            a0 = dp4a_ss((int)(Fd & 0x03030303u), xv.x, a0);
            a1 = dp4a_ss((int)(Fd & 0x0C0C0C0Cu), xv.y, a1);
            a2 = dp4a_ss((int)(Fd & 0x30303030u), xv.z, a2);
            a3 = dp4a_us(Fd & 0xC0C0C0C0u, xv.w, a3);
          }
        }
        // release the slot: reads done before the refill
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        const int fx = a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6);
        atomicAdd(&sacc[(part - pa) * 32 + lane], (pre[c + nc] - pre[c]) - fx);
      }
      if (!good) break;
    }
    nchunk += (unsigned)ci;
    if (!good) raise_abort(ctl);
    named_sync();
    int* P = reinterpret_cast<int*>(p.ws + p.off_part[gt]);
    for (int i = tid; i < (pb - pa) * 32; i += kDT) P[(size_t)pa * 32 + i] = sacc[i];
    return good;
  };

  // request the cached keys and values of this CTA's first attention pass of `layer`
  auto kv_request = [&](int layer) {
    if (cta >= KVH * ns || tid != 0) return;  // kv_pending: thread 0 only
    const int j = cta / ns, sp_ = cta - j * ns;
    const int npos = p.pos + 1;
    const int p0 = (int)((long long)npos * sp_ / ns);
    const int p1 = min((int)((long long)npos * (sp_ + 1) / ns), p.pos);  // cached rows only
    const int cnt = min(kKvPass, p1 - p0);
    if (cnt <= 0) return;
    kv_pending = true;
    const size_t row = ((size_t)(layer * KVH + j) * p.max_pos + p0) * kHD;
    const uint32_t bytes = (uint32_t)cnt * kHD * 2;
    mbar_arrive_expect_tx(kvbar, 2 * bytes);
    const uint64_t pol = policy_evict_first();
    bulk_g2s(kvs, p.kc + row, bytes, kvbar, pol);
    bulk_g2s(kvs + kKvPass * kHD, p.vc + row, bytes, kvbar, pol);
  };
  auto kv_wait = [&]() -> bool {
    const bool r = mbar_wait_bounded(kvbar, kvphase & 1u);
    ++kvphase;
    return r;
  };

  // attention of `layer` (stage S2)
  auto attention_stage = [&](int layer) -> bool {
    if (cta >= KVH * ns) return true;
    const int j = cta / ns, sp_ = cta - j * ns;
    const int npos = p.pos + 1;
    const int p0 = (int)((long long)npos * sp_ / ns);
    const int p1 = (int)((long long)npos * (sp_ + 1) / ns);
    float* qs = scr;                        // [rep][128] q heads, then k, v
    float* ks = scr + rep * kHD;
    float* vs = ks + kHD;
    const float sq = tensor_scale(layer, 0), sk = tensor_scale(layer, 1), sv = tensor_scale(layer, 2);
    for (int i = tid; i < (rep + 2) * kHD; i += kDT) {
      const int r = i / kHD, d = i - r * kHD;
      float val;
      if (r < rep)
        val = linear_out(0, 0, (j * rep + r) * kHD + d, sq);
      else if (r == rep)
        val = linear_out(0, 1, j * kHD + d, sk);
      else
        val = linear_out(0, 2, j * kHD + d, sv);
      scr[i] = val;
    }
    named_sync();
    // RoPE, rotate_half, on the query heads and the key: pair (i, i + 64)
    const float* cs = p.rope + (size_t)p.pos * kHD;  // [64][2] cos, sin
    for (int i = tid; i < (rep + 1) * (kHD / 2); i += kDT) {
      const int r = i / (kHD / 2), f = i - r * (kHD / 2);
      float* v = scr + r * kHD;
      const float c = __ldg(cs + 2 * f), s = __ldg(cs + 2 * f + 1);
      const float a = v[f], b = v[f + kHD / 2];
      v[f] = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
      v[f + kHD / 2] = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
    }
    named_sync();
    if (p.trace && sp_ == 0) {
      float* tr = p.trace + (size_t)layer * p.trace_stride;
      for (int i = tid; i < (rep + 2) * kHD; i += kDT) {
        const int r = i / kHD, d = i - r * kHD;
        const size_t o = r < rep ? (size_t)(j * rep + r) * kHD + d
                                 : (size_t)HQ + (size_t)(r - rep) * KVH * kHD + (size_t)j * kHD + d;
        tr[o] = scr[i];
      }
    }
    named_sync();
    // the new key and value: bf16 as stored, used from here on as the cache holds them
    for (int d = tid; d < kHD; d += kDT) {
      const uint32_t kb = f32_to_bf16_rn(ks[d]), vb = f32_to_bf16_rn(vs[d]);
      if (sp_ == ns - 1) {
        const size_t at = ((size_t)(layer * KVH + j) * p.max_pos + p.pos) * kHD + d;
        p.kc[at] = (uint16_t)kb;
        p.vc[at] = (uint16_t)vb;
      }
      ks[d] = bf16_to_f32(kb);
      vs[d] = bf16_to_f32(vb);
    }
    named_sync();
    // scores and running softmax: warp = (query head hh, position group pg)
    const int hh = warp >> 2, pg = warp & 3;
    const bool active = hh < rep;
    float qv[4] = {0.f, 0.f, 0.f, 0.f};
    if (active)
#pragma unroll
      for (int e = 0; e < 4; ++e) qv[e] = qs[hh * kHD + 4 * lane + e];
    float m = -INFINITY, l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    const float kScale = 0.08838834764831845f;  // 1/sqrt(128)
    auto visit = [&](const float* kv4, const float* vv4) {
      float part = qv[0] * kv4[0];
      part = fmaf(qv[1], kv4[1], part);
      part = fmaf(qv[2], kv4[2], part);
      part = fmaf(qv[3], kv4[3], part);
#pragma unroll
      for (int off = 16; off; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      const float sc = part * kScale;
      const float mn = fmaxf(m, sc);
      const float corr = expf(m - mn), pe = expf(sc - mn);
      l = fmaf(l, corr, pe);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = fmaf(o[e], corr, pe * vv4[e]);
      m = mn;
    };
    const int pc1 = min(p1, p.pos);  // cached positions of this range: [p0, pc1)
    bool good = true;
    for (int base = p0; base < pc1; base += kKvPass) {
      const int cnt = min(kKvPass, pc1 - base);
      if (base != p0) {
        // a further pass: issued and awaited here (long contexts)
        named_sync();
        if (tid == 0) {
          const size_t row = ((size_t)(layer * KVH + j) * p.max_pos + base) * kHD;
          const uint32_t bytes = (uint32_t)cnt * kHD * 2;
          mbar_arrive_expect_tx(kvbar, 2 * bytes);
          const uint64_t pol = policy_evict_first();
          bulk_g2s(kvs, p.kc + row, bytes, kvbar, pol);
          bulk_g2s(kvs + kKvPass * kHD, p.vc + row, bytes, kvbar, pol);
        }
      }
      kv_pending = false;
      good = __all_sync(0xffffffffu, kv_wait()) && good;
      if (!good) break;
      if (active) {
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
    }
    if (!good) {
      raise_abort(ctl);
      return false;
    }
    // the current position (in the last range)
    if (active && p1 == npos && pg == ((npos - 1 - p0) & 3)) visit(ks + 4 * lane, vs + 4 * lane);
    named_sync();
    // merge the four position groups of each query head
    float* st = scr + (rep + 2) * kHD;  // [16 warps][130]
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
        const float w = expf(e[0] - M);
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
    __threadfence();
    named_sync();
    if (tid == 0) *s_flag = atomicAdd(&ctl->att[j], 1u) == (unsigned)(ns - 1) ? 2 : 0;
    named_sync();
    if (*s_flag == 2) {
      __threadfence();
      float* out = reinterpret_cast<float*>(p.ws + p.off_attn);
      for (int i = tid; i < rep * kHD; i += kDT) {
        const int r = i / kHD, d = i - r * kHD;
        float M = -INFINITY;
        for (int s = 0; s < ns; ++s) {
          const float* e = Pa + ((size_t)(j * ns + s) * rep + r) * (kHD + 2);
          if (__ldcg(e + 1) != 0.f) M = fmaxf(M, __ldcg(e));
        }
        float L = 0.f, O = 0.f;
        for (int s = 0; s < ns; ++s) {
          const float* e = Pa + ((size_t)(j * ns + s) * rep + r) * (kHD + 2);
          const float ls = __ldcg(e + 1);
          if (ls == 0.f) continue;
          const float w = expf(__ldcg(e) - M);
          L = fmaf(ls, w, L);
          O = fmaf(__ldcg(e + 2 + d), w, O);
        }
        const float val = O / L;
        out[(size_t)(j * rep + r) * kHD + d] = val;
        if (p.trace) p.trace[(size_t)layer * p.trace_stride + HQ + 2 * KVH * kHD + (size_t)(j * rep + r) * kHD + d] = val;
      }
      named_sync();
      if (tid == 0) ctl->att[j] = 0u;
    }
    return true;
  };

  // ---- the stages
  for (int si = p.first; si <= p.last && ok; ++si) {
    const int layer = si / 5, st = si % 5;
    const float* gains = p.gains + (size_t)layer * p.gain_stride;
    if (st == 0) {
      if (si + 1 <= p.last) kv_request(layer);  // the attention of this layer is in the run
      const bool fresh = si == p.first;
      const float sd = fresh ? 0.f : tensor_scale(layer - 1, 6);
      // h += down(previous layer), unless the run starts here
      build_image(D, gains, 0, [&](int i) {
        float x = h[i];
        if (!fresh) {
          x = __fadd_rn(x, linear_out(3, 0, i, sd));
          h[i] = x;
        }
        return x;
      });
      ok = gemv_stage(0) && grid_sync(ctl, epoch, s_flag);
    } else if (st == 1) {
      // a run that starts at S2 is refused on the host
      ok = attention_stage(layer) && grid_sync(ctl, epoch, s_flag);
    } else if (st == 2) {
      const float* src = si == p.first ? p.attn_in : reinterpret_cast<const float*>(p.ws + p.off_attn);
      const bool ext = si == p.first;
      build_image(HQ, gains + D, 1, [&](int i) { return ext ? __ldg(src + i) : __ldcg(src + i); });
      ok = gemv_stage(1) && grid_sync(ctl, epoch, s_flag);
    } else if (st == 3) {
      const bool fresh = si == p.first;
      const float so = tensor_scale(layer, 3);
      build_image(D, gains + D + HQ, 2, [&](int i) {
        float x = h[i];
        if (!fresh) {
          x = __fadd_rn(x, linear_out(1, 0, i, so));
          h[i] = x;
        }
        return x;
      });
      ok = gemv_stage(2) && grid_sync(ctl, epoch, s_flag);
    } else {
      const float sg = tensor_scale(layer, 4), su = tensor_scale(layer, 5);
      build_image(F, gains + 2 * D + HQ, 3, [&](int i) {
        const float g = linear_out(2, 0, i, sg), u = linear_out(2, 1, i, su);
        const float r = g > 0.f ? g : 0.f;
        return __fmul_rn(__fmul_rn(r, r), u);
      });
      ok = gemv_stage(3) && grid_sync(ctl, epoch, s_flag);
    }
  }

  // ---- the residual stream after the last stage run (CTA 0)
  if (ok && cta == 0) {
    const int layer = p.last / 5, st = p.last % 5;
    if (st == 2 || st == 4) {
      const float sw = tensor_scale(layer, st == 2 ? 3 : 6);
      for (int i = tid; i < D; i += kDT) p.h_out[i] = __fadd_rn(h[i], linear_out(st == 2 ? 1 : 3, 0, i, sw));
    } else {
      for (int i = tid; i < D; i += kDT) p.h_out[i] = h[i];
    }
  }
  // ---- a copy of cached keys and values that an aborted run never awaited
  if (kv_pending) (void)mbar_wait_bounded(kvbar, kvphase & 1u);
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
  cudaError_t e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
  if (e != cudaSuccess) return (int)e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel, kDBlock, sp.total);
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
  return (int)cudaLaunchKernelEx(&cfg, decode_kernel, p);
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
    int sp = (grid + t - 1) / t;
    if (sp > S.cols) sp = S.cols;
    if (sp > kDecMaxSplits) sp = kDecMaxSplits;
    S.splits = sp;
    S.parts = t * sp;
    if ((S.parts + grid - 1) / grid > kDecMaxPartsPerCta) return TERN_EUNSUPPORTED;
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
