// extern "C" entry points: argument validation, launch planning and dispatch.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <cstdint>

#include "tern_internal.h"

namespace tern {
namespace {

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    return 148;
  }
  return sms;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int xmode_of(tern_act act) {
  return act == TERN_ACT_INT8 ? kXInt8 : act == TERN_ACT_BF16 ? kXBf16 : kXBf16Q8;
}

struct Plan2 {
  int ks, cps, wpc, stage_cols, nstage, cluster, grid_x;
  size_t ws_cnt_bytes, ws_part_bytes;
  bool ok;
};

// Launch plan of the 2-bit GEMV for problems that share K and format.
//  * K is split into `ks` ranges of whole scale groups so that about twelve
//    warps per SM have work (small layers are latency-bound; splitting K
//    spreads their bytes over all SMs), and so that the staged activations of
//    one split fit in shared memory;
//  * up to 16 splits reduce through a thread-block cluster; beyond that (huge
//    K only) a single problem reduces through the caller's workspace;
//  * each warp streams its range in stages of about 4 KB, up to 3 in flight
//    (small stages keep enough warps resident to hide the latency).
Plan2 plan_gemv2(const Layout& L, const int* row_tiles, int nprob, int m, int xmode, int sms, bool ws_ok) {
  Plan2 pl{};
  const bool tq = L.fmt == TERN_FMT_TQ;
  const bool bt3 = L.fmt == TERN_FMT_BT3;
  const int gc = (tq && L.group >= 64) ? L.group / 64 : 1;  // columns per group
  const int units = (L.cols + gc - 1) / gc;
  const int P = L.planes;
  const int colk = bt3 ? kColK3 : kColK2;                      // k per column
  const int colb = bt3 ? bt_col_bytes(P) : P * kPlaneColBytes;  // bytes per column of a row tile
  const int mt = bt3 ? gemv3_mt(m) : gemv2_mt(xmode, m);
  int rt_total = 0;
  for (int i = 0; i < nprob; ++i) rt_total += row_tiles[i];
  pl.wpc = 4;
  const int sc_target = std::max(gc, (4096 / colb) / gc * gc);
  const int ks_par = std::min(units, std::max(1, (12 * sms + rt_total - 1) / rt_total));
  // staged bytes per k (bf16: the 24-bit image; balanced ternary: one per token)
  const int bpk = xmode == kXInt8 ? mt : xmode == kXBf16Q8 ? 3 * mt : (bt3 ? 3 * mt : 3);
  int ks_x = 1;
  while (ks_x < units && (size_t)((units + ks_x - 1) / ks_x) * gc * colk * bpk > 96 * 1024) ++ks_x;
  int ks = std::max(ks_par, ks_x);
  const size_t elem = (xmode != kXBf16 && tq) ? 8 : 4;
  if (bt3 && ks_x > kMaxCluster) {
    pl.ok = false;
    return pl;
  }
  if (ks > kMaxCluster && ks_x <= kMaxCluster) ks = kMaxCluster;
  pl.cluster = 0;
  if (ks > 1 && ks <= kMaxCluster) {
    while ((size_t)ks * mt * pl.wpc * 32 * elem > 32 * 1024 && pl.wpc > 1) pl.wpc /= 2;
    if ((size_t)ks * mt * pl.wpc * 32 * elem <= 32 * 1024) pl.cluster = 1;
  }
  if (ks > 1 && !pl.cluster && (!ws_ok || nprob != 1 || xmode == kXBf16Q8 || bt3)) {
    pl.ok = false;
    return pl;
  }
  pl.cps = ((units + ks - 1) / ks) * gc;
  pl.ks = (L.cols + pl.cps - 1) / pl.cps;
  if (pl.ks == 1) pl.cluster = 0;
  pl.stage_cols = std::min(sc_target, pl.cps);
  pl.nstage = std::min(3, (pl.cps + pl.stage_cols - 1) / pl.stage_cols);
  // fit shared memory: fewer stages in flight, then fewer warps per CTA
  for (;;) {
    Gemv2Params t{};
    t.tq = tq;
    t.k = L.k;
    t.planes = P;
    t.group = L.group;
    t.groups = L.groups;
    t.cols = L.cols;
    t.m = m;
    t.ks = pl.ks;
    t.cluster = pl.cluster;
    t.cols_per_split = pl.cps;
    t.wpc = pl.wpc;
    t.stage_cols = pl.stage_cols;
    t.nstage = pl.nstage;
    if ((bt3 ? gemv3_smem_bytes(t) : gemv2_smem_bytes(t, xmode)) <= 227 * 1024) break;
    if (pl.nstage > 2) {
      --pl.nstage;
    } else if (pl.wpc > 1) {
      pl.wpc /= 2;
    } else {
      pl.ok = false;
      return pl;
    }
  }
  pl.grid_x = 0;
  for (int i = 0; i < nprob; ++i) pl.grid_x += (row_tiles[i] + pl.wpc - 1) / pl.wpc;
  if (pl.ks > 1 && !pl.cluster) {
    pl.ws_cnt_bytes = ((size_t)pl.grid_x * 4 + 255) / 256 * 256;
    pl.ws_part_bytes = (size_t)pl.ks * m * row_tiles[0] * kTileRows * elem;
  }
  pl.ok = true;
  return pl;
}

// Plan of the single-token kernel with one CTA per SM (gemv2w): tile ranges
// of equal column counts per CTA (gemv2w_cta_tile), 4-6 KB stages, as many
// warps and stages in flight as shared memory allows next to the resident
// activation images. Applies when the launch has at least four tiles per SM
// (smaller launches are spread over the SMs by K splits in the row-group
// kernel), or one tile per SM with bf16 activations: there the exact 24-bit
// image makes the launch compute-bound, and sixteen warps on whole tiles beat
// the K-split kernel (a dependent TQ3P / d = 3 launch of 14336x4096, 448
// tiles: 19.6 / 29.9 us against 22.6 / 35.3 us; at 128 tiles the K split
// stays faster).
// With mt > 1 tokens (one problem, integer activations) a launch of half a
// tile per SM is enough: each tile carries mt tokens' work. L is the layout of
// the widest problem (its K sizes the activation images); prob_cols gives
// each problem's column count when K differs between problems (else NULL).
bool plan_gemv2w(const Layout& L, const int* row_tiles, int nprob, int xmode, int sms, Gemv2wParams& p,
                 int mt = 1, const int* prob_cols = nullptr) {
  const bool bt3 = L.fmt == TERN_FMT_BT3;
  if (bt3 && (xmode != kXBf16 || L.planes != 3)) return false;  // d = 2, 4: the row-group kernel
  if (nprob > kMaxProblemsW) return false;
  if (mt > 1 && (nprob != 1 || bt3 || xmode == kXBf16 || mt > kMaxTokensW)) return false;
  int begin[kMaxProblemsW + 1];
  long long cbeg[kMaxProblemsW + 1];
  begin[0] = 0;
  cbeg[0] = 0;
  for (int i = 0; i < nprob; ++i) {
    begin[i + 1] = begin[i] + row_tiles[i];
    cbeg[i + 1] = cbeg[i] + (long long)row_tiles[i] * (prob_cols ? prob_cols[i] : L.cols);
  }
  const int T = begin[nprob];
  if (T < (mt > 1 ? (sms + 1) / 2 : (xmode == kXBf16 ? sms : 4 * sms))) return false;
  p.mt = mt;
  // the kernel's index arithmetic is 32-bit: all columns, and a CTA's columns
  // x warps, stay below 2^31
  if (cbeg[nprob] * 16 >= (1ll << 31) || (cbeg[nprob] / sms + L.cols) * 16 >= (1ll << 31)) return false;
  const bool tq = L.fmt == TERN_FMT_TQ;
  p.tq = tq;
  p.k = L.k;
  p.planes = L.planes;
  p.group = L.group;
  p.groups = L.groups;
  p.cols = L.cols;
  p.bt3 = bt3;
  p.gcols = (tq && L.group >= 64) ? L.group / 64 : 1;
  p.nprob = nprob;
  p.tiles_total = T;
  p.grid = std::min(sms, T);
  for (int i = 0; i <= nprob; ++i) {
    p.tile_begin[i] = begin[i];
    p.col_begin[i] = (int)cbeg[i];
  }
  auto prob_of = [&](int t) {
    int q = 0;
    while (q + 1 < nprob && t >= begin[q + 1]) ++q;
    return q;
  };
  // CTA tile ranges balance columns (the kernel computes the same ones); every
  // CTA needs at least one tile
  int xs = 1;
  for (int c = 0; c < p.grid; ++c) {
    const int t0 = gemv2w_cta_tile(p.tile_begin, p.col_begin, nprob, c, p.grid);
    const int t1 = gemv2w_cta_tile(p.tile_begin, p.col_begin, nprob, c + 1, p.grid);
    if (t1 <= t0) return false;
    xs = std::max(xs, prob_of(t1 - 1) - prob_of(t0) + 1);
  }
  if (xs > kMaxSlotsW) return false;
  p.xslots = xs;
  const int colb = bt3 ? kBt3ColBytes : L.planes * kPlaneColBytes;
  // (warps, stages, stage bytes): sixteen warps with two stages each, the
  // stages as large as shared memory allows next to the activation images.
  // Every stage costs the warp a fixed ~115 instructions (barrier wait, copy
  // issue, stage bookkeeping; ncu instruction counts per 16-k word at 3, 4 and
  // 5.5 KB stages), so larger stages cut instructions per weight: on the
  // BitNet-2B layer set (whose images leave no room for 6 KB) 5.5 KB stages
  // took 169k SM cycles per step against 186k with 4 KB. Three stages of
  // 3.5 KB, or twelve warps with 7.5 KB stages, were slower. Smaller stages
  // and then fewer warps serve long K.
  static const int kShapes[][3] = {{16, 2, 6144}, {16, 2, 5632}, {16, 2, 5120}, {16, 2, 4096},
                                   {16, 2, 3072}, {12, 2, 4096}, {8, 3, 4096},  {8, 2, 4096},
                                   {4, 3, 4096},  {4, 2, 4096}};
  for (const auto& sh : kShapes) {
    p.nw = sh[0];
    p.nstage = sh[1];
    p.stage_cols = std::max(p.gcols, (sh[2] / colb) / p.gcols * p.gcols);
    // the kernel adds its shared copy of the parameter block's head and of
    // its problems
    if (gemv2w_smem_bytes(p, xmode) + offsetof(Gemv2wParams, prob) + sizeof(Gemv2wProblem) * kMaxSlotsW <=
        227 * 1024)
      return true;
  }
  return false;
}

// Plan of the tensor-core batched GEMM (int8 tokens padded to 16, 2-bit formats)
// for one launch of up to kTcMaxTokens tokens. The digit count D of the scales
// is read by the kernel from the packed header, so the token passes and the
// activation slot are sized here for every D the kernel may meet.
// Workspace: arrival counters [tiles][4] | int64 partial sums [256][n_pad]
// (both zero on entry and left zero; sized and placed for the largest launch,
// so that calls with any token count can share one workspace) | activations
// in MMA order | (bf16 input) int8 activations and their scales.
struct PlanTc {
  GemmTcParams p;
  int kchunks, mp;  // 16-k chunks; the largest passes x tokens per pass
  size_t cnt_off, part_off, xp_off, xq_off, sx_off, total;
  bool ok;
};

PlanTc plan_tc(const Layout& L, int mb, int xmode, int sms) {
  PlanTc t{};
  const bool tq = L.fmt == TERN_FMT_TQ;
  if (L.fmt == TERN_FMT_BT3 || (xmode != kXInt8 && xmode != kXBf16Q8) || mb < 1 || mb > kTcMaxTokens) return t;
  // every digit accumulator stays below 2^31: 127 * 127 * K (the planes share
  // one int8 operand); the kernel's positions (128-row tiles x token passes x
  // columns) fit in 31 bits
  if ((long long)127 * 127 * L.k >= (1ll << 31)) return t;
  if ((long long)(L.row_tiles + 3) / 4 * kTcMaxMerged * L.cols >= (1ll << 31)) return t;
  GemmTcParams& p = t.p;
  p.tq = tq;
  p.n = L.n;
  p.k = L.k;
  p.planes = L.planes;
  p.group = tq ? L.group : 0;
  p.cols = L.cols;
  p.row_tiles = L.row_tiles;
  p.tiles = (L.row_tiles + 3) / 4;
  p.n_pad = p.tiles * kTcRows;
  p.m = mb;
  p.m16 = (mb + 15) & ~15;
  // every digit count the header may hold must have a shared-memory plan
  int mp = 0, pcap = 0;
  for (int d7 = 1; d7 <= (tq ? kTcMaxDigits : 1); ++d7) {
    int ps, tp;
    const int dm = tc_merged_digits(L.planes, d7);
    tc_passes(dm, p.m16, &ps, &tp);
    TcLayout lay;
    if (!tc_layout(L.planes, tq, p.group, dm, tp, &lay)) return t;
    mp = std::max(mp, ps * tp);
    pcap = std::max(pcap, ps);
  }
  t.mp = mp;
  p.passes_cap = pcap;
  p.grid = (int)std::min<long long>(sms, (long long)p.tiles * p.cols);
  t.kchunks = L.cols * 4;
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) / 256 * 256;
    return o;
  };
  int pmax = 0, tdummy = 0;
  tc_passes(kTcMaxMerged, kTcMaxTokens, &pmax, &tdummy);
  t.cnt_off = take((size_t)p.tiles * pmax * 4);
  t.part_off = take((size_t)kTcMaxTokens * p.n_pad * 8);
  t.xp_off = take((size_t)t.kchunks * mp * 16);
  if (xmode == kXBf16Q8) {
    t.xq_off = take((size_t)mb * L.k);
    t.sx_off = take((size_t)mb * 4);
  }
  t.total = off;
  t.ok = true;
  return t;
}

tern_status check_one(const tern_desc* desc, const void* d_packed, tern_act act, const void* d_x,
                      const float* d_xscale, tern_out out, void* d_y, Layout* L) {
  tern_status st = layout_of(desc, L);
  if (st != TERN_OK) return st;
  if (!d_packed || !d_x || !d_y) return TERN_EINVAL;
  if (act != TERN_ACT_INT8 && act != TERN_ACT_BF16 && act != TERN_ACT_BF16_Q8) return TERN_EINVAL;
  if (out != TERN_OUT_F32 && out != TERN_OUT_BF16) return TERN_EINVAL;
  if (act == TERN_ACT_INT8 && !d_xscale) return TERN_EINVAL;
  if (!aligned16(d_packed)) return TERN_EALIGN;
  if ((reinterpret_cast<uintptr_t>(d_y) & 3u) != 0) return TERN_EALIGN;
  return TERN_OK;
}

// What the kernels support for this layout and activation mode.
tern_status supported_2bit(const Layout& L, int xmode) {
  const bool tq = L.fmt == TERN_FMT_TQ;
  // balanced ternary: bf16 activations (depth 3 on both kernels, 2 and 4 on the row-group kernel)
  if (L.fmt == TERN_FMT_BT3) return xmode == kXBf16 ? TERN_OK : TERN_EUNSUPPORTED;
  if (xmode == kXBf16 && !tq) return TERN_EUNSUPPORTED;
  if (tq && L.k % kColK2 != 0) return TERN_EUNSUPPORTED;
  if (!tq && (long long)L.k * 127 >= (1ll << 24)) return TERN_EUNSUPPORTED;  // exact int32 -> fp32
  return TERN_OK;
}

void fill_common(Gemv2Params& p, const Layout& L, const Plan2& pl, int m, tern_out out) {
  p.tq = L.fmt == TERN_FMT_TQ;
  p.k = L.k;
  p.planes = L.planes;
  p.group = L.group;
  p.groups = L.groups;
  p.cols = L.cols;
  p.m = m;
  p.out_bf16 = out == TERN_OUT_BF16;
  p.ks = pl.ks;
  p.cluster = pl.cluster;
  p.cols_per_split = pl.cps;
  p.wpc = pl.wpc;
  p.stage_cols = pl.stage_cols;
  p.nstage = pl.nstage;
  p.grid_x = pl.grid_x;
}

tern_status run_single(const tern_desc* desc, const Layout& L, const void* d_packed, int m, tern_act act,
                       const void* d_x, const float* d_xscale, tern_out out, void* d_y, void* d_ws, size_t ws_bytes,
                       void* stream) {
  const int xmode = xmode_of(act);
  tern_status st = supported_2bit(L, xmode);
  if (st != TERN_OK) return st;
  const int sms = device_sms();
  const uint8_t* base = static_cast<const uint8_t*>(d_packed);
  const bool pdl = (desc->flags & TERN_F_PDL) != 0;
  // tensor cores from 16 tokens, and from 9 when a workspace is given (the
  // CUDA-core path below takes more than eight tokens in two passes, slower
  // than one tensor-core launch padded to 16 tokens); also from 5 when the
  // CUDA-core pass's activation images leave room for fewer than 16 warps
  // (long K)
  bool use_tc = m >= 16 || (m >= 9 && d_ws);
  if (!use_tc && m >= 2 && d_ws && xmode != kXBf16 && L.fmt != TERN_FMT_BT3) {
    if (!gemv2w_mt_has_kernel(L.planes, L.fmt == TERN_FMT_TQ, L.group)) {
      use_tc = true;  // no CUDA-core kernel for several tokens of this plane count and group size
    } else if (m >= 5) {
      Gemv2wParams w{};
      const int rt = L.row_tiles;
      use_tc = plan_gemv2w(L, &rt, 1, xmode, sms, w, std::min(m, kMaxTokensW)) && w.nw < 16;
    }
  }
  if (use_tc) {
    const int mb = std::min(m, kTcMaxTokens);
    const PlanTc tp = plan_tc(L, mb, xmode, sms);
    if (tp.ok) {
      if (!d_ws || ws_bytes < tp.total) return TERN_ENOSPACE;
      if ((reinterpret_cast<uintptr_t>(d_ws) & 255u) != 0) return TERN_EALIGN;
      uint8_t* ws = static_cast<uint8_t*>(d_ws);
      const size_t in_elem = xmode == kXInt8 ? 1 : 2;
      const size_t out_elem = out == TERN_OUT_F32 ? 4 : 2;
      for (int t0 = 0; t0 < m; t0 += kTcMaxTokens) {
        const int mc = std::min(kTcMaxTokens, m - t0);
        PlanTc pc = plan_tc(L, mc, xmode, sms);
        if (!pc.ok) return TERN_EUNSUPPORTED;
        GemmTcParams& p = pc.p;
        const uint8_t* xin = static_cast<const uint8_t*>(d_x) + (size_t)t0 * L.k * in_elem;
        const int8_t* xq = reinterpret_cast<const int8_t*>(xin);
        const float* sx = d_xscale ? d_xscale + t0 : nullptr;
        if (xmode == kXBf16Q8) {
          xq = reinterpret_cast<const int8_t*>(ws + pc.xq_off);
          sx = reinterpret_cast<const float*>(ws + pc.sx_off);
          if (launch_quantize(reinterpret_cast<const uint16_t*>(xin), mc, L.k, const_cast<int8_t*>(xq),
                              const_cast<float*>(sx), stream) != 0)
            return TERN_ECUDA;
        }
        p.trit = base + L.trit_offset;
        p.scale = p.tq ? reinterpret_cast<const uint16_t*>(base + L.scale_offset) : nullptr;
        p.header = base;
        if (launch_tc_prep_x(xq, mc, L.k, pc.kchunks, pc.kchunks * pc.mp, p, ws + pc.xp_off, stream) != 0)
          return TERN_ECUDA;
        p.xp = ws + pc.xp_off;
        p.xscale = sx;
        p.y = static_cast<uint8_t*>(d_y) + (size_t)t0 * L.n * out_elem;
        p.part = reinterpret_cast<unsigned long long*>(ws + pc.part_off);
        p.cnt = reinterpret_cast<unsigned*>(ws + pc.cnt_off);
        p.out_bf16 = out == TERN_OUT_BF16;
        p.tensor_scale = desc->tensor_scale;
        const int rc = launch_gemm_tc(p, stream);
        if (rc < 0) return TERN_EUNSUPPORTED;
        if (rc != 0) return TERN_ECUDA;
      }
      return TERN_OK;
    }
  }
  if (m == 1) {
    Gemv2wParams w{};
    const int rt = L.row_tiles;
    if (plan_gemv2w(L, &rt, 1, xmode, sms, w)) {
      w.out_bf16 = out == TERN_OUT_BF16;
      Gemv2wProblem& q = w.prob[0];
      q.trit = base + L.trit_offset;
      q.scale = w.tq ? reinterpret_cast<const uint16_t*>(base + L.scale_offset) : nullptr;
      q.x = d_x;
      q.xscale = d_xscale;
      q.y = d_y;
      q.n = L.n;
      q.row_tiles = L.row_tiles;
      q.tensor_scale = desc->tensor_scale;
      q.k = L.k;
      q.cols = L.cols;
      q.groups = L.groups;
      w.x_vec = aligned16(d_x) && L.k % 16 == 0;
      const int rc = launch_gemv2w(w, xmode, pdl, stream);
      if (rc >= 0) return rc == 0 ? TERN_OK : TERN_ECUDA;
      // no kernel for this plane count and group size: the row-group kernel below
    }
  }
  const size_t in_elem = xmode == kXInt8 ? 1 : 2;
  const size_t out_elem = out == TERN_OUT_F32 ? 4 : 2;
  if (m >= 2 && xmode != kXBf16 && L.fmt != TERN_FMT_BT3) {
    // several tokens on the one-CTA-per-SM kernel, up to eight per pass over
    // the weights (more tokens: passes of near-equal size, at least two
    // tokens each), when the layer has half a tile per SM and the images fit
    Gemv2wParams w{};
    const int rt = L.row_tiles;
    const int passes = (m + kMaxTokensW - 1) / kMaxTokensW;
    if (plan_gemv2w(L, &rt, 1, xmode, sms, w, (m + passes - 1) / passes)) {
      for (int c = 0, t0 = 0; c < passes; ++c) {
        const int mc = (m - t0) / (passes - c);
        if (mc != w.mt && !plan_gemv2w(L, &rt, 1, xmode, sms, w, mc)) return TERN_EUNSUPPORTED;
        w.out_bf16 = out == TERN_OUT_BF16;
        Gemv2wProblem& q = w.prob[0];
        q.trit = base + L.trit_offset;
        q.scale = w.tq ? reinterpret_cast<const uint16_t*>(base + L.scale_offset) : nullptr;
        q.x = static_cast<const uint8_t*>(d_x) + (size_t)t0 * L.k * in_elem;
        q.xscale = d_xscale ? d_xscale + t0 : nullptr;
        q.y = static_cast<uint8_t*>(d_y) + (size_t)t0 * L.n * out_elem;
        q.n = L.n;
        q.row_tiles = L.row_tiles;
        q.tensor_scale = desc->tensor_scale;
        q.k = L.k;
        q.cols = L.cols;
        q.groups = L.groups;
        w.x_vec = aligned16(q.x) && L.k % 16 == 0;
        const int rc = launch_gemv2w(w, xmode, pdl, stream);
        if (rc < 0 && c == 0) break;  // no kernel for this plane count and group size: the row-group kernel below
        if (rc < 0) return TERN_EUNSUPPORTED;
        if (rc != 0) return TERN_ECUDA;
        t0 += mc;
        if (c + 1 == passes) return TERN_OK;
      }
    }
  }
  // the row-group kernels: passes of up to 8 tokens (balanced ternary), 4 or
  // 16 (integer activations) or one (bf16 activations over 2-bit planes)
  const int mt_max = L.fmt == TERN_FMT_BT3 ? 8 : gemv2_mt(xmode, m);
  for (int t0 = 0; t0 < m; t0 += mt_max) {
    const int mc = std::min(mt_max, m - t0);
    const int rt = L.row_tiles;
    const Plan2 pl = plan_gemv2(L, &rt, 1, mc, xmode, sms, d_ws != nullptr);
    if (!pl.ok) return d_ws ? TERN_EUNSUPPORTED : TERN_ENOSPACE;
    if (pl.ks > 1 && !pl.cluster && ws_bytes < pl.ws_cnt_bytes + pl.ws_part_bytes) return TERN_ENOSPACE;
    Gemv2Params p{};
    fill_common(p, L, pl, mc, out);
    p.nprob = 1;
    Gemv2Problem& q = p.prob[0];
    q.trit = base + L.trit_offset;
    q.scale = p.tq ? reinterpret_cast<const uint16_t*>(base + L.scale_offset) : nullptr;
    q.x = static_cast<const uint8_t*>(d_x) + (size_t)t0 * L.k * in_elem;
    q.xscale = d_xscale ? d_xscale + t0 : nullptr;
    q.y = static_cast<uint8_t*>(d_y) + (size_t)t0 * L.n * out_elem;
    q.n = L.n;
    q.row_tiles = L.row_tiles;
    q.cta_begin = 0;
    q.tensor_scale = desc->tensor_scale;
    p.x_vec = aligned16(q.x) && L.k % 16 == 0;
    if (pl.ks > 1 && !pl.cluster) {
      p.ws_cnt = static_cast<unsigned*>(d_ws);
      p.ws_part = static_cast<uint8_t*>(d_ws) + pl.ws_cnt_bytes;
    }
    const int rc = L.fmt == TERN_FMT_BT3 ? launch_gemv3(p, pdl, stream) : launch_gemv2(p, xmode, pdl, stream);
    if (rc < 0) return TERN_EUNSUPPORTED;
    if (rc != 0) return TERN_ECUDA;
  }
  return TERN_OK;
}

}  // namespace
}  // namespace tern

using namespace tern;

extern "C" tern_status tern_workspace_size(const tern_desc* desc, int32_t m, size_t* bytes) {
  if (!bytes) return TERN_EINVAL;
  Layout L;
  tern_status st = layout_of(desc, &L);
  if (st != TERN_OK) return st;
  if (m < 0) return TERN_EINVAL;
  const int sms = device_sms();
  size_t need = 0;
  if (m >= 2) {  // tensor-core paths (a few tokens: group accumulators; more: scale digits)
    for (int xmode = 0; xmode < 3; ++xmode) {
      const PlanTc tp = plan_tc(L, std::min<int>(m, kTcMaxTokens), xmode, sms);
      if (tp.ok) need = std::max(need, tp.total);
    }
  }
  if (L.fmt != TERN_FMT_BT3) {
    const int rt = L.row_tiles;
    for (int xmode = 0; xmode < 3; ++xmode) {
      const int mc = std::max(1, std::min(m, gemv2_mt(xmode, std::max(1, m))));
      const Plan2 pl = plan_gemv2(L, &rt, 1, mc, xmode, sms, true);
      if (pl.ok) need = std::max(need, pl.ws_cnt_bytes + pl.ws_part_bytes);
    }
  }
  *bytes = need;
  return TERN_OK;
}

extern "C" tern_status tern_quantize_act(const uint16_t* d_x_bf16, int32_t m, int32_t k, int8_t* d_xq,
                                         float* d_xscale, void* stream) {
  if (m < 0 || k < 1 || (m > 0 && (!d_x_bf16 || !d_xq || !d_xscale))) return TERN_EINVAL;
  return launch_quantize(d_x_bf16, m, k, d_xq, d_xscale, stream) == 0 ? TERN_OK : TERN_ECUDA;
}

extern "C" tern_status tern_gemm_batched(const tern_desc* desc, const void* d_packed, int32_t m, tern_act act,
                                         const void* d_x, const float* d_xscale, tern_out out, void* d_y, void* d_ws,
                                         size_t ws_bytes, void* stream) {
  Layout L;
  if (m < 1) return TERN_EINVAL;
  tern_status st = check_one(desc, d_packed, act, d_x, d_xscale, out, d_y, &L);
  if (st != TERN_OK) return st;
  return run_single(desc, L, d_packed, m, act, d_x, d_xscale, out, d_y, d_ws, ws_bytes, stream);
}

extern "C" tern_status tern_gemv(const tern_desc* desc, const void* d_packed, tern_act act, const void* d_x,
                                 const float* d_xscale, tern_out out, void* d_y, void* d_ws, size_t ws_bytes,
                                 void* stream) {
  return tern_gemm_batched(desc, d_packed, 1, act, d_x, d_xscale, out, d_y, d_ws, ws_bytes, stream);
}

extern "C" tern_status tern_gemv_grouped(int32_t count, const tern_desc* descs, const void* const* d_packed,
                                         tern_act act, const void* const* d_x, const float* const* d_xscale,
                                         tern_out out, void* const* d_y, void* stream) {
  if (count < 1 || count > kMaxProblemsW || !descs || !d_packed || !d_x || !d_y) return TERN_EINVAL;
  if (act == TERN_ACT_INT8 && !d_xscale) return TERN_EINVAL;
  static thread_local Layout L[kMaxProblemsW];
  int rt[kMaxProblemsW];
  for (int i = 0; i < count; ++i) {
    tern_status st = check_one(&descs[i], d_packed[i], act, d_x[i], d_xscale ? d_xscale[i] : nullptr, out, d_y[i],
                               &L[i]);
    if (st != TERN_OK) return st;
    // the group size matters for TQ only (BitNet: the whole row; d = 3: 16)
    if (L[i].fmt != L[0].fmt || L[i].planes != L[0].planes ||
        (L[0].fmt == TERN_FMT_TQ && L[i].group != L[0].group) || descs[i].flags != descs[0].flags)
      return TERN_EINVAL;
    rt[i] = L[i].row_tiles;
  }
  const int xmode = xmode_of(act);
  int widest = 0;  // the problem with the largest K sizes the activation images
  bool all_vec = true;
  for (int i = 0; i < count; ++i) {
    tern_status st = supported_2bit(L[i], xmode);
    if (st != TERN_OK) return st;
    if (L[i].k > L[widest].k) widest = i;
    all_vec = all_vec && L[i].k % 16 == 0;
  }
  const int sms = device_sms();
  const bool pdl = (descs[0].flags & TERN_F_PDL) != 0;
  {
    static thread_local Gemv2wParams w;
    w = Gemv2wParams{};
    int pcols[kMaxProblemsW];
    for (int i = 0; i < count; ++i) pcols[i] = L[i].cols;
    if (plan_gemv2w(L[widest], rt, count, xmode, sms, w, 1, pcols)) {
      w.out_bf16 = out == TERN_OUT_BF16;
      bool vec = all_vec;
      for (int i = 0; i < count; ++i) {
        const uint8_t* base = static_cast<const uint8_t*>(d_packed[i]);
        Gemv2wProblem& q = w.prob[i];
        q.trit = base + L[i].trit_offset;
        q.scale = w.tq ? reinterpret_cast<const uint16_t*>(base + L[i].scale_offset) : nullptr;
        q.x = d_x[i];
        q.xscale = d_xscale ? d_xscale[i] : nullptr;
        q.y = d_y[i];
        q.n = L[i].n;
        q.row_tiles = L[i].row_tiles;
        q.tensor_scale = descs[i].tensor_scale;
        q.k = L[i].k;
        q.cols = L[i].cols;
        q.groups = L[i].groups;
        vec = vec && aligned16(q.x);
      }
      w.x_vec = vec;
      const int rc = launch_gemv2w(w, xmode, pdl, stream);
      if (rc >= 0) return rc == 0 ? TERN_OK : TERN_ECUDA;
      // no kernel for this plane count and group size: the row-group kernel below
    }
  }
  // the row-group kernel takes up to kMaxProblems problems of one K per launch
  for (int c0 = 0, nc = 0; c0 < count; c0 += nc) {
    nc = 1;
    while (c0 + nc < count && nc < kMaxProblems && L[c0 + nc].k == L[c0].k) ++nc;
    const Plan2 pl = plan_gemv2(L[c0], rt + c0, nc, 1, xmode, sms, false);
    if (!pl.ok) return TERN_EUNSUPPORTED;
    Gemv2Params p{};
    fill_common(p, L[c0], pl, 1, out);
    p.nprob = nc;
    int cta = 0;
    bool vec = L[c0].k % 16 == 0;
    for (int j = 0; j < nc; ++j) {
      const int i = c0 + j;
      const uint8_t* base = static_cast<const uint8_t*>(d_packed[i]);
      Gemv2Problem& q = p.prob[j];
      q.trit = base + L[i].trit_offset;
      q.scale = p.tq ? reinterpret_cast<const uint16_t*>(base + L[i].scale_offset) : nullptr;
      q.x = d_x[i];
      q.xscale = d_xscale ? d_xscale[i] : nullptr;
      q.y = d_y[i];
      q.n = L[i].n;
      q.row_tiles = L[i].row_tiles;
      q.cta_begin = cta;
      q.tensor_scale = descs[i].tensor_scale;
      cta += (L[i].row_tiles + pl.wpc - 1) / pl.wpc;
      vec = vec && aligned16(q.x);
    }
    p.x_vec = vec;
    const int rc = L[0].fmt == TERN_FMT_BT3 ? launch_gemv3(p, pdl, stream) : launch_gemv2(p, xmode, pdl, stream);
    if (rc < 0) return TERN_EUNSUPPORTED;
    if (rc != 0) return TERN_ECUDA;
  }
  return TERN_OK;
}

extern "C" tern_status tern_device_error(void* stream) {
  unsigned v = 0;
  if (read_clear_dev_error_gemv2(stream, &v) != 0) return TERN_ECUDA;
  if (read_clear_dev_error_gemv2w(stream, &v) != 0) return TERN_ECUDA;
  if (read_clear_dev_error_gemv2w_mt(stream, &v) != 0) return TERN_ECUDA;
  if (read_clear_dev_error_stream(stream, &v) != 0) return TERN_ECUDA;
  if (read_clear_dev_error_gemv3(stream, &v) != 0) return TERN_ECUDA;
  if (read_clear_dev_error_gemm_tc(stream, &v) != 0) return TERN_ECUDA;
  if (read_clear_dev_error_selftest(stream, &v) != 0) return TERN_ECUDA;
  if (read_clear_dev_error_decode(stream, &v) != 0) return TERN_ECUDA;
  if (v & TERN_DEVERR_TIMEOUT) return TERN_ETIMEOUT;
  return v ? TERN_EFORMAT : TERN_OK;
}

extern "C" tern_status tern_stream_read(const void* d_src, size_t bytes, int32_t mode, int32_t chunk, int32_t depth,
                                        int32_t ctas_per_sm, int32_t warps, unsigned* d_sink, void* stream) {
  if (!d_src || !d_sink) return TERN_EINVAL;
  const int rc = launch_stream_read(d_src, bytes, mode, chunk, depth, ctas_per_sm, warps, d_sink, stream);
  if (rc < 0) return TERN_EINVAL;
  return rc == 0 ? TERN_OK : TERN_ECUDA;
}
