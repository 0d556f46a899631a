// extern "C" entry points: argument validation, launch planning and dispatch.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "tern_internal.h"

namespace tern {
namespace {

constexpr int kMaxGemvTokens = 16;  // tokens per pass of the GEMV kernels

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

struct Plan2 {
  int ks, cps, wpc, stage_cols, nstage, grid_x;
  size_t ws_cnt_bytes, ws_part_bytes;
};

// Launch plan of the 2-bit GEMV for m tokens in one pass.
//  * K is split into `ks` ranges of whole scale groups so that about four warps
//    per SM have work (small layers are latency-bound; splitting K spreads
//    their bytes over all SMs);
//  * each warp streams its range in stages of about 8 KB, up to 4 in flight.
Plan2 plan_gemv2(const Layout& L, int m, int xmode, int sms, bool allow_split) {
  Plan2 pl{};
  const bool tq = L.fmt == TERN_FMT_TQ;
  const int gc = (tq && L.group >= 64) ? L.group / 64 : 1;  // columns per group
  const int units = (L.cols + gc - 1) / gc;
  const int P = L.planes;
  pl.wpc = 4;
  int sc_target = std::max(gc, (8192 / (P * kPlaneColBytes)) / gc * gc);
  int ks = 1;
  if (allow_split) {
    const int target_warps = 4 * sms;
    ks = std::min(units, std::max(1, (target_warps + L.row_tiles - 1) / L.row_tiles));
  }
  // x staging must fit: m tokens x k-range bytes (int8) or 2 bytes (bf16) <= 96 KB
  const int mt = xmode == kXBf16 ? 1 : (m <= 1 ? 1 : m <= 4 ? 4 : 16);
  const int per_k = xmode == kXBf16 ? 2 : mt;
  while (ks < units && (size_t)((units + ks - 1) / ks) * gc * kColK2 * per_k > 96 * 1024) ++ks;
  int cps_units = (units + ks - 1) / ks;
  pl.cps = cps_units * gc;
  pl.ks = (L.cols + pl.cps - 1) / pl.cps;
  pl.stage_cols = std::min(sc_target, pl.cps);
  pl.nstage = std::min(4, (pl.cps + pl.stage_cols - 1) / pl.stage_cols);
  pl.grid_x = (L.row_tiles + pl.wpc - 1) / pl.wpc;
  if (pl.ks > 1) {
    const size_t elem = (xmode == kXInt8 && tq) ? 8 : 4;
    pl.ws_cnt_bytes = ((size_t)pl.grid_x * 4 + 255) / 256 * 256;
    pl.ws_part_bytes = (size_t)pl.ks * m * L.row_tiles * kTileRows * elem;
  }
  return pl;
}

tern_status check_common(const tern_desc* desc, const void* d_packed, int m, tern_act act, const void* d_x,
                         const float* d_xscale, tern_out out, void* d_y, Layout* L) {
  tern_status st = layout_of(desc, L);
  if (st != TERN_OK) return st;
  if (m < 1) return TERN_EINVAL;
  if (!d_packed || !d_x || !d_y) return TERN_EINVAL;
  if (act != TERN_ACT_INT8 && act != TERN_ACT_BF16) return TERN_EINVAL;
  if (out != TERN_OUT_F32 && out != TERN_OUT_BF16) return TERN_EINVAL;
  if (act == TERN_ACT_INT8 && !d_xscale) return TERN_EINVAL;
  if (!aligned16(d_packed)) return TERN_EALIGN;
  if ((reinterpret_cast<uintptr_t>(d_y) & 3u) != 0) return TERN_EALIGN;
  return TERN_OK;
}

tern_status run_gemv2(const tern_desc* desc, const Layout& L, const void* d_packed, int m, tern_act act,
                      const void* d_x, const float* d_xscale, tern_out out, void* d_y, void* d_ws, size_t ws_bytes,
                      void* stream) {
  const int xmode = act == TERN_ACT_INT8 ? kXInt8 : kXBf16;
  const bool tq = L.fmt == TERN_FMT_TQ;
  if (xmode == kXBf16 && (!tq || m != 1)) return TERN_EUNSUPPORTED;
  if (tq && L.k % kColK2 != 0) return TERN_EUNSUPPORTED;
  if (!tq && (long long)L.k * 127 >= (1ll << 24)) return TERN_EUNSUPPORTED;  // exact int32 -> fp32
  const int sms = device_sms();
  const uint8_t* base = static_cast<const uint8_t*>(d_packed);
  const size_t in_elem = xmode == kXInt8 ? 1 : 2;
  const size_t out_elem = out == TERN_OUT_F32 ? 4 : 2;
  for (int t0 = 0; t0 < m; t0 += kMaxGemvTokens) {
    const int mc = std::min(kMaxGemvTokens, m - t0);
    Plan2 pl = plan_gemv2(L, mc, xmode, sms, d_ws != nullptr);
    if (pl.ks > 1 && ws_bytes < pl.ws_cnt_bytes + pl.ws_part_bytes) return TERN_ENOSPACE;
    Gemv2Params p{};
    p.trit = base + L.trit_offset;
    p.scale = tq ? reinterpret_cast<const uint16_t*>(base + L.scale_offset) : nullptr;
    p.n = L.n;
    p.k = L.k;
    p.planes = L.planes;
    p.group = L.group;
    p.groups = L.groups;
    p.row_tiles = L.row_tiles;
    p.cols = L.cols;
    p.tensor_scale = desc->tensor_scale;
    p.m = mc;
    p.x = static_cast<const uint8_t*>(d_x) + (size_t)t0 * L.k * in_elem;
    p.xscale = d_xscale ? d_xscale + t0 : nullptr;
    p.y = static_cast<uint8_t*>(d_y) + (size_t)t0 * L.n * out_elem;
    p.out_bf16 = out == TERN_OUT_BF16;
    p.ks = pl.ks;
    p.cols_per_split = pl.cps;
    p.wpc = pl.wpc;
    p.stage_cols = pl.stage_cols;
    p.nstage = pl.nstage;
    p.ws_cnt = pl.ks > 1 ? static_cast<unsigned*>(d_ws) : nullptr;
    p.ws_part = pl.ks > 1 ? static_cast<uint8_t*>(d_ws) + pl.ws_cnt_bytes : nullptr;
    if (gemv2_smem_bytes(p, xmode) > 227 * 1024) return TERN_EUNSUPPORTED;
    const int rc = launch_gemv2(p, xmode, (desc->flags & TERN_F_PDL) != 0, stream);
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
  if (L.fmt != TERN_FMT_BT3) {
    const int mc = std::max(1, std::min<int>(m, kMaxGemvTokens));
    for (int xmode = 0; xmode < 2; ++xmode) {
      Plan2 pl = plan_gemv2(L, mc, xmode, sms, true);
      need = std::max(need, pl.ws_cnt_bytes + pl.ws_part_bytes);
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
  tern_status st = check_common(desc, d_packed, m, act, d_x, d_xscale, out, d_y, &L);
  if (st != TERN_OK) return st;
  if (L.fmt == TERN_FMT_BT3) return TERN_EUNSUPPORTED;
  return run_gemv2(desc, L, d_packed, m, act, d_x, d_xscale, out, d_y, d_ws, ws_bytes, stream);
}

extern "C" tern_status tern_gemv(const tern_desc* desc, const void* d_packed, tern_act act, const void* d_x,
                                 const float* d_xscale, tern_out out, void* d_y, void* d_ws, size_t ws_bytes,
                                 void* stream) {
  return tern_gemm_batched(desc, d_packed, 1, act, d_x, d_xscale, out, d_y, d_ws, ws_bytes, stream);
}

extern "C" tern_status tern_device_error(void* stream) {
  unsigned v = 0;
  if (read_clear_dev_error_gemv2(stream, &v) != 0) return TERN_ECUDA;
  return v ? TERN_ETIMEOUT : TERN_OK;
}
