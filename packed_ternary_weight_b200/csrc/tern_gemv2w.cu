// Launches of the one-CTA-per-SM decode GEMV for one token per problem (the
// kernel template and its design notes are in tern_gemv2w_kernel.cuh).
#include "tern_gemv2w_kernel.cuh"

namespace tern {

int read_clear_dev_error_gemv2w(void* stream, unsigned* out) { return read_clear_dev_error_tu(stream, out); }

size_t gemv2w_smem_bytes(const Gemv2wParams& p, int xmode) { return plan2w(p, xmode).total; }

// TQ with 1-4 planes at g = 32, 64, 128 or 256 (sasori README, "K and g").
#define TERN_W_TQ_CASES(XM) \
  switch (p.planes * 100 + wg) { \
    case 102: return launch_w<XM, 1, 2, 1>(p, pdl, stream); \
    case 104: return launch_w<XM, 1, 4, 1>(p, pdl, stream); \
    case 108: return launch_w<XM, 1, 8, 1>(p, pdl, stream); \
    case 116: return launch_w<XM, 1, 16, 1>(p, pdl, stream); \
    case 202: return launch_w<XM, 2, 2, 1>(p, pdl, stream); \
    case 204: return launch_w<XM, 2, 4, 1>(p, pdl, stream); \
    case 208: return launch_w<XM, 2, 8, 1>(p, pdl, stream); \
    case 216: return launch_w<XM, 2, 16, 1>(p, pdl, stream); \
    case 302: return launch_w<XM, 3, 2, 1>(p, pdl, stream); \
    case 304: return launch_w<XM, 3, 4, 1>(p, pdl, stream); \
    case 308: return launch_w<XM, 3, 8, 1>(p, pdl, stream); \
    case 316: return launch_w<XM, 3, 16, 1>(p, pdl, stream); \
    case 402: return launch_w<XM, 4, 2, 1>(p, pdl, stream); \
    case 404: return launch_w<XM, 4, 4, 1>(p, pdl, stream); \
    case 408: return launch_w<XM, 4, 8, 1>(p, pdl, stream); \
    case 416: return launch_w<XM, 4, 16, 1>(p, pdl, stream); \
    default: return -1; \
  }

int launch_gemv2w(const Gemv2wParams& p, int xmode, bool pdl, void* stream) {
  if (p.mt > 1) return launch_gemv2w_mt(p, xmode, pdl, stream);
  if (p.bt3) return (xmode == kXBf16 && p.planes == 3) ? launch_w<kXBf16, 3, -1, 1>(p, pdl, stream) : -1;
  if (!p.tq) {
    if (p.planes != 1) return -1;
    if (xmode == kXInt8) return launch_w<kXInt8, 1, 0, 1>(p, pdl, stream);
    if (xmode == kXBf16Q8) return launch_w<kXBf16Q8, 1, 0, 1>(p, pdl, stream);
    return -1;
  }
  const int wg = p.group / 16;
  if (xmode == kXInt8) TERN_W_TQ_CASES(kXInt8)
  if (xmode == kXBf16Q8) TERN_W_TQ_CASES(kXBf16Q8)
  TERN_W_TQ_CASES(kXBf16)
}
#undef TERN_W_TQ_CASES

}  // namespace tern
