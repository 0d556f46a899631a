// Launches of the one-CTA-per-SM decode GEMV for several tokens of one
// problem (2..8 int8 tokens sharing one pass over the packed weights, padded
// to 2, 4 or 8 with zero images); the kernel template is in
// tern_gemv2w_kernel.cuh.
#include "tern_gemv2w_kernel.cuh"

namespace tern {

int read_clear_dev_error_gemv2w_mt(void* stream, unsigned* out) { return read_clear_dev_error_tu(stream, out); }

namespace {

template <int XM, int MT>
int launch_mt_fmt(const Gemv2wParams& p, bool pdl, void* stream) {
  if (!p.tq) return p.planes == 1 ? launch_w<XM, 1, 0, MT>(p, pdl, stream) : -1;
  switch (p.planes * 100 + p.group / 16) {
    case 116: return launch_w<XM, 1, 16, MT>(p, pdl, stream);
    case 216: return launch_w<XM, 2, 16, MT>(p, pdl, stream);
    case 316: return launch_w<XM, 3, 16, MT>(p, pdl, stream);
    case 416: return launch_w<XM, 4, 16, MT>(p, pdl, stream);
    case 202: return launch_w<XM, 2, 2, MT>(p, pdl, stream);
    case 304: return launch_w<XM, 3, 4, MT>(p, pdl, stream);
    default: return -1;
  }
}

}  // namespace

bool gemv2w_mt_has_kernel(int planes, int tq, int group) {
  if (!tq) return planes == 1;
  switch (planes * 100 + group / 16) {
    case 116: case 216: case 316: case 416: case 202: case 304: return true;
    default: return false;
  }
}

int launch_gemv2w_mt(const Gemv2wParams& p, int xmode, bool pdl, void* stream) {
  if (p.bt3 || p.nprob != 1 || p.mt < 2 || p.mt > kMaxTokensW) return -1;
  const int mtp = gemv2w_mt_pad(p.mt);  // the kernel's token count (zero images beyond p.mt)
  if (xmode == kXInt8) {
    if (mtp == 2) return launch_mt_fmt<kXInt8, 2>(p, pdl, stream);
    return mtp == 4 ? launch_mt_fmt<kXInt8, 4>(p, pdl, stream) : launch_mt_fmt<kXInt8, 8>(p, pdl, stream);
  }
  if (xmode == kXBf16Q8) {
    if (mtp == 2) return launch_mt_fmt<kXBf16Q8, 2>(p, pdl, stream);
    return mtp == 4 ? launch_mt_fmt<kXBf16Q8, 4>(p, pdl, stream) : launch_mt_fmt<kXBf16Q8, 8>(p, pdl, stream);
  }
  return -1;
}

}  // namespace tern
