// Host-side layout computation and packer (no device work).
//
// Packed buffer = 256-byte header + trit stream (+ scale stream for TQ).
// Header (version 2): magic, version, format, N, K, planes, group, tensor
// scale, row tiles, columns, stream offsets and sizes, at byte 72 the number
// of base-128 digits of the largest TQ scale in units of 2^-24 (1 for BitNet,
// 0 for balanced ternary), and the balanced-ternary codebook at byte 128.
//
// 2-bit planes (BitNet b1.58 layout of the QORA-LLM-2B page, "Ternary GEMV";
// sasori TQ{K}P planes): each weight is a 2-bit code 00 -> 0, 01 -> +1,
// 10 -> -1, four per byte. A 16-byte chunk holds 64 consecutive k of one row
// of one plane as four little-endian u32 words; word w covers k = 64c + 16w + j
// with trit j at bit 8*(j%4) + 2*(j/4), so that masking one 2-bit field in each
// byte of a word selects four consecutive k. Chunks are ordered
// [row tile of 32 rows][column c][plane p][row r], so one column of a row tile
// is 512*P contiguous bytes and any range of columns is one contiguous run.
// TQ scales (fp16, one per plane per group of g along K) are ordered
// [row tile][group][plane][row].
//
// Balanced ternary of depth d (Entrit card, "Quantization details": d = 3;
// d = 2 and 4 by the same rule): digits u = t + 1 are packed five per byte in
// base 3 (first digit least significant). A column covers 80 k of a 32-row
// tile. Per row it holds 16 tuples of d bytes: tuple i carries the 5d trits
// of the five weights k = 80c + 16j + i (j = 0..4, one weight of each of the
// column's five groups of 16), weight by weight (t0 .. t(d-1) of weight j are
// trits dj .. dj+d-1 of the tuple, trits 5b..5b+4 in byte b); byte b of tuple
// i sits at b * 512 + 16 r + i. Then one triple per row (bytes at
// 512 d + 32 b + r) holding the five groups' codebook indices in the same
// order (digit q of index j is trit 3j + q). Keeping the trits of a weight
// together lets the decoder read a weight's level U = u0 + 3 u1 + 9 u2 (d = 3)
// with a few divisions by 3, 9 and 27 instead of extracting every digit.
#include <cmath>
#include <cstring>
#include <vector>

#include "tern_internal.h"

namespace tern {

static inline bool valid_group(int g) { return g == 16 || g == 32 || g == 64 || g == 128 || g == 256; }

tern_status layout_of(const tern_desc* d, Layout* L) {
  if (!d || !L) return TERN_EINVAL;
  if (d->n < 1 || d->k < 1 || d->n > (1 << 24) || d->k > (1 << 24)) return TERN_EINVAL;
  Layout l{};
  l.fmt = d->fmt;
  l.n = d->n;
  l.k = d->k;
  l.row_tiles = (d->n + kTileRows - 1) / kTileRows;
  l.trit_offset = kHeaderBytes;
  switch (d->fmt) {
    case TERN_FMT_BITNET:
      if (d->planes != 1) return TERN_EINVAL;
      if (!std::isfinite(d->tensor_scale)) return TERN_EFORMAT;
      l.planes = 1;
      l.group = d->k;
      l.groups = 1;
      l.cols = (d->k + kColK2 - 1) / kColK2;
      l.trit_bytes = (size_t)l.row_tiles * l.cols * kPlaneColBytes;
      l.scale_bytes = 0;
      break;
    case TERN_FMT_TQ:
      if (d->planes < 1 || d->planes > 4) return TERN_EINVAL;
      if (!valid_group(d->group) || d->k % d->group != 0) return TERN_EINVAL;
      l.planes = d->planes;
      l.group = d->group;
      l.groups = d->k / d->group;
      l.cols = (d->k + kColK2 - 1) / kColK2;
      l.trit_bytes = (size_t)l.row_tiles * l.cols * l.planes * kPlaneColBytes;
      l.scale_bytes = (size_t)l.row_tiles * l.groups * l.planes * kTileRows * 2;
      break;
    case TERN_FMT_BT3:
      if (d->planes < 2 || d->planes > 4 || d->group != 16 || d->k % 16 != 0) return TERN_EINVAL;
      l.planes = d->planes;
      l.group = 16;
      l.groups = d->k / 16;
      l.cols = (d->k + kColK3 - 1) / kColK3;
      l.trit_bytes = (size_t)l.row_tiles * l.cols * bt_col_bytes(l.planes);
      l.scale_bytes = 0;
      break;
    default:
      return TERN_EINVAL;
  }
  l.scale_offset = l.trit_offset + l.trit_bytes;
  l.total = l.scale_offset + l.scale_bytes;
  *L = l;
  return TERN_OK;
}

static inline uint32_t code2(int8_t t) { return t == 1 ? 1u : (t == -1 ? 2u : 0u); }

static void write_header(uint8_t* out, const Layout& L, const tern_desc* d, const float* codebook) {
  std::memset(out, 0, kHeaderBytes);
  uint32_t u[7] = {kMagic, kVersion, (uint32_t)L.fmt, (uint32_t)L.n, (uint32_t)L.k, (uint32_t)L.planes,
                   (uint32_t)L.group};
  std::memcpy(out, u, sizeof(u));
  float ts = L.fmt == TERN_FMT_BITNET ? d->tensor_scale : 0.0f;
  std::memcpy(out + 28, &ts, 4);
  uint32_t tc[2] = {(uint32_t)L.row_tiles, (uint32_t)L.cols};
  std::memcpy(out + 32, tc, 8);
  uint64_t q[4] = {L.trit_offset, L.trit_bytes, L.scale_offset, L.scale_bytes};
  std::memcpy(out + 40, q, 32);
  if (L.fmt == TERN_FMT_BT3) std::memcpy(out + kCodebookOffset, codebook, 27 * sizeof(float));
  const uint32_t digits = L.fmt == TERN_FMT_BITNET ? 1u : 0u;  // TQ: set by pack_tq_scales
  std::memcpy(out + kDigitsOffset, &digits, 4);
}

static bool fp16_finite(uint16_t h) { return ((h >> 10) & 0x1F) != 0x1F; }

// |s| / 2^-24 as an exact double (fp16 values are m * 2^e with e >= -24).
static double fp16_units(uint16_t h) {
  int ex = (h >> 10) & 0x1F, man = h & 0x3FF;
  double m = ex ? (1024.0 + man) : (double)man;
  int sh = ex ? ex - 1 : 0;
  return std::ldexp(m, sh);
}

static tern_status pack_2bit(const Layout& L, const int8_t* trits, uint8_t* out) {
  const int P = L.planes, N = L.n, K = L.k;
  for (size_t i = 0; i < (size_t)P * N * K; ++i)
    if (trits[i] < -1 || trits[i] > 1) return TERN_EFORMAT;
  uint8_t* base = out + L.trit_offset;
#pragma omp parallel for schedule(static)
  for (int T = 0; T < L.row_tiles; ++T) {
    for (int c = 0; c < L.cols; ++c)
      for (int p = 0; p < P; ++p)
        for (int r = 0; r < kTileRows; ++r) {
          const int n = T * kTileRows + r;
          uint32_t words[4] = {0, 0, 0, 0};
          if (n < N) {
            const int8_t* row = trits + ((size_t)p * N + n) * K;
            for (int w = 0; w < 4; ++w)
              for (int j = 0; j < 16; ++j) {
                const int k = c * kColK2 + 16 * w + j;
                if (k < K) words[w] |= code2(row[k]) << (8 * (j % 4) + 2 * (j / 4));
              }
          }
          uint8_t* dst = base + (((size_t)T * L.cols + c) * P + p) * kPlaneColBytes + (size_t)r * kChunkBytes;
          std::memcpy(dst, words, 16);  // little-endian host
        }
  }
  return TERN_OK;
}

static tern_status pack_tq_scales(const Layout& L, const uint16_t* s, uint8_t* out) {
  const int P = L.planes, N = L.n, G = L.groups;
  for (size_t i = 0; i < (size_t)P * N * G; ++i)
    if (!fp16_finite(s[i])) return TERN_EFORMAT;
  // Exactness bound of the int8 path: sum over planes and groups of
  // |s| * 127 * g, counted in units of 2^-24, must stay below 2^62.
  for (int n = 0; n < N; ++n) {
    double tot = 0.0;
    for (int p = 0; p < P; ++p)
      for (int g = 0; g < G; ++g) tot += fp16_units(s[((size_t)p * N + n) * G + g]) * 127.0 * L.group;
    if (tot >= std::ldexp(1.0, 62)) return TERN_EFORMAT;
  }
  // Digit count of the largest |s| / 2^-24 in base 128 (at least 1): the
  // batched tensor-core kernel splits every scale into that many 7-bit digits.
  uint64_t umax = 0;
  for (size_t i = 0; i < (size_t)P * N * G; ++i) {
    const uint32_t ex = (s[i] >> 10) & 0x1F, man = s[i] & 0x3FF;
    const uint64_t u = ex ? (uint64_t)(1024 + man) << (ex - 1) : man;
    umax = u > umax ? u : umax;
  }
  uint32_t digits = 1;
  while (digits < 6 && (umax >> (7 * digits)) != 0) ++digits;
  std::memcpy(out + kDigitsOffset, &digits, 4);
  uint16_t* dst = reinterpret_cast<uint16_t*>(out + L.scale_offset);
  for (int T = 0; T < L.row_tiles; ++T)
    for (int g = 0; g < G; ++g)
      for (int p = 0; p < P; ++p)
        for (int r = 0; r < kTileRows; ++r) {
          const int n = T * kTileRows + r;
          dst[(((size_t)T * G + g) * P + p) * kTileRows + r] = n < N ? s[((size_t)p * N + n) * G + g] : 0;
        }
  return TERN_OK;
}

static tern_status pack_bt(const Layout& L, const int8_t* trits, const uint8_t* idx, uint8_t* out) {
  const int N = L.n, K = L.k, G = L.groups, D = L.planes, colb = bt_col_bytes(L.planes);
  for (size_t i = 0; i < (size_t)D * N * K; ++i)
    if (trits[i] < -1 || trits[i] > 1) return TERN_EFORMAT;
  for (size_t i = 0; i < (size_t)N * G; ++i)
    if (idx[i] > 26) return TERN_EFORMAT;
  uint8_t* base = out + L.trit_offset;
#pragma omp parallel for schedule(static)
  for (int T = 0; T < L.row_tiles; ++T) {
    for (int c = 0; c < L.cols; ++c) {
      uint8_t* col = base + ((size_t)T * L.cols + c) * colb;
      for (int r = 0; r < kTileRows; ++r) {
        const int n = T * kTileRows + r;
        for (int i = 0; i < 16; ++i) {
          unsigned dig[20];  // the tuple's trits, weight-major
          for (int j = 0; j < 5; ++j) {
            const int k = c * kColK3 + 16 * j + i;
            for (int p = 0; p < D; ++p)
              dig[D * j + p] = (n < N && k < K) ? (unsigned)(trits[((size_t)p * N + n) * K + k] + 1) : 1u;
          }
          for (int b = 0; b < D; ++b) {
            unsigned v = 0, pw = 1;
            for (int q = 0; q < 5; ++q, pw *= 3) v += dig[5 * b + q] * pw;
            col[b * kPlaneColBytes + r * kChunkBytes + i] = (uint8_t)v;
          }
        }
      }
      // the five groups' codebook indices (3 base-3 digits each) as one more
      // triple per row, index by index: digit q of index j is trit 3j + q
      for (int r = 0; r < kTileRows; ++r) {
        const int n = T * kTileRows + r;
        unsigned dig[15];
        for (int j = 0; j < 5; ++j) {
          const int g = c * kBt3Groups + j;
          const unsigned id = (n < N && g < G) ? idx[(size_t)n * G + g] : 0u;
          dig[3 * j] = id % 3;
          dig[3 * j + 1] = (id / 3) % 3;
          dig[3 * j + 2] = id / 9;
        }
        for (int b = 0; b < 3; ++b) {
          unsigned v = 0, pw = 1;
          for (int q = 0; q < 5; ++q, pw *= 3) v += dig[5 * b + q] * pw;
          col[D * kPlaneColBytes + b * kTileRows + r] = (uint8_t)v;
        }
      }
    }
  }
  return TERN_OK;
}

}  // namespace tern

using namespace tern;

extern "C" tern_status tern_packed_size(const tern_desc* desc, size_t* bytes) {
  if (!bytes) return TERN_EINVAL;
  Layout L;
  tern_status st = layout_of(desc, &L);
  if (st != TERN_OK) return st;
  *bytes = L.total;
  return TERN_OK;
}

extern "C" tern_status tern_pack(const tern_desc* desc, const int8_t* trits, const uint16_t* scales_fp16,
                                 const uint8_t* scale_idx, const float* codebook, void* out, size_t out_cap,
                                 size_t* out_used) {
  Layout L;
  tern_status st = layout_of(desc, &L);
  if (st != TERN_OK) return st;
  if (!trits || !out) return TERN_EINVAL;
  if (L.fmt == TERN_FMT_TQ && !scales_fp16) return TERN_EINVAL;
  if (L.fmt == TERN_FMT_BT3) {
    if (!scale_idx || !codebook) return TERN_EINVAL;
    for (int i = 0; i < 27; ++i)
      if (!std::isfinite(codebook[i])) return TERN_EFORMAT;
  }
  if (out_used) *out_used = L.total;
  if (out_cap < L.total) return TERN_ENOSPACE;
  uint8_t* o = static_cast<uint8_t*>(out);
  std::memset(o, 0, L.total);
  write_header(o, L, desc, codebook);
  if (L.fmt == TERN_FMT_BT3) return pack_bt(L, trits, scale_idx, o);
  st = pack_2bit(L, trits, o);
  if (st != TERN_OK) return st;
  if (L.fmt == TERN_FMT_TQ) st = pack_tq_scales(L, scales_fp16, o);
  return st;
}

extern "C" const char* tern_status_string(tern_status s) {
  switch (s) {
    case TERN_OK: return "ok";
    case TERN_EINVAL: return "invalid argument";
    case TERN_EFORMAT: return "invalid data (trit, index, scale or header)";
    case TERN_EALIGN: return "device pointer not 16-byte aligned";
    case TERN_ENOSPACE: return "buffer or workspace too small";
    case TERN_EUNSUPPORTED: return "no kernel for this combination";
    case TERN_ECUDA: return "CUDA runtime error";
    case TERN_ETIMEOUT: return "bounded wait expired inside a kernel";
  }
  return "unknown status";
}
