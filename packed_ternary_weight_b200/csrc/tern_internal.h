// Internal definitions shared by the host API, the packer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/tern.h"

#define TERN_DEVERR_TIMEOUT 1u

namespace tern {

// ---------------------------------------------------------------- format
constexpr uint32_t kMagic = 0x4E524554u;  // "TERN"
constexpr uint32_t kVersion = 1;
constexpr size_t kHeaderBytes = 256;
constexpr size_t kCodebookOffset = 128;
constexpr int kTileRows = 32;       // rows per row tile (one per lane)
constexpr int kColK2 = 64;          // k per 16-byte chunk, 2-bit planes
constexpr int kColK3 = 80;          // k per 16-byte chunk, base-3 planes
constexpr int kChunkBytes = 16;
constexpr int kPlaneColBytes = kTileRows * kChunkBytes;   // 512
constexpr int kBt3ColBytes = 3 * kPlaneColBytes + 3 * kTileRows;  // 1632
constexpr int kBt3Groups = 5;       // groups of 16 per base-3 column

struct Layout {
  int fmt, n, k, planes, group, groups, row_tiles, cols;
  size_t trit_offset, trit_bytes, scale_offset, scale_bytes, total;
};

// Validates the descriptor and computes the packed layout. Host only.
tern_status layout_of(const tern_desc* d, Layout* L);

// ------------------------------------------------------------ kernels
enum XMode : int { kXInt8 = 0, kXBf16 = 1 };

struct Gemv2Params {
  const uint8_t* trit;      // trit stream (device)
  const uint16_t* scale;    // TQ scale stream (fp16 bits) or nullptr
  int n, k, planes, group, groups, row_tiles, cols;
  float tensor_scale;       // BitNet
  int m;                    // tokens
  const void* x;            // int8 [m][k] or bf16 [m][k]
  const float* xscale;      // int8 path: [m]
  void* y;                  // float [m][n] or bf16 [m][n]
  int out_bf16;
  int ks;                   // K splits (grid.y)
  int cols_per_split;       // multiple of the group's column count
  int wpc;                  // warps (row tiles) per CTA
  int stage_cols;           // columns per pipeline stage
  int nstage;               // stages per warp ring
  void* ws_part;            // split partials [ks][m][row_tiles*32] (int32 / int64 / float)
  unsigned* ws_cnt;         // per-CTA-row arrival counters [grid.x]
};

// Launchers return cudaError_t values as int (0 = success).
int launch_gemv2(const Gemv2Params& p, int xmode, bool pdl, void* stream);
int launch_quantize(const uint16_t* x, int m, int k, int8_t* xq, float* xs, void* stream);

int read_clear_dev_error_gemv2(void* stream, unsigned* out);

// Shared-memory bytes a 2-bit GEMV CTA needs for these parameters.
size_t gemv2_smem_bytes(const Gemv2Params& p, int xmode);

}  // namespace tern
