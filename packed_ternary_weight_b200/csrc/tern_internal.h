// Internal definitions shared by the host API, the packer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/tern.h"

#define TERN_DEVERR_TIMEOUT 1u
#define TERN_DEVERR_FORMAT 2u  /* a kernel found packed data it cannot use */

#if defined(__CUDACC__)
#define TERN_HD __host__ __device__
#else
#define TERN_HD
#endif

namespace tern {

// ---------------------------------------------------------------- format
constexpr uint32_t kMagic = 0x4E524554u;  // "TERN"
constexpr uint32_t kVersion = 2;
constexpr size_t kHeaderBytes = 256;
constexpr size_t kCodebookOffset = 128;
constexpr size_t kDigitsOffset = 72;  // u32: 7-bit digits of the largest TQ scale in units of 2^-24
constexpr int kTileRows = 32;       // rows per row tile (one per lane)
constexpr int kColK2 = 64;          // k per 16-byte chunk, 2-bit planes
constexpr int kColK3 = 80;          // k per 16-byte chunk, base-3 planes
constexpr int kChunkBytes = 16;
constexpr int kPlaneColBytes = kTileRows * kChunkBytes;   // 512
// balanced ternary of depth d: d base-3 bytes per 5 weights of a row, then the group-index triple
TERN_HD constexpr int bt_col_bytes(int d) { return d * kPlaneColBytes + 3 * kTileRows; }
constexpr int kBt3ColBytes = bt_col_bytes(3);  // 1632: d = 3, the depth the kernels take
constexpr int kBt3Groups = 5;       // groups of 16 per base-3 column

struct Layout {
  int fmt, n, k, planes, group, groups, row_tiles, cols;
  size_t trit_offset, trit_bytes, scale_offset, scale_bytes, total;
};

// Validates the descriptor and computes the packed layout. Host only.
tern_status layout_of(const tern_desc* d, Layout* L);

// ------------------------------------------------------------ kernels
// Activation modes of the 2-bit GEMV:
//   kXInt8   int8 activations with one fp32 scale per token (exact path);
//   kXBf16   bf16 activations (24-bit fixed-point image, fp32 group fold);
//   kXBf16Q8 bf16 activations quantised per token inside the kernel, then the
//            exact int8 path (same result as tern_quantize_act + kXInt8).
enum XMode : int { kXInt8 = 0, kXBf16 = 1, kXBf16Q8 = 2 };

constexpr int kMaxProblems = 32;   // independent GEMVs in one launch of the row-group kernel
constexpr int kMaxProblemsW = 256; // ... of the one-CTA-per-SM kernel (parameter block < 32 KB)
constexpr int kMaxSlotsW = 16;     // problems one CTA of that kernel may touch
constexpr int kMaxTokensW = 8;     // tokens of one problem per launch of that kernel
// Activation images of a multi-token launch: the tokens padded to 2, 4 or 8
// (the padding images are zero), so the kernel's token loops have no bounds.
TERN_HD inline int gemv2w_mt_pad(int mt) { return mt <= 1 ? 1 : (mt <= 2 ? 2 : (mt <= 4 ? 4 : 8)); }
constexpr int kMaxCluster = 16;   // K-splits reduced through one thread-block cluster

struct Gemv2Problem {
  const uint8_t* trit;      // trit stream (device)
  const uint16_t* scale;    // TQ scale stream (fp16 bits) or nullptr
  const void* x;            // activations [m][k]
  const float* xscale;      // kXInt8: [m]
  void* y;                  // [m][n] float or bf16
  int n, row_tiles;
  int cta_begin;            // first blockIdx.x of this problem
  float tensor_scale;       // BitNet
};

struct Gemv2Params {
  Gemv2Problem prob[kMaxProblems];
  int nprob;
  int grid_x;               // sum over problems of ceil(row_tiles / wpc): the row groups
  int groups_total;         // set at launch: row groups in all problems
  int persistent;           // set at launch: CTAs walk ranges of row groups (no K split)
  int tq;                   // fp16 group scales (TQ) rather than one per-tensor scale
  int k, planes, group, groups, cols;   // shared by all problems
  int m;                    // tokens
  int out_bf16;
  int ks;                   // K splits (grid.y)
  int cluster;              // 1: splits reduce through a (1, ks, 1) cluster; 0: through ws
  int cols_per_split;       // multiple of the group's column count
  int wpc;                  // warps (row tiles) per CTA
  int stage_cols;           // columns per pipeline stage
  int nstage;               // stages per warp ring
  int x_vec;                // activations may be read with 16-byte loads
  int mt;                   // tokens of the (single) problem sharing the weight stream, or 1
  void* ws_part;            // global fallback: partials [ks][m][row_tiles*32]
  unsigned* ws_cnt;         // global fallback: arrival counters [grid.x]
};

// Single-token 2-bit GEMV with one CTA per SM ("whole-K" kernel, gemv2w):
// the row tiles of all problems are split into equal contiguous ranges, one
// per CTA, and each CTA's columns (tiles x columns) into equal contiguous
// ranges, one per warp; tiles that two or more warps share are combined in
// shared memory in warp order.
struct Gemv2wProblem {
  const uint8_t* trit;
  const uint16_t* scale;
  const void* x;            // [k]
  const float* xscale;      // kXInt8: [1]
  void* y;                  // [n]
  int n, row_tiles;
  float tensor_scale;
  int k, cols, groups;      // input width, its 64-k (80-k for d = 3) columns, scale groups
};

// Scalars first and the tiles' problem boundaries as one compact array, so
// that a CTA's start-up reads touch few lines of the parameter buffer (every
// SM misses on the same lines at once).
struct Gemv2wParams {
  int nprob, tiles_total;
  int grid;                 // CTAs (at most one per SM)
  int tq, k, planes, group, groups, cols;  // k, groups, cols: the largest of the launch's problems
  int bt3;                  // balanced ternary d = 3 columns (80 k, 1632 bytes per tile column)
  int gcols;                // columns per granule of the warp ranges (a whole scale group)
  int out_bf16;
  int nw;                   // warps per CTA
  int stage_cols, nstage;   // per-warp ring: columns per stage, stages
  int xslots;               // activation images resident per CTA
  int x_vec;                // activations may be read with 16-byte loads
  int mt;                   // tokens of the (single) problem sharing the weight stream, or 1
  int early_w;              // set at launch: weights may be requested before the dependency wait
  int tile_begin[kMaxProblemsW + 1];  // first tile of each problem; [nprob] = tiles_total
  int col_begin[kMaxProblemsW + 1];   // first column (tiles x columns) of each problem; [nprob] = total
  Gemv2wProblem prob[kMaxProblemsW];  // last member: the kernel copies only its own problems
};

// CTA c of G takes the tiles [gemv2w_cta_tile(c), gemv2w_cta_tile(c + 1)): the
// first tile whose first column is at or after the c-th equal share of all
// columns, so that CTAs get equal work when problems differ in K. Host and
// device call the same function.
TERN_HD inline int gemv2w_cta_tile(const int* tile_begin, const int* col_begin, int nprob, int c, int G) {
  const long long ctot = col_begin[nprob];
  const long long cg = ctot * c / G;
  if (cg >= ctot) return tile_begin[nprob];
  int lo = 0, hi = nprob - 1;  // the last problem whose first column is <= cg
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (col_begin[mid] <= cg) lo = mid; else hi = mid - 1;
  }
  const int ncol = (col_begin[lo + 1] - col_begin[lo]) / (tile_begin[lo + 1] - tile_begin[lo]);
  const int d = (int)(cg - col_begin[lo]);
  return tile_begin[lo] + (d + ncol - 1) / ncol;
}

// Batched GEMM on the tensor cores (tcgen05 kind::i8): tokens padded to a
// multiple of 16 (the host routes here from 16 tokens, or from 9 when the
// caller gives a workspace). The
// fp16 group scale s of every (plane, row, group) is an integer u = |s| / 2^-24
// written in D' digits of b bits (b = 7, 6, 5 for one, two, three or four
// planes); the A operand of digit d holds sum_p sign(s_p) * t_p * u_{p,d}
// (int8), so one int32 accumulator per digit sums over all groups and planes
// and the exact result is sum_d 2^(b d) * acc_d (int64).
constexpr int kTcRows = 128;       // weight rows per MMA tile (four 32-row tiles)
constexpr int kTcMaxDigits = 6;    // 7-bit digits: fp16 magnitudes are below 2^40 units of 2^-24
constexpr int kTcMaxMerged = 9;    // merged digits (5 bits for three or four planes)
constexpr int kTcMaxTokens = 256;  // tokens per launch (MMA N <= 256)
constexpr int kTcSmemBytes = 227 * 1024;   // dynamic shared memory of every launch
constexpr int kTcSlotBytes = kTcRows * 64;  // one A tile: 128 rows x 64 k, int8
constexpr int kTcMaxStages = 12;
constexpr int kTcMaxSlots = 18;             // A tiles: groups of D' tiles (see tc_layout)
constexpr int kTcMaxColsPerStage = 4;

struct GemmTcParams {
  const uint8_t* trit;           // trit stream
  const uint16_t* scale;         // TQ scale stream, or nullptr
  const uint8_t* header;         // packed header (digit count at kDigitsOffset)
  const uint8_t* xp;             // activations in MMA order [passes][cols*4][tpass][16] (workspace)
  const float* xscale;           // [m]
  void* y;                       // [m][n]
  unsigned long long* part;      // [m][n_pad] int64 partial sums (zero on entry and exit)
  unsigned* cnt;                 // [tiles][passes_cap] arrival counters (zero on entry and exit)
  int n, k, planes, group, cols, row_tiles, tiles, n_pad;
  int m, m16, passes_cap;
  int tq, out_bf16;
  float tensor_scale;
  int grid;
};

// Digits of the merged A operand for P planes and D 7-bit digits of the
// largest scale: b = 7 (one plane), 6 (two), 5 (three, four) bits per digit.
TERN_HD inline int tc_merged_digits(int planes, int d7) {
  const int b = planes == 1 ? 7 : (planes == 2 ? 6 : 5);
  return (7 * d7 + b - 1) / b;
}

// Token passes for D digits: the D accumulators of one pass share the 512
// tensor-memory columns. Host and device compute the same values.
TERN_HD inline void tc_passes(int digits, int m16, int* passes, int* tpass) {
  int tmax = (512 / digits) & ~15;
  if (tmax > kTcMaxTokens) tmax = kTcMaxTokens;
  const int ps = (m16 + tmax - 1) / tmax;
  const int t = ((m16 + ps - 1) / ps + 15) & ~15;
  *passes = ps;
  *tpass = t;
}

// Shared-memory plan of one launch, from the merged digit count D and the
// tokens per pass: mbarriers and misc words | input stages | A tiles (at the
// top). A stage holds C consecutive 64-k columns of four row tiles (trits,
// scale blocks, activations), so that one bulk-copy instruction per stage
// fetches all of them; C is the widest of 4, 2, 1 that leaves three stages.
struct TcLayout {
  uint32_t bars, misc, stages, slots;  // byte offsets
  uint32_t raw_bytes, sc_bytes, xcol_bytes, stage_bytes;
  int C, NS, nslot, NG, sgroups;       // columns per stage, stages, A tiles, A groups, scale blocks per row tile
};
TERN_HD inline bool tc_layout(int planes, int tq, int group, int digits, int tpass, TcLayout* L) {
  L->NG = digits <= 4 ? 4 : (digits <= 6 ? 3 : 2);
  L->nslot = L->NG * digits;
  L->bars = 0;
  L->misc = (uint32_t)(2 * kTcMaxStages + 2 * kTcMaxSlots + 3) * 8u;
  L->stages = 1024;
  L->slots = (uint32_t)kTcSmemBytes - (uint32_t)L->nslot * kTcSlotBytes;
  L->xcol_bytes = 4u * (uint32_t)tpass * 16u;
  for (int C = kTcMaxColsPerStage; C >= 1; C >>= 1) {
    const int sg = tq ? (64 * C >= group ? 64 * C / group : 1) : 0;
    L->C = C;
    L->sgroups = sg;
    L->raw_bytes = 4u * (uint32_t)(C * planes * kPlaneColBytes);
    L->sc_bytes = ((uint32_t)(4 * sg * planes * 64) + 127u) & ~127u;
    L->stage_bytes = L->raw_bytes + L->sc_bytes + (((uint32_t)C * L->xcol_bytes + 127u) & ~127u);
    const int ns = L->slots > L->stages ? (int)((L->slots - L->stages) / L->stage_bytes) : 0;
    L->NS = ns < kTcMaxStages ? ns : kTcMaxStages;
    if (L->NS >= 3) break;
  }
  return L->misc + 64u <= L->stages && L->nslot <= kTcMaxSlots && L->NS >= 2;
}

int launch_gemm_tc(const GemmTcParams& p, void* stream);  // -1: no kernel for this shape
int launch_tc_prep_x(const int8_t* xq, int m, int k, int kchunks, int total_max, const GemmTcParams& p, uint8_t* xp,
                     void* stream);
int read_clear_dev_error_gemm_tc(void* stream, unsigned* out);

// Launchers return cudaError_t values as int (0 = success).
int launch_gemv2(const Gemv2Params& p, int xmode, bool pdl, void* stream);  // -1: no kernel
int launch_gemv2w(const Gemv2wParams& p, int xmode, bool pdl, void* stream);  // -1: no kernel
int launch_gemv2w_mt(const Gemv2wParams& p, int xmode, bool pdl, void* stream);  // p.mt > 1
bool gemv2w_mt_has_kernel(int planes, int tq, int group);  // the plane / group combinations of launch_gemv2w_mt
size_t gemv2w_smem_bytes(const Gemv2wParams& p, int xmode);
int read_clear_dev_error_gemv2w(void* stream, unsigned* out);
int read_clear_dev_error_gemv2w_mt(void* stream, unsigned* out);
int launch_quantize(const uint16_t* x, int m, int k, int8_t* xq, float* xs, void* stream);

int read_clear_dev_error_gemv2(void* stream, unsigned* out);
int read_clear_dev_error_stream(void* stream, unsigned* out);
int read_clear_dev_error_gemv3(void* stream, unsigned* out);
int read_clear_dev_error_selftest(void* stream, unsigned* out);
int launch_gemv3(const Gemv2Params& p, bool pdl, void* stream);  // balanced ternary, bf16 x, m = 1..8
// tokens per launch of the balanced-ternary kernel: m padded to 1, 2, 4 or 8
TERN_HD inline int gemv3_mt(int m) { return m <= 1 ? 1 : (m <= 2 ? 2 : (m <= 4 ? 4 : 8)); }
size_t gemv3_smem_bytes(const Gemv2Params& p);
int launch_stream_read(const void* src, size_t bytes, int mode, int chunk, int depth, int ctas_per_sm, int warps,
                       unsigned* sink, void* stream);

// ------------------------------------------------ persistent decode step
constexpr int kDecMaxLayers = 64;
constexpr int kDecHeadDim = 128;
constexpr int kDecMaxVec = 14336;        // largest hidden / FFN / attention width
constexpr int kDecMaxKvHeads = 16;
constexpr int kDecMaxRep = 4;            // query heads per KV head
constexpr int kDecMaxSplits = 4;         // column ranges per row tile
constexpr int kDecMaxPartsPerCta = 8;
constexpr int kDecMaxSlots = 32;         // 8 KB weight slots of the ring
constexpr size_t kDecSmemBytes = 227 * 1024;

// One GEMV stage of a decode layer (the same shapes in every layer): the
// projections' row tiles, each cut into `splits` column ranges ("parts").
struct DecStage {
  int nprob;           // projections in the stage (q, k, v: 3; gate, up: 2; else 1)
  int proj[3];         // their indices among q, k, v, o, gate, up, down
  int tile0[4];        // first stage tile of each projection; tile0[nprob] = tiles
  int cols;            // 64-k columns (K / 64)
  int splits, parts;   // parts = tiles * splits
};

struct DecParams {
  const uint8_t* packed[kDecMaxLayers][7];   // BitNet packed buffers (device)
  const float* gains;       // [layers][gain_stride]: input D | attn_sub H*128 | post D | ffn_sub F
  uint16_t* kc;             // bf16 [layers][KVH][max_pos][128]
  uint16_t* vc;
  const float* rope;        // [max_pos][64][2] cos, sin
  const float* h_in;        // [D]
  float* h_out;             // [D]
  const float* attn_in;     // [H*128] when the run starts at an o_proj stage
  float* trace;             // optional [layers][trace_stride]
  uint8_t* ws;
  size_t off_ctl, off_part[4], off_att, off_attn, ws_bytes;
  int layers, D, F, H, KVH, max_pos, pos, first, last;
  int gain_stride, trace_stride;
  int vmax;                 // max(D, F, H*128): the image width
  int grid, ns;             // CTAs; attention position ranges per KV head
  float eps;
  DecStage st[4];           // qkv, o, gate/up, down
};

int launch_decode(const DecParams& p, void* stream);  // -1: does not fit one CTA per SM
size_t decode_smem_bytes(const DecParams& p);
int decode_ring_slots(const DecParams& p);
int read_clear_dev_error_decode(void* stream, unsigned* out);

// Shared-memory bytes a 2-bit GEMV CTA needs for these parameters.
size_t gemv2_smem_bytes(const Gemv2Params& p, int xmode);
int gemv2_mt(int xmode, int m);   // tokens per pass of the kernel instantiated for m

}  // namespace tern
