// C entry points over helpers that the host and the kernels share (launch
// planning in tern_internal.h, balanced-ternary level decoding in
// tern_bt_levels.h), built with the host compiler by tests/test_plan_cpu.py so
// that they are checked without a GPU.
#include "packed_ternary_weight_b200/csrc/tern_internal.h"

extern "C" {

int h_cta_tile(const int* tile_begin, const int* col_begin, int nprob, int c, int grid) {
  return tern::gemv2w_cta_tile(tile_begin, col_begin, nprob, c, grid);
}

int h_mt_pad(int mt) { return tern::gemv2w_mt_pad(mt); }

int h_merged_digits(int planes, int d7) { return tern::tc_merged_digits(planes, d7); }

void h_passes(int digits, int m16, int* passes, int* tpass) { tern::tc_passes(digits, m16, passes, tpass); }

// out: bars, misc, stages, slots, raw_bytes, sc_bytes, xcol_bytes, stage_bytes, C, NS, nslot, NG, sgroups
int h_layout(int planes, int tq, int group, int digits, int tpass, long long* out) {
  tern::TcLayout L{};
  const bool ok = tern::tc_layout(planes, tq, group, digits, tpass, &L);
  const long long v[13] = {L.bars, L.misc, L.stages, L.slots, L.raw_bytes, L.sc_bytes, L.xcol_bytes,
                           L.stage_bytes, L.C, L.NS, L.nslot, L.NG, L.sgroups};
  for (int i = 0; i < 13; ++i) out[i] = v[i];
  return ok ? 1 : 0;
}

int h_const(int which) {
  switch (which) {
    case 0: return tern::kTcSmemBytes;
    case 1: return tern::kTcSlotBytes;
    case 2: return tern::kTcMaxStages;
    case 3: return tern::kTcMaxSlots;
    case 4: return tern::kTcMaxTokens;
    case 5: return tern::kTcMaxMerged;
    case 6: return tern::kTcMaxDigits;
    case 7: return tern::kPlaneColBytes;
    case 8: return tern::kMaxTokensW;
    default: return -1;
  }
}

}  // extern "C"

// Balanced-ternary level decoders of depth 2 and 4 (tern_bt_levels.h).
#include "packed_ternary_weight_b200/csrc/tern_bt_levels.h"

extern "C" {

// n packed argument words per byte position; out[5 i + j] = level j of word i
void h_pair_levels(const uint32_t* b0, const uint32_t* b1, int n, uint32_t* out) {
  for (int i = 0; i < n; ++i) {
    uint32_t U[5];
    tern::pair_levels(b0[i], b1[i], U);
    for (int j = 0; j < 5; ++j) out[5 * i + j] = U[j];
  }
}

void h_quad_levels(const uint32_t* b0, const uint32_t* b1, const uint32_t* b2, const uint32_t* b3, int n,
                   uint32_t* out) {
  for (int i = 0; i < n; ++i) {
    uint32_t U[5];
    tern::quad_levels(b0[i], b1[i], b2[i], b3[i], U);
    for (int j = 0; j < 5; ++j) out[5 * i + j] = U[j];
  }
}

}  // extern "C"
