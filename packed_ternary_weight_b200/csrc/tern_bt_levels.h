// Levels of balanced-ternary weights of depth 2 and 4 from their packed byte
// tuples (the format of tern_pack.cpp: five weights per tuple of d base-3
// bytes, five digits u = t + 1 per byte, first digit least significant, a
// weight's d digits consecutive). A weight's level is U = sum_p 3^p u_p, in
// 0 .. 3^d - 1; U minus (3^d - 1) / 2 is sum_p 3^p t_p, the level of the
// Entrit card's rule ("Quantization details") at depth d.
//
// Two tuples are decoded at once, one in each 16-bit lane of the arguments
// (every byte <= 242). The divisions are exact multiply-shifts for v <= 242:
// floor(v / 3) = (171 v) >> 9, floor(v / 9) = (57 v) >> 9,
// floor(v / 27) = (19 v) >> 9, floor(v / 81) = (203 v) >> 14. Every product
// stays below 2^16 and every quotient fits the lane's mask, so no lane
// carries into the other. Host and device use the same code.
#pragma once
#include <cstdint>

#include "tern_internal.h"

namespace tern {

constexpr uint32_t kBtLane7 = 0x007F007Fu;  // quotients below 128
constexpr uint32_t kBtLane2 = 0x00030003u;  // quotients below 4 (v / 81)

// Depth 2: byte 0 = digits of weight 0 (u0, u1), weight 1 (u0, u1), weight 2 (u0);
// byte 1 = weight 2 (u1), weight 3 (u0, u1), weight 4 (u0, u1). U = u0 + 3 u1.
TERN_HD inline void pair_levels(uint32_t b0, uint32_t b1, uint32_t (&U)[5]) {
  const uint32_t q0 = ((b0 * 57u) >> 9) & kBtLane7;  // b0 / 9: weight 1's level, then u0 of weight 2
  U[0] = b0 - 9u * q0;
  const uint32_t u20 = ((q0 * 57u) >> 9) & kBtLane7;  // q0 / 9
  U[1] = q0 - 9u * u20;
  const uint32_t r = ((b1 * 171u) >> 9) & kBtLane7;   // b1 / 3
  U[2] = u20 + 3u * (b1 - 3u * r);
  U[4] = ((r * 57u) >> 9) & kBtLane7;                 // r / 9
  U[3] = r - 9u * U[4];
}

// Depth 4: byte 0 = weight 0 (u0..u3), weight 1 (u0); byte 1 = weight 1
// (u1..u3), weight 2 (u0, u1); byte 2 = weight 2 (u2, u3), weight 3 (u0..u2);
// byte 3 = weight 3 (u3), weight 4 (u0..u3). U = u0 + 3 u1 + 9 u2 + 27 u3.
TERN_HD inline void quad_levels(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3, uint32_t (&U)[5]) {
  const uint32_t q0 = ((b0 * 203u) >> 14) & kBtLane2;  // b0 / 81: u0 of weight 1
  U[0] = b0 - 81u * q0;
  const uint32_t q1 = ((b1 * 19u) >> 9) & kBtLane7;    // b1 / 27: u0 + 3 u1 of weight 2
  U[1] = q0 + 3u * (b1 - 27u * q1);
  const uint32_t q2 = ((b2 * 57u) >> 9) & kBtLane7;    // b2 / 9: u0 + 3 u1 + 9 u2 of weight 3
  U[2] = q1 + 9u * (b2 - 9u * q2);
  U[4] = ((b3 * 171u) >> 9) & kBtLane7;                // b3 / 3
  U[3] = q2 + 27u * (b3 - 3u * U[4]);
}

}  // namespace tern
