// sa_fp8.cuh -- the fp8 summary record encoder shared by the summaries kernel and the
// scorer's decode-time refresh.
//
// Record of a (page, KV head): [Dk E4M3 codes of the min row | Dk codes of the max row |
// int8 e | 15 zero bytes]; value = code * 2^e, e the smallest integer with
// max|value| * 2^-e <= 448, codes rounded outward (min toward -inf, max toward +inf), so
// the decoded rows bracket every key of the page (the quantised-KV option the
// SparseEngine blog's hook-point paragraph lists next to Quest; the pages give no
// format).  The encoder works on the bf16 bit fields: no value is rounded before the one
// outward step.
#pragma once

#include "sa_common.cuh"

namespace sa {

// Exponent of an fp8 record from the largest magnitude A (bf16 magnitude bits): with
// A = f * 2^E, f in [0.5, 1), the smallest e with A * 2^-e <= 448 = 0.875 * 2^9 is E - 9
// when f <= 0.875 and E - 8 otherwise; 0 for A = 0.
__device__ __forceinline__ int fp8_record_exp(uint32_t amag) {
  if (amag == 0) return 0;
  int E;
  const float f = frexpf(__uint_as_float(amag << 16), &E);
  return f <= 0.875f ? E - 9 : E - 8;
}

// E4M3 code of (bf16 value v) * 2^-e rounded toward +inf (up) or -inf (!up), for
// |v * 2^-e| <= 448.  v = S * 2^X exactly (S the 8-bit significand); the target binade
// of floor(log2 |x|) = k has the step 2^(k-3), or 2^-9 below the normal range, and the
// code of T steps of 2^q is 8 * (q + 9) + T (T = 16 carries into the next binade, and
// subnormal T = 8 is the smallest normal).  Zero results are the code 0x00.
__device__ __forceinline__ uint32_t e4m3_outward(uint32_t v, int e, bool up) {
  const uint32_t mag = v & 0x7FFFu;
  if (mag == 0) return 0u;
  const bool neg = (v & 0x8000u) != 0;
  const uint32_t E8 = mag >> 7, m7 = mag & 0x7Fu;
  const uint32_t S = E8 ? (0x80u | m7) : m7;
  const int X = (E8 ? (int)E8 : 1) - 134 - e;
  const int k = 31 - __clz(S) + X;
  const int q = max(k - 3, -9);
  const int sh = X - q;
  uint32_t T;
  if (sh >= 0) {
    T = S << sh;
  } else {
    const int r = -sh;
    T = r >= 32 ? 0u : (S >> r);
    const bool inexact = r >= 32 ? true : (S & ((1u << r) - 1u)) != 0u;
    if (inexact && up != neg) ++T;  // the magnitude moves away from zero
  }
  const uint32_t code = 8u * (uint32_t)(q + 9) + T;
  return code == 0u ? 0u : (neg ? (0x80u | code) : code);
}

// the four codes of the bf16 pairs (a, b) as bytes lo..hi of one word
__device__ __forceinline__ uint32_t e4m3_pack(uint32_t a, uint32_t b, int e, bool up) {
  return e4m3_outward(a & 0xFFFFu, e, up) | (e4m3_outward(a >> 16, e, up) << 8) |
         (e4m3_outward(b & 0xFFFFu, e, up) << 16) | (e4m3_outward(b >> 16, e, up) << 24);
}

__device__ __forceinline__ uint32_t max_mag2(uint32_t m, uint32_t w) {
  return max(m, max(w & 0x7FFFu, (w >> 16) & 0x7FFFu));
}

}  // namespace sa
