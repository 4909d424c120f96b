// leanp.cuh -- Lean P: an FP8 (e4m3) softmax probability written directly as
// its code, one multiply-add plus one integer conversion per element, with a
// power-of-two scale per 64-key block.
//
// Method (Zyphra ZYFA, as reported by the-ai.news "Zyphra presenteert ZYFA",
// section "Drie technieken om de bottleneck te omzeilen", and spke.com
// "Zyphra ZYFA", sections "Lean P" and "ブロックごとのスケーリングと丸められた
// 行和"): the e4m3 bit pattern read as an integer grows by 8 per doubling, so
// the code of 2^x is about 8x + 56; each 64-key block of P is multiplied by a
// power of two before rounding and the block-scaled matrix instruction removes
// that factor again.
//
// Exact fp32 steps (every step rounds to nearest-even in fp32; the FMAs are
// fused):
//   A    = (q_s * k_s) * C,  C = fp32(8 log2(e) / sqrt(Dqk))     per head pair
//   j    = 8 if the block has no live key, else
//          min(126, 8 + floor(((m - bmax) * A) * 0.125))         per row, block
//   B    = fma(-m, A, 56 + 8 j)                                   per row, block
//   u    = fma(s, A, B)                                           per element
//   code = trunc(max(u, 0))           (see leanp_code_word)
// s is the raw fp32 score (sum of products of e4m3 values), m the reference
// row maximum after this key tile and bmax the maximum of the element's 64-key
// block.  The reference max is deferred: it moves only when a tile's max
// exceeds it by more than 64 binades, so a block max may lie above m by up to
// that much, (bmax - m) A <= 512, and then j = 8 + floor of a negative number
// is -56..7.  Precondition: s <= bmax (or s = -inf for a masked key) and
// j >= -56.  Then the block max lands at u = 120 - 8 frac(((m - bmax) A) / 8),
// in (112, 120] (one lower where the fp32 steps round across an integer),
// every other u is below it, and the code never exceeds 126 (127 would be
// NaN; the device code does not clamp at 126 and relies on this bound).  The
// weight the matrix unit applies is value(code) * 2^-j: E8M0 scale code
// 127 - j, in 1 .. 183 (2^-126 .. 2^56) for j in -56 .. 126.
#pragma once
#include <cstdint>

namespace zyfa {

__device__ __forceinline__ float leanp_slope(float q_s, float k_s, float C) {
  return __fmul_rn(__fmul_rn(q_s, k_s), C);
}

__device__ __forceinline__ int leanp_block_shift(float m, float bmax, float A) {
  if (bmax == __int_as_float(0xff800000)) return 8;   // -inf: no live key in the block
  const float f = floorf(__fmul_rn(__fmul_rn(__fsub_rn(m, bmax), A), 0.125f));
  return f >= 118.0f ? 126 : 8 + static_cast<int>(f);
}

__device__ __forceinline__ float leanp_row_offset(float m, float A, int j) {
  return __fmaf_rn(-m, A, static_cast<float>(56 + 8 * j));
}

// The code of one score is computed as (leanp_code_word)
//   x = sat(fma(s, A/256, B/256))       (= fp32(u)/256 clamped to [0, 1]; the
//                                         division by 256 is exact and commutes
//                                         with the rounding for normal values)
//   w = fma_rz(x, 2^-141, 0)             (= trunc(256 x) * 2^-149 exactly)
// x * 2^-141 = (256 x) * 2^-149 lies below 2^-126, so the round-toward-zero FMA
// lands on the subnormal grid, whose spacing is 2^-149: w is the subnormal
// with fraction field trunc(256 x), and its bit pattern read as an integer is
// trunc(max(u, 0)) for 0 <= u < 256.  Two FMA-pipe instructions per score, no
// integer conversion; a256 = A/256 and b256 = B/256 are computed once per
// (row, block).
__device__ __forceinline__ float leanp_scaled_u(float s, float a256, float b256) {
  float x;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(x) : "f"(s), "f"(a256), "f"(b256));
  return x;
}

__device__ __forceinline__ uint32_t leanp_word(float x) {
  float w;
  asm("fma.rz.f32 %0, %1, 0f00000100, 0f00000000;" : "=f"(w) : "f"(x));   // x * 2^-141 + 0
  return __float_as_uint(w);
}

// One score -> its code as an integer (a256 = A/256, b256 = B/256).
__device__ __forceinline__ uint32_t leanp_code_word(float s, float a256, float b256) {
  return leanp_word(leanp_scaled_u(s, a256, b256));
}

// leanp_word for two values at once: one packed round-toward-zero FMA
// (fma.rz.f32x2 applies the same IEEE operation to each half, subnormal
// results included, so each word equals leanp_word's).
__device__ __forceinline__ void leanp_word2(float x0, float x1, uint32_t& w0, uint32_t& w1) {
  uint64_t x, w;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(x0), "f"(x1));
  asm("fma.rz.f32x2 %0, %1, %2, %3;" : "=l"(w) : "l"(x), "l"(0x0000010000000100ull), "l"(0ull));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(w0), "=r"(w1) : "l"(w));
}

// Two scores of one (row, block) -> two codes: the saturating FMA per score,
// then leanp_word2.
__device__ __forceinline__ void leanp_code_word2(float s0, float s1, float a256, float b256, uint32_t& w0,
                                                 uint32_t& w1) {
  leanp_word2(leanp_scaled_u(s0, a256, b256), leanp_scaled_u(s1, a256, b256), w0, w1);
}

// Four codes (integers below 256) -> one 32-bit word holding them as bytes in
// order.  cvt.pack.sat.u8.s32.b32 d, a, b, c sets d = sat_u8(b) | sat_u8(a) << 8
// | c << 16, so two of them pack four codes (three byte permutes did it before).
__device__ __forceinline__ uint32_t pack4_codes(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
  uint32_t hi, d;
  asm("cvt.pack.sat.u8.s32.b32 %0, %1, %2, %3;" : "=r"(hi) : "r"(w3), "r"(w2), "r"(0u));
  asm("cvt.pack.sat.u8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(w1), "r"(w0), "r"(hi));
  return d;
}

}  // namespace zyfa
