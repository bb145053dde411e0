// NF4 encode / decode building blocks shared by the quantize, dequantize and
// fused dequant-GEMM kernels.
//
// Decode.  A weight w' = bf16(fp32(q_code * a')) depends only on the 4-bit
// code and the block's constant a', so each 64-element block first builds its
// 16-entry bf16 table with 16 float32 multiplies, then every element is a
// table lookup.  The table lives in eight registers as byte planes (low and
// high byte of entries 0-7 and 8-15); `prmt` looks up four codes per
// instruction and a bit-select on bit 3 of each code merges the two halves.
//
// Encode.  code = argmin_i |fp32(x / c_b) - q_i| (ties to the lower index) is
// computed without the division: the code counts the thresholds
// T_j = RU_bf16(B_j * c_b) that x reaches, where B_j is the rounding boundary
// (in x / c_b) at which the float32 quotient first lands on the j-th
// nearest-level switch point.  B_j has 25 significant bits, so B_j * c_b is
// exact in float64 and never equal to a bfloat16 x; x >= T_j is therefore
// exactly "fp32(x / c_b) is past the j-th midpoint".  The count is a 4-step
// binary search over packed bf16 pairs.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace qlora {

struct Nf4Params {
  float q[16];       // NF4 levels, ascending, float32
  double bnd[15];    // boundary B_j in x / c_b between code j and code j + 1
  int centred;       // constants coded as E4M3 of (c_b - mu), see block_constant
};

// fp32(k / 255): level k of the 8-bit code of the absmax constants.
__device__ __forceinline__ float level2_value(uint32_t k) {
  return __fdiv_rn(static_cast<float>(k), 255.0f);
}

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v) {
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  return bf162_bits(__floats2bfloat162_rn(lo, hi));
}

// ------------------------------------------------------------------ decode
struct Nf4Lut {
  uint32_t la0, la1, lb0, lb1;  // low bytes of entries 0-3, 4-7, 8-11, 12-15
  uint32_t ha0, ha1, hb0, hb1;  // high bytes
};

__device__ __forceinline__ Nf4Lut make_lut(const Nf4Params& P, float a) {
  uint32_t t[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) t[k] = pack_bf16x2_rn(__fmul_rn(P.q[2 * k], a), __fmul_rn(P.q[2 * k + 1], a));
  Nf4Lut L;
  L.la0 = prmt(t[0], t[1], 0x6420);
  L.la1 = prmt(t[2], t[3], 0x6420);
  L.lb0 = prmt(t[4], t[5], 0x6420);
  L.lb1 = prmt(t[6], t[7], 0x6420);
  L.ha0 = prmt(t[0], t[1], 0x7531);
  L.ha1 = prmt(t[2], t[3], 0x7531);
  L.hb0 = prmt(t[4], t[5], 0x7531);
  L.hb1 = prmt(t[6], t[7], 0x7531);
  return L;
}

// One 32-bit word of packed codes (byte j holds elements 2j in the high
// nibble and 2j+1 in the low nibble) -> 8 bf16 values in element order,
// as four bf16x2 words (lower element in the low half).
//
// prmt reads only the low 16 bits of its selector, one nibble per output
// byte; a nibble with bit 3 set returns a sign-replicated byte instead of a
// table byte.  The low table (entries 0-7) is therefore indexed with the code
// word itself -- codes 8-15 give junk there, which the select discards -- and
// the high table (entries 8-15) with the word XOR 0x8888...; the upper half of
// the word is brought down with a multiply-high so that the shift runs on
// the multiply pipe rather than the logic pipe.
__device__ __forceinline__ void decode8(const Nf4Lut& L, uint32_t w, uint32_t (&out)[4]) {
  const uint32_t w4 = w << 4;
  // Byte k of the mask is 0xFF when the code at nibble k has bit 3 set
  // (prmt sign-replicate mode on the byte that carries that bit at its top).
  const uint32_t m0 = prmt(w, w4, 0x9D8C);
  const uint32_t m1 = prmt(w, w4, 0xBFAE);
  const uint32_t wx = w ^ 0x88888888u;
  const uint32_t wh = __umulhi(w, 0x10000u);   // w >> 16
  const uint32_t wxh = __umulhi(wx, 0x10000u);
  // Nibbles 0..3 hold elements 1, 0, 3, 2.
  uint32_t lo = lop3_sel(prmt(L.la0, L.la1, w), prmt(L.lb0, L.lb1, wx), m0);
  uint32_t hi = lop3_sel(prmt(L.ha0, L.ha1, w), prmt(L.hb0, L.hb1, wx), m0);
  out[0] = prmt(lo, hi, 0x4051);
  out[1] = prmt(lo, hi, 0x6273);
  // Nibbles 4..7 hold elements 5, 4, 7, 6.
  lo = lop3_sel(prmt(L.la0, L.la1, wh), prmt(L.lb0, L.lb1, wxh), m1);
  hi = lop3_sel(prmt(L.ha0, L.ha1, wh), prmt(L.hb0, L.hb1, wxh), m1);
  out[2] = prmt(lo, hi, 0x4051);
  out[3] = prmt(lo, hi, 0x6273);
}

// Value of an 8-bit E4M3 code (1 sign, 4 exponent bits with bias 7, 3
// mantissa bits; subnormals at exponent 0).  Exact in float32.
__device__ __forceinline__ float e4m3_value(uint32_t k) {
  const uint32_t e = (k >> 3) & 15u, m = k & 7u;
  const float v = e == 0 ? static_cast<float>(m) * 0.001953125f  // m * 2^-9
                         : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (k & 0x80u) ? -v : v;
}

// Level k of the 8-bit constant code: k / 255 (unsigned linear) or the
// E4M3 value (mean-centred 8-bit float scheme).
__device__ __forceinline__ float level2_value_for(uint32_t k, int centred) {
  return centred ? e4m3_value(k) : level2_value(k);
}

// a' = fp32(fp32(level(k) * c1) + mu), with mu = 0 for the linear scheme
// (adding +0 to a non-negative product leaves its bits unchanged).
__device__ __forceinline__ float block_constant(uint32_t code2, float c1, int centred, float mu) {
  return __fadd_rn(__fmul_rn(level2_value_for(code2, centred), c1), mu);
}

// mu of the mean-centred scheme: stored after the NB2 group scales.
__device__ __forceinline__ float centred_mu(const float* absmax_scale, int64_t nb2, int centred) {
  return centred ? __ldg(absmax_scale + nb2) : 0.0f;
}

// ------------------------------------------------------------------ encode
__device__ __forceinline__ uint32_t set_ge_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.ge.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Smallest bf16 >= the exact product B_j * c, replicated in both halves.
__device__ __forceinline__ uint32_t threshold_pair(double bnd, float c) {
  const float f = __double2float_ru(bnd * static_cast<double>(c));
  const __nv_bfloat16 h = __float2bfloat16_ru(f);
  const uint32_t b = static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&h));
  return b | (b << 16);
}

struct Nf4Thresholds {
  uint32_t t[15];
};

__device__ __forceinline__ Nf4Thresholds make_thresholds(const Nf4Params& P, float c) {
  Nf4Thresholds T;
  const float cc = (c > 0.0f) ? c : 1.0f;  // all-zero block: every x is 0 -> code 7
#pragma unroll
  for (int j = 0; j < 15; ++j) T.t[j] = threshold_pair(P.bnd[j], cc);
  return T;
}

// Codes of two bf16 values (low half, high half): the low byte of each
// 16-bit half holds that value's code in both nibbles (bits 8-15 are not
// defined).  A 4-step binary search over the 15 thresholds.
__device__ __forceinline__ uint32_t encode_pair(const Nf4Thresholds& T, uint32_t x) {
  const uint32_t m3 = set_ge_bf16x2(x, T.t[7]);
  const uint32_t m2 = set_ge_bf16x2(x, lop3_sel(T.t[3], T.t[11], m3));
  const uint32_t c01 = lop3_sel(T.t[1], T.t[5], m2);
  const uint32_t c23 = lop3_sel(T.t[9], T.t[13], m2);
  const uint32_t m1 = set_ge_bf16x2(x, lop3_sel(c01, c23, m3));
  const uint32_t d0 = lop3_sel(T.t[0], T.t[2], m1);
  const uint32_t d1 = lop3_sel(T.t[4], T.t[6], m1);
  const uint32_t d2 = lop3_sel(T.t[8], T.t[10], m1);
  const uint32_t d3 = lop3_sel(T.t[12], T.t[14], m1);
  const uint32_t e0 = lop3_sel(d0, d1, m2);
  const uint32_t e1 = lop3_sel(d2, d3, m2);
  const uint32_t m0 = set_ge_bf16x2(x, lop3_sel(e0, e1, m3));
  const uint32_t r1 = lop3_sel(m2, m3, 0x00880088u);  // bits 3 and 7 from m3, 2 and 6 from m2
  const uint32_t r2 = lop3_sel(m0, m1, 0x00220022u);  // bits 1 and 5 from m1, 0 and 4 from m0
  return lop3_sel(r2, r1, 0x00CC00CCu);
}

// Four encoded pairs (8 elements in order) -> one packed 32-bit code word,
// byte b = code of element 2b in the high nibble, element 2b + 1 in the low.
__device__ __forceinline__ uint32_t pack_codes8(uint32_t d0, uint32_t d1, uint32_t d2, uint32_t d3) {
  // bytes [e0 e0, e1 e1, e2 e2, e3 e3], then byte 0 = e0 | e1, byte 2 = e2 | e3
  const uint32_t wa = prmt(d0, d1, 0x6420u);
  const uint32_t wb = prmt(d2, d3, 0x6420u);
  const uint32_t ya = lop3_sel(wa >> 8, wa, 0xF0F0F0F0u);
  const uint32_t yb = lop3_sel(wb >> 8, wb, 0xF0F0F0F0u);
  return prmt(ya, yb, 0x6420u);
}

}  // namespace qlora
