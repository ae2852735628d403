// kvq_encode.cuh -- per-thread encoders of the three cache formats, shared by
// the append kernels and the fused decode step.
//
// One thread owns 8 consecutive head_dim values of one token; a block or
// group that spans several threads reduces with warp shuffles, so every lane
// of the warp must call these.  Arithmetic is IEEE binary32 with explicit
// round-to-nearest intrinsics, so the codes equal the format definitions:
//   NVFP4 (NVFP4 KV-cache article, glsqs.com/news/814573, section 2.1, with
//         the per-tensor FP32 scale g = amax/(6*448)):
//         bs = E4M3((blockamax / 6) / g), eff = float(bs) * g,
//         code_i = E2M1(x_i / eff)   (eff == 0 -> all codes 0)
//   INT4  ("KV缓存量化技术：提升大模型长文本生成效率", section 2.1):
//         S = (max - min) / 15, Z = rint(-min / S),
//         q = clamp(rint(x / S) + Z, 0, 15); a constant group uses
//         S = |min| (1 when min == 0)
//   FP8   ("KV Cache量化实战", --kv_cache_qformat table, fp8):
//         code = E4M3(x / s)
#pragma once

#include "kvq_device.cuh"

namespace kvq {

__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}

// Codes of quotients x / d without one IEEE division per value.  With
// r = RN(1/d), r_dn = RN(r (1 - 2^-20)) and r_up = RN(r (1 + 2^-20)), the
// products RN(|x| r_dn) and RN(|x| r_up) enclose the correctly rounded
// quotient RN(|x| / d): the roundings of r, of the margin factor and of the
// product move a value by at most 2^-24 of itself each, and RN(|x| / d)
// lies within 2^-24 of |x| / d, all far inside the 2^-20 margin.  Every
// code here is a rounding to a fixed grid (E2M1, E4M3, integers), monotonic
// in the quotient, so where both ends of the enclosure give the same code
// that is the code of RN(x / d).  Otherwise -- a quotient within a few ulps
// of a decision boundary, or a reciprocal too large for the margin -- the
// value is divided exactly.
struct RecipBounds {
  float dn, up;
  bool ok;
};
__device__ __forceinline__ RecipBounds recip_bounds(float d) {
  const float r = __frcp_rn(d);
  RecipBounds q;
  q.dn = __fmul_rn(r, 1.0f - 0x1p-20f);
  q.up = __fmul_rn(r, 1.0f + 0x1p-20f);
  q.ok = r < 3.0e38f;   // finite, and the upper factor stays finite
  return q;
}

// Two E4M3 codes of non-negative floats in one 16-bit word (`lo` in the low byte).
__device__ __forceinline__ uint32_t e4m3x2_rn_sat_nonneg(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// E2M1 pair code (low nibble = a) of RN(|a| / d), RN(|b| / d), signs not attached.
__device__ __forceinline__ uint32_t e2m1x2_of_quotients(float a, float b, float d, const RecipBounds& q) {
  a = fabsf(a);
  b = fabsf(b);
  const uint32_t c = e2m1x2_rn_sat_nonneg(__fmul_rn(a, q.dn), __fmul_rn(b, q.dn));
  if (q.ok && c == e2m1x2_rn_sat_nonneg(__fmul_rn(a, q.up), __fmul_rn(b, q.up))) return c;
  return e2m1x2_rn_sat_nonneg(__fdiv_rn(a, d), __fdiv_rn(b, d));
}

// E4M3 pair codes (low byte = a) of RN(|a| / d), RN(|b| / d), signs not attached.
__device__ __forceinline__ uint32_t e4m3x2_of_quotients(float a, float b, float d, const RecipBounds& q) {
  a = fabsf(a);
  b = fabsf(b);
  const uint32_t c = e4m3x2_rn_sat_nonneg(__fmul_rn(a, q.dn), __fmul_rn(b, q.dn));
  if (q.ok && c == e4m3x2_rn_sat_nonneg(__fmul_rn(a, q.up), __fmul_rn(b, q.up))) return c;
  return e4m3x2_rn_sat_nonneg(__fdiv_rn(a, d), __fdiv_rn(b, d));
}

// rint(RN(x / d)) for the affine formats (|x / d| stays far below 2^31).
__device__ __forceinline__ int rint_of_quotient(float x, float d, const RecipBounds& q) {
  const float lo = rintf(__fmul_rn(x, q.dn)), hi = rintf(__fmul_rn(x, q.up));
  if (q.ok && lo == hi) return (int)lo;
  return (int)rintf(__fdiv_rn(x, d));
}

// Group statistics of the affine formats over the GROUP values that
// GROUP/8 aligned lanes hold: S = (max - min) / QMAX (|min|, or 1, for a
// constant group), Z = rint(-min / S).
template <int GROUP, int QMAX>
__device__ __forceinline__ void affine_group(const float (&x)[8], float& mn, float& S) {
  constexpr int TPG = GROUP / 8;
  mn = x[0];
  float mx = x[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    mn = fminf(mn, x[i]);
    mx = fmaxf(mx, x[i]);
  }
#pragma unroll
  for (int off = 1; off < TPG; off <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  if (mx == mn)
    S = (mn != 0.0f) ? fabsf(mn) : 1.0f;
  else
    S = __fdiv_rn(__fsub_rn(mx, mn), (float)QMAX);
}

// Compact group metadata: S rounded to binary16 (nearest even; saturated at
// 65504, and 2^-24 if it would round to 0); returns that S as a float.
__device__ __forceinline__ float compact_scale(float S32, __half& S16) {
  __half h = __float2half_rn(S32);
  if (__hisinf(h)) h = __ushort_as_half((unsigned short)0x7BFFu);        // 65504
  if (__half2float(h) == 0.0f) h = __ushort_as_half((unsigned short)0x0001u);   // 2^-24
  S16 = h;
  return __half2float(h);
}

// The 8 codes clamp(rint(x_i / S) + Z, 0, QMAX).
template <int QMAX>
__device__ __forceinline__ void affine_codes8(const float (&x)[8], float S, int Z, int (&q)[8]) {
  const RecipBounds rb = recip_bounds(S);
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = min(max(rint_of_quotient(x[i], S, rb) + Z, 0), QMAX);
}

// NVFP4: 8 values of one 16-value block (the partner lane, lane ^ 1, holds
// the other 8).  Codes packed element i -> nibble i; the block's E4M3 scale.
__device__ __forceinline__ void nvfp4_encode8(const float (&x)[8], float g, uint32_t& packed,
                                              uint32_t& bs) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));   // partner half of the block
  const float tq = __fdiv_rn(amax, 6.0f);
  const float u = __fdiv_rn(tq, g);
  bs = e4m3_rn_sat_nonneg(u);
  const float eff = __fmul_rn(e4m3_to_f32(bs), g);
  packed = 0;
  if (eff != 0.0f) {
    const RecipBounds rb = recip_bounds(eff);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      uint32_t c = e2m1x2_of_quotients(x[i], x[i + 1], eff, rb);
      c |= (__float_as_uint(x[i]) >> 28) & 0x8u;        // signs (eff > 0)
      c |= (__float_as_uint(x[i + 1]) >> 24) & 0x80u;
      packed |= c << (4 * i);
    }
  }
}

// Pair-interleaved NVFP4 V bytes of 8 dims: byte i = code_a(i) | code_b(i) << 4
// (token a = the even token of the pair), as two words (dims 0-3, 4-7).
__device__ __forceinline__ uint2 nvfp4_pair_bytes(uint32_t pa, uint32_t pb) {
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    lo |= (((pa >> (4 * i)) & 0xFu) | (((pb >> (4 * i)) & 0xFu) << 4)) << (8 * i);
    hi |= (((pa >> (4 * (i + 4))) & 0xFu) | (((pb >> (4 * (i + 4))) & 0xFu) << 4)) << (8 * i);
  }
  return make_uint2(lo, hi);
}

// FP8: 8 independent E4M3 codes (little-endian bytes).
__device__ __forceinline__ uint2 fp8_encode8(const float (&x)[8], float s) {
  const RecipBounds rb = recip_bounds(s);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    uint32_t c = e4m3x2_of_quotients(x[i], x[i + 1], s, rb);
    c |= (__float_as_uint(x[i]) >> 24) & 0x80u;          // signs (s > 0)
    c |= (__float_as_uint(x[i + 1]) >> 16) & 0x8000u;
    w[i >> 2] |= c << (8 * (i & 3));
  }
  return make_uint2(w[0], w[1]);
}

// INT4 affine: 8 values of a GROUP-value group spread over GROUP/8 lanes
// (aligned).  Codes packed element i -> nibble i; the group's S and Z.
template <int GROUP>
__device__ __forceinline__ uint32_t int4_encode8(const float (&x)[8], float& S, int& Z) {
  float mn;
  affine_group<GROUP, 15>(x, mn, S);
  Z = (int)rintf(__fdiv_rn(-mn, S));
  int q[8];
  affine_codes8<15>(x, S, Z, q);
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) packed |= (uint32_t)q[i] << (4 * i);
  return packed;
}

// INT4 affine with compact group metadata: S is the binary32 (max - min) / 15
// rounded to binary16 (nearest even; saturated at 65504, and 2^-24 if it
// would round to 0); Z = clamp(round(-min / S16), -128, 127) and the codes
// are taken with that S16, so that (q - Z) * S16 decodes them.
template <int GROUP>
__device__ __forceinline__ uint32_t int4_encode8_compact(const float (&x)[8], __half& S16, int& Z) {
  float mn, S32;
  affine_group<GROUP, 15>(x, mn, S32);
  const float S = compact_scale(S32, S16);
  Z = min(max((int)rintf(__fdiv_rn(-mn, S)), -128), 127);
  int q[8];
  affine_codes8<15>(x, S, Z, q);
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) packed |= (uint32_t)q[i] << (4 * i);
  return packed;
}

// INT8 affine: the same scheme with 255 levels; codes one byte per value
// (element i in byte i of the returned pair of words).
template <int GROUP>
__device__ __forceinline__ uint2 int8_encode8(const float (&x)[8], float& S, int& Z) {
  float mn;
  affine_group<GROUP, 255>(x, mn, S);
  Z = (int)rintf(__fdiv_rn(-mn, S));
  int q[8];
  affine_codes8<255>(x, S, Z, q);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i >> 2] |= (uint32_t)q[i] << (8 * (i & 3));
  return make_uint2(w[0], w[1]);
}

// INT8 with compact group metadata: S as binary16 (see compact_scale) and Z
// clamped to the int16 range (zero points of 8-bit groups that span zero
// lie in 0 .. 255, beyond int8).
template <int GROUP>
__device__ __forceinline__ uint2 int8_encode8_compact(const float (&x)[8], __half& S16, int& Z) {
  float mn, S32;
  affine_group<GROUP, 255>(x, mn, S32);
  const float S = compact_scale(S32, S16);
  Z = min(max((int)rintf(__fdiv_rn(-mn, S)), -32768), 32767);
  int q[8];
  affine_codes8<255>(x, S, Z, q);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i >> 2] |= (uint32_t)q[i] << (8 * (i & 3));
  return make_uint2(w[0], w[1]);
}

// INT8 V rows are stored with a fixed permutation of head_dim: byte
// 16r + 2m + h (r, m = 0..7, h = 0, 1) holds dim 16m + r + 8h, so the 16
// dims a decode thread with row index r multiplies are one 16-byte chunk.
// For the 8 dims 8 part + e of a lane: byte 16e + part.
__device__ __forceinline__ int int8_v_byte_of_dim(int d) {
  return 16 * (d & 7) + 2 * (d >> 4) + ((d >> 3) & 1);
}

// The 16 lanes lane_base .. lane_base+15 hold one row's codes in natural
// order (lane `part`: dims 8 part + e in byte e of {lo, hi}); returns words
// `part` and `part` + 16 of the permuted row in w0, w1.  All 32 lanes call it.
__device__ __forceinline__ void int8_v_permute_words(uint2 codes, int part, int lane_base,
                                                     uint32_t& w0, uint32_t& w1) {
  // word w holds bytes 4w .. 4w+3 = 16e + p with e = w / 4, p = 4 (w % 4) + i
  w0 = 0u;
  w1 = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int src = lane_base + 4 * (part & 3) + i;
    const uint32_t lo = __shfl_sync(0xffffffffu, codes.x, src);   // e = 0..3
    const uint32_t hi = __shfl_sync(0xffffffffu, codes.y, src);   // e = 4..7
    const int e = part >> 2;                                      // word part: e = part / 4
    w0 |= ((lo >> (8 * e)) & 0xFFu) << (8 * i);
    w1 |= ((hi >> (8 * e)) & 0xFFu) << (8 * i);                   // word part+16: e = 4 + part / 4
  }
}

// INT4 V rows are stored with a fixed permutation of head_dim: byte 8r + m
// (r, m = 0..7) of a token's 64-byte row holds dim 16m + r in its low nibble
// and dim 16m + r + 8 in its high nibble.  Then the 16 dims a decode thread
// with row index r multiplies are one 8-byte chunk, and the dims of each
// 16-row MMA tile m stay inside one quantization group (32 or 64 dims).
// (The K rows keep the natural order: element 2i in the low nibble of byte i.)
__device__ __forceinline__ int int4_v_byte_of_dim(int d) { return 8 * (d & 7) + (d >> 4); }
__device__ __forceinline__ int int4_v_nibble_of_dim(int d) { return (d >> 3) & 1; }

// The 16 lanes lane_base .. lane_base+15 hold one row's codes in natural
// order (lane `part`: dims 8 part .. 8 part + 7, dim 8 part + e in nibble e);
// returns word `part` of the permuted row.  All 32 lanes of the warp call it.
__device__ __forceinline__ uint32_t int4_v_permute_word(uint32_t packed, int part, int lane_base) {
  const int r = part >> 1;
  uint32_t out = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = 4 * (part & 1) + i;   // byte 4 part + i = 8 r + m
    const uint32_t lo = __shfl_sync(0xffffffffu, packed, lane_base + 2 * m);       // dim 16m + r
    const uint32_t hi = __shfl_sync(0xffffffffu, packed, lane_base + 2 * m + 1);   // dim 16m + r + 8
    out |= (((lo >> (4 * r)) & 0xFu) | (((hi >> (4 * r)) & 0xFu) << 4)) << (8 * i);
  }
  return out;
}

// INT2 affine: the same scheme with 3 levels; a lane's 8 codes fill 16 bits,
// element i in bits 2i .. 2i+1.  Permuted V rows: the code of dim
// d = 16m + 8h + r (r < 8, h < 2) sits in byte 4r + m/2 at bits 2(2(m%2) + h).
template <int GROUP>
__device__ __forceinline__ uint32_t int2_encode8(const float (&x)[8], float& S, int& Z) {
  float mn;
  affine_group<GROUP, 3>(x, mn, S);
  Z = (int)rintf(__fdiv_rn(-mn, S));
  int q[8];
  affine_codes8<3>(x, S, Z, q);
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) packed |= (uint32_t)q[i] << (2 * i);
  return packed;
}

// INT2 with compact group metadata: S as binary16, Z clamped to int8.
template <int GROUP>
__device__ __forceinline__ uint32_t int2_encode8_compact(const float (&x)[8], __half& S16, int& Z) {
  float mn, S32;
  affine_group<GROUP, 3>(x, mn, S32);
  const float S = compact_scale(S32, S16);
  Z = min(max((int)rintf(__fdiv_rn(-mn, S)), -128), 127);
  int q[8];
  affine_codes8<3>(x, S, Z, q);
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) packed |= (uint32_t)q[i] << (2 * i);
  return packed;
}

// Byte and bit position of dim d in a permuted INT2 V row.
__device__ __forceinline__ int int2_v_byte_of_dim(int d) { return 4 * (d & 7) + (d >> 5); }
__device__ __forceinline__ int int2_v_shift_of_dim(int d) { return 2 * ((d >> 3) & 3); }

// The 16 lanes lane_base .. lane_base+15 hold one row's codes in natural
// order (lane `part`: dims 8 part .. 8 part + 7); returns bytes 2 part and
// 2 part + 1 of the permuted row in its low 16 bits.  Byte 4r + j holds dims
// 32j + 8k + r (k = 0..3, bits 2k), which lane 4j + k holds at bits 2r.  All
// 32 lanes of the warp call it.
__device__ __forceinline__ uint32_t int2_v_permute_half(uint32_t packed, int part, int lane_base) {
  const int r = part >> 1;
  uint32_t out = 0;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int j = 2 * (part & 1) + e;      // byte 2 part + e = 4 r + j
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t w = __shfl_sync(0xffffffffu, packed, lane_base + 4 * j + k);
      out |= ((w >> (2 * r)) & 3u) << (8 * e + 2 * k);
    }
  }
  return out;
}

}  // namespace kvq
