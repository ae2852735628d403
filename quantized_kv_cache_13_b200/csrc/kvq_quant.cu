// kvq_quant.cu -- quantize-and-append, calibration, ring copy and
// dequantize kernels for the three cache formats (sm_100a).
//
// Thread mappings: the bulk quantizers give one thread 16 consecutive
// head_dim values of one token (NVFP4: 32, two blocks; two or four 16-byte
// BF16 loads), the per-pair NVFP4 kernel, INT8, the ring copy and the
// dequantizer 8 (one 16-byte load), so a warp covers two to eight tokens
// with fully coalesced loads and stores.  Groups that span several threads
// reduce their max / min with warp shuffles.
//
// Encode arithmetic is IEEE binary32 with explicit round-to-nearest
// intrinsics (no contraction, no approximate division) because the codes
// must be bit-identical to the format definitions:
//   NVFP4 (NVFP4 KV-cache article, glsqs.com/news/814573, section 2.1; the
//         two-level scale with a per-tensor FP32 scale amax/(6*448)):
//         bs = E4M3((blockamax / 6) / g), eff = float(bs) * g,
//         code_i = E2M1(x_i / eff)   (eff == 0 -> all codes 0)
//   INT4  ("KV缓存量化技术：提升大模型长文本生成效率", section 2.1):
//         S = (max - min) / 15, Z = rint(-min / S),
//         q = clamp(rint(x / S) + Z, 0, 15); a constant group uses
//         S = |min| (1 when min == 0)
//   FP8   ("KV Cache量化实战", --kv_cache_qformat table, fp8):
//         code = E4M3(x / s), s = amax / 448
// E2M1 / E4M3 rounding is round-to-nearest-even with saturation (hardware
// cvt ... .satfinite); negative values that round to zero keep their sign
// bit (the bulk encoders convert signed values, the per-value ones attach
// the sign).
#include <cuda_runtime.h>

#include <algorithm>

#include "kvq_device.cuh"
#include "kvq_encode.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int D = kHeadDim;
constexpr int kThreadsPerRow = D / 8;   // 16

// Per-tensor scale: either the stored one, or (calibrating) derived from the
// amax word: g = amax / divisor, 1 for an all-zero tensor.
__device__ __forceinline__ float tensor_scale(const QuantArgs& a, int kv, float divisor) {
  if (a.calibrate) {
    float amax = __uint_as_float(*a.amax[kv]);
    return amax == 0.0f ? 1.0f : __fdiv_rn(amax, divisor);
  }
  return *a.gscale[kv];
}

// The scale of main-cache token dtok: its segment's under scale renewal,
// else the per-tensor one (g).
__device__ __forceinline__ float token_scale(const QuantArgs& a, int kv, int64_t dtok, float g) {
  return a.renewal ? a.gseg[kv][(uint32_t)dtok / (uint32_t)a.renewal] : g;   // (positions < 2^32)
}

__device__ __forceinline__ void store_scale_once(const QuantArgs& a, int kv, float g) {
  if (a.calibrate && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *a.gscale_out[kv] = g;
}

// ---------------------------------------------------------------------------
// Whole-block encoders of the bulk kernels (one thread per 16 values).
// ---------------------------------------------------------------------------

// Packed E2M1 pair (lo nibble first) of signed floats straight from the
// hardware conversion: round to nearest even, saturating, the sign kept
// (a negative value that rounds to zero gives 0x8; checked on B200 against
// the explicit sign attach of e2m1x2_rn_sat over 5.4e8 values).
__device__ __forceinline__ uint32_t e2m1x2_cvt(float lo, float hi) {
  uint16_t d;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u16.u8 %0, t; }"
      : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// Packed E4M3 pair (lo in the low byte) of signed floats straight from the
// hardware conversion: round to nearest even, saturating to +-448, the
// sign kept (a negative value that rounds to zero gives 0x80).
__device__ __forceinline__ uint32_t e4m3x2_cvt(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// max(a, b, c) in one instruction (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// RN(x / d) without a division, by the correction step of Markstein's
// division (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990): with r =
// RN(1 / d) and q0 = RN(x r), within an ulp of x / d, the residual x - d q0
// is exactly representable and one FMA computes it exactly; RN(q0 + r (x -
// d q0)) is then the correctly rounded quotient, for normal operands whose
// quotient neither overflows nor underflows.  The callers keep to that
// range where it decides a code: they take this path only while r <
// kQuotientMaxRecip (d >= 2^-92, so for quotients of 2^-11 and above -- every
// quotient that can round to a nonzero code -- the residual is a multiple of
// 2^-149 and cannot underflow) and, for the float formats, while the
// largest product amax * r stays below 2^126 (no infinite q0, which the
// correction would turn into NaN); otherwise they divide.  The sign of a zero quotient is
// taken from x (the residual loses it for x = -0).  A CPU check over 4e7
// binary32 pairs (BF16 numerators, exact ties and their neighbours
// included) found no difference from the IEEE quotient, and the codes
// derived from it are checked against the oracle bit for bit.
__device__ __forceinline__ float rn_quotient(float x, float d, float r) {
  const float q0 = __fmul_rn(x, r);
  const float q = __fmaf_rn(__fmaf_rn(-q0, d, x), r, q0);
  return __uint_as_float((__float_as_uint(q) & 0x7FFFFFFFu) | (__float_as_uint(x) & 0x80000000u));
}

constexpr float kQuotientMaxRecip = 0x1p92f;
constexpr float kQuotientMaxProduct = 0x1p126f;

// rn_quotient for the integer codes: a zero quotient's sign is irrelevant
// there, so it is left as the FMA gives it.
__device__ __forceinline__ float rn_quotient_int(float x, float d, float r) {
  const float q0 = __fmul_rn(x, r);
  return __fmaf_rn(__fmaf_rn(-q0, d, x), r, q0);
}

// min(a, b, c) in one instruction (sm_100).
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// clamp(v, 0, hi) in one instruction (min with the result clamped at 0).
__device__ __forceinline__ int clamp0(int v, int hi) {
  int d;
  asm("min.relu.s32 %0, %1, %2;" : "=r"(d) : "r"(v), "r"(hi));
  return d;
}

// Minimum and maximum of 16 values with three-input min / max.
__device__ __forceinline__ void minmax16(const float (&x)[16], float& mn, float& mx) {
  mn = fminf(fmin3(fmin3(x[0], x[1], x[2]), fmin3(x[3], x[4], x[5]), fmin3(x[6], x[7], x[8])),
             fmin3(fmin3(x[9], x[10], x[11]), fmin3(x[12], x[13], x[14]), x[15]));
  mx = fmaxf(fmax3(fmax3(x[0], x[1], x[2]), fmax3(x[3], x[4], x[5]), fmax3(x[6], x[7], x[8])),
             fmax3(fmax3(x[9], x[10], x[11]), fmax3(x[12], x[13], x[14]), x[15]));
}

// NVFP4 for one whole 16-value block in one thread.  c6g = RN(1 / RN(6 g)):
// the block scale's argument RN(RN(amax / 6) / g) lies within 2.01 * 2^-24
// of amax / (6 g) and RN(amax * c6g) within 3.01 * 2^-24 of it, so
// RN(amax * c6g) * (1 -+ 2^-20) enclose it; the E4M3 code of both ends is
// the block scale unless they differ (then the two divisions are done
// exactly: one 16-value block per thread makes this branch rare and cheap,
// unlike the per-element one it replaced).  The element codes are the signed
// conversions of RN(x / eff) from rn_quotient (no bracket, no divergent
// exact path: BF16 inputs put quotients exactly on E2M1 midpoints often
// enough that a bracket's exact fallback left warps mostly idle).  Codes as
// nvfp4_encode8: element 2i in the low nibble of byte i of `codes`.
__device__ __forceinline__ void nvfp4_encode16(const float (&x)[16], float g, float c6g, bool c6g_ok,
                                               uint2& codes, uint32_t& bs) {
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(fabsf(x[2 * i]), fabsf(x[2 * i + 1]));
  const float amax = fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
  const float w = __fmul_rn(amax, c6g);
  const uint32_t b2 = e4m3x2_rn_sat_nonneg(__fmul_rn(w, 1.0f - 0x1p-20f), __fmul_rn(w, 1.0f + 0x1p-20f));
  if (c6g_ok && (b2 & 0xFFu) == (b2 >> 8))
    bs = b2 & 0xFFu;
  else
    bs = e4m3_rn_sat_nonneg(__fdiv_rn(__fdiv_rn(amax, 6.0f), g));
  const float eff = __fmul_rn(e4m3_to_f32(bs), g);
  const float r = __frcp_rn(eff);
  uint32_t wd[2] = {0u, 0u};
  if (r < kQuotientMaxRecip && __fmul_rn(amax, r) < kQuotientMaxProduct) {   // (eff != 0)
#pragma unroll
    for (int i = 0; i < 16; i += 2)
      wd[i >> 3] |= e2m1x2_cvt(rn_quotient(x[i], eff, r), rn_quotient(x[i + 1], eff, r)) << (4 * (i & 7));
  } else if (eff != 0.0f) {   // extreme scales: exact divisions
#pragma unroll
    for (int i = 0; i < 16; i += 2)
      wd[i >> 3] |= e2m1x2_cvt(__fdiv_rn(x[i], eff), __fdiv_rn(x[i + 1], eff)) << (4 * (i & 7));
  }   // else an all-zero block: all codes 0
  codes = make_uint2(wd[0], wd[1]);
}

// Interleave the low nibbles of two words' first four bytes' worth of codes:
// byte k of the result (k = 0..3) = nibble k of a | nibble k of b << 4.
__device__ __forceinline__ uint32_t nibble_interleave4(uint32_t a, uint32_t b) {
  auto spread = [](uint32_t v) {   // nibbles 0..3 of v -> low nibbles of bytes 0..3
    v &= 0xFFFFu;
    v = (v | (v << 8)) & 0x00FF00FFu;
    return (v | (v << 4)) & 0x0F0F0F0Fu;
  };
  return spread(a) | (spread(b) << 4);
}

// FP8 for 16 consecutive values: E4M3 codes (little-endian bytes) of the
// signed RN(x / s) from rn_quotient, with exact divisions outside its range
// (a scale below 2^-92, or values whose quotient would pass 2^126: then the
// IEEE quotient saturates, as the code must).
__device__ __forceinline__ uint4 fp8_encode16(const float (&x)[16], float s) {
  const float r = __frcp_rn(s);
  const float amax = fmaxf(
      fmax3(fmax3(fabsf(x[0]), fabsf(x[1]), fabsf(x[2])), fmax3(fabsf(x[3]), fabsf(x[4]), fabsf(x[5])),
            fmax3(fabsf(x[6]), fabsf(x[7]), fabsf(x[8]))),
      fmax3(fmax3(fabsf(x[9]), fabsf(x[10]), fabsf(x[11])), fmax3(fabsf(x[12]), fabsf(x[13]), fabsf(x[14])),
            fabsf(x[15])));
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  if (r < kQuotientMaxRecip && __fmul_rn(amax, r) < kQuotientMaxProduct) {
#pragma unroll
    for (int i = 0; i < 16; i += 2)
      w[i >> 2] |= e4m3x2_cvt(rn_quotient(x[i], s, r), rn_quotient(x[i + 1], s, r)) << (8 * (i & 3));
  } else {
#pragma unroll
    for (int i = 0; i < 16; i += 2)
      w[i >> 2] |= e4m3x2_cvt(__fdiv_rn(x[i], s), __fdiv_rn(x[i + 1], s)) << (8 * (i & 3));
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Quantize grids: x = blocks of 16 rows (16 threads per row, 8 values each),
// y = (batch, kv head) units (a block walks units in steps of gridDim.y),
// z = K (0) / V (1).  A row is a token (a token pair for the NVFP4 V plane),
// so no thread divides by a runtime length.
__device__ __forceinline__ int64_t row_in_unit() {
  return (int64_t)blockIdx.x * (blockDim.x / kThreadsPerRow) + (threadIdx.x / kThreadsPerRow);
}

// Plane row of token t of this launch's unit bh.
__device__ __forceinline__ int64_t qrow(const QuantArgs& a, int64_t bh, int64_t t) {
  return plane_row(a.unit0 + bh, t, a.cap, a.kv_heads, a.pages, a.page_tokens, a.max_pages);
}

// ---------------------------------------------------------------------------
// NVFP4: 2 threads per 16-element block.
// K is stored token-major (64 code bytes per token, element 2i in the low
// nibble of byte i).  V is stored pair-interleaved: byte d of the 128-byte
// row of token pair (2p, 2p+1) holds dim d of token 2p in the low nibble and
// of token 2p+1 in the high nibble, which is the order the decode kernel's
// V fragments want.  Block scales are one byte per (token, 16 dims) for both.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void load8(const QuantArgs& a, int kv, int64_t bh, int64_t t, int part,
                                      bool ok, float (&x)[8]) {
  if (ok) {
    unpack8(*reinterpret_cast<const uint4*>(a.src[kv] + bh * a.src_bh_stride + (a.src_tok0 + t) * D +
                                            part * 8),
            x);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = 0.0f;
  }
}

__global__ void __launch_bounds__(256) quantize_nvfp4_kernel(QuantArgs a) {
  const int kv = blockIdx.z;
  const float g_tensor = a.renewal ? 1.0f : tensor_scale(a, kv, 2688.0f);
  if (!a.renewal) store_scale_once(a, kv, g_tensor);
  const int part = threadIdx.x % kThreadsPerRow;     // 8-element piece of the row
  const int64_t row = row_in_unit();
  if (kv == 0) {
    // K: one 16-thread row per token.  Rows past the end still take part in
    // the shuffles (on token 0) but store nothing.
    const bool valid = row < a.n;
    const int64_t t = valid ? row : 0;
    const float g = token_scale(a, 0, a.dst_tok0 + t, g_tensor);
    for (int64_t bh = blockIdx.y; bh < a.bh; bh += gridDim.y) {
      float x[8];
      load8(a, 0, bh, t, part, true, x);
      uint32_t packed, bs;
      nvfp4_encode8(x, g, packed, bs);
      if (!valid) continue;
      const int64_t dtok = a.dst_tok0 + t;
      const int64_t r = qrow(a, bh, dtok);
      *reinterpret_cast<uint32_t*>(a.dst[0].codes + r * (D / 2) + part * 4) = packed;
      if ((part & 1) == 0) a.dst[0].meta[r * (D / 16) + part / 2] = (uint8_t)bs;
    }
    return;
  }
  // V: one 16-thread row per destination token pair touched by this append.
  const int64_t p_first = a.dst_tok0 >> 1;
  const int64_t npairs = ((a.dst_tok0 + a.n - 1) >> 1) - p_first + 1;
  const bool valid = row < npairs;
  const int64_t pair = p_first + (valid ? row : 0);
  const int64_t ta = 2 * pair - a.dst_tok0, tb = ta + 1;   // source token indices
  const bool va = valid && ta >= 0 && ta < a.n, vb = valid && tb >= 0 && tb < a.n;
  // both tokens of a pair lie in one segment (segments are multiples of 16)
  const float g = token_scale(a, 1, 2 * pair, g_tensor);
  for (int64_t bh = blockIdx.y; bh < a.bh; bh += gridDim.y) {
    float xa[8], xb[8];
    load8(a, 1, bh, ta, part, va, xa);
    load8(a, 1, bh, tb, part, vb, xb);
    uint32_t pa, pb, sa, sb;
    nvfp4_encode8(xa, g, pa, sa);
    nvfp4_encode8(xb, g, pb, sb);
    if (!valid) continue;
    const uint2 pbytes = nvfp4_pair_bytes(pa, pb);   // byte i: dim part*8 + i of both tokens
    uint32_t lo = pbytes.x, hi = pbytes.y;
    const int64_t r = qrow(a, bh, 2 * pair);   // a pair never straddles a page
    uint2* dst = reinterpret_cast<uint2*>(a.dst[1].codes + r * (D / 2) + part * 8);
    if (!(va && vb)) {
      // only one token of the pair is new: keep the other token's nibbles
      const uint2 old = *dst;
      const uint32_t keep = va ? 0xF0F0F0F0u : 0x0F0F0F0Fu;
      lo = (lo & ~keep) | (old.x & keep);
      hi = (hi & ~keep) | (old.y & keep);
    }
    *dst = make_uint2(lo, hi);
    if ((part & 1) == 0) {
      if (va) a.dst[1].meta[r * (D / 16) + part / 2] = (uint8_t)sa;
      if (vb) a.dst[1].meta[(r + 1) * (D / 16) + part / 2] = (uint8_t)sb;
    }
  }
}

// NVFP4 bulk quantizer: one thread per two 16-value blocks (four 16-byte
// loads), four threads per token, 64 tokens per 256-thread CTA; z = K (0) /
// V (1).  Thread j of a token owns dims [32j, 32j + 32).  The destination's
// first token is even (the host sends an odd first token through
// quantize_nvfp4_kernel), so the two tokens of a V pair sit in lanes l and
// l ^ 4 of one warp: the even lane sends its partner the codes of its second
// block and receives the odd token's codes of its first block, so that the
// even lane writes the pair's bytes of dims [32j, 32j + 16) and the odd lane
// those of [32j + 16, 32j + 32).  A pair whose odd token lies past the
// append writes zero nibbles there (beyond the cache length; a later append
// of that token rewrites its nibbles only).
__global__ void __launch_bounds__(256) quantize_nvfp4_blocks_kernel(QuantArgs a) {
  const int kv = blockIdx.z;
  const float g_tensor = a.renewal ? 1.0f : tensor_scale(a, kv, 2688.0f);
  if (!a.renewal) store_scale_once(a, kv, g_tensor);
  const int j = threadIdx.x & 3;                                    // 32-dim chunk of the token
  const int64_t t = (int64_t)blockIdx.x * 64 + (threadIdx.x >> 2);  // token of the append
  const bool valid = t < a.n;
  const int64_t dtok = a.dst_tok0 + t;
  const float g = a.renewal ? a.gseg[kv][(uint32_t)dtok / (uint32_t)a.renewal] : g_tensor;   // (pairs share a segment)
  const float c6g = __frcp_rn(__fmul_rn(6.0f, g));
  const bool c6g_ok = c6g < 3.0e38f;
  const bool odd = (threadIdx.x >> 2) & 1;
  for (int64_t bh = blockIdx.y; bh < a.bh; bh += gridDim.y) {
    uint4 w[4] = {};
    if (valid) {
      const uint4* src = reinterpret_cast<const uint4*>(a.src[kv] + bh * a.src_bh_stride +
                                                        (a.src_tok0 + t) * D + j * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = src[i];
    }
    uint2 codes[2];
    uint32_t bs[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float x[16], lo[8], hi[8];
      unpack8(w[2 * h], lo);
      unpack8(w[2 * h + 1], hi);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        x[i] = lo[i];
        x[8 + i] = hi[i];
      }
      nvfp4_encode16(x, g, c6g, c6g_ok, codes[h], bs[h]);
    }
    const uint16_t scales = (uint16_t)(bs[0] | (bs[1] << 8));
    if (kv == 0) {
      if (valid) {
        const int64_t r = qrow(a, bh, dtok);
        *reinterpret_cast<uint4*>(a.dst[0].codes + r * (D / 2) + j * 16) =
            make_uint4(codes[0].x, codes[0].y, codes[1].x, codes[1].y);
        *reinterpret_cast<uint16_t*>(a.dst[0].meta + r * (D / 16) + 2 * j) = scales;
      }
      continue;
    }
    // V: the even token's second block goes to the odd lane, the odd
    // token's first block to the even lane
    const uint2 send = odd ? codes[0] : codes[1];
    const uint2 recv = make_uint2(__shfl_xor_sync(0xffffffffu, send.x, 4),
                                  __shfl_xor_sync(0xffffffffu, send.y, 4));
    const uint2 e = odd ? recv : codes[0];   // even token's codes of this lane's 16 dims
    const uint2 o = odd ? codes[1] : recv;   // odd token's codes of the same dims
    const int64_t t_even = t & ~(int64_t)1;
    if (t_even < a.n) {
      const int64_t r_even = qrow(a, bh, dtok & ~(int64_t)1);   // a pair never straddles a page
      *reinterpret_cast<uint4*>(a.dst[1].codes + r_even * (D / 2) + j * 32 + (odd ? 16 : 0)) =
          make_uint4(nibble_interleave4(e.x, o.x), nibble_interleave4(e.x >> 16, o.x >> 16),
                     nibble_interleave4(e.y, o.y), nibble_interleave4(e.y >> 16, o.y >> 16));
    }
    if (valid) *reinterpret_cast<uint16_t*>(a.dst[1].meta + qrow(a, bh, dtok) * (D / 16) + 2 * j) = scales;
  }
}

// ---------------------------------------------------------------------------
// FP8: independent elements, 16 per thread.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_fp8_kernel(QuantArgs a) {
  // 16 values per thread (two 16-byte loads), 8 threads per token, 32 tokens
  // per 256-thread CTA
  const int kv = blockIdx.z;
  const float s_tensor = a.renewal ? 1.0f : tensor_scale(a, kv, 448.0f);
  if (!a.renewal) store_scale_once(a, kv, s_tensor);
  const int64_t t = (int64_t)blockIdx.x * 32 + (threadIdx.x >> 3);
  if (t >= a.n) return;
  const float s = token_scale(a, kv, a.dst_tok0 + t, s_tensor);
  const int part = threadIdx.x & 7;
  for (int64_t bh = blockIdx.y; bh < a.bh; bh += gridDim.y) {
    const uint4* src = reinterpret_cast<const uint4*>(a.src[kv] + bh * a.src_bh_stride +
                                                      (a.src_tok0 + t) * D + part * 16);
    const uint4 w0 = src[0], w1 = src[1];
    float x[16], lo[8], hi[8];
    unpack8(w0, lo);
    unpack8(w1, hi);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[i] = lo[i];
      x[8 + i] = hi[i];
    }
    const int64_t dtok = a.dst_tok0 + t;
    *reinterpret_cast<uint4*>(a.dst[kv].codes + qrow(a, bh, dtok) * D + part * 16) = fp8_encode16(x, s);
  }
}

// ---------------------------------------------------------------------------
// INT4 affine, bulk: one thread per 16 consecutive head_dim values of one
// token (two 16-byte loads), 8 threads per token, 32 tokens per 256-thread
// CTA; a group of 64 (32) values is 4 (2) lanes.  The arithmetic is that of
// int4_encode8 / int4_encode8_compact: the group's min and max, S = (max -
// min) / 15 (|min|, or 1, for a constant group; binary16 with compact
// metadata), Z = rint(-min / S), q = clamp(rint(RN(x / S)) + Z, 0, 15).
// rint(RN(x / S)) is the quotient of rn_quotient_int rounded to an integer
// by adding 1.5 * 2^23 (exact for |x / S| < 2^22: BF16 inputs keep |x / S|
// below 15 * 2^8).
// ---------------------------------------------------------------------------
constexpr float kRintMagic = 12582912.0f;   // 1.5 * 2^23
constexpr uint32_t kRintMagicBits = 0x4B400000u;

// rint(qf) by the 1.5 * 2^23 addition.  Plain metadata keeps |qf| below
// QMAX * 2^8 for BF16 inputs; compact metadata may have saturated S at 65504
// below the group's (max - min) / QMAX, so quotients can pass 2^22 there:
// they are clamped to +-2^22 first, where every code saturates anyway (|Z|
// stays below 2^15).
template <bool COMPACT>
__device__ __forceinline__ int rint_code(float qf) {
  if constexpr (COMPACT) qf = fminf(fmaxf(qf, -0x1p22f), 0x1p22f);
  return (int)(__float_as_uint(__fadd_rn(qf, kRintMagic)) - kRintMagicBits);
}

template <int GROUP, bool COMPACT>
__device__ __forceinline__ uint2 int4_encode16(const float (&x)[16], float& S_out, __half& S16, int& Z) {
  constexpr int TPG = GROUP / 16;         // lanes per group (aligned)
  float mn, mx;
  minmax16(x, mn, mx);
#pragma unroll
  for (int off = 1; off < TPG; off <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  float S;
  if (mx == mn)
    S = (mn != 0.0f) ? fabsf(mn) : 1.0f;
  else
    S = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
  if constexpr (COMPACT) {
    S = compact_scale(S, S16);
    Z = min(max((int)rintf(__fdiv_rn(-mn, S)), -128), 127);
  } else {
    Z = (int)rintf(__fdiv_rn(-mn, S));
  }
  S_out = S;
  const float r = __frcp_rn(S);
  const bool rok = r < kQuotientMaxRecip;
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float qf = rok ? rn_quotient_int(x[i], S, r) : __fdiv_rn(x[i], S);
    w[i >> 3] |= (uint32_t)clamp0(rint_code<COMPACT>(qf) + Z, 15) << (4 * (i & 7));
  }
  return make_uint2(w[0], w[1]);
}

// The INT4 V row of one token from its 8 lanes' natural codes.  Lane j
// (dims 16j .. 16j + 15 = m-tile j) owns byte 8r + j of the permuted row for
// r = 0..7 (dim 16j + r in the low nibble, 16j + r + 8 in the high one); a
// three-step exchange among the 8 lanes (xor 4, 2, 1: each lane keeps the
// half whose position bit matches its own and trades the other) transposes
// those 8 x 8 bytes, after which lane t holds bytes 8t .. 8t + 7.
__device__ __forceinline__ uint2 int4_v_row_transpose(uint2 codes, int j) {
  uint32_t lo = 0u, hi = 0u;   // byte r = code r | code r + 8 << 4
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    lo |= (((codes.x >> (4 * r)) & 0xFu) | (((codes.y >> (4 * r)) & 0xFu) << 4)) << (8 * r);
    hi |= (((codes.x >> (4 * (r + 4))) & 0xFu) | (((codes.y >> (4 * (r + 4))) & 0xFu) << 4)) << (8 * r);
  }
  // xor 4: lanes 0-3 keep bytes 0-3 (lo) of their row and take their
  // partner's; lanes 4-7 keep bytes 4-7
  const bool j2 = j & 4, j1 = j & 2, j0 = j & 1;
  const uint32_t r4 = __shfl_xor_sync(0xffffffffu, j2 ? lo : hi, 4);
  const uint32_t a = j2 ? r4 : lo, b = j2 ? hi : r4;
  // xor 2: keep bytes with position bit 1 == j1
  const uint32_t keep2 = prmt(a, b, j1 ? 0x7632u : 0x5410u);
  const uint32_t r2 = __shfl_xor_sync(0xffffffffu, prmt(a, b, j1 ? 0x5410u : 0x7632u), 2);
  // xor 1: keep bytes with position bit 0 == j0
  const uint32_t keep1 = prmt(keep2, r2, j0 ? 0x7531u : 0x6420u);
  const uint32_t r1 = __shfl_xor_sync(0xffffffffu, prmt(keep2, r2, j0 ? 0x6420u : 0x7531u), 1);
  // order the eight bytes by source lane (the order depends on j & 3)
  const uint32_t flip = (j0 ? 0x4444u : 0u) ^ (j1 ? 0x2222u : 0u);
  return make_uint2(prmt(keep1, r1, 0x6240u ^ flip), prmt(keep1, r1, 0x7351u ^ flip));
}

template <int GROUP, bool COMPACT = false>
__global__ void __launch_bounds__(256) quantize_int4_wide_kernel(QuantArgs a) {
  constexpr int NG = D / GROUP;
  constexpr int TPG = GROUP / 16;
  const int kv = blockIdx.z;
  const int j = threadIdx.x & 7;                                      // dims [16j, 16j + 16)
  const int64_t t = (int64_t)blockIdx.x * 32 + (threadIdx.x >> 3);   // token of the append
  const bool valid = t < a.n;
  for (int64_t bh = blockIdx.y; bh < a.bh; bh += gridDim.y) {
    uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
    if (valid) {
      const uint4* src = reinterpret_cast<const uint4*>(a.src[kv] + bh * a.src_bh_stride +
                                                        (a.src_tok0 + t) * D + j * 16);
      w0 = src[0];
      w1 = src[1];
    }
    float x[16], lo[8], hi[8];
    unpack8(w0, lo);
    unpack8(w1, hi);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[i] = lo[i];
      x[8 + i] = hi[i];
    }
    float S;
    __half S16;
    int Z;
    uint2 codes = int4_encode16<GROUP, COMPACT>(x, S, S16, Z);
    if (kv == 1) codes = int4_v_row_transpose(codes, j);   // (block-uniform: all lanes)
    if (!valid) continue;
    const int64_t r = qrow(a, bh, a.dst_tok0 + t);
    *reinterpret_cast<uint2*>(a.dst[kv].codes + r * (D / 2) + j * 8) = codes;
    if (j % TPG == 0) {
      const int gi = j / TPG;
      if constexpr (COMPACT) {   // {f16 S0, f16 S1, i8 Z0, i8 Z1, 0, 0} per token
        uint8_t* m = a.dst[kv].meta + r * 8;
        *reinterpret_cast<__half*>(m + 2 * gi) = S16;
        m[4 + gi] = (uint8_t)(int8_t)Z;
      } else {
        uint32_t* meta = reinterpret_cast<uint32_t*>(a.dst[kv].meta) + (r * NG + gi) * 2;
        *reinterpret_cast<uint2*>(meta) = make_uint2(__float_as_uint(S), (uint32_t)Z);
      }
    }
  }
}

// INT8 affine codes of one lane's 8 values (element i in byte i), group
// statistics as int8_encode8 / int8_encode8_compact, the quotients x / S
// from rn_quotient (exact divisions when 1 / S is not finite).
template <int GROUP, bool COMPACT>
__device__ __forceinline__ uint2 int8_bulk_encode8(const float (&x)[8], float& S, __half& S16, int& Z) {
  float mn;
  affine_group<GROUP, 255>(x, mn, S);
  if constexpr (COMPACT) {
    S = compact_scale(S, S16);
    Z = min(max((int)rintf(__fdiv_rn(-mn, S)), -32768), 32767);
  } else {
    Z = (int)rintf(__fdiv_rn(-mn, S));
  }
  const float r = __frcp_rn(S);
  const bool rok = r < kQuotientMaxRecip;
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float qf = rok ? rn_quotient_int(x[i], S, r) : __fdiv_rn(x[i], S);
    w[i >> 2] |= (uint32_t)clamp0(rint_code<COMPACT>(qf) + Z, 255) << (8 * (i & 3));
  }
  return make_uint2(w[0], w[1]);
}

// INT8 affine: 8 bytes of codes per lane; V rows in the permuted dim order.
template <int GROUP, bool COMPACT = false>
__global__ void __launch_bounds__(256) quantize_int8_kernel(QuantArgs a) {
  constexpr int TPG = GROUP / 8;          // threads per group
  const int kv = blockIdx.z;
  const int part = threadIdx.x % kThreadsPerRow;
  const int64_t row = row_in_unit();
  const bool valid = row < a.n;           // see quantize_nvfp4_kernel
  const int64_t t = valid ? row : 0;
  for (int64_t bh = blockIdx.y; bh < a.bh; bh += gridDim.y) {
    const uint4 w = *reinterpret_cast<const uint4*>(a.src[kv] + bh * a.src_bh_stride +
                                                    (a.src_tok0 + t) * D + part * 8);
    float x[8];
    unpack8(w, x);
    float S;
    int Z;
    __half S16;
    const uint2 codes = int8_bulk_encode8<GROUP, COMPACT>(x, S, S16, Z);
    uint32_t w0 = 0u, w1 = 0u;
    if (kv == 1) int8_v_permute_words(codes, part, threadIdx.x & 16, w0, w1);   // block-uniform
    if (!valid) continue;
    const int64_t r = qrow(a, bh, a.dst_tok0 + t);
    uint8_t* dst = a.dst[kv].codes + r * D;
    if (kv == 0) {
      *reinterpret_cast<uint2*>(dst + part * 8) = codes;
    } else {
      *reinterpret_cast<uint32_t*>(dst + part * 4) = w0;
      *reinterpret_cast<uint32_t*>(dst + (part + 16) * 4) = w1;
    }
    if (part % TPG == 0) {
      constexpr int NG = D / GROUP;
      const int gi = part / TPG;
      if constexpr (COMPACT) {   // {f16 S0, f16 S1, i16 Z0, i16 Z1} per token
        uint8_t* m = a.dst[kv].meta + r * 8;
        *reinterpret_cast<__half*>(m + 2 * gi) = S16;
        *reinterpret_cast<int16_t*>(m + 4 + 2 * gi) = (int16_t)Z;
      } else {
        uint32_t* meta = reinterpret_cast<uint32_t*>(a.dst[kv].meta) + (r * NG + gi) * 2;
        *reinterpret_cast<uint2*>(meta) = make_uint2(__float_as_uint(S), (uint32_t)Z);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// INT2 affine: the same scheme with 3 levels.  A lane's 8 codes fill 16 bits,
// element i in bits 2i .. 2i+1, so K rows keep the natural order (dim d in
// byte d/4, bits 2 (d%4)).  V rows are stored with permuted dims: the code of
// dim d = 16m + 8h + r (r < 8, h < 2) sits in byte 4r + m/2 at bits
// 2 (2 (m%2) + h).  Bytes 4r .. 4r+3 then hold rows r and r+8 of all eight
// 16-dim m-tiles of the PV product (the layout INT4 uses, at 2 bits), and
// every m-tile lies inside one group.
// ---------------------------------------------------------------------------
// INT2 affine, bulk: one thread per 16 consecutive head_dim values of one
// token (two 16-byte loads, one 4-byte code store), 8 threads per token; a
// group of 64 (32) is 4 (2) lanes.  Arithmetic as int2_encode8 /
// int2_encode8_compact with the integer rounding of int4_encode16.
// ---------------------------------------------------------------------------
template <int GROUP, bool COMPACT>
__device__ __forceinline__ void int2_encode16(const float (&x)[16], float& S_out, __half& S16, int& Z,
                                              int (&q)[16]) {
  constexpr int TPG = GROUP / 16;
  float mn, mx;
  minmax16(x, mn, mx);
#pragma unroll
  for (int off = 1; off < TPG; off <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  float S;
  if (mx == mn)
    S = (mn != 0.0f) ? fabsf(mn) : 1.0f;
  else
    S = __fdiv_rn(__fsub_rn(mx, mn), 3.0f);
  if constexpr (COMPACT) {
    S = compact_scale(S, S16);
    Z = min(max((int)rintf(__fdiv_rn(-mn, S)), -128), 127);
  } else {
    Z = (int)rintf(__fdiv_rn(-mn, S));
  }
  S_out = S;
  const float r = __frcp_rn(S);
  const bool rok = r < kQuotientMaxRecip;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float qf = rok ? rn_quotient_int(x[i], S, r) : __fdiv_rn(x[i], S);
    q[i] = clamp0(rint_code<COMPACT>(qf) + Z, 3);
  }
}

// The INT2 V row of one token from its 8 lanes' codes.  Lane j (dims 16j ..
// 16j + 15 = m-tile j) owns nibble 8r + j of the permuted row for r = 0..7
// (dim 16j + r in its bits 0-1, 16j + r + 8 in bits 2-3); three exchange
// steps among the 8 lanes (xor 4: 16-bit halves, xor 2: bytes, xor 1:
// nibbles) transpose those 8 x 8 nibbles, after which lane t holds nibbles
// 8t .. 8t + 7 (bytes 4t .. 4t + 3).
__device__ __forceinline__ uint32_t int2_v_row_transpose(uint32_t w, int j) {
  const bool j2 = j & 4, j1 = j & 2, j0 = j & 1;
  const uint32_t keep4 = j2 ? w >> 16 : w & 0xFFFFu;
  const uint32_t recv4 = __shfl_xor_sync(0xffffffffu, j2 ? w & 0xFFFFu : w >> 16, 4);
  const uint32_t A = j2 ? (recv4 | keep4 << 16) : (keep4 | recv4 << 16);
  const uint32_t keep2 = prmt(A, 0u, j1 ? 0x31u : 0x20u);
  const uint32_t recv2 = __shfl_xor_sync(0xffffffffu, prmt(A, 0u, j1 ? 0x20u : 0x31u), 2);
  const uint32_t B = prmt(keep2, recv2, 0x5410u);
  const uint32_t keep1 = j0 ? (B >> 4) & 0x0F0F0F0Fu : B & 0x0F0F0F0Fu;
  const uint32_t recv1 = __shfl_xor_sync(0xffffffffu, j0 ? B & 0x0F0F0F0Fu : (B >> 4) & 0x0F0F0F0Fu, 1);
  const uint32_t C = j0 ? (recv1 | keep1 << 4) : (keep1 | recv1 << 4);
  return prmt(C, 0u, j1 ? 0x1302u : 0x3120u);
}

template <int GROUP, bool COMPACT = false>
__global__ void __launch_bounds__(256) quantize_int2_wide_kernel(QuantArgs a) {
  constexpr int NG = D / GROUP;
  constexpr int TPG = GROUP / 16;
  const int kv = blockIdx.z;
  const int j = threadIdx.x & 7;                                      // dims [16j, 16j + 16)
  const int64_t t = (int64_t)blockIdx.x * 32 + (threadIdx.x >> 3);   // token of the append
  const bool valid = t < a.n;
  for (int64_t bh = blockIdx.y; bh < a.bh; bh += gridDim.y) {
    uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
    if (valid) {
      const uint4* src = reinterpret_cast<const uint4*>(a.src[kv] + bh * a.src_bh_stride +
                                                        (a.src_tok0 + t) * D + j * 16);
      w0 = src[0];
      w1 = src[1];
    }
    float x[16], lo[8], hi[8];
    unpack8(w0, lo);
    unpack8(w1, hi);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[i] = lo[i];
      x[8 + i] = hi[i];
    }
    float S;
    __half S16;
    int Z, q[16];
    int2_encode16<GROUP, COMPACT>(x, S, S16, Z, q);
    uint32_t word = 0u;
    if (kv == 0) {   // natural order: dim 16j + i at bits 2i
#pragma unroll
      for (int i = 0; i < 16; ++i) word |= (uint32_t)q[i] << (2 * i);
    } else {         // permuted (block-uniform: all lanes exchange)
#pragma unroll
      for (int r = 0; r < 8; ++r) word |= (uint32_t)(q[r] | (q[r + 8] << 2)) << (4 * r);
      word = int2_v_row_transpose(word, j);
    }
    if (!valid) continue;
    const int64_t r = qrow(a, bh, a.dst_tok0 + t);
    *reinterpret_cast<uint32_t*>(a.dst[kv].codes + r * (D / 4) + j * 4) = word;
    if (j % TPG == 0) {
      const int gi = j / TPG;
      if constexpr (COMPACT) {   // {f16 S0, f16 S1, i8 Z0, i8 Z1, 0, 0} per token
        uint8_t* m = a.dst[kv].meta + r * 8;
        *reinterpret_cast<__half*>(m + 2 * gi) = S16;
        m[4 + gi] = (uint8_t)(int8_t)Z;
      } else {
        uint32_t* meta = reinterpret_cast<uint32_t*>(a.dst[kv].meta) + (r * NG + gi) * 2;
        *reinterpret_cast<uint2*>(meta) = make_uint2(__float_as_uint(S), (uint32_t)Z);
      }
    }
  }
}


// ---------------------------------------------------------------------------
// amax over K and V of one append (exact: compare BF16 magnitudes as ints).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* k, const uint16_t* v,
                                                   int64_t n_vec8, uint32_t* amax_k,
                                                   uint32_t* amax_v) {
  const uint16_t* src = blockIdx.y == 0 ? k : v;
  uint32_t* dst = blockIdx.y == 0 ? amax_k : amax_v;
  uint32_t m = 0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 w = reinterpret_cast<const uint4*>(src)[i];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m = max(m, ws[j] & 0x7FFFu);
      m = max(m, (ws[j] >> 16) & 0x7FFFu);
    }
  }
  m = __reduce_max_sync(0xffffffffu, m);
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0u;
    m = __reduce_max_sync(0xffffffffu, m);
    if (threadIdx.x == 0 && m != 0u) atomicMax(dst, m << 16);   // f32 bits of the BF16 value
  }
}

// ---------------------------------------------------------------------------
// Ring copy: BF16 tokens into ring slots.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) ring_copy_kernel(const uint16_t* src_k,
                                                        const uint16_t* src_v,
                                                        int64_t src_bh_stride, int64_t src_tok0,
                                                        uint16_t* ring_k, uint16_t* ring_v, int R,
                                                        int64_t ring_tok0, int64_t n, int bh) {
  const int kv = blockIdx.y;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t rows = (int64_t)bh * n;
  if (tid >= rows * kThreadsPerRow) return;
  const int part = (int)(tid % kThreadsPerRow);
  const int64_t row = tid / kThreadsPerRow;
  const int64_t t = row % n;
  const int64_t b = row / n;
  const uint16_t* src = (kv == 0 ? src_k : src_v) + b * src_bh_stride + (src_tok0 + t) * D + part * 8;
  uint16_t* dst = (kv == 0 ? ring_k : ring_v) + (b * R + ring_tok0 + t) * D + part * 8;
  *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
}

// ---------------------------------------------------------------------------
// Dequantize main-cache tokens to f32 [bh][n][D].  PAIRS: a V plane in its
// decode layout (NVFP4 pair-interleaved, INT4 / INT8 / INT2 dim-permuted),
// undone here.
// ---------------------------------------------------------------------------
template <int FMT, int GROUP, bool PAIRS, bool COMPACT = false>
__global__ void __launch_bounds__(256) dequantize_kernel(Plane p, const float* gscale,
                                                         int64_t cap, int bh, int64_t start,
                                                         int64_t n, float* out, const float* gseg,
                                                         int renewal, RowMap map) {
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t rows = (int64_t)bh * n;
  if (tid >= rows * kThreadsPerRow) return;
  const int part = (int)(tid % kThreadsPerRow);
  const int64_t row = tid / kThreadsPerRow;
  const int64_t t = row % n;
  const int64_t b = row / n;
  const int64_t tok = plane_row(map.unit0 + b, start + t, cap, map.kv_heads, map.pages,
                                map.page_tokens, map.max_pages);
  float y[8];
  if constexpr (FMT == KVQ_NVFP4) {
    const float g = renewal ? gseg[(uint32_t)(start + t) / (uint32_t)renewal] : *gscale;
    uint32_t c;
    if (PAIRS) {   // pair-interleaved V: this token's nibble of each of 8 bytes
      const uint2 w = *reinterpret_cast<const uint2*>(p.codes + (tok & ~(int64_t)1) * (D / 2) + part * 8);
      const int sh = (int)(tok & 1) * 4;
      c = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        c |= ((w.x >> (8 * i + sh)) & 0xFu) << (4 * i);
        c |= ((w.y >> (8 * i + sh)) & 0xFu) << (4 * (i + 4));
      }
    } else {
      c = *reinterpret_cast<const uint32_t*>(p.codes + tok * (D / 2) + part * 4);
    }
    const float bs = e4m3_to_f32(p.meta[tok * (D / 16) + part / 2]);
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(__fmul_rn(e2m1_to_f32((c >> (4 * i)) & 0xFu), bs), g);
  } else if constexpr (FMT == KVQ_FP8) {
    const float s = renewal ? gseg[(uint32_t)(start + t) / (uint32_t)renewal] : *gscale;
    const uint2 c = *reinterpret_cast<const uint2*>(p.codes + tok * D + part * 8);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      y[i] = __fmul_rn(e4m3_to_f32((c.x >> (8 * i)) & 0xFFu), s);
      y[4 + i] = __fmul_rn(e4m3_to_f32((c.y >> (8 * i)) & 0xFFu), s);
    }
  } else if constexpr (FMT == KVQ_INT8) {
    constexpr int NG = D / GROUP;
    const uint8_t* crow = p.codes + tok * D;
    const int gi = (part * 8) / GROUP;
    float S;
    int Z;
    if constexpr (COMPACT) {   // {f16 S0, f16 S1, i16 Z0, i16 Z1}
      S = __half2float(*reinterpret_cast<const __half*>(p.meta + tok * 8 + 2 * gi));
      Z = (int)*reinterpret_cast<const int16_t*>(p.meta + tok * 8 + 4 + 2 * gi);
    } else {
      const uint2 sz = *reinterpret_cast<const uint2*>(p.meta + (tok * NG + gi) * 8);
      S = __uint_as_float(sz.x);
      Z = (int)sz.y;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int d = 8 * part + e;
      const int q = crow[PAIRS ? int8_v_byte_of_dim(d) : d];
      y[e] = __fmul_rn((float)(q - Z), S);
    }
  } else if constexpr (FMT == KVQ_INT2) {
    constexpr int NG = D / GROUP;
    const uint8_t* crow = p.codes + tok * (D / 4);
    uint32_t c;
    if (PAIRS) {   // V row in the permuted dim order: gather dims 8 part + e
      c = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int d = 8 * part + e;
        c |= ((uint32_t)(crow[int2_v_byte_of_dim(d)] >> int2_v_shift_of_dim(d)) & 3u) << (2 * e);
      }
    } else {
      c = *reinterpret_cast<const uint16_t*>(crow + part * 2);
    }
    const int gi = (part * 8) / GROUP;
    float S;
    int Z;
    if constexpr (COMPACT) {   // {f16 S0, f16 S1, i8 Z0, i8 Z1, 0, 0}
      S = __half2float(*reinterpret_cast<const __half*>(p.meta + tok * 8 + 2 * gi));
      Z = (int)(int8_t)p.meta[tok * 8 + 4 + gi];
    } else {
      const uint2 sz = *reinterpret_cast<const uint2*>(p.meta + (tok * NG + gi) * 8);
      S = __uint_as_float(sz.x);
      Z = (int)sz.y;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fmul_rn((float)((int)((c >> (2 * i)) & 3u) - Z), S);
  } else {
    constexpr int NG = D / GROUP;
    uint32_t c;
    if (PAIRS) {   // V row in the permuted dim order: gather dims 8 part + e
      const uint8_t* row = p.codes + tok * (D / 2);
      c = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int d = 8 * part + e;
        c |= ((uint32_t)(row[int4_v_byte_of_dim(d)] >> (4 * int4_v_nibble_of_dim(d))) & 0xFu) << (4 * e);
      }
    } else {
      c = *reinterpret_cast<const uint32_t*>(p.codes + tok * (D / 2) + part * 4);
    }
    const int gi = (part * 8) / GROUP;
    float S;
    int Z;
    if constexpr (COMPACT) {
      S = __half2float(*reinterpret_cast<const __half*>(p.meta + tok * 8 + 2 * gi));
      Z = (int)(int8_t)p.meta[tok * 8 + 4 + gi];
    } else {
      const uint2 sz = *reinterpret_cast<const uint2*>(p.meta + (tok * NG + gi) * 8);
      S = __uint_as_float(sz.x);
      Z = (int)sz.y;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fmul_rn((float)((int)((c >> (4 * i)) & 0xFu) - Z), S);
  }
  float4* o = reinterpret_cast<float4*>(out + row * D + part * 8);
  o[0] = make_float4(y[0], y[1], y[2], y[3]);
  o[1] = make_float4(y[4], y[5], y[6], y[7]);
}

inline unsigned grid_for(int64_t threads) { return (unsigned)((threads + 255) / 256); }

}  // namespace

cudaError_t launch_amax(const uint16_t* k, const uint16_t* v, int64_t elems, uint32_t* amax_k,
                        uint32_t* amax_v, cudaStream_t stream) {
  const int64_t n_vec8 = elems / 8;
  int64_t blocks = (n_vec8 + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  amax_kernel<<<dim3((unsigned)blocks, 2), 256, 0, stream>>>(k, v, n_vec8, amax_k, amax_v);
  return cudaGetLastError();
}

cudaError_t launch_quantize(int format, const QuantArgs& a, cudaStream_t stream) {
  if (a.n <= 0 || a.bh <= 0) return cudaSuccess;
  // rows per unit: n tokens (NVFP4 V: token pairs, never more than n); 16
  // rows per 256-thread block
  const int64_t rows_per_block = 256 / kThreadsPerRow;
  const dim3 grid((unsigned)((a.n + rows_per_block - 1) / rows_per_block),
                  (unsigned)std::min<int64_t>(a.bh, 65535), 2);
  switch (format) {
    case KVQ_NVFP4: {
      // an odd first destination token goes through the per-pair kernel
      // (it completes a pair already in the cache); the rest starts even
      QuantArgs b = a;
      if (a.dst_tok0 & 1) {
        QuantArgs one = a;
        one.n = 1;
        quantize_nvfp4_kernel<<<dim3(1, grid.y, 2), 256, 0, stream>>>(one);
        b.calibrate = 0;          // the scale is stored by the launch above
        b.src_tok0 += 1;
        b.dst_tok0 += 1;
        b.n -= 1;
        if (b.n == 0) break;
      }
      const dim3 g16((unsigned)((b.n + 63) / 64), grid.y, 2);
      quantize_nvfp4_blocks_kernel<<<g16, 256, 0, stream>>>(b);
      break;
    }
    case KVQ_FP8:
      quantize_fp8_kernel<<<dim3((unsigned)((a.n + 31) / 32), grid.y, 2), 256, 0, stream>>>(a);
      break;
    case KVQ_INT8:
      if (a.compact) quantize_int8_kernel<64, true><<<grid, 256, 0, stream>>>(a);
      else quantize_int8_kernel<64><<<grid, 256, 0, stream>>>(a);
      break;
    case KVQ_INT2: {
      const dim3 g32((unsigned)((a.n + 31) / 32), grid.y, 2);
      if (a.compact) quantize_int2_wide_kernel<64, true><<<g32, 256, 0, stream>>>(a);
      else if (a.group == 64) quantize_int2_wide_kernel<64><<<g32, 256, 0, stream>>>(a);
      else quantize_int2_wide_kernel<32><<<g32, 256, 0, stream>>>(a);
      break;
    }
    case KVQ_INT4: {
      const dim3 g32((unsigned)((a.n + 31) / 32), grid.y, 2);
      if (a.compact) quantize_int4_wide_kernel<64, true><<<g32, 256, 0, stream>>>(a);
      else if (a.group == 64) quantize_int4_wide_kernel<64><<<g32, 256, 0, stream>>>(a);
      else quantize_int4_wide_kernel<32><<<g32, 256, 0, stream>>>(a);
      break;
    }
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// Scale renewal: one 16-thread row per token; the row takes the max |x|
// (BF16 magnitudes compared as integers) over every (batch, kv head) unit
// of the append, so one atomic per token and K|V goes to the token's
// segment word.  Grid: x = blocks of 16 tokens, z = K (0) / V (1).
__global__ void __launch_bounds__(256) seg_amax_kernel(const uint16_t* k, const uint16_t* v,
                                                      int64_t src_bh_stride, int64_t n, int bh,
                                                      int64_t dst_tok0, int renewal,
                                                      uint32_t* seg_amax_k, uint32_t* seg_amax_v) {
  const int kv = blockIdx.z;
  const int part = threadIdx.x % kThreadsPerRow;
  const int64_t t = row_in_unit();
  const bool valid = t < n;
  const uint16_t* src = (kv ? v : k) + t * D + part * 8;
  uint32_t* dst = kv ? seg_amax_v : seg_amax_k;
  uint32_t m = 0;
  if (valid) {
    auto fold = [&m](const uint4& w) {
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) m = max(m, max(ws[j] & 0x7FFFu, (ws[j] >> 16) & 0x7FFFu));
    };
    int b = 0;
    for (; b + 4 <= bh; b += 4) {   // four loads in flight
      uint4 w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = *reinterpret_cast<const uint4*>(src + (b + i) * src_bh_stride);
#pragma unroll
      for (int i = 0; i < 4; ++i) fold(w[i]);
    }
    for (; b < bh; ++b) fold(*reinterpret_cast<const uint4*>(src + b * src_bh_stride));
  }
#pragma unroll
  for (int off = 1; off < kThreadsPerRow; off <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (valid && part == 0 && m != 0u)
    atomicMax(&dst[(uint32_t)(dst_tok0 + t) / (uint32_t)renewal], m << 16);
}

__global__ void renew_scales_kernel(const uint32_t* seg_amax_k, const uint32_t* seg_amax_v,
                                    float* seg_scale_k, float* seg_scale_v, int64_t s_first,
                                    int64_t count, float divisor) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 2 * count) return;
  const int kv = (int)(i / count);
  const int64_t seg = s_first + i % count;
  const float amax = __uint_as_float((kv ? seg_amax_v : seg_amax_k)[seg - 1]);
  (kv ? seg_scale_v : seg_scale_k)[seg] = amax == 0.0f ? 1.0f : __fdiv_rn(amax, divisor);
}

__global__ void scale_from_amax_kernel(const uint32_t* amax_k, const uint32_t* amax_v,
                                       float* gscale_k, float* gscale_v, float divisor) {
  const int kv = threadIdx.x;
  if (kv > 1) return;
  const float amax = __uint_as_float(*(kv ? amax_v : amax_k));
  *(kv ? gscale_v : gscale_k) = amax == 0.0f ? 1.0f : __fdiv_rn(amax, divisor);
}

cudaError_t launch_scale_from_amax(const uint32_t* amax_k, const uint32_t* amax_v, float* gscale_k,
                                   float* gscale_v, float divisor, cudaStream_t stream) {
  scale_from_amax_kernel<<<1, 32, 0, stream>>>(amax_k, amax_v, gscale_k, gscale_v, divisor);
  return cudaGetLastError();
}

cudaError_t launch_seg_amax(const uint16_t* k, const uint16_t* v, int64_t src_bh_stride, int64_t n,
                            int bh, int64_t dst_tok0, int renewal, uint32_t* seg_amax_k,
                            uint32_t* seg_amax_v, cudaStream_t stream) {
  if (n <= 0 || bh <= 0) return cudaSuccess;
  const int rows_per_block = 256 / kThreadsPerRow;
  const dim3 grid((unsigned)((n + rows_per_block - 1) / rows_per_block), 1, 2);
  seg_amax_kernel<<<grid, 256, 0, stream>>>(k, v, src_bh_stride, n, bh, dst_tok0, renewal,
                                            seg_amax_k, seg_amax_v);
  return cudaGetLastError();
}

cudaError_t launch_renew_scales(const uint32_t* seg_amax_k, const uint32_t* seg_amax_v,
                                float* seg_scale_k, float* seg_scale_v, int64_t s_first,
                                int64_t s_last, float divisor, cudaStream_t stream) {
  if (s_last < s_first) return cudaSuccess;
  const int64_t count = s_last - s_first + 1;
  renew_scales_kernel<<<(unsigned)((2 * count + 255) / 256), 256, 0, stream>>>(
      seg_amax_k, seg_amax_v, seg_scale_k, seg_scale_v, s_first, count, divisor);
  return cudaGetLastError();
}

cudaError_t launch_ring_copy(const uint16_t* src_k, const uint16_t* src_v, int64_t src_bh_stride,
                             int64_t src_tok0, uint16_t* ring_k, uint16_t* ring_v, int R,
                             int64_t ring_tok0, int64_t n, int bh, cudaStream_t stream) {
  const int64_t threads = (int64_t)bh * n * kThreadsPerRow;
  if (threads == 0) return cudaSuccess;
  ring_copy_kernel<<<dim3(grid_for(threads), 2), 256, 0, stream>>>(
      src_k, src_v, src_bh_stride, src_tok0, ring_k, ring_v, R, ring_tok0, n, bh);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(int format, const Plane& p, const float* gscale, int64_t cap,
                              int group, int bh, int64_t start, int64_t n, float* out, bool v_pairs,
                              cudaStream_t stream, const float* gseg, int renewal, bool compact,
                              const RowMap& map) {
  const int64_t threads = (int64_t)bh * n * kThreadsPerRow;
  if (threads == 0) return cudaSuccess;
  const unsigned grid = grid_for(threads);
  switch (format) {
    case KVQ_NVFP4:
      if (v_pairs) dequantize_kernel<KVQ_NVFP4, 16, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      else dequantize_kernel<KVQ_NVFP4, 16, false><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      break;
    case KVQ_FP8: dequantize_kernel<KVQ_FP8, 0, false><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map); break;
    case KVQ_INT8:
      if (compact) {
        if (v_pairs) dequantize_kernel<KVQ_INT8, 64, true, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
        else dequantize_kernel<KVQ_INT8, 64, false, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      } else if (v_pairs) {
        dequantize_kernel<KVQ_INT8, 64, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      } else {
        dequantize_kernel<KVQ_INT8, 64, false><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      }
      break;
    case KVQ_INT2:
      if (compact) {
        if (v_pairs) dequantize_kernel<KVQ_INT2, 64, true, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
        else dequantize_kernel<KVQ_INT2, 64, false, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      } else if (group == 64) {
        if (v_pairs) dequantize_kernel<KVQ_INT2, 64, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
        else dequantize_kernel<KVQ_INT2, 64, false><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      } else {
        if (v_pairs) dequantize_kernel<KVQ_INT2, 32, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
        else dequantize_kernel<KVQ_INT2, 32, false><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      }
      break;
    case KVQ_INT4:
      if (compact) {
        if (v_pairs) dequantize_kernel<KVQ_INT4, 64, true, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
        else dequantize_kernel<KVQ_INT4, 64, false, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      } else if (group == 64) {
        if (v_pairs) dequantize_kernel<KVQ_INT4, 64, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
        else dequantize_kernel<KVQ_INT4, 64, false><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      } else {
        if (v_pairs) dequantize_kernel<KVQ_INT4, 32, true><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
        else dequantize_kernel<KVQ_INT4, 32, false><<<grid, 256, 0, stream>>>(p, gscale, cap, bh, start, n, out, gseg, renewal, map);
      }
      break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

__global__ void table_update_kernel(int32_t* table, const TableUpdate u) {
  const int i = threadIdx.x;
  if (i < u.n) table[u.idx[i]] = u.val[i];
}

cudaError_t launch_table_update(int32_t* table, const TableUpdate& u, cudaStream_t stream) {
  if (u.n <= 0) return cudaSuccess;
  table_update_kernel<<<1, kTableBatch, 0, stream>>>(table, u);
  return cudaGetLastError();
}

}  // namespace kvq
