// kvq_attn.cu -- split-K decode attention over the quantized cache, plus the
// log-sum-exp combine of the per-split partial results (sm_100a).
//
// Decode reads the quantized cache and dequantizes it on the fly (NVFP4
// KV-cache article, glsqs.com/news/814573, section 2.1; for the INT4 cache
// the BF16 residual ring of the most recent tokens is read as well,
// "KV缓存量化技术：提升大模型长文本生成效率", section 2.2).  The sequence is
// cut into splits (flash-decoding), each split producing (m, l, o) per
// query head, and a second kernel merges the splits.
//
// One CTA = one (batch, KV head, split).  Warp 8 is a producer: its elected
// lane streams the split's tiles (128 tokens of K codes, V codes, K meta,
// V meta) into a ring of shared-memory stages with 1-D bulk copies that
// complete on an mbarrier.  Warps 0..7 each take a 16-token slab of every
// stage and:
//   1. S^T[16 keys x 8 heads] = K_slab[16 x 128] . Q'^T with
//      mma.m16n8k16 (keys on M, the G <= 8 query heads of the KV head on N,
//      head_dim on K); K is dequantized from shared memory straight into
//      the A fragments in FP16 (E2M1 x E4M3 and E4M3 are exact in FP16).
//   2. online softmax in FP32 (base 2, the softmax scale and log2(e) folded
//      into Q', the per-tensor K scale folded into the exponent);
//   3. P^T is transposed in registers (movmatrix) into the B fragment of
//      O^T[128 dims x 8 heads] += V_slab^T[128 x 16 keys] . P^T, again with
//      V dequantized straight into A fragments.
// The head_dim order inside a fragment is permuted (the contraction does
// not care) so that every thread reads whole bytes/words of one token; Q is
// loaded in the same permuted order.  The 8 warps' states merge through
// shared memory into one partial per (split, head).
#include <cuda_runtime.h>
#include <math.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int D = kHeadDim;
constexpr int NW = 8;                        // consumer warps
constexpr int SLAB = 16;                     // tokens per warp per stage
constexpr int TILE = NW * SLAB;              // tokens per stage
constexpr int THREADS = (NW + 1) * 32;
constexpr int REC = D + 2;                   // partial record: m, l, o[D]
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
constexpr float kLog2e = 1.4426950408889634f;

template <int FMT, int GROUP>
struct Fmt {
  static constexpr int CB = (FMT == KVQ_FP8) ? D : D / 2;                 // code bytes / token
  static constexpr int MB = (FMT == KVQ_NVFP4) ? D / 16 : (FMT == KVQ_INT4) ? (D / GROUP) * 8 : 0;
  static constexpr int STAGE_BYTES = TILE * 2 * (CB + MB);
  static constexpr int STAGES = (STAGE_BYTES <= 20 * 1024) ? 4 : 3;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 2 * STAGES * 8 + 16;
};

// Dimension held in half `hf` (0 = low) of Q fragment register i (0..15) of
// a thread with quad index c.  Must match how the K fragments are built.
template <int FMT>
__device__ __forceinline__ int q_dim(int c, int i, int hf) {
  if (FMT == KVQ_INT4) {
    const int s = i >> 1, second = i & 1;
    return 32 * c + 8 * (s >> 1) + 2 * (s & 1) + second + 4 * hf;
  }
  return 32 * c + 2 * i + hf;
}

struct WarpState {
  float m0, m1, l0, l1;   // heads 2c, 2c+1 (base-2 logits)
  float o[8][4];          // O^T fragments: m-tile mt = dims 16r+2mt (+1)
};

__device__ __forceinline__ float quad_rows_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
  return v;
}

// Online-softmax step for one slab.  acc: S^T fragment (keys r, r+8 x heads
// 2c, 2c+1), already in base-2 units after multiplying by kscale.  Returns
// the P^T fragments transposed into the B operand of the PV product.
__device__ __forceinline__ void softmax_slab(float acc[4], bool vr, bool vr8, float kscale,
                                             WarpState& st, uint32_t& pb0, uint32_t& pb1) {
  const float NEG = -INFINITY;
  const float t0 = vr ? acc[0] * kscale : NEG;
  const float t1 = vr ? acc[1] * kscale : NEG;
  const float t2 = vr8 ? acc[2] * kscale : NEG;
  const float t3 = vr8 ? acc[3] * kscale : NEG;
  const float mx0 = quad_rows_max(fmaxf(t0, t2));
  const float mx1 = quad_rows_max(fmaxf(t1, t3));
  if (__any_sync(0xffffffffu, (mx0 > st.m0) || (mx1 > st.m1))) {
    const float n0 = fmaxf(st.m0, mx0), n1 = fmaxf(st.m1, mx1);
    const float a0 = (n0 == NEG) ? 1.0f : ex2(st.m0 - n0);
    const float a1 = (n1 == NEG) ? 1.0f : ex2(st.m1 - n1);
    st.l0 *= a0;
    st.l1 *= a1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      st.o[mt][0] *= a0;
      st.o[mt][2] *= a0;
      st.o[mt][1] *= a1;
      st.o[mt][3] *= a1;
    }
    st.m0 = n0;
    st.m1 = n1;
  }
  const float ref0 = (st.m0 == NEG) ? 0.0f : st.m0;
  const float ref1 = (st.m1 == NEG) ? 0.0f : st.m1;
  const float p0 = ex2(t0 - ref0), p1 = ex2(t1 - ref1);
  const float p2 = ex2(t2 - ref0), p3 = ex2(t3 - ref1);
  st.l0 += p0 + p2;
  st.l1 += p1 + p3;
  pb0 = movmatrix_trans(f32x2_to_f16x2(p0, p1));
  pb1 = movmatrix_trans(f32x2_to_f16x2(p2, p3));
}

__device__ __forceinline__ uint32_t byte_of(uint32_t w, int k) { return (w >> (8 * k)) & 0xFFu; }

__device__ __forceinline__ uint32_t bcast_lo(uint32_t h2) { return prmt(h2, 0, 0x1010); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t h2) { return prmt(h2, 0, 0x3232); }

// f16x2 {1024 + z, 1024 + z} and {s, s}
__device__ __forceinline__ uint32_t h2_const(float lo, float hi) { return f32x2_to_f16x2(lo, hi); }

// ---------------------------------------------------------------------------
// Per-format slab kernels: QK^T into acc, then (after softmax) PV into st.o.
// kc/vc: slab's first token row of K/V codes; km/vm: of K/V meta.
// ---------------------------------------------------------------------------
template <int FMT, int GROUP>
struct Slab;

template <int GROUP>
struct Slab<KVQ_NVFP4, GROUP> {
  static __device__ __forceinline__ void qk(const uint8_t* kc, const uint8_t* km, int r, int c,
                                            const uint32_t* qf, float acc[4]) {
    const uint4 k0 = *reinterpret_cast<const uint4*>(kc + r * 64 + 16 * c);
    const uint4 k1 = *reinterpret_cast<const uint4*>(kc + (r + 8) * 64 + 16 * c);
    const uint32_t s0 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(km + r * 8 + 2 * c));
    const uint32_t s1 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(km + (r + 8) * 8 + 2 * c));
    const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w};
    const uint32_t w1[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t sc0 = (s < 4) ? bcast_lo(s0) : bcast_hi(s0);
      const uint32_t sc1 = (s < 4) ? bcast_lo(s1) : bcast_hi(s1);
      const int wi = s >> 1, bi = 2 * (s & 1);
      const uint32_t a0 = hmul2(e2m1x2_to_f16x2(byte_of(w0[wi], bi)), sc0);
      const uint32_t a2 = hmul2(e2m1x2_to_f16x2(byte_of(w0[wi], bi + 1)), sc0);
      const uint32_t a1 = hmul2(e2m1x2_to_f16x2(byte_of(w1[wi], bi)), sc1);
      const uint32_t a3 = hmul2(e2m1x2_to_f16x2(byte_of(w1[wi], bi + 1)), sc1);
      mma_f16_16816(acc, a0, a1, a2, a3, qf[2 * s], qf[2 * s + 1]);
    }
  }
  static __device__ __forceinline__ void pv(const uint8_t* vc, const uint8_t* vm, int r, int c,
                                            uint32_t pb0, uint32_t pb1, WarpState& st) {
    const int X = 2 * c, Y = 2 * c + 1, Z = 2 * c + 8, W = 2 * c + 9;
    const uint2 vx = *reinterpret_cast<const uint2*>(vc + X * 64 + 8 * r);
    const uint2 vy = *reinterpret_cast<const uint2*>(vc + Y * 64 + 8 * r);
    const uint2 vz = *reinterpret_cast<const uint2*>(vc + Z * 64 + 8 * r);
    const uint2 vw = *reinterpret_cast<const uint2*>(vc + W * 64 + 8 * r);
    const uint32_t sxy = e4m3x2_to_f16x2((uint32_t)vm[X * 8 + r] | ((uint32_t)vm[Y * 8 + r] << 8));
    const uint32_t szw = e4m3x2_to_f16x2((uint32_t)vm[Z * 8 + r] | ((uint32_t)vm[W * 8 + r] << 8));
    const uint32_t xw[2] = {vx.x, vx.y}, yw[2] = {vy.x, vy.y};
    const uint32_t zw[2] = {vz.x, vz.y}, ww[2] = {vw.x, vw.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      // nibble transpose: byte k of lo = (x even dim, y even dim), hi = odd dims
      const uint32_t lo = (xw[h] & 0x0F0F0F0Fu) | ((yw[h] << 4) & 0xF0F0F0F0u);
      const uint32_t hi = ((xw[h] >> 4) & 0x0F0F0F0Fu) | (yw[h] & 0xF0F0F0F0u);
      const uint32_t lo2 = (zw[h] & 0x0F0F0F0Fu) | ((ww[h] << 4) & 0xF0F0F0F0u);
      const uint32_t hi2 = ((zw[h] >> 4) & 0x0F0F0F0Fu) | (ww[h] & 0xF0F0F0F0u);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t a0 = hmul2(e2m1x2_to_f16x2(byte_of(lo, k)), sxy);
        const uint32_t a1 = hmul2(e2m1x2_to_f16x2(byte_of(hi, k)), sxy);
        const uint32_t a2 = hmul2(e2m1x2_to_f16x2(byte_of(lo2, k)), szw);
        const uint32_t a3 = hmul2(e2m1x2_to_f16x2(byte_of(hi2, k)), szw);
        mma_f16_16816(st.o[4 * h + k], a0, a1, a2, a3, pb0, pb1);
      }
    }
  }
};

template <int GROUP>
struct Slab<KVQ_FP8, GROUP> {
  static __device__ __forceinline__ void qk(const uint8_t* kc, const uint8_t*, int r, int c,
                                            const uint32_t* qf, float acc[4]) {
    const uint4* p0 = reinterpret_cast<const uint4*>(kc + r * 128 + 32 * c);
    const uint4* p1 = reinterpret_cast<const uint4*>(kc + (r + 8) * 128 + 32 * c);
    const uint4 k0a = p0[0], k0b = p0[1], k1a = p1[0], k1b = p1[1];
    const uint32_t w0[8] = {k0a.x, k0a.y, k0a.z, k0a.w, k0b.x, k0b.y, k0b.z, k0b.w};
    const uint32_t w1[8] = {k1a.x, k1a.y, k1a.z, k1a.w, k1b.x, k1b.y, k1b.z, k1b.w};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t a0 = e4m3x2_to_f16x2(w0[s] & 0xFFFFu);
      const uint32_t a2 = e4m3x2_to_f16x2(w0[s] >> 16);
      const uint32_t a1 = e4m3x2_to_f16x2(w1[s] & 0xFFFFu);
      const uint32_t a3 = e4m3x2_to_f16x2(w1[s] >> 16);
      mma_f16_16816(acc, a0, a1, a2, a3, qf[2 * s], qf[2 * s + 1]);
    }
  }
  static __device__ __forceinline__ void pv(const uint8_t* vc, const uint8_t*, int r, int c,
                                            uint32_t pb0, uint32_t pb1, WarpState& st) {
    const int X = 2 * c, Y = 2 * c + 1, Z = 2 * c + 8, W = 2 * c + 9;
    const uint4 vx = *reinterpret_cast<const uint4*>(vc + X * 128 + 16 * r);
    const uint4 vy = *reinterpret_cast<const uint4*>(vc + Y * 128 + 16 * r);
    const uint4 vz = *reinterpret_cast<const uint4*>(vc + Z * 128 + 16 * r);
    const uint4 vw = *reinterpret_cast<const uint4*>(vc + W * 128 + 16 * r);
    const uint32_t xw[4] = {vx.x, vx.y, vx.z, vx.w}, yw[4] = {vy.x, vy.y, vy.z, vy.w};
    const uint32_t zw[4] = {vz.x, vz.y, vz.z, vz.w}, ww[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      // bytes [x0, y0, x1, y1] and [x2, y2, x3, y3]
      const uint32_t e01 = prmt(xw[h], yw[h], 0x5140), e23 = prmt(xw[h], yw[h], 0x7362);
      const uint32_t f01 = prmt(zw[h], ww[h], 0x5140), f23 = prmt(zw[h], ww[h], 0x7362);
      mma_f16_16816(st.o[2 * h], e4m3x2_to_f16x2(e01 & 0xFFFFu), e4m3x2_to_f16x2(e01 >> 16),
                    e4m3x2_to_f16x2(f01 & 0xFFFFu), e4m3x2_to_f16x2(f01 >> 16), pb0, pb1);
      mma_f16_16816(st.o[2 * h + 1], e4m3x2_to_f16x2(e23 & 0xFFFFu), e4m3x2_to_f16x2(e23 >> 16),
                    e4m3x2_to_f16x2(f23 & 0xFFFFu), e4m3x2_to_f16x2(f23 >> 16), pb0, pb1);
    }
  }
};

template <int GROUP>
struct Slab<KVQ_INT4, GROUP> {
  static constexpr int MB = (D / GROUP) * 8;
  // {1024 + n_j, 1024 + n_{j+4}} from nibbles j and j+4 of w
  static __device__ __forceinline__ uint32_t magic(uint32_t w, int j) {
    return lop3_and_or(w >> (4 * j), 0x000F000Fu, 0x64006400u);
  }
  static __device__ __forceinline__ void qk(const uint8_t* kc, const uint8_t* km, int r, int c,
                                            const uint32_t* qf, float acc[4]) {
    const uint4 k0 = *reinterpret_cast<const uint4*>(kc + r * 64 + 16 * c);
    const uint4 k1 = *reinterpret_cast<const uint4*>(kc + (r + 8) * 64 + 16 * c);
    const int gi = (32 * c) / GROUP;
    const uint2 m0 = *reinterpret_cast<const uint2*>(km + r * MB + 8 * gi);
    const uint2 m1 = *reinterpret_cast<const uint2*>(km + (r + 8) * MB + 8 * gi);
    const float z0 = 1024.0f + (float)(int)m0.y, z1 = 1024.0f + (float)(int)m1.y;
    const uint32_t zz0 = h2_const(z0, z0), zz1 = h2_const(z1, z1);
    const float S0 = __uint_as_float(m0.x), S1 = __uint_as_float(m1.x);
    const uint32_t ss0 = h2_const(S0, S0), ss1 = h2_const(S1, S1);
    const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w};
    const uint32_t w1[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int wi = s >> 1, j = 2 * (s & 1);
      const uint32_t a0 = hmul2(hsub2(magic(w0[wi], j), zz0), ss0);
      const uint32_t a2 = hmul2(hsub2(magic(w0[wi], j + 1), zz0), ss0);
      const uint32_t a1 = hmul2(hsub2(magic(w1[wi], j), zz1), ss1);
      const uint32_t a3 = hmul2(hsub2(magic(w1[wi], j + 1), zz1), ss1);
      mma_f16_16816(acc, a0, a1, a2, a3, qf[2 * s], qf[2 * s + 1]);
    }
  }
  static __device__ __forceinline__ void pv(const uint8_t* vc, const uint8_t* vm, int r, int c,
                                            uint32_t pb0, uint32_t pb1, WarpState& st) {
    const int X = 2 * c, Y = 2 * c + 1, Z = 2 * c + 8, W = 2 * c + 9;
    const int gi = (16 * r) / GROUP;
    const uint2 vx = *reinterpret_cast<const uint2*>(vc + X * 64 + 8 * r);
    const uint2 vy = *reinterpret_cast<const uint2*>(vc + Y * 64 + 8 * r);
    const uint2 vz = *reinterpret_cast<const uint2*>(vc + Z * 64 + 8 * r);
    const uint2 vw = *reinterpret_cast<const uint2*>(vc + W * 64 + 8 * r);
    const uint2 mx = *reinterpret_cast<const uint2*>(vm + X * MB + 8 * gi);
    const uint2 my = *reinterpret_cast<const uint2*>(vm + Y * MB + 8 * gi);
    const uint2 mz = *reinterpret_cast<const uint2*>(vm + Z * MB + 8 * gi);
    const uint2 mw = *reinterpret_cast<const uint2*>(vm + W * MB + 8 * gi);
    const uint32_t zxy = h2_const(1024.0f + (float)(int)mx.y, 1024.0f + (float)(int)my.y);
    const uint32_t zzw = h2_const(1024.0f + (float)(int)mz.y, 1024.0f + (float)(int)mw.y);
    const uint32_t sxy = h2_const(__uint_as_float(mx.x), __uint_as_float(my.x));
    const uint32_t szw = h2_const(__uint_as_float(mz.x), __uint_as_float(mw.x));
    const uint32_t xw[2] = {vx.x, vx.y}, yw[2] = {vy.x, vy.y};
    const uint32_t zw[2] = {vz.x, vz.y}, ww[2] = {vw.x, vw.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        // low 16 bits: bytes (2half, 2half+1) of x; high 16 bits: same of y
        const uint32_t sel = half ? 0x7632u : 0x5410u;
        const uint32_t e = prmt(xw[h], yw[h], sel);
        const uint32_t f = prmt(zw[h], ww[h], sel);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          const int mt = 4 * h + 2 * half + kb;
          const uint32_t a0 = hmul2(hsub2(magic(e, 2 * kb), zxy), sxy);
          const uint32_t a1 = hmul2(hsub2(magic(e, 2 * kb + 1), zxy), sxy);
          const uint32_t a2 = hmul2(hsub2(magic(f, 2 * kb), zzw), szw);
          const uint32_t a3 = hmul2(hsub2(magic(f, 2 * kb + 1), zzw), szw);
          mma_f16_16816(st.o[mt], a0, a1, a2, a3, pb0, pb1);
        }
      }
    }
  }
};

// magic(e, j) on a prmt'd word: nibble j of the low half pairs with nibble j
// of the high half -> for j = 0: (x byte lo nibble, y byte lo nibble), which
// is the even dim of byte 2*half (+kb) ... see the mapping notes above.

// Ring tokens (BF16, global memory) for one slab, in the INT4 Q order.
__device__ __forceinline__ void ring_qk(const uint16_t* rk, int ntok, int r, int c,
                                        const uint32_t* qf, float acc[4]) {
  // token rows r and r+8; dims of register (s, j): 32c + 8(s>>1) + 2(s&1) + j (+4)
  float x0[32], x1[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w0 = make_uint4(0, 0, 0, 0), w1 = make_uint4(0, 0, 0, 0);
    if (r < ntok) w0 = *reinterpret_cast<const uint4*>(rk + r * D + 32 * c + 8 * q);
    if (r + 8 < ntok) w1 = *reinterpret_cast<const uint4*>(rk + (r + 8) * D + 32 * c + 8 * q);
    const uint32_t a[4] = {w0.x, w0.y, w0.z, w0.w}, b[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x0[8 * q + 2 * e] = bf16_lo(a[e]);
      x0[8 * q + 2 * e + 1] = bf16_hi(a[e]);
      x1[8 * q + 2 * e] = bf16_lo(b[e]);
      x1[8 * q + 2 * e + 1] = bf16_hi(b[e]);
    }
  }
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int base = 8 * (s >> 1) + 2 * (s & 1);
    const uint32_t a0 = f32x2_to_f16x2(x0[base], x0[base + 4]);
    const uint32_t a2 = f32x2_to_f16x2(x0[base + 1], x0[base + 5]);
    const uint32_t a1 = f32x2_to_f16x2(x1[base], x1[base + 4]);
    const uint32_t a3 = f32x2_to_f16x2(x1[base + 1], x1[base + 5]);
    mma_f16_16816(acc, a0, a1, a2, a3, qf[2 * s], qf[2 * s + 1]);
  }
}

__device__ __forceinline__ void ring_pv(const uint16_t* rv, int ntok, int r, int c, uint32_t pb0,
                                        uint32_t pb1, WarpState& st) {
  const int tk[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
  float v[4][16];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint4 w = make_uint4(0, 0, 0, 0);
      if (tk[t] < ntok) w = *reinterpret_cast<const uint4*>(rv + tk[t] * D + 16 * r + 8 * q);
      const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[t][8 * q + 2 * e] = bf16_lo(a[e]);
        v[t][8 * q + 2 * e + 1] = bf16_hi(a[e]);
      }
    }
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const uint32_t a0 = f32x2_to_f16x2(v[0][2 * mt], v[1][2 * mt]);
    const uint32_t a1 = f32x2_to_f16x2(v[0][2 * mt + 1], v[1][2 * mt + 1]);
    const uint32_t a2 = f32x2_to_f16x2(v[2][2 * mt], v[3][2 * mt]);
    const uint32_t a3 = f32x2_to_f16x2(v[2][2 * mt + 1], v[3][2 * mt + 1]);
    mma_f16_16816(st.o[mt], a0, a1, a2, a3, pb0, pb1);
  }
}

__device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");
}

template <int FMT, int GROUP>
__global__ void __launch_bounds__(THREADS) decode_attn_kernel(const AttnArgs a) {
  using F = Fmt<FMT, GROUP>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + F::STAGES * F::STAGE_BYTES);
  uint64_t* empty = full + F::STAGES;

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int S = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bh = (int64_t)b * a.kv_heads + kvh;

  const int64_t tiles = (a.len_main + TILE - 1) / TILE;
  const int64_t t_begin = tiles * split / S, t_end = tiles * (split + 1) / S;
  const int ntiles = (int)(t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < F::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ---------------- producer ----------------
    if (lane == 0) {
      const uint8_t* kc = a.k.codes + bh * a.cap * F::CB;
      const uint8_t* vc = a.v.codes + bh * a.cap * F::CB;
      const uint8_t* km = F::MB ? a.k.meta + bh * a.cap * F::MB : nullptr;
      const uint8_t* vm = F::MB ? a.v.meta + bh * a.cap * F::MB : nullptr;
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % F::STAGES;
        if (i >= F::STAGES &&
            !mbar_wait_bounded(&empty[s], ((i / F::STAGES) - 1) & 1, a.dev_status,
                               kDevErrTimeoutEmpty, kWaitLimitNs))
          break;
        uint8_t* st = smem + s * F::STAGE_BYTES;
        const int64_t tok0 = (t_begin + i) * TILE;
        mbar_arrive_expect_tx(&full[s], F::STAGE_BYTES);
        bulk_g2s(st, kc + tok0 * F::CB, TILE * F::CB, &full[s]);
        bulk_g2s(st + TILE * F::CB, vc + tok0 * F::CB, TILE * F::CB, &full[s]);
        if (F::MB) {
          bulk_g2s(st + 2 * TILE * F::CB, km + tok0 * F::MB, TILE * F::MB, &full[s]);
          bulk_g2s(st + 2 * TILE * F::CB + TILE * F::MB, vm + tok0 * F::MB, TILE * F::MB, &full[s]);
        }
        ++issued;
      }
      // Never leave the CTA with copies still landing in shared memory.
      const int first = issued > F::STAGES ? issued - F::STAGES : 0;
      for (int i = first; i < issued; ++i)
        mbar_wait_bounded(&full[i % F::STAGES], (i / F::STAGES) & 1, a.dev_status,
                          kDevErrTimeoutDrain, kWaitLimitNs);
    }
    return;
  }

  // ---------------- consumers ----------------
  const int r = lane >> 2, c = lane & 3;
  const float qscale = a.softmax_scale * kLog2e;
  uint32_t qf[16];
  {
    const uint16_t* qp = a.q + ((int64_t)b * a.kv_heads * a.G + (int64_t)kvh * a.G + r) * D;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float lo = 0.0f, hi = 0.0f;
      if (r < a.G) {
        lo = __uint_as_float((uint32_t)qp[q_dim<FMT>(c, i, 0)] << 16) * qscale;
        hi = __uint_as_float((uint32_t)qp[q_dim<FMT>(c, i, 1)] << 16) * qscale;
      }
      qf[i] = f32x2_to_f16x2(lo, hi);
    }
  }
  const float kscale = (FMT == KVQ_INT4) ? 1.0f : *a.gscale_k;

  WarpState st;
  st.m0 = st.m1 = -INFINITY;
  st.l0 = st.l1 = 0.0f;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int j = 0; j < 4; ++j) st.o[mt][j] = 0.0f;

  bool ok = true;
  for (int i = 0; i < ntiles; ++i) {
    const int s = i % F::STAGES;
    if (!mbar_wait_bounded(&full[s], (i / F::STAGES) & 1, a.dev_status, kDevErrTimeoutFull,
                           kWaitLimitNs)) {
      ok = false;
      break;
    }
    const int64_t tok = (t_begin + i) * TILE + warp * SLAB;   // first token of this slab
    if (tok < a.len_main) {
      const uint8_t* stg = smem + s * F::STAGE_BYTES;
      const uint8_t* kc = stg + warp * SLAB * F::CB;
      const uint8_t* vc = stg + TILE * F::CB + warp * SLAB * F::CB;
      const uint8_t* km = stg + 2 * TILE * F::CB + warp * SLAB * F::MB;
      const uint8_t* vm = stg + 2 * TILE * F::CB + TILE * F::MB + warp * SLAB * F::MB;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      Slab<FMT, GROUP>::qk(kc, km, r, c, qf, acc);
      uint32_t pb0, pb1;
      softmax_slab(acc, tok + r < a.len_main, tok + r + 8 < a.len_main, kscale, st, pb0, pb1);
      Slab<FMT, GROUP>::pv(vc, vm, r, c, pb0, pb1, st);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // Residual ring (INT4): the last split reads the BF16 ring tokens.
  if (FMT == KVQ_INT4 && ok && split == S - 1 && a.len_ring > 0) {
    const uint16_t* rk = a.k.ring + bh * (int64_t)a.R * D;
    const uint16_t* rv = a.v.ring + bh * (int64_t)a.R * D;
    const int nslab = (int)((a.len_ring + SLAB - 1) / SLAB);
    for (int sl = warp; sl < nslab; sl += NW) {
      const int ntok = (int)min((int64_t)SLAB, a.len_ring - (int64_t)sl * SLAB);
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      ring_qk(rk + (int64_t)sl * SLAB * D, ntok, r, c, qf, acc);
      uint32_t pb0, pb1;
      softmax_slab(acc, r < ntok, r + 8 < ntok, 1.0f, st, pb0, pb1);
      ring_pv(rv + (int64_t)sl * SLAB * D, ntok, r, c, pb0, pb1, st);
    }
  }

  // ---------------- merge the 8 warps ----------------
  st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, 4);
  st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, 8);
  st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, 16);
  st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, 4);
  st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, 8);
  st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, 16);

  consumer_bar();   // every warp is done reading the stages
  float* red_m = reinterpret_cast<float*>(smem);          // [NW][8]
  float* red_l = red_m + NW * 8;                           // [NW][8]
  float* red_o = red_l + NW * 8;                           // [NW][8][D]
  if (r == 0) {
    red_m[warp * 8 + 2 * c] = st.m0;
    red_m[warp * 8 + 2 * c + 1] = st.m1;
    red_l[warp * 8 + 2 * c] = st.l0;
    red_l[warp * 8 + 2 * c + 1] = st.l1;
  }
  float* ow = red_o + warp * 8 * D;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int d0 = 16 * r + 2 * mt;
    ow[(2 * c) * D + d0] = st.o[mt][0];
    ow[(2 * c + 1) * D + d0] = st.o[mt][1];
    ow[(2 * c) * D + d0 + 1] = st.o[mt][2];
    ow[(2 * c + 1) * D + d0 + 1] = st.o[mt][3];
  }
  consumer_bar();

  const int64_t rec0 = ((bh * S + split) * a.G) * REC;
  for (int idx = threadIdx.x; idx < a.G * D; idx += NW * 32) {
    const int h = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w * 8 + h]);
    float o = 0.0f, l = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = red_m[w * 8 + h];
        const float f = (mw == -INFINITY) ? 0.0f : ex2(mw - M);
        o += f * red_o[(w * 8 + h) * D + d];
        l += f * red_l[w * 8 + h];
      }
    }
    float* rec = a.partials + rec0 + (int64_t)h * REC;
    rec[2 + d] = o;
    if (d == 0) {
      rec[0] = M;
      rec[1] = l;
    }
  }
}

// Merge the S split records of every (batch, query head): out = gV * sum_s
// e^(m_s - M) o_s / sum_s e^(m_s - M) l_s (base 2).
__global__ void __launch_bounds__(D) combine_kernel(const float* partials, int S, int G,
                                                    int kv_heads, const float* gscale_v,
                                                    float* out) {
  const int bq = blockIdx.x;                 // b * Hq + hq
  const int Hq = kv_heads * G;
  const int b = bq / Hq, hq = bq % Hq;
  const int kvh = hq / G, h = hq % G;
  const int64_t bh = (int64_t)b * kv_heads + kvh;
  const float* base = partials + (bh * S * G + h) * REC;
  const int64_t stride = (int64_t)G * REC;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, base[s * stride]);
  float o = 0.0f, l = 0.0f;
  for (int s = 0; s < S; ++s) {
    const float* rec = base + s * stride;
    const float f = (rec[0] == -INFINITY) ? 0.0f : ex2(rec[0] - M);
    l += f * rec[1];
    o += f * rec[2 + threadIdx.x];
  }
  const float gv = gscale_v ? *gscale_v : 1.0f;
  out[(int64_t)bq * D + threadIdx.x] = (o / l) * gv;
}

template <int FMT, int GROUP>
cudaError_t launch_impl(const AttnArgs& a, cudaStream_t stream) {
  using F = Fmt<FMT, GROUP>;
  auto kern = decode_attn_kernel<FMT, GROUP>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const dim3 grid(a.splits, a.kv_heads, a.batch);
  kern<<<grid, THREADS, F::SMEM, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  combine_kernel<<<a.batch * a.kv_heads * a.G, D, 0, stream>>>(a.partials, a.splits, a.G,
                                                                a.kv_heads, a.gscale_v, a.out);
  return cudaGetLastError();
}

template <int FMT, int GROUP>
int blocks_impl() {
  using F = Fmt<FMT, GROUP>;
  auto kern = decode_attn_kernel<FMT, GROUP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM) != cudaSuccess)
    return 1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, THREADS, F::SMEM) != cudaSuccess)
    return 1;
  return n > 0 ? n : 1;
}

}  // namespace

int attn_blocks_per_sm(int format) {
  switch (format) {
    case KVQ_NVFP4: return blocks_impl<KVQ_NVFP4, 16>();
    case KVQ_FP8: return blocks_impl<KVQ_FP8, 0>();
    default: return blocks_impl<KVQ_INT4, 64>();
  }
}

cudaError_t launch_decode_attention(const AttnArgs& a, cudaStream_t stream) {
  switch (a.format) {
    case KVQ_NVFP4: return launch_impl<KVQ_NVFP4, 16>(a, stream);
    case KVQ_FP8: return launch_impl<KVQ_FP8, 0>(a, stream);
    case KVQ_INT4:
      return a.group == 64 ? launch_impl<KVQ_INT4, 64>(a, stream)
                           : launch_impl<KVQ_INT4, 32>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kvq
