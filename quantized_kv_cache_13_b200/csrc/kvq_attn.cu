// kvq_attn.cu -- split-K decode attention over the quantized cache with the
// log-sum-exp combine fused in (sm_100a).
//
// Decode reads the quantized cache and dequantizes it on the fly (NVFP4
// KV-cache article, glsqs.com/news/814573, section 2.1; for the INT4 and
// INT8 caches the BF16 residual ring of the most recent tokens is read as
// well, "KV缓存量化技术：提升大模型长文本生成效率", section 2.2).
//
// Work split (flash-decoding with even shares): the cache of every
// (batch, KV head) "unit" is cut into tiles of TILE tokens; the flattened
// sequence of all units' tiles is divided evenly over a single wave of CTAs
// (SMs x resident CTAs per SM), so a CTA may own the tail of one unit and the
// head of the next.  For every unit it touches a CTA produces one partial
// (m, l, o) per query head; the last CTA to finish a unit (an atomic counter
// per unit, reset by that CTA) merges the partials and writes the output.
//
// Inside a CTA, every warp streams its own share of each tile (K codes, V
// codes, K meta, V meta of SPW 16-token slabs) into private shared-memory
// stages with 1-D bulk copies, issued by one elected lane and completing on
// the warp's own mbarrier; a warp refills a stage as soon as it is done with
// it, and no warp waits for another until the merge.  For each slab:
//   1. S^T[16 keys x 8 heads] = K_slab[16 x 128] . Q'^T with mma.m16n8k16
//      (keys on M, the G <= 8 query heads of the KV head on N, head_dim on
//      K); K is dequantized from shared memory straight into A fragments in
//      FP16 (E2M1 x E4M3 and E4M3 are exact in FP16);
//   2. online softmax in FP32, base 2 (softmax scale and log2(e) folded into
//      Q', the per-tensor K scale folded into the exponent), one max update
//      per SPW slabs;
//   3. P^T goes through movmatrix into the B fragment of
//      O^T[128 dims x 8 heads] += V_slab^T[128 x 16 keys] . P^T, with V
//      dequantized straight into A fragments (for the INT formats the group
//      scale is applied to P instead and the zero point is one extra MMA).
// The head_dim order inside the QK fragments is permuted (the contraction
// does not care) so every thread reads whole words of one token; Q is loaded
// in the same order.
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "kvq_device.cuh"
#include "kvq_encode.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int D = kHeadDim;
constexpr int SLAB = 16;                     // tokens per mma tile
constexpr int REC = D + 2;                   // partial record: m, l, o[D]
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;   // logits are kept in base 2

// The affine integer formats: per-group S and Z, no per-tensor scale, an
// optional BF16 ring, group scales applied on the P side of the PV product.
template <int FMT>
constexpr bool kIntAffine =
    FMT == KVQ_INT4 || FMT == KVQ_INT8 || FMT == KVQ_INT2 || FMT == kFmtInt4Compact ||
    FMT == kFmtInt8Compact || FMT == kFmtInt2Compact;

// The format whose code layout (and Q order) a kernel format id uses.
template <int FMT>
constexpr int kCodeFmt = FMT == kFmtInt4Compact ? KVQ_INT4
                         : FMT == kFmtInt8Compact ? KVQ_INT8
                         : FMT == kFmtInt2Compact ? KVQ_INT2 : FMT;

template <int FMT, int GROUP>
struct Fmt {
  // Two 8-warp CTAs per SM (8 warps = 2 per SM sub-partition per CTA, 128
  // registers each); all warps compute.  (One 16-warp CTA per SM measured
  // slower end to end.)
  static constexpr int NW = 8;
  static constexpr int MIN_BLOCKS = 2;
  static constexpr int THREADS = NW * 32;
  static constexpr int MERGE_BYTES = NW * 8 * D * 4;   // per-warp O for the intra-CTA merge
  static constexpr int CF = kCodeFmt<FMT>;
  static constexpr int CB = (CF == KVQ_FP8 || CF == KVQ_INT8) ? D
                            : (CF == KVQ_INT2) ? D / 4 : D / 2;   // code bytes / token
  static constexpr int MB = (FMT == KVQ_NVFP4) ? D / 16
                            : (FMT == kFmtInt4Compact || FMT == kFmtInt8Compact ||
                               FMT == kFmtInt2Compact) ? 8
                            : kIntAffine<FMT> ? (D / GROUP) * 8 : 0;
  // slabs per warp per stage and stage count: as many slabs per stage as
  // two CTAs' shared memory allows with at least two stages (NVFP4 3 x 2,
  // INT4 2 x 2, FP8 1 x 3); more slabs per stage spread the per-tile wait,
  // refill and loop work over more tokens (INT2: 3 x 3)
  static constexpr int SPW = (CF == KVQ_FP8 || CF == KVQ_INT8) ? 1
                             : (CF == KVQ_NVFP4 || (CF == KVQ_INT2 && GROUP == 64)) ? 3 : 2;
  static constexpr int WTOK = SLAB * SPW;                                 // tokens per warp per tile
  static constexpr int TILE = NW * WTOK;                                  // tokens per tile
  static constexpr int WSTAGE = WTOK * 2 * (CB + MB);                     // one warp's part of a stage
  // a warp's slot in a stage: its part, padded so that a stage also holds
  // the intra-CTA merge buffer (only compact INT2's parts are smaller)
  static constexpr int WSTRIDE = WSTAGE > MERGE_BYTES / NW ? WSTAGE : MERGE_BYTES / NW;
  static constexpr int STAGE_BYTES = NW * WSTRIDE;
  static constexpr int STAGES = (CF == KVQ_FP8 || CF == KVQ_INT8 || CF == KVQ_INT2) ? 3 : 2;
  static constexpr int NC = kIntAffine<FMT> ? D / GROUP : 0;   // zero-point accumulators
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  // per-warp full mbarriers, per-warp m/l, flags
  static constexpr int SMEM = BAR_OFF + STAGES * NW * 8 + 2 * NW * 8 * 4 + 16;
  static_assert(STAGE_BYTES >= MERGE_BYTES, "a stage must hold the merge buffer");
  static_assert(WTOK * MB % 16 == 0 && WTOK * CB % 16 == 0, "bulk copies are 16-byte multiples");
};

// head_dim index held in half `hf` (0 = low) of Q fragment register i
// (0..15) of a thread with quad index c.  Must match how each format's K
// fragments are built (k-step s = i / 2 uses registers 2s and 2s+1).
template <int FMT_ID, int GROUP>
__device__ __forceinline__ int q_dim(int c, int i, int hf) {
  // compact-metadata ids share their code format's fragment order (INT4's
  // compact id keeps its own branch below)
  constexpr int FMT = FMT_ID == kFmtInt8Compact ? KVQ_INT8 : FMT_ID == kFmtInt2Compact ? KVQ_INT2 : FMT_ID;
  const int s = i >> 1, second = i & 1;
  if (FMT == KVQ_INT8)                  // k-steps 0-3: group 0, 4-7: group 1; 4 bytes per k-step
    return 64 * (s >> 2) + 16 * c + 4 * (s & 3) + 2 * second + hf;
  if (FMT == KVQ_INT2 && GROUP == 32)   // 32 dims per thread (its group), word s/4, code pairs (j, j+8)
    return 32 * c + 16 * (s >> 2) + 2 * (s & 3) + second + 8 * hf;
  if (FMT == KVQ_INT2)                  // k-steps 0-3: group 0, 4-7: group 1; code pairs (j, j+8)
    return 64 * (s >> 2) + 16 * c + 2 * (s & 3) + second + 8 * hf;
  if ((FMT == KVQ_INT4 && GROUP == 64) || FMT == kFmtInt4Compact)   // k-steps 0-3: group 0, 4-7: group 1
    return 64 * (s >> 2) + 16 * c + 8 * ((s & 3) >> 1) + 2 * (s & 1) + second + 4 * hf;
  if (FMT == KVQ_INT4)                  // 32 contiguous dims per thread, nibble pairs (j, j+4)
    return 32 * c + 8 * (s >> 1) + 2 * (s & 1) + second + 4 * hf;
  return 32 * c + 2 * i + hf;           // 32 contiguous dims per thread, natural pairs
}

// Per-warp online-softmax state.  NC > 0 (INT4): one extra accumulator per
// quantization group for the zero-point term of the P.V product (see
// int4_pv), subtracted from O before the merge.
// l: the softmax denominators as an MMA accumulator of ones^T . P^T over the
// same FP16 probabilities the P.V product uses, so the output is a weighted
// mean of V with exactly normalised weights; every row holds the sums, and
// l[0] / l[1] are those of heads 2c / 2c+1.
template <int NC>
struct WarpState {
  float m0, m1;           // heads 2c, 2c+1 (base-2 logits)
  float l[4];
  float o[8][4];          // O^T fragments (rows of m-tile mt: see o_dim)
  float corr[NC][4];
};
template <>
struct WarpState<0> {
  float m0, m1;
  float l[4];
  float o[8][4];
};
constexpr uint32_t kHalfOnes = 0x3C003C00u;   // FP16 {1.0, 1.0}

// head_dim index of row r (hi = 0) or r + 8 (hi = 1) of O^T m-tile mt.
// NVFP4 / FP8: dims 16r + 2mt (+1); INT formats (permuted V rows): 16mt + r (+8).
template <int FMT>
__device__ __forceinline__ int o_dim(int mt, int r, int hi) {
  return kIntAffine<FMT> ? 16 * mt + r + 8 * hi : 16 * r + 2 * mt + hi;
}

template <int NC>
__device__ __forceinline__ void state_reset(WarpState<NC>& st) {
  st.m0 = st.m1 = -INFINITY;
  st.l[0] = st.l[1] = st.l[2] = st.l[3] = 0.0f;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int j = 0; j < 4; ++j) st.o[mt][j] = 0.0f;
  if constexpr (NC > 0) {
#pragma unroll
    for (int g = 0; g < NC; ++g)
#pragma unroll
      for (int j = 0; j < 4; ++j) st.corr[g][j] = 0.0f;
  }
}

__device__ __forceinline__ float rows_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
  return v;
}

// Online-softmax step over NS slabs.  acc[s]: raw S^T fragment (keys r, r+8
// x heads 2c, 2c+1) of slab s; the logit in base 2 is acc * kscale (kscale >
// 0, so maxima are taken on acc directly).  nvalid[s]: valid keys of slab s
// (ignored when FULL).  Produces the PV B fragments (P^T transposed by
// movmatrix) per slab.  hilo: acc holds the q'_hi scores of head c in
// column 2c and its q'_lo scores in column 2c + 1 (G <= 4, see load_q); they
// are added here first (SUMMED: the slab has added them itself, as the
// factored INT slabs do), and column 2c + 1 carries no probability.
//
// The reference m of each head only has to keep p = 2^(logit - m) in range,
// so it is moved (and O, l rescaled) only when some logit exceeds it by more
// than kLazyMax: p stays below 2^kLazyMax = 256 in the FP16 P operand, and
// the cross-lane max reduction runs only on those rare steps.  When it runs
// it sets m to the exact running maximum.
constexpr float kLazyMax = 8.0f;
template <int NS, bool FULL, int NC, bool SUMMED = false>
__device__ __forceinline__ void softmax_step(float (&acc)[NS][4], const int (&nvalid)[NS], int r,
                                             float kscale, float ik, bool hilo, WarpState<NC>& st,
                                             uint32_t (&pb)[NS][2]) {
  const float NEG = -INFINITY;
  if (hilo) {   // column 2c: q'_hi scores + column 2c+1: q'_lo scores (see load_q)
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      if constexpr (!SUMMED) {
        acc[s][0] += acc[s][1];
        acc[s][2] += acc[s][3];
      }
      acc[s][1] = acc[s][3] = NEG;   // no head in column 2c+1: p = 0 there
    }
  }
  if (!FULL) {
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const bool v0 = r < nvalid[s], v1 = r + 8 < nvalid[s];
      if (!v0) acc[s][0] = acc[s][1] = NEG;
      if (!v1) acc[s][2] = acc[s][3] = NEG;
    }
  }
  // trigger thresholds on the raw scores (kscale > 0; ik = 1 / kscale is
  // computed once per launch, and its rounding only moves the threshold by
  // an ulp)
  const float t0 = (st.m0 + kLazyMax) * ik, t1 = (st.m1 + kLazyMax) * ik;
  bool over = false;
#pragma unroll
  for (int s = 0; s < NS; ++s)
    over |= (fmaxf(acc[s][0], acc[s][2]) > t0) | (fmaxf(acc[s][1], acc[s][3]) > t1);
  if (__any_sync(0xffffffffu, over)) {
    float mx0 = fmaxf(acc[0][0], acc[0][2]), mx1 = fmaxf(acc[0][1], acc[0][3]);
#pragma unroll
    for (int s = 1; s < NS; ++s) {
      mx0 = fmaxf(mx0, fmaxf(acc[s][0], acc[s][2]));
      mx1 = fmaxf(mx1, fmaxf(acc[s][1], acc[s][3]));
    }
    mx0 = rows_max(mx0) * kscale;
    mx1 = rows_max(mx1) * kscale;
    const float n0 = fmaxf(st.m0, mx0), n1 = fmaxf(st.m1, mx1);
    const float a0 = (n0 == NEG) ? 1.0f : ex2(st.m0 - n0);
    const float a1 = (n1 == NEG) ? 1.0f : ex2(st.m1 - n1);
    st.l[0] *= a0;
    st.l[2] *= a0;
    st.l[1] *= a1;
    st.l[3] *= a1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      st.o[mt][0] *= a0;
      st.o[mt][2] *= a0;
      st.o[mt][1] *= a1;
      st.o[mt][3] *= a1;
    }
    if constexpr (NC > 0) {
#pragma unroll
      for (int g = 0; g < NC; ++g) {
        st.corr[g][0] *= a0;
        st.corr[g][2] *= a0;
        st.corr[g][1] *= a1;
        st.corr[g][3] *= a1;
      }
    }
    st.m0 = n0;
    st.m1 = n1;
  }
  // m is finite once any valid key was seen; before that every p is 0
  const float ref0 = (st.m0 == NEG) ? 0.0f : -st.m0;
  const float ref1 = (st.m1 == NEG) ? 0.0f : -st.m1;
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const float p0 = ex2(fmaf(acc[s][0], kscale, ref0)), p2 = ex2(fmaf(acc[s][2], kscale, ref0));
    float p1 = 0.0f, p3 = 0.0f;
    if (!hilo) {
      p1 = ex2(fmaf(acc[s][1], kscale, ref1));
      p3 = ex2(fmaf(acc[s][3], kscale, ref1));
    }
    pb[s][0] = movmatrix_trans(f32x2_to_f16x2(p0, p1));
    pb[s][1] = movmatrix_trans(f32x2_to_f16x2(p2, p3));
    mma_f16_16816(st.l, kHalfOnes, kHalfOnes, kHalfOnes, kHalfOnes, pb[s][0], pb[s][1]);
  }
}

__device__ __forceinline__ uint32_t bcast_lo(uint32_t h2) { return prmt(h2, 0, 0x1010); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t h2) { return prmt(h2, 0, 0x3232); }

// ---------------------------------------------------------------------------
// Per-format slab kernels: qk() accumulates S^T, pv() accumulates O^T.
// kc/vc: the slab's first token row of K/V codes; km/vm: of K/V meta.
// ---------------------------------------------------------------------------
template <int FMT, int GROUP>
struct Slab;

// Slabs whose metadata is converted in shared memory once per part
// (`prepare`, declared with a true kConv) before their slabs are read.
template <typename S, typename = void>
struct HasPrepare : std::false_type {};
template <typename S>
struct HasPrepare<S, std::void_t<decltype(S::kConv)>> : std::bool_constant<S::kConv> {};
// Slabs whose qk() already adds the two Q' parts' columns when hilo
// (declared with a true kHiloSummed).
template <typename S, typename = void>
struct HiloSummed : std::false_type {};
template <typename S>
struct HiloSummed<S, std::void_t<decltype(S::kHiloSummed)>> : std::bool_constant<S::kHiloSummed> {};

template <int GROUP>
struct Slab<KVQ_NVFP4, GROUP> {
  // QK: thread (r, c) covers dims [32c, 32c+32) of keys r and r+8; k-step s
  // uses bytes 2s (a0/a1) and 2s+1 (a2/a3) of that 16-byte chunk; the block
  // scale is that of block 2c (k-steps 0..3) or 2c+1 (4..7).
  static __device__ __forceinline__ void qk(const uint8_t* kc, const uint8_t* km, int r, int c,
                                            const uint32_t (&qf)[16], const float (&)[8],
                                            bool, float (&acc)[4]) {
    const uint4 k0 = *reinterpret_cast<const uint4*>(kc + r * 64 + 16 * c);
    const uint4 k1 = *reinterpret_cast<const uint4*>(kc + (r + 8) * 64 + 16 * c);
    uint32_t s0, s1;   // {scale 2c, scale 2c+1} of keys r and r+8
    {
      uint32_t unused;
      e4m3x4_to_f16x2x2(*reinterpret_cast<const uint16_t*>(km + r * 8 + 2 * c), s0, unused);
      e4m3x4_to_f16x2x2(*reinterpret_cast<const uint16_t*>(km + (r + 8) * 8 + 2 * c), s1, unused);
    }
    const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w};
    const uint32_t w1[4] = {k1.x, k1.y, k1.z, k1.w};
    // two independent accumulator chains (even / odd k-steps) halve the
    // dependent-mma latency
    float ac[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const uint32_t sc0 = (wi < 2) ? bcast_lo(s0) : bcast_hi(s0);
      const uint32_t sc1 = (wi < 2) ? bcast_lo(s1) : bcast_hi(s1);
      uint32_t h0[4], h1[4];
      e2m1x8_to_f16x2x4(w0[wi], h0);
      e2m1x8_to_f16x2x4(w1[wi], h1);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int s = 2 * wi + j;
        mma_f16_16816(ac[j], hmul2(h0[2 * j], sc0), hmul2(h1[2 * j], sc1), hmul2(h0[2 * j + 1], sc0),
                      hmul2(h1[2 * j + 1], sc1), qf[2 * s], qf[2 * s + 1]);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = ac[0][e] + ac[1][e];
  }
  // PV: thread (r, c) covers block r (dims 16r..16r+15) of keys 2c, 2c+1
  // (pair c of the slab) and 2c+8, 2c+9 (pair c+4); V is pair-interleaved, so
  // byte d of a pair row already holds dim d of both keys, i.e. one A
  // register per byte.  m-tile mt holds dims 16r+2mt (row r) and 16r+2mt+1
  // (row r+8).
  static __device__ __forceinline__ void pv(const uint8_t* vc, const uint8_t* vm, int r, int c,
                                            uint32_t pb0, uint32_t pb1, WarpState<0>& st) {
    const uint4 pxy = *reinterpret_cast<const uint4*>(vc + c * 128 + 16 * r);
    const uint4 pzw = *reinterpret_cast<const uint4*>(vc + (c + 4) * 128 + 16 * r);
    const int X = 2 * c, Y = 2 * c + 1, Z = 2 * c + 8, W = 2 * c + 9;
    uint32_t sxy, szw, unused;
    e4m3x4_to_f16x2x2((uint32_t)vm[X * 8 + r] | ((uint32_t)vm[Y * 8 + r] << 8), sxy, unused);
    e4m3x4_to_f16x2x2((uint32_t)vm[Z * 8 + r] | ((uint32_t)vm[W * 8 + r] << 8), szw, unused);
    const uint32_t xw[4] = {pxy.x, pxy.y, pxy.z, pxy.w};
    const uint32_t zw[4] = {pzw.x, pzw.y, pzw.z, pzw.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t a[4], b[4];
      e2m1x8_to_f16x2x4(xw[w], a);
      e2m1x8_to_f16x2x4(zw[w], b);
      mma_f16_16816(st.o[2 * w], hmul2(a[0], sxy), hmul2(a[1], sxy), hmul2(b[0], szw),
                    hmul2(b[1], szw), pb0, pb1);
      mma_f16_16816(st.o[2 * w + 1], hmul2(a[2], sxy), hmul2(a[3], sxy), hmul2(b[2], szw),
                    hmul2(b[3], szw), pb0, pb1);
    }
  }
};

template <int GROUP>
struct Slab<KVQ_FP8, GROUP> {
  static __device__ __forceinline__ void qk(const uint8_t* kc, const uint8_t*, int r, int c,
                                            const uint32_t (&qf)[16], const float (&)[8],
                                            bool, float (&acc)[4]) {
    const uint4* p0 = reinterpret_cast<const uint4*>(kc + r * 128 + 32 * c);
    const uint4* p1 = reinterpret_cast<const uint4*>(kc + (r + 8) * 128 + 32 * c);
    const uint4 k0a = p0[0], k0b = p0[1], k1a = p1[0], k1b = p1[1];
    const uint32_t w0[8] = {k0a.x, k0a.y, k0a.z, k0a.w, k0b.x, k0b.y, k0b.z, k0b.w};
    const uint32_t w1[8] = {k1a.x, k1a.y, k1a.z, k1a.w, k1b.x, k1b.y, k1b.z, k1b.w};
    float ac[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      uint32_t a0, a2, a1, a3;
      e4m3x4_to_f16x2x2(w0[s], a0, a2);
      e4m3x4_to_f16x2x2(w1[s], a1, a3);
      mma_f16_16816(ac[s & 1], a0, a1, a2, a3, qf[2 * s], qf[2 * s + 1]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = ac[0][e] + ac[1][e];
  }
  static __device__ __forceinline__ void pv(const uint8_t* vc, const uint8_t*, int r, int c,
                                            uint32_t pb0, uint32_t pb1, WarpState<0>& st) {
    const int X = 2 * c, Y = 2 * c + 1, Z = 2 * c + 8, W = 2 * c + 9;
    const uint4 vx = *reinterpret_cast<const uint4*>(vc + X * 128 + 16 * r);
    const uint4 vy = *reinterpret_cast<const uint4*>(vc + Y * 128 + 16 * r);
    const uint4 vz = *reinterpret_cast<const uint4*>(vc + Z * 128 + 16 * r);
    const uint4 vw = *reinterpret_cast<const uint4*>(vc + W * 128 + 16 * r);
    const uint32_t xw[4] = {vx.x, vx.y, vx.z, vx.w}, yw[4] = {vy.x, vy.y, vy.z, vy.w};
    const uint32_t zw[4] = {vz.x, vz.y, vz.z, vz.w}, ww[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      // bytes [x0, y0, x1, y1] and [x2, y2, x3, y3] of word h
      uint32_t e0, e1, e2, e3, f0, f1, f2, f3;
      e4m3x4_to_f16x2x2(prmt(xw[h], yw[h], 0x5140), e0, e1);
      e4m3x4_to_f16x2x2(prmt(xw[h], yw[h], 0x7362), e2, e3);
      e4m3x4_to_f16x2x2(prmt(zw[h], ww[h], 0x5140), f0, f1);
      e4m3x4_to_f16x2x2(prmt(zw[h], ww[h], 0x7362), f2, f3);
      mma_f16_16816(st.o[2 * h], e0, e1, f0, f1, pb0, pb1);
      mma_f16_16816(st.o[2 * h + 1], e2, e3, f2, f3, pb0, pb1);
    }
  }
};

// {1024 + Z_a, 1024 + Z_b} as an FP16 pair for the zero-point MMA of the PV
// product.  Z is any int32: it is negative for a group whose values are all
// positive and exceeds 15 (255) for one whose values are all negative.  The
// pair is exact for -3072 <= Z <= 1024; beyond that it is 1024 + Z rounded to
// FP16, an error below 2^-11 of 1024 + Z, while the group's values
// themselves are about |Z| * S.
__device__ __forceinline__ uint32_t zero_point_pair(uint32_t za, uint32_t zb) {
  return f32x2_to_f16x2(1024.0f + (float)(int)za, 1024.0f + (float)(int)zb);
}
constexpr uint32_t kHalf960 = 0x63806380u;    // FP16 {960, 960}

// INT4 PV (any group size).  V rows are stored with permuted dims (byte
// 8r + m holds dims 16m + r and 16m + r + 8), so thread (r, c) reads one
// 8-byte chunk per key (keys 2c, 2c+1, 2c+8, 2c+9) and every 16-row m-tile
// m = dims 16m .. 16m + 15 lies in one group g.  With v = (n - Z_t) S_t,
//   O^T_m = sum_t v_t P_t = sum_t (1024 + n_t) (S_t P_t) - sum_t (1024 + Z_t) (S_t P_t):
// the m-tile MMA runs on the raw codes against P' = S P (the group's scales
// applied to the B fragment, 2 mul.f16x2 per group), and the zero-point term
// is one more MMA per group, accumulated in st.corr[g] and subtracted from
// the group's O rows before the merge.  Rows r (the low nibble of a byte)
// take the codes as 1024 + n and their zero-point rows are 1024 + Z_t; rows
// r + 8 (the high nibble) take them as 64 + n straight from bits 4-7 (0x5400
// | n << 4, one lop3 and no shift) and their zero-point rows are 64 + Z_t
// (the 1024 + Z_t pair minus 960 in FP16).
// CONV (groups of 64, {f32 S, i32 Z} metadata): the part's V metadata was
// rewritten in shared memory by Int4G64Slab::prepare as, per key pair and
// group, the FP16 pairs {S, S'}, {1024 + Z, 1024 + Z'} and {64 + Z, 64 + Z'}
// of the pair's two keys, so a pair's operands of a group are one 16-byte
// load.
template <int GROUP, bool COMPACT = false, bool CONV = false>
__device__ __forceinline__ void int4_pv(const uint8_t* vc, const uint8_t* vm, int r, int c,
                                        uint32_t pb0, uint32_t pb1, WarpState<D / GROUP>& st) {
  constexpr int NG = D / GROUP;          // groups per row
  constexpr int MPG = GROUP / 16;        // m-tiles per group
  // meta bytes per key: {f32 S, i32 Z} per group, or compact {f16 S0, f16 S1, i8 Z0, i8 Z1, 0, 0}
  constexpr int MB = COMPACT ? 8 : NG * 8;
  const int X = 2 * c, Y = 2 * c + 1, Z = 2 * c + 8, W = 2 * c + 9;
  const uint2 vx = *reinterpret_cast<const uint2*>(vc + X * 64 + 8 * r);
  const uint2 vy = *reinterpret_cast<const uint2*>(vc + Y * 64 + 8 * r);
  const uint2 vz = *reinterpret_cast<const uint2*>(vc + Z * 64 + 8 * r);
  const uint2 vw = *reinterpret_cast<const uint2*>(vc + W * 64 + 8 * r);
  // A fragments: word h of a key's chunk holds m-tiles 4h .. 4h+3, byte i =
  // m-tile 4h + i (low nibble row r, high nibble row r + 8); the 16-bit
  // halves of the XY / ZW pairs put key X (Z) low and key Y (W) high.
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    uint32_t q0, q1, zxy, zzw, zxy64, zzw64;
    if constexpr (CONV) {   // slot X + g: group g of keys (X, Y); Z + g: of (Z, W)
      const uint4 cxy = *reinterpret_cast<const uint4*>(vm + (X + g) * 16);
      const uint4 czw = *reinterpret_cast<const uint4*>(vm + (Z + g) * 16);
      q0 = hmul2(pb0, cxy.x);
      q1 = hmul2(pb1, czw.x);
      zxy = cxy.y;
      zzw = czw.y;
      zxy64 = cxy.z;
      zzw64 = czw.z;
    } else if constexpr (COMPACT) {
      // word 0: S0 | S1 (f16), word 1: Z0, Z1 (i8) in its low two bytes
      const uint2 mx = *reinterpret_cast<const uint2*>(vm + X * MB);
      const uint2 my = *reinterpret_cast<const uint2*>(vm + Y * MB);
      const uint2 mz = *reinterpret_cast<const uint2*>(vm + Z * MB);
      const uint2 mw = *reinterpret_cast<const uint2*>(vm + W * MB);
      const uint32_t sel = g ? 0x7632u : 0x5410u;   // half g of each key's S word
      q0 = hmul2(pb0, prmt(mx.x, my.x, sel));
      q1 = hmul2(pb1, prmt(mz.x, mw.x, sel));
      const int sh = 8 * g;
      zxy = zero_point_pair((uint32_t)(int)(int8_t)(mx.y >> sh), (uint32_t)(int)(int8_t)(my.y >> sh));
      zzw = zero_point_pair((uint32_t)(int)(int8_t)(mz.y >> sh), (uint32_t)(int)(int8_t)(mw.y >> sh));
    } else {
      const uint2 mx = *reinterpret_cast<const uint2*>(vm + X * MB + 8 * g);
      const uint2 my = *reinterpret_cast<const uint2*>(vm + Y * MB + 8 * g);
      const uint2 mz = *reinterpret_cast<const uint2*>(vm + Z * MB + 8 * g);
      const uint2 mw = *reinterpret_cast<const uint2*>(vm + W * MB + 8 * g);
      // P' = S P for keys (X, Y) and (Z, W)
      q0 = hmul2(pb0, f32x2_to_f16x2(__uint_as_float(mx.x), __uint_as_float(my.x)));
      q1 = hmul2(pb1, f32x2_to_f16x2(__uint_as_float(mz.x), __uint_as_float(mw.x)));
      zxy = zero_point_pair(mx.y, my.y);
      zzw = zero_point_pair(mz.y, mw.y);
    }
    if constexpr (!CONV) {
      zxy64 = hsub2(zxy, kHalf960);
      zzw64 = hsub2(zzw, kHalf960);
    }
    mma_f16_16816(st.corr[g], zxy, zxy64, zzw, zzw64, q0, q1);
#pragma unroll
    for (int j = 0; j < MPG; j += 2) {
      const int mt = MPG * g + j, h = mt >> 2, half = (mt >> 1) & 1;
      const uint32_t xw = h ? vx.y : vx.x, yw = h ? vy.y : vy.x;
      const uint32_t zw = h ? vz.y : vz.x, ww = h ? vw.y : vw.x;
      const uint32_t sel = half ? 0x7632u : 0x5410u;
      const uint32_t e = prmt(xw, yw, sel), f = prmt(zw, ww, sel);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t ei = e >> (8 * i), fi = f >> (8 * i);
        mma_f16_16816(st.o[mt + i], lop3_and_or(ei, 0x000F000Fu, 0x64006400u),
                      lop3_and_or(ei, 0x00F000F0u, 0x54005400u),
                      lop3_and_or(fi, 0x000F000Fu, 0x64006400u),
                      lop3_and_or(fi, 0x00F000F0u, 0x54005400u), q0, q1);
      }
    }
  }
}

template <int GROUP>
struct Slab<KVQ_INT4, GROUP> {
  static constexpr int MB = (D / GROUP) * 8;
  // {1024 + n_j, 1024 + n_{j+4}} from nibbles j and j+4 of w
  static __device__ __forceinline__ uint32_t magic(uint32_t w, int j) {
    return lop3_and_or(w >> (4 * j), 0x000F000Fu, 0x64006400u);
  }
  static __device__ __forceinline__ void qk(const uint8_t* kc, const uint8_t* km, int r, int c,
                                            const uint32_t (&qf)[16], const float (&)[8],
                                            bool, float (&acc)[4]) {
    const uint4 k0 = *reinterpret_cast<const uint4*>(kc + r * 64 + 16 * c);
    const uint4 k1 = *reinterpret_cast<const uint4*>(kc + (r + 8) * 64 + 16 * c);
    const int gi = (32 * c) / GROUP;
    const uint2 m0 = *reinterpret_cast<const uint2*>(km + r * MB + 8 * gi);
    const uint2 m1 = *reinterpret_cast<const uint2*>(km + (r + 8) * MB + 8 * gi);
    const float z0 = 1024.0f + (float)(int)m0.y, z1 = 1024.0f + (float)(int)m1.y;
    const uint32_t zz0 = f32x2_to_f16x2(z0, z0), zz1 = f32x2_to_f16x2(z1, z1);
    const float S0 = __uint_as_float(m0.x), S1 = __uint_as_float(m1.x);
    const uint32_t ss0 = f32x2_to_f16x2(S0, S0), ss1 = f32x2_to_f16x2(S1, S1);
    const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w};
    const uint32_t w1[4] = {k1.x, k1.y, k1.z, k1.w};
    float ac[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int wi = s >> 1, j = 2 * (s & 1);
      const uint32_t a0 = hmul2(hsub2(magic(w0[wi], j), zz0), ss0);
      const uint32_t a2 = hmul2(hsub2(magic(w0[wi], j + 1), zz0), ss0);
      const uint32_t a1 = hmul2(hsub2(magic(w1[wi], j), zz1), ss1);
      const uint32_t a3 = hmul2(hsub2(magic(w1[wi], j + 1), zz1), ss1);
      mma_f16_16816(ac[s & 1], a0, a1, a2, a3, qf[2 * s], qf[2 * s + 1]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = ac[0][e] + ac[1][e];
  }
  static __device__ __forceinline__ void pv(const uint8_t* vc, const uint8_t* vm, int r, int c,
                                            uint32_t pb0, uint32_t pb1, WarpState<D / GROUP>& st) {
    int4_pv<GROUP>(vc, vm, r, c, pb0, pb1, st);
  }
};

// INT4 with groups of 64, K side factored: the MMA runs on the raw codes
// offset by a constant o_d (exact in FP16), one accumulator per group, and
// the group's S and Z are applied to the FP32 result:
//   score = sum_g S_g * (sum_{d in g} q'_d (o_d + n_d) - sum_{d in g} o_d q'_d - Z_g * sum_{d in g} q'_d).
// A code taken from bits 0-3 of a 16-bit half becomes 1024 + n with one
// lop3 (0x6400 | n); one taken from bits 4-7 becomes 64 + n, also with one
// lop3 (0x5400 | n << 4: the ulp at 64 is 1/16), so a word's eight codes
// cost four lop3 and one shift.  Values with offset 1024 pair with the even
// Q registers, those with offset 64 with the odd ones.  load_q supplies
// -sum o_d q'_d per group and column (qs[4..7]); the group's MMA
// accumulators start there, so the offsets cancel inside the accumulation.
// Thread c covers dims [16c, 16c+16) of each group (bytes 8c.. and 32+8c..).
// COMPACT: the group metadata is {f16 S0, f16 S1, i8 Z0, i8 Z1, 0, 0} per
// token instead of {f32 S, i32 Z} per group.
template <bool COMPACT>
struct Int4G64Slab {
  static constexpr int MB = COMPACT ? 8 : 16;
  static constexpr bool kHiloSummed = true;
  // {f32 S, i32 Z} metadata is converted once per part and key in shared
  // memory (one key per lane), instead of once per slab by each of the 4
  // (K) or 8 (V) lanes that read it: K keeps {S0, float(Z0), S1, float(Z1)}.
  // V is regrouped by key pair (2j, 2j + 1), the pairs the PV A operand
  // takes together: slot 2j + g holds group g of the pair as {FP16 pair
  // S(2j) | S(2j+1), FP16 pair 1024 + Z(2j) | 1024 + Z(2j+1), FP16 pair
  // 64 + Z(2j) | 64 + Z(2j+1), 0} (the two lanes of a pair trade their
  // converted values with one exchange each).  The values are those the
  // per-slab conversions gave.  Called by the whole warp before the part's
  // slabs, with `nkeys` the part's keys, a multiple of 32 (all of them,
  // stale ones included: cache memory beyond the valid tokens holds finite
  // metadata, zero or earlier tokens').
  static constexpr bool kConv = !COMPACT;
  static __device__ __forceinline__ void prepare(uint8_t* km, uint8_t* vm, int nkeys, int lane) {
    if constexpr (kConv) {
      for (int k = lane; k < nkeys; k += 32) {   // (nkeys % 32 == 0: every lane exchanges)
        uint4 m = *reinterpret_cast<const uint4*>(km + k * MB);
        m.y = __float_as_uint((float)(int)m.y);
        m.w = __float_as_uint((float)(int)m.w);
        *reinterpret_cast<uint4*>(km + k * MB) = m;
        const uint4 v = *reinterpret_cast<const uint4*>(vm + k * MB);
        const float z0 = (float)(int)v.y, z1 = (float)(int)v.w;
        const uint32_t s2 = f32x2_to_f16x2(__uint_as_float(v.x), __uint_as_float(v.z));   // S0 | S1
        const uint32_t z2 = f32x2_to_f16x2(1024.0f + z0, 1024.0f + z1);
        const uint32_t ps = __shfl_xor_sync(0xffffffffu, s2, 1);   // the pair's other key
        const uint32_t pz = __shfl_xor_sync(0xffffffffu, z2, 1);
        uint4 o;   // even key: group 0 {own, partner}; odd key: group 1 {partner, own}
        if (k & 1) {
          o.x = prmt(ps, s2, 0x7632u), o.y = prmt(pz, z2, 0x7632u);
        } else {
          o.x = prmt(s2, ps, 0x5410u), o.y = prmt(z2, pz, 0x5410u);
        }
        o.z = hsub2(o.y, kHalf960);   // 64 + Z of both keys
        o.w = 0u;
        *reinterpret_cast<uint4*>(vm + k * MB) = o;
      }
    }
  }
  // codes j of both 16-bit halves of w (j = 0..3): 1024 + n for even j, 64 + n for odd j
  static __device__ __forceinline__ uint32_t magic(uint32_t w, int j) {
    const uint32_t x = j >= 2 ? w >> 8 : w;
    return (j & 1) ? lop3_and_or(x, 0x00F000F0u, 0x54005400u) : lop3_and_or(x, 0x000F000Fu, 0x64006400u);
  }
  static __device__ __forceinline__ void qk(const uint8_t* kc, const uint8_t* km, int r, int c,
                                            const uint32_t (&qf)[16], const float (&qs)[8],
                                            bool hilo, float (&acc)[4]) {
    const uint2 c00 = *reinterpret_cast<const uint2*>(kc + r * 64 + 8 * c);
    const uint2 c01 = *reinterpret_cast<const uint2*>(kc + r * 64 + 32 + 8 * c);
    const uint2 c10 = *reinterpret_cast<const uint2*>(kc + (r + 8) * 64 + 8 * c);
    const uint2 c11 = *reinterpret_cast<const uint2*>(kc + (r + 8) * 64 + 32 + 8 * c);
    const uint32_t wr[2][2] = {{c00.x, c00.y}, {c01.x, c01.y}};
    const uint32_t wr8[2][2] = {{c10.x, c10.y}, {c11.x, c11.y}};
    float ac[2][4] = {{qs[4], qs[5], qs[4], qs[5]}, {qs[6], qs[7], qs[6], qs[7]}};   // -offset sums
#pragma unroll
    for (int g = 0; g < 2; ++g) {
#pragma unroll
      for (int sp = 0; sp < 4; ++sp) {
        const int s = 4 * g + sp, wi = sp >> 1, j = 2 * (sp & 1);
        mma_f16_16816(ac[g], magic(wr[g][wi], j), magic(wr8[g][wi], j), magic(wr[g][wi], j + 1),
                      magic(wr8[g][wi], j + 1), qf[2 * s], qf[2 * s + 1]);
      }
    }
    float zr0, zr1, z80, z81, sr0, sr1, s80, s81;
    if constexpr (COMPACT) {
      const uint2 m0 = *reinterpret_cast<const uint2*>(km + r * MB);       // S0 | S1, Z0 Z1
      const uint2 m1 = *reinterpret_cast<const uint2*>(km + (r + 8) * MB);
      const float2 s0 = __half22float2(*reinterpret_cast<const __half2*>(&m0.x));
      const float2 s1 = __half22float2(*reinterpret_cast<const __half2*>(&m1.x));
      sr0 = s0.x, sr1 = s0.y, s80 = s1.x, s81 = s1.y;
      zr0 = (float)(int8_t)(m0.y & 0xFFu);
      zr1 = (float)(int8_t)((m0.y >> 8) & 0xFFu);
      z80 = (float)(int8_t)(m1.y & 0xFFu);
      z81 = (float)(int8_t)((m1.y >> 8) & 0xFFu);
    } else {   // converted by prepare: S0, float(Z0), S1, float(Z1)
      const uint4 m0 = *reinterpret_cast<const uint4*>(km + r * MB);
      const uint4 m1 = *reinterpret_cast<const uint4*>(km + (r + 8) * MB);
      zr0 = __uint_as_float(m0.y), zr1 = __uint_as_float(m0.w);
      z80 = __uint_as_float(m1.y), z81 = __uint_as_float(m1.w);
      sr0 = __uint_as_float(m0.x), sr1 = __uint_as_float(m0.z);
      s80 = __uint_as_float(m1.x), s81 = __uint_as_float(m1.z);
    }
    if (hilo) {   // one score per head from both Q' parts (see factored_scores)
      const float a0 = ac[0][0] + ac[0][1], a1 = ac[1][0] + ac[1][1];
      const float a8 = ac[0][2] + ac[0][3], a9 = ac[1][2] + ac[1][3];
      acc[0] = sr0 * fmaf(-zr0, qs[0], a0) + sr1 * fmaf(-zr1, qs[2], a1);
      acc[2] = s80 * fmaf(-z80, qs[0], a8) + s81 * fmaf(-z81, qs[2], a9);
      acc[1] = acc[3] = 0.0f;
    } else {
      acc[0] = sr0 * fmaf(-zr0, qs[0], ac[0][0]) + sr1 * fmaf(-zr1, qs[2], ac[1][0]);
      acc[1] = sr0 * fmaf(-zr0, qs[1], ac[0][1]) + sr1 * fmaf(-zr1, qs[3], ac[1][1]);
      acc[2] = s80 * fmaf(-z80, qs[0], ac[0][2]) + s81 * fmaf(-z81, qs[2], ac[1][2]);
      acc[3] = s80 * fmaf(-z80, qs[1], ac[0][3]) + s81 * fmaf(-z81, qs[3], ac[1][3]);
    }
  }
  static __device__ __forceinline__ void pv(const uint8_t* vc, const uint8_t* vm, int r, int c,
                                            uint32_t pb0, uint32_t pb1, WarpState<2>& st) {
    int4_pv<64, COMPACT, kConv>(vc, vm, r, c, pb0, pb1, st);
  }
};

template <>
struct Slab<KVQ_INT4, 64> : Int4G64Slab<false> {};
template <>
struct Slab<kFmtInt4Compact, 64> : Int4G64Slab<true> {};

// Group metadata forms of the factored INT slabs (groups of 64, two per
// token row):
//   kMetaF32: {f32 S, i32 Z} per group, 16 bytes per token;
//   kMetaC8:  {f16 S0, f16 S1, i8 Z0, i8 Z1, 0, 0}, 8 bytes (INT2, INT4);
//   kMetaC16: {f16 S0, f16 S1, i16 Z0, i16 Z1}, 8 bytes (INT8).
constexpr int kMetaF32 = 0, kMetaC8 = 1, kMetaC16 = 2;

// A row's S0, S1 and 1024 + Z0, 1024 + Z1 (the K side; Z0, Z1 when
// OFF1024 is false).
template <int META, bool OFF1024 = true>
__device__ __forceinline__ void row_meta(const uint8_t* m, float& S0, float& S1, float& zf0,
                                         float& zf1) {
  constexpr float o = OFF1024 ? 1024.0f : 0.0f;
  if constexpr (META == kMetaF32) {
    const uint4 v = *reinterpret_cast<const uint4*>(m);   // S0, Z0, S1, Z1
    S0 = __uint_as_float(v.x);
    S1 = __uint_as_float(v.z);
    zf0 = o + (float)(int)v.y;
    zf1 = o + (float)(int)v.w;
  } else {
    const uint2 v = *reinterpret_cast<const uint2*>(m);
    const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
    S0 = sf.x;
    S1 = sf.y;
    if constexpr (META == kMetaC8) {
      zf0 = o + (float)(int8_t)(v.y & 0xFFu);
      zf1 = o + (float)(int8_t)((v.y >> 8) & 0xFFu);
    } else {
      zf0 = o + (float)(int16_t)(v.y & 0xFFFFu);
      zf1 = o + (float)(int16_t)(v.y >> 16);
    }
  }
}

// Group g of keys a and b (meta rows ma, mb): the FP16 pair {S_a, S_b} and
// the zero-point pair {1024 + Z_a, 1024 + Z_b} (the V side).
template <int META>
__device__ __forceinline__ void pair_meta(const uint8_t* ma, const uint8_t* mb, int g, uint32_t& s2,
                                          uint32_t& z2) {
  if constexpr (META == kMetaF32) {
    const uint2 a = *reinterpret_cast<const uint2*>(ma + 8 * g);
    const uint2 b = *reinterpret_cast<const uint2*>(mb + 8 * g);
    s2 = f32x2_to_f16x2(__uint_as_float(a.x), __uint_as_float(b.x));
    z2 = zero_point_pair(a.y, b.y);
  } else {
    const uint2 a = *reinterpret_cast<const uint2*>(ma);
    const uint2 b = *reinterpret_cast<const uint2*>(mb);
    s2 = prmt(a.x, b.x, g ? 0x7632u : 0x5410u);   // half g of each key's S word
    if constexpr (META == kMetaC8)
      z2 = zero_point_pair((uint32_t)(int)(int8_t)(a.y >> (8 * g)), (uint32_t)(int)(int8_t)(b.y >> (8 * g)));
    else
      z2 = zero_point_pair((uint32_t)(int)(int16_t)(a.y >> (16 * g)),
                           (uint32_t)(int)(int16_t)(b.y >> (16 * g)));
  }
}

// The factored K-side score of rows r and r+8 from the two groups' raw MMA
// sums ac[g]: sum_g S_g (ac_g - (1024 + Z_g) * sum of the group's Q').
// OFFS: the raw sums carry per-value offsets o_d instead of 1024, and they
// started from load_q's qs[4..7] = -sum o_d q'_d, so that they hold
// sum q'_d n_d already: sum_g S_g * (ac_g - Z_g * sum of Q').
// hilo (G <= 4): columns 2c and 2c + 1 hold the scores of Q''s high and
// low FP16 parts of one head, and qs[0], qs[2] the sums of both parts
// (load_q); the two columns' raw sums are added first and one score is
// formed, in column 2c (column 2c + 1 is left 0).
template <int META, bool OFFS = false>
__device__ __forceinline__ void factored_scores(const uint8_t* km, int r, int MB, const float (&ac)[2][4],
                                                const float (&qs)[8], bool hilo, float (&acc)[4]) {
  float sr0, sr1, zr0, zr1, s80, s81, z80, z81;
  row_meta<META, !OFFS>(km + r * MB, sr0, sr1, zr0, zr1);
  row_meta<META, !OFFS>(km + (r + 8) * MB, s80, s81, z80, z81);
  if (hilo) {
    const float a0 = ac[0][0] + ac[0][1], a1 = ac[1][0] + ac[1][1];
    const float a8 = ac[0][2] + ac[0][3], a9 = ac[1][2] + ac[1][3];
    acc[0] = sr0 * fmaf(-zr0, qs[0], a0) + sr1 * fmaf(-zr1, qs[2], a1);
    acc[2] = s80 * fmaf(-z80, qs[0], a8) + s81 * fmaf(-z81, qs[2], a9);
    acc[1] = acc[3] = 0.0f;
  } else {
    acc[0] = sr0 * fmaf(-zr0, qs[0], ac[0][0]) + sr1 * fmaf(-zr1, qs[2], ac[1][0]);
    acc[1] = sr0 * fmaf(-zr0, qs[1], ac[0][1]) + sr1 * fmaf(-zr1, qs[3], ac[1][1]);
    acc[2] = s80 * fmaf(-z80, qs[0], ac[0][2]) + s81 * fmaf(-z81, qs[2], ac[1][2]);
    acc[3] = s80 * fmaf(-z80, qs[1], ac[0][3]) + s81 * fmaf(-z81, qs[3], ac[1][3]);
  }
}

// INT8 affine, groups of 64, both sides factored like INT4 g64.  An FP16
// pair {1024 + q_a, 1024 + q_b} is one prmt of the code bytes with 0x64
// (the high byte of 1024.0).
__device__ __forceinline__ uint32_t u8pair_magic(uint32_t w, uint32_t sel) {
  return prmt(w, 0x64646464u, sel);
}

template <int META>
struct Int8Slab {
  static constexpr int MB = META == kMetaF32 ? 16 : 8;
  static constexpr bool kHiloSummed = true;
  // QK: thread c covers dims [64g + 16c, 64g + 16c + 16) of group g, k-step
  // 4g + j taking bytes 4j .. 4j+3 (pairs (0,1) -> a0/a1, (2,3) -> a2/a3).
  static __device__ __forceinline__ void qk(const uint8_t* kc, const uint8_t* km, int r, int c,
                                            const uint32_t (&qf)[16], const float (&qs)[8],
                                            bool hilo, float (&acc)[4]) {
    const uint4 kr0 = *reinterpret_cast<const uint4*>(kc + r * 128 + 16 * c);
    const uint4 kr1 = *reinterpret_cast<const uint4*>(kc + r * 128 + 64 + 16 * c);
    const uint4 k80 = *reinterpret_cast<const uint4*>(kc + (r + 8) * 128 + 16 * c);
    const uint4 k81 = *reinterpret_cast<const uint4*>(kc + (r + 8) * 128 + 64 + 16 * c);
    const uint32_t wr[2][4] = {{kr0.x, kr0.y, kr0.z, kr0.w}, {kr1.x, kr1.y, kr1.z, kr1.w}};
    const uint32_t w8[2][4] = {{k80.x, k80.y, k80.z, k80.w}, {k81.x, k81.y, k81.z, k81.w}};
    float ac[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
#pragma unroll
    for (int g = 0; g < 2; ++g) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s = 4 * g + j;
        mma_f16_16816(ac[g], u8pair_magic(wr[g][j], 0x4140u), u8pair_magic(w8[g][j], 0x4140u),
                      u8pair_magic(wr[g][j], 0x4342u), u8pair_magic(w8[g][j], 0x4342u), qf[2 * s],
                      qf[2 * s + 1]);
      }
    }
    factored_scores<META>(km, r, MB, ac, qs, hilo, acc);
  }
  // PV: V rows are dim-permuted (byte 16r + 2m + h = dim 16m + r + 8h), so
  // thread (r, c) reads one 16-byte chunk per key; m-tile m = dims 16m ..
  // 16m + 15, group m / 4.  Scale on P and zero point as in int4_pv.
  static __device__ __forceinline__ void pv(const uint8_t* vc, const uint8_t* vm, int r, int c,
                                            uint32_t pb0, uint32_t pb1, WarpState<2>& st) {
    const int X = 2 * c, Y = 2 * c + 1, Z = 2 * c + 8, W = 2 * c + 9;
    const uint4 vx = *reinterpret_cast<const uint4*>(vc + X * 128 + 16 * r);
    const uint4 vy = *reinterpret_cast<const uint4*>(vc + Y * 128 + 16 * r);
    const uint4 vz = *reinterpret_cast<const uint4*>(vc + Z * 128 + 16 * r);
    const uint4 vw = *reinterpret_cast<const uint4*>(vc + W * 128 + 16 * r);
    const uint32_t xw[4] = {vx.x, vx.y, vx.z, vx.w}, yw[4] = {vy.x, vy.y, vy.z, vy.w};
    const uint32_t zw[4] = {vz.x, vz.y, vz.z, vz.w}, ww[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      uint32_t sxy, szw, zxy, zzw;
      pair_meta<META>(vm + X * MB, vm + Y * MB, g, sxy, zxy);
      pair_meta<META>(vm + Z * MB, vm + W * MB, g, szw, zzw);
      const uint32_t q0 = hmul2(pb0, sxy), q1 = hmul2(pb1, szw);
      mma_f16_16816(st.corr[g], zxy, zxy, zzw, zzw, q0, q1);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int mt = 4 * g + j, wi = mt >> 1;
        // bytes 2m, 2m+1 of the chunk (rows r, r+8) of keys X, Y (and Z, W)
        const uint32_t sel = (mt & 1) ? 0x7632u : 0x5410u;
        const uint32_t txy = prmt(xw[wi], yw[wi], sel), tzw = prmt(zw[wi], ww[wi], sel);
        mma_f16_16816(st.o[mt], u8pair_magic(txy, 0x4240u), u8pair_magic(txy, 0x4341u),
                      u8pair_magic(tzw, 0x4240u), u8pair_magic(tzw, 0x4341u), q0, q1);
      }
    }
  }
};

template <>
struct Slab<KVQ_INT8, 64> : Int8Slab<kMetaF32> {};
template <>
struct Slab<kFmtInt8Compact, 64> : Int8Slab<kMetaC16> {};

// INT2 affine, groups of 64, both sides factored like INT4 g64.  A 32-bit
// word holds 16 codes of 2 bits, eight per 16-bit half.  The code at bits
// b, b+1 of a half becomes the FP16 value o_b + n with one lop3 (the bits
// OR-ed into the mantissa of o_b, whose ulp is 2^-b):
//   b = 0, 2, 4, 6, 8:  o_b = 1024, 256, 64, 16, 4;
// the codes at b = 10, 12, 14 are taken the same way from the word shifted
// right by 8 (offsets 256, 64, 16), so a word's 16 codes cost eight lop3 and
// one shift.  Used on the K side, where the offsets leave the scores through
// load_q's FP32 sums of o_d q'_d.
__device__ __forceinline__ uint32_t int2_magic(uint32_t w, uint32_t w_sh8, int b) {
  const uint32_t x = b >= 10 ? w_sh8 : w;
  const int bb = b >= 10 ? b - 8 : b;
  const uint32_t mag = bb == 0 ? 0x64006400u : bb == 2 ? 0x5C005C00u : bb == 4 ? 0x54005400u
                       : bb == 6 ? 0x4C004C00u : 0x44004400u;
  return lop3_and_or(x, 0x00030003u << bb, mag);
}
__host__ __device__ constexpr float int2_offset(int b) {
  return b >= 10 ? int2_offset(b - 8) : b == 0 ? 1024.0f : b == 2 ? 256.0f : b == 4 ? 64.0f
                                      : b == 6 ? 16.0f : 4.0f;
}
// INT2 PV (groups of 64 or 32).  V rows are dim-permuted (dim 16m + r + 8h
// in byte 4r + m/2 at bits 2(2(m%2) + h)), so thread (r, c) reads one word
// per key (keys 2c, 2c+1, 2c+8, 2c+9): rows r and r+8 of all eight m-tiles,
// m-tiles 2b and 2b+1 in byte b.  Group g holds m-tiles g*MPG .. g*MPG +
// MPG - 1.  Scale on P and zero point as in int4_pv.
template <int GROUP, int META = kMetaF32>
__device__ __forceinline__ void int2_pv(const uint8_t* vc, const uint8_t* vm, int r, int c,
                                        uint32_t pb0, uint32_t pb1, WarpState<D / GROUP>& st) {
  constexpr int NG = D / GROUP, MPG = GROUP / 16, MB = META == kMetaF32 ? NG * 8 : 8;
  const int X = 2 * c, Y = 2 * c + 1, Z = 2 * c + 8, W = 2 * c + 9;
  const uint32_t xw = *reinterpret_cast<const uint32_t*>(vc + X * 32 + 4 * r);
  const uint32_t yw = *reinterpret_cast<const uint32_t*>(vc + Y * 32 + 4 * r);
  const uint32_t zw = *reinterpret_cast<const uint32_t*>(vc + Z * 32 + 4 * r);
  const uint32_t ww = *reinterpret_cast<const uint32_t*>(vc + W * 32 + 4 * r);
  // (V codes as 1024 + n: the zero-point MMA then removes the same offset
  // from the same FP16 P', so the two FP32 accumulations' rounding of the
  // offset term largely cancels)
  auto magic = [](uint32_t w, int sh) { return lop3_and_or(w >> sh, 0x00030003u, 0x64006400u); };
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    uint32_t sxy, szw, zxy, zzw;
    pair_meta<META>(vm + X * MB, vm + Y * MB, g, sxy, zxy);
    pair_meta<META>(vm + Z * MB, vm + W * MB, g, szw, zzw);
    const uint32_t q0 = hmul2(pb0, sxy), q1 = hmul2(pb1, szw);
    mma_f16_16816(st.corr[g], zxy, zxy, zzw, zzw, q0, q1);
    // the group's bytes of keys X | Y (and Z | W) side by side in 16-bit
    // halves: bytes 2g, 2g+1 (groups of 64) or byte g (groups of 32)
    const uint32_t gb = (uint32_t)g;   // (groups of 32: bytes [x_g, x_g, y_g, y_g])
    const uint32_t sel = MPG == 4 ? (g ? 0x7632u : 0x5410u)
                                  : (gb | (gb << 4) | ((4u + gb) << 8) | ((4u + gb) << 12));
    const uint32_t e = prmt(xw, yw, sel), f = prmt(zw, ww, sel);
#pragma unroll
    for (int i = 0; i < MPG; ++i) {
      const int sh = 8 * (i >> 1) + 4 * (i & 1);   // m-tile g*MPG + i, row r; row r+8 at sh + 2
      mma_f16_16816(st.o[MPG * g + i], magic(e, sh), magic(e, sh + 2), magic(f, sh), magic(f, sh + 2),
                    q0, q1);
    }
  }
}

template <int META>
struct Int2G64Slab {
  static constexpr int MB = META == kMetaF32 ? 16 : 8;
  static constexpr bool kHiloSummed = true;
  // QK: thread c covers dims [64g + 16c, 64g + 16c + 16) of group g, one
  // word per row and group (bytes 16g + 4c .. 16g + 4c + 3); k-step 4g + sp
  // takes code pairs (2sp, 2sp + 8) for a0/a1 and (2sp + 1, 2sp + 9) for
  // a2/a3 (bits 4sp and 4sp + 2 of each half: see int2_magic).
  static __device__ __forceinline__ void qk(const uint8_t* kc, const uint8_t* km, int r, int c,
                                            const uint32_t (&qf)[16], const float (&qs)[8],
                                            bool hilo, float (&acc)[4]) {
    const uint32_t wr[2] = {*reinterpret_cast<const uint32_t*>(kc + r * 32 + 4 * c),
                            *reinterpret_cast<const uint32_t*>(kc + r * 32 + 16 + 4 * c)};
    const uint32_t w8[2] = {*reinterpret_cast<const uint32_t*>(kc + (r + 8) * 32 + 4 * c),
                            *reinterpret_cast<const uint32_t*>(kc + (r + 8) * 32 + 16 + 4 * c)};
    float ac[2][4] = {{qs[4], qs[5], qs[4], qs[5]}, {qs[6], qs[7], qs[6], qs[7]}};   // -offset sums
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const uint32_t wrs = wr[g] >> 8, w8s = w8[g] >> 8;
#pragma unroll
      for (int sp = 0; sp < 4; ++sp) {
        const int s = 4 * g + sp;
        mma_f16_16816(ac[g], int2_magic(wr[g], wrs, 4 * sp), int2_magic(w8[g], w8s, 4 * sp),
                      int2_magic(wr[g], wrs, 4 * sp + 2), int2_magic(w8[g], w8s, 4 * sp + 2),
                      qf[2 * s], qf[2 * s + 1]);
      }
    }
    factored_scores<META, true>(km, r, MB, ac, qs, hilo, acc);
  }
  static __device__ __forceinline__ void pv(const uint8_t* vc, const uint8_t* vm, int r, int c,
                                            uint32_t pb0, uint32_t pb1, WarpState<2>& st) {
    int2_pv<64, META>(vc, vm, r, c, pb0, pb1, st);
  }
};

template <>
struct Slab<KVQ_INT2, 64> : Int2G64Slab<kMetaF32> {};
template <>
struct Slab<kFmtInt2Compact, 64> : Int2G64Slab<kMetaC8> {};

// INT2 with groups of 32: thread c's 32 dims of a row are exactly group c,
// so the K side dequantizes in FP16 like INT4 with groups of 32,
// (1024 + q - (1024 + Z)) * S per pair (q - Z exact; S rounded to FP16).
template <>
struct Slab<KVQ_INT2, 32> {
  static constexpr int MB = 32;
  static __device__ __forceinline__ uint32_t magic(uint32_t w, int sh) {
    return lop3_and_or(w >> sh, 0x00030003u, 0x64006400u);
  }
  static __device__ __forceinline__ void qk(const uint8_t* kc, const uint8_t* km, int r, int c,
                                            const uint32_t (&qf)[16], const float (&)[8],
                                            bool, float (&acc)[4]) {
    const uint2 k0 = *reinterpret_cast<const uint2*>(kc + r * 32 + 8 * c);
    const uint2 k1 = *reinterpret_cast<const uint2*>(kc + (r + 8) * 32 + 8 * c);
    const uint2 m0 = *reinterpret_cast<const uint2*>(km + r * MB + 8 * c);
    const uint2 m1 = *reinterpret_cast<const uint2*>(km + (r + 8) * MB + 8 * c);
    const float z0 = 1024.0f + (float)(int)m0.y, z1 = 1024.0f + (float)(int)m1.y;
    const uint32_t zz0 = f32x2_to_f16x2(z0, z0), zz1 = f32x2_to_f16x2(z1, z1);
    const float S0 = __uint_as_float(m0.x), S1 = __uint_as_float(m1.x);
    const uint32_t ss0 = f32x2_to_f16x2(S0, S0), ss1 = f32x2_to_f16x2(S1, S1);
    const uint32_t w0[2] = {k0.x, k0.y}, w1[2] = {k1.x, k1.y};
    float ac[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int wi = s >> 2, j = 2 * (s & 3);   // code pairs (j, j+8) and (j+1, j+9) of word wi
      const uint32_t a0 = hmul2(hsub2(magic(w0[wi], 2 * j), zz0), ss0);
      const uint32_t a2 = hmul2(hsub2(magic(w0[wi], 2 * j + 2), zz0), ss0);
      const uint32_t a1 = hmul2(hsub2(magic(w1[wi], 2 * j), zz1), ss1);
      const uint32_t a3 = hmul2(hsub2(magic(w1[wi], 2 * j + 2), zz1), ss1);
      mma_f16_16816(ac[s & 1], a0, a1, a2, a3, qf[2 * s], qf[2 * s + 1]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = ac[0][e] + ac[1][e];
  }
  static __device__ __forceinline__ void pv(const uint8_t* vc, const uint8_t* vm, int r, int c,
                                            uint32_t pb0, uint32_t pb1, WarpState<4>& st) {
    int2_pv<32>(vc, vm, r, c, pb0, pb1, st);
  }
};

// Ring tokens (BF16, global memory) for one slab, in the format's Q order.
template <int FMT, int GROUP>
__device__ __forceinline__ void ring_qk(const uint16_t* rk, int ntok, int r, int c,
                                        const uint32_t (&qf)[16], float (&acc)[4]) {
  acc[0] = acc[1] = acc[2] = acc[3] = 0.0f;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    uint32_t a[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {   // a0: row r, reg 2s; a1: row r+8, reg 2s; a2/a3: reg 2s+1
      const int row = r + 8 * (e & 1), i = 2 * s + (e >> 1);
      float lo = 0.0f, hi = 0.0f;
      if (row < ntok) {
        lo = __uint_as_float((uint32_t)rk[row * D + q_dim<FMT, GROUP>(c, i, 0)] << 16);
        hi = __uint_as_float((uint32_t)rk[row * D + q_dim<FMT, GROUP>(c, i, 1)] << 16);
      }
      a[e] = f32x2_to_f16x2(lo, hi);
    }
    mma_f16_16816(acc, a[0], a[1], a[2], a[3], qf[2 * s], qf[2 * s + 1]);
  }
}

// Ring tokens (BF16, natural dim order in global memory) for one slab, into
// the format's O layout (o_dim: INT formats 16mt + r (+8), NVFP4 / FP8
// 16r + 2mt (+1)).  NVFP4 / FP8 scale the values by vscale = 1 / g_V.
template <int FMT, int NC>
__device__ __forceinline__ void ring_pv(const uint16_t* rv, int ntok, int r, int c, uint32_t pb0,
                                        uint32_t pb1, float vscale, WarpState<NC>& st) {
  const int tk[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
  float v[4][16];   // v[t][2mt + hi] = dim o_dim(mt, r, hi) of key tk[t]
#pragma unroll
  for (int t = 0; t < 4; ++t) {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float x = tk[t] < ntok ? __uint_as_float((uint32_t)rv[tk[t] * D + o_dim<FMT>(k >> 1, r, k & 1)] << 16)
                             : 0.0f;
      if constexpr (!kIntAffine<FMT>) x *= vscale;
      v[t][k] = x;
    }
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
    mma_f16_16816(st.o[mt], f32x2_to_f16x2(v[0][2 * mt], v[1][2 * mt]),
                  f32x2_to_f16x2(v[0][2 * mt + 1], v[1][2 * mt + 1]),
                  f32x2_to_f16x2(v[2][2 * mt], v[3][2 * mt]),
                  f32x2_to_f16x2(v[2][2 * mt + 1], v[3][2 * mt + 1]), pb0, pb1);
}

__device__ __forceinline__ void consumer_bar() { __syncthreads(); }

// Q' = q * softmax_scale * log2(e), in this thread's fragment order, as
// FP16 parts: q'_hi = FP16(q') and q'_lo = FP16(q' - q'_hi), so that the
// scores K . (q'_hi + q'_lo) carry q' to about 2^-22 of itself rather than
// FP16's 2^-11 (with large keys the logit error of a plain FP16 Q' alone
// moves the softmax weights visibly).  With G <= 4 query heads the lo parts
// ride in the MMA's spare columns: column 2h (B-fragment lanes 8h..8h+3)
// holds q'_hi of head h and column 2h + 1 its q'_lo, so every lane's score
// fragment holds both parts of head c side by side and softmax_step adds
// them in place; head h's softmax state, P and O then live in column 2h
// (see merge_unit).  With G > 4 column h holds head h's q'_hi only.  For
// the INT formats also the per-group sums of the column's FP16 values for
// the two columns 2c, 2c+1 this thread's score fragment holds: qs[0..3] =
// {group 0 column 2c, group 0 column 2c+1, group 1 column 2c, group 1 column
// 2c+1}.  INT4 and INT2 with groups of 64 also take qs[4..7], the same
// columns' sums of o_d q'_d, negated, o_d being the offset the K value
// paired with q'_d carries (INT4: 1024 for an even Q register, 64 for an
// odd one, see Int4G64Slab; INT2: by bit position, see int2_magic); their
// K-side MMA accumulators start from these.  With hilo (G <= 4) qs[0] and
// qs[2] hold the sums of both Q' parts of head c (qs[1] = qs[3] = 0).
template <int FMT, int GROUP>
__device__ __forceinline__ void load_q(const AttnArgs& a, int b, int kvh, int r, int c,
                                       uint32_t (&qf)[16], float (&qs)[8]) {
  const float qscale = a.softmax_scale * kLog2e;
  const bool hilo = a.G <= 4;
  const int head = hilo ? (r >> 1) : r;
  const bool lo_part = hilo && (r & 1);
  const uint16_t* qp = a.q + (((int64_t)b * a.kv_heads + kvh) * a.G + head) * D;
  constexpr bool kInt4Off = (FMT == KVQ_INT4 && GROUP == 64) || FMT == kFmtInt4Compact;
  constexpr bool kInt2Off = (FMT == KVQ_INT2 && GROUP == 64) || FMT == kFmtInt2Compact;
  constexpr bool kOff = kInt4Off || kInt2Off;
  float g0 = 0.0f, g1 = 0.0f, o0 = 0.0f, o1 = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float lo = 0.0f, hi = 0.0f;
    if (head < a.G) {
      lo = __fmul_rn(__uint_as_float((uint32_t)qp[q_dim<FMT, GROUP>(c, i, 0)] << 16), qscale);
      hi = __fmul_rn(__uint_as_float((uint32_t)qp[q_dim<FMT, GROUP>(c, i, 1)] << 16), qscale);
    }
    uint32_t h2 = f32x2_to_f16x2(lo, hi);
    if (lo_part) {   // the residual is exact in FP32
      const float2 r2 = __half22float2(*reinterpret_cast<const __half2*>(&h2));
      h2 = f32x2_to_f16x2(__fsub_rn(lo, r2.x), __fsub_rn(hi, r2.y));
    }
    qf[i] = h2;
    if ((FMT == KVQ_INT4 && GROUP == 64) || FMT == KVQ_INT8 || FMT == KVQ_INT2 ||
        FMT == kFmtInt4Compact || FMT == kFmtInt8Compact || FMT == kFmtInt2Compact) {
      const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&qf[i]));
      if ((i >> 1) < 4) g0 += h.x + h.y; else g1 += h.x + h.y;
      if (kOff) {
        // the offset of the K values register i pairs with: INT4 g64 by
        // parity; INT2 g64 by the code's bit position 4 (s & 3) + 2 (i & 1)
        const float off = kInt4Off ? ((i & 1) ? 64.0f : 1024.0f)
                                   : int2_offset(4 * ((i >> 1) & 3) + 2 * (i & 1));
        if ((i >> 1) < 4) o0 = fmaf(off, h.x + h.y, o0); else o1 = fmaf(off, h.x + h.y, o1);
      }
    }
  }
  if ((FMT == KVQ_INT4 && GROUP == 64) || FMT == KVQ_INT8 || FMT == KVQ_INT2 ||
      FMT == kFmtInt4Compact || FMT == kFmtInt8Compact || FMT == kFmtInt2Compact) {
    g0 += __shfl_xor_sync(0xffffffffu, g0, 1);
    g0 += __shfl_xor_sync(0xffffffffu, g0, 2);
    g1 += __shfl_xor_sync(0xffffffffu, g1, 1);
    g1 += __shfl_xor_sync(0xffffffffu, g1, 2);
    qs[0] = __shfl_sync(0xffffffffu, g0, 8 * c);       // column 2c lives in lanes 8c..8c+3
    qs[1] = __shfl_sync(0xffffffffu, g0, 8 * c + 4);   // column 2c+1
    qs[2] = __shfl_sync(0xffffffffu, g1, 8 * c);
    qs[3] = __shfl_sync(0xffffffffu, g1, 8 * c + 4);
  } else {
    qs[0] = qs[1] = qs[2] = qs[3] = 0.0f;
  }
  if (kOff) {
    o0 += __shfl_xor_sync(0xffffffffu, o0, 1);
    o0 += __shfl_xor_sync(0xffffffffu, o0, 2);
    o1 += __shfl_xor_sync(0xffffffffu, o1, 1);
    o1 += __shfl_xor_sync(0xffffffffu, o1, 2);
    qs[4] = -__shfl_sync(0xffffffffu, o0, 8 * c);
    qs[5] = -__shfl_sync(0xffffffffu, o0, 8 * c + 4);
    qs[6] = -__shfl_sync(0xffffffffu, o1, 8 * c);
    qs[7] = -__shfl_sync(0xffffffffu, o1, 8 * c + 4);
  } else {
    qs[4] = qs[5] = qs[6] = qs[7] = 0.0f;
  }
  if (hilo) {   // both Q' parts of head c in column 2c's sums (see factored_scores)
    qs[0] += qs[1], qs[2] += qs[3];
    qs[1] = qs[3] = 0.0f;
  }
}

// Fused append (kvq_decode_step): one warp writes unit u's new token -- K
// by lanes 0-15, V by lanes 16-31, 8 head_dim values each -- in the cache
// format, exactly as the append kernels would.  Main-cache writes are
// followed by a proxy fence so that a later bulk copy of the same bytes by
// this CTA sees them.
// Max |x| of the 8 values of each lane over its 16-lane half (K or V), as
// f32 bits of the BF16 magnitude; the half's first lane adds it to the
// token's scale segment (scale renewal).
__device__ __forceinline__ void add_segment_amax(const uint4& w, uint32_t* seg_amax, int part) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) m = max(m, max(ws[j] & 0x7FFFu, (ws[j] >> 16) & 0x7FFFu));
#pragma unroll
  for (int off = 1; off < 16; off <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (part == 0 && m != 0u) atomicMax(seg_amax, m << 16);
}

// pos: the token's main-cache position (new_kind 1; `row` is its plane
// row) or ring slot (new_kind 2).
template <int FMT, int GROUP, bool RENEW = false>
__device__ __forceinline__ void write_new_token(const AttnArgs& a, int64_t u, int lane, int64_t pos,
                                                int64_t row) {
  const int kv = lane >> 4, part = lane & 15;
  const uint16_t* src = (kv ? a.v_new : a.k_new) + u * D + part * 8;
  const uint4 w = *reinterpret_cast<const uint4*>(src);
  const Plane& P = kv ? a.v : a.k;
  if (a.new_kind == 2) {   // a cache with a ring: the token goes to its ring slot as is
    *reinterpret_cast<uint4*>(P.ring + (u * a.R + pos) * D + part * 8) = w;
    return;
  }
  float x[8];
  unpack8(w, x);
  if constexpr (RENEW) {   // NVFP4 / FP8: this token's segment and its amax
    add_segment_amax(w, (kv ? a.seg_amax_v : a.seg_amax_k) + (uint32_t)pos / (uint32_t)a.renewal, part);
  }
  if constexpr (FMT == KVQ_NVFP4) {
    const float g = RENEW ? (kv ? a.gseg_v : a.gseg_k)[(uint32_t)pos / (uint32_t)a.renewal]
                          : (kv ? *a.gscale_v : *a.gscale_k);
    uint32_t packed, bs;
    nvfp4_encode8(x, g, packed, bs);
    if (kv == 0) {
      *reinterpret_cast<uint32_t*>(P.codes + row * (D / 2) + part * 4) = packed;
    } else {   // pair-interleaved V: replace this token's nibbles only (rows
               // and positions have the same parity: capacities and pages are even)
      uint2* dst = reinterpret_cast<uint2*>(P.codes + (row & ~(int64_t)1) * (D / 2) + part * 8);
      const bool odd = pos & 1;
      const uint2 nb = odd ? nvfp4_pair_bytes(0u, packed) : nvfp4_pair_bytes(packed, 0u);
      const uint32_t keep = odd ? 0x0F0F0F0Fu : 0xF0F0F0F0u;
      const uint2 old = *dst;
      *dst = make_uint2((nb.x & ~keep) | (old.x & keep), (nb.y & ~keep) | (old.y & keep));
    }
    if ((part & 1) == 0) P.meta[row * (D / 16) + part / 2] = (uint8_t)bs;
  } else if constexpr (FMT == KVQ_FP8) {
    const float sc = RENEW ? (kv ? a.gseg_v : a.gseg_k)[(uint32_t)pos / (uint32_t)a.renewal]
                           : (kv ? *a.gscale_v : *a.gscale_k);
    *reinterpret_cast<uint2*>(P.codes + row * D + part * 8) = fp8_encode8(x, sc);
  } else if constexpr (FMT == kFmtInt2Compact) {
    __half S16;
    int Z;
    const uint32_t packed = int2_encode8_compact<GROUP>(x, S16, Z);
    const uint32_t vhalf = int2_v_permute_half(packed, part, lane & 16);
    *reinterpret_cast<uint16_t*>(P.codes + row * (D / 4) + part * 2) = (uint16_t)(kv ? vhalf : packed);
    if (part % (GROUP / 8) == 0) {   // {f16 S0, f16 S1, i8 Z0, i8 Z1, 0, 0}
      const int gi = part / (GROUP / 8);
      *reinterpret_cast<__half*>(P.meta + row * 8 + 2 * gi) = S16;
      P.meta[row * 8 + 4 + gi] = (uint8_t)(int8_t)Z;
    }
  } else if constexpr (FMT == kFmtInt8Compact) {
    __half S16;
    int Z;
    const uint2 codes = int8_encode8_compact<GROUP>(x, S16, Z);
    uint32_t w0, w1;
    int8_v_permute_words(codes, part, lane & 16, w0, w1);
    uint8_t* dst = P.codes + row * D;
    if (kv == 0) {
      *reinterpret_cast<uint2*>(dst + part * 8) = codes;
    } else {
      *reinterpret_cast<uint32_t*>(dst + part * 4) = w0;
      *reinterpret_cast<uint32_t*>(dst + (part + 16) * 4) = w1;
    }
    if (part % (GROUP / 8) == 0) {   // {f16 S0, f16 S1, i16 Z0, i16 Z1}
      const int gi = part / (GROUP / 8);
      *reinterpret_cast<__half*>(P.meta + row * 8 + 2 * gi) = S16;
      *reinterpret_cast<int16_t*>(P.meta + row * 8 + 4 + 2 * gi) = (int16_t)Z;
    }
  } else if constexpr (FMT == KVQ_INT2) {
    float S;
    int Z;
    const uint32_t packed = int2_encode8<GROUP>(x, S, Z);
    // V rows in the permuted dim order (both halves of the warp shuffle)
    const uint32_t vhalf = int2_v_permute_half(packed, part, lane & 16);
    *reinterpret_cast<uint16_t*>(P.codes + row * (D / 4) + part * 2) = (uint16_t)(kv ? vhalf : packed);
    constexpr int TPG = GROUP / 8;
    if (part % TPG == 0)
      *reinterpret_cast<uint2*>(P.meta + (row * (D / GROUP) + part / TPG) * 8) =
          make_uint2(__float_as_uint(S), (uint32_t)Z);
  } else if constexpr (FMT == KVQ_INT8) {
    float S;
    int Z;
    const uint2 codes = int8_encode8<GROUP>(x, S, Z);
    // V rows in the permuted dim order (both halves of the warp shuffle)
    uint32_t w0, w1;
    int8_v_permute_words(codes, part, lane & 16, w0, w1);
    uint8_t* dst = P.codes + row * D;
    if (kv == 0) {
      *reinterpret_cast<uint2*>(dst + part * 8) = codes;
    } else {
      *reinterpret_cast<uint32_t*>(dst + part * 4) = w0;
      *reinterpret_cast<uint32_t*>(dst + (part + 16) * 4) = w1;
    }
    constexpr int TPG = GROUP / 8;
    if (part % TPG == 0)
      *reinterpret_cast<uint2*>(P.meta + (row * (D / GROUP) + part / TPG) * 8) =
          make_uint2(__float_as_uint(S), (uint32_t)Z);
  } else if constexpr (FMT == kFmtInt4Compact) {
    __half S16;
    int Z;
    const uint32_t packed = int4_encode8_compact<GROUP>(x, S16, Z);
    const uint32_t vword = int4_v_permute_word(packed, part, lane & 16);
    *reinterpret_cast<uint32_t*>(P.codes + row * (D / 2) + part * 4) = kv ? vword : packed;
    if (part % (GROUP / 8) == 0) {   // {f16 S0, f16 S1, i8 Z0, i8 Z1, 0, 0}
      const int gi = part / (GROUP / 8);
      *reinterpret_cast<__half*>(P.meta + row * 8 + 2 * gi) = S16;
      P.meta[row * 8 + 4 + gi] = (uint8_t)(int8_t)Z;
    }
  } else {
    float S;
    int Z;
    const uint32_t packed = int4_encode8<GROUP>(x, S, Z);
    // V rows in the permuted dim order (both halves of the warp shuffle)
    const uint32_t vword = int4_v_permute_word(packed, part, lane & 16);
    *reinterpret_cast<uint32_t*>(P.codes + row * (D / 2) + part * 4) = kv ? vword : packed;
    constexpr int TPG = GROUP / 8;
    if (part % TPG == 0)
      *reinterpret_cast<uint2*>(P.meta + (row * (D / GROUP) + part / TPG) * 8) =
          make_uint2(__float_as_uint(S), (uint32_t)Z);
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Each warp streams its own share of every tile -- tokens [w*WTOK, (w+1)*WTOK)
// of it, w the warp -- through STAGES private stage buffers, each filled by
// one group of 1-D bulk copies completing on the warp's own mbarrier.  No
// warp waits for another in the main loop; the CTA synchronises only to
// merge at the end of a unit's segment.

// The next tile part this warp requests: the count requested so far, the
// stage it goes to, its tile index within its unit and its first token row
// in the planes (unit * cap + tile * TILE + this warp's offset).
struct Feed {
  int k;
  int stage;
  int lt;
  int64_t row;
};

// Request the next tile part and advance the feed by one tile.  Called by
// the whole warp: every lane keeps the same (warp-uniform) feed state, and
// one elected lane issues the copies.
template <int FMT, int GROUP>
__device__ __forceinline__ void feed_next(const AttnArgs& a, uint8_t* wsm, uint64_t* full, Feed& f,
                                          int tpu) {
  using F = Fmt<FMT, GROUP>;
  uint8_t* dst = wsm + f.stage * F::STAGE_BYTES;
  uint64_t* bar = &full[f.stage];
  if (elect_one()) {
    mbar_arrive_expect_tx(bar, F::WSTAGE);
    bulk_g2s(dst, a.k.codes + f.row * F::CB, F::WTOK * F::CB, bar);
    bulk_g2s(dst + F::WTOK * F::CB, a.v.codes + f.row * F::CB, F::WTOK * F::CB, bar);
    if (F::MB) {
      bulk_g2s(dst + 2 * F::WTOK * F::CB, a.k.meta + f.row * F::MB, F::WTOK * F::MB, bar);
      bulk_g2s(dst + 2 * F::WTOK * F::CB + F::WTOK * F::MB, a.v.meta + f.row * F::MB,
               F::WTOK * F::MB, bar);
    }
  }
  ++f.k;
  if (++f.stage == F::STAGES) f.stage = 0;
  f.row += F::TILE;
  if (++f.lt == tpu) {
    f.lt = 0;
    f.row += a.cap - (int64_t)tpu * F::TILE;
  }
}

// Give back the stage just consumed: its refill is the warp's next tile
// part, requested once every lane's reads of the stage are done.
template <int FMT, int GROUP>
__device__ __forceinline__ void refill(const AttnArgs& a, uint8_t* wsm, uint64_t* full, Feed& f,
                                       int ntiles, int tpu) {
  __syncwarp();
  if (f.k < ntiles) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    feed_next<FMT, GROUP>(a, wsm, full, f, tpu);
  }
}

// Scores, online softmax and P.V for this warp's part of one tile (`ws`:
// the part in its stage).  FULL: all WTOK tokens exist; otherwise `left` of
// them do (the unit's last, partial tile).
// RENEW (scale renewal, NVFP4 / FP8): the slab starting at token tok0 + 16 sp
// of the unit has the K and V scales of its segment; its scores are scaled
// by g_K before the softmax (kscale is then 1).  O is kept in units of the V
// scale of segment *vseg (the last one this warp read): when a slab of
// another segment comes, O is rescaled in FP32 by the ratio of the two
// scales, so the values enter the P.V product unscaled and no per-key
// factor is rounded to FP16.
template <int FMT, int GROUP, bool FULL, bool RENEW = false>
__device__ __forceinline__ void attend_part(const uint8_t* ws, int r, int c,
                                            const uint32_t (&qf)[16], const float (&qs)[8],
                                            float kscale, float ik, bool hilo, int64_t left,
                                            WarpState<Fmt<FMT, GROUP>::NC>& st,
                                            const AttnArgs* a = nullptr, int64_t tok0 = 0,
                                            int* vseg = nullptr) {
  using F = Fmt<FMT, GROUP>;
  if constexpr (HasPrepare<Slab<FMT, GROUP>>::value) {   // per-part metadata conversion
    static_assert(F::WTOK % 32 == 0, "prepare pairs keys across lanes: whole warps of keys");
    Slab<FMT, GROUP>::prepare(const_cast<uint8_t*>(ws) + 2 * F::WTOK * F::CB,
                              const_cast<uint8_t*>(ws) + 2 * F::WTOK * F::CB + F::WTOK * F::MB, F::WTOK,
                              threadIdx.x & 31);
    __syncwarp();
  }
  float acc[F::SPW][4];
#pragma unroll
  for (int sp = 0; sp < F::SPW; ++sp)
    Slab<FMT, GROUP>::qk(ws + sp * SLAB * F::CB, ws + 2 * F::WTOK * F::CB + sp * SLAB * F::MB, r, c,
                         qf, qs, hilo, acc[sp]);
  int segs[F::SPW];
  if constexpr (RENEW) {
    // segment of each slab: one division per part (positions < 2^32; a
    // segment is at least 16 tokens, so the part's WTOK <= 48 tokens cross
    // at most three boundaries)
    const uint32_t P = (uint32_t)a->renewal;
    const uint32_t s0 = (uint32_t)tok0 / P, r0 = (uint32_t)tok0 - s0 * P;
#pragma unroll
    for (int sp = 0; sp < F::SPW; ++sp) {
      const uint32_t t = r0 + sp * SLAB;
      segs[sp] = (int)(s0 + (t >= P) + (t >= 2 * P) + (t >= 3 * P));
      const float ks = __ldg(a->gseg_k + segs[sp]);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[sp][e] *= ks;
    }
  }
  uint32_t pb[F::SPW][2];
  int nvalid[F::SPW];
#pragma unroll
  for (int sp = 0; sp < F::SPW; ++sp) {
    const int64_t l2 = left - sp * SLAB;
    nvalid[sp] = l2 >= SLAB ? SLAB : (l2 > 0 ? (int)l2 : 0);
  }
  softmax_step<F::SPW, FULL, F::NC, HiloSummed<Slab<FMT, GROUP>>::value>(acc, nvalid, r, kscale, ik, hilo,
                                                                      st, pb);
#pragma unroll
  for (int sp = 0; sp < F::SPW; ++sp) {
    if constexpr (RENEW) {
      // (a slab without valid keys adds nothing, and its segment's scale may
      // not exist yet)
      if (nvalid[sp] > 0 && segs[sp] != *vseg) {
        if (*vseg >= 0) {
          const float f = __fdiv_rn(__ldg(a->gseg_v + *vseg), __ldg(a->gseg_v + segs[sp]));
#pragma unroll
          for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int j = 0; j < 4; ++j) st.o[mt][j] *= f;
        }
        *vseg = segs[sp];
      }
    }
    Slab<FMT, GROUP>::pv(ws + F::WTOK * F::CB + sp * SLAB * F::CB,
                         ws + 2 * F::WTOK * F::CB + F::WTOK * F::MB + sp * SLAB * F::MB, r, c,
                         pb[sp][0], pb[sp][1], st);
  }
}

// The residual ring of unit u (len_ring BF16 tokens), read after the main
// cache by the CTA that owns the unit's last tile; warp w takes the ring's
// 16-token slabs w, w + NW, ...
template <int FMT, int GROUP>
__device__ __forceinline__ void attend_ring(const AttnArgs& a, int64_t u, int64_t len_ring,
                                            int warp, int r, int c, const uint32_t (&qf)[16],
                                            float ring_vscale,
                                            WarpState<Fmt<FMT, GROUP>::NC>& st) {
  constexpr int NW = Fmt<FMT, GROUP>::NW;
  if (len_ring > 0) {
    const uint16_t* rk = a.k.ring + u * (int64_t)a.R * D;
    const uint16_t* rv = a.v.ring + u * (int64_t)a.R * D;
    const int nslab = (int)((len_ring + SLAB - 1) / SLAB);
    for (int sl = warp; sl < nslab; sl += NW) {
      float acc[1][4] = {{0.0f, 0.0f, 0.0f, 0.0f}};
      const int nv[1] = {(int)min((int64_t)SLAB, len_ring - (int64_t)sl * SLAB)};
      ring_qk<FMT, GROUP>(rk + (int64_t)sl * SLAB * D, nv[0], r, c, qf, acc[0]);
      uint32_t pb[1][2];
      softmax_step<1, false>(acc, nv, r, 1.0f, 1.0f, a.G <= 4, st, pb);
      ring_pv<FMT>(rv + (int64_t)sl * SLAB * D, nv[0], r, c, pb[0][0], pb[0][1], ring_vscale, st);
    }
  }
}

// End of unit u's segment in this CTA: merge the NW warps' softmax states
// through shared memory (the held stage, or stage 0, as the buffer); a unit
// owned by this CTA alone (first == last) is written out directly, otherwise
// the CTA writes one (m, l, o) record per query head and the last CTA of the
// unit to finish (an atomic count) merges the records and writes the output.
// An empty unit (l = 0: a sequence of a ragged batch with no tokens) gives
// output 0 and log-sum-exp -inf.
template <int FMT, int GROUP>
__device__ __forceinline__ void merge_unit(const AttnArgs& a, uint8_t* smem, int held_stage,
                                           WarpState<Fmt<FMT, GROUP>::NC>& st, int warp, int r,
                                           int c, int64_t u, int cta, int first, int last,
                                           float gv, float* red_m, float* red_l,
                                           volatile int* flags) {
  using F = Fmt<FMT, GROUP>;
  constexpr int NW = F::NW;
  const float l0 = st.l[0], l1 = st.l[1];   // (every row of the ones-MMA holds the whole sum)
  float* red_o = reinterpret_cast<float*>(smem + (held_stage >= 0 ? held_stage : 0) * F::STAGE_BYTES);
  consumer_bar();   // every warp is done with the held stage's data
  if (r == 0) {
    red_m[warp * 8 + 2 * c] = st.m0;
    red_m[warp * 8 + 2 * c + 1] = st.m1;
    red_l[warp * 8 + 2 * c] = l0;
    red_l[warp * 8 + 2 * c + 1] = l1;
  }
  float* ow = red_o + warp * 8 * D;
  if constexpr (F::NC > 0) {   // INT formats: the zero-point term of each group's rows
    constexpr int MPG = 8 / F::NC;   // m-tiles per group
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int g = mt / MPG;
#pragma unroll
      for (int j = 0; j < 4; ++j) st.o[mt][j] -= st.corr[g][j];
    }
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int d0 = o_dim<FMT>(mt, r, 0), d1 = o_dim<FMT>(mt, r, 1);
    ow[(2 * c) * D + d0] = st.o[mt][0];
    ow[(2 * c + 1) * D + d0] = st.o[mt][1];
    ow[(2 * c) * D + d1] = st.o[mt][2];
    ow[(2 * c + 1) * D + d1] = st.o[mt][3];
  }
  consumer_bar();

  const int nct = last - first + 1;
  float* out_u = a.out + u * a.G * D;
  float* rec_u = a.partials + (u * a.maxc) * (int64_t)a.G * REC;
  const int col_step = a.G <= 4 ? 2 : 1;   // head h's column (see load_q)
  for (int idx = threadIdx.x; idx < a.G * D; idx += NW * 32) {
    const int h = idx / D, d = idx % D, hc = h * col_step;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w * 8 + hc]);
    float o = 0.0f, l = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = red_m[w * 8 + hc];
        const float f = (mw == -INFINITY) ? 0.0f : ex2(mw - M);
        o += f * red_o[(w * 8 + hc) * D + d];
        l += f * red_l[w * 8 + hc];
      }
    }
    if (nct == 1) {
      // l == 0: the unit holds no token (a ragged batch's empty sequence)
      out_u[h * D + d] = l > 0.0f ? (o / l) * gv : 0.0f;
      if (a.lse != nullptr && d == 0)
        a.lse[u * a.G + h] = l > 0.0f ? (M + log2f(l)) * kLn2 : -INFINITY;
    } else {
      float* rec = rec_u + ((int64_t)(cta - first) * a.G + h) * REC;
      rec[2 + d] = o;
      if (d == 0) {
        rec[0] = M;
        rec[1] = l;
      }
    }
  }
  if (nct > 1) {
    consumer_bar();   // all record writes issued (and red_o no longer read)
    if (threadIdx.x == 0) {
      __threadfence();   // cumulative: orders the CTA's record writes before the count
      const int old = atomicAdd(&a.counters[u], 1);
      flags[1] = (old == nct - 1) ? 1 : 0;
      if (old == nct - 1) {
        __threadfence();
        atomicExch(&a.counters[u], 0);
      }
    }
    consumer_bar();
    if (flags[1]) {
      // Last CTA of the unit: merge the nct records (L2).  First every
      // record's (m, l) into shared memory in one parallel pass ...
      float* ml = red_o;   // merge buffer is free now: [nct * G][2]
      for (int i = threadIdx.x; i < nct * a.G; i += NW * 32) {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(rec_u + (int64_t)i * REC));
        ml[2 * i] = v.x;
        ml[2 * i + 1] = v.y;
      }
      consumer_bar();
      // ... then each output element with its o loads issued together.
      for (int idx = threadIdx.x; idx < a.G * D; idx += NW * 32) {
        const int h = idx / D, d = idx % D;
        float M = -INFINITY;
        for (int j = 0; j < nct; ++j) M = fmaxf(M, ml[2 * (j * a.G + h)]);
        float o = 0.0f, l = 0.0f;
        for (int j0 = 0; j0 < nct; j0 += 8) {
          float ov[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            ov[jj] = (j0 + jj < nct) ? __ldcg(rec_u + ((int64_t)(j0 + jj) * a.G + h) * REC + 2 + d) : 0.0f;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            if (j0 + jj < nct) {
              const float mj = ml[2 * ((j0 + jj) * a.G + h)];
              const float f = (mj == -INFINITY) ? 0.0f : ex2(mj - M);
              l += f * ml[2 * ((j0 + jj) * a.G + h) + 1];
              o += f * ov[jj];
            }
          }
        }
        out_u[h * D + d] = l > 0.0f ? (o / l) * gv : 0.0f;
        if (a.lse != nullptr && d == 0)
          a.lse[u * a.G + h] = l > 0.0f ? (M + log2f(l)) * kLn2 : -INFINITY;
      }
    }
  }
  consumer_bar();   // merge buffer free again
}

// RING: the kernel reads a BF16 residual ring after the main cache.  The
// INT formats always carry that code (their ring is optional at run time);
// NVFP4 and FP8 get a separate instantiation for caches created with a ring,
// so the ring-less kernel is unchanged.
// RENEW: NVFP4 / FP8 caches with scale renewal (per-segment scales).
template <int FMT, int GROUP, bool RING = kIntAffine<FMT>, bool RENEW = false>
__global__ void __launch_bounds__(Fmt<FMT, GROUP>::THREADS, Fmt<FMT, GROUP>::MIN_BLOCKS)
    decode_attn_kernel(const AttnArgs a) {
  using F = Fmt<FMT, GROUP>;
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NW = F::NW;
  // the warp index, visibly the same in every lane (uniform datapath)
  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + F::BAR_OFF) + warp * F::STAGES;   // this warp's
  float* red_m = reinterpret_cast<float*>(smem + F::BAR_OFF + F::STAGES * NW * 8);      // [NW][8]
  float* red_l = red_m + NW * 8;                                                         // [NW][8]
  volatile int* flags = reinterpret_cast<volatile int*>(red_l + NW * 8);   // [0] abort, [1] last
  uint8_t* wsm = smem + warp * F::WSTRIDE;   // this warp's part of stage 0

  const int cta = blockIdx.x, C = gridDim.x;
  const int units = a.batch * a.kv_heads;
  const bool ring_only = a.tpu == 0;
  // flattened tile range of this CTA (ring-only: one unit per "tile")
  const int tpu = ring_only ? 1 : a.tpu;
  const int64_t wb = ring_only ? 0 : a.wb;
  const int64_t W = (int64_t)units * (tpu + wb);
  const int64_t t_begin = split_first_tile_at(W * cta / C, units, tpu, wb);
  const int64_t t_end = split_first_tile_at(W * (cta + 1) / C, units, tpu, wb);
  const int ntiles = ring_only ? 0 : (int)(t_end - t_begin);

  Feed f;
  f.k = 0;
  f.stage = 0;
  f.lt = (int)(t_begin % tpu);
  f.row = (t_begin / tpu) * a.cap + (int64_t)f.lt * F::TILE + warp * F::WTOK;

  // Fused append (kvq_decode_step): the new token of every unit whose last
  // tile this CTA owns is written by the one warp that reads it -- the warp
  // whose part of the last tile holds it, or, for a ring, the warp
  // whose ring slab holds it -- before that warp requests or reads it.
  const int64_t u_lo = t_begin / tpu;
  const int n_new = (a.new_kind != 0 && t_end > t_begin) ? (int)(t_end / tpu - u_lo) : 0;
  const int w_new = a.new_kind == 1 ? (int)((a.new_pos % F::TILE) / F::WTOK)
                                    : (int)((a.new_pos / SLAB) % NW);
  const bool writer = n_new > 0 && warp == w_new;
  // this warp's first tile part holds a new token
  const bool first_new = writer && a.new_kind == 1 && ntiles > 0 && (t_begin + 1) % tpu == 0;

  if (lane == 0) {
    for (int s = 0; s < F::STAGES; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  // Only the first tile now: requested by every warp at once, the first
  // tiles all land early; the rest of the stages follow once it is in.  A
  // first tile that lies wholly below pre_len (tokens no kernel that may
  // still be running writes) is requested before the wait for the previous
  // kernel of the stream, so its copy overlaps that kernel's tail.
  const bool pre = ntiles > 0 && !first_new &&
                   (int64_t)f.lt * F::TILE + (warp + 1) * F::WTOK <= a.pre_len;
  if (pre) feed_next<FMT, GROUP>(a, wsm, full, f, tpu);
  griddep_wait();
  griddep_launch_dependents();
  if (ntiles > 0 && !first_new && !pre) feed_next<FMT, GROUP>(a, wsm, full, f, tpu);
  if (threadIdx.x == 0) {
    flags[0] = 0;
    flags[1] = 0;
  }
  if (writer) {
    for (int j = 0; j < n_new; ++j)
      write_new_token<FMT, GROUP, RENEW>(a, u_lo + j, lane, a.new_pos, (u_lo + j) * a.cap + a.new_pos);
    __syncwarp();
    if (first_new) feed_next<FMT, GROUP>(a, wsm, full, f, tpu);
  }
  __syncthreads();

  const int r = lane >> 2, c = lane & 3;
  const float kscale = (kIntAffine<FMT> || RENEW) ? 1.0f : *a.gscale_k;
  const float ik = __frcp_rn(kscale);
  // RENEW: each warp's O is brought to absolute units before the merge (its
  // segment's V scale), so the merge multiplies by 1
  const float gv = (kIntAffine<FMT> || RENEW) ? 1.0f : *a.gscale_v;
  // ring values enter O divided by the per-tensor V scale, which the output
  // multiplies back (the quantized part of O is accumulated without it)
  const float ring_vscale = kIntAffine<FMT> ? 1.0f : __frcp_rn(gv);
  int consumed = 0;        // tile parts of this warp processed so far
  int stage = 0;           // consumed % STAGES
  uint32_t phase = 0;      // (consumed / STAGES) & 1
  // the unit's last tile holds fewer than TILE tokens
  const bool partial_last = (a.len_main % F::TILE) != 0;

  for (int64_t seg = t_begin; seg < t_end;) {
    const int64_t u = seg / tpu;
    const int64_t seg_end = min(t_end, (u + 1) * tpu);
    const int b = (int)(u / a.kv_heads), kvh = (int)(u % a.kv_heads);
    uint32_t qf[16];
    float qs[8];
    load_q<FMT, GROUP>(a, b, kvh, r, c, qf, qs);
    const bool hilo = a.G <= 4;
    WarpState<F::NC> st;
    state_reset(st);
    int vseg = -1;         // RENEW: the V-scale segment O is in units of (none yet)

    int held_stage = -1;   // stage kept as the merge buffer
    if (!ring_only) {
      const int lt_end = (int)(seg_end - u * tpu);
      // A partial last tile is taken out of the main loop, which then needs
      // no masking.
      const bool tail = partial_last && seg_end == (u + 1) * tpu;
      const int lt_full = tail ? lt_end - 1 : lt_end;
      // wait for the current tile part; after the first, request the rest
      // of the first stage set
      auto arrive = [&]() {
        const bool ok = mbar_wait_bounded(&full[stage], phase, a.dev_status, kDevErrTimeoutFull,
                                          kWaitLimitNs, flags);
        if (consumed == 0) {
          while (f.k < ntiles && f.k < F::STAGES) feed_next<FMT, GROUP>(a, wsm, full, f, tpu);
        }
        return ok;
      };
      // done with tile lt: refill its stage, or keep it for the merge
      auto release = [&](int lt) {
        if (lt + 1 == lt_end)
          held_stage = stage;   // refilled after the merge below
        else
          refill<FMT, GROUP>(a, wsm, full, f, ntiles, tpu);
        ++consumed;
        if (++stage == F::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      };
      int lt = (int)(seg - u * tpu);
      for (; lt < lt_full; ++lt) {
        if (arrive())
          attend_part<FMT, GROUP, true, RENEW>(wsm + stage * F::STAGE_BYTES, r, c, qf, qs, kscale, ik, hilo,
                                               F::WTOK, st, &a,
                                               (int64_t)lt * F::TILE + warp * F::WTOK, &vseg);
        release(lt);
      }
      if (lt < lt_end) {
        const int64_t left = a.len_main - ((int64_t)lt * F::TILE + warp * F::WTOK);
        if (arrive() && left > 0)
          attend_part<FMT, GROUP, false, RENEW>(wsm + stage * F::STAGE_BYTES, r, c, qf, qs, kscale, ik, hilo,
                                                left, st, &a,
                                                (int64_t)lt * F::TILE + warp * F::WTOK, &vseg);
        release(lt);
      }
    }

    // Residual ring: read by the CTA that owns the unit's last tile.
    if (RING && seg_end == (u + 1) * tpu && !flags[0])
      attend_ring<FMT, GROUP>(a, u, a.len_ring, warp, r, c, qf, ring_vscale, st);

    if constexpr (RENEW) {   // O to absolute units
      if (vseg >= 0) {
        const float gsv = __ldg(a.gseg_v + vseg);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
          for (int j = 0; j < 4; ++j) st.o[mt][j] *= gsv;
      }
    }
    {
      const int64_t u_first = u * tpu;
      const int first = (int)split_cta_of_tile(u_first, tpu, wb, W, C);
      const int last = (int)split_cta_of_tile(u_first + tpu - 1, tpu, wb, W, C);
      merge_unit<FMT, GROUP>(a, smem, held_stage, st, warp, r, c, u, cta, first, last, gv, red_m,
                             red_l, flags);
    }
    if (held_stage >= 0) refill<FMT, GROUP>(a, wsm, full, f, ntiles, tpu);
    seg = seg_end;
  }

  // Copies can still be in flight here only if a wait gave up (every tile
  // part is requested and consumed even then): let this warp's last ones
  // land before exiting.
  if (lane == 0 && flags[0]) {
    for (int k = f.k > F::STAGES ? f.k - F::STAGES : 0; k < f.k; ++k)
      mbar_wait_bounded(&full[k % F::STAGES], (k / F::STAGES) & 1, a.dev_status,
                        kDevErrTimeoutDrain, kWaitLimitNs, nullptr);
  }
}


// ---------------------------------------------------------------------------
// Ragged batches and paged planes.  Sequence b holds seq_main[b] main-cache
// and seq_ring[b] ring tokens; each of its units owns s_b = max(1, tiles)
// consecutive slots of the flattened slot line (one slot per main-cache tile;
// a unit without main-cache tokens owns one slot for its ring, or for an
// output of zeros when it holds nothing).  CTA i owns slots
// [cta_slot[i], cta_slot[i+1]) -- the host splits the line with the same
// unit-start weights as the uniform kernel -- and streams the tiles among
// them exactly as the uniform kernel does; only the unit bookkeeping and the
// plane rows (the block table of a paged cache) differ.
// ---------------------------------------------------------------------------

// Largest b < n with seq_slot0[b] <= x (seq_slot0 is strictly increasing:
// every sequence owns at least kv_heads slots).
__device__ __forceinline__ int ragged_seq_of_slot(const RaggedArgs& ra, int n, int x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ra.seq_slot0[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The CTA whose slot range holds slot x: the largest i < C with
// cta_slot[i] <= x (empty ranges have equal bounds and never qualify over
// the next non-empty one).
__device__ __forceinline__ int ragged_cta_of_slot(const RaggedArgs& ra, int C, int x) {
  int lo = 0, hi = C - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ra.cta_slot[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int TILE>
__device__ __forceinline__ int ragged_tiles(const RaggedArgs& ra, int b) {
  return (ra.seq_main[b] + TILE - 1) / TILE;
}

// Next tile part this warp requests: unit (b, h), tile lt of that unit's
// `tiles`, plus the request count and stage as in Feed.
struct RaggedFeed {
  int k;
  int stage;
  int b, h, lt, tiles;
};

// Move the feed to the next main-cache tile: the next tile of the unit, or
// the first tile of the next unit that has any (units of empty sequences and
// ring-only units are skipped).
template <int TILE>
__device__ __forceinline__ void ragged_feed_advance(const RaggedArgs& ra, int nseq, int H,
                                                    RaggedFeed& f) {
  if (++f.lt < f.tiles) return;
  f.lt = 0;
  for (;;) {
    if (++f.h >= H) {
      f.h = 0;
      if (++f.b >= nseq) {
        f.tiles = 0;
        return;
      }
      f.tiles = ragged_tiles<TILE>(ra, f.b);
    }
    if (f.tiles > 0) return;
  }
}

template <int FMT, int GROUP>
__device__ __forceinline__ void ragged_feed_next(const AttnArgs& a, const RaggedArgs& ra,
                                                 uint8_t* wsm, uint64_t* full, RaggedFeed& f,
                                                 int warp) {
  using F = Fmt<FMT, GROUP>;
  uint8_t* dst = wsm + f.stage * F::STAGE_BYTES;
  uint64_t* bar = &full[f.stage];
  if (elect_one()) {
    // a warp share never crosses a page: pages hold whole tiles
    const int64_t row = plane_row((int64_t)f.b * a.kv_heads + f.h, (int64_t)f.lt * F::TILE + warp * F::WTOK,
                                  a.cap, a.kv_heads, ra.pages, ra.page_tokens, ra.max_pages);
    mbar_arrive_expect_tx(bar, F::WSTAGE);
    bulk_g2s(dst, a.k.codes + row * F::CB, F::WTOK * F::CB, bar);
    bulk_g2s(dst + F::WTOK * F::CB, a.v.codes + row * F::CB, F::WTOK * F::CB, bar);
    if (F::MB) {
      bulk_g2s(dst + 2 * F::WTOK * F::CB, a.k.meta + row * F::MB, F::WTOK * F::MB, bar);
      bulk_g2s(dst + 2 * F::WTOK * F::CB + F::WTOK * F::MB, a.v.meta + row * F::MB,
               F::WTOK * F::MB, bar);
    }
  }
  ++f.k;
  if (++f.stage == F::STAGES) f.stage = 0;
  ragged_feed_advance<F::TILE>(ra, a.batch, a.kv_heads, f);
}

template <int FMT, int GROUP>
__device__ __forceinline__ void ragged_refill(const AttnArgs& a, const RaggedArgs& ra, uint8_t* wsm,
                                              uint64_t* full, RaggedFeed& f, int ntiles, int warp) {
  __syncwarp();
  if (f.k < ntiles) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    ragged_feed_next<FMT, GROUP>(a, ra, wsm, full, f, warp);
  }
}

template <int FMT, int GROUP, bool RING = kIntAffine<FMT>>
__global__ void __launch_bounds__(Fmt<FMT, GROUP>::THREADS, Fmt<FMT, GROUP>::MIN_BLOCKS)
    decode_attn_ragged_kernel(const AttnArgs a, const __grid_constant__ RaggedArgs ra) {
  using F = Fmt<FMT, GROUP>;
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NW = F::NW;
  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + F::BAR_OFF) + warp * F::STAGES;
  float* red_m = reinterpret_cast<float*>(smem + F::BAR_OFF + F::STAGES * NW * 8);
  float* red_l = red_m + NW * 8;
  volatile int* flags = reinterpret_cast<volatile int*>(red_l + NW * 8);
  uint8_t* wsm = smem + warp * F::WSTRIDE;

  const int cta = blockIdx.x, C = gridDim.x;
  const int nseq = a.batch, H = a.kv_heads;
  const int X0 = ra.cta_slot[cta], X1 = ra.cta_slot[cta + 1];
  const int b0 = X0 < X1 ? ragged_seq_of_slot(ra, nseq, X0) : 0;

  // Tile parts this warp consumes: every slot in range of a sequence with
  // main-cache tokens is a tile.
  int ntiles = 0;
  for (int b = b0, x = X0; x < X1 && b < nseq; ++b) {
    const int end = min(X1, ra.seq_slot0[b + 1]);
    if (ra.seq_main[b] > 0) ntiles += end - x;
    x = end;
  }

  RaggedFeed f;
  f.k = 0;
  f.stage = 0;
  f.b = nseq;   // an empty range feeds nothing
  f.h = f.lt = f.tiles = 0;
  if (X0 < X1) {
    const int tiles = ragged_tiles<F::TILE>(ra, b0);
    const int s = max(1, tiles), off = X0 - ra.seq_slot0[b0];
    f.b = b0;
    f.h = off / s;
    f.lt = off % s;
    f.tiles = tiles;
    if (tiles == 0) {   // the first unit has no tile: start at the next one that does
      f.lt = 0;
      ragged_feed_advance<F::TILE>(ra, nseq, H, f);
    }
  }

  if (lane == 0) {
    for (int s = 0; s < F::STAGES; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  griddep_wait();   // nothing of the cache is read before the previous kernel is done
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    flags[0] = 0;
    flags[1] = 0;
  }
  // Fused append (kvq_decode_step): the new token of every unit whose last
  // slot this CTA owns is written by the warp that reads it (the warp whose
  // share of the unit's last tile, or whose ring slab, holds it), before
  // that warp requests anything.
  if (a.new_kind != 0 && X0 < X1) {
    for (int b = b0, x = X0; x < X1 && b < nseq; ++b) {
      const int tiles = ragged_tiles<F::TILE>(ra, b), s = max(1, tiles);
      const int base = ra.seq_slot0[b];
      const int end = min(X1, ra.seq_slot0[b + 1]);
      for (int h = (x - base) / s; h < H && base + h * s < end; ++h) {
        if (base + (h + 1) * s > X1) break;   // the unit's last slot is not ours
        const int64_t u = (int64_t)b * H + h;
        const int64_t pos = a.new_kind == 1 ? (int64_t)ra.seq_main[b] - 1 : (int64_t)ra.seq_ring[b] - 1;
        const int w_new = a.new_kind == 1 ? (int)((pos % F::TILE) / F::WTOK) : (int)((pos / SLAB) % NW);
        if (warp == w_new)
          write_new_token<FMT, GROUP>(a, u, lane, pos,
                                      a.new_kind == 1 ? plane_row(u, pos, a.cap, H, ra.pages, ra.page_tokens,
                                                                  ra.max_pages)
                                                      : 0);
      }
      x = end;
    }
    __syncwarp();
  }
  if (ntiles > 0) ragged_feed_next<FMT, GROUP>(a, ra, wsm, full, f, warp);
  __syncthreads();

  const int r = lane >> 2, c = lane & 3;
  const float kscale = kIntAffine<FMT> ? 1.0f : *a.gscale_k;
  const float ik = __frcp_rn(kscale);
  const float gv = kIntAffine<FMT> ? 1.0f : *a.gscale_v;
  const float ring_vscale = kIntAffine<FMT> ? 1.0f : __frcp_rn(gv);
  int consumed = 0, stage = 0;
  uint32_t phase = 0;

  int b = b0, h = 0;
  if (X0 < X1) {
    const int s = max(1, ragged_tiles<F::TILE>(ra, b0));
    h = (X0 - ra.seq_slot0[b0]) / s;
  }
  for (int x = X0; x < X1;) {
    const int tiles = ragged_tiles<F::TILE>(ra, b), s = max(1, tiles);
    const int U0 = ra.seq_slot0[b] + h * s;
    const int seg_end = min(X1, U0 + s);
    const int64_t u = (int64_t)b * H + h;
    uint32_t qf[16];
    float qs[8];
    load_q<FMT, GROUP>(a, b, h, r, c, qf, qs);
    const bool hilo = a.G <= 4;
    WarpState<F::NC> st;
    state_reset(st);

    int held_stage = -1;
    if (tiles > 0) {
      const int64_t len = ra.seq_main[b];
      const int lt_end = seg_end - U0;
      const bool tail = (len % F::TILE) != 0 && lt_end == tiles;
      const int lt_full = tail ? lt_end - 1 : lt_end;
      auto arrive = [&]() {
        const bool ok = mbar_wait_bounded(&full[stage], phase, a.dev_status, kDevErrTimeoutFull,
                                          kWaitLimitNs, flags);
        if (consumed == 0) {
          while (f.k < ntiles && f.k < F::STAGES) ragged_feed_next<FMT, GROUP>(a, ra, wsm, full, f, warp);
        }
        return ok;
      };
      auto release = [&](int lt) {
        if (lt + 1 == lt_end)
          held_stage = stage;
        else
          ragged_refill<FMT, GROUP>(a, ra, wsm, full, f, ntiles, warp);
        ++consumed;
        if (++stage == F::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      };
      int lt = x - U0;
      for (; lt < lt_full; ++lt) {
        if (arrive())
          attend_part<FMT, GROUP, true>(wsm + stage * F::STAGE_BYTES, r, c, qf, qs, kscale, ik, hilo, F::WTOK, st);
        release(lt);
      }
      if (lt < lt_end) {
        const int64_t left = len - ((int64_t)lt * F::TILE + warp * F::WTOK);
        if (arrive() && left > 0)
          attend_part<FMT, GROUP, false>(wsm + stage * F::STAGE_BYTES, r, c, qf, qs, kscale, ik, hilo, left, st);
        release(lt);
      }
    }
    if (RING && seg_end == U0 + s && !flags[0])
      attend_ring<FMT, GROUP>(a, u, ra.seq_ring[b], warp, r, c, qf, ring_vscale, st);
    const int first = ragged_cta_of_slot(ra, C, U0);
    const int last = ragged_cta_of_slot(ra, C, U0 + s - 1);
    merge_unit<FMT, GROUP>(a, smem, held_stage, st, warp, r, c, u, cta, first, last, gv, red_m,
                           red_l, flags);
    if (held_stage >= 0) ragged_refill<FMT, GROUP>(a, ra, wsm, full, f, ntiles, warp);
    x = seg_end;
    if (++h == H) {
      h = 0;
      ++b;
    }
  }

  if (lane == 0 && flags[0]) {
    for (int k = f.k > F::STAGES ? f.k - F::STAGES : 0; k < f.k; ++k)
      mbar_wait_bounded(&full[k % F::STAGES], (k / F::STAGES) & 1, a.dev_status,
                        kDevErrTimeoutDrain, kWaitLimitNs, nullptr);
  }
}

// Launch configuration of the attention kernels: with `pdl`, programmatic
// stream serialization (the kernel may start while the previous kernel of
// the stream finishes; it waits for it with griddep_wait).
inline void launch_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute (&attr)[1], int grid,
                          int threads, int smem, cudaStream_t stream, int pdl) {
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
}

template <int FMT, int GROUP, bool RING = kIntAffine<FMT>, bool RENEW = false>
cudaError_t set_smem_attr() {
  using F = Fmt<FMT, GROUP>;
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<FMT, GROUP, RING, RENEW>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(decode_attn_kernel<FMT, GROUP, RING, RENEW>,
                              cudaFuncAttributePreferredSharedMemoryCarveout,
                              cudaSharedmemCarveoutMaxShared);
}

template <int FMT, int GROUP, bool RING = kIntAffine<FMT>, bool RENEW = false>
cudaError_t launch_impl(const AttnArgs& a, cudaStream_t stream) {
  using F = Fmt<FMT, GROUP>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = set_smem_attr<FMT, GROUP, RING, RENEW>();
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  launch_config(cfg, attr, a.ctas, F::THREADS, F::SMEM, stream, a.pdl);
  return cudaLaunchKernelEx(&cfg, decode_attn_kernel<FMT, GROUP, RING, RENEW>, a);
}

template <int FMT, int GROUP, bool RING = kIntAffine<FMT>, bool RENEW = false>
int blocks_impl() {
  using F = Fmt<FMT, GROUP>;
  if (set_smem_attr<FMT, GROUP, RING, RENEW>() != cudaSuccess) return 1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_attn_kernel<FMT, GROUP, RING, RENEW>, F::THREADS,
                                                    F::SMEM) != cudaSuccess)
    return 1;
  return n > 0 ? n : 1;
}

template <int FMT, int GROUP, bool RING = kIntAffine<FMT>>
cudaError_t launch_ragged_impl(const AttnArgs& a, const RaggedArgs& r, cudaStream_t stream) {
  using F = Fmt<FMT, GROUP>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_attn_ragged_kernel<FMT, GROUP, RING>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_attn_ragged_kernel<FMT, GROUP, RING>,
                               cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  launch_config(cfg, attr, a.ctas, F::THREADS, F::SMEM, stream, a.pdl);
  return cudaLaunchKernelEx(&cfg, decode_attn_ragged_kernel<FMT, GROUP, RING>, a, r);
}

}  // namespace

int attn_tile_tokens(int format, int group) {
  switch (format) {
    case KVQ_NVFP4: return Fmt<KVQ_NVFP4, 16>::TILE;
    case KVQ_FP8: return Fmt<KVQ_FP8, 0>::TILE;
    case KVQ_INT8: return Fmt<KVQ_INT8, 64>::TILE;
    case KVQ_INT2: return group == 32 ? Fmt<KVQ_INT2, 32>::TILE : Fmt<KVQ_INT2, 64>::TILE;
    default:
      static_assert(Fmt<KVQ_INT4, 64>::TILE == Fmt<KVQ_INT4, 32>::TILE &&
                        Fmt<KVQ_INT4, 64>::TILE == Fmt<kFmtInt4Compact, 64>::TILE,
                    "INT4 variants share a tile");
      return Fmt<KVQ_INT4, 64>::TILE;
  }
}

int attn_page_granularity(int format) {
  // a multiple of the tile of every kernel variant of the format
  if (format == KVQ_INT2) {
    static_assert((Fmt<KVQ_INT2, 32>::TILE * 3) % Fmt<KVQ_INT2, 64>::TILE == 0, "INT2 tiles");
    return 3 * Fmt<KVQ_INT2, 32>::TILE;   // 768: both INT2 tiles divide it
  }
  return attn_tile_tokens(format, 0);
}

int attn_blocks_per_sm(int format, bool ring, bool renew, bool compact) {
  switch (format) {
    case KVQ_NVFP4:
      return renew ? blocks_impl<KVQ_NVFP4, 16, false, true>()
                   : ring ? blocks_impl<KVQ_NVFP4, 16, true>() : blocks_impl<KVQ_NVFP4, 16>();
    case KVQ_FP8:
      return renew ? blocks_impl<KVQ_FP8, 0, false, true>()
                   : ring ? blocks_impl<KVQ_FP8, 0, true>() : blocks_impl<KVQ_FP8, 0>();
    case KVQ_INT8: return compact ? blocks_impl<kFmtInt8Compact, 64>() : blocks_impl<KVQ_INT8, 64>();
    case KVQ_INT2:
      if (compact) return blocks_impl<kFmtInt2Compact, 64>();
      return std::min(blocks_impl<KVQ_INT2, 64>(), blocks_impl<KVQ_INT2, 32>());
    default:
      if (compact) return blocks_impl<kFmtInt4Compact, 64>();
      return std::min(blocks_impl<KVQ_INT4, 64>(), blocks_impl<KVQ_INT4, 32>());
  }
}

cudaError_t launch_decode_attention(const AttnArgs& a, cudaStream_t stream) {
  switch (a.format) {
    case KVQ_NVFP4:
      if (a.renewal) return launch_impl<KVQ_NVFP4, 16, false, true>(a, stream);
      return a.R > 0 ? launch_impl<KVQ_NVFP4, 16, true>(a, stream) : launch_impl<KVQ_NVFP4, 16>(a, stream);
    case KVQ_FP8:
      if (a.renewal) return launch_impl<KVQ_FP8, 0, false, true>(a, stream);
      return a.R > 0 ? launch_impl<KVQ_FP8, 0, true>(a, stream) : launch_impl<KVQ_FP8, 0>(a, stream);
    case KVQ_INT4:
      if (a.compact) return launch_impl<kFmtInt4Compact, 64>(a, stream);
      return a.group == 64 ? launch_impl<KVQ_INT4, 64>(a, stream)
                           : launch_impl<KVQ_INT4, 32>(a, stream);
    case KVQ_INT8:
      return a.compact ? launch_impl<kFmtInt8Compact, 64>(a, stream) : launch_impl<KVQ_INT8, 64>(a, stream);
    case KVQ_INT2:
      if (a.compact) return launch_impl<kFmtInt2Compact, 64>(a, stream);
      return a.group == 64 ? launch_impl<KVQ_INT2, 64>(a, stream) : launch_impl<KVQ_INT2, 32>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode_attention_ragged(const AttnArgs& a, const RaggedArgs& r,
                                           cudaStream_t stream) {
  switch (a.format) {
    case KVQ_NVFP4:
      return a.R > 0 ? launch_ragged_impl<KVQ_NVFP4, 16, true>(a, r, stream)
                     : launch_ragged_impl<KVQ_NVFP4, 16>(a, r, stream);
    case KVQ_FP8:
      return a.R > 0 ? launch_ragged_impl<KVQ_FP8, 0, true>(a, r, stream)
                     : launch_ragged_impl<KVQ_FP8, 0>(a, r, stream);
    case KVQ_INT4:
      if (a.compact) return launch_ragged_impl<kFmtInt4Compact, 64>(a, r, stream);
      return a.group == 64 ? launch_ragged_impl<KVQ_INT4, 64>(a, r, stream)
                           : launch_ragged_impl<KVQ_INT4, 32>(a, r, stream);
    case KVQ_INT8:
      return a.compact ? launch_ragged_impl<kFmtInt8Compact, 64>(a, r, stream)
                       : launch_ragged_impl<KVQ_INT8, 64>(a, r, stream);
    case KVQ_INT2:
      if (a.compact) return launch_ragged_impl<kFmtInt2Compact, 64>(a, r, stream);
      return a.group == 64 ? launch_ragged_impl<KVQ_INT2, 64>(a, r, stream)
                           : launch_ragged_impl<KVQ_INT2, 32>(a, r, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kvq
