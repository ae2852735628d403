/*
 * kvq_oracle.c -- plain, slow CPU oracle for the quantized KV-cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke check
 * and the benchmark's CPU-baseline leg may load this library.  It shares no
 * code, header, table or constant generator with the CUDA library under
 * quantized_kv_cache_13_b200/csrc, and it never calls into it.
 *
 * Sources (untrusted web pages; cited by title and section):
 *   [P1] NVFP4 KV-cache article, glsqs.com/news/814573
 *        ("NVFP4 KV缓存技术详解", section 2.1: 16-value groups sharing one
 *        FP8 scale; prefill quantize, decode dequantize, append-on-update).
 *   [P2] "KV Cache量化实战：Model Optimizer为大模型长上下文省下50%显存",
 *        m.nxbn.cn/news/90317 (KV size formula; --kv_cache_qformat table:
 *        fp8 = per-tensor amax calibration, *_cast = constant scale).
 *   [P3] "KV缓存量化技术：提升大模型长文本生成效率", rkmt.cn/news/1711363
 *        (section 2.1 affine formulas for S and Z, grouping of 64;
 *        section 2.2 residual cache of the most recent 128 tokens).
 *   [P1] only says the NVFP4 scales are derived from tensor statistics.
 *   The per-tensor second-level scale amax/(6*448) (the largest E2M1 value
 *   times the largest E4M3 value, so the largest block maps onto the top of
 *   both grids) and round-to-nearest-even on the grid are the readings taken
 *   where it is silent.
 *
 * Precision: every encode decision (scales, codes, zero points) is taken in
 * IEEE binary32 with round-to-nearest, exactly as written below, because the
 * format fixes FP32 scales.  Attention is computed in binary64.  Build with
 * -ffp-contract=off and without -ffast-math so that no operation is fused or
 * reordered.
 *
 * Parity status: every function here is pinned by tests/test_oracle_*.py
 * (library cross-checks, closed forms, invariants, brute force, the pages'
 * printed tables).  No function is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <stdlib.h>

/* ------------------------------------------------------------------------ */
/* E4M3 (OCP FP8, "fn" variant: no infinities, 0x7F/0xFF are NaN).          */
/* Bit layout: s eeee mmm, exponent bias 7; exponent field 0 = subnormal.   */
/* ------------------------------------------------------------------------ */

/* Value of a non-negative E4M3 code 0x00..0x7E (0x7F is NaN, never produced). */
static double e4m3_magnitude(int code)
{
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    if (e == 0)
        return ldexp((double)m / 8.0, -6);           /* subnormal: m/8 * 2^-6 */
    return ldexp(1.0 + (double)m / 8.0, e - 7);      /* normal: (1+m/8)*2^(e-7) */
}

float kvqo_e4m3_decode(uint8_t code)
{
    if ((code & 0x7F) == 0x7F)
        return NAN;
    double v = e4m3_magnitude(code & 0x7F);
    return (float)((code & 0x80) ? -v : v);
}

/*
 * Round-to-nearest-even onto the E4M3 grid with saturation to the largest
 * finite value (448).  Written as a search over the 127 non-negative finite
 * codes: pick the nearest grid value; on an exact tie pick the even code
 * (even mantissa LSB).  The sign of x is kept, so a negative input that
 * rounds to zero gives 0x80.
 */
uint8_t kvqo_e4m3_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);
    int best = 0;
    double best_err = a;                          /* distance to code 0 (= 0.0) */
    for (int c = 1; c <= 0x7E; ++c) {
        double err = fabs(a - e4m3_magnitude(c));
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------------ */
/* E2M1 (FP4): s ee m, grid {0, 0.5, 1, 1.5, 2, 3, 4, 6}, codes 0..7.       */
/* ------------------------------------------------------------------------ */

static const double E2M1_GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

float kvqo_e2m1_decode(uint8_t code)
{
    double v = E2M1_GRID[code & 0x7];
    return (float)((code & 0x8) ? -v : v);
}

/* Nearest grid value, ties to the even code, saturating at 6, sign kept. */
uint8_t kvqo_e2m1_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs((double)x);
    if (a >= 6.0)
        return (uint8_t)(sign | 0x7);
    int best = 0;
    double best_err = a;
    for (int c = 1; c < 8; ++c) {
        double err = fabs(a - E2M1_GRID[c]);
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(sign | best);
}

/* Element-wise wrappers (used by the encoder cross-checks). */
void kvqo_e4m3_encode_array(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = kvqo_e4m3_encode(x[i]);
}
void kvqo_e2m1_encode_array(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = kvqo_e2m1_encode(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Per-tensor scales ([P2] format table: fp8 and nvfp4 calibrate one scale  */
/* per tensor from its amax; the *_cast variants use a constant 1.0).       */
/* ------------------------------------------------------------------------ */

float kvqo_amax(const float* x, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > m) m = a;
    }
    return m;
}

/* NVFP4 second-level scale: amax / (6 * 448); an all-zero tensor gives 1. */
float kvqo_nvfp4_global_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    return amax / 2688.0f;
}

/* FP8 per-tensor scale: amax / 448; an all-zero tensor gives 1. */
float kvqo_fp8_global_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    return amax / 448.0f;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 ([P1] section 2.1): blocks of 16 consecutive values along head_dim */
/* share one E4M3 scale; values are E2M1, two per byte (even index in the   */
/* low nibble).                                                              */
/* ------------------------------------------------------------------------ */

/*
 * Encode `rows` vectors of length D (D a multiple of 16).
 * codes: rows x D/2 bytes; scales: rows x D/16 E4M3 bytes.
 */
void kvqo_nvfp4_encode(const float* x, int64_t rows, int D, float g,
                       uint8_t* codes, uint8_t* scales)
{
    int nb = D / 16;
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * D;
        uint8_t* cr = codes + r * (D / 2);
        for (int b = 0; b < nb; ++b) {
            const float* blk = xr + 16 * b;
            float a = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float v = fabsf(blk[i]);
                if (v > a) a = v;
            }
            float t = a / 6.0f;               /* block amax over the E2M1 max */
            float u = t / g;                  /* relative to the tensor scale */
            uint8_t bs = kvqo_e4m3_encode(u);
            float eff = kvqo_e4m3_decode(bs) * g;
            scales[r * nb + b] = bs;
            for (int i = 0; i < 16; i += 2) {
                uint8_t lo = 0, hi = 0;
                if (eff != 0.0f) {
                    lo = kvqo_e2m1_encode(blk[i] / eff);
                    hi = kvqo_e2m1_encode(blk[i + 1] / eff);
                }
                cr[8 * b + i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

void kvqo_nvfp4_decode(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                       int D, float g, float* out)
{
    int nb = D / 16;
    for (int64_t r = 0; r < rows; ++r) {
        for (int d = 0; d < D; ++d) {
            uint8_t byte = codes[r * (D / 2) + d / 2];
            uint8_t c = (d & 1) ? (byte >> 4) : (byte & 0xF);
            float bs = kvqo_e4m3_decode(scales[r * nb + d / 16]);
            out[r * D + d] = kvqo_e2m1_decode(c) * bs * g;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* MXFP4, for comparison only (an external definition, not from the pages:  */
/* the OCP Microscaling Formats specification v1.0, MXFP4 = E2M1 elements   */
/* with one E8M0 power-of-two scale per block of 32).  [P1] section 3.2     */
/* compares NVFP4 with MXFP4; the comparison study uses this encoder.       */
/* Shared scale X = 2^(floor(log2(max|x|)) - 2), 2 being the exponent of    */
/* E2M1's largest normal (6 = 1.5 * 2^2), clamped to E8M0's 2^-127..2^127;  */
/* elements are E2M1(x / X) with the same rounding and saturation as NVFP4  */
/* (values in [6, 8) * X saturate to 6).  An all-zero block gets the        */
/* smallest scale.  Codes packed as NVFP4's; one E8M0 byte (exponent + 127) */
/* per 32 values.                                                           */
/* ------------------------------------------------------------------------ */

void kvqo_mxfp4_encode(const float* x, int64_t rows, int D, uint8_t* codes, uint8_t* scales)
{
    const int nb = D / 32;
    for (int64_t r = 0; r < rows; ++r) {
        for (int b = 0; b < nb; ++b) {
            const float* blk = x + r * D + b * 32;
            float a = 0.0f;
            for (int i = 0; i < 32; ++i)
                if (fabsf(blk[i]) > a) a = fabsf(blk[i]);
            int e = -127;
            if (a > 0.0f) {
                int ex;
                frexpf(a, &ex);          /* a = m * 2^ex, m in [0.5, 1): floor(log2 a) = ex - 1 */
                e = ex - 1 - 2;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            scales[r * nb + b] = (uint8_t)(e + 127);
            const float X = ldexpf(1.0f, e);
            for (int i = 0; i < 32; ++i) {
                uint8_t c = kvqo_e2m1_encode(blk[i] / X);
                int d = b * 32 + i;
                uint8_t* byte = &codes[r * (D / 2) + d / 2];
                if (d & 1) *byte = (uint8_t)((*byte & 0x0F) | (c << 4));
                else       *byte = (uint8_t)((*byte & 0xF0) | c);
            }
        }
    }
}

void kvqo_mxfp4_decode(const uint8_t* codes, const uint8_t* scales, int64_t rows, int D,
                       float* out)
{
    const int nb = D / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int d = 0; d < D; ++d) {
            uint8_t byte = codes[r * (D / 2) + d / 2];
            uint8_t c = (d & 1) ? (byte >> 4) : (byte & 0xF);
            out[r * D + d] = kvqo_e2m1_decode(c) * ldexpf(1.0f, (int)scales[r * nb + d / 32] - 127);
        }
}

/* ------------------------------------------------------------------------ */
/* FP8-E4M3 with one per-tensor scale ([P2] format table, fp8 / fp8_cast).   */
/* ------------------------------------------------------------------------ */

void kvqo_fp8_encode(const float* x, int64_t n, float s, uint8_t* codes)
{
    for (int64_t i = 0; i < n; ++i) codes[i] = kvqo_e4m3_encode(x[i] / s);
}

void kvqo_fp8_decode(const uint8_t* codes, int64_t n, float s, float* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = kvqo_e4m3_decode(codes[i]) * s;
}

/* ------------------------------------------------------------------------ */
/* INT affine ([P3] section 2.1): per group of `group` values along         */
/* head_dim, S = (max - min) / (2^nbits - 1), Z = round(-min / S),           */
/* q = clamp(round(x / S) + Z, 0, 2^nbits - 1), x^ = (q - Z) * S.            */
/* "round" is round-half-to-even.  The page prints "- Z" in the quantize    */
/* formula; with its own definition of Z that would send the minimum to     */
/* -2*round(min/S), so the consistent reading "+ Z" is used.  A constant     */
/* group (max == min) has no defined S; S = |min| (1 when min == 0) makes   */
/* the code 0 and the reconstruction exact.  4-bit codes are packed two per  */
/* byte, even index in the low nibble.                                       */
/* ------------------------------------------------------------------------ */

void kvqo_int4_encode(const float* x, int64_t rows, int D, int group,
                      uint8_t* codes, float* S_out, int32_t* Z_out)
{
    const int qmax = 15;
    int ng = D / group;
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * D;
        for (int gi = 0; gi < ng; ++gi) {
            const float* grp = xr + gi * group;
            float mn = grp[0], mx = grp[0];
            for (int i = 1; i < group; ++i) {
                if (grp[i] < mn) mn = grp[i];
                if (grp[i] > mx) mx = grp[i];
            }
            float S;
            if (mx == mn)
                S = (mn != 0.0f) ? fabsf(mn) : 1.0f;
            else
                S = (mx - mn) / (float)qmax;
            int32_t Z = (int32_t)rintf(-mn / S);
            S_out[r * ng + gi] = S;
            Z_out[r * ng + gi] = Z;
            for (int i = 0; i < group; ++i) {
                int32_t q = (int32_t)rintf(grp[i] / S) + Z;
                if (q < 0) q = 0;
                if (q > qmax) q = qmax;
                int d = gi * group + i;
                uint8_t* byte = &codes[r * (D / 2) + d / 2];
                if (d & 1) *byte = (uint8_t)((*byte & 0x0F) | (q << 4));
                else       *byte = (uint8_t)((*byte & 0xF0) | q);
            }
        }
    }
}

void kvqo_int4_decode(const uint8_t* codes, const float* S, const int32_t* Z,
                      int64_t rows, int D, int group, float* out)
{
    int ng = D / group;
    for (int64_t r = 0; r < rows; ++r) {
        for (int d = 0; d < D; ++d) {
            uint8_t byte = codes[r * (D / 2) + d / 2];
            int32_t q = (d & 1) ? (byte >> 4) : (byte & 0xF);
            int gi = d / group;
            out[r * D + d] = (float)(q - Z[r * ng + gi]) * S[r * ng + gi];
        }
    }
}

/* The same affine scheme with 8-bit codes (qmax = 255), one code per byte. */
/* [P3] section 2.1 gives the scheme for any bit width; the INT8 variant is */
/* the "nbits = 8" setting of the residual-cache quantizer it describes.    */
void kvqo_int8_encode(const float* x, int64_t rows, int D, int group,
                      uint8_t* codes, float* S_out, int32_t* Z_out)
{
    const int qmax = 255;
    int ng = D / group;
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * D;
        for (int gi = 0; gi < ng; ++gi) {
            const float* grp = xr + gi * group;
            float mn = grp[0], mx = grp[0];
            for (int i = 1; i < group; ++i) {
                if (grp[i] < mn) mn = grp[i];
                if (grp[i] > mx) mx = grp[i];
            }
            float S;
            if (mx == mn)
                S = (mn != 0.0f) ? fabsf(mn) : 1.0f;
            else
                S = (mx - mn) / (float)qmax;
            int32_t Z = (int32_t)rintf(-mn / S);
            S_out[r * ng + gi] = S;
            Z_out[r * ng + gi] = Z;
            for (int i = 0; i < group; ++i) {
                int32_t q = (int32_t)rintf(grp[i] / S) + Z;
                if (q < 0) q = 0;
                if (q > qmax) q = qmax;
                codes[r * D + gi * group + i] = (uint8_t)q;
            }
        }
    }
}

void kvqo_int8_decode(const uint8_t* codes, const float* S, const int32_t* Z,
                      int64_t rows, int D, int group, float* out)
{
    int ng = D / group;
    for (int64_t r = 0; r < rows; ++r) {
        for (int d = 0; d < D; ++d) {
            int gi = d / group;
            out[r * D + d] = (float)((int32_t)codes[r * D + d] - Z[r * ng + gi]) * S[r * ng + gi];
        }
    }
}

/* The same affine scheme with 2-bit codes (qmax = 3): the INT2 row of      */
/* [P3] section 3.1's table, and the strong quantization its section 4.2    */
/* suggests for old chunks of a long context.  Four codes per byte, the     */
/* lowest index in the lowest two bits (the nibble order carried on).       */
void kvqo_int2_encode(const float* x, int64_t rows, int D, int group,
                      uint8_t* codes, float* S_out, int32_t* Z_out)
{
    const int qmax = 3;
    int ng = D / group;
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * D;
        uint8_t* cr = codes + r * (D / 4);
        for (int i = 0; i < D / 4; ++i) cr[i] = 0;
        for (int gi = 0; gi < ng; ++gi) {
            const float* grp = xr + gi * group;
            float mn = grp[0], mx = grp[0];
            for (int i = 1; i < group; ++i) {
                if (grp[i] < mn) mn = grp[i];
                if (grp[i] > mx) mx = grp[i];
            }
            float S;
            if (mx == mn)
                S = (mn != 0.0f) ? fabsf(mn) : 1.0f;
            else
                S = (mx - mn) / (float)qmax;
            int32_t Z = (int32_t)rintf(-mn / S);
            S_out[r * ng + gi] = S;
            Z_out[r * ng + gi] = Z;
            for (int i = 0; i < group; ++i) {
                int32_t q = (int32_t)rintf(grp[i] / S) + Z;
                if (q < 0) q = 0;
                if (q > qmax) q = qmax;
                int d = gi * group + i;
                cr[d / 4] = (uint8_t)(cr[d / 4] | (q << (2 * (d % 4))));
            }
        }
    }
}

void kvqo_int2_decode(const uint8_t* codes, const float* S, const int32_t* Z,
                      int64_t rows, int D, int group, float* out)
{
    int ng = D / group;
    for (int64_t r = 0; r < rows; ++r) {
        for (int d = 0; d < D; ++d) {
            int32_t q = (codes[r * (D / 4) + d / 4] >> (2 * (d % 4))) & 3;
            int gi = d / group;
            out[r * D + d] = (float)(q - Z[r * ng + gi]) * S[r * ng + gi];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Decode attention (the definition, in binary64).                          */
/* For one sequence and one query vector: s_j = scale * <q, k_j>,            */
/* p = softmax(s) (max-subtracted), o = sum_j p_j v_j.                       */
/* K, V: L x D (float); q: D (float); out: D (double).                       */
/* ------------------------------------------------------------------------ */

void kvqo_attention_lse(const float* q, const float* K, const float* V, int64_t L,
                        int D, double scale, double* out, double* lse)
{
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (lse) *lse = -INFINITY;
    if (L <= 0) return;
    double* s = (double*)malloc(sizeof(double) * (size_t)L);
    if (!s) return;
    double smax = -INFINITY;
    for (int64_t j = 0; j < L; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += (double)q[d] * (double)K[j * D + d];
        s[j] = scale * acc;
        if (s[j] > smax) smax = s[j];
    }
    double denom = 0.0;
    for (int64_t j = 0; j < L; ++j) {
        s[j] = exp(s[j] - smax);
        denom += s[j];
    }
    for (int64_t j = 0; j < L; ++j) {
        double p = s[j] / denom;
        for (int d = 0; d < D; ++d) out[d] += p * (double)V[j * D + d];
    }
    /* log of the softmax denominator: log sum_j exp(s_j) */
    if (lse) *lse = smax + log(denom);
    free(s);
}

void kvqo_attention(const float* q, const float* K, const float* V, int64_t L,
                    int D, double scale, double* out)
{
    kvqo_attention_lse(q, K, V, L, D, scale, out, NULL);
}

/*
 * Merge of attention over disjoint parts of one key sequence: part r gave
 * the normalised output o_r and the log-sum-exp lse_r of its scores.  Over
 * the union, exp(lse) = sum_r exp(lse_r) and o = sum_r exp(lse_r - lse) o_r.
 * A part with no keys has lse_r = -inf and weight 0; if every part is empty
 * the result is o = 0, lse = -inf.
 */
void kvqo_combine(int n, int D, const double* o_parts, const double* lse_parts,
                  double* out, double* lse)
{
    double m = -INFINITY;
    for (int r = 0; r < n; ++r)
        if (lse_parts[r] > m) m = lse_parts[r];
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (m == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double wsum = 0.0;
    for (int r = 0; r < n; ++r) {
        double w = (lse_parts[r] == -INFINITY) ? 0.0 : exp(lse_parts[r] - m);
        wsum += w;
        for (int d = 0; d < D; ++d) out[d] += w * o_parts[(int64_t)r * D + d];
    }
    for (int d = 0; d < D; ++d) out[d] /= wsum;
    *lse = m + log(wsum);
}

/*
 * Grouped-query form: q is G x D (the G query heads that share one KV head),
 * out is G x D.  Each head is the single-query definition above.
 */
void kvqo_attention_gqa(const float* q, int G, const float* K, const float* V,
                        int64_t L, int D, double scale, double* out)
{
    for (int h = 0; h < G; ++h)
        kvqo_attention(q + (int64_t)h * D, K, V, L, D, scale, out + (int64_t)h * D);
}
