/*
 * kvq.h -- C ABI of the B200 quantized KV-cache library (libkvq.so).
 *
 * The library quantizes each new token's K/V into a per-layer cache and runs
 * split-K decode attention that reads the quantized cache and dequantizes it
 * in registers.  Five cache formats:
 *
 *   KVQ_NVFP4  E2M1 values, two per byte (even head_dim index in the low
 *              nibble), one E4M3 scale per 16 consecutive values along
 *              head_dim, and one FP32 scale per tensor (K or V of a layer).
 *              Source: NVFP4 KV-cache article (glsqs.com/news/814573),
 *              section 2.1 "technical principle": groups of 16 values share
 *              one FP8 scale; prefill quantizes, decode dequantizes on the
 *              fly, each generated token is quantized and appended.
 *   KVQ_INT4   affine 4-bit codes per group of `group_size` values along
 *              head_dim with S = (max-min)/15, Z = round(-min/S),
 *              q = clamp(round(x/S)+Z, 0, 15); a BF16 residual ring keeps the
 *              most recent `residual_length` tokens and is quantized into
 *              the main cache when it fills.  Source: "KV缓存量化技术：
 *              提升大模型长文本生成效率" (rkmt.cn/news/1711363), section 2.1
 *              (formulas, groups of 64) and section 2.2 (residual cache).
 *   KVQ_INT8   the same affine scheme with 8-bit codes (one per byte, 255
 *              levels), group_size 64, with the same residual ring: the
 *              8-bit setting of the residual-cache quantizer of section 2.1
 *              of the same page.
 *   KVQ_INT2   the same affine scheme with 2-bit codes (four per byte, 3
 *              levels), group_size 64 or 32, with the same residual ring,
 *              which may hold up to 16384 tokens: the INT2 row of section
 *              3.1 of the same page, and the age tiers of its section 4.2
 *              (old chunks in INT2, the newest chunk of 8K-16K tokens kept
 *              in BF16, i.e. a ring of one chunk).
 *   KVQ_FP8    E4M3 codes with one FP32 scale per tensor.  Source:
 *              "KV Cache量化实战：Model Optimizer为大模型长上下文省下50%显存"
 *              (m.nxbn.cn/news/90317), --kv_cache_qformat table (fp8:
 *              per-tensor amax calibration; fp8_cast: constant scale).
 *
 * Conventions for every call:
 *   - Device pointers are CUDA device addresses on the current device; host
 *     pointers are plain host memory.  Nothing here allocates device memory:
 *     the cache buffer, inputs, outputs and the attention workspace all
 *     belong to the caller.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; token counts are kept on
 *     the host, so no call on the append / attention path synchronizes.
 *   - Every call returns a kvq_status.  Arguments are checked on the host
 *     before anything is launched; a failed check leaves the cache
 *     unchanged.  kvq_last_error() gives a message for the last failure on
 *     the calling thread.  No C++ exception crosses this interface.
 *   - A cache handle must not be used from two threads at once.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct kvq_cache* kvq_cache_t;

enum kvq_format {
    KVQ_NVFP4 = 1,
    KVQ_INT4 = 2,
    KVQ_FP8 = 3,
    KVQ_INT8 = 4,
    KVQ_INT2 = 5
};

enum kvq_status {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,     /* bad shape, pointer, alignment or index */
    KVQ_ERR_CAPACITY = 2,        /* append would exceed max_len tokens */
    KVQ_ERR_WORKSPACE = 3,       /* buffer or workspace too small */
    KVQ_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
    KVQ_ERR_DEVICE_TIMEOUT = 5,  /* a kernel gave up a bounded wait */
    KVQ_ERR_UNSUPPORTED = 6,     /* valid but not implemented combination */
    KVQ_ERR_EMPTY = 7            /* attention over a cache with no tokens */
};

/*
 * Raw device layout of one (layer, K|V) pair, for inspection and tests.
 * codes: u8 [batch][kv_heads][capacity][code_bytes].  Token-major for K and
 * for FP8 V (NVFP4/INT4 K: element 2i of a token in the low nibble of its
 * byte i; INT8 K: element d in byte d; INT2 K: element d in byte d/4 at
 * bits 2(d%4)).  The V planes of the NVFP4, INT4 and
 * INT8 formats are stored in the order the decode kernel's V fragments use;
 * the code values are the same:
 *   NVFP4 V is pair-interleaved: the 128 bytes of tokens 2p and 2p+1 hold,
 *     at byte d, dim d of token 2p in the low nibble and dim d of token 2p+1
 *     in the high nibble;
 *   INT4 V rows are dim-permuted: byte 8r + m (r, m = 0..7) of a token's 64
 *     bytes holds dim 16m + r in the low nibble and dim 16m + r + 8 in the
 *     high nibble;
 *   INT8 V rows are dim-permuted: byte 16r + 2m + h (r, m = 0..7, h = 0, 1)
 *     of a token's 128 bytes holds dim 16m + r + 8h;
 *   INT2 V rows are dim-permuted: byte 4r + m/2 (r, m = 0..7) of a token's
 *     32 bytes holds dim 16m + r + 8h (h = 0, 1) at bits 2(2(m%2) + h).
 */
struct kvq_layout {
    void* codes;           /* see above                                       */
    void* meta;            /* NVFP4: u8 E4M3 [batch][kv_heads][capacity][head_dim/16]
                              INT4, INT8, INT2: {f32 S, i32 Z} [batch][kv_heads][capacity][head_dim/group]
                              INT4, INT2 with compact_meta: {f16 S0, f16 S1, i8 Z0, i8 Z1, 0, 0}
                                [batch][kv_heads][capacity]; INT8 with compact_meta:
                                {f16 S0, f16 S1, i16 Z0, i16 Z1}
                              FP8:   NULL                                       */
    void* ring;            /* residual_length > 0: bf16
                              [batch][kv_heads][residual_length][head_dim]; else NULL */
    float* global_scale;   /* device f32 per-tensor scale (NVFP4, FP8); else NULL */
    int64_t capacity;      /* token stride of codes/meta planes (>= max_len) */
    int32_t code_bytes;    /* code bytes per token per head */
    int32_t meta_bytes;    /* meta bytes per token per head */
    int32_t compact_meta;  /* 1: INT4 compact group metadata (see kvq_options) */
    int32_t scale_renewal; /* segment length of scale renewal, 0 if none; then
                              global_scale points at scale_segments f32 per-
                              segment scales (segment s: tokens [s*len, (s+1)*len)) */
    int32_t scale_segments;
    int32_t page_tokens;   /* paged cache: tokens per page, else 0.  Then codes /
                              meta are pools [num_pages][kv_heads][page_tokens][bytes]
                              and `capacity` equals page_tokens */
    int32_t num_pages;
    int32_t max_pages;     /* block-table entries per sequence */
    int32_t reserved;
    const int32_t* pages;  /* device block table [batch][max_pages] (-1: none), or NULL */
};

/*
 * Options of kvq_cache_bytes_ex / kvq_cache_create_ex (zero-initialise;
 * NULL means all defaults).
 *   scale_renewal  NVFP4/FP8 caches without a ring: renew the per-tensor
 *                  scales every `scale_renewal` tokens, a multiple of 16
 *                  (0 = never, the default).  Source: NVFP4 KV-cache
 *                  article, section 3.1 (the scale factors are updated
 *                  every 512 processed tokens).  Token positions fall into
 *                  segments [sP, (s+1)P).  Segment 0 uses the calibrated
 *                  (or given) scale; segment s >= 1 uses the scale of the
 *                  amax of segment s-1's tokens (all batch rows and heads of
 *                  the layer).  Tokens are never re-encoded.  kvq_truncate
 *                  keeps the amax of dropped tokens of a partial segment.
 */
struct kvq_options {
    int32_t scale_renewal;
    int32_t compact_meta;   /* INT4, INT8 or INT2 with group_size 64: store each
                               group's S as binary16 and Z as a small integer,
                               8 meta bytes per token instead of 16: {f16 S0,
                               f16 S1, i8 Z0, i8 Z1, 2 zero bytes} for INT4 and
                               INT2, {f16 S0, f16 S1, i16 Z0, i16 Z1} for INT8
                               (whose zero points, 0..255 for groups that span
                               zero, do not fit int8).  S is the binary32 S
                               rounded to binary16 (nearest even; saturated at
                               65504; 2^-24 if it would round to 0); Z and the
                               codes are computed with that S; Z is clamped to
                               its integer type's range. */
    int32_t page_tokens;    /* paged blocks (0 = one contiguous region per
                               sequence): the main-cache planes of every layer
                               become a pool of `num_pages` pages, each holding
                               page_tokens consecutive tokens of one sequence
                               for all its KV heads.  A sequence takes pages
                               from the pool as its main cache grows (the
                               first layer to need a page takes it for every
                               layer) and gives them back at kvq_seq_reset or
                               kvq_cache_reset; a per-sequence block table maps
                               its token t to page table[t / page_tokens].
                               page_tokens must be a positive multiple of
                               kvq_page_granularity(format).  Not with
                               scale_renewal.  Source: the globally addressed
                               KV cache of the NVFP4 article's section 5.2. */
    int32_t num_pages;      /* pages in the pool (paged caches) */
    int32_t reserved[4];
};

/*
 * Bytes of device memory a cache needs (all layers, K and V, the residual
 * ring, per-tensor scales and a status word).  0 if the arguments are
 * invalid.  Size model: see the KV size formula on the Model Optimizer page
 * (2 x layers x kv_heads x head_dim x len x bytes per element) plus scale
 * and padding bytes.
 *   format           KVQ_NVFP4 | KVQ_INT4 | KVQ_FP8 | KVQ_INT8 | KVQ_INT2
 *   head_dim         128
 *   group_size       NVFP4: 16 (or 0 = 16); INT4, INT2: 64 or 32; INT8: 64;
 *                    FP8: 0
 *   residual_length  NVFP4, FP8, INT4, INT8: 0..4096 tokens (0 = no ring);
 *                    INT2: 0..16384
 */
size_t kvq_cache_bytes(int format, int layers, int batch, int kv_heads, int head_dim,
                       int64_t max_len, int group_size, int residual_length);
/* kvq_cache_bytes with options (NULL: the same as kvq_cache_bytes). */
size_t kvq_cache_bytes_ex(int format, int layers, int batch, int kv_heads, int head_dim,
                          int64_t max_len, int group_size, int residual_length,
                          const struct kvq_options* options);

/*
 * Bind a cache to caller-owned device memory `device_buf` (at least
 * kvq_cache_bytes(...) bytes, 256-byte aligned).  The buffer is zeroed
 * (synchronously) and all lengths start at 0.
 *   global_scales  host float[layers][2] (K, V): per-tensor scales to use for
 *                  NVFP4/FP8 (1.0 gives the *_cast variants).  NULL: each
 *                  layer's K and V scale is calibrated on the device from the
 *                  amax of that layer's first append (NVFP4: amax/(6*448),
 *                  FP8: amax/448, 1.0 for an all-zero tensor).  Ignored for
 *                  INT4, INT8 and INT2.
 * The handle is host memory owned by the library; free it with
 * kvq_cache_destroy.  Errors: INVALID_ARG, WORKSPACE (buffer too small),
 * UNSUPPORTED (head_dim != 128), CUDA.
 */
int kvq_cache_create(kvq_cache_t* out, int format, int layers, int batch, int kv_heads,
                     int head_dim, int64_t max_len, int group_size, int residual_length,
                     void* device_buf, size_t buf_bytes, const float* global_scales);
/* kvq_cache_create with options (NULL: the same as kvq_cache_create); the
 * buffer must hold kvq_cache_bytes_ex(..., options) bytes.  Options the
 * format cannot take give INVALID_ARG. */
int kvq_cache_create_ex(kvq_cache_t* out, int format, int layers, int batch, int kv_heads,
                        int head_dim, int64_t max_len, int group_size, int residual_length,
                        void* device_buf, size_t buf_bytes, const float* global_scales,
                        const struct kvq_options* options);

/* Free the host handle.  The device buffer stays the caller's. */
int kvq_cache_destroy(kvq_cache_t cache);

/*
 * Empty every layer (lengths to 0) and forget calibrated scales (scales given
 * at creation are kept).  Enqueued on `stream`.
 */
int kvq_cache_reset(kvq_cache_t cache, void* stream);

/*
 * Quantize n new tokens of K and V into `layer` and append them.
 *   k, v   device bf16 [batch][kv_heads][n][head_dim], contiguous, 16-byte
 *          aligned.
 * Without a ring, tokens go straight to the main cache.  With a ring (any
 * format), tokens enter the ring; each time it fills it is quantized into
 * the main cache and emptied, exactly as if the tokens had been appended one
 * at a time.  NVFP4/FP8: the first append of an uncalibrated layer first
 * reduces amax over this call's K and V and sets the per-tensor scales,
 * whether its tokens go to the main cache or to the ring (a ring on NVFP4 /
 * FP8 is the combination compared in the NVFP4 article's section 3.2
 * setting; its tokens are encoded at the flush with the layer's scale).
 * Attention reads NVFP4 / FP8 ring values as FP16 multiples of the V
 * scale, so a ring value above 24 (NVFP4) or 146 (FP8) times the
 * calibration amax overflows; in the main cache it would saturate.
 * Errors: INVALID_ARG, CAPACITY (nothing is written), CUDA.
 */
int kvq_append(kvq_cache_t cache, int layer, const void* k, const void* v, int64_t n,
               void* stream);

/* Quantize whatever the ring holds (possibly fewer than
 * residual_length tokens) into the main cache and empty the ring.  A no-op
 * for an empty ring or a format without one. */
int kvq_flush_residual(kvq_cache_t cache, int layer, void* stream);

/* Workspace bytes kvq_decode_attention needs for `q_heads` query heads (0
 * for invalid arguments).  Enough for any sequence lengths the cache can
 * hold, ragged batches included. */
size_t kvq_workspace_bytes(kvq_cache_t cache, int q_heads);

/*
 * Decode attention for one new query token per sequence:
 *   out[b][h][:] = softmax_j(scale * q[b][h] . k_j) . v_j over the layer's
 *   main cache (dequantized) followed by the ring tokens, with query head h
 *   reading KV head h / (q_heads / kv_heads).
 *   q          device bf16 [batch][q_heads][head_dim], 16-byte aligned
 *   q_heads    a multiple of kv_heads with q_heads/kv_heads in 1..8
 *   softmax_scale  <= 0 selects 1/sqrt(head_dim)
 *   out        device f32 [batch][q_heads][head_dim]
 *   workspace  device scratch of kvq_workspace_bytes(cache, q_heads) bytes,
 *              256-byte aligned, not used by another call at the same time
 * Scores accumulate in FP32 on tensor cores with FP16 operands, and the
 * softmax is FP32.  The probabilities enter the P.V product as FP16 values
 * (2^-11 relative rounding each) and the denominators are summed from the
 * same FP16 values, so the output is an exactly normalised weighted mean of
 * the dequantized values: each weight is off by at most 2^-11 relative, so
 * the output's error is at most 2^-10 * max_j |v_j - out| (plus FP32
 * accumulation), however large the values are (with scale renewal too: the
 * output accumulator is rescaled in FP32 when the segment changes).  The
 * INT formats multiply each FP16 probability by its group's S in FP16, one
 * more rounding per weight, which adds up to 2^-11 * max_j |v_j|.  With
 * values within +-10 of the output this is inside a max-abs of 1e-2.
 * Q' = q * softmax_scale * log2(e) enters the score product in FP16: with
 * q_heads / kv_heads <= 4 as two parts, FP16(q') and FP16 of the rest, in
 * otherwise unused MMA columns, which carries q' to about 2^-22 of itself;
 * with 5..8 query heads per KV head as one FP16 value (2^-11 relative
 * rounding per element), which moves a base-2 logit by at most
 * 2^-11 * sum_d |q'_d k_d|.  |q| * softmax_scale must stay below 45,000
 * (with 1/sqrt(128): |q| below 500,000).
 *   NVFP4 and FP8 values are exact in FP16.
 *   INT4/INT8/INT2 codes enter as the exact FP16 values 1024 + q.  S and Z
 *     are applied to the FP32 scores on the K side; on the V side S scales
 *     the FP16 probabilities and the zero-point term sum (1024 + Z) S P is
 *     subtracted in FP32.  1024 + Z is an FP16 operand: exact for
 *     -3072 <= Z <= 1024 (Z < 0 when all of a group's values are positive,
 *     Z above the top code when all are negative), rounded to FP16 beyond.
 *     BF16 inputs bound it: a non-constant group spans at least one BF16
 *     spacing, more than 2^-8 of its largest magnitude, so
 *     |Z| < 256 (2^bits - 1).  That is exact for INT2 and within 2^-11
 *     relative for INT4.  For INT8 the same holds up to Z = 64480; only a
 *     group whose values are two adjacent BF16 numbers near the top of a
 *     binade reaches beyond, where the FP16 operand overflows.
 *   The FP16 probabilities stay below 256 (the softmax reference moves
 *     only when a logit passes it by 8 in base 2), so the scaled operand
 *     S * p of the INT formats holds groups whose value range is below
 *     about 3,800 (INT4), 65,000 (INT8) or 760 (INT2); a V group with a wider
 *     range can overflow it.
 * Errors: INVALID_ARG, EMPTY, WORKSPACE, CUDA.
 */
int kvq_decode_attention(kvq_cache_t cache, int layer, const void* q, int q_heads,
                         float softmax_scale, float* out, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * One decode step in one launch: append one new token of K and V (as
 * kvq_append with n = 1) and run decode attention over the cache that
 * includes it (as kvq_decode_attention).  In the attention kernel, the warp
 * that streams the part of a sequence's last cache tile holding the new
 * token quantizes and stores the token before it requests that part (or
 * stores it into the ring slot whose slab it reads), so the step costs one
 * kernel instead of two.
 *   k, v   device bf16 [batch][kv_heads][1][head_dim], 16-byte aligned
 *   other arguments as kvq_decode_attention
 * When the step is the layer's first (calibrating) append, when the token
 * fills the ring (which must be flushed), or, under scale renewal, when the
 * token starts a new segment (whose scale is renewed first), it runs as
 * kvq_append followed by kvq_decode_attention.  Same results as those two
 * calls.  Errors: those
 * of both calls; on an error the layer's lengths are unchanged.
 */
int kvq_decode_step(kvq_cache_t cache, int layer, const void* k, const void* v, const void* q,
                    int q_heads, float softmax_scale, float* out, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * Dequantize main-cache tokens [start, start+n) of K (kv=0) or V (kv=1) into
 * device f32 out[batch][kv_heads][n][head_dim].  NVFP4: e2m1*e4m3*g;
 * INT4, INT8, INT2: (q-Z)*S; FP8: e4m3*s, in FP32.  Errors: INVALID_ARG, CUDA.
 */
int kvq_dequantize(kvq_cache_t cache, int layer, int kv, int64_t start, int64_t n, float* out,
                   void* stream);

/*
 * Drop tokens so that `layer` holds `total_len` tokens (main + ring), e.g. to
 * roll back speculative tokens.  If total_len >= the main-cache length only
 * ring tokens are dropped; otherwise the main cache is cut to total_len and
 * the ring emptied.  Host bookkeeping only; nothing is launched and the
 * per-tensor scales are kept.  Errors: INVALID_ARG (total_len above the
 * current length or negative).
 */
int kvq_truncate(kvq_cache_t cache, int layer, int64_t total_len);

/* Host-side token counts of a layer. */
int kvq_get_lengths(kvq_cache_t cache, int layer, int64_t* len_main, int64_t* len_ring);

/* Device layout of (layer, kv). */
int kvq_get_layout(kvq_cache_t cache, int layer, int kv, struct kvq_layout* out);

/*
 * Synchronize `stream` and read the device status word: 0 if no kernel has
 * given up a bounded wait, else a nonzero code (and the call returns
 * KVQ_ERR_DEVICE_TIMEOUT): 1 a tile's copy did not land within 2 s, 3 copies
 * were still pending when the kernel exited.  The word is cleared after
 * reading.
 */
int kvq_device_status(kvq_cache_t cache, void* stream, int* device_error);

/*
 * kvq_decode_attention without a workspace argument, for callers that cannot
 * allocate device memory: host frameworks whose callbacks must not allocate
 * (an inference-engine plugin's enqueue, for example), or decode loops that
 * must never call cudaMalloc because it can block and synchronise the
 * device.  The pages have no counterpart to this call; it exists for such
 * callers only.  Same arguments, layout and errors as kvq_decode_attention.
 *
 * The partial records go to a static 4 MiB device array inside libkvq.so,
 * which every GPU that loads the library keeps until the process exits.  A
 * cache/q_heads combination whose kvq_workspace_bytes() exceeds 4 MiB is
 * refused with KVQ_ERR_WORKSPACE (use kvq_decode_attention then).  The
 * first call on each device resolves the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls share the one array: calls whose
 * kernels overlap on the GPU (other streams, other caches) race and must be
 * ordered by the caller.  Nothing in the array has to start at zero; each
 * call writes every record before reading it.
 */
int kvq_decode_attention_noalloc(kvq_cache_t cache, int layer, const void* q, int q_heads,
                                 float softmax_scale, float* out, void* stream);

/*
 * kvq_decode_attention that also writes, per query head, the log-sum-exp of
 * its scores over this cache:
 *   lse[b][h] = log sum_j exp(scale * q[b][h] . k_j)   (natural log, f32)
 * so that attention over a sequence split into parts held by several caches
 * (several GPUs: context parallelism) can be merged with
 * kvq_combine_partials.  A layer with no tokens is not an error here: out
 * is set to 0 and lse to -inf, a part without weight in the merge.
 *   lse    device f32 [batch][q_heads], 4-byte aligned
 *   other arguments as kvq_decode_attention
 * The log-sum-exp merge is the combine step of split-K decode attention
 * (flash decoding), taken across devices.  Errors: those of
 * kvq_decode_attention except EMPTY.
 */
int kvq_decode_attention_lse(kvq_cache_t cache, int layer, const void* q, int q_heads,
                             float softmax_scale, float* out, float* lse, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * Merge attention results over n_parts disjoint parts of the same key
 * sequences.  Part r of row i (a row is one query head of one sequence) has
 * its output at o_parts + r*o_stride + i*head_dim and its log-sum-exp at
 * lse_parts + r*lse_stride + i, as written by kvq_decode_attention_lse:
 *   out[i]     = sum_r exp(lse_r - L) o_r,  L = log sum_r exp(lse_r)
 *   lse_out[i] = L (optional: NULL skips it)
 * Parts with lse = -inf carry no weight; a row no part covers gets out 0
 * and lse -inf.  All pointers are device f32, 4-byte aligned; out may not
 * alias the inputs.  head_dim must be 128.  Errors: INVALID_ARG,
 * UNSUPPORTED, CUDA.
 */
int kvq_combine_partials(int n_parts, int64_t rows, int head_dim, const float* o_parts,
                         int64_t o_stride, const float* lse_parts, int64_t lse_stride, float* out,
                         float* lse_out, void* stream);

/*
 * Sequences of different lengths (a ragged batch).  Every call above works
 * on a batch whose sequences hold different numbers of tokens: kvq_append
 * and kvq_decode_step add their tokens to each sequence at that sequence's
 * own end (its ring, if any, filling and flushing on its own),
 * kvq_flush_residual flushes every sequence's ring, and the attention calls
 * attend each sequence over its own tokens; a sequence holding no token
 * gets output 0 (and log-sum-exp -inf), and KVQ_ERR_EMPTY is returned only
 * when no sequence holds a token.  kvq_get_lengths reports sequence 0,
 * kvq_truncate cuts every sequence longer than total_len to total_len, and
 * kvq_dequantize's token range must lie inside every sequence's main cache.
 * Limits of a ragged or paged batch: at most 256 sequences; no scale
 * renewal.  NVFP4 / FP8 calibrate their per-tensor scales from the first
 * append to the layer, whichever sequences it feeds, over the tokens it
 * appends.
 */

/* Append n tokens to sequence `seq` only.  k, v: device bf16
 * [kv_heads][n][head_dim], contiguous, 16-byte aligned.  Same rules as
 * kvq_append for that one sequence.  Errors: INVALID_ARG, CAPACITY (the
 * sequence's max_len, or no free page), UNSUPPORTED (scale renewal), CUDA. */
int kvq_append_seq(kvq_cache_t cache, int layer, int seq, const void* k, const void* v, int64_t n,
                   void* stream);

/* Empty sequence `seq` in every layer (for the next request in its batch
 * slot); a paged cache returns its pages to the pool.  Calibrated scales
 * are kept.  Host bookkeeping, plus block-table updates enqueued on
 * `stream` for a paged cache. */
int kvq_seq_reset(kvq_cache_t cache, int seq, void* stream);

/* Token counts of one sequence. */
int kvq_get_seq_lengths(kvq_cache_t cache, int layer, int seq, int64_t* len_main,
                        int64_t* len_ring);

/* kvq_truncate for one sequence. */
int kvq_truncate_seq(kvq_cache_t cache, int layer, int seq, int64_t total_len);

/* kvq_dequantize for one sequence: main-cache tokens [start, start+n) of
 * sequence `seq` into device f32 out[kv_heads][n][head_dim]. */
int kvq_dequantize_seq(kvq_cache_t cache, int layer, int kv, int seq, int64_t start, int64_t n,
                       float* out, void* stream);

/* Page ids of sequence `seq` (host copy of its block-table row; -1 for
 * entries without a page) into pages[0 .. n).  Paged caches only. */
int kvq_get_block_table(kvq_cache_t cache, int seq, int32_t* pages, int64_t n);

/* page_tokens of a paged cache must be a multiple of this (the decode
 * kernel's tile for the format); 0 for an unknown format. */
int kvq_page_granularity(int format);

/* Message for the last failed call on this thread ("" if none). */
const char* kvq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
