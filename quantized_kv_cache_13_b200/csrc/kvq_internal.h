// kvq_internal.h -- host-side cache structure and kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kHeadDim = 128;
constexpr int kCapacityAlign = 768;      // token padding of every plane: a multiple of every attention tile (384, 256, 128)
constexpr int kMaxG = 8;                 // query heads per KV head handled per CTA

// Device pointers of one (layer, K|V) pair.
struct Plane {
  uint8_t* codes = nullptr;     // [B][H][cap][code_bytes]
  uint8_t* meta = nullptr;      // [B][H][cap][meta_bytes]
  uint16_t* ring = nullptr;     // bf16 [B][H][R][D]
};

struct LayerState {
  Plane kv[2];
  float* gscale[2] = {nullptr, nullptr};   // device per-tensor scale (K, V)
  uint32_t* amax[2] = {nullptr, nullptr};  // device amax accumulators (f32 bits)
  // Token counts.  While every sequence of the batch holds the same number
  // of tokens (`ragged` false) len_main / len_ring are those counts; once a
  // per-sequence call makes them differ, seq_main / seq_ring ([batch]) hold
  // each sequence's counts and len_main / len_ring are sequence 0's.
  int64_t len_main = 0;
  int64_t len_ring = 0;
  // Lowest main-cache position written by the layer's most recent call that
  // wrote main-cache tokens (an append, a flush, a fused decode step).  A
  // decode kernel may read tokens below it before waiting for the previous
  // kernel of its stream: every kernel that wrote them has completed.
  int64_t write_lo = 0;
  bool ragged = false;
  int64_t* seq_main = nullptr;
  int64_t* seq_ring = nullptr;
  bool calibrated[2] = {false, false};
  // scale renewal: per-segment scales and amax accumulators (f32 bits) of K, V
  float* seg_scale[2] = {nullptr, nullptr};
  uint32_t* seg_amax[2] = {nullptr, nullptr};
};

}  // namespace kvq

struct kvq_cache {
  int format = 0;
  int layers = 0, batch = 0, kv_heads = 0, head_dim = 0;
  int64_t max_len = 0;
  int64_t capacity = 0;
  int group = 0;            // NVFP4 16, INT4 32/64, INT8 64
  int R = 0;                // ring length (0: no ring)
  int code_bytes = 0, meta_bytes = 0;
  bool scales_given = false;
  int renewal = 0;          // scale renewal period in tokens (0: never)
  int compact = 0;          // INT4 g64: compact group metadata (f16 S, i8 Z)
  int64_t nseg = 0;         // scale segments per (layer, K|V)
  int* dev_status = nullptr;
  int* counters = nullptr;   // device [layers][batch * kv_heads]
  int device = 0;
  int sm_count = 0;
  int ctas_env = 0;         // KVQ_CTAS override of the attention grid (0 = automatic)
  int pdl = 1;              // launch attention kernels with programmatic dependent launch (KVQ_PDL=0: off)
  int split_wb = 3;         // unit-start weight of the attention work split (set per format at create; KVQ_UNIT_WEIGHT)
  kvq::LayerState* L = nullptr;
  // Paged blocks (page_tokens > 0): the main-cache planes of every layer are
  // pools of num_pages pages of page_tokens tokens x kv_heads; sequence b's
  // token t lives in page pages[b * max_pages + t / page_tokens].  The block
  // table is shared by all layers; host copy `host_pages` (-1: unassigned),
  // device copy `dev_pages` in the cache header.
  int page_tokens = 0;
  int64_t num_pages = 0;
  int64_t max_pages = 0;    // table entries per sequence: ceil(max_len / page_tokens)
  int32_t* host_pages = nullptr;
  int32_t* dev_pages = nullptr;
  int32_t* free_pages = nullptr;   // stack of unassigned page ids
  int64_t n_free = 0;
  int64_t* seq_pages = nullptr;    // [batch] pages assigned to each sequence
};

namespace kvq {

// Launchers (kvq_quant.cu / kvq_attn.cu).  All enqueue on `stream`.
cudaError_t launch_amax(const uint16_t* k, const uint16_t* v, int64_t elems, uint32_t* amax_k,
                        uint32_t* amax_v, cudaStream_t stream);

// Quantize n tokens per (b,h) from src (bf16; token t of (b,h) at
// src + bh*src_bh_stride + (src_tok0+t)*D) into main-cache tokens
// [dst_tok0, dst_tok0+n).  kv_count = 1 or 2 (K then V).
struct QuantArgs {
  const uint16_t* src[2];
  int64_t src_bh_stride;    // elements
  int64_t src_tok0;
  Plane dst[2];
  int64_t dst_tok0;
  int64_t n;
  int bh;                   // batch * kv_heads
  int64_t cap;
  int group;
  const float* gscale[2];   // NVFP4/FP8 per-tensor scale (read), or
  const uint32_t* amax[2];  // amax words when calibrating (then gscale is written)
  float* gscale_out[2];
  int calibrate;            // 1: derive the scale from amax and store it
  const float* gseg[2];     // scale renewal: per-segment scales of K, V (else null)
  int renewal;              // segment length in tokens (0: the per-tensor scale)
  int compact;              // INT4 g64: f16 S + i8 Z group metadata
  // Plane rows: unit bh of this launch is cache unit unit0 + bh (unit =
  // batch index * kv_heads + kv head); its token t is row
  // unit * cap + t, or, with pages, the page-table row (see plane_row).
  int64_t unit0;
  int kv_heads;
  const int32_t* pages;     // block table [batch][max_pages] or null
  int page_tokens;
  int max_pages;
};

// Row of token t of cache unit u in a main-cache plane: contiguous planes
// hold each unit's tokens at u * cap + t; paged planes hold token t of
// sequence b = u / kv_heads in page pages[b * max_pages + t / page_tokens],
// whose rows are [kv_heads][page_tokens].
__host__ __device__ inline int64_t plane_row(int64_t u, int64_t t, int64_t cap, int kv_heads,
                                             const int32_t* pages, int page_tokens, int max_pages) {
  if (!pages) return u * cap + t;
  const int64_t b = u / kv_heads, h = u - b * kv_heads;
  const int64_t page = pages[b * max_pages + t / page_tokens];
  return (page * kv_heads + h) * page_tokens + t % page_tokens;
}

// Scale renewal (NVFP4 / FP8): atomic max of |x| of n appended tokens per
// (b,h) into the segment words seg_amax[kv][(dst_tok0 + t) / renewal], and
// the scales of segments s_first .. s_last from the amax of the segment
// before each: g[s] = amax[s-1] / divisor (1 for a zero segment).
cudaError_t launch_seg_amax(const uint16_t* k, const uint16_t* v, int64_t src_bh_stride, int64_t n,
                            int bh, int64_t dst_tok0, int renewal, uint32_t* seg_amax_k,
                            uint32_t* seg_amax_v, cudaStream_t stream);
cudaError_t launch_renew_scales(const uint32_t* seg_amax_k, const uint32_t* seg_amax_v,
                                float* seg_scale_k, float* seg_scale_v, int64_t s_first,
                                int64_t s_last, float divisor, cudaStream_t stream);
cudaError_t launch_quantize(int format, const QuantArgs& a, cudaStream_t stream);

// Per-tensor scales from the amax words: g = amax / divisor (1 for a zero
// tensor), for K and V (NVFP4 / FP8 caches with a ring calibrate this way,
// since their first append may quantize nothing).
cudaError_t launch_scale_from_amax(const uint32_t* amax_k, const uint32_t* amax_v, float* gscale_k,
                                   float* gscale_v, float divisor, cudaStream_t stream);

// Copy n bf16 tokens per (b,h) into ring slots [ring_tok0, ring_tok0+n).
cudaError_t launch_ring_copy(const uint16_t* src_k, const uint16_t* src_v, int64_t src_bh_stride,
                             int64_t src_tok0, uint16_t* ring_k, uint16_t* ring_v, int R,
                             int64_t ring_tok0, int64_t n, int bh, cudaStream_t stream);

// v_pairs: the plane is a V plane in its decode layout (NVFP4: pair-interleaved
// codes; INT4, INT8: permuted dims), which the dequantize undoes.
// gseg / renewal: per-segment scales of a renewing NVFP4 / FP8 cache (else
// null / 0, and gscale is the per-tensor scale).
struct RowMap {             // see plane_row
  int64_t unit0;
  int kv_heads;
  const int32_t* pages;
  int page_tokens;
  int max_pages;
};
cudaError_t launch_dequantize(int format, const Plane& p, const float* gscale, int64_t cap,
                              int group, int bh, int64_t start, int64_t n, float* out, bool v_pairs,
                              cudaStream_t stream, const float* gseg, int renewal, bool compact,
                              const RowMap& map);

// Set block-table entries: table[idx[i]] = val[i] for i < n (n <= kTableBatch).
constexpr int kTableBatch = 64;
struct TableUpdate {
  int n;
  int32_t idx[kTableBatch];
  int32_t val[kTableBatch];
};
cudaError_t launch_table_update(int32_t* table, const TableUpdate& u, cudaStream_t stream);

// Kernel-internal format id of INT4 g64 with compact group metadata: per
// token {f16 S0, f16 S1, i8 Z0, i8 Z1, 2 zero bytes}.
constexpr int kFmtInt4Compact = 16;
// INT8 g64 with compact metadata {f16 S0, f16 S1, i16 Z0, i16 Z1}, and INT2
// g64 with {f16 S0, f16 S1, i8 Z0, i8 Z1, 2 zero bytes}, per token.
constexpr int kFmtInt8Compact = 17;
constexpr int kFmtInt2Compact = 18;

struct AttnArgs {
  int format;
  Plane k, v;
  const float* gscale_k;     // device, NVFP4/FP8 (nullptr for the INT formats)
  const float* gscale_v;
  int64_t cap;
  int R;
  int64_t len_main;
  int64_t len_ring;
  int batch, kv_heads, G;
  int group;
  const uint16_t* q;          // bf16 [B][Hq][D]
  float softmax_scale;
  float* out;                 // f32 [B][Hq][D]
  float* lse;                 // f32 [B][Hq] log-sum-exp of the scores, or nullptr
  float* partials;            // workspace: [units][maxc][G][D + 2]
  int* counters;              // per unit, zero between calls (cache header)
  int ctas;                   // grid size
  int tpu;                    // main-cache tiles per unit (0: ring only)
  int maxc;                   // record slots per unit
  int wb;                     // unit-start weight of the work split, in tiles
  // Fused append of this step's token (kvq_decode_step): 0 none; 1 written
  // to main-cache position new_pos; 2 copied to ring slot new_pos.  The
  // lengths above already include it.
  int new_kind;
  int64_t new_pos;
  const uint16_t* k_new;      // bf16 [B][Hkv][1][D]
  const uint16_t* v_new;
  int* dev_status;
  // scale renewal (NVFP4 / FP8): per-segment scales and amax words of K, V
  const float* gseg_k;
  const float* gseg_v;
  uint32_t* seg_amax_k;
  uint32_t* seg_amax_v;
  int renewal;                // segment length in tokens (0: per-tensor scales)
  int compact;                // INT4 g64 with f16 S + i8 Z group metadata
  // Programmatic dependent launch: pdl = 1 launches the kernel so that it
  // may start while the previous kernel of the stream finishes; main-cache
  // tokens [0, pre_len) are written by no kernel that can still be running
  // then, so a warp may request its first tile before the grid-dependency
  // wait when the tile lies wholly below pre_len.
  int pdl;
  int64_t pre_len;
};

// Sequences of different lengths, and paged planes: the second argument of
// the ragged attention kernel (kernel parameter space; up to kMaxSeqs
// sequences and kMaxCtas CTAs).  Every (batch, KV head) unit of sequence b
// owns s_b = max(1, ceil(seq_main[b] / TILE)) consecutive "slots" of the
// flattened slot line (a slot is one main-cache tile; a unit without
// main-cache tokens still owns one slot, in which only its ring is read);
// CTA i owns slots [cta_slot[i], cta_slot[i+1]).
constexpr int kMaxSeqs = 256;
constexpr int kMaxCtas = 512;
struct RaggedArgs {
  int32_t seq_main[kMaxSeqs];      // main-cache tokens of each sequence
  int32_t seq_ring[kMaxSeqs];      // ring tokens of each sequence
  int32_t seq_slot0[kMaxSeqs + 1]; // first slot of sequence b's unit (b, 0); [batch] = total
  int32_t cta_slot[kMaxCtas + 1];
  const int32_t* pages;            // block table [batch][max_pages], or null
  int32_t page_tokens;
  int32_t max_pages;
};
cudaError_t launch_decode_attention_ragged(const AttnArgs& a, const RaggedArgs& r,
                                           cudaStream_t stream);

// Log-sum-exp merge of per-part attention results (kvq_cp.cu): part r of
// row i has o at o_parts + r*o_stride + i*D and lse at lse_parts +
// r*lse_stride + i.  lse_out may be null.
cudaError_t launch_combine(int n, int64_t rows, const float* o_parts, int64_t o_stride,
                           const float* lse_parts, int64_t lse_stride, float* out, float* lse_out,
                           cudaStream_t stream);
// o = 0 and lse = -inf for `rows` rows (attention over no keys).
cudaError_t launch_empty_part(int64_t rows, float* out, float* lse, cudaStream_t stream);

// Tile ownership of the decode-attention grid (shared by host and kernel).
// Every (batch, KV head) unit has tpu tiles; unit u occupies positions
// [u*(tpu+wb), (u+1)*(tpu+wb)) of a weighted line whose first wb positions
// stand for the fixed cost of starting a unit (query load, end-of-unit
// merge) and whose tile k sits at u*(tpu+wb) + wb + k.  CTA i of C owns the
// tiles at positions [i*W/C, (i+1)*W/C), W = units*(tpu+wb): contiguous in
// flattened (unit-major) tile order, each tile owned once, and a CTA whose
// range starts a unit gets that many fewer tiles.
__host__ __device__ inline int64_t split_first_tile_at(int64_t p, int64_t units, int64_t tpu,
                                                       int64_t wb) {
  const int64_t span = tpu + wb;
  const int64_t u = p / span;
  if (u >= units) return units * tpu;
  const int64_t o = p - u * span;
  return u * tpu + (o <= wb ? 0 : o - wb);
}
__host__ __device__ inline int64_t split_cta_of_tile(int64_t t, int64_t tpu, int64_t wb, int64_t W,
                                                     int64_t C) {
  const int64_t pos = t + (t / tpu + 1) * wb;
  return ((pos + 1) * C + W - 1) / W - 1;
}

// Tokens per shared-memory stage of the attention kernel for `format`.
int attn_tile_tokens(int format, int group);
// Page sizes of a paged cache must be multiples of this (every kernel
// variant's tile of the format divides it).
int attn_page_granularity(int format);
// Blocks per SM the attention kernel of `format` reaches (occupancy query);
// `ring` / `renew`: the NVFP4 / FP8 instantiations for caches with a
// residual ring / with scale renewal.
int attn_blocks_per_sm(int format, bool ring, bool renew, bool compact);
cudaError_t launch_decode_attention(const AttnArgs& a, cudaStream_t stream);

// Record `msg` as this thread's kvq_last_error() message; returns `code`.
int report_error(int code, const char* msg);

}  // namespace kvq
