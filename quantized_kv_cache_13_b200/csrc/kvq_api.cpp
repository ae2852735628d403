// kvq_api.cpp -- host side of the kvq C ABI: argument checks, the device
// buffer layout, token bookkeeping (main cache + residual ring) and kernel
// launch routing.  No device memory is allocated here; every byte lives in
// caller-owned buffers.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "kvq.h"
#include "kvq_internal.h"

using namespace kvq;

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int ok() {
  g_err[0] = '\0';
  return KVQ_OK;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

struct Geometry {
  int code_bytes = 0, meta_bytes = 0, group = 0;
  int renewal = 0;         // scale renewal period (0: per-tensor scales only)
  int compact = 0;         // INT4 g64 with f16 S + i8 Z group metadata
  int64_t nseg = 0;        // scale segments per (layer, K|V) when renewing
  size_t seg_off = 0;      // byte offset of the segment scales, then the segment amaxes
  int64_t cap = 0;
  size_t header = 0;       // scales, amax words, status word, attention counters
  size_t counters_off = 0; // byte offset of the per-(layer, unit) counters
  size_t codes = 0, meta = 0, ring = 0;   // bytes per (layer, kv) plane
  size_t per_layer = 0;
  size_t total = 0;
  int page_tokens = 0;     // paged planes: tokens per page (0: contiguous)
  int64_t num_pages = 0;
  int64_t max_pages = 0;   // block-table entries per sequence
  size_t table_off = 0;    // byte offset of the block table in the header
};

// Check the arguments and compute the layout:
//   [header: per layer {gscale K, gscale V, amax K, amax V} x f32/u32, status
//    word, per (layer, batch x kv_head) attention completion counters]
//   then per layer, per K/V: codes plane, meta plane, ring plane,
// every plane 256-byte aligned.
inline bool int_affine_format(int format) {
  return format == KVQ_INT4 || format == KVQ_INT8 || format == KVQ_INT2;
}

int geometry(int format, int layers, int batch, int kv_heads, int head_dim, int64_t max_len,
             int group_size, int residual_length, const kvq_options* opt, Geometry* g) {
  if (format != KVQ_NVFP4 && format != KVQ_INT4 && format != KVQ_FP8 && format != KVQ_INT8 &&
      format != KVQ_INT2)
    return fail(KVQ_ERR_INVALID_ARG, "unknown format %d", format);
  if (layers <= 0 || batch <= 0 || kv_heads <= 0 || max_len <= 0)
    return fail(KVQ_ERR_INVALID_ARG, "layers, batch, kv_heads and max_len must be positive");
  if (head_dim != kHeadDim)
    return fail(KVQ_ERR_UNSUPPORTED, "head_dim %d: only %d is implemented", head_dim, kHeadDim);
  if (max_len > (int64_t(1) << 31))
    return fail(KVQ_ERR_INVALID_ARG, "max_len %lld too large", (long long)max_len);
  // the kernels index (batch, kv head) units and layers with 32-bit ints
  if ((int64_t)batch * kv_heads > (int64_t(1) << 24) || layers > (1 << 16))
    return fail(KVQ_ERR_INVALID_ARG, "batch x kv_heads %lld or layers %d too large",
                (long long)batch * kv_heads, layers);
  // INT2's ring may hold a whole recent chunk of 8K-16K tokens (age tiers)
  const int max_ring = format == KVQ_INT2 ? 16384 : 4096;
  if (residual_length < 0 || residual_length > max_ring)
    return fail(KVQ_ERR_INVALID_ARG, "residual_length %d outside 0..%d", residual_length, max_ring);
  switch (format) {
    case KVQ_NVFP4:
      if (group_size != 0 && group_size != 16)
        return fail(KVQ_ERR_INVALID_ARG, "NVFP4 blocks are 16 values (group_size %d)", group_size);
      g->group = 16;
      g->code_bytes = head_dim / 2;
      g->meta_bytes = head_dim / 16;
      break;
    case KVQ_INT4:
      if (group_size != 64 && group_size != 32)
        return fail(KVQ_ERR_INVALID_ARG, "INT4 group_size must be 64 or 32 (got %d)", group_size);
      g->group = group_size;
      g->code_bytes = head_dim / 2;
      g->meta_bytes = (head_dim / group_size) * 8;
      break;
    case KVQ_INT2:
      if (group_size != 64 && group_size != 32)
        return fail(KVQ_ERR_INVALID_ARG, "INT2 group_size must be 64 or 32 (got %d)", group_size);
      g->group = group_size;
      g->code_bytes = head_dim / 4;
      g->meta_bytes = (head_dim / group_size) * 8;
      break;
    case KVQ_INT8:
      if (group_size != 64)
        return fail(KVQ_ERR_INVALID_ARG, "INT8 group_size must be 64 (got %d)", group_size);
      g->group = group_size;
      g->code_bytes = head_dim;
      g->meta_bytes = (head_dim / group_size) * 8;
      break;
    case KVQ_FP8:
      if (group_size != 0)
        return fail(KVQ_ERR_INVALID_ARG, "FP8 has no groups (group_size %d)", group_size);
      g->code_bytes = head_dim;
      g->meta_bytes = 0;
      break;
  }
  g->cap = (int64_t)align_up((size_t)max_len, kCapacityAlign);
  const size_t bh = (size_t)batch * kv_heads;
  const int renewal = opt ? opt->scale_renewal : 0;
  if (renewal != 0) {
    if (format != KVQ_NVFP4 && format != KVQ_FP8)
      return fail(KVQ_ERR_INVALID_ARG, "scale renewal is defined for NVFP4 and FP8");
    if (residual_length != 0)
      return fail(KVQ_ERR_INVALID_ARG, "scale renewal is defined for caches without a ring");
    if (renewal < 16 || renewal % 16 != 0)
      return fail(KVQ_ERR_INVALID_ARG, "scale_renewal %d must be a positive multiple of 16", renewal);
  }
  g->renewal = renewal;
  g->nseg = renewal ? (g->cap + renewal - 1) / renewal : 0;
  if (opt && opt->compact_meta) {
    if (!int_affine_format(format) || g->group != 64)
      return fail(KVQ_ERR_INVALID_ARG,
                  "compact group metadata is implemented for INT4, INT8 and INT2 with groups of 64");
    g->compact = 1;
    g->meta_bytes = 8;   // {f16 S0, f16 S1, Z0, Z1}: i8 Z (INT4, INT2, 2 zero bytes) or i16 Z (INT8)
  }
  const int page_tokens = opt ? opt->page_tokens : 0;
  if (page_tokens != 0) {
    const int gran = attn_page_granularity(format);
    if (page_tokens < 0 || page_tokens % gran != 0)
      return fail(KVQ_ERR_INVALID_ARG, "page_tokens %d must be a positive multiple of %d", page_tokens,
                  gran);
    if (opt->num_pages <= 0) return fail(KVQ_ERR_INVALID_ARG, "a paged cache needs num_pages > 0");
    if (renewal != 0) return fail(KVQ_ERR_INVALID_ARG, "scale renewal is not defined for paged caches");
    if (batch > kMaxSeqs)
      return fail(KVQ_ERR_INVALID_ARG, "a paged cache holds at most %d sequences", kMaxSeqs);
    g->page_tokens = page_tokens;
    g->num_pages = opt->num_pages;
    g->max_pages = (max_len + page_tokens - 1) / page_tokens;
    g->cap = page_tokens;   // row stride inside a page
  }
  g->counters_off = align_up((size_t)layers * 4 * sizeof(float) + sizeof(int), 16);
  g->seg_off = align_up(g->counters_off + (size_t)layers * bh * sizeof(int), 16);
  g->table_off = align_up(g->seg_off + (size_t)layers * 2 * g->nseg * 8, 16);
  g->header = align_up(g->table_off + (size_t)batch * g->max_pages * sizeof(int32_t), 256);
  const size_t rows = g->page_tokens ? (size_t)g->num_pages * kv_heads * g->page_tokens
                                     : bh * (size_t)g->cap;
  g->codes = align_up(rows * g->code_bytes, 256);
  g->meta = align_up(rows * g->meta_bytes, 256);
  g->ring = align_up(bh * (size_t)residual_length * head_dim * 2, 256);
  g->per_layer = 2 * (g->codes + g->meta + g->ring);
  // (sizes stay far below 2^64 with the limits above; reject absurd totals)
  if ((double)g->per_layer * layers + (double)g->header > 0x1p50)
    return fail(KVQ_ERR_INVALID_ARG, "cache of %.3g bytes is too large",
                (double)g->per_layer * layers + (double)g->header);
  g->total = g->header + (size_t)layers * g->per_layer;
  return KVQ_OK;
}

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// The affine integer formats: no per-tensor scale, optional residual ring.
inline bool int_affine(int format) {
  return format == KVQ_INT4 || format == KVQ_INT8 || format == KVQ_INT2;
}

int check_cache(kvq_cache_t c, int layer) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "null cache");
  if (layer < 0 || layer >= c->layers)
    return fail(KVQ_ERR_INVALID_ARG, "layer %d outside 0..%d", layer, c->layers - 1);
  return KVQ_OK;
}

void free_host_state(kvq_cache_t c) {
  if (c->L) {
    for (int l = 0; l < c->layers; ++l) {
      delete[] c->L[l].seq_main;
      delete[] c->L[l].seq_ring;
    }
  }
  delete[] c->L;
  delete[] c->host_pages;
  delete[] c->free_pages;
  delete[] c->seq_pages;
  delete c;
}

// Every page free (ids handed out in increasing order), every table entry
// unassigned (host copy; the caller clears the device copy).
void reset_page_pool(kvq_cache_t c) {
  for (int64_t i = 0; i < c->num_pages; ++i) c->free_pages[i] = (int32_t)(c->num_pages - 1 - i);
  c->n_free = c->num_pages;
  for (int64_t i = 0; i < (int64_t)c->batch * c->max_pages; ++i) c->host_pages[i] = -1;
  for (int b = 0; b < c->batch; ++b) c->seq_pages[b] = 0;
}

// ---- token counts: one per batch, or one per sequence (ragged) ----------

inline int64_t seq_main(const LayerState& L, int b) { return L.ragged ? L.seq_main[b] : L.len_main; }
inline int64_t seq_ring(const LayerState& L, int b) { return L.ragged ? L.seq_ring[b] : L.len_ring; }

// Keep per-sequence counts (before a change that may make them differ).
void make_ragged(kvq_cache_t c, LayerState& L) {
  if (L.ragged) return;
  for (int b = 0; b < c->batch; ++b) {
    L.seq_main[b] = L.len_main;
    L.seq_ring[b] = L.len_ring;
  }
  L.ragged = true;
}

// Back to one count for the batch when all sequences agree; otherwise keep
// len_main / len_ring equal to sequence 0's.
void normalize(kvq_cache_t c, LayerState& L) {
  if (!L.ragged) return;
  L.len_main = L.seq_main[0];
  L.len_ring = L.seq_ring[0];
  for (int b = 1; b < c->batch; ++b)
    if (L.seq_main[b] != L.len_main || L.seq_ring[b] != L.len_ring) return;
  L.ragged = false;
}

// Set the counts of sequences [b0, b0 + nb) (all of them when the layer
// is not ragged and nb is the batch).
void set_counts(kvq_cache_t c, LayerState& L, int b0, int nb, int64_t m, int64_t r) {
  if (!L.ragged && b0 == 0 && nb == c->batch) {
    L.len_main = m;
    L.len_ring = r;
    return;
  }
  make_ragged(c, L);
  for (int b = b0; b < b0 + nb; ++b) {
    L.seq_main[b] = m;
    L.seq_ring[b] = r;
  }
  normalize(c, L);
}

// True when the attention / decode-step kernels must take per-sequence
// counts and plane rows (the ragged kernel).
inline bool needs_ragged_kernel(kvq_cache_t c, const LayerState& L) { return L.ragged || c->page_tokens; }

// ---- pages ----------------------------------------------------------------

inline int64_t pages_for(kvq_cache_t c, int64_t tokens) {
  return (tokens + c->page_tokens - 1) / c->page_tokens;
}

// Pages sequence b still has to take so that `tokens` main-cache tokens fit.
inline int64_t pages_missing(kvq_cache_t c, int b, int64_t tokens) {
  if (!c->page_tokens) return 0;
  const int64_t need = pages_for(c, tokens) - c->seq_pages[b];
  return need > 0 ? need : 0;
}

int flush_table_update(kvq_cache_t c, TableUpdate& up, cudaStream_t s) {
  if (up.n == 0) return KVQ_OK;
  cudaError_t e = launch_table_update(c->dev_pages, up, s);
  up.n = 0;
  if (e != cudaSuccess) return cuda_fail(e, "block-table update launch");
  return KVQ_OK;
}

// Give sequence b pages for its first `tokens` main-cache tokens (the caller
// has checked that the pool holds enough free pages).
int ensure_pages(kvq_cache_t c, int b, int64_t tokens, cudaStream_t s) {
  if (!c->page_tokens) return KVQ_OK;
  const int64_t need = pages_for(c, tokens);
  TableUpdate up{};
  while (c->seq_pages[b] < need) {
    if (c->n_free == 0) return fail(KVQ_ERR_CAPACITY, "no free page left in the pool");
    const int32_t id = c->free_pages[--c->n_free];
    const int64_t slot = (int64_t)b * c->max_pages + c->seq_pages[b]++;
    c->host_pages[slot] = id;
    up.idx[up.n] = (int32_t)slot;
    up.val[up.n++] = id;
    if (up.n == kTableBatch) {
      int st = flush_table_update(c, up, s);
      if (st != KVQ_OK) return st;
    }
  }
  return flush_table_update(c, up, s);
}

// Return sequence b's pages to the pool.
int release_pages(kvq_cache_t c, int b, cudaStream_t s) {
  if (!c->page_tokens) return KVQ_OK;
  TableUpdate up{};
  while (c->seq_pages[b] > 0) {
    const int64_t slot = (int64_t)b * c->max_pages + --c->seq_pages[b];
    c->free_pages[c->n_free++] = c->host_pages[slot];
    c->host_pages[slot] = -1;
    up.idx[up.n] = (int32_t)slot;
    up.val[up.n++] = -1;
    if (up.n == kTableBatch) {
      int st = flush_table_update(c, up, s);
      if (st != KVQ_OK) return st;
    }
  }
  return flush_table_update(c, up, s);
}

// Main-cache tokens a sequence holds after appending n tokens to (m, r).
inline int64_t main_after(kvq_cache_t c, int64_t m, int64_t r, int64_t n) {
  return c->R ? m + ((r + n) / c->R) * c->R : m + n;
}

// ---- quantize-append ------------------------------------------------------

// Quantize n tokens per unit from a bf16 source into the main cache of
// `layer`, sequences [b0, b0 + nb), at main-cache positions dst_tok0 ...
int quantize_units(kvq_cache_t c, int layer, int b0, int nb, const uint16_t* sk, const uint16_t* sv,
                   int64_t src_bh_stride, int64_t src_tok0, int64_t n, int64_t dst_tok0,
                   bool calibrate, cudaStream_t stream) {
  LayerState& L = c->L[layer];
  for (int b = b0; b < b0 + nb; ++b) {
    int st = ensure_pages(c, b, dst_tok0 + n, stream);
    if (st != KVQ_OK) return st;
  }
  QuantArgs a{};
  a.src[0] = sk;
  a.src[1] = sv;
  a.src_bh_stride = src_bh_stride;
  a.src_tok0 = src_tok0;
  a.dst[0] = L.kv[0];
  a.dst[1] = L.kv[1];
  a.dst_tok0 = dst_tok0;
  a.n = n;
  a.bh = nb * c->kv_heads;
  a.cap = c->capacity;
  a.group = c->group;
  for (int kv = 0; kv < 2; ++kv) {
    a.gscale[kv] = L.gscale[kv];
    a.amax[kv] = L.amax[kv];
    a.gscale_out[kv] = L.gscale[kv];
  }
  a.calibrate = calibrate ? 1 : 0;
  a.gseg[0] = L.seg_scale[0];
  a.gseg[1] = L.seg_scale[1];
  a.renewal = c->renewal;
  a.compact = c->compact;
  a.unit0 = (int64_t)b0 * c->kv_heads;
  a.kv_heads = c->kv_heads;
  a.pages = c->dev_pages;
  a.page_tokens = c->page_tokens;
  a.max_pages = (int)c->max_pages;
  cudaError_t e = launch_quantize(c->format, a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  // the lowest main-cache position this kernel writes (per-sequence writes:
  // no decode kernel reads ahead of its grid-dependency wait until a
  // whole-batch write sets it again)
  L.write_lo = (b0 == 0 && nb == c->batch && !L.ragged) ? dst_tok0 : 0;
  return KVQ_OK;
}

// Uniform-batch form used by the scale-renewal path (all sequences, at the
// layer's main-cache end), advancing len_main.
int quantize_into_main(kvq_cache_t c, int layer, const uint16_t* sk, const uint16_t* sv,
                       int64_t src_bh_stride, int64_t src_tok0, int64_t n, bool calibrate,
                       cudaStream_t stream) {
  LayerState& L = c->L[layer];
  int st = quantize_units(c, layer, 0, c->batch, sk, sv, src_bh_stride, src_tok0, n, L.len_main,
                          calibrate, stream);
  if (st != KVQ_OK) return st;
  L.len_main += n;
  return KVQ_OK;
}

// Ring planes of sequence b0's first unit.
inline uint16_t* ring_of(kvq_cache_t c, const LayerState& L, int kv, int b0) {
  return L.kv[kv].ring + (size_t)b0 * c->kv_heads * c->R * c->head_dim;
}

// Append n tokens to sequences [b0, b0 + nb), which hold the same counts
// (the per-tensor scales are already calibrated).  With a ring this equals
// appending the tokens one by one: top up the ring, flush it when it is
// full, quantize whole rings straight from the input, keep the rest.
int append_group(kvq_cache_t c, int layer, int b0, int nb, const uint16_t* sk, const uint16_t* sv,
                 int64_t bh_stride, int64_t n, cudaStream_t s) {
  LayerState& L = c->L[layer];
  int64_t m = seq_main(L, b0), r = seq_ring(L, b0);
  int st;
  if (c->R == 0) {
    st = quantize_units(c, layer, b0, nb, sk, sv, bh_stride, 0, n, m, false, s);
    if (st != KVQ_OK) return st;
    set_counts(c, L, b0, nb, m + n, 0);
    return KVQ_OK;
  }
  const int bh = nb * c->kv_heads;
  uint16_t* rk = ring_of(c, L, 0, b0);
  uint16_t* rv = ring_of(c, L, 1, b0);
  const int64_t ring_stride = (int64_t)c->R * c->head_dim;
  int64_t done = 0;
  const int64_t a = std::min<int64_t>(n, c->R - r);
  if (a > 0) {
    cudaError_t e = launch_ring_copy(sk, sv, bh_stride, 0, rk, rv, c->R, r, a, bh, s);
    if (e != cudaSuccess) return cuda_fail(e, "ring copy launch");
    r += a;
    done = a;
  }
  if (r == c->R) {   // the ring is full: quantize it into the main cache
    st = quantize_units(c, layer, b0, nb, rk, rv, ring_stride, 0, r, m, false, s);
    if (st != KVQ_OK) return st;
    m += r;
    r = 0;
  }
  const int64_t whole = ((n - done) / c->R) * c->R;   // whole rings straight from the input
  if (whole > 0) {
    st = quantize_units(c, layer, b0, nb, sk, sv, bh_stride, done, whole, m, false, s);
    if (st != KVQ_OK) return st;
    m += whole;
    done += whole;
  }
  if (done < n) {   // the rest goes to the (now empty) ring
    const int64_t rem = n - done;
    cudaError_t e = launch_ring_copy(sk, sv, bh_stride, done, rk, rv, c->R, 0, rem, bh, s);
    if (e != cudaSuccess) return cuda_fail(e, "ring copy launch");
    r = rem;
  }
  set_counts(c, L, b0, nb, m, r);
  return KVQ_OK;
}

// Quantize the rings of sequences [b0, b0 + nb) (equal counts) into the
// main cache and empty them.
int flush_group(kvq_cache_t c, int layer, int b0, int nb, cudaStream_t s) {
  LayerState& L = c->L[layer];
  const int64_t m = seq_main(L, b0), r = seq_ring(L, b0);
  if (r == 0) return KVQ_OK;
  int st = quantize_units(c, layer, b0, nb, ring_of(c, L, 0, b0), ring_of(c, L, 1, b0),
                          (int64_t)c->R * c->head_dim, 0, r, m, false, s);
  if (st != KVQ_OK) return st;
  set_counts(c, L, b0, nb, m + r, 0);
  return KVQ_OK;
}

// NVFP4 / FP8: set the layer's per-tensor scales from the amax of `elems`
// values of k and of v (the layer's first append).
int calibrate_layer(kvq_cache_t c, int layer, const uint16_t* sk, const uint16_t* sv, int64_t elems,
                    cudaStream_t s) {
  LayerState& L = c->L[layer];
  if (int_affine(c->format) || (L.calibrated[0] && L.calibrated[1])) return KVQ_OK;
  cudaError_t e = launch_amax(sk, sv, elems, L.amax[0], L.amax[1], s);
  if (e == cudaSuccess)
    e = launch_scale_from_amax(L.amax[0], L.amax[1], L.gscale[0], L.gscale[1],
                               c->format == KVQ_NVFP4 ? 2688.0f : 448.0f, s);
  if (e != cudaSuccess) return cuda_fail(e, "calibration launch");
  L.calibrated[0] = L.calibrated[1] = true;
  return KVQ_OK;
}

}  // namespace

int kvq::report_error(int code, const char* msg) { return fail(code, "%s", msg); }

extern "C" {

size_t kvq_cache_bytes_ex(int format, int layers, int batch, int kv_heads, int head_dim,
                          int64_t max_len, int group_size, int residual_length,
                          const kvq_options* options) {
  Geometry g;
  if (geometry(format, layers, batch, kv_heads, head_dim, max_len, group_size, residual_length,
               options, &g) != KVQ_OK)
    return 0;
  return g.total;
}

size_t kvq_cache_bytes(int format, int layers, int batch, int kv_heads, int head_dim,
                       int64_t max_len, int group_size, int residual_length) {
  return kvq_cache_bytes_ex(format, layers, batch, kv_heads, head_dim, max_len, group_size,
                            residual_length, nullptr);
}

int kvq_cache_create(kvq_cache_t* out, int format, int layers, int batch, int kv_heads,
                     int head_dim, int64_t max_len, int group_size, int residual_length,
                     void* device_buf, size_t buf_bytes, const float* global_scales) {
  return kvq_cache_create_ex(out, format, layers, batch, kv_heads, head_dim, max_len, group_size,
                             residual_length, device_buf, buf_bytes, global_scales, nullptr);
}

int kvq_cache_create_ex(kvq_cache_t* out, int format, int layers, int batch, int kv_heads,
                        int head_dim, int64_t max_len, int group_size, int residual_length,
                        void* device_buf, size_t buf_bytes, const float* global_scales,
                        const kvq_options* options) {
  if (!out) return fail(KVQ_ERR_INVALID_ARG, "null output handle");
  *out = nullptr;
  Geometry g;
  int st = geometry(format, layers, batch, kv_heads, head_dim, max_len, group_size,
                    residual_length, options, &g);
  if (st != KVQ_OK) return st;
  if (!device_buf) return fail(KVQ_ERR_INVALID_ARG, "null device buffer");
  if (((uintptr_t)device_buf & 255u) != 0)
    return fail(KVQ_ERR_INVALID_ARG, "device buffer must be 256-byte aligned");
  if (buf_bytes < g.total)
    return fail(KVQ_ERR_WORKSPACE, "device buffer has %zu bytes, %zu needed", buf_bytes, g.total);
  if (global_scales) {
    for (int i = 0; i < 2 * layers; ++i)
      if (!(global_scales[i] > 0.0f) || global_scales[i] > 3.0e38f)
        return fail(KVQ_ERR_INVALID_ARG, "global scale %d must be positive and finite", i);
  }
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, device_buf);
  if (e != cudaSuccess) return cuda_fail(e, "cudaPointerGetAttributes");
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail(KVQ_ERR_INVALID_ARG, "cache buffer is not device memory");

  kvq_cache* c = new (std::nothrow) kvq_cache();
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "out of host memory");
  c->L = new (std::nothrow) LayerState[layers];
  if (!c->L) {
    delete c;
    return fail(KVQ_ERR_INVALID_ARG, "out of host memory");
  }
  c->format = format;
  c->layers = layers;
  c->batch = batch;
  c->kv_heads = kv_heads;
  c->head_dim = head_dim;
  c->max_len = max_len;
  c->capacity = g.cap;
  c->group = g.group;
  c->R = residual_length;
  c->code_bytes = g.code_bytes;
  c->meta_bytes = g.meta_bytes;
  c->scales_given = global_scales != nullptr;
  c->renewal = g.renewal;
  c->nseg = g.nseg;
  c->compact = g.compact;
  c->page_tokens = g.page_tokens;
  c->num_pages = g.num_pages;
  c->max_pages = g.max_pages;
  c->device = attr.device;
  if (const char* env = getenv("KVQ_CTAS")) c->ctas_env = atoi(env);
  if (const char* env = getenv("KVQ_PDL")) c->pdl = atoi(env) != 0;
  // unit-start weight in tiles: about the time of a query load plus a merge
  // (measured optima on B200: 2 of NVFP4's 384-token tiles, 3 of INT4's
  // 256-token tiles; FP8's 128-token tiles take 4)
  c->split_wb = format == KVQ_NVFP4 ? 2 : (format == KVQ_INT4 || format == KVQ_INT2) ? 3 : 4;
  if (const char* env = getenv("KVQ_UNIT_WEIGHT")) c->split_wb = atoi(env) < 0 ? 0 : atoi(env);

  bool host_ok = true;
  for (int l = 0; l < layers && host_ok; ++l) {
    c->L[l].seq_main = new (std::nothrow) int64_t[batch]();
    c->L[l].seq_ring = new (std::nothrow) int64_t[batch]();
    host_ok = c->L[l].seq_main && c->L[l].seq_ring;
  }
  if (host_ok && g.page_tokens) {
    c->host_pages = new (std::nothrow) int32_t[(size_t)batch * g.max_pages];
    c->free_pages = new (std::nothrow) int32_t[g.num_pages];
    c->seq_pages = new (std::nothrow) int64_t[batch]();
    host_ok = c->host_pages && c->free_pages && c->seq_pages;
  }
  if (!host_ok) {
    free_host_state(c);
    return fail(KVQ_ERR_INVALID_ARG, "out of host memory");
  }
  uint8_t* base = static_cast<uint8_t*>(device_buf);
  float* hdr = reinterpret_cast<float*>(base);
  if (g.page_tokens) {
    c->dev_pages = reinterpret_cast<int32_t*>(base + g.table_off);
    reset_page_pool(c);
  }
  c->dev_status = reinterpret_cast<int*>(hdr + (size_t)layers * 4);
  c->counters = reinterpret_cast<int*>(base + g.counters_off);
  uint8_t* p = base + g.header;
  for (int l = 0; l < layers; ++l) {
    LayerState& L = c->L[l];
    for (int kv = 0; kv < 2; ++kv) {
      L.gscale[kv] = hdr + l * 4 + kv;
      L.amax[kv] = reinterpret_cast<uint32_t*>(hdr + l * 4 + 2 + kv);
      L.kv[kv].codes = p;
      p += g.codes;
      L.kv[kv].meta = g.meta_bytes ? p : nullptr;
      p += g.meta;
      L.kv[kv].ring = residual_length ? reinterpret_cast<uint16_t*>(p) : nullptr;
      p += g.ring;
      L.calibrated[kv] = int_affine(format) || c->scales_given;
      if (g.renewal) {
        float* seg = reinterpret_cast<float*>(base + g.seg_off);
        L.seg_scale[kv] = seg + ((size_t)l * 2 + kv) * g.nseg;
        L.seg_amax[kv] = reinterpret_cast<uint32_t*>(seg + (size_t)layers * 2 * g.nseg) +
                         ((size_t)l * 2 + kv) * g.nseg;
      }
    }
  }
  int dev_prev = 0;
  cudaGetDevice(&dev_prev);
  if (dev_prev != c->device) cudaSetDevice(c->device);
  e = cudaMemset(device_buf, 0, g.total);
  if (e == cudaSuccess && g.page_tokens)   // every block-table entry starts unassigned (-1)
    e = cudaMemset(c->dev_pages, 0xFF, (size_t)batch * g.max_pages * sizeof(int32_t));
  if (e == cudaSuccess) {
    float* init = static_cast<float*>(calloc((size_t)layers * 4, sizeof(float)));
    if (!init) {
      e = cudaErrorMemoryAllocation;
    } else {
      for (int l = 0; l < layers; ++l) {
        init[l * 4 + 0] = global_scales ? global_scales[2 * l] : 1.0f;
        init[l * 4 + 1] = global_scales ? global_scales[2 * l + 1] : 1.0f;
      }
      e = cudaMemcpy(hdr, init, (size_t)layers * 4 * sizeof(float), cudaMemcpyHostToDevice);
      free(init);
    }
  }
  if (e == cudaSuccess && g.renewal && global_scales) {
    // segment 0 of every layer starts from the given scales
    const size_t nf = (size_t)layers * 2 * g.nseg;
    float* seg = static_cast<float*>(calloc(nf, sizeof(float)));
    if (!seg) {
      e = cudaErrorMemoryAllocation;
    } else {
      for (int l = 0; l < layers; ++l)
        for (int kv = 0; kv < 2; ++kv) seg[((size_t)l * 2 + kv) * g.nseg] = global_scales[2 * l + kv];
      e = cudaMemcpy(base + g.seg_off, seg, nf * sizeof(float), cudaMemcpyHostToDevice);
      free(seg);
    }
  }
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, c->device);
  if (dev_prev != c->device) cudaSetDevice(dev_prev);
  if (e != cudaSuccess) {
    free_host_state(c);
    return cuda_fail(e, "cache initialisation");
  }
  *out = c;
  return ok();
}

int kvq_cache_destroy(kvq_cache_t c) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "null cache");
  free_host_state(c);
  return ok();
}

int kvq_cache_reset(kvq_cache_t c, void* stream) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "null cache");
  if (c->page_tokens) {
    reset_page_pool(c);
    cudaError_t e = cudaMemsetAsync(c->dev_pages, 0xFF, (size_t)c->batch * c->max_pages * sizeof(int32_t),
                                    S(stream));
    if (e != cudaSuccess) return cuda_fail(e, "reset");
  }
  for (int l = 0; l < c->layers; ++l) {
    LayerState& L = c->L[l];
    L.len_main = L.len_ring = 0;
    L.ragged = false;
    L.write_lo = 0;
    for (int kv = 0; kv < 2; ++kv) {
      if (!int_affine(c->format) && !c->scales_given) {
        L.calibrated[kv] = false;
        cudaError_t e = cudaMemsetAsync(L.amax[kv], 0, sizeof(uint32_t), S(stream));
        if (e != cudaSuccess) return cuda_fail(e, "reset");
      }
      if (c->renewal) {
        cudaError_t e = cudaMemsetAsync(L.seg_amax[kv], 0, c->nseg * sizeof(uint32_t), S(stream));
        // Segment scales past the first are cleared too, so that no scale of
        // the previous history is read for a slot the new history has not
        // written yet.  Segment 0 keeps a given scale; without one, the next
        // calibrating append rewrites it.
        const int64_t keep = c->scales_given ? 1 : 0;
        if (e == cudaSuccess && c->nseg > keep)
          e = cudaMemsetAsync(L.seg_scale[kv] + keep, 0, (c->nseg - keep) * sizeof(float), S(stream));
        if (e != cudaSuccess) return cuda_fail(e, "reset");
      }
    }
  }
  return ok();
}

int kvq_append(kvq_cache_t c, int layer, const void* k, const void* v, int64_t n, void* stream) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (n < 0) return fail(KVQ_ERR_INVALID_ARG, "negative token count");
  if (n == 0) return ok();
  if (!k || !v) return fail(KVQ_ERR_INVALID_ARG, "null k or v");
  if (!aligned16(k) || !aligned16(v)) return fail(KVQ_ERR_INVALID_ARG, "k and v must be 16-byte aligned");
  LayerState& L = c->L[layer];
  int64_t new_pages = 0;
  for (int b = 0; b < c->batch; ++b) {
    const int64_t m = seq_main(L, b), r = seq_ring(L, b);
    if (m + r + n > c->max_len)
      return fail(KVQ_ERR_CAPACITY, "append of %lld tokens exceeds max_len %lld (sequence %d holds %lld)",
                  (long long)n, (long long)c->max_len, b, (long long)(m + r));
    new_pages += pages_missing(c, b, main_after(c, m, r, n));
  }
  if (new_pages > c->n_free)
    return fail(KVQ_ERR_CAPACITY, "append needs %lld more pages, %lld are free", (long long)new_pages,
                (long long)c->n_free);
  cudaStream_t s = S(stream);
  const uint16_t* sk = static_cast<const uint16_t*>(k);
  const uint16_t* sv = static_cast<const uint16_t*>(v);
  const int64_t bh_stride = n * c->head_dim;

  if (c->renewal) {
    if (L.ragged) return fail(KVQ_ERR_UNSUPPORTED, "scale renewal needs equal sequence lengths");
    // Scale renewal: segment 0 takes the scale calibrated from the first
    // append; every segment whose first token this append brings takes the
    // scale of the previous segment's amax, which this append may complete.
    const float divisor = c->format == KVQ_NVFP4 ? 2688.0f : 448.0f;
    cudaError_t e = cudaSuccess;
    if (!(L.calibrated[0] && L.calibrated[1])) {
      const int64_t elems = (int64_t)c->batch * c->kv_heads * n * c->head_dim;
      e = launch_amax(sk, sv, elems, L.amax[0], L.amax[1], s);
      if (e == cudaSuccess)
        e = launch_scale_from_amax(L.amax[0], L.amax[1], L.seg_scale[0], L.seg_scale[1], divisor, s);
    }
    const int64_t pos0 = L.len_main, P = c->renewal;
    if (e == cudaSuccess)
      e = launch_seg_amax(sk, sv, bh_stride, n, c->batch * c->kv_heads, pos0, c->renewal,
                          L.seg_amax[0], L.seg_amax[1], s);
    const int64_t s_first = std::max<int64_t>(1, (pos0 + P - 1) / P), s_last = (pos0 + n - 1) / P;
    if (e == cudaSuccess)
      e = launch_renew_scales(L.seg_amax[0], L.seg_amax[1], L.seg_scale[0], L.seg_scale[1], s_first,
                              s_last, divisor, s);
    if (e != cudaSuccess) return cuda_fail(e, "scale renewal launch");
    L.calibrated[0] = L.calibrated[1] = true;
    st = quantize_into_main(c, layer, sk, sv, bh_stride, 0, n, false, s);
    return st == KVQ_OK ? ok() : st;
  }
  const int64_t elems = (int64_t)c->batch * c->kv_heads * n * c->head_dim;
  if (!L.ragged && c->R == 0 && !int_affine(c->format) && !(L.calibrated[0] && L.calibrated[1])) {
    // the calibrating append without a ring: amax, then the quantize kernel
    // derives the scales from it (and stores them) itself
    cudaError_t e = launch_amax(sk, sv, elems, L.amax[0], L.amax[1], s);
    if (e != cudaSuccess) return cuda_fail(e, "amax launch");
    st = quantize_units(c, layer, 0, c->batch, sk, sv, bh_stride, 0, n, L.len_main, true, s);
    if (st != KVQ_OK) return st;
    L.len_main += n;
    L.calibrated[0] = L.calibrated[1] = true;
    return ok();
  }
  // NVFP4 / FP8 calibrate from the first append even when all of its
  // tokens go to a ring
  st = calibrate_layer(c, layer, sk, sv, elems, s);
  if (st != KVQ_OK) return st;
  if (!L.ragged) {
    st = append_group(c, layer, 0, c->batch, sk, sv, bh_stride, n, s);
    return st == KVQ_OK ? ok() : st;
  }
  // sequences of different lengths: each at its own end
  const int64_t seq_stride = (int64_t)c->kv_heads * n * c->head_dim;
  for (int b = 0; b < c->batch; ++b) {
    st = append_group(c, layer, b, 1, sk + b * seq_stride, sv + b * seq_stride, bh_stride, n, s);
    if (st != KVQ_OK) return st;
  }
  return ok();
}

int kvq_append_seq(kvq_cache_t c, int layer, int seq, const void* k, const void* v, int64_t n,
                   void* stream) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (seq < 0 || seq >= c->batch) return fail(KVQ_ERR_INVALID_ARG, "sequence %d outside 0..%d", seq, c->batch - 1);
  if (n < 0) return fail(KVQ_ERR_INVALID_ARG, "negative token count");
  if (n == 0) return ok();
  if (!k || !v) return fail(KVQ_ERR_INVALID_ARG, "null k or v");
  if (!aligned16(k) || !aligned16(v)) return fail(KVQ_ERR_INVALID_ARG, "k and v must be 16-byte aligned");
  if (c->renewal) return fail(KVQ_ERR_UNSUPPORTED, "scale renewal needs equal sequence lengths");
  if (c->batch > kMaxSeqs)
    return fail(KVQ_ERR_UNSUPPORTED, "per-sequence lengths are implemented for at most %d sequences", kMaxSeqs);
  LayerState& L = c->L[layer];
  const int64_t m = seq_main(L, seq), r = seq_ring(L, seq);
  if (m + r + n > c->max_len)
    return fail(KVQ_ERR_CAPACITY, "append of %lld tokens exceeds max_len %lld (sequence %d holds %lld)",
                (long long)n, (long long)c->max_len, seq, (long long)(m + r));
  if (pages_missing(c, seq, main_after(c, m, r, n)) > c->n_free)
    return fail(KVQ_ERR_CAPACITY, "no free page left in the pool");
  cudaStream_t s = S(stream);
  const uint16_t* sk = static_cast<const uint16_t*>(k);
  const uint16_t* sv = static_cast<const uint16_t*>(v);
  st = calibrate_layer(c, layer, sk, sv, (int64_t)c->kv_heads * n * c->head_dim, s);
  if (st != KVQ_OK) return st;
  st = append_group(c, layer, seq, 1, sk, sv, n * c->head_dim, n, s);
  return st == KVQ_OK ? ok() : st;
}

int kvq_flush_residual(kvq_cache_t c, int layer, void* stream) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (c->R == 0) return ok();
  LayerState& L = c->L[layer];
  int64_t new_pages = 0;
  for (int b = 0; b < c->batch; ++b)
    new_pages += pages_missing(c, b, seq_main(L, b) + seq_ring(L, b));
  if (new_pages > c->n_free) return fail(KVQ_ERR_CAPACITY, "no free page left in the pool");
  if (!L.ragged) {
    st = flush_group(c, layer, 0, c->batch, S(stream));
    return st == KVQ_OK ? ok() : st;
  }
  for (int b = 0; b < c->batch; ++b) {
    st = flush_group(c, layer, b, 1, S(stream));
    if (st != KVQ_OK) return st;
  }
  return ok();
}

// CTAs the attention kernel can keep resident at once (one wave).
static int resident_ctas(kvq_cache_t c) {
  // attention CTAs resident per SM, per format id (KVQ_NVFP4 .. KVQ_INT2)
  // and kernel variant (NVFP4 / FP8: plain, with a ring, with scale renewal;
  // INT4: compact group metadata)
  static int bps[KVQ_INT2 + 1][4] = {};
  static_assert(KVQ_NVFP4 >= 0 && KVQ_INT4 <= KVQ_INT2 && KVQ_FP8 <= KVQ_INT2 && KVQ_INT8 <= KVQ_INT2,
                "format ids index bps");
  const int var = c->compact ? 3 : c->renewal ? 2 : c->R > 0 ? 1 : 0;
  if (bps[c->format][var] == 0)
    bps[c->format][var] = attn_blocks_per_sm(c->format, var == 1, var == 2, var == 3);
  int n = c->sm_count * bps[c->format][var];
  if (c->ctas_env > n) n = c->ctas_env;
  return n < 1 ? 1 : n;
}


size_t kvq_workspace_bytes(kvq_cache_t c, int q_heads) {
  if (!c || q_heads <= 0 || q_heads % c->kv_heads != 0)
    return 0;
  const int G = q_heads / c->kv_heads;
  const size_t units = (size_t)c->batch * c->kv_heads;
  // A unit is touched by at most floor(C / kv_heads) + 2 CTAs of a C-CTA
  // grid, whatever the sequence lengths: the grid splits a line on which
  // the kv_heads units of one sequence have equal spans, and each CTA takes
  // 1/C of the line.  (With equal lengths the bound is C / units + 2.)
  const size_t C = (size_t)resident_ctas(c);
  const size_t maxc = std::min(C, C / (size_t)c->kv_heads + 2);
  return align_up(units * maxc * G * (kHeadDim + 2) * sizeof(float), 256);
}

}  // extern "C"

namespace {

// The common fields of an attention launch.
AttnArgs attn_args(kvq_cache_t c, int layer, const void* q, int G, float softmax_scale, float* out,
                   void* workspace, float* lse) {
  const LayerState& L = c->L[layer];
  AttnArgs a{};
  a.format = c->format;
  a.k = L.kv[0];
  a.v = L.kv[1];
  a.gscale_k = int_affine(c->format) ? nullptr : L.gscale[0];
  a.gscale_v = int_affine(c->format) ? nullptr : L.gscale[1];
  a.cap = c->capacity;
  a.R = c->R;
  a.len_main = L.len_main;
  a.len_ring = L.len_ring;
  a.batch = c->batch;
  a.kv_heads = c->kv_heads;
  a.G = G;
  a.group = c->group;
  a.q = static_cast<const uint16_t*>(q);
  a.softmax_scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf((float)c->head_dim);
  a.out = out;
  a.partials = static_cast<float*>(workspace);
  a.counters = c->counters + (size_t)layer * c->batch * c->kv_heads;
  a.dev_status = c->dev_status;
  a.lse = lse;
  a.gseg_k = L.seg_scale[0];
  a.gseg_v = L.seg_scale[1];
  a.seg_amax_k = L.seg_amax[0];
  a.seg_amax_v = L.seg_amax[1];
  a.renewal = c->renewal;
  a.compact = c->compact;
  a.pdl = c->pdl;
  a.pre_len = 0;
  return a;
}

// Decode attention over sequences of their own lengths and/or paged
// planes: the host lays out the slot line (see RaggedArgs), splits it over
// the grid with the uniform kernel's unit-start weights, and checks the
// workspace against the actual records per unit.
int ragged_attention(kvq_cache_t c, int layer, const void* q, int q_heads, float softmax_scale,
                     float* out, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                     int new_kind, const void* k_new, const void* v_new, float* lse) {
  const LayerState& L = c->L[layer];
  if (c->batch > kMaxSeqs)
    return fail(KVQ_ERR_UNSUPPORTED, "per-sequence lengths are implemented for at most %d sequences", kMaxSeqs);
  const int G = q_heads / c->kv_heads;
  const int H = c->kv_heads;
  const int tile = attn_tile_tokens(c->format, c->group);
  static thread_local RaggedArgs ra;   // large (it is the kernel's parameter block)
  std::memset(&ra, 0, sizeof(ra));
  const int64_t wb = c->split_wb;
  int64_t slots = 0, line = 0;
  for (int b = 0; b < c->batch; ++b) {
    const int64_t m = seq_main(L, b), r = seq_ring(L, b);
    const int64_t sb = std::max<int64_t>(1, (m + tile - 1) / tile);
    ra.seq_main[b] = (int32_t)m;
    ra.seq_ring[b] = (int32_t)r;
    ra.seq_slot0[b] = (int32_t)slots;
    slots += H * sb;
    line += H * (sb + wb);
  }
  ra.seq_slot0[c->batch] = (int32_t)slots;
  if (slots >= (int64_t(1) << 31)) return fail(KVQ_ERR_UNSUPPORTED, "too many tiles for one launch");
  int64_t C = c->ctas_env > 0 ? c->ctas_env : resident_ctas(c);
  C = std::min<int64_t>(std::min<int64_t>(C, kMaxCtas), slots);
  // CTA i owns line positions [i*line/C, (i+1)*line/C): the first slot at
  // or after each boundary
  {
    int b = 0;
    int64_t pos0 = 0;   // line position of sequence b
    for (int64_t i = 0; i <= C; ++i) {
      const int64_t p = line * i / C;
      int64_t sb = b < c->batch ? std::max<int64_t>(1, ((int64_t)ra.seq_main[b] + tile - 1) / tile) : 1;
      while (b < c->batch && p >= pos0 + H * (sb + wb)) {
        pos0 += H * (sb + wb);
        ++b;
        if (b < c->batch) sb = std::max<int64_t>(1, ((int64_t)ra.seq_main[b] + tile - 1) / tile);
      }
      if (b >= c->batch) {
        ra.cta_slot[i] = (int32_t)slots;
        continue;
      }
      const int64_t off = p - pos0, span = sb + wb;
      const int64_t h = off / span, o = off % span;
      ra.cta_slot[i] = (int32_t)(ra.seq_slot0[b] + h * sb + (o <= wb ? 0 : o - wb));
    }
  }
  // records per unit: the CTAs whose range holds a slot of the unit
  auto cta_of = [&](int64_t x) {
    int64_t lo = 0, hi = C - 1;
    while (lo < hi) {
      const int64_t mid = (lo + hi + 1) / 2;
      if (ra.cta_slot[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  int64_t maxc = 1;
  for (int b = 0; b < c->batch; ++b) {
    const int64_t sb = std::max<int64_t>(1, ((int64_t)ra.seq_main[b] + tile - 1) / tile);
    for (int h = 0; h < H; ++h) {
      const int64_t U0 = ra.seq_slot0[b] + h * sb;
      maxc = std::max<int64_t>(maxc, cta_of(U0 + sb - 1) - cta_of(U0) + 1);
    }
  }
  const size_t need = (size_t)c->batch * H * maxc * G * (kHeadDim + 2) * sizeof(float);
  if (workspace_bytes < need)
    return fail(KVQ_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, need);
  ra.pages = c->dev_pages;
  ra.page_tokens = c->page_tokens;
  ra.max_pages = (int32_t)c->max_pages;

  AttnArgs a = attn_args(c, layer, q, G, softmax_scale, out, workspace, lse);
  a.ctas = (int)C;
  a.maxc = (int)maxc;
  a.wb = (int)wb;
  a.new_kind = new_kind;
  a.k_new = static_cast<const uint16_t*>(k_new);
  a.v_new = static_cast<const uint16_t*>(v_new);
  cudaError_t e = launch_decode_attention_ragged(a, ra, stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode attention launch");
  return ok();
}

// kvq_decode_step over sequences of their own lengths or paged planes:
// every sequence's token goes to its own end (main cache or ring slot),
// written by the attention kernel itself; the two-launch fallback covers the
// calibrating append and any ring that this token fills.
int ragged_decode_step(kvq_cache_t c, int layer, const void* k, const void* v, const void* q,
                       int q_heads, float softmax_scale, float* out, void* workspace,
                       size_t workspace_bytes, cudaStream_t s) {
  LayerState& L = c->L[layer];
  const bool ring = c->R > 0;
  bool fills = false;
  int64_t new_pages = 0;
  for (int b = 0; b < c->batch; ++b) {
    const int64_t m = seq_main(L, b), r = seq_ring(L, b);
    if (m + r + 1 > c->max_len)
      return fail(KVQ_ERR_CAPACITY, "decode step exceeds max_len %lld (sequence %d)", (long long)c->max_len, b);
    fills |= ring && r + 1 == c->R;
    if (!ring) new_pages += pages_missing(c, b, m + 1);
  }
  const bool calibrated = int_affine(c->format) || (L.calibrated[0] && L.calibrated[1]);
  if (!calibrated || fills) {
    int st = kvq_append(c, layer, k, v, 1, s);
    if (st != KVQ_OK) return st;
    return kvq_decode_attention(c, layer, q, q_heads, softmax_scale, out, workspace, workspace_bytes, s);
  }
  if (new_pages > c->n_free) return fail(KVQ_ERR_CAPACITY, "no free page left in the pool");
  // counts including the new token
  const bool was_ragged = L.ragged;
  const int64_t old_main = L.len_main, old_ring = L.len_ring;
  make_ragged(c, L);
  for (int b = 0; b < c->batch; ++b) {
    if (ring) ++L.seq_ring[b]; else ++L.seq_main[b];
    if (!ring) {
      int st = ensure_pages(c, b, L.seq_main[b], s);
      if (st != KVQ_OK) return st;   // (cannot happen: checked above)
    }
  }
  int st = ragged_attention(c, layer, q, q_heads, softmax_scale, out, workspace, workspace_bytes, s,
                            ring ? 2 : 1, k, v, nullptr);
  if (st == KVQ_OK && !ring) L.write_lo = 0;
  if (st != KVQ_OK) {
    for (int b = 0; b < c->batch; ++b) {
      if (ring) --L.seq_ring[b]; else --L.seq_main[b];
    }
    if (!was_ragged) {
      L.ragged = false;
      L.len_main = old_main;
      L.len_ring = old_ring;
      return st;
    }
  }
  normalize(c, L);
  return st;
}

// Shared by kvq_decode_attention and kvq_decode_step.  new_kind/new_pos/k/v
// describe a token the kernel appends itself (0 = none); the layer's lengths
// must already include it.
int decode_attention_impl(kvq_cache_t c, int layer, const void* q, int q_heads, float softmax_scale,
                          float* out, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                          int new_kind, int64_t new_pos, const void* k_new, const void* v_new,
                          float* lse = nullptr) {
  const LayerState& L = c->L[layer];
  if (needs_ragged_kernel(c, L))
    return ragged_attention(c, layer, q, q_heads, softmax_scale, out, workspace, workspace_bytes, stream,
                            new_kind, k_new, v_new, lse);
  const int G = q_heads / c->kv_heads;
  const int64_t units = (int64_t)c->batch * c->kv_heads;
  const int tile = attn_tile_tokens(c->format, c->group);
  const int64_t tpu = (L.len_main + tile - 1) / tile;
  const int64_t T = tpu > 0 ? units * tpu : units;
  int64_t C = c->ctas_env > 0 ? c->ctas_env : resident_ctas(c);
  if (C > T) C = T;
  const int64_t wb = tpu > 0 ? c->split_wb : 0;
  const int64_t W = units * ((tpu > 0 ? tpu : 1) + wb);
  int64_t maxc = 1;
  if (tpu > 0) {
    for (int64_t u = 0; u < units; ++u) {
      const int64_t n = split_cta_of_tile(u * tpu + tpu - 1, tpu, wb, W, C) -
                        split_cta_of_tile(u * tpu, tpu, wb, W, C) + 1;
      if (n > maxc) maxc = n;
    }
  }
  const size_t need = (size_t)units * maxc * G * (kHeadDim + 2) * sizeof(float);
  if (workspace_bytes < need)
    return fail(KVQ_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, need);

  AttnArgs a = attn_args(c, layer, q, G, softmax_scale, out, workspace, lse);
  a.ctas = (int)C;
  a.tpu = (int)tpu;
  a.maxc = (int)maxc;
  a.wb = (int)wb;
  a.new_kind = new_kind;
  a.new_pos = new_pos;
  a.k_new = static_cast<const uint16_t*>(k_new);
  a.v_new = static_cast<const uint16_t*>(v_new);
  // tokens no still-running kernel writes: below the previous main-cache
  // write of the layer, and below this step's own token
  a.pre_len = std::min<int64_t>(L.write_lo, new_kind == 1 ? new_pos : L.len_main);
  cudaError_t e = launch_decode_attention(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode attention launch");
  if (new_kind == 1) c->L[layer].write_lo = new_pos;
  return ok();
}

// Some sequence of the layer holds a token.
bool any_tokens(kvq_cache_t c, const LayerState& L) {
  if (!L.ragged) return L.len_main + L.len_ring > 0;
  for (int b = 0; b < c->batch; ++b)
    if (L.seq_main[b] + L.seq_ring[b] > 0) return true;
  return false;
}

// Argument checks of the attention calls (nothing is modified).
int check_attention_args(kvq_cache_t c, int layer, const void* q, int q_heads, float* out,
                         void* workspace) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (!q || !out || !workspace) return fail(KVQ_ERR_INVALID_ARG, "null q, out or workspace");
  if (!aligned16(q) || !aligned16(out) || ((uintptr_t)workspace & 255u))
    return fail(KVQ_ERR_INVALID_ARG, "q/out must be 16-byte and workspace 256-byte aligned");
  if (q_heads <= 0 || q_heads % c->kv_heads != 0)
    return fail(KVQ_ERR_INVALID_ARG, "q_heads %d is not a multiple of kv_heads %d", q_heads,
                c->kv_heads);
  if (q_heads / c->kv_heads > kMaxG)
    return fail(KVQ_ERR_UNSUPPORTED, "more than %d query heads per KV head", kMaxG);
  return KVQ_OK;
}

}  // namespace

extern "C" {

int kvq_decode_attention(kvq_cache_t c, int layer, const void* q, int q_heads,
                         float softmax_scale, float* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
  int st = check_attention_args(c, layer, q, q_heads, out, workspace);
  if (st != KVQ_OK) return st;
  const LayerState& L = c->L[layer];
  if (!any_tokens(c, L)) return fail(KVQ_ERR_EMPTY, "layer %d holds no tokens", layer);
  return decode_attention_impl(c, layer, q, q_heads, softmax_scale, out, workspace, workspace_bytes,
                               S(stream), 0, 0, nullptr, nullptr);
}

int kvq_decode_attention_lse(kvq_cache_t c, int layer, const void* q, int q_heads,
                             float softmax_scale, float* out, float* lse, void* workspace,
                             size_t workspace_bytes, void* stream) {
  int st = check_attention_args(c, layer, q, q_heads, out, workspace);
  if (st != KVQ_OK) return st;
  if (!lse || ((uintptr_t)lse & 3u)) return fail(KVQ_ERR_INVALID_ARG, "lse must be a 4-byte aligned pointer");
  const LayerState& L = c->L[layer];
  if (!any_tokens(c, L)) {
    // a part of the sequence without keys: no weight in the merge
    cudaError_t e = launch_empty_part((int64_t)c->batch * q_heads, out, lse, S(stream));
    if (e != cudaSuccess) return cuda_fail(e, "empty-part launch");
    return ok();
  }
  return decode_attention_impl(c, layer, q, q_heads, softmax_scale, out, workspace, workspace_bytes,
                               S(stream), 0, 0, nullptr, nullptr, lse);
}

int kvq_combine_partials(int n_parts, int64_t rows, int head_dim, const float* o_parts,
                         int64_t o_stride, const float* lse_parts, int64_t lse_stride, float* out,
                         float* lse_out, void* stream) {
  if (n_parts < 1 || rows < 0) return fail(KVQ_ERR_INVALID_ARG, "n_parts %d, rows %lld", n_parts, (long long)rows);
  if (head_dim != kHeadDim)
    return fail(KVQ_ERR_UNSUPPORTED, "head_dim %d: only %d is implemented", head_dim, kHeadDim);
  if (!o_parts || !lse_parts || !out) return fail(KVQ_ERR_INVALID_ARG, "null o_parts, lse_parts or out");
  if (n_parts > 1 && (o_stride < rows * head_dim || lse_stride < rows))
    return fail(KVQ_ERR_INVALID_ARG, "part strides %lld, %lld smaller than a part", (long long)o_stride,
                (long long)lse_stride);
  if (((uintptr_t)o_parts | (uintptr_t)lse_parts | (uintptr_t)out | (uintptr_t)lse_out) & 3u)
    return fail(KVQ_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  cudaError_t e = launch_combine(n_parts, rows, o_parts, o_stride, lse_parts, lse_stride, out, lse_out,
                                 S(stream));
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  return ok();
}

int kvq_decode_step(kvq_cache_t c, int layer, const void* k, const void* v, const void* q,
                    int q_heads, float softmax_scale, float* out, void* workspace,
                    size_t workspace_bytes, void* stream) {
  int st = check_attention_args(c, layer, q, q_heads, out, workspace);
  if (st != KVQ_OK) return st;
  if (!k || !v) return fail(KVQ_ERR_INVALID_ARG, "null k or v");
  if (!aligned16(k) || !aligned16(v)) return fail(KVQ_ERR_INVALID_ARG, "k and v must be 16-byte aligned");
  LayerState& L = c->L[layer];
  if (needs_ragged_kernel(c, L))
    return ragged_decode_step(c, layer, k, v, q, q_heads, softmax_scale, out, workspace, workspace_bytes,
                              S(stream));
  if (L.len_main + L.len_ring + 1 > c->max_len)
    return fail(KVQ_ERR_CAPACITY, "decode step exceeds max_len %lld", (long long)c->max_len);
  const bool ring = c->R > 0;
  const bool calibrated = int_affine(c->format) || (L.calibrated[0] && L.calibrated[1]);
  const bool renews = c->renewal && L.len_main % c->renewal == 0;
  if (!calibrated || (ring && L.len_ring + 1 == c->R) || renews) {
    // the first (calibrating) append, a ring flush, or the first token of a
    // new scale segment (its scale is renewed first): two separate launches
    st = kvq_append(c, layer, k, v, 1, stream);
    if (st != KVQ_OK) return st;
    return kvq_decode_attention(c, layer, q, q_heads, softmax_scale, out, workspace,
                                workspace_bytes, stream);
  }
  const int64_t old_main = L.len_main, old_ring = L.len_ring;
  int kind;
  int64_t pos;
  if (ring) {
    kind = 2;
    pos = L.len_ring++;
  } else {
    kind = 1;
    pos = L.len_main++;
  }
  st = decode_attention_impl(c, layer, q, q_heads, softmax_scale, out, workspace, workspace_bytes,
                             S(stream), kind, pos, k, v);
  if (st != KVQ_OK) {
    L.len_main = old_main;
    L.len_ring = old_ring;
  }
  return st;
}

}  // extern "C"

namespace {

int dequantize_units(kvq_cache_t c, int layer, int kv, int b0, int nb, int64_t start, int64_t n,
                     float* out, void* stream) {
  const LayerState& L = c->L[layer];
  if (n == 0) return ok();
  if (!out || !aligned16(out)) return fail(KVQ_ERR_INVALID_ARG, "out must be 16-byte aligned");
  const RowMap map{(int64_t)b0 * c->kv_heads, c->kv_heads, c->dev_pages, c->page_tokens,
                   (int)c->max_pages};
  cudaError_t e = launch_dequantize(c->format, L.kv[kv], L.gscale[kv], c->capacity, c->group,
                                    nb * c->kv_heads, start, n, out,
                                    (c->format == KVQ_NVFP4 || int_affine(c->format)) && kv == 1,
                                    S(stream), L.seg_scale[kv], c->renewal, c->compact != 0, map);
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return ok();
}

}  // namespace

extern "C" {

int kvq_dequantize(kvq_cache_t c, int layer, int kv, int64_t start, int64_t n, float* out,
                   void* stream) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (kv != 0 && kv != 1) return fail(KVQ_ERR_INVALID_ARG, "kv must be 0 (K) or 1 (V)");
  const LayerState& L = c->L[layer];
  int64_t len = L.len_main;
  for (int b = 0; L.ragged && b < c->batch; ++b) len = std::min(len, L.seq_main[b]);
  if (start < 0 || n < 0 || start + n > len)
    return fail(KVQ_ERR_INVALID_ARG, "token range [%lld, %lld) outside the main cache (%lld)",
                (long long)start, (long long)(start + n), (long long)len);
  return dequantize_units(c, layer, kv, 0, c->batch, start, n, out, stream);
}

int kvq_dequantize_seq(kvq_cache_t c, int layer, int kv, int seq, int64_t start, int64_t n, float* out,
                       void* stream) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (kv != 0 && kv != 1) return fail(KVQ_ERR_INVALID_ARG, "kv must be 0 (K) or 1 (V)");
  if (seq < 0 || seq >= c->batch) return fail(KVQ_ERR_INVALID_ARG, "sequence %d outside 0..%d", seq, c->batch - 1);
  const int64_t len = seq_main(c->L[layer], seq);
  if (start < 0 || n < 0 || start + n > len)
    return fail(KVQ_ERR_INVALID_ARG, "token range [%lld, %lld) outside sequence %d's main cache (%lld)",
                (long long)start, (long long)(start + n), seq, (long long)len);
  return dequantize_units(c, layer, kv, seq, 1, start, n, out, stream);
}

int kvq_truncate(kvq_cache_t c, int layer, int64_t total_len) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  LayerState& L = c->L[layer];
  if (!L.ragged) {
    if (total_len < 0 || total_len > L.len_main + L.len_ring)
      return fail(KVQ_ERR_INVALID_ARG, "cannot truncate %lld tokens to %lld",
                  (long long)(L.len_main + L.len_ring), (long long)total_len);
    if (total_len >= L.len_main) {
      L.len_ring = total_len - L.len_main;
    } else {
      L.len_main = total_len;
      L.len_ring = 0;
    }
    return ok();
  }
  if (total_len < 0) return fail(KVQ_ERR_INVALID_ARG, "negative length %lld", (long long)total_len);
  for (int b = 0; b < c->batch; ++b) {
    if (L.seq_main[b] + L.seq_ring[b] <= total_len) continue;
    if (total_len >= L.seq_main[b]) {
      L.seq_ring[b] = total_len - L.seq_main[b];
    } else {
      L.seq_main[b] = total_len;
      L.seq_ring[b] = 0;
    }
  }
  normalize(c, L);
  return ok();
}

int kvq_truncate_seq(kvq_cache_t c, int layer, int seq, int64_t total_len) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (seq < 0 || seq >= c->batch) return fail(KVQ_ERR_INVALID_ARG, "sequence %d outside 0..%d", seq, c->batch - 1);
  LayerState& L = c->L[layer];
  const int64_t m = seq_main(L, seq), r = seq_ring(L, seq);
  if (total_len < 0 || total_len > m + r)
    return fail(KVQ_ERR_INVALID_ARG, "cannot truncate %lld tokens to %lld", (long long)(m + r),
                (long long)total_len);
  if (total_len >= m)
    set_counts(c, L, seq, 1, m, total_len - m);
  else
    set_counts(c, L, seq, 1, total_len, 0);
  return ok();
}

int kvq_get_lengths(kvq_cache_t c, int layer, int64_t* len_main, int64_t* len_ring) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (len_main) *len_main = c->L[layer].len_main;
  if (len_ring) *len_ring = c->L[layer].len_ring;
  return ok();
}

int kvq_get_seq_lengths(kvq_cache_t c, int layer, int seq, int64_t* len_main, int64_t* len_ring) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (seq < 0 || seq >= c->batch) return fail(KVQ_ERR_INVALID_ARG, "sequence %d outside 0..%d", seq, c->batch - 1);
  if (len_main) *len_main = seq_main(c->L[layer], seq);
  if (len_ring) *len_ring = seq_ring(c->L[layer], seq);
  return ok();
}

int kvq_seq_reset(kvq_cache_t c, int seq, void* stream) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "null cache");
  if (seq < 0 || seq >= c->batch) return fail(KVQ_ERR_INVALID_ARG, "sequence %d outside 0..%d", seq, c->batch - 1);
  if (c->renewal) return fail(KVQ_ERR_UNSUPPORTED, "scale renewal needs equal sequence lengths");
  int st = release_pages(c, seq, S(stream));
  if (st != KVQ_OK) return st;
  for (int l = 0; l < c->layers; ++l) set_counts(c, c->L[l], seq, 1, 0, 0);
  return ok();
}

int kvq_get_block_table(kvq_cache_t c, int seq, int32_t* pages, int64_t n) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "null cache");
  if (!c->page_tokens) return fail(KVQ_ERR_INVALID_ARG, "not a paged cache");
  if (seq < 0 || seq >= c->batch) return fail(KVQ_ERR_INVALID_ARG, "sequence %d outside 0..%d", seq, c->batch - 1);
  if (n < 0 || (n > 0 && !pages)) return fail(KVQ_ERR_INVALID_ARG, "bad output array");
  for (int64_t j = 0; j < n; ++j)
    pages[j] = j < c->max_pages ? c->host_pages[(int64_t)seq * c->max_pages + j] : -1;
  return ok();
}

int kvq_page_granularity(int format) {
  if (format != KVQ_NVFP4 && format != KVQ_INT4 && format != KVQ_FP8 && format != KVQ_INT8 &&
      format != KVQ_INT2)
    return 0;
  return attn_page_granularity(format);
}

int kvq_get_layout(kvq_cache_t c, int layer, int kv, struct kvq_layout* out) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if ((kv != 0 && kv != 1) || !out) return fail(KVQ_ERR_INVALID_ARG, "bad kv or null output");
  const LayerState& L = c->L[layer];
  out->codes = L.kv[kv].codes;
  out->meta = L.kv[kv].meta;
  out->ring = L.kv[kv].ring;
  out->global_scale = int_affine(c->format) ? nullptr : c->renewal ? L.seg_scale[kv] : L.gscale[kv];
  out->scale_renewal = c->renewal;
  out->compact_meta = c->compact;
  out->scale_segments = c->nseg;
  out->capacity = c->capacity;
  out->code_bytes = c->code_bytes;
  out->meta_bytes = c->meta_bytes;
  out->page_tokens = c->page_tokens;
  out->num_pages = (int32_t)c->num_pages;
  out->max_pages = (int32_t)c->max_pages;
  out->reserved = 0;
  out->pages = c->dev_pages;
  return ok();
}

int kvq_device_status(kvq_cache_t c, void* stream, int* device_error) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "null cache");
  int h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, c->dev_status, sizeof(int), cudaMemcpyDeviceToHost, S(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(S(stream));
  if (e != cudaSuccess) return cuda_fail(e, "device status read");
  if (device_error) *device_error = h;
  if (h != 0) {
    e = cudaMemsetAsync(c->dev_status, 0, sizeof(int), S(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(S(stream));
    if (e != cudaSuccess) return cuda_fail(e, "device status clear");
    return fail(KVQ_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded wait (code %d)", h);
  }
  return ok();
}

const char* kvq_last_error(void) { return g_err; }

}  // extern "C"
