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
};

// Check the arguments and compute the layout:
//   [header: per layer {gscale K, gscale V, amax K, amax V} x f32/u32, status
//    word, per (layer, batch x kv_head) attention completion counters]
//   then per layer, per K/V: codes plane, meta plane, ring plane,
// every plane 256-byte aligned.
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
    if (format != KVQ_INT4 || g->group != 64)
      return fail(KVQ_ERR_INVALID_ARG, "compact group metadata is implemented for INT4 with groups of 64");
    g->compact = 1;
    g->meta_bytes = 8;   // {f16 S0, f16 S1, i8 Z0, i8 Z1, 0, 0}
  }
  g->counters_off = align_up((size_t)layers * 4 * sizeof(float) + sizeof(int), 16);
  g->seg_off = align_up(g->counters_off + (size_t)layers * bh * sizeof(int), 16);
  g->header = align_up(g->seg_off + (size_t)layers * 2 * g->nseg * 8, 256);
  g->codes = align_up(bh * g->cap * g->code_bytes, 256);
  g->meta = align_up(bh * g->cap * g->meta_bytes, 256);
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
// Caches the decode attention kernel implements (INT2: groups of 64 only).
inline bool has_attention(int format, int group) { return format != KVQ_INT2 || group == 64; }

int check_cache(kvq_cache_t c, int layer) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "null cache");
  if (layer < 0 || layer >= c->layers)
    return fail(KVQ_ERR_INVALID_ARG, "layer %d outside 0..%d", layer, c->layers - 1);
  return KVQ_OK;
}

// Quantize n tokens from a bf16 source into the main cache of `layer`.
int quantize_into_main(kvq_cache_t c, int layer, const uint16_t* sk, const uint16_t* sv,
                       int64_t src_bh_stride, int64_t src_tok0, int64_t n, bool calibrate,
                       cudaStream_t stream) {
  LayerState& L = c->L[layer];
  QuantArgs a{};
  a.src[0] = sk;
  a.src[1] = sv;
  a.src_bh_stride = src_bh_stride;
  a.src_tok0 = src_tok0;
  a.dst[0] = L.kv[0];
  a.dst[1] = L.kv[1];
  a.dst_tok0 = L.len_main;
  a.n = n;
  a.bh = c->batch * c->kv_heads;
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
  cudaError_t e = launch_quantize(c->format, a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  L.len_main += n;
  return KVQ_OK;
}

int flush_ring(kvq_cache_t c, int layer, cudaStream_t stream) {
  LayerState& L = c->L[layer];
  if (L.len_ring == 0) return KVQ_OK;
  const int64_t r = L.len_ring;
  int st = quantize_into_main(c, layer, L.kv[0].ring, L.kv[1].ring, (int64_t)c->R * c->head_dim, 0,
                              r, false, stream);
  if (st != KVQ_OK) return st;
  L.len_ring = 0;
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
  c->device = attr.device;
  if (const char* env = getenv("KVQ_CTAS")) c->ctas_env = atoi(env);
  // unit-start weight in tiles: about the time of a query load plus a merge
  // (measured optima on B200: 2 of NVFP4's 384-token tiles, 3 of INT4's
  // 256-token tiles; FP8's 128-token tiles take 4)
  c->split_wb = format == KVQ_NVFP4 ? 2 : (format == KVQ_INT4 || format == KVQ_INT2) ? 3 : 4;
  if (const char* env = getenv("KVQ_UNIT_WEIGHT")) c->split_wb = atoi(env) < 0 ? 0 : atoi(env);

  uint8_t* base = static_cast<uint8_t*>(device_buf);
  float* hdr = reinterpret_cast<float*>(base);
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
    delete[] c->L;
    delete c;
    return cuda_fail(e, "cache initialisation");
  }
  *out = c;
  return ok();
}

int kvq_cache_destroy(kvq_cache_t c) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "null cache");
  delete[] c->L;
  delete c;
  return ok();
}

int kvq_cache_reset(kvq_cache_t c, void* stream) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "null cache");
  for (int l = 0; l < c->layers; ++l) {
    LayerState& L = c->L[l];
    L.len_main = L.len_ring = 0;
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
  if (L.len_main + L.len_ring + n > c->max_len)
    return fail(KVQ_ERR_CAPACITY, "append of %lld tokens exceeds max_len %lld (holding %lld)",
                (long long)n, (long long)c->max_len, (long long)(L.len_main + L.len_ring));
  cudaStream_t s = S(stream);
  const uint16_t* sk = static_cast<const uint16_t*>(k);
  const uint16_t* sv = static_cast<const uint16_t*>(v);
  const int64_t bh_stride = n * c->head_dim;

  if (c->renewal) {
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
  if (c->R == 0) {
    bool calibrate = false;
    if (!int_affine(c->format) && !(L.calibrated[0] && L.calibrated[1])) {
      const int64_t elems = (int64_t)c->batch * c->kv_heads * n * c->head_dim;
      cudaError_t e = launch_amax(sk, sv, elems, L.amax[0], L.amax[1], s);
      if (e != cudaSuccess) return cuda_fail(e, "amax launch");
      calibrate = true;
    }
    st = quantize_into_main(c, layer, sk, sv, bh_stride, 0, n, calibrate, s);
    if (st != KVQ_OK) return st;
    if (calibrate) L.calibrated[0] = L.calibrated[1] = true;
    return ok();
  }

  // With a residual ring: identical to appending token by token.  NVFP4 /
  // FP8 still calibrate their per-tensor scales from the first append,
  // before its tokens enter the ring.
  if (!int_affine(c->format) && !(L.calibrated[0] && L.calibrated[1])) {
    const int64_t elems = (int64_t)c->batch * c->kv_heads * n * c->head_dim;
    cudaError_t e = launch_amax(sk, sv, elems, L.amax[0], L.amax[1], s);
    if (e == cudaSuccess)
      e = launch_scale_from_amax(L.amax[0], L.amax[1], L.gscale[0], L.gscale[1],
                                 c->format == KVQ_NVFP4 ? 2688.0f : 448.0f, s);
    if (e != cudaSuccess) return cuda_fail(e, "calibration launch");
    L.calibrated[0] = L.calibrated[1] = true;
  }
  const int bh = c->batch * c->kv_heads;
  int64_t done = 0;
  // 1. top up the ring
  int64_t a = std::min<int64_t>(n, c->R - L.len_ring);
  if (a > 0) {
    cudaError_t e = launch_ring_copy(sk, sv, bh_stride, 0, L.kv[0].ring, L.kv[1].ring, c->R,
                                     L.len_ring, a, bh, s);
    if (e != cudaSuccess) return cuda_fail(e, "ring copy launch");
    L.len_ring += a;
    done = a;
  }
  if (L.len_ring == c->R) {
    st = flush_ring(c, layer, s);
    if (st != KVQ_OK) return st;
  }
  // 2. whole rings straight from the input
  const int64_t whole = ((n - done) / c->R) * c->R;
  if (whole > 0) {
    st = quantize_into_main(c, layer, sk, sv, bh_stride, done, whole, false, s);
    if (st != KVQ_OK) return st;
    done += whole;
  }
  // 3. the remainder goes to the (now empty) ring
  if (done < n) {
    const int64_t rem = n - done;
    cudaError_t e = launch_ring_copy(sk, sv, bh_stride, done, L.kv[0].ring, L.kv[1].ring, c->R,
                                     0, rem, bh, s);
    if (e != cudaSuccess) return cuda_fail(e, "ring copy launch");
    L.len_ring = rem;
  }
  return ok();
}

int kvq_flush_residual(kvq_cache_t c, int layer, void* stream) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (c->R == 0) return ok();
  st = flush_ring(c, layer, S(stream));
  return st == KVQ_OK ? ok() : st;
}

// CTAs the attention kernel can keep resident at once (one wave).
static int resident_ctas(kvq_cache_t c) {
  // attention CTAs resident per SM, per format id (KVQ_NVFP4 .. KVQ_INT2)
  // and kernel variant (NVFP4 / FP8: plain, with a ring, with scale renewal;
  // INT4: compact group metadata)
  static int bps[KVQ_INT2 + 1][4] = {};
  static_assert(KVQ_NVFP4 >= 0 && KVQ_INT4 <= KVQ_INT2 && KVQ_FP8 <= KVQ_INT2 && KVQ_INT8 <= KVQ_INT2,
                "format ids index bps");
  if (!has_attention(c->format, c->group)) return 1;
  const int var = c->compact ? 3 : c->renewal ? 2 : c->R > 0 ? 1 : 0;
  if (bps[c->format][var] == 0)
    bps[c->format][var] = attn_blocks_per_sm(c->format, var == 1, var == 2, var == 3);
  int n = c->sm_count * bps[c->format][var];
  if (c->ctas_env > n) n = c->ctas_env;
  return n < 1 ? 1 : n;
}


size_t kvq_workspace_bytes(kvq_cache_t c, int q_heads) {
  if (!c || q_heads <= 0 || q_heads % c->kv_heads != 0 || !has_attention(c->format, c->group))
    return 0;
  const int G = q_heads / c->kv_heads;
  const size_t units = (size_t)c->batch * c->kv_heads;
  // a unit is touched by at most floor(C / units) + 2 CTAs of a C-CTA grid
  const size_t maxc = (size_t)resident_ctas(c) / units + 2;
  return align_up(units * maxc * G * (kHeadDim + 2) * sizeof(float), 256);
}

}  // extern "C"

namespace {

// Shared by kvq_decode_attention and kvq_decode_step.  new_kind/new_pos/k/v
// describe a token the kernel appends itself (0 = none); the layer's lengths
// must already include it.
int decode_attention_impl(kvq_cache_t c, int layer, const void* q, int q_heads, float softmax_scale,
                          float* out, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                          int new_kind, int64_t new_pos, const void* k_new, const void* v_new,
                          float* lse = nullptr) {
  const LayerState& L = c->L[layer];
  const int G = q_heads / c->kv_heads;
  const int64_t units = (int64_t)c->batch * c->kv_heads;
  const int tile = attn_tile_tokens(c->format);
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
  a.counters = c->counters + (size_t)layer * units;
  a.ctas = (int)C;
  a.tpu = (int)tpu;
  a.maxc = (int)maxc;
  a.wb = (int)wb;
  a.new_kind = new_kind;
  a.new_pos = new_pos;
  a.k_new = static_cast<const uint16_t*>(k_new);
  a.v_new = static_cast<const uint16_t*>(v_new);
  a.dev_status = c->dev_status;
  a.lse = lse;
  a.gseg_k = L.seg_scale[0];
  a.gseg_v = L.seg_scale[1];
  a.seg_amax_k = L.seg_amax[0];
  a.seg_amax_v = L.seg_amax[1];
  a.renewal = c->renewal;
  a.compact = c->compact;
  cudaError_t e = launch_decode_attention(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode attention launch");
  return ok();
}

// Argument checks of the attention calls (nothing is modified).
int check_attention_args(kvq_cache_t c, int layer, const void* q, int q_heads, float* out,
                         void* workspace) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (!has_attention(c->format, c->group))
    return fail(KVQ_ERR_UNSUPPORTED, "decode attention over INT2 is implemented for groups of 64 only");
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
  if (L.len_main + L.len_ring == 0) return fail(KVQ_ERR_EMPTY, "layer %d holds no tokens", layer);
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
  if (L.len_main + L.len_ring == 0) {
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

int kvq_dequantize(kvq_cache_t c, int layer, int kv, int64_t start, int64_t n, float* out,
                   void* stream) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (kv != 0 && kv != 1) return fail(KVQ_ERR_INVALID_ARG, "kv must be 0 (K) or 1 (V)");
  const LayerState& L = c->L[layer];
  if (start < 0 || n < 0 || start + n > L.len_main)
    return fail(KVQ_ERR_INVALID_ARG, "token range [%lld, %lld) outside the main cache (%lld)",
                (long long)start, (long long)(start + n), (long long)L.len_main);
  if (n == 0) return ok();
  if (!out || !aligned16(out)) return fail(KVQ_ERR_INVALID_ARG, "out must be 16-byte aligned");
  cudaError_t e = launch_dequantize(c->format, L.kv[kv], L.gscale[kv], c->capacity, c->group,
                                    c->batch * c->kv_heads, start, n, out,
                                    (c->format == KVQ_NVFP4 || int_affine(c->format)) && kv == 1,
                                    S(stream), L.seg_scale[kv], c->renewal, c->compact != 0);
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return ok();
}

int kvq_truncate(kvq_cache_t c, int layer, int64_t total_len) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  LayerState& L = c->L[layer];
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

int kvq_get_lengths(kvq_cache_t c, int layer, int64_t* len_main, int64_t* len_ring) {
  int st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (len_main) *len_main = c->L[layer].len_main;
  if (len_ring) *len_ring = c->L[layer].len_ring;
  return ok();
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
