"""B200 quantized KV cache: Python binding of libkvq.so.

Argument marshalling only: every step of the path (calibration, quantize,
ring flush, split-K decode attention, combine, dequantize) runs in the CUDA
kernels of libkvq.so.  PyTorch provides device memory and streams.  There is
no CPU fallback: if the library cannot be loaded, every call raises.

The functions below carry the names of the C entry points in include/kvq.h
and take torch tensors or raw integers; ``KVCache`` wraps them with the
buffer allocation done by torch.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

NVFP4, INT4, FP8, INT8, INT2 = 1, 2, 3, 4, 5
FORMATS = {"nvfp4": NVFP4, "int4": INT4, "fp8": FP8, "int8": INT8, "int2": INT2}
INT_AFFINE = (INT4, INT8, INT2)

KVQ_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "CAPACITY", 3: "WORKSPACE", 4: "CUDA",
                5: "DEVICE_TIMEOUT", 6: "UNSUPPORTED", 7: "EMPTY"}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_build", "libkvq.so")
_lib = None


class KVQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s (%d): %s" % (STATUS_NAMES.get(status, "?"), status, message))
        self.status = status


class kvq_layout(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("meta", ctypes.c_void_p), ("ring", ctypes.c_void_p),
                ("global_scale", ctypes.c_void_p), ("capacity", ctypes.c_int64),
                ("code_bytes", ctypes.c_int32), ("meta_bytes", ctypes.c_int32),
                ("compact_meta", ctypes.c_int32), ("scale_renewal", ctypes.c_int32),
                ("scale_segments", ctypes.c_int32), ("page_tokens", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("max_pages", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("pages", ctypes.c_void_p)]


class kvq_options(ctypes.Structure):
    _fields_ = [("scale_renewal", ctypes.c_int32), ("compact_meta", ctypes.c_int32),
                ("page_tokens", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 4)]


EXPORTS = ["kvq_cache_bytes", "kvq_cache_create", "kvq_cache_destroy", "kvq_cache_reset",
           "kvq_append", "kvq_flush_residual", "kvq_workspace_bytes", "kvq_decode_attention",
           "kvq_dequantize", "kvq_truncate", "kvq_get_lengths", "kvq_get_layout",
           "kvq_device_status", "kvq_last_error", "kvq_decode_attention_noalloc",
           "kvq_decode_step", "kvq_decode_attention_lse", "kvq_combine_partials",
           "kvq_cache_bytes_ex", "kvq_cache_create_ex", "kvq_append_seq", "kvq_seq_reset",
           "kvq_get_seq_lengths", "kvq_truncate_seq", "kvq_dequantize_seq", "kvq_get_block_table",
           "kvq_page_granularity"]


def load_library(path: Optional[str] = None):
    """Load libkvq.so (built by quantized_kv_cache_13_b200/build.py)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError("libkvq.so not found at %s: run `python -m quantized_kv_cache_13_b200.build`"
                           % p)
    L = ctypes.CDLL(p)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    L.kvq_cache_bytes.restype = sz
    L.kvq_cache_bytes.argtypes = [i32, i32, i32, i32, i32, i64, i32, i32]
    L.kvq_cache_create.restype = i32
    L.kvq_cache_create.argtypes = [ctypes.POINTER(vp), i32, i32, i32, i32, i32, i64, i32, i32, vp,
                                   sz, ctypes.POINTER(ctypes.c_float)]
    L.kvq_cache_bytes_ex.restype = sz
    L.kvq_cache_bytes_ex.argtypes = [i32, i32, i32, i32, i32, i64, i32, i32, ctypes.POINTER(kvq_options)]
    L.kvq_cache_create_ex.restype = i32
    L.kvq_cache_create_ex.argtypes = [ctypes.POINTER(vp), i32, i32, i32, i32, i32, i64, i32, i32, vp,
                                      sz, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(kvq_options)]
    L.kvq_cache_destroy.restype = i32
    L.kvq_cache_destroy.argtypes = [vp]
    L.kvq_cache_reset.restype = i32
    L.kvq_cache_reset.argtypes = [vp, vp]
    L.kvq_append.restype = i32
    L.kvq_append.argtypes = [vp, i32, vp, vp, i64, vp]
    L.kvq_flush_residual.restype = i32
    L.kvq_flush_residual.argtypes = [vp, i32, vp]
    L.kvq_workspace_bytes.restype = sz
    L.kvq_workspace_bytes.argtypes = [vp, i32]
    L.kvq_decode_attention.restype = i32
    L.kvq_decode_attention.argtypes = [vp, i32, vp, i32, ctypes.c_float, vp, vp, sz, vp]
    L.kvq_dequantize.restype = i32
    L.kvq_dequantize.argtypes = [vp, i32, i32, i64, i64, vp, vp]
    L.kvq_truncate.restype = i32
    L.kvq_truncate.argtypes = [vp, i32, i64]
    L.kvq_get_lengths.restype = i32
    L.kvq_get_lengths.argtypes = [vp, i32, ctypes.POINTER(i64), ctypes.POINTER(i64)]
    L.kvq_get_layout.restype = i32
    L.kvq_get_layout.argtypes = [vp, i32, i32, ctypes.POINTER(kvq_layout)]
    L.kvq_device_status.restype = i32
    L.kvq_device_status.argtypes = [vp, vp, ctypes.POINTER(i32)]
    L.kvq_decode_step.restype = i32
    L.kvq_decode_step.argtypes = [vp, i32, vp, vp, vp, i32, ctypes.c_float, vp, vp, sz, vp]
    L.kvq_decode_attention_noalloc.restype = i32
    L.kvq_decode_attention_noalloc.argtypes = [vp, i32, vp, i32, ctypes.c_float, vp, vp]
    L.kvq_decode_attention_lse.restype = i32
    L.kvq_decode_attention_lse.argtypes = [vp, i32, vp, i32, ctypes.c_float, vp, vp, vp, sz, vp]
    L.kvq_combine_partials.restype = i32
    L.kvq_combine_partials.argtypes = [i32, i64, i32, vp, i64, vp, i64, vp, vp, vp]
    L.kvq_append_seq.restype = i32
    L.kvq_append_seq.argtypes = [vp, i32, i32, vp, vp, i64, vp]
    L.kvq_seq_reset.restype = i32
    L.kvq_seq_reset.argtypes = [vp, i32, vp]
    L.kvq_get_seq_lengths.restype = i32
    L.kvq_get_seq_lengths.argtypes = [vp, i32, i32, ctypes.POINTER(i64), ctypes.POINTER(i64)]
    L.kvq_truncate_seq.restype = i32
    L.kvq_truncate_seq.argtypes = [vp, i32, i32, i64]
    L.kvq_dequantize_seq.restype = i32
    L.kvq_dequantize_seq.argtypes = [vp, i32, i32, i32, i64, i64, vp, vp]
    L.kvq_get_block_table.restype = i32
    L.kvq_get_block_table.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_int32), i64]
    L.kvq_page_granularity.restype = i32
    L.kvq_page_granularity.argtypes = [i32]
    L.kvq_last_error.restype = ctypes.c_char_p
    L.kvq_last_error.argtypes = []
    if path is None:
        _lib = L
    return L


def lib():
    return load_library()


def _check(status: int):
    if status != KVQ_OK:
        raise KVQError(status, lib().kvq_last_error().decode())


def _stream_ptr(stream=None) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _ptr(t) -> int:
    return int(t.data_ptr()) if t is not None else 0


# --------------------------------------------------------------------------
# C entry points, same names, tensors in and status checked.
# --------------------------------------------------------------------------

def _options(scale_renewal: int = 0, compact_meta: bool = False, page_tokens: int = 0,
             num_pages: int = 0):
    if not scale_renewal and not compact_meta and not page_tokens:
        return None
    o = kvq_options()
    o.scale_renewal = scale_renewal
    o.compact_meta = 1 if compact_meta else 0
    o.page_tokens = page_tokens
    o.num_pages = num_pages
    return ctypes.byref(o)


def kvq_cache_bytes(fmt: int, layers: int, batch: int, kv_heads: int, head_dim: int, max_len: int,
                    group_size: int, residual_length: int, scale_renewal: int = 0,
                    compact_meta: bool = False, page_tokens: int = 0, num_pages: int = 0) -> int:
    return int(lib().kvq_cache_bytes_ex(fmt, layers, batch, kv_heads, head_dim, max_len, group_size,
                                        residual_length,
                                        _options(scale_renewal, compact_meta, page_tokens, num_pages)))


def kvq_cache_create(fmt, layers, batch, kv_heads, head_dim, max_len, group_size, residual_length,
                     device_buf, global_scales=None, scale_renewal: int = 0,
                     compact_meta: bool = False, page_tokens: int = 0, num_pages: int = 0) -> int:
    """kvq_cache_create_ex (no options: the same as kvq_cache_create)."""
    h = ctypes.c_void_p()
    gs = None
    if global_scales is not None:
        flat = [float(x) for row in global_scales for x in row]
        gs = (ctypes.c_float * len(flat))(*flat)
    _check(lib().kvq_cache_create_ex(ctypes.byref(h), fmt, layers, batch, kv_heads, head_dim, max_len,
                                     group_size, residual_length, _ptr(device_buf),
                                     device_buf.numel() * device_buf.element_size(), gs,
                                     _options(scale_renewal, compact_meta, page_tokens, num_pages)))
    return h.value


def kvq_cache_destroy(handle: int):
    _check(lib().kvq_cache_destroy(handle))


def kvq_cache_reset(handle: int, stream=None):
    _check(lib().kvq_cache_reset(handle, _stream_ptr(stream)))


def kvq_append(handle: int, layer: int, k, v, stream=None):
    n = k.shape[2]
    _check(lib().kvq_append(handle, layer, _ptr(k), _ptr(v), n, _stream_ptr(stream)))


def kvq_flush_residual(handle: int, layer: int, stream=None):
    _check(lib().kvq_flush_residual(handle, layer, _stream_ptr(stream)))


def kvq_workspace_bytes(handle: int, q_heads: int) -> int:
    return int(lib().kvq_workspace_bytes(handle, q_heads))


def kvq_decode_attention(handle: int, layer: int, q, out, workspace, softmax_scale: float = 0.0,
                         stream=None):
    _check(lib().kvq_decode_attention(handle, layer, _ptr(q), q.shape[1], softmax_scale, _ptr(out),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream_ptr(stream)))


def kvq_decode_attention_lse(handle: int, layer: int, q, out, lse, workspace,
                             softmax_scale: float = 0.0, stream=None):
    """Decode attention plus the per-head log-sum-exp of the scores (f32
    [B, Hq]), for merging parts of a sequence held by several caches."""
    _check(lib().kvq_decode_attention_lse(handle, layer, _ptr(q), q.shape[1], softmax_scale, _ptr(out),
                                          _ptr(lse), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          _stream_ptr(stream)))


def kvq_combine_partials(o_parts, lse_parts, out, lse_out=None, stream=None):
    """Log-sum-exp merge of attention over disjoint parts: o_parts f32 [n, rows,
    D] (or any tensor whose parts are equally strided), lse_parts f32 [n, rows]
    -> out f32 [rows, D] (and lse_out f32 [rows] if given)."""
    n = o_parts.shape[0]
    rows = lse_parts.shape[1]
    D = o_parts.shape[-1]
    if o_parts.dim() != 3 or o_parts.shape[1] != rows or o_parts.stride(2) != 1 or o_parts.stride(1) != D:
        raise ValueError("o_parts must be [n, rows, D] with contiguous rows")
    if lse_parts.stride(1) != 1:
        raise ValueError("lse_parts must be [n, rows] with contiguous rows")
    _check(lib().kvq_combine_partials(n, rows, o_parts.shape[-1], _ptr(o_parts), o_parts.stride(0),
                                      _ptr(lse_parts), lse_parts.stride(0), _ptr(out),
                                      _ptr(lse_out) if lse_out is not None else None,
                                      _stream_ptr(stream)))


def kvq_decode_step(handle: int, layer: int, k, v, q, out, workspace, softmax_scale: float = 0.0,
                    stream=None):
    """Append one token (k, v: [B, Hkv, 1, D] bf16) and run decode attention
    over the cache including it, in one launch."""
    _check(lib().kvq_decode_step(handle, layer, _ptr(k), _ptr(v), _ptr(q), q.shape[1], softmax_scale,
                                 _ptr(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream_ptr(stream)))


def kvq_decode_attention_noalloc(handle: int, layer: int, q, out, softmax_scale: float = 0.0,
                                 stream=None):
    """Decode attention with the library's built-in scratch instead of a
    caller workspace, for callers that cannot allocate device memory."""
    _check(lib().kvq_decode_attention_noalloc(handle, layer, _ptr(q), q.shape[1], softmax_scale,
                                              _ptr(out), _stream_ptr(stream)))


def kvq_dequantize(handle: int, layer: int, kv: int, start: int, n: int, out, stream=None):
    _check(lib().kvq_dequantize(handle, layer, kv, start, n, _ptr(out), _stream_ptr(stream)))


def kvq_truncate(handle: int, layer: int, total_len: int):
    _check(lib().kvq_truncate(handle, layer, total_len))


def kvq_get_lengths(handle: int, layer: int) -> Tuple[int, int]:
    a, b = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().kvq_get_lengths(handle, layer, ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def kvq_append_seq(handle: int, layer: int, seq: int, k, v, stream=None):
    """Append n tokens (k, v: [Hkv, n, D] bf16) to sequence `seq` only."""
    _check(lib().kvq_append_seq(handle, layer, seq, _ptr(k), _ptr(v), k.shape[-2], _stream_ptr(stream)))


def kvq_seq_reset(handle: int, seq: int, stream=None):
    _check(lib().kvq_seq_reset(handle, seq, _stream_ptr(stream)))


def kvq_get_seq_lengths(handle: int, layer: int, seq: int) -> Tuple[int, int]:
    a, b = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().kvq_get_seq_lengths(handle, layer, seq, ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def kvq_truncate_seq(handle: int, layer: int, seq: int, total_len: int):
    _check(lib().kvq_truncate_seq(handle, layer, seq, total_len))


def kvq_dequantize_seq(handle: int, layer: int, kv: int, seq: int, start: int, n: int, out, stream=None):
    _check(lib().kvq_dequantize_seq(handle, layer, kv, seq, start, n, _ptr(out), _stream_ptr(stream)))


def kvq_get_block_table(handle: int, seq: int, n: int):
    arr = (ctypes.c_int32 * max(n, 1))()
    _check(lib().kvq_get_block_table(handle, seq, arr, n))
    return list(arr)[:n]


def kvq_page_granularity(fmt: int) -> int:
    return int(lib().kvq_page_granularity(fmt))


def kvq_get_layout(handle: int, layer: int, kv: int) -> kvq_layout:
    out = kvq_layout()
    _check(lib().kvq_get_layout(handle, layer, kv, ctypes.byref(out)))
    return out


def kvq_device_status(handle: int, stream=None) -> int:
    code = ctypes.c_int()
    st = lib().kvq_device_status(handle, _stream_ptr(stream), ctypes.byref(code))
    if st not in (KVQ_OK, 5):
        _check(st)
    return code.value


# --------------------------------------------------------------------------
# Convenience wrapper owning torch buffers.
# --------------------------------------------------------------------------

class KVCache:
    """A quantized KV cache for `layers` attention layers on one GPU.

    fmt: NVFP4 | INT4 | FP8 | INT8 | INT2 (or "nvfp4" | "int4" | "fp8" |
    "int8" | "int2").  INT2 decode attention needs group_size 64.
    global_scales: None (calibrate each layer from its first append) or a
    [layers][2] list of per-tensor K/V scales (1.0 = the *_cast variants).
    """

    def __init__(self, fmt, layers: int, batch: int, kv_heads: int, max_len: int,
                 head_dim: int = 128, group_size: int = 0, residual_length: int = 0,
                 global_scales=None, device=None, scale_renewal: int = 0,
                 compact_meta: bool = False, page_tokens: int = 0, num_pages: int = 0):
        import torch
        self.fmt = FORMATS.get(fmt, fmt) if isinstance(fmt, str) else fmt
        if self.fmt in INT_AFFINE and group_size == 0:
            group_size = 64
        self.layers, self.batch, self.kv_heads, self.head_dim = layers, batch, kv_heads, head_dim
        self.max_len, self.group_size, self.residual_length = max_len, group_size, residual_length
        self.device = torch.device(device if device is not None else "cuda")
        self.scale_renewal = scale_renewal
        self.compact_meta = compact_meta
        self.page_tokens, self.num_pages = page_tokens, num_pages
        nbytes = kvq_cache_bytes(self.fmt, layers, batch, kv_heads, head_dim, max_len, group_size,
                                 residual_length, scale_renewal, compact_meta, page_tokens, num_pages)
        if nbytes == 0:
            # reproduce the error message through create's checks
            raise KVQError(1, "invalid cache arguments")
        self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.handle = kvq_cache_create(self.fmt, layers, batch, kv_heads, head_dim, max_len,
                                       group_size, residual_length, self.buffer, global_scales,
                                       scale_renewal, compact_meta, page_tokens, num_pages)
        self._ws = {}

    def __del__(self):
        h = getattr(self, "handle", None)
        if h:
            try:
                kvq_cache_destroy(h)
            except Exception:
                pass
            self.handle = None

    def append(self, layer: int, k, v, stream=None):
        kvq_append(self.handle, layer, k, v, stream)

    def flush_residual(self, layer: int, stream=None):
        kvq_flush_residual(self.handle, layer, stream)

    def reset(self, stream=None):
        kvq_cache_reset(self.handle, stream)

    def truncate(self, layer: int, total_len: int):
        kvq_truncate(self.handle, layer, total_len)

    def lengths(self, layer: int) -> Tuple[int, int]:
        """(main, ring) token counts of the layer (of sequence 0 in a ragged batch)."""
        return kvq_get_lengths(self.handle, layer)

    # -- sequences of different lengths ------------------------------------
    def append_seq(self, layer: int, seq: int, k, v, stream=None):
        kvq_append_seq(self.handle, layer, seq, k, v, stream)

    def seq_reset(self, seq: int, stream=None):
        kvq_seq_reset(self.handle, seq, stream)

    def seq_lengths(self, layer: int, seq: int) -> Tuple[int, int]:
        return kvq_get_seq_lengths(self.handle, layer, seq)

    def truncate_seq(self, layer: int, seq: int, total_len: int):
        kvq_truncate_seq(self.handle, layer, seq, total_len)

    def dequantize_seq(self, layer: int, kv: int, seq: int, start: int, n: int, stream=None):
        import torch
        out = torch.empty((self.kv_heads, n, self.head_dim), dtype=torch.float32, device=self.device)
        kvq_dequantize_seq(self.handle, layer, kv, seq, start, n, out, stream)
        return out

    def block_table(self, seq: int):
        """Page ids of sequence `seq` (paged caches; -1: no page)."""
        return kvq_get_block_table(self.handle, seq, self.layout(0, 0).max_pages)

    def seq_rows(self, seq: int, n: int):
        """Plane rows (int64 [H, n]) of tokens [0, n) of sequence `seq`, for
        indexing the flattened codes / meta planes of raw()."""
        import torch
        H = self.kv_heads
        t = torch.arange(n, dtype=torch.int64)
        h = torch.arange(H, dtype=torch.int64)[:, None]
        lay = self.layout(0, 0)
        if not lay.page_tokens:
            return ((seq * H + h) * lay.capacity + t[None, :]).to(self.device)
        P = lay.page_tokens
        table = torch.tensor(self.block_table(seq), dtype=torch.int64)
        page = table[t // P]
        return ((page[None, :] * H + h) * P + (t % P)[None, :]).to(self.device)

    def seq_raw(self, layer: int, kv: int, seq: int, n: int):
        """Sequence `seq`'s main-cache planes of tokens [0, n), gathered from
        contiguous or paged storage: dict with 'codes' [1, H, n, code_bytes]
        and 'meta' shaped as in raw() with a batch of 1."""
        lay = self.layout(layer, kv)
        rows = self.seq_rows(seq, n)
        raw = self.raw(layer, kv)
        out = {}
        for name in ("codes", "meta", "meta_s16", "meta_z8"):
            if name in raw:
                x = raw[name]
                flat = x.reshape(-1, *x.shape[3:])
                out[name] = flat[rows].unsqueeze(0)
        return out

    def workspace(self, q_heads: int):
        import torch
        ws = self._ws.get(q_heads)
        if ws is None:
            ws = torch.empty(kvq_workspace_bytes(self.handle, q_heads), dtype=torch.uint8,
                             device=self.device)
            self._ws[q_heads] = ws
        return ws

    def decode_attention(self, layer: int, q, out=None, softmax_scale: float = 0.0, stream=None):
        import torch
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        kvq_decode_attention(self.handle, layer, q, out, self.workspace(q.shape[1]), softmax_scale,
                             stream)
        return out

    def decode_attention_lse(self, layer: int, q, out=None, lse=None, softmax_scale: float = 0.0,
                             stream=None):
        """(out f32 [B, Hq, D], lse f32 [B, Hq]): attention over this cache and
        the log-sum-exp of the scores (0 and -inf for an empty layer)."""
        import torch
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        if lse is None:
            lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
        kvq_decode_attention_lse(self.handle, layer, q, out, lse, self.workspace(q.shape[1]),
                                 softmax_scale, stream)
        return out, lse

    def decode_step(self, layer: int, k, v, q, out=None, softmax_scale: float = 0.0, stream=None):
        """Append one token and attend, in one launch (kvq_decode_step)."""
        import torch
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        kvq_decode_step(self.handle, layer, k, v, q, out, self.workspace(q.shape[1]), softmax_scale,
                        stream)
        return out

    def dequantize(self, layer: int, kv: int, start: int, n: int, stream=None):
        import torch
        out = torch.empty((self.batch, self.kv_heads, n, self.head_dim), dtype=torch.float32,
                          device=self.device)
        kvq_dequantize(self.handle, layer, kv, start, n, out, stream)
        return out

    def layout(self, layer: int, kv: int) -> kvq_layout:
        return kvq_get_layout(self.handle, layer, kv)

    def raw(self, layer: int, kv: int):
        """Views of the device planes of (layer, kv): dict with 'codes'
        [B,H,cap,code_bytes] u8, 'meta' (NVFP4 u8 [..,16th], INT4/INT8/INT2 int32
        [..,groups,2]), 'ring' bf16 [B,H,R,D], 'scale' f32 [1]."""
        lay = self.layout(layer, kv)
        base = self.buffer.data_ptr()
        B, H, cap = self.batch, self.kv_heads, lay.capacity
        if lay.page_tokens:   # pools [num_pages][H][page_tokens][bytes]
            B = lay.num_pages

        def view(ptr, nbytes):
            off = ptr - base
            return self.buffer[off:off + nbytes]

        out = {"codes": view(lay.codes, B * H * cap * lay.code_bytes).view(B, H, cap, lay.code_bytes)}
        if lay.meta:
            m = view(lay.meta, B * H * cap * lay.meta_bytes)
            if lay.compact_meta:
                # {f16 S0, f16 S1, Z0, Z1} per token: i8 Z (INT4, INT2; 2 zero
                # bytes) or i16 Z (INT8)
                import torch
                m = m.view(B, H, cap, 8)
                out["meta_s16"] = m[..., :4].contiguous().view(torch.float16)
                if self.fmt == INT8:
                    out["meta_z16"] = m[..., 4:8].contiguous().view(torch.int16)
                else:
                    out["meta_z8"] = m[..., 4:6].contiguous().view(torch.int8)
                out["meta"] = m
            elif self.fmt in INT_AFFINE:
                import torch
                out["meta"] = m.view(torch.int32).view(B, H, cap, lay.meta_bytes // 8, 2)
            else:
                out["meta"] = m.view(B, H, cap, lay.meta_bytes)
        if lay.ring:
            import torch
            R = self.residual_length
            out["ring"] = view(lay.ring, self.batch * H * R * self.head_dim * 2).view(torch.bfloat16).view(
                self.batch, H, R, self.head_dim)
        if lay.global_scale:
            import torch
            # one f32 per tensor, or one per scale segment under scale renewal
            n = lay.scale_segments if lay.scale_renewal else 1
            out["scale"] = view(lay.global_scale, 4 * n).view(torch.float32)
        return out

    def canonical_codes(self, layer: int, kv: int, start: int = 0, n: int = None):
        """Main-cache codes of tokens [start, start+n) as [B, H, n, code_bytes]
        uint8 in token-major order (NVFP4/INT4: element 2i in the low nibble
        of byte i).  The V planes are stored in the decode kernel's order and
        this undoes it: NVFP4 V is pair-interleaved (byte d of the row of
        tokens 2p, 2p+1 holds dim d of token 2p in the low nibble and of token
        2p+1 in the high nibble); INT4 V rows are dim-permuted (byte 8r + m
        holds dim 16m + r in the low nibble and dim 16m + r + 8 in the high
        nibble); INT8 V rows are dim-permuted (byte 16r + 2m + h holds dim
        16m + r + 8h); INT2 V rows are dim-permuted (byte 4r + m/2 holds dim
        16m + r + 8h at bits 2(2(m%2) + h)).  Inspection helper (plain torch indexing), not part of
        the decode path."""
        if n is None:
            n = self.lengths(layer)[0] - start
        return self._canonical(self.raw(layer, kv)["codes"], kv, start, n)

    def seq_canonical_codes(self, layer: int, kv: int, seq: int, n: int):
        """canonical_codes of tokens [0, n) of sequence `seq` ([1, H, n, bytes]),
        from contiguous or paged storage (n even for an NVFP4 V plane, or the
        sequence's last token: pairs are whole)."""
        n_rows = n + (n & 1) if (self.fmt == NVFP4 and kv == 1) else n
        return self._canonical(self.seq_raw(layer, kv, seq, n_rows)["codes"], kv, 0, n)

    def _canonical(self, codes, kv: int, start: int, n: int):
        import torch
        if self.fmt == INT8 and kv == 1:
            c = codes[:, :, start:start + n]
            d = torch.arange(self.head_dim, device=c.device)
            byte_of = 16 * (d % 8) + 2 * (d // 16) + (d // 8) % 2
            return c[..., byte_of]
        if self.fmt == INT2 and kv == 1:
            return int2_v_canonical(codes[:, :, start:start + n])
        if self.fmt == INT4 and kv == 1:
            c = codes[:, :, start:start + n]
            nib = torch.stack([c & 0xF, c >> 4], dim=-1).reshape(*c.shape[:3], 2 * c.shape[3])
            # nibble 2b + h of the permuted row is dim 16 (b % 8) + b // 8 + 8 h
            b = torch.arange(c.shape[3], device=c.device)
            dim_of = torch.stack([16 * (b % 8) + b // 8, 16 * (b % 8) + b // 8 + 8], dim=-1).reshape(-1)
            dims = torch.empty_like(nib)
            dims[..., dim_of] = nib
            return dims[..., 0::2] | (dims[..., 1::2] << 4)
        if not (self.fmt == NVFP4 and kv == 1):
            return codes[:, :, start:start + n]
        p0, p1 = start // 2, (start + n + 1) // 2
        B, H = codes.shape[0], codes.shape[1]
        P = codes[:, :, 2 * p0:2 * p1].reshape(B, H, p1 - p0, self.head_dim)
        tok = torch.stack([P & 0xF, P >> 4], dim=3).reshape(B, H, 2 * (p1 - p0), self.head_dim)
        canon = tok[..., 0::2] | (tok[..., 1::2] << 4)
        off = start - 2 * p0
        return canon[:, :, off:off + n]

    def device_status(self, stream=None) -> int:
        return kvq_device_status(self.handle, stream)


def int2_v_canonical(c):
    """INT2 V rows [..., 32] uint8 in the permuted order (dim d = 16m + 8h + r
    in byte 4r + m/2 at bits 2(2(m%2) + h)) -> natural packing (dim d in byte
    d/4 at bits 2(d%4)).  Plain torch indexing, for inspection and tests."""
    import torch
    d = torch.arange(4 * c.shape[-1], device=c.device)
    byte_of = 4 * (d % 8) + d // 32
    shift = (2 * ((d // 8) % 4)).to(torch.uint8)
    vals = torch.bitwise_right_shift(c[..., byte_of], shift) & 3
    vals = vals.reshape(*c.shape[:-1], c.shape[-1], 4)
    return vals[..., 0] | (vals[..., 1] << 2) | (vals[..., 2] << 4) | (vals[..., 3] << 6)
