"""CPU oracle for the quantized KV-cache hot path.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library (``quantized_kv_cache_13_b200``) and never imports it.

Sources, cited by page title and section:
  [P1] NVFP4 KV-cache article, glsqs.com/news/814573, section 2.1 (NVFP4
       groups of 16 with one FP8 scale; quantize at prefill, dequantize on the
       fly at decode, quantize-and-append each new token).
  [P2] "KV Cache量化实战：Model Optimizer为大模型长上下文省下50%显存",
       m.nxbn.cn/news/90317 (KV size formula and savings table;
       --kv_cache_qformat table: fp8/nvfp4 calibrate a per-tensor amax,
       *_cast use a constant scale).
  [P3] "KV缓存量化技术：提升大模型长文本生成效率", rkmt.cn/news/1711363
       (section 1 per-layer size; section 2.1 affine S/Z formulas and groups
       of 64; section 2.2 residual cache of the most recent 128 tokens,
       quantized and merged into the main cache when full; section 3.1 table).

The element-level arithmetic lives in ``kvq_oracle.c`` (binary32 encode
decisions, binary64 attention).  This module holds the ctypes glue, the
cache bookkeeping (main cache + residual ring, appended token by token) and
the size formula.  Every function is pinned by tests/test_oracle_*.py.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

from . import build as _build

_lib = None

NVFP4, INT4, FP8, INT8, INT2 = 1, 2, 3, 4, 5
FORMAT_NAMES = {NVFP4: "nvfp4", INT4: "int4", FP8: "fp8", INT8: "int8", INT2: "int2"}
INT_AFFINE = (INT4, INT8, INT2)

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64 = ctypes.c_int64


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.kvqo_e4m3_decode.restype = ctypes.c_float
        L.kvqo_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.kvqo_e2m1_decode.restype = ctypes.c_float
        L.kvqo_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.kvqo_e4m3_encode.restype = ctypes.c_uint8
        L.kvqo_e4m3_encode.argtypes = [ctypes.c_float]
        L.kvqo_e2m1_encode.restype = ctypes.c_uint8
        L.kvqo_e2m1_encode.argtypes = [ctypes.c_float]
        L.kvqo_e4m3_encode_array.argtypes = [_f32p, _i64, _u8p]
        L.kvqo_e2m1_encode_array.argtypes = [_f32p, _i64, _u8p]
        L.kvqo_amax.restype = ctypes.c_float
        L.kvqo_amax.argtypes = [_f32p, _i64]
        L.kvqo_nvfp4_global_scale.restype = ctypes.c_float
        L.kvqo_nvfp4_global_scale.argtypes = [ctypes.c_float]
        L.kvqo_fp8_global_scale.restype = ctypes.c_float
        L.kvqo_fp8_global_scale.argtypes = [ctypes.c_float]
        L.kvqo_nvfp4_encode.argtypes = [_f32p, _i64, ctypes.c_int, ctypes.c_float, _u8p, _u8p]
        L.kvqo_nvfp4_decode.argtypes = [_u8p, _u8p, _i64, ctypes.c_int, ctypes.c_float, _f32p]
        L.kvqo_fp8_encode.argtypes = [_f32p, _i64, ctypes.c_float, _u8p]
        L.kvqo_fp8_decode.argtypes = [_u8p, _i64, ctypes.c_float, _f32p]
        L.kvqo_int4_encode.argtypes = [_f32p, _i64, ctypes.c_int, ctypes.c_int, _u8p, _f32p, _i32p]
        L.kvqo_int4_decode.argtypes = [_u8p, _f32p, _i32p, _i64, ctypes.c_int, ctypes.c_int, _f32p]
        L.kvqo_mxfp4_encode.argtypes = [_f32p, _i64, ctypes.c_int, _u8p, _u8p]
        L.kvqo_mxfp4_decode.argtypes = [_u8p, _u8p, _i64, ctypes.c_int, _f32p]
        L.kvqo_int8_encode.argtypes = [_f32p, _i64, ctypes.c_int, ctypes.c_int, _u8p, _f32p, _i32p]
        L.kvqo_int8_decode.argtypes = [_u8p, _f32p, _i32p, _i64, ctypes.c_int, ctypes.c_int, _f32p]
        L.kvqo_int2_encode.argtypes = [_f32p, _i64, ctypes.c_int, ctypes.c_int, _u8p, _f32p, _i32p]
        L.kvqo_int2_decode.argtypes = [_u8p, _f32p, _i32p, _i64, ctypes.c_int, ctypes.c_int, _f32p]
        L.kvqo_attention.argtypes = [_f32p, _f32p, _f32p, _i64, ctypes.c_int, ctypes.c_double, _f64p]
        L.kvqo_attention_lse.argtypes = [_f32p, _f32p, _f32p, _i64, ctypes.c_int, ctypes.c_double,
                                         _f64p, _f64p]
        L.kvqo_combine.argtypes = [ctypes.c_int, ctypes.c_int, _f64p, _f64p, _f64p, _f64p]
        L.kvqo_attention_gqa.argtypes = [_f32p, ctypes.c_int, _f32p, _f32p, _i64, ctypes.c_int,
                                         ctypes.c_double, _f64p]
        _lib = L
    return _lib


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


# --------------------------------------------------------------------------
# Scalar formats
# --------------------------------------------------------------------------

def e4m3_encode(x) -> np.ndarray:
    """E4M3 codes (RNE, saturating at 448, sign kept) of float32 values."""
    x = _f32(x)
    out = np.empty(x.shape, np.uint8)
    lib().kvqo_e4m3_encode_array(_p(x, _f32p), x.size, _p(out, _u8p))
    return out


def e4m3_decode(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    L = lib()
    return np.array([L.kvqo_e4m3_decode(int(v)) for v in c.ravel()],
                    np.float32).reshape(c.shape)


def e2m1_encode(x) -> np.ndarray:
    """E2M1 codes 0..15 (RNE on the grid, saturating at 6, sign kept)."""
    x = _f32(x)
    out = np.empty(x.shape, np.uint8)
    lib().kvqo_e2m1_encode_array(_p(x, _f32p), x.size, _p(out, _u8p))
    return out


def e2m1_decode(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    L = lib()
    return np.array([L.kvqo_e2m1_decode(int(v)) for v in c.ravel()],
                    np.float32).reshape(c.shape)


def amax(x) -> float:
    x = _f32(x)
    return float(lib().kvqo_amax(_p(x, _f32p), x.size))


def global_scale(fmt: int, amax_value: float) -> float:
    """Per-tensor scale from a calibration amax ([P2] format table)."""
    L = lib()
    if fmt == NVFP4:
        return float(L.kvqo_nvfp4_global_scale(amax_value))
    if fmt == FP8:
        return float(L.kvqo_fp8_global_scale(amax_value))
    raise ValueError("only NVFP4 and FP8 carry a per-tensor scale")


# --------------------------------------------------------------------------
# Row encoders / decoders.  x: float32 [..., D]; leading dims are rows.
# --------------------------------------------------------------------------

def nvfp4_quantize(x, g: float):
    x = _f32(x)
    D = x.shape[-1]
    rows = x.size // D
    codes = np.zeros(x.shape[:-1] + (D // 2,), np.uint8)
    scales = np.zeros(x.shape[:-1] + (D // 16,), np.uint8)
    lib().kvqo_nvfp4_encode(_p(x, _f32p), rows, D, g, _p(codes, _u8p), _p(scales, _u8p))
    return codes, scales


def nvfp4_dequantize(codes, scales, g: float) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    D = codes.shape[-1] * 2
    rows = codes.size // (D // 2)
    out = np.empty(codes.shape[:-1] + (D,), np.float32)
    lib().kvqo_nvfp4_decode(_p(codes, _u8p), _p(scales, _u8p), rows, D, g, _p(out, _f32p))
    return out


def fp8_quantize(x, s: float) -> np.ndarray:
    x = _f32(x)
    codes = np.empty(x.shape, np.uint8)
    lib().kvqo_fp8_encode(_p(x, _f32p), x.size, s, _p(codes, _u8p))
    return codes


def fp8_dequantize(codes, s: float) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, np.float32)
    lib().kvqo_fp8_decode(_p(codes, _u8p), codes.size, s, _p(out, _f32p))
    return out


def int4_quantize(x, group: int = 64):
    x = _f32(x)
    D = x.shape[-1]
    rows = x.size // D
    codes = np.zeros(x.shape[:-1] + (D // 2,), np.uint8)
    S = np.zeros(x.shape[:-1] + (D // group,), np.float32)
    Z = np.zeros(x.shape[:-1] + (D // group,), np.int32)
    lib().kvqo_int4_encode(_p(x, _f32p), rows, D, group, _p(codes, _u8p), _p(S, _f32p), _p(Z, _i32p))
    return codes, S, Z


def int4_dequantize(codes, S, Z, group: int = 64) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    S = np.ascontiguousarray(S, dtype=np.float32)
    Z = np.ascontiguousarray(Z, dtype=np.int32)
    D = codes.shape[-1] * 2
    rows = codes.size // (D // 2)
    out = np.empty(codes.shape[:-1] + (D,), np.float32)
    lib().kvqo_int4_decode(_p(codes, _u8p), _p(S, _f32p), _p(Z, _i32p), rows, D, group, _p(out, _f32p))
    return out


# --------------------------------------------------------------------------
# Attention (definition, binary64)
# --------------------------------------------------------------------------

def attention(q, K, V, scale: Optional[float] = None) -> np.ndarray:
    """Softmax attention of G query vectors over L keys/values.

    q: [G, D], K/V: [L, D] (float32 values).  Returns float64 [G, D].
    """
    q = _f32(q)
    K = _f32(K)
    V = _f32(V)
    if q.ndim == 1:
        q = q[None, :]
    G, D = q.shape
    L = K.shape[0] if K.size else 0
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = np.zeros((G, D), np.float64)
    if L == 0:
        return out
    lib().kvqo_attention_gqa(_p(q, _f32p), G, _p(K, _f32p), _p(V, _f32p), L, D,
                             float(scale), _p(out, _f64p))
    return out


def attention_lse(q, K, V, scale: Optional[float] = None):
    """attention() plus the log-sum-exp of each query's scores:
    (out float64 [G, D], lse float64 [G]); no keys gives out 0, lse -inf."""
    q = _f32(q)
    K = _f32(K)
    V = _f32(V)
    if q.ndim == 1:
        q = q[None, :]
    G, D = q.shape
    L = K.shape[0] if K.size else 0
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = np.zeros((G, D), np.float64)
    lse = np.full(G, -np.inf)
    for h in range(G):
        o = np.zeros(D, np.float64)
        l = ctypes.c_double()
        lib().kvqo_attention_lse(_p(np.ascontiguousarray(q[h]), _f32p), _p(K, _f32p), _p(V, _f32p),
                                 L, D, float(scale), _p(o, _f64p), ctypes.byref(l))
        out[h], lse[h] = o, l.value
    return out, lse


def combine_partials(o_parts, lse_parts):
    """Merge attention over disjoint key parts: o_parts [n, ..., D], lse_parts
    [n, ...] -> (out [..., D], lse [...]) in float64."""
    o_parts = np.asarray(o_parts, np.float64)
    lse_parts = np.asarray(lse_parts, np.float64)
    n, D = o_parts.shape[0], o_parts.shape[-1]
    rows = int(np.prod(o_parts.shape[1:-1], dtype=np.int64))
    o2 = o_parts.reshape(n, rows, D)
    l2 = lse_parts.reshape(n, rows)
    out = np.zeros((rows, D), np.float64)
    lse = np.zeros(rows, np.float64)
    for i in range(rows):
        op = np.ascontiguousarray(o2[:, i])
        lp = np.ascontiguousarray(l2[:, i])
        o = np.zeros(D, np.float64)
        l = ctypes.c_double()
        lib().kvqo_combine(n, D, _p(op, _f64p), _p(lp, _f64p), _p(o, _f64p), ctypes.byref(l))
        out[i], lse[i] = o, l.value
    return out.reshape(o_parts.shape[1:]), lse.reshape(lse_parts.shape[1:])


# --------------------------------------------------------------------------
# KV size formula ([P2] "why long context runs out of memory": bytes =
# 2 x layers x kv_heads x head_dim x seq_len x bytes_per_element).
def mxfp4_quantize(x):
    """MXFP4 (an external definition for the comparison of [P1] section 3.2:
    OCP Microscaling v1.0, E2M1 elements with one E8M0 scale per 32 values)
    -> (codes packed like NVFP4's, E8M0 scale bytes)."""
    x = _f32(x)
    D = x.shape[-1]
    rows = x.size // D
    codes = np.zeros(x.shape[:-1] + (D // 2,), np.uint8)
    scales = np.zeros(x.shape[:-1] + (D // 32,), np.uint8)
    lib().kvqo_mxfp4_encode(_p(x, _f32p), rows, D, _p(codes, _u8p), _p(scales, _u8p))
    return codes, scales


def mxfp4_dequantize(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    D = codes.shape[-1] * 2
    rows = codes.size // (D // 2)
    out = np.empty(codes.shape[:-1] + (D,), np.float32)
    lib().kvqo_mxfp4_decode(_p(codes, _u8p), _p(scales, _u8p), rows, D, _p(out, _f32p))
    return out


def int8_quantize(x, group: int = 64):
    """INT8 affine groups ([P3] section 2.1 with 8-bit codes): codes one byte
    per value, S and Z per group."""
    x = _f32(x)
    D = x.shape[-1]
    rows = x.size // D
    codes = np.zeros(x.shape, np.uint8)
    S = np.zeros(x.shape[:-1] + (D // group,), np.float32)
    Z = np.zeros(x.shape[:-1] + (D // group,), np.int32)
    lib().kvqo_int8_encode(_p(x, _f32p), rows, D, group, _p(codes, _u8p), _p(S, _f32p), _p(Z, _i32p))
    return codes, S, Z


def int8_dequantize(codes, S, Z, group: int = 64) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    S = np.ascontiguousarray(S, dtype=np.float32)
    Z = np.ascontiguousarray(Z, dtype=np.int32)
    D = codes.shape[-1]
    rows = codes.size // D
    out = np.empty(codes.shape, np.float32)
    lib().kvqo_int8_decode(_p(codes, _u8p), _p(S, _f32p), _p(Z, _i32p), rows, D, group, _p(out, _f32p))
    return out


def int2_quantize(x, group: int = 64):
    """INT2 affine groups ([P3] section 2.1 with 2-bit codes; the INT2 row of
    its section 3.1 table): four codes per byte, S and Z per group."""
    x = _f32(x)
    D = x.shape[-1]
    rows = x.size // D
    codes = np.zeros(x.shape[:-1] + (D // 4,), np.uint8)
    S = np.zeros(x.shape[:-1] + (D // group,), np.float32)
    Z = np.zeros(x.shape[:-1] + (D // group,), np.int32)
    lib().kvqo_int2_encode(_p(x, _f32p), rows, D, group, _p(codes, _u8p), _p(S, _f32p), _p(Z, _i32p))
    return codes, S, Z


def int2_dequantize(codes, S, Z, group: int = 64) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    S = np.ascontiguousarray(S, dtype=np.float32)
    Z = np.ascontiguousarray(Z, dtype=np.int32)
    D = codes.shape[-1] * 4
    rows = codes.size // (D // 4)
    out = np.empty(codes.shape[:-1] + (D,), np.float32)
    lib().kvqo_int2_decode(_p(codes, _u8p), _p(S, _f32p), _p(Z, _i32p), rows, D, group, _p(out, _f32p))
    return out


def int_compact_quantize(x, bits: int, group: int = 64, zbits: int = 8):
    """The affine scheme ([P3] section 2.1) with compact group metadata: S
    stored as IEEE binary16 and Z as a signed zbits-bit integer (int8: 3
    bytes per group instead of 8).

    Reading taken (the pages give no compact form): S is computed in binary32
    as usual, then rounded to binary16 (round to nearest even; saturated to
    65504, and raised to 2^-24 if it would round to zero); Z and the codes are
    computed with that stored S, so decoding (q - Z) * S reproduces what the
    encoder aimed at; Z is clamped to the zbits-bit signed range, and a group
    whose Z does not fit saturates its codes at the ends of the range.  The
    cache keeps int8 zero points for 2- and 4-bit codes and int16 ones for
    8-bit codes (zero points of groups that span zero lie in 0 .. 2^bits - 1,
    which int8 holds only below 8 bits).  Codes are unpacked here (one per
    value, uint8).  Steps use numpy binary32 arithmetic and numpy's binary16
    conversion.
    """
    x = _f32(x)
    D = x.shape[-1]
    g = x.reshape(x.shape[:-1] + (D // group, group))
    qmax = np.float32(2 ** bits - 1)
    mn = g.min(axis=-1)
    mx = g.max(axis=-1)
    with np.errstate(over="ignore"):
        S32 = np.where(mx == mn, np.where(mn != 0, np.abs(mn), np.float32(1.0)),
                       (mx - mn) / qmax).astype(np.float32)
        S16 = S32.astype(np.float16)
    S16 = np.where(np.isinf(S16), np.float16(65504.0), S16)
    S16 = np.where(S16 == 0, np.float16(2.0 ** -24), S16)
    S = S16.astype(np.float32)
    zlo, zhi = -(2 ** (zbits - 1)), 2 ** (zbits - 1) - 1
    Z = np.clip(np.rint(-mn / S), zlo, zhi).astype(np.int32)
    q = np.clip(np.rint(g / S[..., None]) + Z[..., None], 0, qmax).astype(np.uint8)
    return q.reshape(x.shape), S16, Z.astype(np.int8 if zbits == 8 else np.int16)


def compact_zbits(bits: int) -> int:
    """Zero-point width of the cache's compact metadata for `bits`-bit codes."""
    return 16 if bits == 8 else 8


def int_compact_dequantize(q, S16, Z, group: int = 64) -> np.ndarray:
    q = np.asarray(q)
    D = q.shape[-1]
    g = q.reshape(q.shape[:-1] + (D // group, group)).astype(np.int32)
    S = np.asarray(S16, np.float16).astype(np.float32)
    out = ((g - np.asarray(Z, np.int32)[..., None]).astype(np.float32) * S[..., None]).astype(np.float32)
    return out.reshape(q.shape)


# --------------------------------------------------------------------------

def kv_cache_bytes(layers: int, kv_heads: int, head_dim: int, seq_len: int,
                   bytes_per_element: float) -> float:
    return 2 * layers * kv_heads * head_dim * seq_len * bytes_per_element


def cache_storage_bytes_per_token_head(fmt: int, head_dim: int, group: int = 64,
                                       compact: bool = False) -> int:
    """Bytes one token of one KV head occupies in the main cache, K or V.

    NVFP4: head_dim/2 code bytes + head_dim/16 E4M3 scale bytes.
    INT4:  head_dim/2 code bytes + (f32 S + i32 Z) per group of `group`.
    INT8:  head_dim code bytes + (f32 S + i32 Z) per group of `group`.
    INT2:  head_dim/4 code bytes + (f32 S + i32 Z) per group of `group`.
    FP8:   head_dim code bytes.
    compact=True (INT formats): f16 S + an int8 Z (2, 4 bits: 3 bytes per
    group) or int16 Z (8 bits: 4 bytes per group).
    """
    if fmt == NVFP4:
        return head_dim // 2 + head_dim // 16
    if compact and fmt in INT_AFFINE:
        bits = {INT4: 4, INT8: 8, INT2: 2}[fmt]
        return head_dim * bits // 8 + (2 + compact_zbits(bits) // 8) * (head_dim // group)
    if fmt == INT4:
        return head_dim // 2 + 8 * (head_dim // group)
    if fmt == INT8:
        return head_dim + 8 * (head_dim // group)
    if fmt == INT2:
        return head_dim // 4 + 8 * (head_dim // group)
    if fmt == FP8:
        return head_dim
    raise ValueError(fmt)


# --------------------------------------------------------------------------
# Cache bookkeeping: main quantized cache plus (INT4) residual ring.
# --------------------------------------------------------------------------

@dataclass
class _Layer:
    # main cache, per K/V: list of per-chunk arrays, concatenated lazily, and
    # the per-tensor scale each chunk was encoded with
    main: List[list] = field(default_factory=lambda: [[], []])
    main_scale: List[list] = field(default_factory=lambda: [[], []])
    ring: List[list] = field(default_factory=lambda: [[], []])   # float32 [B,H,D] tokens
    len_main: int = 0
    scale: List[Optional[float]] = field(default_factory=lambda: [None, None])
    # recalibration: (first token, scale) of every scale segment, and the
    # amax of the tokens of the current segment so far
    segments: List[list] = field(default_factory=lambda: [[], []])
    seg_amax: List[float] = field(default_factory=lambda: [0.0, 0.0])


class OracleCache:
    """The cache as the pages describe it, kept in host memory.

    * NVFP4 / FP8 ([P1] section 2.1): every appended token is quantized and
      placed at the end of the main cache.  The per-tensor scale of K (and of
      V) is calibrated from the amax of the layer's first append unless it
      was given ([P2] format table).
    * INT4 / INT8 / INT2 affine with residual ring ([P3] section 2.2): tokens
      enter a BF16 ring of `residual_length` slots one by one; as soon as the
      ring is full its contents are quantized, merged into the main cache and
      the ring is emptied.  `flush_residual` quantizes a partial ring the same
      way.  residual_length == 0 quantizes every token immediately.
    * NVFP4 / FP8 with a residual ring (the combination [P1] section 3.2's
      comparison leaves open): the same ring; the ring's tokens are encoded
      at the flush with the layer's per-tensor scale, which is still
      calibrated from the first append.
    * compact=True (INT formats): group metadata S as binary16 and Z as int8
      (INT2, INT4) or int16 (INT8), encoded by int_compact_quantize (main arrays: one code per value, S16,
      Z8).
    * Scale recalibration ([P1] section 3.1: the scale is renewed every 512
      processed tokens; NVFP4 / FP8 without a ring): `recalibrate_every` = P
      splits the token positions into segments [sP, (s+1)P).  Segment 0 uses
      the calibrated (or given) scale; segment s >= 1 uses the scale computed
      from the amax of segment s-1's tokens (all batch rows and heads of the
      layer).  Tokens are never re-encoded: each keeps the scale that was in
      force at its position, so the rule is causal and a bulk append equals
      the same tokens appended one by one.
    """

    def __init__(self, fmt: int, layers: int, batch: int, kv_heads: int, head_dim: int,
                 max_len: int, group_size: int = 0, residual_length: int = 0,
                 global_scales=None, recalibrate_every: int = 0, compact: bool = False):
        if fmt not in FORMAT_NAMES:
            raise ValueError("unknown format")
        if recalibrate_every and (fmt not in (NVFP4, FP8) or residual_length):
            raise ValueError("recalibration is defined for NVFP4 / FP8 without a ring")
        if compact and fmt not in INT_AFFINE:
            raise ValueError("compact group metadata is defined for the INT formats")
        self.compact = compact
        self.fmt = fmt
        self.layers = layers
        self.batch = batch
        self.kv_heads = kv_heads
        self.head_dim = head_dim
        self.max_len = max_len
        self.group = group_size if fmt in INT_AFFINE else 16 if fmt == NVFP4 else 0
        self.R = residual_length
        self.P = recalibrate_every
        self.L = [_Layer() for _ in range(layers)]
        self._given = None
        if global_scales is not None:
            self._given = np.asarray(global_scales, np.float32).reshape(layers, 2)
        self.reset()

    # -- encoding of a block of whole tokens [B, H, n, D] ------------------
    def _encode(self, x: np.ndarray, scale: Optional[float]):
        if self.compact:
            bits = {INT4: 4, INT8: 8, INT2: 2}[self.fmt]
            return int_compact_quantize(x, bits, self.group, compact_zbits(bits))
        if self.fmt == NVFP4:
            return nvfp4_quantize(x, scale)
        if self.fmt == FP8:
            return (fp8_quantize(x, scale),)
        if self.fmt == INT8:
            return int8_quantize(x, self.group)
        if self.fmt == INT2:
            return int2_quantize(x, self.group)
        return int4_quantize(x, self.group)

    def _put(self, st: _Layer, kv: int, x: np.ndarray):
        st.main[kv].append(self._encode(x, st.scale[kv]))
        st.main_scale[kv].append(st.scale[kv])

    def append(self, layer: int, k, v):
        """Append n tokens: k, v float32 [B, H, n, D] (values exact in BF16)."""
        st = self.L[layer]
        k = _f32(k)
        v = _f32(v)
        n = k.shape[2]
        if n == 0:
            return
        if st.len_main + len(st.ring[0]) + n > self.max_len:
            raise ValueError("capacity exceeded")
        for kv, x in ((0, k), (1, v)):
            if self.fmt in (NVFP4, FP8) and st.scale[kv] is None:
                st.scale[kv] = global_scale(self.fmt, amax(x))
                st.segments[kv] = [(0, st.scale[kv])]
        if self.P:
            self._append_recalibrating(st, k, v)
            return
        if self.R == 0:
            for kv, x in ((0, k), (1, v)):
                self._put(st, kv, x)
            st.len_main += n
            return
        # Residual ring: push token by token; flush whenever the ring fills.
        for t in range(n):
            for kv, x in ((0, k), (1, v)):
                st.ring[kv].append(x[:, :, t, :])
            if len(st.ring[0]) == self.R:
                self._flush(layer)

    def _append_recalibrating(self, st: _Layer, k: np.ndarray, v: np.ndarray):
        n = k.shape[2]
        t = 0
        while t < n:
            pos = st.len_main
            run = min(n - t, self.P - pos % self.P)     # tokens left in this segment
            for kv, x in ((0, k), (1, v)):
                part = x[:, :, t:t + run]
                if pos % self.P == 0 and pos > 0:
                    # first token of a new segment: renew the scale from the
                    # previous segment's amax, then start a new running amax
                    st.scale[kv] = global_scale(self.fmt, st.seg_amax[kv])
                    st.segments[kv].append((pos, st.scale[kv]))
                    st.seg_amax[kv] = 0.0
                st.seg_amax[kv] = max(st.seg_amax[kv], amax(part))
                self._put(st, kv, part)
            st.len_main += run
            t += run

    def _flush(self, layer: int):
        st = self.L[layer]
        r = len(st.ring[0])
        if r == 0:
            return
        for kv in (0, 1):
            block = np.stack(st.ring[kv], axis=2)          # [B, H, r, D]
            self._put(st, kv, block)
            st.ring[kv] = []
        st.len_main += r

    def flush_residual(self, layer: int):
        self._flush(layer)

    def reset(self):
        self.L = [_Layer() for _ in range(self.layers)]
        if self._given is not None:
            for li in range(self.layers):
                self.L[li].scale = [float(self._given[li, 0]), float(self._given[li, 1])]
                self.L[li].segments = [[(0, self.L[li].scale[0])], [(0, self.L[li].scale[1])]]

    # -- views --------------------------------------------------------------
    def lengths(self, layer: int):
        st = self.L[layer]
        return st.len_main, len(st.ring[0])

    def scale(self, layer: int, kv: int) -> Optional[float]:
        """The per-tensor scale in force for the next token."""
        return self.L[layer].scale[kv]

    def segment_scales(self, layer: int, kv: int):
        """[(first token, scale)] of every scale segment so far."""
        return list(self.L[layer].segments[kv])

    def main_arrays(self, layer: int, kv: int):
        """Concatenated main-cache arrays along the token axis (axis 2)."""
        parts = self.L[layer].main[kv]
        if not parts:
            return None
        return tuple(np.concatenate([p[i] for p in parts], axis=2) for i in range(len(parts[0])))

    def ring_tokens(self, layer: int, kv: int) -> np.ndarray:
        ring = self.L[layer].ring[kv]
        if not ring:
            return np.zeros((self.batch, self.kv_heads, 0, self.head_dim), np.float32)
        return np.stack(ring, axis=2)

    def dequantize_main(self, layer: int, kv: int) -> np.ndarray:
        st = self.L[layer]
        if not st.main[kv]:
            return np.zeros((self.batch, self.kv_heads, 0, self.head_dim), np.float32)
        if self.compact:
            return np.concatenate([int_compact_dequantize(*part, self.group) for part in st.main[kv]],
                                  axis=2)
        return np.concatenate([dequantize_arrays(self.fmt, part, sc, self.group)
                               for part, sc in zip(st.main[kv], st.main_scale[kv])], axis=2)

    def decode_attention(self, layer: int, q, scale: Optional[float] = None) -> np.ndarray:
        """q: float32 [B, Hq, D] -> float64 [B, Hq, D]; kv head of query
        head h is h // (Hq / kv_heads)."""
        K = np.concatenate([self.dequantize_main(layer, 0), self.ring_tokens(layer, 0)], axis=2)
        V = np.concatenate([self.dequantize_main(layer, 1), self.ring_tokens(layer, 1)], axis=2)
        return gqa_decode_attention(q, K, V, scale)


def dequantize_arrays(fmt: int, arrs, scale: Optional[float], group: int) -> np.ndarray:
    """Dequantize main-cache arrays (as returned by the encoders) to float32."""
    if fmt == NVFP4:
        return nvfp4_dequantize(arrs[0], arrs[1], scale)
    if fmt == FP8:
        return fp8_dequantize(arrs[0], scale)
    if fmt == INT8:
        return int8_dequantize(arrs[0], arrs[1], arrs[2], group)
    if fmt == INT2:
        return int2_dequantize(arrs[0], arrs[1], arrs[2], group)
    return int4_dequantize(arrs[0], arrs[1], arrs[2], group)


def gqa_decode_attention(q, K, V, scale: Optional[float] = None) -> np.ndarray:
    """q [B, Hq, D]; K, V [B, Hkv, L, D] -> float64 [B, Hq, D]."""
    q = _f32(q)
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D), np.float64)
    for b in range(B):
        for h in range(Hkv):
            out[b, h * G:(h + 1) * G] = attention(q[b, h * G:(h + 1) * G], K[b, h], V[b, h], scale)
    return out


class RaggedOracleCache:
    """A batch of sequences of different lengths: the per-sequence view of a
    KV cache whose address space is shared by all sequences of a batch
    ([P1] section 5.2 speaks of a globally addressed KV cache; serving
    batches hold sequences of unequal length).

    Each sequence b is its own one-sequence OracleCache (same format, ring
    and group size), so every per-token rule -- encoding, ring, flush -- is
    the single-sequence rule.  The only state shared across sequences is
    each layer's per-tensor K and V scale (NVFP4 / FP8): it is calibrated by
    the layer's first append, whichever sequences that append feeds, from
    the amax of the tokens it appends, and every sequence uses it from then
    on ([P2] format table: one amax per tensor).  Scale renewal is not
    defined here: sequences reach a segment at different times.

    A sequence with no tokens attends to nothing: its output is 0.
    """

    def __init__(self, fmt: int, layers: int, batch: int, kv_heads: int, head_dim: int,
                 max_len: int, group_size: int = 0, residual_length: int = 0,
                 global_scales=None, compact: bool = False):
        self.fmt, self.layers, self.batch = fmt, layers, batch
        self.kv_heads, self.head_dim, self.max_len = kv_heads, head_dim, max_len
        self.R = residual_length
        self.group = group_size if fmt in INT_AFFINE else 16 if fmt == NVFP4 else 0
        self._args = (fmt, layers, 1, kv_heads, head_dim, max_len, group_size, residual_length)
        self.compact = compact
        self._given = None if global_scales is None else np.asarray(global_scales, np.float32).reshape(layers, 2)
        self.seqs = [OracleCache(*self._args, global_scales=self._given, compact=compact)
                     for _ in range(batch)]
        # per layer: the shared per-tensor (K, V) scales, None until calibrated
        self.shared = [None if self._given is None else (float(self._given[li, 0]), float(self._given[li, 1]))
                       for li in range(layers)]

    def _calibrate(self, layer: int, ks, vs):
        """ks, vs: the [H, n, D] token blocks one append brings."""
        if self.fmt not in (NVFP4, FP8) or self.shared[layer] is not None:
            return
        gk = global_scale(self.fmt, max([amax(x) for x in ks] + [0.0]))
        gv = global_scale(self.fmt, max([amax(x) for x in vs] + [0.0]))
        self.shared[layer] = (gk, gv)
        for oc in self.seqs:
            st = oc.L[layer]
            st.scale = [gk, gv]
            st.segments = [[(0, gk)], [(0, gv)]]

    def append_seq(self, layer: int, seq: int, k, v):
        """Append n tokens to sequence `seq`: k, v float32 [H, n, D]."""
        k, v = _f32(k), _f32(v)
        if k.shape[1] == 0:
            return
        self._calibrate(layer, [k], [v])
        self.seqs[seq].append(layer, k[None], v[None])

    def append(self, layer: int, k, v, n=None):
        """Append to every sequence: k, v float32 [B, H, n_max, D]; sequence b
        takes its first n[b] tokens (all n_max when n is None)."""
        k, v = _f32(k), _f32(v)
        n = [k.shape[2]] * self.batch if n is None else list(n)
        if sum(n) == 0:
            return
        self._calibrate(layer, [k[b, :, :n[b]] for b in range(self.batch) if n[b]],
                        [v[b, :, :n[b]] for b in range(self.batch) if n[b]])
        for b in range(self.batch):
            if n[b]:
                self.seqs[b].append(layer, k[b:b + 1, :, :n[b]], v[b:b + 1, :, :n[b]])

    def flush_residual(self, layer: int):
        for oc in self.seqs:
            oc.flush_residual(layer)

    def reset_seq(self, seq: int):
        """Empty sequence `seq` in every layer (the shared scales stay)."""
        oc = OracleCache(*self._args, global_scales=self._given, compact=self.compact)
        for li in range(self.layers):
            if self.shared[li] is not None:
                oc.L[li].scale = list(self.shared[li])
                oc.L[li].segments = [[(0, self.shared[li][0])], [(0, self.shared[li][1])]]
        self.seqs[seq] = oc

    def lengths(self, layer: int, seq: int):
        return self.seqs[seq].lengths(layer)

    def scale(self, layer: int, kv: int):
        return None if self.shared[layer] is None else self.shared[layer][kv]

    def main_arrays(self, layer: int, kv: int, seq: int):
        """Main-cache arrays of one sequence, [1, H, n, ...] (None if empty)."""
        return self.seqs[seq].main_arrays(layer, kv)

    def ring_tokens(self, layer: int, kv: int, seq: int) -> np.ndarray:
        return self.seqs[seq].ring_tokens(layer, kv)

    def decode_attention(self, layer: int, q, scale: Optional[float] = None) -> np.ndarray:
        """q float32 [B, Hq, D] -> float64 [B, Hq, D]; a sequence holding no
        tokens gives 0."""
        q = _f32(q)
        out = np.zeros(q.shape, np.float64)
        for b, oc in enumerate(self.seqs):
            if sum(oc.lengths(layer)):
                out[b] = oc.decode_attention(layer, q[b:b + 1], scale)[0]
        return out
