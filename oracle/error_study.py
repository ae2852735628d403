"""Reconstruction and attention-output error of the cache formats on
synthetic long sequences.

TEST INFRASTRUCTURE: calls only the oracle and the seeded input generators.
Usage:  python -m oracle.error_study [--lengths 1100,16500,102500] [--drift] [--compact]

Three studies, each on one (batch, kv head) unit with G = 8 query heads:

* Formats (the NVFP4-vs-MXFP4 comparison of the NVFP4 KV-cache article,
  section 3.2, on synthetic data instead of models).  NVFP4 and FP8 use a
  per-tensor scale calibrated on the whole sequence.  MXFP4 uses its
  per-block power-of-two scales.  INT4 / INT8 / INT2 use affine groups of 64.
* Cache configurations with a BF16 residual ring:
  - HF's 128-token ring on INT4 and INT2 (section 2.2 of the KV-cache
    long-text article);
  - its troubleshooting setting, INT4 groups of 32 with a 256-token ring
    (section 4.3);
  - NVFP4 with a 128-token ring;
  - the age-based tiers of its section 4.2: older chunks in INT2, the most
    recent (incomplete) 8192-token chunk kept in full precision, i.e. INT2
    with an 8192-token ring.
  A cache of L tokens holds the first R*floor(L/R) tokens quantized and the
  rest exact.
* Drift (the NVFP4 article's section 3.1, scale renewal every 512 tokens):
  K and V magnitudes change by 2x every 4096 tokens after a 512-token
  calibrating prefill.  NVFP4 and FP8 are run with a frozen scale and with
  the scale renewed every 512 tokens.

* Compact group metadata (f16 S, i8 Z) against f32 S + i32 Z for the INT
  formats, on N(0,1) tokens and on groups shifted away from zero.

Reported: rel-RMSE of the cached K and V (quantized part and ring together)
and the rel-L2 error of the fp64 attention output against fp64 attention
over the exact (BF16) K and V.
"""
from __future__ import annotations

import argparse

import numpy as np

import oracle
from quantized_kv_cache_13_b200 import workloads as W

FORMATS = ("nvfp4", "mxfp4", "int4", "int8", "int2", "fp8")

# name -> (format, group, residual ring length)
CACHE_CONFIGS = {
    "int4 g64 R128": ("int4", 64, 128),
    "int4 g32 R256": ("int4", 32, 256),
    "int2 g64 R128": ("int2", 64, 128),
    "int2 g64 + 8192-token BF16 chunk": ("int2", 64, 8192),
    "nvfp4 R128": ("nvfp4", 16, 128),
}


def roundtrip(fmt: str, x: np.ndarray, group: int = 64, calib=None) -> np.ndarray:
    """Quantize and dequantize x [L, 128] with the oracle.  NVFP4 / FP8
    calibrate their per-tensor scale on `calib` (default: x itself)."""
    if x.shape[0] == 0:
        return x.copy()
    c = x if calib is None else calib
    if fmt == "nvfp4":
        g = oracle.global_scale(oracle.NVFP4, oracle.amax(c))
        return oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(x, g), g)
    if fmt == "mxfp4":
        return oracle.mxfp4_dequantize(*oracle.mxfp4_quantize(x))
    if fmt == "int4":
        return oracle.int4_dequantize(*oracle.int4_quantize(x, group), group)
    if fmt == "int8":
        return oracle.int8_dequantize(*oracle.int8_quantize(x, group), group)
    if fmt == "int2":
        return oracle.int2_dequantize(*oracle.int2_quantize(x, group), group)
    if fmt == "fp8":
        s = oracle.global_scale(oracle.FP8, oracle.amax(c))
        return oracle.fp8_dequantize(oracle.fp8_quantize(x, s), s)
    raise ValueError(fmt)


def cached(fmt: str, group: int, R: int, x: np.ndarray) -> np.ndarray:
    """What a cache with an R-token ring holds after x [L, 128] was appended:
    the first R*floor(L/R) tokens through the quantizer, the rest exact."""
    n_q = (x.shape[0] // R) * R if R else x.shape[0]
    return np.concatenate([roundtrip(fmt, x[:n_q], group, calib=x), x[n_q:]], axis=0)


def rel(a: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(a.astype(np.float64) - ref) / np.linalg.norm(ref))


def _unit(dist: str, Lmax: int, seed: int, G: int):
    w = W.custom(oracle.INT4, 1, 1, G, Lmax, seed, k_dist=dist, v_dist=dist)
    return W.kv_slice(w, "k", 0, 0, 0, Lmax), W.kv_slice(w, "v", 0, 0, 0, Lmax), W.q_tensor(w)[0]


def study(dist: str, lengths, seed: int = 2024, G: int = 8, configs=None):
    """Errors for one input distribution: {name: (k_rmse, v_rmse, {L: attn_err})}
    over the plain formats and the ring configurations."""
    Lmax = max(lengths)
    K, V, q = _unit(dist, Lmax, seed, G)
    todo = [(f, (f, 64, 0)) for f in FORMATS]
    todo += list((CACHE_CONFIGS if configs is None else configs).items())
    out = {}
    for name, (fmt, grp, R) in todo:
        att = {}
        for L in lengths:
            Kh, Vh = cached(fmt, grp, R, K[:L]), cached(fmt, grp, R, V[:L])
            ref = oracle.attention(q, K[:L], V[:L])
            att[L] = rel(oracle.attention(q, Kh, Vh), ref)
        Kh, Vh = cached(fmt, grp, R, K), cached(fmt, grp, R, V)
        out[name] = (rel(Kh, K), rel(Vh, V), att)
    return out


def drifting(x: np.ndarray, period: int, factor_log2: int) -> np.ndarray:
    """x with token t multiplied by 2^(factor_log2 * floor(t / period)) (exact
    in BF16)."""
    e = (np.arange(x.shape[0]) // period) * factor_log2
    return (x * np.exp2(e).astype(np.float32)[:, None]).astype(np.float32)


def drift_study(L: int = 16384, period: int = 4096, factor_log2: int = 1, P: int = 512,
                prefill: int = 512, seed: int = 2025, G: int = 8):
    """{(fmt, "frozen"|"renewed"): (k_rmse, v_rmse, attn_err)} for NVFP4 and
    FP8 caches fed a 512-token prefill, then the rest in P-token appends
    (equal, bit for bit, to token-by-token appends)."""
    K, V, q = _unit("normal", L, seed, G)
    K = drifting(K, period, factor_log2)
    V = drifting(V, period, factor_log2)
    ref = oracle.attention(q, K, V)
    out = {}
    for fmt in (oracle.NVFP4, oracle.FP8):
        for mode, every in (("frozen", 0), ("renewed", P)):
            c = oracle.OracleCache(fmt, 1, 1, 1, 128, L, recalibrate_every=every)
            c.append(0, K[None, None, :prefill], V[None, None, :prefill])
            for t in range(prefill, L, P):
                c.append(0, K[None, None, t:t + P], V[None, None, t:t + P])
            Kh = c.dequantize_main(0, 0)[0, 0]
            Vh = c.dequantize_main(0, 1)[0, 0]
            out[(oracle.FORMAT_NAMES[fmt], mode)] = (
                rel(Kh, K), rel(Vh, V), rel(oracle.attention(q, Kh, Vh), ref))
    return out


def shifted_groups(rng, L: int, group: int = 64, shift: float = 2.0, sigma: float = 0.3):
    """Tokens whose groups of `group` values are N(0, sigma) shifted by -shift,
    0 or +shift (a stand-in for channels with large offsets): many groups
    hold values of one sign only, whose zero points lie far outside the code
    range."""
    x = sigma * rng.standard_normal((L, 128))
    x = x + np.repeat(rng.choice([-shift, 0.0, shift], size=(L, 128 // group)), group, axis=-1)
    return W.to_bf16_values(x.astype(np.float32))


def compact_study(L: int = 4096, seed: int = 2026):
    """Reconstruction rel-RMSE of the INT formats with f32 S + i32 Z group
    metadata against the compact f16 S + i8 Z form, on N(0,1) tokens and on
    shifted groups: {(inputs, bits): (f32-meta error, compact error, share of
    groups whose Z was clamped)}.  compact_study_cache_form gives the form
    the cache stores (an int16 Z for 8-bit codes)."""
    rng = np.random.default_rng(seed)
    inputs = {"N(0,1)": W.to_bf16_values(rng.standard_normal((L, 128)).astype(np.float32)),
              "shifted groups": shifted_groups(rng, L)}
    quant = {2: (oracle.int2_quantize, oracle.int2_dequantize),
             4: (oracle.int4_quantize, oracle.int4_dequantize),
             8: (oracle.int8_quantize, oracle.int8_dequantize)}
    out = {}
    for name, x in inputs.items():
        for bits, (qf, dq) in quant.items():
            c, S, Z = qf(x, 64)
            full = rel(dq(c, S, Z, 64), x)
            q16, S16, Z8 = oracle.int_compact_quantize(x, bits, 64)
            comp = rel(oracle.int_compact_dequantize(q16, S16, Z8, 64), x)
            clamped = float(np.mean((Z < -128) | (Z > 127)))
            out[(name, bits)] = (full, comp, clamped)
    return out


def compact_study_cache_form(L: int = 4096, seed: int = 2026):
    """As compact_study, with each width's zero point as the cache stores it
    (int8 for 2 and 4 bits, int16 for 8 bits): {(inputs, bits): (f32-meta
    error, compact error)}."""
    rng = np.random.default_rng(seed)
    inputs = {"N(0,1)": W.to_bf16_values(rng.standard_normal((L, 128)).astype(np.float32)),
              "shifted groups": shifted_groups(rng, L)}
    quant = {2: (oracle.int2_quantize, oracle.int2_dequantize),
             4: (oracle.int4_quantize, oracle.int4_dequantize),
             8: (oracle.int8_quantize, oracle.int8_dequantize)}
    out = {}
    for name, x in inputs.items():
        for bits, (qf, dq) in quant.items():
            c, S, Z = qf(x, 64)
            full = rel(dq(c, S, Z, 64), x)
            qc, S16, Zc = oracle.int_compact_quantize(x, bits, 64, oracle.compact_zbits(bits))
            out[(name, bits)] = (full, rel(oracle.int_compact_dequantize(qc, S16, Zc, 64), x))
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--lengths", default="1100,16500,102500")
    ap.add_argument("--dists", default="normal,lognormal_outlier,offset_uniform")
    ap.add_argument("--drift", action="store_true", help="run the scale-renewal study only")
    ap.add_argument("--compact", action="store_true", help="run the compact-metadata study only")
    args = ap.parse_args()
    if args.compact:
        res = compact_study()
        print("| inputs | format | rel-RMSE, f32 S + i32 Z | rel-RMSE, f16 S + i8 Z | groups with Z outside int8 |")
        print("|---|---|---|---|---|")
        for (name, bits), (full, comp, clamped) in res.items():
            print("| %s | INT%d g64 | %.4f | %.4f | %.1f %% |" % (name, bits, full, comp, 100 * clamped))
        return
    if args.drift:
        for f2 in (1, -1):
            res = drift_study(factor_log2=f2)
            print("\n### magnitude x%s every 4096 tokens, 16384 tokens\n" % ("2" if f2 > 0 else "1/2"))
            print("| format | scale | K rel-RMSE | V rel-RMSE | attention rel-L2 |")
            print("|---|---|---|---|---|")
            for (fmt, mode), (k, v, a) in res.items():
                print("| %s | %s | %.4f | %.4f | %.2e |" % (fmt, mode, k, v, a))
        return
    lengths = [int(x) for x in args.lengths.split(",")]
    for dist in args.dists.split(","):
        res = study(dist, lengths)
        print("\n### inputs: %s\n" % dist)
        print("| configuration | K rel-RMSE | V rel-RMSE | " +
              " | ".join("attention rel-L2 @ %d" % L for L in lengths) + " |")
        print("|---|---|---|" + "---|" * len(lengths))
        for name, (k, v, att) in res.items():
            print("| %s | %.4f | %.4f | %s |" % (name, k, v, " | ".join("%.2e" % att[L] for L in lengths)))
        print("\nNVFP4 / MXFP4 attention error: " +
              ", ".join("%.2f @ %d" % (res["nvfp4"][2][L] / res["mxfp4"][2][L], L) for L in lengths))


if __name__ == "__main__":
    main()
