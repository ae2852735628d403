"""Reconstruction and attention-output error of the cache formats on
synthetic long sequences (the NVFP4-vs-MXFP4 comparison the NVFP4 KV-cache
article draws in its section 3.2, on synthetic data instead of models).

TEST INFRASTRUCTURE: calls only the oracle and the seeded input generators.
Usage:  python -m oracle.error_study [--lengths 1024,16384,102400]

For one (batch, kv head) unit and G = 8 query heads, each format quantizes
the unit's K and V (NVFP4 and FP8 with a per-tensor scale calibrated on the
whole sequence, MXFP4 with its per-block power-of-two scales, INT4 / INT8
affine groups of 64).  Reported, per format:
  rel-RMSE of the reconstructed K and V,
  rel-L2 error of the fp64 attention output against fp64 attention over
  the exact (BF16) K and V, for each sequence length.
"""
from __future__ import annotations

import argparse

import numpy as np

import oracle
from quantized_kv_cache_13_b200 import workloads as W

FORMATS = ("nvfp4", "mxfp4", "int4", "int8", "fp8")


def roundtrip(fmt: str, x: np.ndarray) -> np.ndarray:
    """Quantize and dequantize x [L, 128] with the oracle."""
    if fmt == "nvfp4":
        g = oracle.global_scale(oracle.NVFP4, oracle.amax(x))
        return oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(x, g), g)
    if fmt == "mxfp4":
        return oracle.mxfp4_dequantize(*oracle.mxfp4_quantize(x))
    if fmt == "int4":
        return oracle.int4_dequantize(*oracle.int4_quantize(x, 64), 64)
    if fmt == "int8":
        return oracle.int8_dequantize(*oracle.int8_quantize(x, 64), 64)
    if fmt == "fp8":
        s = oracle.global_scale(oracle.FP8, oracle.amax(x))
        return oracle.fp8_dequantize(oracle.fp8_quantize(x, s), s)
    raise ValueError(fmt)


def rel(a: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(a.astype(np.float64) - ref) / np.linalg.norm(ref))


def study(dist: str, lengths, seed: int = 2024, G: int = 8):
    """Errors for one input distribution: {fmt: (k_rmse, v_rmse, {L: attn_err})}."""
    Lmax = max(lengths)
    w = W.custom(oracle.INT4, 1, 1, G, Lmax, seed, k_dist=dist, v_dist=dist)
    K = W.kv_slice(w, "k", 0, 0, 0, Lmax)
    V = W.kv_slice(w, "v", 0, 0, 0, Lmax)
    q = W.q_tensor(w)[0]                                  # [G, 128]
    out = {}
    for fmt in FORMATS:
        att = {}
        for L in lengths:
            Kh, Vh = roundtrip(fmt, K[:L]), roundtrip(fmt, V[:L])
            ref = oracle.attention(q, K[:L], V[:L])
            att[L] = rel(oracle.attention(q, Kh, Vh), ref)
        Kh, Vh = roundtrip(fmt, K), roundtrip(fmt, V)
        out[fmt] = (rel(Kh, K), rel(Vh, V), att)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--lengths", default="1024,16384,102400")
    ap.add_argument("--dists", default="normal,lognormal_outlier,offset_uniform")
    args = ap.parse_args()
    lengths = [int(x) for x in args.lengths.split(",")]
    for dist in args.dists.split(","):
        res = study(dist, lengths)
        print("\n### inputs: %s\n" % dist)
        print("| format | K rel-RMSE | V rel-RMSE | " +
              " | ".join("attention rel-L2 @ %d" % L for L in lengths) + " |")
        print("|---|---|---|" + "---|" * len(lengths))
        for fmt in FORMATS:
            k, v, att = res[fmt]
            print("| %s | %.4f | %.4f | %s |" % (fmt, k, v, " | ".join("%.2e" % att[L] for L in lengths)))
        print("\nNVFP4 / MXFP4 attention error: " +
              ", ".join("%.2f @ %d" % (res["nvfp4"][2][L] / res["mxfp4"][2][L], L) for L in lengths))


if __name__ == "__main__":
    main()
