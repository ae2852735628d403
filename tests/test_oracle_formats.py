"""Pins for the oracle's scalar formats and block encoders (CPU only).

The oracle's E2M1 / E4M3 encoders are written as grid searches; here they are
checked against independent library casts (ml_dtypes, torch) and against
exact properties of the formats: grid round trips, scaling by powers of two,
error bounds, and the INT affine min/max invariants of the affine formulas in
section 2.1 of "KV缓存量化技术：提升大模型长文本生成效率".
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _sweep_points(grid, lo, hi):
    """Dense float32 sweep plus every grid point, midpoint and their float32
    neighbours (the places where a rounding mistake would show)."""
    pts = [np.linspace(lo, hi, 200001, dtype=np.float32)]
    g = np.array(sorted(set(grid)), np.float64)
    mids = (g[1:] + g[:-1]) / 2
    special = np.concatenate([g, mids]).astype(np.float32)
    pts.append(special)
    pts.append(np.nextafter(special, np.float32(np.inf)))
    pts.append(np.nextafter(special, np.float32(-np.inf)))
    x = np.concatenate(pts)
    return np.concatenate([x, -x, np.array([0.0, -0.0], np.float32)])


E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e4m3_values():
    return [float(np.uint8(c).view(ml_dtypes.float8_e4m3fn)) for c in range(0x7F)]


def test_e2m1_encode_matches_ml_dtypes():
    x = _sweep_points(E2M1_VALUES, 0.0, 8.0)
    ours = oracle.e2m1_encode(x)
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(ours, ref)


def test_e2m1_decode_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    assert np.array_equal(oracle.e2m1_decode(codes), ref)
    # sign of zero kept
    assert math.copysign(1.0, float(oracle.e2m1_decode(np.uint8(8)))) == -1.0


def test_e2m1_ties_to_even_and_saturation():
    # midpoints between neighbouring grid values go to the even code
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 1e30, -0.25, -5.0], np.float32)
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(oracle.e2m1_encode(x), ref)
    assert list(oracle.e2m1_encode(x)[:7]) == [0, 2, 2, 4, 4, 6, 6]
    assert oracle.e2m1_encode(np.float32(1e30)) == 7
    assert oracle.e2m1_encode(np.float32(-1e30)) == 15


def test_e4m3_encode_matches_ml_dtypes_and_torch():
    # ml_dtypes / torch cast to NaN above 464; below that all three agree.
    x = _sweep_points(_e4m3_values(), 0.0, 464.0)
    x = x[np.abs(x) <= 464.0]
    ours = oracle.e4m3_encode(x)
    ref = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, ref)
    ref_t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref_t)


def test_e4m3_subnormal_sweep_matches_ml_dtypes():
    x = _sweep_points(_e4m3_values()[:16], 0.0, 2.0 ** -5)
    assert np.array_equal(oracle.e4m3_encode(x), x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8))


def test_e4m3_saturates_to_448():
    x = np.array([448.0, 465.0, 1e6, np.float32(3e38), -500.0], np.float32)
    assert list(oracle.e4m3_encode(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_e4m3_decode_all_finite_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    ref = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    ours = oracle.e4m3_decode(codes)
    assert np.array_equal(ours, ref)
    assert np.isnan(oracle.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


@pytest.mark.parametrize("k", [-3, 0, 5])
def test_fp8_round_trip_all_codes(k):
    """Every finite E4M3 code times a power-of-two scale encodes back to itself."""
    s = float(2.0 ** k)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    x = oracle.e4m3_decode(codes) * np.float32(s)
    back = oracle.fp8_quantize(x, s)
    assert np.array_equal(back, codes)
    assert np.array_equal(oracle.fp8_dequantize(back, s), x)


def test_fp8_relative_error_bound():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(20000).astype(np.float32)
    s = oracle.global_scale(oracle.FP8, oracle.amax(x))
    xh = oracle.fp8_dequantize(oracle.fp8_quantize(x, s), s)
    u = np.abs(x) / s
    normal = u >= 2.0 ** -6
    rel = np.abs(xh[normal] - x[normal]) / np.abs(x[normal])
    assert rel.max() <= 2.0 ** -4 * (1 + 1e-6)
    # subnormal range: absolute error at most half the subnormal step
    assert np.all(np.abs(xh[~normal] - x[~normal]) <= s * 2.0 ** -10 * (1 + 1e-6))


def test_global_scales():
    assert oracle.global_scale(oracle.NVFP4, 2688.0) == 1.0
    assert oracle.global_scale(oracle.FP8, 448.0) == 1.0
    assert oracle.global_scale(oracle.NVFP4, 0.0) == 1.0
    assert oracle.global_scale(oracle.FP8, 0.0) == 1.0
    assert oracle.amax(np.array([-3.5, 2.0, 0.0], np.float32)) == 3.5


# --------------------------------------------------------------------------
# NVFP4 blocks
# --------------------------------------------------------------------------

def _nvfp4_grid_input(rng, rows, D, g):
    """Rows whose blocks are E2M1 values x one E4M3 block scale x g, each block
    holding a +-6 so that block amax / 6 is exactly the block scale."""
    e2m1 = rng.integers(0, 16, size=(rows, D)).astype(np.uint8)
    e2m1[:, ::16] = rng.choice([7, 15], size=(rows, D // 16))
    # normal E4M3 block scales (subnormal ones would not survive /6 exactly)
    bs = rng.integers(0x08, 0x7F, size=(rows, D // 16)).astype(np.uint8)
    vals = oracle.e2m1_decode(e2m1).astype(np.float64)
    bsv = oracle.e4m3_decode(bs).astype(np.float64)
    x = vals * np.repeat(bsv, 16, axis=1) * g
    return x.astype(np.float32), e2m1, bs


@pytest.mark.parametrize("g", [1.0, 2.0 ** -7, 2.0 ** 5])
def test_nvfp4_grid_round_trip(g):
    rng = np.random.default_rng(11)
    x, e2m1, bs = _nvfp4_grid_input(rng, 64, 128, g)
    codes, scales = oracle.nvfp4_quantize(x, g)
    assert np.array_equal(scales, bs)
    unpacked = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(64, 128)
    # a zero may come back as either signed zero only if the input was -0:
    assert np.array_equal(unpacked, e2m1)
    assert np.array_equal(oracle.nvfp4_dequantize(codes, scales, g), x)


def test_nvfp4_packing_low_nibble_first():
    g = 1.0
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.0     # code 7, low nibble of byte 0
    x[0, 1] = -1.0    # code 0xA, high nibble of byte 0
    x[0, 3] = 0.5     # code 1, high nibble of byte 1
    codes, scales = oracle.nvfp4_quantize(x, g)
    assert scales[0, 0] == oracle.e4m3_encode(np.float32(1.0))
    assert codes[0, 0] == 0xA7
    assert codes[0, 1] == 0x10


@pytest.mark.parametrize("k", [-6, -1, 3, 9])
def test_nvfp4_power_of_two_invariance(k):
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((40, 128)) * rng.lognormal(0, 1, (40, 1))).astype(np.float32)
    g = oracle.global_scale(oracle.NVFP4, oracle.amax(x))
    c0, s0 = oracle.nvfp4_quantize(x, g)
    xs = (x * np.float32(2.0 ** k)).astype(np.float32)
    gs = oracle.global_scale(oracle.NVFP4, oracle.amax(xs))
    assert gs == g * 2.0 ** k
    c1, s1 = oracle.nvfp4_quantize(xs, gs)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)


def test_nvfp4_error_bound_and_zero_block():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((300, 128)).astype(np.float32)
    x[7, 16:32] = 0.0                           # an all-zero block
    g = oracle.global_scale(oracle.NVFP4, oracle.amax(x))
    codes, scales = oracle.nvfp4_quantize(x, g)
    assert scales[7, 1] == 0 and np.all(codes[7, 8:16] == 0)
    xh = oracle.nvfp4_dequantize(codes, scales, g)
    eff = oracle.e4m3_decode(scales).astype(np.float64) * g
    err = np.abs(xh.astype(np.float64) - x).reshape(300, 8, 16).max(axis=2)
    # half the widest grid step (4 -> 6) is one block unit
    assert np.all(err <= eff * (1 + 1e-6))
    # and the block maximum never saturates by more than the E4M3 rounding
    assert np.all(np.abs(x).reshape(300, 8, 16).max(axis=2) <= 6 * eff * (1 + 2.0 ** -4) + 1e-30)


def test_nvfp4_negative_zero_code():
    g = 1.0
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.0
    x[0, 2] = -0.1      # rounds to -0 on the grid (sign kept, as ml_dtypes does)
    codes, _ = oracle.nvfp4_quantize(x, g)
    assert codes[0, 1] & 0xF == 0x8


# --------------------------------------------------------------------------
# INT4 affine groups
# --------------------------------------------------------------------------

@pytest.mark.parametrize("k", [-9, -2, 0, 4])
def test_int4_grid_round_trip(k):
    """x = (q - Z0) * 2^k with q covering 0 and 15 in every group gives back
    S = 2^k, Z = Z0 and q exactly."""
    rng = np.random.default_rng(21)
    rows, D, grp = 50, 128, 64
    q = rng.integers(0, 16, size=(rows, D))
    q[:, 0::grp] = 0
    q[:, 1::grp] = 15
    Z0 = rng.integers(-20, 36, size=(rows, D // grp))
    S0 = 2.0 ** k
    x = ((q - np.repeat(Z0, grp, axis=1)) * S0).astype(np.float32)
    codes, S, Z = oracle.int4_quantize(x, grp)
    assert np.all(S == np.float32(S0))
    assert np.array_equal(Z, Z0)
    unpacked = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(rows, D)
    assert np.array_equal(unpacked, q)
    assert np.array_equal(oracle.int4_dequantize(codes, S, Z, grp), x)


def test_int4_min_max_invariants_and_error():
    rng = np.random.default_rng(22)
    rows, D, grp = 2000, 128, 64
    x = (rng.standard_normal((rows, D)) + rng.uniform(-1, 1, (1, D))).astype(np.float32)
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    codes, S, Z = oracle.int4_quantize(x, grp)
    q = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(rows, D).astype(np.int64)
    xg = x.reshape(rows, 2, grp)
    qg = q.reshape(rows, 2, grp)
    amin = xg.argmin(axis=2)
    amax = xg.argmax(axis=2)
    qmin = np.take_along_axis(qg, amin[..., None], axis=2)[..., 0]
    qmax = np.take_along_axis(qg, amax[..., None], axis=2)[..., 0]
    assert np.all(qmin == 0)
    # the maximum maps to 15, or to 14 when the roundings of max/S and min/S
    # fall on opposite sides of a half-integer (rare)
    assert np.all((qmax == 15) | (qmax == 14))
    assert (qmax == 15).mean() > 0.99
    # reconstruction error at most S/2 (+ rounding of x/S) where nothing clamps
    xh = oracle.int4_dequantize(codes, S, Z, grp).reshape(rows, 2, grp)
    Sg = S[..., None].astype(np.float64)
    inside = (qg > 0) & (qg < 15)
    err = np.abs(xh.astype(np.float64) - xg)
    assert np.all(err[inside] <= (0.5 * Sg * (1 + 1e-5) + 1e-7 * np.abs(xg))[inside] + 1e-12)


def test_int4_constant_and_zero_groups():
    x = np.zeros((3, 128), np.float32)
    x[0, :64] = 2.5
    x[1, 64:] = -1.75
    codes, S, Z = oracle.int4_quantize(x, 64)
    assert S[0, 0] == 2.5 and Z[0, 0] == -1
    assert S[1, 1] == 1.75 and Z[1, 1] == 1
    assert S[2, 0] == 1.0 and Z[2, 0] == 0
    assert np.all(codes == 0)
    assert np.array_equal(oracle.int4_dequantize(codes, S, Z, 64), x)


@pytest.mark.parametrize("k", [-5, 3])
def test_int4_power_of_two_invariance(k):
    rng = np.random.default_rng(23)
    x = rng.standard_normal((100, 128)).astype(np.float32)
    c0, S0, Z0 = oracle.int4_quantize(x, 64)
    c1, S1, Z1 = oracle.int4_quantize(x * np.float32(2.0 ** k), 64)
    assert np.array_equal(c0, c1) and np.array_equal(Z0, Z1)
    assert np.array_equal(S1, S0 * np.float32(2.0 ** k))


# --------------------------------------------------------------------------
# INT8 affine groups (the same scheme with 8-bit codes, one per byte)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("k", [-12, -3, 0, 2])
def test_int8_grid_round_trip(k):
    """x = (q - Z0) * 2^k with q covering 0 and 255 in every group gives back
    S = 2^k, Z = Z0 and q exactly."""
    rng = np.random.default_rng(31)
    rows, D, grp = 50, 128, 64
    q = rng.integers(0, 256, size=(rows, D))
    q[:, 0::grp] = 0
    q[:, 1::grp] = 255
    Z0 = rng.integers(-40, 300, size=(rows, D // grp))
    S0 = 2.0 ** k
    x = ((q - np.repeat(Z0, grp, axis=1)) * S0).astype(np.float32)
    codes, S, Z = oracle.int8_quantize(x, grp)
    assert np.all(S == np.float32(S0))
    assert np.array_equal(Z, Z0)
    assert np.array_equal(codes.astype(np.int64), q)
    assert np.array_equal(oracle.int8_dequantize(codes, S, Z, grp), x)


def test_int8_min_max_invariants_and_error():
    rng = np.random.default_rng(32)
    rows, D, grp = 2000, 128, 64
    x = (rng.standard_normal((rows, D)) + rng.uniform(-1, 1, (1, D))).astype(np.float32)
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    codes, S, Z = oracle.int8_quantize(x, grp)
    q = codes.astype(np.int64)
    xg = x.reshape(rows, 2, grp)
    qg = q.reshape(rows, 2, grp)
    amin = xg.argmin(axis=2)
    amax = xg.argmax(axis=2)
    qmin = np.take_along_axis(qg, amin[..., None], axis=2)[..., 0]
    qmax = np.take_along_axis(qg, amax[..., None], axis=2)[..., 0]
    assert np.all(qmin == 0)
    # the maximum maps to 255, or to 254 when the roundings of max/S and
    # min/S fall on opposite sides of a half-integer (rare)
    assert np.all((qmax == 255) | (qmax == 254))
    assert (qmax == 255).mean() > 0.99
    # reconstruction error at most S/2 (+ rounding of x/S) where nothing clamps
    xh = oracle.int8_dequantize(codes, S, Z, grp).reshape(rows, 2, grp)
    Sg = S[..., None].astype(np.float64)
    inside = (qg > 0) & (qg < 255)
    err = np.abs(xh.astype(np.float64) - xg)
    assert np.all(err[inside] <= (0.5 * Sg * (1 + 1e-5) + 1e-7 * np.abs(xg))[inside] + 1e-12)
    # 8 bits: the step is (max - min) / 255, 17x finer than INT4's / 15
    S4 = oracle.int4_quantize(x, grp)[1]
    assert np.allclose(S4 / S, 255.0 / 15.0, rtol=1e-5)


def test_int8_constant_and_zero_groups():
    x = np.zeros((3, 128), np.float32)
    x[0, :64] = 2.5
    x[1, 64:] = -1.75
    codes, S, Z = oracle.int8_quantize(x, 64)
    assert S[0, 0] == 2.5 and Z[0, 0] == -1
    assert S[1, 1] == 1.75 and Z[1, 1] == 1
    assert S[2, 0] == 1.0 and Z[2, 0] == 0
    assert np.all(codes == 0)
    assert np.array_equal(oracle.int8_dequantize(codes, S, Z, 64), x)


@pytest.mark.parametrize("k", [-5, 3])
def test_int8_power_of_two_invariance(k):
    rng = np.random.default_rng(33)
    x = rng.standard_normal((100, 128)).astype(np.float32)
    c0, S0, Z0 = oracle.int8_quantize(x, 64)
    c1, S1, Z1 = oracle.int8_quantize(x * np.float32(2.0 ** k), 64)
    assert np.array_equal(c0, c1) and np.array_equal(Z0, Z1)
    assert np.array_equal(S1, S0 * np.float32(2.0 ** k))


def test_int8_brute_force_against_exhaustive_code_search():
    """For sampled values, the code is one of the integers 0..255 whose
    reconstruction (q - Z) * S lies nearest to the value, found by trying
    all 256 codes (ties admit either neighbour)."""
    rng = np.random.default_rng(34)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    codes, S, Z = oracle.int8_quantize(x, 64)
    cand = np.arange(256, dtype=np.float64)
    for r in range(0, 64, 7):
        for g in range(2):
            s, z = np.float64(S[r, g]), int(Z[r, g])
            for i in range(0, 64, 5):
                v = np.float64(x[r, 64 * g + i])
                dist = np.abs((cand - z) * s - v)
                best = np.flatnonzero(dist <= dist.min() * (1 + 1e-9) + 1e-30)
                assert codes[r, 64 * g + i] in best


# --------------------------------------------------------------------------
# INT2 affine groups (the same scheme with 2-bit codes, four per byte)
# --------------------------------------------------------------------------

def _int2_unpack(codes, D):
    rows = codes.shape[0]
    return np.stack([(codes >> (2 * j)) & 3 for j in range(4)], axis=-1).reshape(rows, D)


@pytest.mark.parametrize("k", [-10, -1, 0, 5])
@pytest.mark.parametrize("grp", [32, 64, 128])
def test_int2_grid_round_trip(k, grp):
    """x = (q - Z0) * 2^k with q covering 0 and 3 in every group gives back
    S = 2^k, Z = Z0 and q exactly; the lowest index sits in the lowest two
    bits of its byte."""
    rng = np.random.default_rng(41)
    rows, D = 50, 128
    q = rng.integers(0, 4, size=(rows, D))
    q[:, 0::grp] = 0
    q[:, 1::grp] = 3
    Z0 = rng.integers(-6, 10, size=(rows, D // grp))
    S0 = 2.0 ** k
    x = ((q - np.repeat(Z0, grp, axis=1)) * S0).astype(np.float32)
    codes, S, Z = oracle.int2_quantize(x, grp)
    assert codes.shape == (rows, D // 4)
    assert np.all(S == np.float32(S0))
    assert np.array_equal(Z, Z0)
    assert np.array_equal(_int2_unpack(codes, D), q)
    assert codes[0, 0] == q[0, 0] | (q[0, 1] << 2) | (q[0, 2] << 4) | (q[0, 3] << 6)
    assert np.array_equal(oracle.int2_dequantize(codes, S, Z, grp), x)


def test_int2_min_max_invariants_and_error():
    rng = np.random.default_rng(42)
    rows, D, grp = 2000, 128, 64
    x = (rng.standard_normal((rows, D)) + rng.uniform(-1, 1, (1, D))).astype(np.float32)
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    codes, S, Z = oracle.int2_quantize(x, grp)
    q = _int2_unpack(codes, D).astype(np.int64)
    xg = x.reshape(rows, 2, grp)
    qg = q.reshape(rows, 2, grp)
    amin = xg.argmin(axis=2)
    amax = xg.argmax(axis=2)
    qmin = np.take_along_axis(qg, amin[..., None], axis=2)[..., 0]
    qmax = np.take_along_axis(qg, amax[..., None], axis=2)[..., 0]
    assert np.all(qmin == 0)
    # the maximum maps to 3, or to 2 when the roundings of max/S and min/S
    # fall on opposite sides of a half-integer
    assert np.all((qmax == 3) | (qmax == 2))
    assert (qmax == 3).mean() > 0.99
    # reconstruction error at most S/2 (+ rounding of x/S) where nothing clamps
    xh = oracle.int2_dequantize(codes, S, Z, grp).reshape(rows, 2, grp)
    Sg = S[..., None].astype(np.float64)
    inside = (qg > 0) & (qg < 3)
    err = np.abs(xh.astype(np.float64) - xg)
    assert np.all(err[inside] <= (0.5 * Sg * (1 + 1e-5) + 1e-7 * np.abs(xg))[inside] + 1e-12)
    # 2 bits: the step is (max - min) / 3, 5x coarser than INT4's / 15
    S4 = oracle.int4_quantize(x, grp)[1]
    assert np.allclose(S / S4, 15.0 / 3.0, rtol=1e-5)


def test_int2_constant_and_zero_groups():
    x = np.zeros((3, 128), np.float32)
    x[0, :64] = 2.5
    x[1, 64:] = -1.75
    codes, S, Z = oracle.int2_quantize(x, 64)
    assert S[0, 0] == 2.5 and Z[0, 0] == -1
    assert S[1, 1] == 1.75 and Z[1, 1] == 1
    assert S[2, 0] == 1.0 and Z[2, 0] == 0
    assert np.all(codes == 0)
    assert np.array_equal(oracle.int2_dequantize(codes, S, Z, 64), x)


@pytest.mark.parametrize("k", [-5, 3])
def test_int2_power_of_two_invariance(k):
    rng = np.random.default_rng(43)
    x = rng.standard_normal((100, 128)).astype(np.float32)
    c0, S0, Z0 = oracle.int2_quantize(x, 64)
    c1, S1, Z1 = oracle.int2_quantize(x * np.float32(2.0 ** k), 64)
    assert np.array_equal(c0, c1) and np.array_equal(Z0, Z1)
    assert np.array_equal(S1, S0 * np.float32(2.0 ** k))


def test_int2_brute_force_against_exhaustive_code_search():
    """Every code is one of the integers 0..3 whose reconstruction
    (q - Z) * S lies nearest to the value (ties admit either neighbour)."""
    rng = np.random.default_rng(44)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    codes, S, Z = oracle.int2_quantize(x, 32)
    q = _int2_unpack(codes, 128)
    cand = np.arange(4, dtype=np.float64)
    for r in range(64):
        for d in range(128):
            s, z = np.float64(S[r, d // 32]), int(Z[r, d // 32])
            dist = np.abs((cand - z) * s - np.float64(x[r, d]))
            best = np.flatnonzero(dist <= dist.min() * (1 + 1e-9) + 1e-30)
            assert q[r, d] in best


# --------------------------------------------------------------------------
# Compact group metadata (f16 S, i8 Z) for the INT formats
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("k", [-14, -3, 0, 9])
def test_compact_grid_round_trip(bits, k):
    """x = (q - Z0) * 2^k with q covering 0 and 2^bits - 1 in every group and
    Z0 inside int8: S = 2^k exactly in binary16, Z = Z0, q exact."""
    rng = np.random.default_rng(51 + bits)
    rows, D, grp = 40, 128, 64
    top = 2 ** bits - 1
    q = rng.integers(0, top + 1, size=(rows, D))
    q[:, 0::grp] = 0
    q[:, 1::grp] = top
    Z0 = rng.integers(-128, 128, size=(rows, D // grp))
    x = ((q - np.repeat(Z0, grp, axis=1)) * 2.0 ** k).astype(np.float32)
    codes, S, Z = oracle.int_compact_quantize(x, bits, grp)
    assert S.dtype == np.float16 and Z.dtype == np.int8
    assert np.all(S == np.float16(2.0 ** k))
    assert np.array_equal(Z.astype(np.int64), Z0)
    assert np.array_equal(codes.astype(np.int64), q)
    assert np.array_equal(oracle.int_compact_dequantize(codes, S, Z, grp), x)


def test_compact_matches_f32_metadata_on_its_grid():
    """Where S is exact in binary16 and Z fits int8, the compact codes are the
    f32-metadata codes."""
    rng = np.random.default_rng(52)
    q = rng.integers(0, 16, size=(30, 128))
    q[:, 0::64] = 0
    q[:, 1::64] = 15
    Z0 = rng.integers(-20, 36, size=(30, 2))
    x = ((q - np.repeat(Z0, 64, axis=1)) * 0.125).astype(np.float32)
    c16, S16, Z16 = oracle.int_compact_quantize(x, 4, 64)
    c32, S32, Z32 = oracle.int4_quantize(x, 64)
    unpacked = np.stack([c32 & 0xF, c32 >> 4], axis=-1).reshape(30, 128)
    assert np.array_equal(c16, unpacked)
    assert np.array_equal(S16.astype(np.float32), S32) and np.array_equal(Z16.astype(np.int32), Z32)


def test_compact_error_bound_and_z_clamp():
    rng = np.random.default_rng(53)
    # groups spanning zero: nothing clamps, error within S/2 of the stored S
    x = torch.from_numpy(rng.standard_normal((500, 128)).astype(np.float32)).bfloat16().float().numpy()
    q, S, Z = oracle.int_compact_quantize(x, 4, 64)
    xh = oracle.int_compact_dequantize(q, S, Z, 64)
    Sg = np.repeat(S.astype(np.float64), 64, axis=1)
    inside = (q > 0) & (q < 15)
    assert np.all(np.abs(xh - x)[inside] <= 0.5 * Sg[inside] * (1 + 1e-3) + 1e-6 * np.abs(x)[inside])
    # a group far above zero: its true Z is below -128, so Z clamps and the
    # codes saturate at 15; no reconstruction exceeds (15 + 128) * S
    y = (10.0 + 0.1 * rng.standard_normal((4, 128))).astype(np.float32)
    q, S, Z = oracle.int_compact_quantize(y, 4, 64)
    assert np.all(Z == -128)
    yh = oracle.int_compact_dequantize(q, S, Z, 64)
    top = (15 + 128) * np.repeat(S.astype(np.float32), 64, axis=1)
    assert np.all(yh <= top) and np.any(q == 15)


@pytest.mark.parametrize("k", [-10, 0, 7])
def test_compact_int16_zero_point_round_trip(k):
    """8-bit codes with int16 zero points: x = (q - Z0) * 2^k with Z0 over
    the whole int16 range and q covering 0 and 255 gives S = 2^k, Z = Z0 and
    q exactly; symmetric groups (Z near 128) no longer clamp."""
    rng = np.random.default_rng(55)
    q = rng.integers(0, 256, size=(40, 128))
    q[:, 0::64] = 0
    q[:, 1::64] = 255
    Z0 = rng.integers(-2000, 2000, size=(40, 2))
    Z0[0] = [128, 127]
    x = ((q - np.repeat(Z0, 64, axis=1)) * 2.0 ** k).astype(np.float32)
    codes, S, Z = oracle.int_compact_quantize(x, 8, 64, zbits=16)
    assert Z.dtype == np.int16 and np.all(S == np.float16(2.0 ** k))
    assert np.array_equal(Z.astype(np.int64), Z0) and np.array_equal(codes.astype(np.int64), q)
    assert np.array_equal(oracle.int_compact_dequantize(codes, S, Z, 64), x)
    assert oracle.compact_zbits(8) == 16 and oracle.compact_zbits(4) == oracle.compact_zbits(2) == 8


def test_compact_int8_with_int16_zero_matches_f32_metadata_on_its_grid():
    """Where S is exact in binary16, the compact INT8 codes and zero points
    (int16) equal the f32-metadata ones, including symmetric groups."""
    rng = np.random.default_rng(56)
    q = rng.integers(0, 256, size=(30, 128))
    q[:, 0::64] = 0
    q[:, 1::64] = 255
    Z0 = rng.integers(100, 160, size=(30, 2))
    x = ((q - np.repeat(Z0, 64, axis=1)) * 0.0625).astype(np.float32)
    c16, S16, Z16 = oracle.int_compact_quantize(x, 8, 64, zbits=16)
    c32, S32, Z32 = oracle.int8_quantize(x, 64)
    assert np.array_equal(c16, c32)
    assert np.array_equal(S16.astype(np.float32), S32) and np.array_equal(Z16.astype(np.int32), Z32)


def test_compact_power_of_two_invariance():
    rng = np.random.default_rng(54)
    x = rng.standard_normal((50, 128)).astype(np.float32)
    a = oracle.int_compact_quantize(x, 4, 64)
    b = oracle.int_compact_quantize(x * np.float32(8.0), 4, 64)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[2], b[2])
    assert np.array_equal(b[1].astype(np.float32), a[1].astype(np.float32) * 8)


def test_compact_storage_bytes():
    assert oracle.cache_storage_bytes_per_token_head(oracle.INT4, 128, 64, compact=True) == 70
    # INT8 keeps an int16 zero point (4 bytes per group)
    assert oracle.cache_storage_bytes_per_token_head(oracle.INT8, 128, 64, compact=True) == 136
    assert oracle.cache_storage_bytes_per_token_head(oracle.INT2, 128, 64, compact=True) == 38


# --------------------------------------------------------------------------
# MXFP4 (an external definition, for the comparison of [P1] section 3.2)
# --------------------------------------------------------------------------

E2M1_VALUES = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


@pytest.mark.parametrize("k", [-20, -3, 0, 5])
def test_mxfp4_grid_round_trip(k):
    """Blocks of E2M1 grid values times 2^k whose largest magnitude is 4 or 6
    (exponent 2) come back exactly, with the E8M0 scale byte k + 127."""
    rng = np.random.default_rng(41)
    rows, D = 40, 128
    mag = rng.integers(0, 8, size=(rows, D))
    sign = rng.choice([-1.0, 1.0], size=(rows, D))
    mag[:, 0::32] = rng.choice([6, 7], size=(rows, D // 32))     # 4.0 or 6.0 in each block
    x = (sign * E2M1_VALUES[mag] * 2.0 ** k).astype(np.float32)
    codes, scales = oracle.mxfp4_quantize(x)
    assert np.all(scales == k + 127)
    assert np.array_equal(oracle.mxfp4_dequantize(codes, scales), x)


def test_mxfp4_scale_is_power_of_two_below_the_block_max():
    """X = 2^(floor(log2 amax) - 2): the block max lands in [4, 8) * X, and
    values in [6, 8) * X saturate to 6 * X."""
    rng = np.random.default_rng(42)
    x = (rng.standard_normal((500, 128)) * rng.lognormal(0, 2, (500, 1))).astype(np.float32)
    codes, scales = oracle.mxfp4_quantize(x)
    X = np.ldexp(1.0, scales.astype(np.int64) - 127)                   # [500, 4]
    amax = np.abs(x.reshape(500, 4, 32)).max(axis=2)
    ratio = amax / X
    assert np.all((ratio >= 4.0) & (ratio < 8.0))
    xh = oracle.mxfp4_dequantize(codes, scales).reshape(500, 4, 32)
    assert np.all(np.abs(xh) <= 6.0 * X[..., None])
    # the largest element saturates exactly when it is at or beyond 6 X
    big = ratio >= 6.0
    top = np.abs(xh).max(axis=2)
    assert np.all(top[big] == 6.0 * X[big])


def test_mxfp4_zero_block_and_element_rounding_match_e2m1():
    x = np.zeros((2, 128), np.float32)
    x[1] = np.random.default_rng(43).standard_normal(128).astype(np.float32)
    codes, scales = oracle.mxfp4_quantize(x)
    assert np.all(scales[0] == 0) and np.all(codes[0] == 0)
    # element codes are the (pinned) E2M1 encoder of x / X
    X = np.ldexp(np.float32(1.0), scales[1].astype(np.int64) - 127).astype(np.float32)
    expect = oracle.e2m1_encode(x[1] / np.repeat(X, 32))
    got = np.stack([codes[1] & 0xF, codes[1] >> 4], axis=-1).reshape(128)
    assert np.array_equal(got, expect)
