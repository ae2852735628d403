"""Error studies over the oracle, at small sizes.

* NVFP4 vs MXFP4 (NVFP4 KV-cache article, section 3.2), on synthetic data.
  NVFP4 has 16-value blocks with E4M3 scales; MXFP4 has 32-value blocks
  with power-of-two scales.  NVFP4 reconstructs K and V more closely, and
  the attention output over its cache is closer to the exact one.
* Bit width: INT8 < INT4 < INT2 error, the order of the Llama-2 table in
  section 3.1 of the KV-cache long-text article.  A residual ring and a
  full-precision recent chunk (its sections 2.2 and 4.2) lower the error.
* Scale renewal every P tokens (NVFP4 article, section 3.1): it follows
  growing magnitudes that saturate a frozen scale.
"""
import pytest

from oracle import error_study


@pytest.mark.parametrize("dist", ["normal", "lognormal_outlier", "offset_uniform"])
def test_nvfp4_error_below_mxfp4(dist):
    res = error_study.study(dist, [2048], seed=77, configs={})
    nk, nv, natt = res["nvfp4"]
    mk, mv, matt = res["mxfp4"]
    assert nk < mk and nv < mv
    assert natt[2048] < matt[2048]
    # and the expected order of the other formats' reconstruction error
    assert res["int8"][0] < res["fp8"][0] < nk


def test_bit_width_order_and_rings():
    cfg = {"int2 R128": ("int2", 64, 128), "int2 + 1024 chunk": ("int2", 64, 1024),
           "int4 g32": ("int4", 32, 0)}
    res = error_study.study("normal", [1500], seed=78, configs=cfg)
    err = {k: v[2][1500] for k, v in res.items()}
    rmse = {k: v[0] for k, v in res.items()}
    assert rmse["int8"] < rmse["int4"] < rmse["int2"]
    assert err["int8"] < err["int4"] < err["int2"]
    # 2-bit steps are 5x the 4-bit ones: about 5x the reconstruction error
    assert 3.5 < rmse["int2"] / rmse["int4"] < 6.5
    # exact tokens in the ring / the recent chunk only lower the error
    assert err["int2 + 1024 chunk"] < err["int2 R128"] < err["int2"]
    # smaller groups: a finer S per group
    assert rmse["int4 g32"] < rmse["int4"]


def test_scale_renewal_follows_growth():
    res = error_study.drift_study(L=3072, period=1024, factor_log2=1, P=256, prefill=256)
    for fmt in ("nvfp4", "fp8"):
        frozen, renewed = res[(fmt, "frozen")], res[(fmt, "renewed")]
        # a frozen scale saturates the 2x and 4x regimes
        assert frozen[0] > 0.25 and renewed[0] < 0.12
        # the renewed scale lags one segment behind each jump, which the
        # attention output still feels, but less than half as much
        assert renewed[2] < 0.55 * frozen[2]


def test_study_is_deterministic():
    a = error_study.study("normal", [1024], seed=5, configs={})
    b = error_study.study("normal", [1024], seed=5, configs={})
    assert a == b


def test_compact_metadata_costs_nothing_for_int4_but_breaks_int8():
    """f16 S + i8 Z: INT4 / INT2 zero points of groups that span zero lie in
    0 .. 15 and those of groups shifted by about 7 sigma stay inside int8, so
    the compact form matches the f32 metadata; INT8 zero points of symmetric
    groups sit near 128, just past int8, so about half the groups clamp."""
    res = error_study.compact_study(L=512, seed=3)
    for name in ("N(0,1)", "shifted groups"):
        for bits in (2, 4):
            full, comp, clamped = res[(name, bits)]
            assert clamped == 0.0 and comp <= full * 1.01
    full, comp, clamped = res[("N(0,1)", 8)]
    assert 0.3 < clamped < 0.7 and comp > 3 * full


def test_compact_cache_form_costs_nothing_for_every_width():
    """With the zero point as the cache stores it (int16 for 8-bit codes),
    the compact form matches the f32 metadata for INT2, INT4 and INT8 alike,
    up to S rounded to binary16."""
    res = error_study.compact_study_cache_form(L=512, seed=3)
    for name in ("N(0,1)", "shifted groups"):
        for bits in (2, 4, 8):
            full, comp = res[(name, bits)]
            assert comp <= full * 1.02 + 1e-6, (name, bits, full, comp)
