"""The NVFP4-vs-MXFP4 comparison of the NVFP4 KV-cache article (section 3.2),
on synthetic data: NVFP4's 16-value blocks with E4M3 scales reconstruct K and
V more closely than MXFP4's 32-value blocks with power-of-two scales, and the
attention output over the quantized cache is closer to the exact one."""
import pytest

from oracle import error_study


@pytest.mark.parametrize("dist", ["normal", "lognormal_outlier", "offset_uniform"])
def test_nvfp4_error_below_mxfp4(dist):
    res = error_study.study(dist, [2048], seed=77)
    nk, nv, natt = res["nvfp4"]
    mk, mv, matt = res["mxfp4"]
    assert nk < mk and nv < mv
    assert natt[2048] < matt[2048]
    # and the expected order of the other formats' reconstruction error
    assert res["int8"][0] < res["fp8"][0] < nk


def test_study_is_deterministic():
    a = error_study.study("normal", [1024], seed=5)
    b = error_study.study("normal", [1024], seed=5)
    assert a == b
