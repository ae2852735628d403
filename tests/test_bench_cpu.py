"""bench.py pieces that need no GPU: the algorithmic byte model, the
weak-scaling arithmetic and the reference arm (the oracle on the host)."""
import importlib.util
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_token_bytes_per_format(bench):
    W = bench.W
    # K + V per token per KV head: codes + scales (NVFP4 64 + 8, INT4 64 + 16,
    # INT8 128 + 16, FP8 128), twice
    assert bench.token_bytes(W.WORKLOADS["gqa_nvfp4_32k"]) == 144
    assert bench.token_bytes(W.WORKLOADS["mha_int4_16k"]) == 160
    assert bench.token_bytes(W.WORKLOADS["mha_int8_16k"]) == 288
    assert bench.token_bytes(W.WORKLOADS["gqa_fp8_32k"]) == 256
    assert bench.token_bytes(W.WORKLOADS["mha_int2_16k"]) == 96


def test_decode_and_step_bytes(bench):
    w = bench.W.WORKLOADS["gqa_nvfp4_32k"]
    L = w.context + 1
    # the cache of all 64 units, plus Q (bf16) and O (f32)
    assert bench.decode_bytes(w, L, 0) == 64 * L * 144 + 8 * 32 * 128 * 6
    # the fused step also reads the new token (bf16 K, V) and writes it quantized
    assert bench.step_bytes(w, L, 0) == bench.decode_bytes(w, L, 0) + 64 * (512 + 144)
    wi = bench.W.WORKLOADS["mha_int4_16k"]
    # ring tokens are read as bf16; the ring write is bf16 too
    assert bench.decode_bytes(wi, 16384, 1) == 128 * (16384 * 160 + 512) + 4 * 32 * 128 * 6
    assert bench.step_bytes(wi, 16384, 1) == bench.decode_bytes(wi, 16384, 1) + 128 * (512 + 512)


def test_weak_scaling_value_single_rank(bench):
    # (the max over ranks with world > 1 is covered by test_dist_replicas.py)
    ms, value = bench.weak_scaling_value(0.05, 8, 1)
    assert ms == pytest.approx(0.05) and value == pytest.approx(8 / 0.05e-3)


def test_reference_arm_runs_the_oracle():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_nvfp4", "--steps", "2", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"] == "tiny_nvfp4"


def test_staged_inputs_round_trip(bench):
    """The end-to-end leg's single staging buffer: each view sees exactly its
    tensor, and each piece starts on a 16-byte boundary."""
    import torch
    g = torch.Generator().manual_seed(0)
    k = torch.randn(8, 8, 1, 128, generator=g).bfloat16()
    v = torch.randn(8, 8, 1, 128, generator=g).bfloat16()
    q = torch.randn(8, 32, 128, generator=g).bfloat16()
    buf, offs = bench.staged_inputs([k, v, q], pinned=False)
    assert buf.numel() == k.numel() + v.numel() + q.numel()
    assert offs == [0, k.numel(), k.numel() + v.numel()]
    dev = buf.clone()                      # stands in for the device copy
    kd, vd, qd = bench.staged_views(dev, [k, v, q])
    for a, b in ((kd, k), (vd, v), (qd, q)):
        assert a.shape == b.shape and a.is_contiguous() and torch.equal(a, b)
        assert (a.data_ptr() - dev.data_ptr()) % 16 == 0
    with pytest.raises(AssertionError):
        bench.staged_inputs([torch.zeros(3, dtype=torch.bfloat16), q], pinned=False)


def test_traffic_record_follows_the_kernel_sources(bench):
    """roofline.traffic is the committed capture only while the kernel
    sources hash to the recorded value; the note says which case holds."""
    import json
    rec = json.load(open(bench.TRAFFIC_FILE))
    current = rec["kernel_sha256"] == bench.kernel_source_hash()
    t = bench.recorded_traffic("gqa_nvfp4_32k")
    note = bench.traffic_note("gqa_nvfp4_32k")
    if current:
        assert t == rec["workloads"]["gqa_nvfp4_32k"]["dram_bytes_per_launch"]
        assert note.startswith("ncu capture")
    else:
        assert t is None and note.startswith("null")
    assert bench.recorded_traffic("no_such_workload") is None


def test_variant_workloads(bench):
    """The cache-option workloads: byte model and the oracle sample of one
    unit (a short context, so the sample stays quick)."""
    import dataclasses
    W = bench.W
    assert bench.token_bytes(W.WORKLOADS["mha_int4_16k_compact"]) == 144
    assert bench.token_bytes(W.WORKLOADS["gqa_nvfp4_32k_renew512"]) == 144
    assert W.WORKLOADS["gqa_nvfp4_32k_renew512"].context % 512 != 0
    for name in ("mha_int4_16k_compact", "gqa_nvfp4_32k_renew512", "gqa_nvfp4_32k_ring128"):
        w = dataclasses.replace(W.WORKLOADS[name], context=1100)
        assert bench.oracle_decode_sample(w, [(0, 0)], 1101) > 0
