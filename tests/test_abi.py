"""The C ABI library loads, exports every symbol include/kvq.h declares, and
its host-side checks and size arithmetic work without a GPU."""
import ctypes
import os
import re

import pytest

import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kvq.load_library()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ["kvq_cache_create", "kvq_append", "kvq_flush_residual", "kvq_decode_attention",
              "kvq_dequantize"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert sorted(kvq.EXPORTS) == _declared_functions()


def test_cache_bytes_layout(lib):
    # NVFP4, 1 layer, B1, H2, max_len 768: header 256 + per K/V (codes + scales)
    cap = 768
    per = 2 * (1 * 2 * cap * 64 + 1 * 2 * cap * 8)
    assert kvq.kvq_cache_bytes(kvq.NVFP4, 1, 1, 2, 128, 768, 16, 0) == 256 + per
    # capacity rounds up to 768 tokens, a multiple of every attention tile
    # (384 NVFP4, 256 INT4, 128 FP8), so whole tiles can always be copied
    assert kvq.kvq_cache_bytes(kvq.FP8, 1, 1, 1, 128, 300, 0, 0) == 256 + 2 * 768 * 128
    assert kvq.kvq_cache_bytes(kvq.FP8, 1, 1, 1, 128, 769, 0, 0) == 256 + 2 * 1536 * 128
    # INT4 g64 with a 128-token BF16 ring
    b = kvq.kvq_cache_bytes(kvq.INT4, 2, 1, 1, 128, 768, 64, 128)
    assert b == 256 + 2 * 2 * (768 * 64 + 768 * 16 + 128 * 128 * 2)
    # INT8 g64: one code byte per value, {S, Z} per group, the same ring
    b = kvq.kvq_cache_bytes(kvq.INT8, 2, 1, 1, 128, 768, 64, 128)
    assert b == 256 + 2 * 2 * (768 * 128 + 768 * 16 + 128 * 128 * 2)
    # INT2 g64: four codes per byte, the same {S, Z} groups; its ring may
    # hold a whole 8192-token chunk (age tiers)
    b = kvq.kvq_cache_bytes(kvq.INT2, 2, 1, 1, 128, 768, 64, 128)
    assert b == 256 + 2 * 2 * (768 * 32 + 768 * 16 + 128 * 128 * 2)
    b = kvq.kvq_cache_bytes(kvq.INT2, 1, 1, 1, 128, 8200, 32, 8192)
    assert b == 256 + 2 * (8448 * 32 + 8448 * 32 + 8192 * 128 * 2)   # 11 x 768 tokens
    # NVFP4 and FP8 may have a BF16 ring too
    b = kvq.kvq_cache_bytes(kvq.NVFP4, 1, 1, 1, 128, 768, 16, 128)
    assert b == 256 + 2 * (768 * 64 + 768 * 8 + 128 * 128 * 2)
    b = kvq.kvq_cache_bytes(kvq.FP8, 1, 1, 1, 128, 768, 0, 48)
    assert b == 256 + 2 * (768 * 128 + 48 * 128 * 2)
    # the quantized main cache is 4x / 2x smaller than BF16 codes-wise
    bf16 = 2 * 256 * 128 * 2
    assert 2 * 256 * 64 * 4 == bf16 and 2 * 256 * 128 * 2 == bf16


@pytest.mark.parametrize("args", [
    (9, 1, 1, 1, 128, 16, 0, 0),        # bad format
    (kvq.NVFP4, 1, 1, 1, 64, 16, 0, 0),     # head_dim
    (kvq.NVFP4, 1, 1, 1, 128, 16, 32, 0),   # NVFP4 block size
    (kvq.NVFP4, 1, 1, 1, 128, 16, 0, 5000),  # ring too long
    (kvq.INT4, 1, 1, 1, 128, 16, 48, 0),    # INT4 group
    (kvq.FP8, 0, 1, 1, 128, 16, 0, 0),      # no layers
    (kvq.INT4, 1, 1, 1, 128, 16, 64, 5000),  # ring too long
    (kvq.INT8, 1, 1, 1, 128, 16, 32, 0),    # INT8 group (64 only)
    (kvq.INT8, 1, 1, 1, 128, 16, 64, 5000),  # ring too long
    (kvq.INT2, 1, 1, 1, 128, 16, 16, 0),    # INT2 group (64 or 32)
    (kvq.INT2, 1, 1, 1, 128, 16, 64, 16385),  # ring longer than a 16K chunk
    (6, 1, 1, 1, 128, 16, 64, 0),           # no format 6
    (kvq.FP8, 1, 1 << 13, 1 << 12, 128, 16, 0, 0),   # 2^25 (batch, kv head) units
    (kvq.FP8, 1 << 17, 1, 1, 128, 16, 0, 0),         # layers
    (kvq.NVFP4, 4096, 64, 64, 128, 1 << 31, 16, 0),  # petabytes
])
def test_invalid_arguments_rejected(lib, args):
    assert kvq.kvq_cache_bytes(*args) == 0
    h = ctypes.c_void_p()
    st = lib.kvq_cache_create(ctypes.byref(h), *args, None, 0, None)
    assert st in (1, 6)
    assert h.value is None
    assert len(lib.kvq_last_error()) > 0


def test_null_handles_rejected(lib):
    assert lib.kvq_cache_destroy(None) == 1
    assert lib.kvq_append(None, 0, None, None, 1, None) == 1
    assert lib.kvq_decode_attention(None, 0, None, 8, 0.0, None, None, 0, None) == 1
    assert lib.kvq_workspace_bytes(None, 8) == 0


def test_combine_and_lse_argument_checks(lib):
    """Checked on the host before anything is launched (no GPU needed)."""
    fake = ctypes.c_void_p(1 << 20)       # never dereferenced: every call below fails its checks
    assert lib.kvq_combine_partials(0, 8, 128, fake, 1024, fake, 8, fake, None, None) == 1
    assert lib.kvq_combine_partials(2, -1, 128, fake, 1024, fake, 8, fake, None, None) == 1
    assert lib.kvq_combine_partials(2, 8, 64, fake, 1024, fake, 8, fake, None, None) == 6
    assert lib.kvq_combine_partials(2, 8, 128, None, 1024, fake, 8, fake, None, None) == 1
    assert lib.kvq_combine_partials(2, 8, 128, fake, 1000, fake, 8, fake, None, None) == 1
    assert lib.kvq_combine_partials(2, 8, 128, fake, 1024, fake, 7, fake, None, None) == 1
    assert lib.kvq_combine_partials(2, 8, 128, ctypes.c_void_p((1 << 20) + 2), 1024, fake, 8, fake,
                                    None, None) == 1
    assert lib.kvq_decode_attention_lse(None, 0, None, 8, 0.0, None, None, None, 0, None) == 1
    assert len(lib.kvq_last_error()) > 0


def test_scale_renewal_option_sizes_and_checks(lib):
    # per layer and K|V: one f32 scale and one amax word per segment, in the header
    base = kvq.kvq_cache_bytes(kvq.NVFP4, 2, 1, 2, 128, 768, 16, 0)
    with_renewal = kvq.kvq_cache_bytes(kvq.NVFP4, 2, 1, 2, 128, 768, 16, 0, scale_renewal=64)
    nseg = 768 // 64
    # header: 2 layers x 4 words + status word -> counters at 48, 2 x 2 counters -> 64, segments after
    assert with_renewal - base == -(-(64 + 2 * 2 * nseg * 8) // 256) * 256 - 256
    assert kvq.kvq_cache_bytes(kvq.FP8, 1, 1, 1, 128, 100, 0, 0, scale_renewal=512) > 0
    # options the format cannot take
    assert kvq.kvq_cache_bytes(kvq.INT4, 1, 1, 1, 128, 768, 64, 0, scale_renewal=512) == 0
    assert kvq.kvq_cache_bytes(kvq.NVFP4, 1, 1, 1, 128, 768, 16, 128, scale_renewal=512) == 0
    assert kvq.kvq_cache_bytes(kvq.NVFP4, 1, 1, 1, 128, 768, 16, 0, scale_renewal=24) == 0
    assert kvq.kvq_cache_bytes(kvq.NVFP4, 1, 1, 1, 128, 768, 16, 0, scale_renewal=-16) == 0
    # no options = the plain call
    assert lib.kvq_cache_bytes_ex(kvq.NVFP4, 2, 1, 2, 128, 768, 16, 0, None) == base


def test_compact_meta_option_sizes_and_checks():
    # INT4 g64: 8 meta bytes per token (f16 S0, f16 S1, i8 Z0, i8 Z1, 2 zero bytes) instead of 16
    assert kvq.kvq_cache_bytes(kvq.INT4, 1, 1, 1, 128, 768, 64, 0, compact_meta=True) == \
        256 + 2 * (768 * 64 + 768 * 8)
    assert kvq.kvq_cache_bytes(kvq.INT4, 1, 1, 1, 128, 768, 64, 128, compact_meta=True) == \
        256 + 2 * (768 * 64 + 768 * 8 + 128 * 128 * 2)
    # INT8 g64 (f16 S0, f16 S1, i16 Z0, i16 Z1) and INT2 g64 (as INT4): 8 bytes too
    assert kvq.kvq_cache_bytes(kvq.INT8, 1, 1, 1, 128, 768, 64, 0, compact_meta=True) == \
        256 + 2 * (768 * 128 + 768 * 8)
    assert kvq.kvq_cache_bytes(kvq.INT2, 1, 1, 1, 128, 768, 64, 0, compact_meta=True) == \
        256 + 2 * (768 * 32 + 768 * 8)
    for fmt, grp in ((kvq.INT4, 32), (kvq.INT2, 32), (kvq.NVFP4, 16), (kvq.FP8, 0)):
        assert kvq.kvq_cache_bytes(fmt, 1, 1, 1, 128, 768, grp, 0, compact_meta=True) == 0


def test_paged_option_sizes_and_checks():
    """Paged caches: the planes are pools of num_pages pages of page_tokens
    tokens x kv_heads, plus a block table [batch][max_pages] in the header;
    page_tokens must be a multiple of the format's page granularity."""
    assert kvq.kvq_page_granularity(kvq.NVFP4) == 384
    assert kvq.kvq_page_granularity(kvq.INT4) == 256
    assert kvq.kvq_page_granularity(kvq.FP8) == kvq.kvq_page_granularity(kvq.INT8) == 128
    assert kvq.kvq_page_granularity(kvq.INT2) == 768    # groups of 64 (384) and of 32 (256)
    assert kvq.kvq_page_granularity(99) == 0
    # NVFP4, B2, H3, max_len 1000 -> 3 table entries per sequence; 5 pages of 384 tokens
    b = kvq.kvq_cache_bytes(kvq.NVFP4, 1, 2, 3, 128, 1000, 16, 0, page_tokens=384, num_pages=5)
    assert b == 256 + 2 * (5 * 3 * 384 * 64 + 5 * 3 * 384 * 8)
    assert kvq.kvq_cache_bytes(kvq.NVFP4, 1, 2, 3, 128, 1000, 16, 0, page_tokens=128, num_pages=5) == 0
    assert kvq.kvq_cache_bytes(kvq.NVFP4, 1, 2, 3, 128, 1000, 16, 0, page_tokens=384, num_pages=0) == 0
    assert kvq.kvq_cache_bytes(kvq.NVFP4, 1, 2, 3, 128, 1000, 16, 0, scale_renewal=512,
                               page_tokens=384, num_pages=5) == 0


def test_header_is_plain_c_and_links_from_c(tmp_path, lib):
    """include/kvq.h is valid C99 (no C++ in the boundary), and a C program
    using it links against libkvq.so and calls a host-only entry point."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_kvq.c"
    src.write_text(
        '#include "kvq.h"\n#include <stdio.h>\n'
        "int main(void) {\n"
        "  struct kvq_options o = {0};\n"
        "  o.scale_renewal = 16;\n"
        "  size_t a = kvq_cache_bytes(KVQ_NVFP4, 1, 1, 1, 128, 768, 16, 0);\n"
        "  size_t b = kvq_cache_bytes_ex(KVQ_NVFP4, 1, 1, 1, 128, 768, 16, 0, &o);\n"
        '  printf("%zu %zu\\n", a, b);\n'
        "  return (a > 0 && b > a) ? 0 : 1;\n}\n")
    libdir = os.path.dirname(kvq.LIB_PATH)
    exe = tmp_path / "use_kvq"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lkvq", "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
