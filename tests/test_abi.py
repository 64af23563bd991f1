"""The C ABI library loads and exports every symbol include/mxq.h declares;
host-only behaviour (size queries, statuses returned before any CUDA call).
No kernel runs here."""
import os
import re
import subprocess

import pytest

import oracle
from block_scaled_microscaling_b200 import build as mxq_build
from block_scaled_microscaling_b200 import mxq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxq.h")
FMTS = ["axs6", "mxfp6_e2m3", "mxfp6_e3m2", "mxfp8", "mxfp4"]


@pytest.fixture(scope="module")
def L():
    mxq_build.build()
    return mxq.lib()


def declared_symbols():
    src = open(HEADER).read()
    return re.findall(r"MXQ_API\s+[\w\s\*]+?\b(mxq_\w+)\s*\(", src)


def test_exports_every_declared_symbol(L):
    syms = declared_symbols()
    assert len(syms) == 22
    out = subprocess.run(["nm", "-D", "--defined-only", mxq.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(mxq_\w+)", out))
    for s in syms:
        assert s in exported, s
        assert hasattr(L, s)
    assert set(mxq.EXPORTS) == set(syms)


def test_enum_values_match_header():
    src = open(HEADER).read()
    for name, v in [("MXQ_AXS6", 0), ("MXQ_MXFP6_E2M3", 1), ("MXQ_MXFP6_E3M2", 2), ("MXQ_MXFP8_E4M3", 3),
                    ("MXQ_MXFP4_E2M1", 4), ("MXQ_F32", 0), ("MXQ_BF16", 1), ("MXQ_OK", 0),
                    ("MXQ_ERR_INVALID_ARG", 1), ("MXQ_ERR_SHAPE", 2), ("MXQ_ERR_ALIGN", 3),
                    ("MXQ_ERR_UNSUPPORTED", 4), ("MXQ_ERR_CUDA", 5), ("MXQ_ERR_TIMEOUT", 6),
                    ("MXQ_OP_QUANTIZE", 0), ("MXQ_OP_DEQUANTIZE", 1), ("MXQ_OP_FAKE_QUANTIZE", 2)]:
        assert re.search(rf"\b{name}\s*=\s*{v}\b", src), name
    assert list(mxq.FORMATS.values()) == [0, 1, 2, 3, 4]
    assert re.search(r"#define MXQ_MAX_GROUP\s+(\d+)", src).group(1) == str(mxq.MAX_GROUP)
    assert re.search(r"#define MXQ_MAX_BATCH\s+(\d+)", src).group(1) == "64"
    assert mxq.OP_KINDS == {"quantize": 0, "dequantize": 1, "fake_quantize": 2}


def test_block_bits_match_page_facts(L):
    # 8 scale bits + 32 elements, plus AXS-6's 2-bit config ("AXS-6" block figure)
    assert [mxq.mxq_block_bits(i) for i in range(5)] == [202, 200, 200, 264, 136]
    assert round(mxq.mxq_block_bits(0) / 32, 2) == 6.31
    assert mxq.mxq_block_bits(7) == -1


@pytest.mark.parametrize("fmt", FMTS)
def test_size_queries_match_oracle(L, fmt):
    for rows, cols in [(1, 32), (3, 96), (4096, 4096), (16384, 8192), (0, 64)]:
        f = mxq.FORMATS[fmt]
        assert mxq.mxq_codes_bytes(f, rows, cols) == oracle.lib().orc_codes_bytes(oracle.FORMATS[fmt], rows, cols)
        assert mxq.mxq_scales_bytes(f, rows, cols) == oracle.lib().orc_scales_bytes(oracle.FORMATS[fmt], rows, cols)
    assert mxq.mxq_codes_bytes(mxq.FORMATS[fmt], 2, 33) == 0
    assert mxq.mxq_scales_bytes(mxq.FORMATS[fmt], -1, 32) == 0


def test_statuses_before_any_cuda_call(L):
    q = mxq.mxq_quantize
    assert q(9, None, 0, 1, 32, None, None, None) == 1          # bad format
    assert q(1, None, 5, 1, 32, None, None, None) == 1          # bad dtype
    assert q(1, None, 0, 1, 33, None, None, None) == 2          # cols % 32
    assert q(1, None, 0, -1, 32, None, None, None) == 2         # rows < 0
    assert q(1, None, 0, 1, 0, None, None, None) == 2           # cols == 0
    assert q(1, None, 0, 1 << 40, 1 << 20, None, None, None) == 2  # size overflow
    assert q(1, None, 0, 0, 32, None, None, None) == 0          # empty: no-op
    assert q(1, None, 0, 1, 32, None, None, None) == 1          # null pointer
    assert mxq.mxq_dequantize(1, None, None, 0, 64, None, 1, None) == 0
    assert mxq.mxq_dequantize(1, None, None, 2, 64, None, 3, None) == 1
    assert mxq.mxq_fake_quantize(0, None, 0, 0, 64, None, None) == 0
    assert mxq.mxq_fake_quantize(0, None, 0, 1, 48, None, None) == 2
    assert mxq.mxq_exp_quantize(4, None, 0, 64, None, None, None) == 0
    assert mxq.mxq_exp_quantize(4, None, 2, 40, None, None, None) == 2
    assert mxq.mxq_quantize_grouped(1, 1, [], None) == 1
    assert mxq.mxq_quantize_grouped(1, 1, [(0, 0, 0, 0, 64)], None) == 0
    assert mxq.mxq_quantize_grouped(1, 1, [(0, 0, 0, 0, 64)] * 65, None) == 1
    assert mxq.mxq_quantize_mma(0, None, 1, 128, 128, None, None, None) == 4   # AXS-6 header is 16 bits
    assert mxq.mxq_quantize_mma(1, None, 1, 128, 100, None, None, None) == 2
    assert mxq.mxq_quantize_mma(3, None, 1, 0, 128, None, None, None) == 0
    assert mxq.mxq_quantize_mma(3, None, 1, 1, 128, None, None, None) == 1
    assert mxq.mxq_swizzle_scales(None, -1, 4, None, None) == 2
    assert mxq.mxq_swizzle_scales(None, 4, 0, None, None) == 2
    assert mxq.mxq_swizzle_scales(None, 0, 4, None, None) == 0
    assert mxq.mxq_swizzle_scales(None, 4, 4, None, None) == 1
    b = mxq.mxq_run_batch
    assert b(1, [], None) == 1                                          # n = 0
    assert b(1, [(0, 1, 0, 0, 0, 0, 0, 64)] * 65, None) == 1            # n > 64
    assert b(1, [(3, 1, 0, 0, 0, 0, 0, 64)], None) == 1                 # bad kind
    assert b(1, [(0, 9, 0, 0, 0, 0, 0, 64)], None) == 1                 # bad format
    assert b(7, [(0, 1, 0, 0, 0, 0, 0, 64)], None) == 1                 # bad dtype
    assert b(1, [(1, 1, 0, 0, 0, 0, 2, 48)], None) == 2                 # cols % 32
    assert b(1, [(0, 1, 0, 0, 0, 0, 0, 64), (2, 0, 0, 0, 0, 0, 0, 32)], None) == 0  # all empty
    assert b(1, [(0, 1, 0, 0, 0, 0, 1, 64)], None) == 1                 # null pointers
    assert b(1, [(0, 1, 0, 0, 0, 0, 1 << 40, 1 << 30)], None) == 2      # size overflow
    assert b(1, [(2, 1, 0, 0, 0, 0, -1, 64)], None) == 2                # rows < 0
    assert b(1, [(5, 1, 0, 0, 0, 0, -1, 64)], None) == 1                # bad kind beats bad shape
    ef = mxq.mxq_exp_free_quantize
    assert ef(None, 0, 64, None, None, None) == 0
    assert ef(None, 2, 40, None, None, None) == 2
    assert ef(None, 1, 64, None, None, None) == 1
    assert ef(None, 1 << 40, 1 << 20, None, None, None) == 2
    qc, dc = mxq.mxq_quantize_cols, mxq.mxq_dequantize_cols
    assert qc(1, None, 1, 0, 64, None, None, None) == 0
    assert qc(1, None, 1, 48, 64, None, None, None) == 2                # rows % 32
    assert qc(1, None, 1, 64, 48, None, None, None) == 2                # cols % 32
    assert qc(1, None, 1, 1 << 40, 64, None, None, None) == 2           # too many tile rows
    assert qc(1, None, 1, 64, 64, None, None, None) == 1
    assert qc(8, None, 1, 64, 64, None, None, None) == 1
    assert dc(1, None, None, 0, 64, None, 1, None) == 0
    assert dc(1, None, None, 64, 1 << 50, None, 1, None) == 2
    assert dc(1, None, None, 64, 64, None, 1, None) == 1
    qx, dx, fx = mxq.mxq_quantize_exmy, mxq.mxq_dequantize_exmy, mxq.mxq_fake_quantize_exmy
    assert qx(2, 3, None, 0, 0, 64, None, None, None) == 0
    assert qx(6, 1, None, 0, 1, 64, None, None, None) == 4              # E > 5
    assert qx(2, 7, None, 0, 1, 64, None, None, None) == 4              # W = 10
    assert qx(1, 0, None, 0, 1, 64, None, None, None) == 4              # M = 0
    assert qx(2, 3, None, 4, 1, 64, None, None, None) == 1              # bad dtype
    assert qx(2, 3, None, 0, 1, 48, None, None, None) == 2
    assert qx(2, 3, None, 0, 1, 64, None, None, None) == 1
    assert dx(0, 5, None, None, 0, 64, None, 0, None) == 0
    assert dx(0, 5, None, None, 1, 64, None, 0, None) == 1
    assert fx(5, 3, None, 1, 1 << 40, 1 << 20, None, None) == 2
    assert fx(5, 3, None, 1, 1, 64, None, None) == 1
    sw = mxq.mxq_swizzle_scales
    assert sw(None, 8, 4 * (0x7FFFFFFF // 128) + 1, None, None) == 2  # one tile-row's words beyond 32 bits
    assert sw(None, 8, 0, None, None) == 2 and sw(None, -1, 4, None, None) == 2
    assert sw(None, 0, 4, None, None) == 0
    assert mxq.mxq_selftest_timeout(0) == 1 and mxq.mxq_selftest_timeout(1001) == 1
    for s in range(7):
        assert mxq.mxq_status_string(s)
    assert mxq.mxq_status_string(99) == "unknown status"
    assert mxq.mxq_version().count(".") == 2


def test_mma_scales_bytes_match_oracle(L):
    for rows, cols in [(1, 32), (127, 96), (128, 128), (129, 160), (4096, 4096), (0, 64)]:
        assert mxq.mxq_mma_scales_bytes(rows, cols) == oracle.mma_scales_bytes(rows, cols // 32)
    assert mxq.mxq_mma_scales_bytes(4, 33) == 0 and mxq.mxq_mma_scales_bytes(-1, 32) == 0


def test_block_size_other_than_32_is_rejected():
    with pytest.raises(mxq.MXQError) as e:
        mxq.fake_quantize(None, "axs6", block_size=16)
    assert e.value.status == 4


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(mxq, "LIB_PATH", str(tmp_path / "libmxq.so"))
    monkeypatch.setattr(mxq, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        mxq.lib()


C_PROGRAM = r"""
#include <stdio.h>
#include "mxq.h"

/* a plain C caller of the ABI, linked against libmxq.so: the host-only queries */
int main(void) {
    printf("%zu %zu %zu %d %d %s\n", mxq_codes_bytes(MXQ_MXFP6_E2M3, 4096, 4096),
           mxq_scales_bytes(MXQ_AXS6, 4096, 4096), mxq_codes_bytes(MXQ_MXFP4_E2M1, 3, 96),
           mxq_block_bits(MXQ_AXS6), mxq_block_bits(MXQ_MXFP8_E4M3), mxq_status_string(MXQ_ERR_SHAPE));
    return 0;
}
"""


@pytest.mark.parametrize("compiler,std,ext", [("gcc", "c99", "c"), ("g++", "c++11", "cpp")])
def test_plain_c_caller(L, tmp_path, compiler, std, ext):
    """The boundary is a C ABI: a C99 program (and the same source as C++11) built against
    include/mxq.h alone (no CUDA headers) links with libmxq.so and calls it. Host-only queries;
    no kernel runs."""
    src = tmp_path / f"caller.{ext}"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(mxq.LIB_PATH)
    r = subprocess.run([compiler, f"-std={std}", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                        os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-lmxq",
                        "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    a, b, c, d, e, msg = out.stdout.split(" ", 5)
    assert int(a) == 4096 * 4096 // 32 * 24 and int(b) == 4096 * 4096 // 32 * 2 and int(c) == 3 * 3 * 16
    assert int(d) == 202 and int(e) == 264
    assert msg.strip() == mxq.mxq_status_string(2)
