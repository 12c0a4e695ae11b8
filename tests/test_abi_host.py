"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/nvfp4w4a4.h declares, and rejects bad arguments with
the documented status codes before touching the device."""
import ctypes
import os
import re

import pytest

from nvfp4_w4a4_quantized_06_b200 import build, native

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "nvfp4w4a4.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return native.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][A-Za-z0-9_ \*]*?\b((?:nvfp4|w4a4)_[a-z0-9_]+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_size_helpers(L):
    assert L.nvfp4_codes_bytes(64, 256) == 64 * 128
    assert L.nvfp4_sf_bytes(64, 256) == 128 * 16
    assert L.nvfp4_sf_bytes(129, 5120) == 256 * 320
    assert L.nvfp4_codes_bytes(-1, 64) == 0


def test_status_strings(L):
    for s in range(10):
        assert L.nvfp4_status_string(s)


FAKE = 1 << 20   # a 16-byte-aligned non-null stand-in; validation fails before any use


def test_quantize_validation(L):
    q = L.nvfp4_quantize
    assert q(FAKE, 7, 4, 64, 64, FAKE, FAKE, FAKE, 0, 4, None) == 4            # dtype
    assert q(FAKE, 0, 4, 100, 100, FAKE, FAKE, FAKE, 0, 4, None) == 2          # K % 64
    assert q(FAKE, 0, 4, 64, 32, FAKE, FAKE, FAKE, 0, 4, None) == 2           # ld < K
    assert q(FAKE, 0, 4, 64, 64, FAKE, FAKE, FAKE, 2, 4, None) == 2           # rows past the fused total
    assert q(None, 0, 4, 64, 64, FAKE, FAKE, FAKE, 0, 4, None) == 1           # null x
    assert q(FAKE + 2, 0, 4, 64, 64, FAKE, FAKE, FAKE, 0, 4, None) == 3       # misaligned x
    assert q(FAKE, 0, 4, 64, 68, FAKE, FAKE, FAKE, 0, 4, None) == 3           # row stride not 16 B


def test_gemm_validation(L):
    g = L.nvfp4_gemm
    args = [FAKE] * 7
    assert g(*args, 0, 64, 8, 64, 100, None, 0, None) == 2                    # K % 64
    assert g(*args, 5, 64, 8, 64, 128, None, 0, None) == 4                    # out dtype
    assert g(*args, 0, 32, 8, 64, 128, None, 0, None) == 2                    # ld_y < N
    assert g(None, *args[1:], 0, 64, 8, 64, 128, None, 0, None) == 1          # null
    assert g(*args[:6], FAKE + 4, 0, 64, 8, 64, 128, None, 0, None) == 3      # misaligned y


def test_linear_validation(L):
    w = L.w4a4_gemm
    assert w(FAKE, 0, 256, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 8, 64, 256, None, 0, None) == 8   # no workspace
    assert w(FAKE, 0, 256, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 8, 64, 256, FAKE, 16, None) == 8  # too small
    assert w(FAKE, 3, 256, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 8, 64, 256, FAKE, 0, None) == 4
    assert w(FAKE, 0, 100, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 8, 64, 256, FAKE, 0, None) == 2


def test_harmonize_validation(L):
    h = L.nvfp4_harmonize_group
    offs = (ctypes.c_int64 * 3)(0, 48, 96)
    bad = (ctypes.c_int64 * 3)(0, 48, 90)
    po = ctypes.cast(offs, ctypes.c_void_p)
    assert h(FAKE, 96, 256, 2, ctypes.cast(bad, ctypes.c_void_p), FAKE, FAKE, None) == 2
    assert h(FAKE, 96, 256, 0, po, FAKE, FAKE, None) == 2
    assert h(FAKE, 96, 256, 17, po, FAKE, FAKE, None) == 2
    assert h(None, 96, 256, 2, po, FAKE, FAKE, None) == 1
    assert h(FAKE, 96, 100, 2, po, FAKE, FAKE, None) == 2


def test_empty_inputs_are_no_ops(L):
    # zero rows with no padding to write, M == 0 or N == 0: OK without a launch
    assert L.nvfp4_quantize(None, 0, 0, 64, 64, None, None, None, 0, 0, None) == 0
    assert L.nvfp4_gemm(*([None] * 7), 0, 8, 0, 8, 64, None, 0, None) == 0
    assert L.w4a4_gemm(None, 0, 64, None, None, None, None, None, 0, 8, 0, 8, 64, None, 0, None) == 0


def test_next_rows_validation(L):
    g = L.w4a4_gdn_gates
    base = [FAKE, 0, 256, FAKE, FAKE, FAKE, FAKE, FAKE, 96]
    assert g(*base, 64, 96, 48, 256, FAKE, 1 << 30, None) != 2              # well-formed up to here
    assert g(*base, 64, 200, 48, 256, FAKE, 1 << 30, None) == 5             # N > 128: not a gate projection
    assert g(*base, 64, 96, 97, 256, FAKE, 1 << 30, None) == 2              # n_a beyond N
    assert g(*base, 64, 96, 48, 100, FAKE, 1 << 30, None) == 2              # K % 64
    assert g(FAKE, 7, 256, FAKE, FAKE, FAKE, FAKE, FAKE, 96, 64, 96, 48, 256, FAKE, 1 << 30, None) == 4
    f = L.nvfp4_fake_quant
    assert f(FAKE, 0, 4, 100, 100, FAKE, FAKE, 1, 100, None, None) == 2      # K % 64
    assert f(FAKE, 0, 4, 64, 64, FAKE, FAKE, 9, 64, None, None) == 4         # output dtype
    assert f(FAKE + 2, 0, 4, 64, 64, FAKE, FAKE, 1, 64, None, None) == 3     # misaligned x
    assert f(FAKE, 0, 4, 64, 64, FAKE, FAKE, 1, 64, FAKE + 4, None) == 3     # misaligned statistics
    q = L.nvfp4_fp8_quantize
    assert q(FAKE, 0, 12, FAKE, FAKE, None) == 2                             # n % 8
    assert q(FAKE, 3, 16, FAKE, FAKE, None) == 4
    assert q(FAKE, 0, 16, None, FAKE, None) == 1
    assert q(FAKE + 8, 0, 16, FAKE, FAKE, None) == 3
    assert q(FAKE, 0, 0, None, None, None) == 0                              # empty: nothing to do


def test_requant_and_rmsnorm_validation(L):
    h = L.nvfp4_harmonize_requant
    offs = (ctypes.c_int64 * 3)(0, 48, 96)
    bad = (ctypes.c_int64 * 3)(0, 48, 90)
    po = ctypes.cast(offs, ctypes.c_void_p)
    assert h(FAKE, FAKE, 96, 256, 2, ctypes.cast(bad, ctypes.c_void_p), FAKE, FAKE, None) == 2
    assert h(FAKE, FAKE, 96, 100, 2, po, FAKE, FAKE, None) == 2              # K % 64
    assert h(None, FAKE, 96, 256, 2, po, FAKE, FAKE, None) == 1              # null codes
    assert h(FAKE + 4, FAKE, 96, 256, 2, po, FAKE, FAKE, None) == 3          # codes not 8-byte aligned
    r = L.nvfp4_rmsnorm_quantize
    tail = [FAKE, FAKE, FAKE, None, None]                                     # gscale, codes, sf, inv, stream
    assert r(FAKE, 0, 4, 256, 256, FAKE, 0, 0.0, *tail) == 2                # eps must be > 0
    assert r(FAKE, 0, 4, 256, 256, FAKE, 0, float("nan"), *tail) == 2
    assert r(FAKE, 0, 4, 256, 256, FAKE, 0, float("inf"), *tail) == 2
    assert r(FAKE, 2, 4, 256, 256, FAKE, 0, 1e-6, *tail) == 4               # dtype
    assert r(FAKE, 0, 4, 100, 100, FAKE, 0, 1e-6, *tail) == 2               # K % 64
    assert r(FAKE, 0, 4, 256, 256, None, 0, 1e-6, *tail) == 1               # null weight
    assert r(FAKE, 0, 4, 256, 256, FAKE + 8, 0, 1e-6, *tail) == 3           # misaligned weight
    assert r(FAKE, 0, 4, 256, 256, FAKE, 0, 1e-6, FAKE, FAKE, FAKE, FAKE + 2, None) == 3   # misaligned inv
    # the norm weight must fit in one CTA's shared memory beside the staging
    assert r(FAKE, 0, 4, 111936, 111936, FAKE, 0, 1e-6, *tail) == 5
    assert r(FAKE, 1, 4, 111936, 111936, FAKE, 0, 1e-6, *tail) == 5
    assert r(FAKE, 0, 4, 111872, 111872, FAKE, 0, 1e-6, *tail) not in (2, 3, 5)
    assert r(FAKE, 1, 4, 111872, 111872, FAKE, 0, 1e-6, *tail) not in (2, 3, 5)


def test_error_word_bits_match_the_header(L):
    """The flag values nvfp4_last_device_status documents are the values the
    kernels OR into the device error word."""
    src = os.path.join(os.path.dirname(HEADER), "..", "nvfp4_w4a4_quantized_06_b200", "csrc", "ptx.cuh")
    enum = re.search(r"enum\s*:\s*unsigned\s*\{([^}]*)\}", open(src).read()).group(1)
    code_bits = {n: int(v) for n, v in re.findall(r"(ERR_[A-Z]+)\s*=\s*(\d+)u", enum)}
    assert code_bits == {"ERR_PRODUCER": 1, "ERR_MMA": 2, "ERR_EPILOGUE": 4, "ERR_TMEM": 8, "ERR_SELFTEST": 16}
    doc = open(HEADER).read()
    block = doc[doc.index("Reports and clears the library's device error word"):doc.index("nvfp4_last_device_status(nvfp4_stream_t")]
    listed = {int(b): int(v) for b, v in re.findall(r"bit (\d+) \((\d+)\)", block)}
    assert listed == {0: 1, 1: 2, 2: 4, 3: 8, 4: 16}
    assert set(listed.values()) == set(code_bits.values())
    assert "bit 4 (value 16)" in doc[doc.index("Failure-detection self-test"):]


def test_last_device_status_takes_a_stream(L):
    assert L.nvfp4_last_device_status.argtypes[0] is ctypes.c_void_p
    assert L.nvfp4_last_device_status(None, None) == 1                       # null flags: rejected first
