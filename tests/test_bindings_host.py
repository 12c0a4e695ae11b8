"""Host-side checks of the Python binding (no GPU needed).  The C ABI takes
bare pointers, so the binding validates every tensor's layout, dtype and size
before a pointer reaches the library.  Rejected layouts raise their own
errors; accepted ones get as far as the device check, which CPU tensors fail
with "tensors must live on the GPU" -- so a call that reaches that message
passed every layout check."""
import pytest
import torch

from nvfp4_w4a4_quantized_06_b200 import build, native

ON_GPU = "live on the GPU"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    native.lib()


def f32(n=1):
    return torch.zeros(n, dtype=torch.float32)


def u8(*shape):
    return torch.zeros(shape, dtype=torch.uint8)


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_quantize_layouts():
    x = bf16(96, 320)
    with pytest.raises(ValueError, match=ON_GPU):
        native.quantize(x, f32())
    # a strided row view and the codes slice of a fused buffer are fine
    big = bf16(96, 384)
    with pytest.raises(ValueError, match=ON_GPU):
        native.quantize(big[:, :320], f32())
    codes = u8(144, 160)
    sf = u8(native.sf_bytes(144, 320))
    with pytest.raises(ValueError, match=ON_GPU):
        native.quantize(x, f32(), codes=codes[48:144], sf=sf, sf_row0=48, sf_rows_total=144)
    # rejected
    with pytest.raises(ValueError, match="column stride"):
        native.quantize(bf16(320, 96).t(), f32())
    with pytest.raises(ValueError, match=r"\[96, 160\]"):
        native.quantize(x, f32(), codes=u8(96, 80))
    with pytest.raises(TypeError, match="uint8"):
        native.quantize(x, f32(), codes=torch.zeros(96, 160, dtype=torch.int8))
    with pytest.raises(ValueError, match="row stride"):
        native.quantize(x, f32(), codes=u8(96, 320)[:, :160])
    with pytest.raises(ValueError, match="needs"):
        native.quantize(x, f32(), sf=u8(native.sf_bytes(96, 320) - 1))
    with pytest.raises(ValueError, match="needs"):                  # sized for this call, not the fused total
        native.quantize(x, f32(), sf=u8(native.sf_bytes(96, 320)), sf_row0=100, sf_rows_total=196)
    with pytest.raises(TypeError, match="float32"):
        native.quantize(x, torch.zeros(1, dtype=torch.float64))
    with pytest.raises(ValueError, match="2-D"):
        native.quantize(bf16(320), f32())


def test_linear_and_gemm_layouts():
    M, N, K = 32, 96, 256
    x, wc, ws = bf16(M, K), u8(N, K // 2), u8(native.sf_bytes(N, K))
    for fn in (native.linear, native.linear_noalloc, native.linear_fused):
        with pytest.raises(ValueError, match=ON_GPU):
            fn(x, f32(), wc, ws, f32())
        with pytest.raises(ValueError, match="needs"):
            fn(x, f32(), wc, u8(100), f32())
        with pytest.raises(ValueError, match=r"\[32, 96\]"):
            fn(x, f32(), wc, ws, f32(), out=bf16(M, N + 1))
        with pytest.raises(ValueError, match=r"\[96, 128\]"):
            fn(x, f32(), u8(N, K // 4), ws, f32())
    with pytest.raises(TypeError, match="uint8"):
        native.linear(x, f32(), wc, ws, f32(), workspace=f32(1 << 20))
    with pytest.raises(ValueError, match=ON_GPU):
        native.gdn_gates(x, f32(), wc, ws, f32(), n_a=48)
    with pytest.raises(TypeError, match="float32"):
        native.gdn_gates(x, f32(), wc, ws, f32(), n_a=48, out=bf16(M, N))
    ac, asf = u8(M, K // 2), u8(native.sf_bytes(M, K))
    with pytest.raises(ValueError, match=ON_GPU):
        native.gemm(ac, asf, f32(), wc, ws, f32())
    with pytest.raises(ValueError, match=r"\[96, 128\]"):                # K of B differs from K of A
        native.gemm(ac, asf, f32(), u8(N, K // 2 + 16), ws, f32())
    with pytest.raises(ValueError, match="needs"):
        native.gemm(ac, u8(16), f32(), wc, ws, f32())


def test_group_and_next_row_layouts():
    K = 320
    codes, sf = u8(96, K // 2), u8(native.sf_bytes(96, K))
    with pytest.raises(ValueError, match=ON_GPU):
        native.harmonize(sf, 96, K, [0, 48, 96], f32(2))
    with pytest.raises(ValueError, match="needs 2"):
        native.harmonize(sf, 96, K, [0, 48, 96], f32(1))
    with pytest.raises(ValueError, match="two entries"):
        native.harmonize(sf, 96, K, [96], f32(1))
    with pytest.raises(ValueError, match=ON_GPU):
        native.harmonize_requant(codes, sf, K, [0, 48, 96], f32(2))
    with pytest.raises(ValueError, match=r"\[100, 160\]"):
        native.harmonize_requant(codes, sf, K, [0, 48, 100], f32(2))
    x = bf16(64, K)
    with pytest.raises(ValueError, match=ON_GPU):
        native.rmsnorm_quantize(x, bf16(K), 1e-6, f32())
    with pytest.raises(TypeError, match="norm weight"):
        native.rmsnorm_quantize(x, bf16(K + 64), 1e-6, f32())
    with pytest.raises(TypeError, match="norm weight"):
        native.rmsnorm_quantize(x, f32(K), 1e-6, f32())
    with pytest.raises(ValueError, match="needs 64"):
        native.rmsnorm_quantize(x, bf16(K), 1e-6, f32(), inv=f32(63))
    with pytest.raises(ValueError, match=ON_GPU):
        native.fake_quant(x, f32())
    with pytest.raises(TypeError, match="float64"):
        native.fake_quant(x, f32(), stats=f32(2))
    with pytest.raises(ValueError, match=ON_GPU):
        native.fp8_quantize(bf16(1024), f32())
    with pytest.raises(ValueError, match="needs 1024"):
        native.fp8_quantize(bf16(1024), f32(), out=u8(1000))
    with pytest.raises(ValueError, match=ON_GPU):
        native.amax_gscale(x)
    with pytest.raises(TypeError, match="float32"):
        native.amax_gscale(x, out=torch.zeros(1, dtype=torch.float64))


def test_every_entry_point_has_a_ctypes_signature():
    """Every function the header declares has its argument and result types
    set in the binding (an unset signature would pass 64-bit sizes and
    pointers as C ints)."""
    import ctypes
    import os
    import re
    header = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "nvfp4w4a4.h")
    text = re.sub(r"/\*.*?\*/", "", open(header).read(), flags=re.S)
    names = sorted(set(re.findall(r"^[A-Za-z_][A-Za-z0-9_ \*]*?\b((?:nvfp4|w4a4)_[a-z0-9_]+)\s*\(", text, re.M)))
    L = native.lib()
    assert len(names) >= 18
    missing = [n for n in names if getattr(L, n).argtypes is None]
    assert not missing, missing
    # the functions that return something other than a status code say so
    wide = [n for n in names if n.endswith("_bytes") or n in ("nvfp4_launch_count", "nvfp4_status_string")]
    untyped = [n for n in wide if getattr(L, n).restype is ctypes.c_int]
    assert wide and not untyped, untyped


def test_debug_mode_reports_device_flags_at_the_call(monkeypatch):
    """With NVFP4_DEBUG set, a call that left a device error flag raises at
    once, naming the entry point; without it, flags wait for the next
    explicit status read."""
    monkeypatch.setattr(native, "last_device_status", lambda: 4)
    monkeypatch.setattr(native, "DEBUG", False)
    native._check("nvfp4_quantize", 0)
    monkeypatch.setattr(native, "DEBUG", True)
    with pytest.raises(native.Nvfp4Error, match=r"nvfp4_quantize \(device error flags 0x4\)"):
        native._check("nvfp4_quantize", 0)
    with pytest.raises(native.Nvfp4Error, match="bad shape"):
        native._check("nvfp4_quantize", 2)
    monkeypatch.setattr(native, "last_device_status", lambda: 0)
    native._check("nvfp4_quantize", 0)
