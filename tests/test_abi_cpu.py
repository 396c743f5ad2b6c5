"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
symbol that ``include/bitlinear.h`` declares, reports workspace sizes, and rejects bad
arguments before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT

pytestmark = pytest.mark.cpu

HEADER = os.path.join(ROOT, "include", "bitlinear.h")


@pytest.fixture(scope="module")
def L():
    from ternary_weight_bit_absmean_b200 import build_lib, binding
    build_lib.build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"BL_API\s+[\w\s\*]+?\b(bitlinear_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ["bitlinear_quantize_weights", "bitlinear_quantize_weights_with_scale",
                 "bitlinear_pack", "bitlinear_quantize_act", "bitlinear_forward",
                 "bitlinear_workspace_size"]:
        assert want in names


def test_library_exports_every_declared_symbol(L):
    from ternary_weight_bit_absmean_b200 import binding
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)
    # nothing but the declared API is exported
    assert {n for n in exported if n.startswith("bitlinear_")} == set(declared_functions())


def test_binding_covers_every_declared_function(L):
    """The Python binding gives every entry point of the header a ctypes prototype and
    calls it from a wrapper (the path and layout variants through the keyword arguments
    of the plain wrapper; the workspace-free weight quantiser through the library handle
    in its own test)."""
    import inspect
    from ternary_weight_bit_absmean_b200 import binding
    declared = set(declared_functions())
    assert set(binding.EXPORTED) | {"bitlinear_quantize_weights_noalloc"} == declared
    src = inspect.getsource(binding)
    for name in binding.EXPORTED:
        assert "L.%s.argtypes" % name in src and "L.%s.restype" % name in src, name
        assert "lib().%s(" % name in src, name


def test_library_has_no_driver_or_torch_dependency():
    from ternary_weight_bit_absmean_b200 import binding
    out = subprocess.run(["ldd", binding.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libtorch" not in out and "libcudart" not in out


def test_header_compiles_as_c():
    src = '#include "bitlinear.h"\nint main(void){ return (int)bitlinear_workspace_size(1, 4) < 0; }\n'
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I",
                    os.path.join(ROOT, "include"), "-x", "c", "-"], input=src, text=True, check=True)


def test_workspace_size(L):
    assert L.bitlinear_workspace_size(0, 4) == 0
    assert L.bitlinear_workspace_size(4, 0) == 0
    assert L.bitlinear_workspace_size(1, 4) == 8
    sizes = [L.bitlinear_workspace_size(n, 4096) for n in (1, 64, 4096, 65536)]
    assert sizes == sorted(sizes) and sizes[-1] <= 148 * 8 * 8


BL_OK, INVALID, SHAPE, MISALIGNED, WORKSPACE = 0, 1, 2, 3, 4
FAKE = 1 << 20          # 16-byte aligned, never dereferenced: every case fails validation first
ODD = FAKE + 4


def test_quantize_weights_validation(L):
    f = L.bitlinear_quantize_weights
    ws = L.bitlinear_workspace_size(8, 64)
    assert f(None, 8, 64, 1e-5, FAKE, FAKE, FAKE, ws, None) == INVALID
    assert f(FAKE, 0, 64, 1e-5, FAKE, FAKE, FAKE, ws, None) == INVALID
    assert f(FAKE, 8, -4, 1e-5, FAKE, FAKE, FAKE, ws, None) == INVALID
    assert f(FAKE, 8, 64, 0.0, FAKE, FAKE, FAKE, ws, None) == INVALID
    assert f(FAKE, 8, 64, float("nan"), FAKE, FAKE, FAKE, ws, None) == INVALID
    assert f(FAKE, 8, 66, 1e-5, FAKE, FAKE, FAKE, ws, None) == SHAPE
    assert f(ODD, 8, 64, 1e-5, FAKE, FAKE, FAKE, ws, None) == MISALIGNED
    assert f(FAKE, 8, 64, 1e-5, FAKE, ODD, FAKE, ws, None) == MISALIGNED
    assert f(FAKE, 8, 64, 1e-5, FAKE, FAKE, None, ws, None) == WORKSPACE
    assert f(FAKE, 8, 64, 1e-5, FAKE, FAKE, FAKE, ws - 1, None) == WORKSPACE


def test_other_entry_points_validation(L):
    assert L.bitlinear_quantize_weights_with_scale(FAKE, 8, 64, None, FAKE, None) == INVALID
    assert L.bitlinear_quantize_weights_with_scale(FAKE, 8, 6, FAKE, FAKE, None) == SHAPE
    assert L.bitlinear_pack(FAKE, 8, 10, FAKE, None, None) == SHAPE
    assert L.bitlinear_pack(ODD, 8, 64, FAKE, None, None) == MISALIGNED
    assert L.bitlinear_quantize_act(FAKE, 0, 64, 1e-5, FAKE, FAKE, None) == INVALID
    assert L.bitlinear_quantize_act(FAKE, 4, 64, -1.0, FAKE, FAKE, None) == INVALID
    assert L.bitlinear_quantize_act(FAKE, 4, 64, 1e-5, ODD, FAKE, None) == MISALIGNED
    fwd = L.bitlinear_forward
    assert fwd(None, FAKE, FAKE, FAKE, 4, 8, 64, FAKE, 0, None, None) == INVALID
    assert fwd(FAKE, FAKE, FAKE, FAKE, 4, 8, 66, FAKE, 0, None, None) == SHAPE
    assert fwd(FAKE, FAKE, FAKE, FAKE, 4, 8, 64, FAKE, 7, None, None) == INVALID
    assert fwd(FAKE, FAKE, FAKE, FAKE, 4, 8, 1 << 25, FAKE, 0, None, None) == SHAPE
    assert fwd(FAKE, ODD, FAKE, FAKE, 4, 8, 64, FAKE, 0, None, None) == MISALIGNED
    path = L.bitlinear_forward_path
    for p in (2, 3, 4):  # every tcgen05 variant needs K % 64 == 0
        assert path(FAKE, FAKE, FAKE, FAKE, 40, 8, 96, FAKE, 0, None, p, None) == SHAPE
    assert path(FAKE, FAKE, FAKE, FAKE, 4, 8, 64, FAKE, 0, None, 9, None) == INVALID
    for p in (6, 7):  # the two forced decode GEMV kernels read x_q in the stride-4 layout only
        assert path(FAKE, FAKE, FAKE, FAKE, 4, 8192, 256, FAKE, 0, None, p, None) == SHAPE
    assert L.bitlinear_status_string(3) == b"BL_ERR_MISALIGNED"
    lay = L.bitlinear_forward_layout
    for k16 in (1, 2):  # the k16 layouts need K % 16 == 0
        assert lay(FAKE, FAKE, FAKE, FAKE, 4, 8, 72, FAKE, 0, None, k16, 0, None) == SHAPE
    assert lay(FAKE, FAKE, FAKE, FAKE, 4, 8, 64, FAKE, 0, None, 5, 0, None) == INVALID
    assert lay(FAKE, FAKE, FAKE, FAKE, 4, 8, 64, FAKE, 0, None, 3, 0, None) == INVALID
    # stride-4 x_q on a forced tensor-core path needs K <= 2^17
    for p in (2, 3, 4):
        assert lay(FAKE, FAKE, FAKE, FAKE, 40, 8, (1 << 17) + 64, FAKE, 0, None, 2, p, None) == SHAPE
    nq = L.bitlinear_norm_quantize_act
    assert nq(None, None, 4, 64, 0, 1e-5, 1e-5, FAKE, FAKE, 0, None) == INVALID
    assert nq(FAKE, None, 4, 64, 2, 1e-5, 1e-5, FAKE, FAKE, 0, None) == INVALID        # unknown norm kind
    assert nq(FAKE, None, 4, 64, 0, -1.0, 1e-5, FAKE, FAKE, 0, None) == INVALID        # norm_eps < 0
    assert nq(FAKE, None, 4, 64, 1, 1e-5, 0.0, FAKE, FAKE, 0, None) == INVALID         # eps <= 0
    assert nq(FAKE, None, 4, 64, 0, 1e-5, 1e-5, FAKE, FAKE, 3, None) == INVALID        # unknown layout
    assert nq(FAKE, None, 4, 60, 0, 1e-5, 1e-5, FAKE, FAKE, 0, None) == SHAPE          # K % 8
    assert nq(FAKE, None, 4, 40, 1, 1e-5, 1e-5, FAKE, FAKE, 2, None) == SHAPE          # k16 layout needs K % 16
    assert nq(ODD, None, 4, 64, 0, 1e-5, 1e-5, FAKE, FAKE, 0, None) == MISALIGNED
    assert nq(FAKE, ODD, 4, 64, 0, 1e-5, 1e-5, FAKE, FAKE, 0, None) == MISALIGNED      # norm weight
    qa = L.bitlinear_quantize_act_layout
    assert qa(FAKE, 4, 24, 1e-5, FAKE, FAKE, 1, None) == SHAPE
    assert qa(FAKE, 4, 24, 1e-5, FAKE, FAKE, 2, None) == SHAPE
    assert qa(FAKE, 4, 32, 1e-5, FAKE, FAKE, 3, None) == INVALID


def test_tl5_entry_points_validation(L):
    """The five-codes-per-byte entry points reject bad arguments on the host."""
    rb = L.bitlinear_tl5_row_bytes
    assert [rb(k) for k in (16, 80, 96, 8192, 28672)] == [16, 16, 32, 1648, 5744]
    assert rb(0) == 0 and rb(-16) == 0 and rb(24) == 0
    pk = L.bitlinear_pack_tl5
    assert pk(None, 8, 64, FAKE, None, None) == INVALID
    assert pk(FAKE, 0, 64, FAKE, None, None) == INVALID
    assert pk(FAKE, 8, 72, FAKE, None, None) == SHAPE          # K % 16
    assert pk(ODD, 8, 64, FAKE, None, None) == MISALIGNED
    assert pk(FAKE, 8, 64, ODD, None, None) == MISALIGNED
    rp = L.bitlinear_repack_tl5
    assert rp(FAKE, 8, 64, None, None) == INVALID
    assert rp(FAKE, 8, 40, FAKE, None) == SHAPE
    assert rp(ODD, 8, 64, FAKE, None) == MISALIGNED
    f = L.bitlinear_forward_tl5
    assert f(None, FAKE, FAKE, FAKE, 4, 8, 64, FAKE, 0, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 8, 64, FAKE, 0, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, 4, 8, 64, FAKE, 7, None) == INVALID          # unknown dtype
    assert f(FAKE, FAKE, FAKE, FAKE, 4, 8, 72, FAKE, 0, None) == SHAPE            # K % 16
    assert f(FAKE, FAKE, FAKE, FAKE, 4, 8, 1 << 25, FAKE, 0, None) == SHAPE       # int32 accumulators
    assert f(FAKE, FAKE, FAKE, FAKE, 65535 * 16 + 1, 8, 64, FAKE, 0, None) == SHAPE
    assert f(FAKE, FAKE, ODD, FAKE, 4, 8, 64, FAKE, 0, None) == MISALIGNED
    assert f(FAKE, FAKE, FAKE, FAKE, 4, 8, 64, ODD, 0, None) == MISALIGNED


def test_ste_backward_validation(L):
    fi = L.bitlinear_ste_backward_input
    assert fi(None, FAKE, FAKE, 4, 8, 64, FAKE, None) == INVALID
    assert fi(FAKE, FAKE, FAKE, 0, 8, 64, FAKE, None) == INVALID
    assert fi(FAKE, FAKE, FAKE, 4, 8, 66, FAKE, None) == SHAPE          # K % 4
    assert fi(FAKE, FAKE, FAKE, 1 << 31, 8, 64, FAKE, None) == SHAPE
    assert fi(FAKE, ODD, FAKE, 4, 8, 64, FAKE, None) == MISALIGNED
    fw = L.bitlinear_ste_backward_weight
    assert fw(FAKE, FAKE, FAKE, None, 4, 8, 64, FAKE, None) == INVALID
    assert fw(FAKE, FAKE, FAKE, FAKE, 4, -8, 64, FAKE, None) == INVALID
    assert fw(FAKE, FAKE, FAKE, FAKE, 4, 1 << 31, 64, FAKE, None) == SHAPE
    assert fw(FAKE, FAKE, FAKE, FAKE, 4, 8, 66, FAKE, None) == SHAPE      # K % 4
    assert fw(FAKE, FAKE, ODD, FAKE, 4, 8, 64, FAKE, None) == MISALIGNED
    assert fw(FAKE, FAKE, FAKE, FAKE, 4, 8, 64, ODD, None) == MISALIGNED


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from ternary_weight_bit_absmean_b200 import binding
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        binding.lib()
