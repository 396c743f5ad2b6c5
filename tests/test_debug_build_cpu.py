"""The device index checks of the debugging build compile (nvcc cross-compiles for sm_100a
without a GPU), and the normal build leaves them out: the source that carries them
compiles with BL_DEBUG_CHECKS=1, and the library's normal objects are built without it."""
import os
import subprocess

import pytest

from ternary_weight_bit_absmean_b200 import build_lib


@pytest.mark.skipif(not os.path.exists(build_lib.NVCC), reason="nvcc not available")
def test_debug_checks_compile(tmp_path):
    obj = tmp_path / "k_gemv_tc_debug.o"
    subprocess.run([build_lib.NVCC, *build_lib.FLAGS, "-DBL_DEBUG_CHECKS=1", "-I", build_lib.INCLUDE, "-I",
                    build_lib.CSRC, "-c", os.path.join(build_lib.CSRC, "k_gemv_tc.cu"), "-o", str(obj)], check=True)
    assert obj.stat().st_size > 0


def test_normal_build_has_no_debug_flag():
    assert "-DBL_DEBUG_CHECKS=1" not in build_lib.FLAGS
    assert build_lib.DEBUG_LIB != build_lib.LIB
