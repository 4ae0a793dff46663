"""The C-ABI library loads and exports every symbol include/mxmoe.h declares,
and rejects invalid arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "mxmoe.h")).read()
    return re.findall(r"^MX_API\s+(?:int|size_t|unsigned long long)\s+([a-z0-9_]+)\(", src, flags=re.M)


@pytest.fixture(scope="module")
def mx():
    from fp8_moe_numerics_b200 import build, _lib
    build.build()
    return _lib.lib()


def test_every_declared_symbol_is_exported(mx):
    names = _declared()
    assert len(names) >= 16
    for n in names:
        assert hasattr(mx, n), n
    from fp8_moe_numerics_b200._lib import SIGNATURES
    assert set(SIGNATURES) == set(names)


def test_wait_selftest_limit_checked_on_host(mx):
    assert mx.mx_wait_selftest(0, None) == 1
    assert mx.mx_wait_selftest(10 * 1000 * 1000 + 1, None) == 1


def test_launch_counter_ignores_rejected_calls(mx):
    before = mx.mx_kernel_launches()
    assert isinstance(before, int) and before >= 0
    # rejected on the host: no kernel is launched
    assert mx.nvfp4_quantize(None, 16, 64, 1, None, None, None, 1, None) == 1
    assert mx.mx_kernel_launches() == before


def test_sizes_and_version(mx):
    assert mx.mx_version() == 1
    assert mx.mx_sf_bytes(256, 4096, 16, 1) == 256 * 256
    assert mx.mx_sf_bytes(100, 4096, 16, 1) == 0          # MMA layout needs rows % 128
    assert mx.mx_sf_bytes(100, 4096, 16, 0) == 100 * 256
    assert mx.mx_sf_bytes(128, 96, 32, 1) == 0            # 3 scale columns: not a multiple of 4
    assert mx.mx_route_workspace_bytes(32768, 384) == (128 * 384 + 384) * 4


def test_invalid_arguments_are_rejected_before_launch(mx):
    buf = (ctypes.c_uint8 * 4096)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    null = ctypes.c_void_p(0)
    EINVAL = 1
    # null input
    assert mx.nvfp4_quantize(null, 16, 64, 1, p, p, p, 0, null) == EINVAL
    # cols not a multiple of 16
    assert mx.nvfp4_quantize(p, 16, 40, 1, p, p, p, 0, null) == EINVAL
    # MMA layout with rows % 128 != 0
    assert mx.nvfp4_quantize(p, 16, 64, 1, p, p, p, 1, null) == EINVAL
    # misaligned input pointer
    assert mx.nvfp4_quantize(ctypes.c_void_p(ctypes.addressof(buf) + 1), 16, 64, 1, p, p, p, 0, null) == EINVAL
    # bad rbits
    assert mx.mxfp8_requant_transpose_sr(p, p, p, 128, 64, 1, 0, null, 0, 0, 7, p, p, 0, null) == EINVAL
    # K not a multiple of 256 for the NVFP4 GEMM
    assert mx.grouped_gemm_nvfp4(p, p, p, p, p, p, p, 1, 128, 256, 128, p, 0, null) == EINVAL
    # unknown GEMM mode
    assert mx.grouped_gemm_mxfp8(5, p, p, p, p, p, 1, 128, 128, 128, p, 0, null) == EINVAL
    # routing capacity too small
    assert mx.moe_route(p, 16, 2, 4, 128, p, p, p, p, 4096, null) == EINVAL


def test_c_program_compiles_links_and_calls_the_library(mx, tmp_path):
    # the boundary from C itself: the header as C99, the library linked by
    # name, host-side calls that need no GPU
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text(
        '#include "mxmoe.h"\n'
        '#include <stdio.h>\n'
        'int main(void) {\n'
        '    unsigned long long n0 = mx_kernel_launches();\n'
        '    int bad = nvfp4_quantize(0, 128, 100, 1, 0, 0, 0, MX_SF_ROWMAJOR, 0);  /* cols % 16 != 0 */\n'
        '    size_t sf = mx_sf_bytes(256, 4096, 16, MX_SF_MMA);\n'
        '    printf("%d %d %zu %llu\\n", mx_version(), bad, sf, mx_kernel_launches() - n0);\n'
        '    return 0;\n'
        '}\n')
    lib_dir = os.path.join(ROOT, "fp8_moe_numerics_b200")
    exe = tmp_path / "use"
    cuda_inc = next((d for d in ("/usr/local/cuda/include", os.environ.get("CUDA_HOME", "") + "/include")
                     if os.path.exists(os.path.join(d, "cuda_runtime.h"))), None)
    if cuda_inc is None:
        pytest.skip("no CUDA headers")
    subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src), "-o", str(exe),
                    "-L", lib_dir, "-lmxmoe", "-Wl,-rpath," + lib_dir], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert int(out[0]) == mx.mx_version() and int(out[1]) == 1          # MX_EINVAL
    assert int(out[2]) == 256 * 4096 // 16 and int(out[3]) == 0          # nothing launched


def test_bounds_checked_build_exports_the_same_symbols(mx):
    """libmxmoe_debug.so (-DMX_DEBUG_BOUNDS) builds from the same sources, exports
    every declared symbol, reports itself as the bounds-checked build, and the
    normal library reports 0 and never counts anything."""
    import ctypes
    from fp8_moe_numerics_b200 import build
    path = build.build(debug_bounds=True)
    dbg = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(dbg, n), n
    dbg.mx_debug_bounds_build.restype = ctypes.c_int
    dbg.mx_debug_bounds_violations.restype = ctypes.c_ulonglong
    dbg.mx_debug_bounds_violations.argtypes = [ctypes.c_int]
    assert dbg.mx_debug_bounds_build() == 1
    assert mx.mx_debug_bounds_build() == 0
    assert mx.mx_debug_bounds_violations(1) == 0
