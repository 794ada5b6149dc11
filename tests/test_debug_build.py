"""The bounds-checking debug build (compiled with -DSV_DEBUG_BOUNDS=1): it
compiles, exports what the headers declare, and the binding loads it when
SPECVERIFY_DEBUG_BOUNDS=1.  Host-side only: no compute call is made here (the
GPU parity of the debug build is in test_gpu_debug_bounds.py)."""
import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

from test_abi import _declared  # noqa: E402


@pytest.fixture(scope="module")
def debug_lib():
    from speculative_decoding_verification_90_b200 import build
    return build.build(debug=True)


def test_debug_build_compiles_with_the_checks_on(debug_lib):
    """The flag reaches the kernels: the device code of the verification
    kernels compiles with the checks on (a separate object, so that a build
    that dropped the flag would still be caught by this compile)."""
    from speculative_decoding_verification_90_b200 import build
    src = os.path.join(build.CSRC, "specverify.cu")
    out = os.path.join(ROOT, "_build_debug_check.o")
    try:
        r = subprocess.run([build.nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O1",
                            "-std=c++17", "-DSV_DEBUG_BOUNDS=1", "-I", build.INCLUDE, "-I",
                            build.CSRC, "-c", src, "-o", out], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr[-2000:]
    finally:
        if os.path.exists(out):
            os.remove(out)


def test_debug_library_exports_every_declared_symbol(debug_lib):
    lib = ctypes.CDLL(debug_lib)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_loads_the_debug_library_on_request(debug_lib):
    code = ("from speculative_decoding_verification_90_b200 import specverify as S; "
            "print(S.LIB_PATH); print(S.specverify_status_string(S.SV_ERR_BOUNDS))")
    env = dict(os.environ, SPECVERIFY_DEBUG_BOUNDS="1")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    path, msg = r.stdout.strip().splitlines()[-2:]
    assert os.path.basename(path) == "libspecverify_debug.so"
    assert "bounds" in msg
