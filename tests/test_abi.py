"""Host-side checks of the C-ABI library: it loads without a GPU, exports every
function that include/specverify.h declares, and the binding covers them all.
No compute call is made here."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))
PREFIX = r"(?:specverify|specfold_gate|specverify_lmhead)_\w+"


def _declared():
    names = set()
    for header in HEADERS:
        text = open(header).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(rf"\b({PREFIX})\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib_path():
    from speculative_decoding_verification_90_b200 import build
    return build.build()


def test_header_declares_the_entry_points():
    names = _declared()
    for required in ("specverify_create", "specverify_run", "specverify_destroy"):
        assert required in names
    assert len(names) >= 10


def test_library_exports_every_declared_symbol(lib_path):
    lib = ctypes.CDLL(lib_path)
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(rf"\bT ({PREFIX})", out))
    assert set(_declared()) == exported


def test_binding_covers_the_header(lib_path):
    from speculative_decoding_verification_90_b200 import specverify
    assert set(specverify.SIGNATURES) == set(_declared())
    for name in _declared():
        assert callable(getattr(specverify, name)), name


def test_library_holds_no_oracle_code(lib_path):
    out = subprocess.run(["nm", "-D", lib_path], capture_output=True, text=True, check=True).stdout
    assert "oracle" not in out


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "speculative_decoding_verification_90_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "liboracle" not in text, f


def test_status_strings_without_gpu(lib_path):
    from speculative_decoding_verification_90_b200 import specverify as S
    assert S.specverify_status_string(S.SV_OK) == "ok"
    assert "token" in S.specverify_status_string(S.SV_ERR_TOKEN_RANGE)
    assert S.specverify_status_string(12345) == "unknown status"


def test_create_argument_checks_without_gpu(lib_path):
    from speculative_decoding_verification_90_b200 import specverify as S
    with pytest.raises(S.SpecVerifyError) as e:
        S.specverify_create(-1, 2, 100, S.SV_DTYPE_F32, 0)
    assert e.value.status == S.SV_ERR_INVALID_ARG
    with pytest.raises(S.SpecVerifyError) as e:
        S.specverify_create(1, 2, 100, 7, 0)
    assert e.value.status == S.SV_ERR_INVALID_ARG


def test_null_handle_is_rejected(lib_path):
    from speculative_decoding_verification_90_b200 import specverify as S
    lib = S._lib
    assert lib.specverify_run(None, None, None, None, None, None, 1.0, None, None, None) == \
        S.SV_ERR_INVALID_ARG
    assert lib.specverify_set_launch(None, 1, 256, 0) == S.SV_ERR_INVALID_ARG
    lib.specverify_destroy(None)
