"""GPU parity of the bounds-checking debug build (libspecverify_debug.so).

The debug build checks, in the verification kernels, the indices derived
from the launch geometry and from each sequence's decision before it touches
the workspace or the outputs; a failed check sets a status bit
(SV_ERR_BOUNDS) and skips the access.  A child process loads the debug build
(SPECVERIFY_DEBUG_BOUNDS=1) and runs small workloads through the C ABI: every
check must pass (status 0) and the outputs must match the oracle like the
normal build's."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)

CHILD = r"""
import numpy as np
from speculative_decoding_verification_90_b200 import specverify as S, workloads
from parity import assert_parity, compare, gpu_run, oracle_run
assert S.LIB_PATH.endswith("libspecverify_debug.so"), S.LIB_PATH

def small(seed, B, G, V, dtype):
    rng = np.random.default_rng(seed)
    t = (rng.standard_normal((B, G + 1, V)) * 3).astype(np.float32)
    d = (0.8 * t[:, :G] + 0.2 * rng.standard_normal((B, G, V)) * 3).astype(np.float32)
    return workloads._finish(f"debug_{B}_{G}_{V}_{dtype}", dtype, 1.0, t, d, rng)

for wl in (workloads.b8_g3_v32000(seed=0), small(3, 24, 4, 4099, "f32"), small(4, 16, 3, 50257, "bf16"),
           small(5, 6, 0, 1000, "bf16")):
    for fused in (False, True):
        g = gpu_run(wl, fused=fused)
        assert g["status"] == 0 and g["bits"] == 0, (wl.name, fused, g["status"], g["bits"])
        assert_parity(compare(wl, g, oracle_run(wl)))
print("debug build ok")
"""


def test_debug_build_passes_its_checks_and_matches_the_oracle():
    from speculative_decoding_verification_90_b200 import build
    build.build(debug=True)
    env = dict(os.environ, SPECVERIFY_DEBUG_BOUNDS="1",
               PYTHONPATH=os.pathsep.join([ROOT, TESTS, os.environ.get("PYTHONPATH", "")]))
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=TESTS, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    assert "debug build ok" in r.stdout
