"""bench.py's command line, checked on the CPU: unknown sampling settings are
rejected by the parser before anything runs."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=300, cwd=ROOT)


def test_unknown_sampling_setting_is_an_argument_error():
    r = _bench("--sampling", "greedy,top_p0.5")
    assert r.returncode == 2
    assert "unknown setting(s) ['top_p0.5']" in r.stderr


def test_help_lists_the_sampling_settings():
    r = _bench("--help")
    assert r.returncode == 0
    for name in ("greedy", "top_k50_top_p0.9", "top_p0.9", "top_k2000"):
        assert name in r.stdout
