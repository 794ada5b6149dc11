import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))
for path in (ROOT, TESTS):
    if path not in sys.path:
        sys.path.insert(0, path)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the host")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Decision-parity counts of every GPU comparison of the session, one line
    per workload: sequences compared, hard differences, decisions whose oracle
    margin is below 1e-6 (allowed, counted) and residual draws whose residual
    mass is below what fp32 resolves (checked for validity, counted)."""
    try:
        import parity
    except ImportError:
        return
    if not parity.REPORT:
        return
    agg = {}
    for name, seqs, hard, margin, unres in parity.REPORT:
        a = agg.setdefault(name, [0, 0, 0, 0, 0])
        for i, v in enumerate((1, seqs, hard, margin, unres)):
            a[i] += v
    tot = [sum(a[i] for a in agg.values()) for i in range(5)]
    tr = terminalreporter
    tr.write_line(f"parity: {tot[0]} comparisons, {tot[1]} sequences, hard {tot[2]}, "
                  f"margin cases {tot[3]}, unresolved draws {tot[4]}")
    noted = [(n, a) for n, a in agg.items() if a[2] or a[3] or a[4]]
    for name, a in sorted(noted)[:12]:
        tr.write_line(f"  {name}: {a[1]} seqs in {a[0]} calls, hard {a[2]}, margin {a[3]}, "
                      f"unresolved {a[4]}")
