"""Write ``exactness_beta.json``: the draft mixing weight of the exactness workload.

The exactness experiment of "Speculative decoding - the small model writes
first and the big model checks" (section 4) draws 60 000 samples at the
position where the draft and target distributions differ most, with total
variation TV(p, q) = 0.6571 (section 4 table).  The synthetic stand-in uses a
fixed target row z ~ N(0, 3^2) and a draft row (1-beta) z + beta w with
w ~ N(0, 3^2); this script finds beta by bisection so that TV(p, q) matches
the page's value.  It calls only the CPU oracle's softmax (no CUDA code).

Run from the repository root:  python tests/golden/make_exactness_beta.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from speculative_decoding_verification_90_b200 import workloads  # noqa: E402

PAGE_TV = 0.6571   # section 4 table: the draft model's own distribution vs the target's
SEED = 0
VOCAB = 4096


def tv_at(beta, z, w):
    q, _, _ = oracle.softmax(z[0], 1.0)
    p, _, _ = oracle.softmax(workloads.exactness_draft_row(z, w, beta), 1.0)
    return 0.5 * float(np.abs(p - q).sum())


def main():
    z, w = workloads.exactness_rows(SEED, VOCAB)
    lo, hi = 0.0, 1.0
    assert tv_at(lo, z, w) < PAGE_TV < tv_at(hi, z, w)
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        if tv_at(mid, z, w) < PAGE_TV:
            lo = mid
        else:
            hi = mid
    beta = 0.5 * (lo + hi)
    out = {
        "beta": beta,
        "tv_pq": tv_at(beta, z, w),
        "page_tv_pq": PAGE_TV,
        "seed": SEED,
        "vocab": VOCAB,
        "source": "Speculative decoding - the small model writes first and the big model "
                  "checks, section 4 (exactness experiment: TV 0.6571, 60 000 samples; "
                  "speculative samples 0.0018, direct samples 0.0035)",
        "written_by": "tests/golden/make_exactness_beta.py (oracle softmax only)",
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "exactness_beta.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
