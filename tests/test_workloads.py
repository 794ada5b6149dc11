"""Host checks of the seeded input generators' shared-row layout (no GPU)."""
import numpy as np

from speculative_decoding_verification_90_b200 import workloads


def _check_layout(wl):
    m = wl.meta
    assert wl.mapped
    np.testing.assert_array_equal(m["target_rows"][m["target_map"]], wl.target)
    np.testing.assert_array_equal(m["draft_rows"][m["draft_map"]], wl.draft)
    assert m["target_map"].dtype == np.int32 and m["draft_map"].dtype == np.int32
    # every distinct row is referenced
    assert len(np.unique(m["target_map"])) == m["target_rows"].shape[0]
    assert len(np.unique(m["draft_map"])) == m["draft_rows"].shape[0]


def test_multibranch_rows_and_maps():
    wl = workloads.multibranch(seed=1, sequences=5, branches=3, gamma=5, vocab=700)
    _check_layout(wl)
    S, K, G = 5, 3, 5
    pts = wl.meta["branch_points"]
    tm, dm = wl.meta["target_map"], wl.meta["draft_map"]
    for s in range(S):
        bp = pts[s]
        rows = slice(s * K, (s + 1) * K)
        # shared positions: one row, one token for all branches
        assert (tm[rows, :bp] == tm[s * K, :bp]).all()
        assert (dm[rows, :bp] == dm[s * K, :bp]).all()
        assert (wl.tokens[rows, :bp] == wl.tokens[s * K, :bp]).all()
        # private positions: a row of their own
        priv = tm[rows, bp:].ravel()
        assert len(np.unique(priv)) == priv.size
    n_rows = wl.meta["target_rows"].shape[0] + wl.meta["draft_rows"].shape[0]
    assert wl.unique_logit_bytes == n_rows * wl.vocab * 2 < wl.logit_bytes


def test_multibranch_slice_drops_row_tables():
    wl = workloads.multibranch(seed=1, sequences=4, branches=2, gamma=3, vocab=300)
    part = wl.slice(2, 6)
    assert not part.mapped
    np.testing.assert_array_equal(part.target, wl.target[2:6])


def test_random_maps_layouts():
    for kw in ({}, {"dtype": "bf16"}, {"gamma": 0, "target_rows": 7, "draft_rows": 0},
               {"batch": 3, "gamma": 2, "target_rows": 9, "draft_rows": 6}):
        wl = workloads.random_maps(seed=2, vocab=300, **kw)
        _check_layout(wl)
        assert wl.tokens.shape == (wl.batch, wl.gamma)
        assert ((wl.tokens >= 0) & (wl.tokens < wl.vocab)).all()
