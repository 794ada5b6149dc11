"""Pins of the fold-gate oracle (oracle/gate.c) to what the page and plain
mathematics fix, independent of the oracle's own code.

The SpecFold explainer (blog.ontle.kr, post 356) defines the gate's measure as
the relative difference ||H_child - H_parent|| / ||H_parent|| at the same layer
input (observation paragraph), recomputation of the positions above tau packed
from all branches into one batch (the paragraph after the per-position path),
and provenance of folded positions followed along the fold chain (the
implementer's note).  Each pin below fails on a plausible mistake: a dropped
square root or a swapped numerator and denominator (closed forms), a wrong
parent index or position (tree fixture), the comparison's direction or
strictness (threshold cases), the chain walk (sources), the packing order.
"""
import math

import numpy as np
import pytest

import oracle
from speculative_decoding_verification_90_b200.workloads import bf16_bits, bits_to_f32


def _gate(h, parent, tau):
    return oracle.gate(np.ascontiguousarray(h, np.float32), np.asarray(parent, np.int32), tau)


def test_scaled_child_gives_the_scale_factor():
    """H_child = (1 + a) H_parent gives d = |a| (the products are exact; only the
    square roots round)."""
    rng = np.random.default_rng(0)
    parent_row = bits_to_f32(bf16_bits(rng.standard_normal((3, 64)).astype(np.float32)))
    for a in (0.5, -0.75, 0.25, 2.0, -1.0):
        h = np.stack([parent_row, (1.0 + a) * parent_row])
        r = _gate(h, [-1, 0], 1.0)
        np.testing.assert_allclose(r["rel_diff"][1], abs(a), rtol=1e-14, atol=0)
        assert np.all(np.isinf(r["rel_diff"][0]))


def test_three_four_twelve():
    """Parent (3, 4, 0), child (3, 4, 12): ||diff|| = 12, ||parent|| = 5, d = 2.4."""
    h = np.zeros((2, 1, 3), np.float32)
    h[0, 0] = [3, 4, 0]
    h[1, 0] = [3, 4, 12]
    r = _gate(h, [-1, 0], 2.4)
    assert r["rel_diff"][1, 0] == pytest.approx(2.4, rel=0, abs=1e-15)
    assert r["recompute"][1, 0] == 0           # d == tau folds (recompute only above tau)
    r = _gate(h, [-1, 0], math.nextafter(2.4, 0.0))
    assert r["recompute"][1, 0] == 1


def test_orthogonal_difference():
    """Child = parent + b e_1 with parent = a e_0: d = |b| / |a|."""
    h = np.zeros((2, 2, 5), np.float32)
    h[0, :, 0] = [2.0, 8.0]
    h[1] = h[0]
    h[1, :, 1] = [1.0, -2.0]
    r = _gate(h, [-1, 0], 0.3)
    np.testing.assert_array_equal(r["rel_diff"][1], [0.5, 0.25])
    np.testing.assert_array_equal(r["recompute"][1], [1, 0])


def test_zero_norms():
    """0/0 reads as 0 (folded), x/0 as +inf (recomputed)."""
    h = np.zeros((3, 2, 4), np.float32)
    h[2, 1, 3] = 1.0
    r = _gate(h, [-1, 0, 0], 0.0)
    assert r["rel_diff"][1, 0] == 0.0 and r["recompute"][1, 0] == 0
    assert r["rel_diff"][2, 0] == 0.0 and r["recompute"][2, 0] == 0
    assert np.isinf(r["rel_diff"][2, 1]) and r["recompute"][2, 1] == 1


def test_nan_recomputes():
    h = np.ones((2, 2, 4), np.float32)
    h[1, 0, 2] = np.nan
    r = _gate(h, [-1, 0], 10.0)
    assert r["recompute"][1, 0] == 1 and r["recompute"][1, 1] == 0


def test_tree_provenance_sources_and_packing():
    """A hand-made tree with the expected rows written out.

    Branches: 0 (no parent) <- 1 <- 2, 0 <- 3, and 4 (no parent); 3 positions.
    Copies fold (d = 0); a row marked X below differs strongly (d = 1) and is
    recomputed:
        branch 0: X X X     (no parent: always recomputed)
        branch 1: . X .
        branch 2: X . .
        branch 3: . . X
        branch 4: X X X     (no parent)
    """
    P, D = 3, 4
    base = np.arange(1, 1 + 5 * P * D, dtype=np.float32).reshape(5, P, D)
    h = base.copy()
    parent = [-1, 0, 1, 0, -1]
    for c in (1, 2, 3):
        h[c] = h[parent[c]]
    h[1, 1] *= 2.0
    h[2, 0] *= 2.0
    h[3, 2] *= 2.0
    r = _gate(h, parent, 0.5)
    row = lambda c, j: c * P + j  # noqa: E731
    rec = [[1, 1, 1], [0, 1, 0], [1, 0, 0], [0, 0, 1], [1, 1, 1]]
    np.testing.assert_array_equal(r["recompute"], rec)
    expect_prov = [[-1, -1, -1],
                   [row(0, 0), -1, row(0, 2)],
                   [-1, row(1, 1), row(1, 2)],
                   [row(0, 0), row(0, 1), -1],
                   [-1, -1, -1]]
    np.testing.assert_array_equal(r["provenance"], expect_prov)
    # branch 2, position 2 folds onto branch 1, which folds onto branch 0
    expect_src = [[row(0, 0), row(0, 1), row(0, 2)],
                  [row(0, 0), row(1, 1), row(0, 2)],
                  [row(2, 0), row(1, 1), row(0, 2)],
                  [row(0, 0), row(0, 1), row(3, 2)],
                  [row(4, 0), row(4, 1), row(4, 2)]]
    np.testing.assert_array_equal(r["source"], expect_src)
    np.testing.assert_array_equal(
        r["packed"], [row(0, 0), row(0, 1), row(0, 2), row(1, 1), row(2, 0), row(3, 2),
                      row(4, 0), row(4, 1), row(4, 2)])
    assert r["status"] == oracle.GATE_OK


@pytest.mark.parametrize("parent,bad", [
    ([-1, 0, 5], [2]),                  # out of range
    ([-1, 1, 1], [1, 2]),               # self link, and a child of it
    ([-1, 2, 1], [1, 2]),               # two-cycle
    ([-1, 2, 3, 2, 0], [1, 2, 3]),      # a chain that runs into a cycle
    ([-7, 0, 1], [0, 1, 2]),            # negative other than -1 at the top
])
def test_invalid_parents_are_roots(parent, bad):
    nb = len(parent)
    h = np.ones((nb, 2, 3), np.float32)
    r = _gate(h, parent, 0.1)
    assert r["status"] == oracle.GATE_ERR_PARENT
    for c in range(nb):
        if c in bad:
            assert r["parent_used"][c] == -1
            assert (r["recompute"][c] == 1).all()
        else:
            assert r["parent_used"][c] == parent[c]


def test_tau_extremes():
    rng = np.random.default_rng(3)
    h = rng.standard_normal((4, 5, 16)).astype(np.float32)
    parent = [-1, 0, 0, 1]
    r = _gate(h, parent, np.inf)
    assert (r["recompute"][1:] == 0).all()                      # every parented row folds
    assert r["packed"].tolist() == list(range(5))               # only the root's rows
    r = _gate(h, parent, 0.0)
    assert (r["recompute"] == 1).all()                          # any difference recomputes


def test_invariants_on_random_trees():
    """Packed rows ascending and exactly the recomputed ones; sources are recomputed
    rows; a folded row's source is its provenance row's source."""
    from speculative_decoding_verification_90_b200.workloads import gate_tree
    g = gate_tree(seed=1, sequences=6, branches=5, positions=9, dim=40, dtype="f32", tau=0.08)
    r = oracle.gate(g.hidden, g.parent, g.tau)
    rec = r["recompute"].ravel()
    np.testing.assert_array_equal(r["packed"], np.flatnonzero(rec))
    assert (np.diff(r["packed"]) > 0).all()
    src = r["source"].ravel()
    prov = r["provenance"].ravel()
    assert (rec[src] == 1).all()
    folded = np.flatnonzero(rec == 0)
    np.testing.assert_array_equal(src[folded], src[prov[folded]])
    np.testing.assert_array_equal(src[rec == 1], np.flatnonzero(rec))
    # the decision is d > tau everywhere
    d = r["rel_diff"].ravel()
    assert ((d > g.tau) == (rec == 1)).all()
    # the perturbation peaks at the revealed position, so it is recomputed there
    rev = g.meta["revealed"]
    for c in range(g.branches):
        if rev[c] >= 0:
            assert r["recompute"][c, rev[c]] == 1


def test_bf16_input_reads_the_stored_values():
    """bf16 bits and their float32 values give the same result."""
    rng = np.random.default_rng(4)
    f = rng.standard_normal((3, 4, 24)).astype(np.float32)
    bits = bf16_bits(f)
    r16 = oracle.gate(bits, np.array([-1, 0, 1], np.int32), 0.5)
    r32 = oracle.gate(bits_to_f32(bits), np.array([-1, 0, 1], np.int32), 0.5)
    np.testing.assert_array_equal(r16["rel_diff"], r32["rel_diff"])
    np.testing.assert_array_equal(r16["packed"], r32["packed"])
