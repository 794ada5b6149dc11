"""Pins of the CPU oracle against what the pages and the mathematics fix.

Every check here compares the oracle with something other than itself: values
worked out by hand from the verify rule, closed forms, a library softmax on the
cases that reduce to it, brute force over uniform grids on tiny vocabularies,
invariants of the method, and the pages' own exactness experiment.

Sources: "Speculative decoding - the small model writes first and the big model
checks" (sections 1-4) and "Speculative decoding: how to run big models fast"
(section "How it works").
"""
import json
import os

import numpy as np
import pytest
import torch

from speculative_decoding_verification_90_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _logits_from_probs(prob):
    return np.log(np.asarray(prob, np.float64)).astype(np.float32)


# --------------------------------------------------------------------------
# softmax (section 1 notation; temperature as an adjusted distribution)
# --------------------------------------------------------------------------

def test_softmax_uniform_is_one_over_v(oracle_mod):
    for V in (1, 2, 7, 256, 4096):
        prob, mx, sm = oracle_mod.softmax(np.full(V, 1.25, np.float32), 0.7)
        assert np.max(np.abs(prob - 1.0 / V)) < 1e-15
        assert mx == 1.25 and abs(sm - V) < 1e-9


def test_softmax_closed_forms(oracle_mod):
    prob, _, _ = oracle_mod.softmax(_logits_from_probs([1, 2, 3]), 1.0)
    assert np.allclose(prob, [1 / 6, 2 / 6, 3 / 6], atol=2e-7)
    # T = 2 on logits (0, 2 ln 2): exp(y) = (1, 2)
    x = np.array([0.0, 2 * np.log(2.0)], np.float32)
    prob, _, _ = oracle_mod.softmax(x, 2.0)
    assert np.allclose(prob, [1 / 3, 2 / 3], atol=2e-7)
    # bf16 storage: bits 0x0000 (0.0) and 0x3F80 (1.0)
    prob, mx, _ = oracle_mod.softmax(np.array([0x0000, 0x3F80], np.uint16), 1.0)
    e = np.e
    assert mx == 1.0
    assert np.allclose(prob, [1 / (1 + e), e / (1 + e)], atol=1e-15)
    # -inf entries carry no mass
    prob, _, _ = oracle_mod.softmax(np.array([-np.inf, 0.0, -np.inf, 0.0], np.float32), 1.0)
    assert prob.tolist() == [0.0, 0.5, 0.0, 0.5]


@pytest.mark.parametrize("T", [0.3, 0.7, 1.0, 2.5])
def test_softmax_matches_library_routine(oracle_mod, T):
    rng = np.random.default_rng(1)
    for V in (5, 1000, 32000):
        x = (rng.standard_normal(V) * 3).astype(np.float32)
        ref = torch.softmax(torch.from_numpy(x).double() / T, dim=0).numpy()
        prob, mx, sm = oracle_mod.softmax(x, T)
        assert np.max(np.abs(prob - ref)) < 1e-13    # summation order differs
        assert mx == float(x.max())
        assert abs(prob.sum() - 1.0) < 1e-12


def test_softmax_rejects_invalid_rows(oracle_mod):
    for bad in ([0.0, np.nan], [0.0, np.inf], [-np.inf, -np.inf]):
        with pytest.raises(ValueError):
            oracle_mod.softmax(np.array(bad, np.float32), 1.0)


# --------------------------------------------------------------------------
# the verify rule on a hand-worked example (section 1)
# --------------------------------------------------------------------------

def _one_call(oracle_mod, q_rows, p_rows, t, ua, ur, T=1.0):
    tgt = np.stack([_logits_from_probs(r) for r in q_rows])[None]
    G = len(p_rows)
    drf = (np.stack([_logits_from_probs(r) for r in p_rows])[None] if G
           else np.zeros((1, 0, tgt.shape[-1]), np.float32))
    return oracle_mod.verify(tgt, drf, np.array([t], np.int32).reshape(1, G),
                             np.array([ua], np.float32).reshape(1, G),
                             np.array([ur], np.float32), T)


def test_hand_worked_example(oracle_mod):
    ex = _load("hand_example.json")
    for case in ex["cases"]:
        out = _one_call(oracle_mod, [ex["q"], ex["q_bonus"]], [ex["p"]], [case["t"]],
                        [case["u_accept"]], case["u_resample"])
        assert out["out_num_accepted"][0] == case["num_accepted"], case
        assert out["out_tokens"][0].tolist() == case["tokens"], case
        assert abs(out["ratio"][0, 0] - ex["ratio"][case["t"]]) < 1e-6
        if case["num_accepted"] == 0:
            assert abs(out["resid_mass"][0] - ex["residual_mass"]) < 1e-6


def test_inverse_cdf_follows_index_order(oracle_mod):
    ex = _load("hand_example.json")["inverse_cdf"]
    for u, tok in zip(ex["u"], ex["token"]):
        out = _one_call(oracle_mod, [ex["distribution"]], [], [], [], u)
        assert out["out_num_accepted"][0] == 0
        assert out["out_tokens"][0].tolist() == [tok], (u, tok)


# --------------------------------------------------------------------------
# brute force: the output law equals q (section 4 claim; rejection sampling)
# --------------------------------------------------------------------------

def _grid(n):
    return ((np.arange(n) + 0.5) / n).astype(np.float32)


@pytest.mark.parametrize("V", [2, 3, 5, 8])
def test_bruteforce_law_equals_target(oracle_mod, V):
    """gamma = 1: sweep both uniforms over midpoint grids, for every draft token t.

    P(out = x) = sum_t p(t) [P(accept | t) 1{x = t} + P(reject | t) P(draw = x | reject, t)]
    is estimated by counting grid outcomes; it must equal q(x) up to the grid's
    resolution.  A flipped comparison, a residual of max(0, p - q), or a draw
    from the wrong row all break it.
    """
    rng = np.random.default_rng(V)
    n = 20000
    for trial in range(3):
        q = rng.dirichlet(np.ones(V) * 0.7)
        p = rng.dirichlet(np.ones(V) * 0.7)
        qb = rng.dirichlet(np.ones(V))
        q_seen = torch.softmax(torch.from_numpy(_logits_from_probs(q)).double(), 0).numpy()
        p_seen = torch.softmax(torch.from_numpy(_logits_from_probs(p)).double(), 0).numpy()
        law = np.zeros(V)
        ug = _grid(n)
        for t in range(V):
            B = n
            tgt = np.broadcast_to(np.stack([_logits_from_probs(q), _logits_from_probs(qb)]),
                                  (B, 2, V))
            drf = np.broadcast_to(_logits_from_probs(p)[None], (B, 1, V))
            tok = np.full((B, 1), t, np.int32)
            # accept frequency over a grid of u_accept
            out = oracle_mod.verify(tgt, drf, tok, ug.reshape(B, 1),
                                    np.full(B, 0.5, np.float32), 1.0)
            acc = float(np.mean(out["out_num_accepted"] == 1))
            # residual law over a grid of u_resample at a rejecting u_accept
            out = oracle_mod.verify(tgt, drf, tok, np.full((B, 1), 0.99999994, np.float32), ug, 1.0)
            rejected = out["out_num_accepted"] == 0
            if rejected.all():
                res = np.bincount(out["out_tokens"][:, 0], minlength=V) / B
            else:
                assert q_seen[t] / p_seen[t] > 0.99999994
                res = np.zeros(V)
            law += p_seen[t] * (acc * np.eye(V)[t] + (1.0 - acc) * res)
        assert np.max(np.abs(law - q_seen)) < 3.0 * V / n, (trial, law, q_seen)


def test_bonus_law_is_target_at_last_position(oracle_mod):
    """When every draft is accepted the extra token is drawn from q_gamma."""
    rng = np.random.default_rng(7)
    V, n = 6, 30000
    q_last = rng.dirichlet(np.ones(V))
    same = rng.dirichlet(np.ones(V))
    tgt = np.broadcast_to(np.stack([_logits_from_probs(same), _logits_from_probs(q_last)]), (n, 2, V))
    drf = np.broadcast_to(_logits_from_probs(same)[None], (n, 1, V))
    tok = np.full((n, 1), 2, np.int32)
    out = oracle_mod.verify(tgt, drf, tok, np.zeros((n, 1), np.float32), _grid(n), 1.0)
    assert (out["out_num_accepted"] == 1).all()
    law = np.bincount(out["out_tokens"][:, 1], minlength=V) / n
    ref = torch.softmax(torch.from_numpy(_logits_from_probs(q_last)).double(), 0).numpy()
    assert np.max(np.abs(law - ref)) < 2.0 / n


# --------------------------------------------------------------------------
# invariants ("How it works": 1..gamma+1 tokens per target call)
# --------------------------------------------------------------------------

def _random_problem(rng, B, G, V, dtype, mix):
    tgt = (rng.standard_normal((B, G + 1, V)) * 3).astype(np.float32)
    drf = (mix * tgt[:, :G] + (1 - mix) * rng.standard_normal((B, G, V)) * 3).astype(np.float32)
    if dtype == "bf16":
        tgt, drf = workloads.bf16_bits(tgt), workloads.bf16_bits(drf)
        seen = workloads.bits_to_f32(drf)
    else:
        seen = drf
    tok = workloads.gumbel_max_tokens(rng, seen, 1.0) if G else np.zeros((B, 0), np.int32)
    return tgt, drf, tok, rng.random((B, G), dtype=np.float32), rng.random(B, dtype=np.float32)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_output_invariants(oracle_mod, dtype):
    rng = np.random.default_rng(3)
    for (B, G, V, T, mix) in [(40, 4, 64, 1.0, 0.8), (30, 1, 17, 0.5, 0.3), (20, 7, 33, 1.7, 0.95),
                              (10, 0, 50, 1.0, 0.0)]:
        tgt, drf, tok, ua, ur = _random_problem(rng, B, G, V, dtype, mix)
        out = oracle_mod.verify(tgt, drf, tok, ua, ur, T)
        n = out["out_num_accepted"]
        assert ((n >= 0) & (n <= G)).all()
        for b in range(B):
            row = out["out_tokens"][b]
            emitted = row[row >= 0]
            assert len(emitted) == n[b] + 1            # 1 .. gamma+1 tokens per call
            assert (row[: n[b]] == tok[b, : n[b]]).all()  # accepted prefix is the drafts
            assert (row[n[b] + 1:] == -1).all()
            assert 0 <= row[n[b]] < V
        assert (out["seq_status"] == 0).all()


def test_identical_distributions_always_accept(oracle_mod):
    rng = np.random.default_rng(4)
    B, G, V = 50, 5, 40
    tgt = (rng.standard_normal((B, G + 1, V)) * 3).astype(np.float32)
    drf = tgt[:, :G].copy()
    tok = workloads.gumbel_max_tokens(rng, drf, 1.0)
    out = oracle_mod.verify(tgt, drf, tok, rng.random((B, G), dtype=np.float32),
                            rng.random(B, dtype=np.float32), 1.0)
    assert (out["out_num_accepted"] == G).all()
    assert np.allclose(out["ratio"], 1.0, atol=1e-12)


def test_disjoint_supports_reject_first_and_draw_from_target(oracle_mod):
    rng = np.random.default_rng(5)
    B, G, V = 60, 3, 20
    tgt = (rng.standard_normal((B, G + 1, V)) * 2).astype(np.float32)
    drf = (rng.standard_normal((B, G, V)) * 2).astype(np.float32)
    tgt[:, :, V // 2:] = -np.inf   # target mass on the lower half
    drf[:, :, : V // 2] = -np.inf  # draft mass on the upper half
    tok = workloads.gumbel_max_tokens(rng, drf, 1.0)
    out = oracle_mod.verify(tgt, drf, tok, rng.random((B, G), dtype=np.float32),
                            rng.random(B, dtype=np.float32), 1.0)
    assert (out["out_num_accepted"] == 0).all()
    assert (out["out_tokens"][:, 0] < V // 2).all()
    assert np.allclose(out["resid_mass"], 1.0, atol=1e-12)


def test_zero_residual_mass_falls_back_to_target(oracle_mod):
    """A rejection whose residual max(0, q - p) has no mass in double precision:
    target and draft rows equal except at the drafted token t, where q(t)
    underflows to 0 (logit -1000) and p(t) is about 1e-301 (logit -690).  The
    ratio is 0, so t is rejected; every other q(i) equals p(i) bit for bit
    (the tiny p(t) does not move the draft's normaliser), so Z = 0.  The draw
    then comes from q at that position (inverse CDF with the same uniform,
    checked against a library softmax) and the ZERO_MASS warning is set."""
    rng = np.random.default_rng(12)
    B, G, V, T = 24, 2, 64, 1.0
    tgt = (rng.standard_normal((B, G + 1, V)) * 2).astype(np.float32)
    drf = tgt[:, :G].copy()
    n = rng.integers(0, G, size=B)          # the position that rejects
    tok = np.zeros((B, G), np.int32)
    for b in range(B):
        for j in range(G):
            tok[b, j] = int(np.argmax(tgt[b, j]))  # accepted (ratio 1) before n
        t = int(rng.integers(0, V))
        tok[b, n[b]] = t
        tgt[b, n[b], t] = -1000.0
        drf[b, n[b], t] = -690.0
    u_acc = np.full((B, G), 0.5, np.float32)
    u_res = rng.random(B, dtype=np.float32)
    out = oracle_mod.verify(tgt, drf, tok, u_acc, u_res, T)
    np.testing.assert_array_equal(out["out_num_accepted"], n)
    assert (out["seq_status"] == 18).all()
    for b in range(B):
        q = torch.softmax(torch.from_numpy(tgt[b, n[b]].astype(np.float64)) / T, 0).numpy()
        c = np.cumsum(q)
        expect = int(np.searchsorted(c, float(u_res[b]) * c[-1], side="right"))
        assert abs(float(u_res[b]) * c[-1] - c[min(expect, V - 1)]) > 1e-9   # away from an edge
        assert out["out_tokens"][b, n[b]] == expect
        np.testing.assert_array_equal(out["out_tokens"][b, :n[b]], tok[b, :n[b]])
        assert (out["out_tokens"][b, n[b] + 1:] == -1).all()
        assert out["q_tok"][b, n[b]] == 0.0 and out["p_tok"][b, n[b]] > 0.0


def test_data_errors(oracle_mod):
    rng = np.random.default_rng(6)
    tgt, drf, tok, ua, ur = _random_problem(rng, 4, 3, 16, "f32", 0.5)
    tok = tok.copy()
    tok[1, 2] = 16          # out of range
    tok[2, 0] = -1          # out of range
    tgt = tgt.copy()
    tgt[3, 3, 5] = np.nan   # non-finite in the bonus row
    out = oracle_mod.verify(tgt, drf, tok, ua, ur, 1.0)
    assert out["seq_status"].tolist() == [0, 16, 16, 17]
    for b in (1, 2, 3):
        assert out["out_num_accepted"][b] == 0
        assert (out["out_tokens"][b] == -1).all()
    assert out["errors"] == 3


def test_threads_do_not_change_results(oracle_mod):
    rng = np.random.default_rng(8)
    tgt, drf, tok, ua, ur = _random_problem(rng, 37, 3, 100, "bf16", 0.7)
    a = oracle_mod.verify(tgt, drf, tok, ua, ur, 0.8, threads=1)
    b = oracle_mod.verify(tgt, drf, tok, ua, ur, 0.8, threads=5)
    for k in a:
        if isinstance(a[k], np.ndarray):
            assert np.array_equal(a[k], b[k], equal_nan=True), k


# --------------------------------------------------------------------------
# acceptance count: closed form E[n] = sum_k prod_{j<k} (1 - TV_j)
# --------------------------------------------------------------------------

def test_mean_accepted_matches_closed_form(oracle_mod):
    """With t ~ p, P(accept_j) = sum_x min(p_j, q_j) = 1 - TV(p_j, q_j), independently per position."""
    wl = workloads.char_level(calls=1000, seed=0)
    out = oracle_mod.verify(wl.target, wl.draft, wl.tokens, wl.u_accept, wl.u_resample, 1.0)
    n = out["out_num_accepted"].astype(np.float64)
    q = torch.softmax(torch.from_numpy(wl.target[:, :4]).double(), -1)
    p = torch.softmax(torch.from_numpy(wl.draft).double(), -1)
    alpha = torch.minimum(p, q).sum(-1).numpy()          # [calls, gamma]
    surv = np.cumprod(alpha, axis=1)                     # P(n >= k) = prod_{j<k} alpha_j
    expected = surv.sum(axis=1)
    second = (2 * np.arange(1, 5) - 1) @ surv.T          # E[n^2] = sum_k (2k-1) P(n >= k)
    var = second - expected ** 2
    z = (n.mean() - expected.mean()) / np.sqrt(var.sum() / len(n) ** 2)
    assert abs(z) < 3.5, (n.mean(), expected.mean(), z)


# --------------------------------------------------------------------------
# the pages' bookkeeping tables (section 2 and 3): tokens per step = accepted + 1
# --------------------------------------------------------------------------

def test_page_tables_bookkeeping():
    t = _load("page_tables.json")
    for k, acc, tok, ms, sp in zip(t["k"], t["mean_accepted"], t["tokens_per_step"],
                                   t["time_ms"], t["speedup"]):
        assert abs(tok - (acc + 1.0)) < 1e-9                       # the corrected/bonus token
        # the printed call times are rounded to 1 us, so sums drift by up to 1 us
        assert abs(ms - (t["target_ms"] + k * t["draft_ms"])) < 1.5e-3
        assert abs(sp - tok / (ms / t["target_ms"])) < 0.006
    assert max(zip(t["speedup"], t["k"]))[1] == 3


# --------------------------------------------------------------------------
# the pages' exactness experiment (section 4), restated on a synthetic position
# --------------------------------------------------------------------------

@pytest.mark.slow
def test_exactness_experiment(oracle_mod):
    beta = _load("exactness_beta.json")["beta"]
    wl = workloads.exactness(beta, batch=60000, seed=0)
    q0, _, _ = oracle_mod.softmax(wl.target[0, 0], 1.0)
    p0, _, _ = oracle_mod.softmax(wl.draft[0, 0], 1.0)
    tv_pq = 0.5 * np.abs(p0 - q0).sum()
    assert abs(tv_pq - 0.6571) < 0.002                      # the page's worst position
    out = oracle_mod.verify(wl.target, wl.draft, wl.tokens, wl.u_accept, wl.u_resample, 1.0,
                            threads=os.cpu_count() or 1)
    first = out["out_tokens"][:, 0]
    N, V = len(first), wl.vocab
    emp = np.bincount(first, minlength=V) / N
    tv_spec = 0.5 * np.abs(emp - q0).sum()
    rng = np.random.default_rng(1234)
    direct = [0.5 * np.abs(np.bincount(rng.choice(V, N, p=q0), minlength=V) / N - q0).sum()
              for _ in range(20)]
    mu, sd = float(np.mean(direct)), float(np.std(direct))
    assert tv_spec <= mu + 3 * sd, (tv_spec, mu, sd)
    # draft tokens alone sit at TV ~ 0.657 from q: the correction is what closes the gap
    emp_draft = np.bincount(wl.tokens[:, 0], minlength=V) / N
    assert 0.5 * np.abs(emp_draft - q0).sum() > 0.6
    # goodness of fit on well-populated tokens
    big = q0 * N >= 5
    chi2 = float((((emp - q0) * N) ** 2 / (q0 * N))[big].sum())
    dof = int(big.sum()) - 1
    assert chi2 < dof + 5 * np.sqrt(2 * dof), (chi2, dof)
