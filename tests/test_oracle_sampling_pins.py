"""Pins of the sampling-variant oracle (oracle/sampling.c): greedy, top-k,
nucleus and per-sequence temperature as standard sampling from an adjusted
distribution ("Speculative decoding: how to run big models fast", section "How
it works", guarantee paragraph), verified with the rule of "Speculative
decoding - the small model writes first and the big model checks", section 1.

Each check compares the oracle with something other than itself: the pinned
plain oracle where the variants reduce to it, the greedy rule written with
numpy's argmax, hand-worked top-k / top-p examples, and brute force over
uniform grids showing that the output law is the adjusted target distribution.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_90_b200 import workloads


def _grid(n):
    return ((np.arange(n) + 0.5) / n).astype(np.float32)


def _run(wl, T, **kw):
    return oracle.verify_sampling(wl.target, wl.draft, wl.tokens, wl.u_accept, wl.u_resample,
                                  T, threads=4, **kw)


def test_no_filter_equals_the_plain_oracle():
    wl = workloads.b8_g3_v32000(seed=4)
    T = float(np.float32(wl.temperature))
    a = oracle.verify(wl.target, wl.draft, wl.tokens, wl.u_accept, wl.u_resample, T)
    for kw in ({}, {"top_k": wl.vocab}, {"top_p": 1.0}, {"top_k": wl.vocab, "top_p": 1.0}):
        b = _run(wl, T, **kw)
        np.testing.assert_array_equal(a["out_tokens"], b["out_tokens"])
        np.testing.assert_array_equal(a["out_num_accepted"], b["out_num_accepted"])
        np.testing.assert_allclose(b["q_tok"], a["q_tok"], rtol=1e-12, atol=1e-300)
        np.testing.assert_allclose(b["p_tok"], a["p_tok"], rtol=1e-12, atol=1e-300)
        assert (b["kept_target"] == wl.vocab).all()


def _greedy_expected(wl):
    am = wl.target.astype(np.float64) if wl.dtype == "f32" else \
        workloads.bits_to_f32(wl.target).astype(np.float64)
    best = np.argmax(am, axis=2)          # first index of the maximum
    B, G = wl.tokens.shape
    out = np.full((B, G + 1), -1, np.int32)
    nacc = np.zeros(B, np.int32)
    for b in range(B):
        n = 0
        while n < G and wl.tokens[b, n] == best[b, n]:
            n += 1
        out[b, :n] = wl.tokens[b, :n]
        out[b, n] = best[b, n]
        nacc[b] = n
    return out, nacc


def test_greedy_is_argmax_prefix():
    """T = 0: accept exactly while t_j = argmax q_j, then emit argmax q_n."""
    wl = workloads.b8_g3_v32000(seed=5)
    # make some drafts agree with the target's argmax so that prefixes are accepted
    tgt = workloads.bits_to_f32(wl.target)
    best = np.argmax(tgt, axis=2)
    wl.tokens[:4, :2] = best[:4, :2]
    wl.tokens[2, 2] = best[2, 2]
    out, nacc = _greedy_expected(wl)
    for kw in ({}, {"top_k": 5}, {"top_p": 0.3}):
        r = _run(wl, 0.0, **kw)
        np.testing.assert_array_equal(r["out_tokens"], out)
        np.testing.assert_array_equal(r["out_num_accepted"], nacc)
    assert nacc.max() == 3 and nacc[:4].min() >= 2


def test_greedy_ties_take_the_first_index():
    V = 6
    tgt = np.zeros((1, 2, V), np.float32)
    tgt[0, 0, [2, 4]] = 3.0
    tgt[0, 1, [1, 5]] = 7.0
    drf = np.zeros((1, 1, V), np.float32)
    r = oracle.verify_sampling(tgt, drf, np.array([[4]], np.int32), np.zeros((1, 1), np.float32),
                               np.array([0.9], np.float32), 0.0)
    assert r["out_tokens"].tolist() == [[2, -1]]
    r = oracle.verify_sampling(tgt, drf, np.array([[2]], np.int32), np.zeros((1, 1), np.float32),
                               np.array([0.9], np.float32), 0.0)
    assert r["out_tokens"].tolist() == [[2, 1]]


def test_top_k_worked_example():
    """Logits (2, 1, 0, -1, 5, 3), T = 1, k = 3: kept {4, 5, 0}; q(4) = e^5 / (e^5 + e^3 + e^2)."""
    x = np.array([2, 1, 0, -1, 5, 3], np.float32)
    tgt = np.stack([x, x])[None]
    drf = np.zeros((1, 1, 6), np.float32)   # uniform draft: p(t) = 1/3 after top-3 of ties...
    drf[0, 0] = [0, 0, 0, -5, 0, -5]        # draft top-3 with ties at 0: keeps {0, 1, 2, 4}
    r = oracle.verify_sampling(tgt, drf, np.array([[4]], np.int32),
                               np.array([[0.999]], np.float32), np.array([0.5], np.float32),
                               1.0, top_k=3)
    z = np.exp(5.0) + np.exp(3.0) + np.exp(2.0)
    assert r["q_tok"][0, 0] == pytest.approx(np.exp(5.0) / z, rel=1e-14)
    assert r["p_tok"][0, 0] == pytest.approx(0.25, rel=1e-14)     # 4 tied entries kept
    assert r["kept_target"].tolist() == [[3, 3]]
    assert r["kept_draft"].tolist() == [[4]]
    assert r["out_num_accepted"][0] == 1                          # ratio 3.6 > 0.999
    # the bonus draw is from q restricted to {4, 5, 0}: u = 0.5 lands on index 4
    # (cumulative in index order: e^2/z = 0.04, then e^5/z = 0.88 > 0.5)
    assert r["out_tokens"].tolist() == [[4, 4]]


def test_top_p_worked_example():
    """Probabilities (0.5, 0.3, 0.15, 0.05): top_p 0.79 keeps two, 0.81 keeps three."""
    probs = np.array([0.5, 0.3, 0.15, 0.05])
    x = np.log(probs).astype(np.float32)
    tgt = np.stack([x, x])[None]
    drf = tgt[:, :1].copy()
    tok = np.array([[1]], np.int32)
    ua = np.array([[0.0]], np.float32)
    ur = np.array([0.7], np.float32)
    seen = np.exp(x.astype(np.float64))
    seen /= seen.sum()
    for top_p, keep in ((0.79, 2), (0.81, 3), (0.4, 1), (0.999, 4)):
        r = oracle.verify_sampling(tgt, drf, tok, ua, ur, 1.0, top_p=top_p)
        assert r["kept_target"][0, 0] == keep
        expect = seen[1] / seen[:keep].sum() if keep >= 2 else 0.0
        assert r["q_tok"][0, 0] == pytest.approx(expect, rel=1e-12, abs=1e-300)
        assert r["filter_margin"][0] > 0


def test_top_k_ties_are_kept():
    x = np.array([3, 1, 1, 1, 0], np.float32)
    tgt = np.stack([x, x])[None]
    r = oracle.verify_sampling(tgt, tgt[:, :1], np.array([[0]], np.int32),
                               np.zeros((1, 1), np.float32), np.array([0.5], np.float32), 1.0,
                               top_k=2)
    assert r["kept_target"].tolist() == [[4, 4]]


def test_top_k_one_is_greedy():
    wl = workloads.b8_g3_v32000(seed=6)
    g = _run(wl, 0.0)
    k1 = _run(wl, 0.7, top_k=1)
    np.testing.assert_array_equal(g["out_tokens"], k1["out_tokens"])


def test_temperature_errors():
    wl = workloads.b8_g3_v32000(seed=7)
    T = np.full(wl.batch, 0.7, np.float32)
    T[1], T[3], T[5] = -0.5, np.nan, np.inf
    r = _run(wl, T, top_k=10)
    for b in (1, 3, 5):
        assert r["seq_status"][b] == oracle.ERR_TEMPERATURE
        assert r["out_num_accepted"][b] == 0 and (r["out_tokens"][b] == -1).all()
    assert (r["seq_status"][[0, 2, 4, 6, 7]] == 0).all()


def test_per_sequence_temperature_equals_separate_calls():
    wl = workloads.b8_g3_v32000(seed=8)
    T = np.array([0.5, 1.0, 0.0, 2.0, 0.7, 0.0, 1.3, 0.9], np.float32)
    r = _run(wl, T, top_k=40, top_p=0.95)
    for b in range(wl.batch):
        s = wl.slice(b, b + 1)
        rb = oracle.verify_sampling(s.target, s.draft, s.tokens, s.u_accept, s.u_resample,
                                    T[b], top_k=40, top_p=0.95)
        np.testing.assert_array_equal(r["out_tokens"][b], rb["out_tokens"][0])


@pytest.mark.parametrize("top_k,top_p", [(2, 1.0), (0, 0.7), (3, 0.8)])
def test_bruteforce_law_equals_adjusted_target(top_k, top_p):
    """gamma = 1, V = 5: with t drawn from the adjusted p, the output law is the
    adjusted q (the rejection-sampling argument on adjusted distributions).

    The adjusted distributions are built here from their definition: the kept
    sets are fixed by construction (distinct logits), then a library softmax
    over the kept entries.
    """
    V, n = 5, 20000
    rng = np.random.default_rng(top_k * 10 + int(top_p * 10))
    for trial in range(3):
        xq = np.sort(rng.normal(0, 1.5, V))[::-1].astype(np.float32)
        xp = np.sort(rng.normal(0, 1.5, V))[::-1].astype(np.float32)
        xq = xq[rng.permutation(V)]
        xp = xp[rng.permutation(V)]

        def adjusted(x):
            order = np.argsort(-x.astype(np.float64), kind="stable")
            keep = np.zeros(V, bool)
            k = top_k if 0 < top_k < V else V
            keep[order[:k]] = True
            w = torch.softmax(torch.from_numpy(x.astype(np.float64)), 0).numpy()
            if top_p < 1.0:
                w_k = np.where(keep, w, 0.0)
                w_k /= w_k.sum()
                c = np.cumsum(w_k[order])
                m = int(np.searchsorted(c, top_p)) + 1   # first prefix with mass >= top_p
                keep = np.zeros(V, bool)
                keep[order[:m]] = True
            a = np.where(keep, w, 0.0)
            return a / a.sum()

        q, p = adjusted(xq), adjusted(xp)
        ug = _grid(n)
        tgt = np.broadcast_to(np.stack([xq, xq])[None], (n, 2, V))
        drf = np.broadcast_to(xp[None, None], (n, 1, V))
        law = np.zeros(V)
        for t in np.flatnonzero(p > 0):
            tok = np.full((n, 1), t, np.int32)
            out = oracle.verify_sampling(tgt, drf, tok, ug.reshape(n, 1),
                                         np.full(n, 0.5, np.float32), 1.0, top_k=top_k,
                                         top_p=top_p)
            acc = float(np.mean(out["out_num_accepted"] == 1))
            out = oracle.verify_sampling(tgt, drf, tok, np.full((n, 1), 0.99999994, np.float32),
                                         ug, 1.0, top_k=top_k, top_p=top_p)
            if (out["out_num_accepted"] == 0).all():
                res = np.bincount(out["out_tokens"][:, 0], minlength=V) / n
            else:
                assert q[t] / p[t] > 0.99999994
                res = np.zeros(V)
            law += p[t] * (acc * np.eye(V)[t] + (1.0 - acc) * res)
        assert np.max(np.abs(law - q)) < 3.0 * V / n, (trial, law, q)


def test_top_p_keeps_tied_values_together():
    """Probabilities (0.4, 0.2, 0.2, 0.2): top_p 0.4 stops at the first value
    (mass 0.4 reaches it) and keeps one entry; top_p 0.5 must take the next
    value, which three entries share, so all four are kept (q(t) = 0.2)."""
    probs = np.array([0.4, 0.2, 0.2, 0.2])
    x = np.log(probs).astype(np.float32)
    tgt = np.stack([x, x])[None]
    drf = tgt[:, :1].copy()
    tok = np.array([[2]], np.int32)
    ua = np.array([[0.0]], np.float32)
    ur = np.array([0.3], np.float32)
    seen = np.exp(x.astype(np.float64))
    seen /= seen.sum()
    for top_p, keep in ((0.39, 1), (0.5, 4), (0.9, 4)):
        r = oracle.verify_sampling(tgt, drf, tok, ua, ur, 1.0, top_p=top_p)
        assert r["kept_target"][0].tolist() == [keep, keep]
        expect = seen[2] / seen[:keep].sum() if keep > 2 else 0.0
        assert r["q_tok"][0, 0] == pytest.approx(expect, rel=1e-12, abs=1e-300)
