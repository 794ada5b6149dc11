"""Pins of the oracle's output-layer logits (oracle.lm_logits) and of its
float64-logit input path, used by the fused LM-head parity tests."""
import numpy as np

import oracle
from speculative_decoding_verification_90_b200 import workloads


def test_one_hot_rows_pick_weight_columns():
    """hidden = e_i gives logits = W[:, i] exactly."""
    rng = np.random.default_rng(0)
    D, V = 16, 40
    w = workloads.bits_to_f32(workloads.bf16_bits(rng.standard_normal((V, D)).astype(np.float32)))
    h = np.zeros((3, D), np.float32)
    h[0, 2] = 1.0
    h[1, 15] = 1.0
    h[2, 7] = -2.0
    x = oracle.lm_logits(h, w)
    np.testing.assert_array_equal(x[0], w[:, 2])
    np.testing.assert_array_equal(x[1], w[:, 15])
    np.testing.assert_array_equal(x[2], -2.0 * w[:, 7].astype(np.float64))


def test_hand_example():
    """(1, 2) . ((3, 4), (5, 6), (-1, 0.5))^T = (11, 17, 0)."""
    x = oracle.lm_logits(np.array([[1.0, 2.0]], np.float32),
                         np.array([[3.0, 4.0], [5.0, 6.0], [-1.0, 0.5]], np.float32))
    np.testing.assert_array_equal(x, [[11.0, 17.0, 0.0]])


def test_float64_logits_match_the_float32_path():
    """The verification of float64 logits equals that of the same values as
    float32 / bf16 (the loader only widens)."""
    wl = workloads.b8_g3_v32000(seed=3)
    a = oracle.verify(wl.target, wl.draft, wl.tokens, wl.u_accept, wl.u_resample, 0.7)
    t = workloads.bits_to_f32(wl.target).astype(np.float64)
    d = workloads.bits_to_f32(wl.draft).astype(np.float64)
    b = oracle.verify(t, d, wl.tokens, wl.u_accept, wl.u_resample, 0.7)
    for k in ("out_tokens", "out_num_accepted"):
        np.testing.assert_array_equal(a[k], b[k])
    np.testing.assert_array_equal(a["q_tok"], b["q_tok"])


def test_lmhead_workload_layout():
    w = workloads.lmhead(seed=1, batch=3, gamma=2, vocab=500, hidden=128)
    assert w.target_hidden.shape == (3, 3, 128) and w.draft_hidden.shape == (3, 2, 128)
    assert w.target_weight.shape == (500, 128) and w.draft_weight is w.target_weight
    assert ((w.tokens >= 0) & (w.tokens < 500)).all()
    w2 = workloads.lmhead(seed=1, batch=3, gamma=2, vocab=500, hidden=128, shared_weight=False)
    assert w2.draft_weight is not w2.target_weight


def test_integer_valued_inputs_give_exact_dot_products():
    """Small integers are exact in bf16 and every partial sum below 2^53 is exact
    in float64: the logits equal Python integer arithmetic (brute force)."""
    rng = np.random.default_rng(7)
    D, V, R = 96, 33, 5
    h = rng.integers(-8, 9, size=(R, D))
    w = rng.integers(-8, 9, size=(V, D))
    hb = workloads.bits_to_f32(workloads.bf16_bits(h.astype(np.float32)))
    wb = workloads.bits_to_f32(workloads.bf16_bits(w.astype(np.float32)))
    assert (hb == h).all() and (wb == w).all()
    x = oracle.lm_logits(hb, wb)
    for r in range(R):
        for v in range(V):
            assert x[r, v] == sum(int(h[r, k]) * int(w[v, k]) for k in range(D))


def test_scaling_a_hidden_row_scales_its_logits():
    """h -> 2h doubles every logit exactly (a power of two is exact in both
    bf16 and float64); the other rows are untouched."""
    rng = np.random.default_rng(8)
    D, V = 64, 50
    h = workloads.bits_to_f32(workloads.bf16_bits(rng.standard_normal((2, D)).astype(np.float32)))
    w = workloads.bits_to_f32(workloads.bf16_bits(rng.standard_normal((V, D)).astype(np.float32)))
    x = oracle.lm_logits(h, w)
    h2 = h.copy()
    h2[1] *= 2.0
    x2 = oracle.lm_logits(h2, w)
    np.testing.assert_array_equal(x2[0], x[0])
    np.testing.assert_array_equal(x2[1], 2.0 * x[1])
