"""The decision-parity rules of the GPU tests, checked on the CPU: outputs equal
to the oracle's pass, a changed decision with a resolvable margin fails, and a
residual draw whose residual mass is below what fp32 resolves is accepted only
when the emitted token is valid."""
import numpy as np
import pytest

from speculative_decoding_verification_90_b200 import workloads

from parity import RESID_RESOLVE, compare, compare_sampling, oracle_run, oracle_run_sampling

oracle = pytest.importorskip("oracle")


def _copy(o):
    return {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in o.items()}


def _small(seed=41):
    return workloads.b8_g3_v32000(seed=seed)


def _rejected(o, G):
    """Sequences with a residual draw (a rejection before the bonus position)."""
    return [b for b in range(len(o["out_num_accepted"]))
            if o["seq_status"][b] == 0 and o["out_num_accepted"][b] < G]


def test_identical_outputs_pass():
    wl = _small()
    o = oracle_run_sampling(wl, 1.0, 20, 0.9)
    s = compare_sampling(wl, _copy(o), o, 20)
    assert not s["hard"] and not s["margin_cases"] and not s["unresolved"]


def test_changed_draw_with_resolvable_mass_is_hard():
    wl = _small()
    o = oracle_run_sampling(wl, 1.0, 0, 1.0)
    rej = [b for b in _rejected(o, wl.gamma) if o["resid_mass"][b] >= RESID_RESOLVE
           and o["cdf_margin_norm"][b] >= 1e-6]
    assert rej
    b = rej[0]
    g = _copy(o)
    n = int(o["out_num_accepted"][b])
    g["out_tokens"][b, n] = (g["out_tokens"][b, n] + 1) % wl.vocab
    s = compare_sampling(wl, g, o)
    assert [h[0] for h in s["hard"]] == [b]
    s = compare(wl, g, o, check_probs=False)
    assert [h[0] for h in s["hard"]] == [b]


def test_unresolved_draw_checks_validity():
    wl = _small()
    o = oracle_run_sampling(wl, 1.0, 50, 1.0)
    b = _rejected(o, wl.gamma)[0]
    n = int(o["out_num_accepted"][b])
    o["resid_mass"][b] = 1e-12   # as if q and p agreed to fp32 resolution
    x = workloads.bits_to_f32(wl.target[b, n])
    order = np.argsort(-x, kind="stable")
    inside, outside = int(order[1]), int(order[5000])
    assert inside != o["out_tokens"][b, n]
    g = _copy(o)
    g["out_tokens"][b, n] = inside          # another token of the top-50 set: valid
    s = compare_sampling(wl, g, o, 50)
    assert not s["hard"] and [u[0] for u in s["unresolved"]] == [b]
    g["out_tokens"][b, n] = outside         # outside the top-k set: invalid
    s = compare_sampling(wl, g, o, 50)
    assert [h[0] for h in s["hard"]] == [b]
    g["out_tokens"][b, n] = wl.vocab        # out of range
    s = compare(wl, g, o, check_probs=False)
    assert [h[0] for h in s["hard"]] == [b]


def test_unresolved_plain_draw_needs_residual_support():
    """Plain step: an unresolved residual draw passes only with a token of the
    residual's support (q_n > p_n at fp32 precision); a token the draft
    favours, or one outside [0, V), is a hard difference; the count of
    unresolved draws is capped."""
    from parity import assert_parity
    wl = _small()
    o = oracle_run(wl)
    b = _rejected(o, wl.gamma)[0]
    n = int(o["out_num_accepted"][b])
    o["resid_mass"][b] = 1e-12
    T = float(np.float32(wl.temperature))
    q = oracle.softmax(wl.target[b, n], T)[0]
    p = oracle.softmax(wl.draft[b, n], T)[0]
    d = q - p
    d[int(o["out_tokens"][b, n])] = 0.0
    favoured_by_q, favoured_by_p = int(np.argmax(d)), int(np.argmin(d))
    assert d[favoured_by_q] > 0 > d[favoured_by_p]
    g = _copy(o)
    g["out_tokens"][b, n] = favoured_by_q
    s = compare(wl, g, o, check_probs=False)
    assert not s["hard"] and [u[0] for u in s["unresolved"]] == [b]
    assert_parity(s, max_unresolved_frac=0.0, report=False)   # one unresolved draw is allowed
    g["out_tokens"][b, n] = favoured_by_p
    s = compare(wl, g, o, check_probs=False)
    assert [h[0] for h in s["hard"]] == [b]
    # a second unresolved sequence exceeds the cap of max(1, 1% of 8)
    b2 = [c for c in _rejected(o, wl.gamma) if c != b][0]
    n2 = int(o["out_num_accepted"][b2])
    o["resid_mass"][b2] = 1e-12
    q2 = oracle.softmax(wl.target[b2, n2], T)[0]
    p2 = oracle.softmax(wl.draft[b2, n2], T)[0]
    d2 = q2 - p2
    d2[int(o["out_tokens"][b2, n2])] = 0.0
    g["out_tokens"][b, n] = favoured_by_q
    g["out_tokens"][b2, n2] = int(np.argmax(d2))
    s = compare(wl, g, o, check_probs=False)
    assert not s["hard"] and len(s["unresolved"]) == 2
    with pytest.raises(AssertionError):
        assert_parity(s, report=False)
