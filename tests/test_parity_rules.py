"""The decision-parity rules of the GPU tests, checked on the CPU: outputs equal
to the oracle's pass, a changed decision with a resolvable margin fails, and a
residual draw whose residual mass is below what fp32 resolves is accepted only
when the emitted token is valid."""
import numpy as np
import pytest

from speculative_decoding_verification_90_b200 import workloads

from parity import RESID_RESOLVE, compare, compare_sampling, oracle_run_sampling

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
