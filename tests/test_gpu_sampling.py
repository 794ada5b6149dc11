"""GPU parity of the sampling-variant step (specverify_run_sampling) against the
CPU oracle of adjusted distributions (greedy, top-k, nucleus, per-sequence
temperature).  Every call goes through the C ABI."""
import ctypes

import numpy as np
import pytest

from speculative_decoding_verification_90_b200 import workloads

from parity import (assert_parity, compare_sampling, gpu_run_sampling, oracle_run_sampling,
                    to_device)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _check(wl, temps, name, top_k=0, top_p=1.0, max_margin_frac=0.02, max_unresolved_frac=0.01):
    g = gpu_run_sampling(wl, temps, top_k, top_p)
    o = oracle_run_sampling(wl, temps, top_k, top_p)
    s = compare_sampling(wl, g, o, top_k)
    print(f"\n[{name}] seqs={s['sequences']} hard={len(s['hard'])} margin={len(s['margin_cases'])} "
          f"unresolved={len(s['unresolved'])} "
          f"dq={s.get('max_dq')} dp={s.get('max_dp')} dz={s.get('max_dz')} "
          f"kept_t(mean)={float(np.mean(o['kept_target'])):.1f}")
    assert_parity(s, max_margin_frac=max_margin_frac, max_unresolved_frac=max_unresolved_frac)
    return g, o, s


@pytest.mark.parametrize("top_k,top_p", [(50, 0.9), (0, 0.9), (20, 1.0), (0, 1.0), (1, 1.0),
                                         (200, 0.5)])
def test_b8_filters(top_k, top_p):
    wl = workloads.b8_g3_v32000(seed=11)
    _check(wl, wl.temperature, f"b8 k={top_k} p={top_p}", top_k, top_p)


def test_b64_greedy_full_size():
    wl = workloads.b64_g8_v128256(seed=1)
    # let some drafts agree with the target's argmax so greedy prefixes are accepted
    tgt = workloads.bits_to_f32(wl.target)
    best = np.argmax(tgt, axis=2)
    wl.tokens[::2, :4] = best[::2, :4]
    g, o, _ = _check(wl, 0.0, "b64 greedy")
    assert g["out_num_accepted"].max() >= 4


@pytest.mark.parametrize("top_k,top_p", [(50, 0.9), (0, 0.95), (40, 1.0)])
def test_b64_filters_full_size(top_k, top_p):
    wl = workloads.b64_g8_v128256(seed=2)
    _check(wl, wl.temperature, f"b64 k={top_k} p={top_p}", top_k, top_p)


@pytest.mark.parametrize("T,top_k,top_p", [(1.0, 2000, 1.0), (0.7, 2000, 0.9), (1.3, 5000, 0.95),
                                           (0.05, 0, 0.9), (2.5, 0, 0.5), (1.0, 0, 0.9999),
                                           (1.0, 0, 0.02), (0.05, 3000, 1.0)])
def test_b64_band_cuts_full_size(T, top_k, top_p):
    """Large top-k sets (count bands) and nucleus cuts alone (mass bands) over
    temperatures that move the cut from the top band to the far tail.  At
    T = 0.05 q and p concentrate on a few entries, and after the cut the two
    agree to fp64 rounding at some rejected positions (the oracle's own
    residual mass there is 1e-80 or 2e-15): up to 5 % of the sequences may hold
    such an unresolved draw, each still checked for validity."""
    wl = workloads.b64_g8_v128256(seed=5)
    _check(wl, T, f"b64 T={T} k={top_k} p={top_p}", top_k, top_p,
           max_unresolved_frac=0.05 if T <= 0.05 else 0.01)


def test_flat_and_neg_inf_rows():
    """Rows of one repeated value (every entry in one band: more candidates than
    fit) and rows mostly -inf (the last band), with large top-k and nucleus cuts."""
    rng = np.random.default_rng(31)
    B, G, V = 6, 3, 40000
    tgt = (rng.standard_normal((B, G + 1, V)) * 2.0).astype(np.float32)
    drf = (0.8 * tgt[:, :G] + 0.2 * rng.standard_normal((B, G, V)) * 2.0).astype(np.float32)
    tgt[0] = 1.5
    drf[0] = 1.5
    tgt[1, :, 100:] = -np.inf
    drf[1, :, 200:] = -np.inf
    tgt[2, 1, :] = np.where(np.arange(V) % 3 == 0, 0.25, -np.inf)
    tok = workloads.gumbel_max_tokens(rng, drf, 1.0)
    wl = workloads.Workload("flat_inf", B, G, V, "f32", 1.0, tgt, drf, tok,
                            rng.random((B, G), dtype=np.float32), rng.random(B, dtype=np.float32))
    for k, p in ((0, 0.5), (0, 0.97), (3000, 1.0), (20000, 0.9), (300, 0.8)):
        _check(wl, 1.0, f"flat/-inf k={k} p={p}", k, p)


def test_multibranch_filters_full_size():
    wl = workloads.multibranch(seed=3)
    _check(wl, 1.0, "multibranch k=50 p=0.9", 50, 0.9)


def test_mixed_temperatures_and_errors():
    wl = workloads.b8_g3_v32000(seed=12)
    temps = np.array([0.7, 0.0, 1.5, -1.0, 0.3, np.nan, 0.0, 2.0], np.float32)
    g, o, _ = _check(wl, temps, "mixed temperatures", 30, 0.85)
    for b in (3, 5):
        assert o["seq_status"][b] == 21
        assert g["out_num_accepted"][b] == 0 and (g["out_tokens"][b] == -1).all()
    assert g["status"] == 21 and g["bits"] & 16


def test_top_k_one_equals_greedy():
    wl = workloads.b8_g3_v32000(seed=13)
    a = gpu_run_sampling(wl, 0.0)
    b = gpu_run_sampling(wl, 0.7, top_k=1)
    np.testing.assert_array_equal(a["out_tokens"], b["out_tokens"])


@pytest.mark.parametrize("V", [256, 50257, 1000])
def test_f32_and_ragged_vocab(V):
    rng = np.random.default_rng(V)
    B, G = 12, 4
    tgt = (rng.standard_normal((B, G + 1, V)) * 2.0).astype(np.float32)
    drf = (0.8 * tgt[:, :G] + 0.2 * rng.standard_normal((B, G, V)) * 2.0).astype(np.float32)
    tok = workloads.gumbel_max_tokens(rng, drf, 1.0)
    wl = workloads.Workload(f"ragged_{V}", B, G, V, "f32", 1.0, tgt, drf, tok,
                            rng.random((B, G), dtype=np.float32), rng.random(B, dtype=np.float32))
    _check(wl, 1.0, f"f32 V={V} k=10 p=0.8", 10, 0.8)
    _check(wl, 0.8, f"f32 V={V} p=0.97", 0, 0.97)


def test_tied_logits():
    """Integer-valued logits: many ties at the top-k and top-p thresholds."""
    rng = np.random.default_rng(21)
    B, G, V = 16, 3, 4096
    tgt = np.round(rng.standard_normal((B, G + 1, V)) * 2.0).astype(np.float32)
    drf = np.round(0.8 * tgt[:, :G] + 0.5 * rng.standard_normal((B, G, V))).astype(np.float32)
    tok = workloads.gumbel_max_tokens(rng, drf, 1.0)
    wl = workloads.Workload("tied", B, G, V, "f32", 1.0, tgt, drf, tok,
                            rng.random((B, G), dtype=np.float32), rng.random(B, dtype=np.float32))
    for k, p in ((7, 1.0), (0, 0.6), (100, 0.9)):
        _check(wl, 1.0, f"ties k={k} p={p}", k, p)


def test_sampling_invalid_arguments():
    from speculative_decoding_verification_90_b200 import specverify as m
    wl = workloads.b8_g3_v32000(seed=14)
    d = to_device(wl)
    temps = torch.full((wl.batch,), 0.7, device="cuda")
    ot = torch.empty((wl.batch, wl.gamma + 1), dtype=torch.int32, device="cuda")
    on = torch.empty((wl.batch,), dtype=torch.int32, device="cuda")
    with m.SpecVerify(wl.batch, wl.gamma, wl.vocab, wl.dtype) as sv:
        def call(k, p, t=temps.data_ptr()):
            return m._lib.specverify_run_sampling(
                sv.handle, d["target"].data_ptr(), d["draft"].data_ptr(), d["tokens"].data_ptr(),
                d["u_accept"].data_ptr(), d["u_resample"].data_ptr(), t, k, ctypes.c_float(p),
                ot.data_ptr(), on.data_ptr(), None)
        assert call(-1, 0.9) == m.SV_ERR_INVALID_ARG
        assert call(5, 0.0) == m.SV_ERR_INVALID_ARG
        assert call(5, float("nan")) == m.SV_ERR_INVALID_ARG
        assert call(5, 0.9, 0) == m.SV_ERR_INVALID_ARG
        assert call(5, 0.9) == m.SV_OK
        torch.cuda.synchronize()
        assert sv.status()[0] == m.SV_OK
