"""GPU parity of the shared-row entry point (specverify_run_mapped).

Each distinct logit row is given once, with int32 maps from every (sequence,
position) to its row.  The oracle knows nothing of maps: it runs on the rows
the maps pick out, materialised on the host by plain indexing.  The mapped
step must also reproduce the plain entry point bit for bit on those rows,
since it performs the same arithmetic on the same data.
"""
import ctypes

import numpy as np
import pytest

from speculative_decoding_verification_90_b200 import workloads

from parity import assert_parity, compare, gpu_run, oracle_run, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

READBACK = ("target_lse", "draft_lse", "q_tok", "p_tok", "ratio", "resid_mass")


def _report(name, s):
    print(f"\n[{name}] seqs={s['sequences']} hard={len(s['hard'])} "
          f"margin={len(s['margin_cases'])} dq={s.get('max_dq')} dp={s.get('max_dp')} "
          f"lseT={s.get('max_target_lse_abs')} lseD={s.get('max_draft_lse_abs')} dz={s.get('max_dz')}")


def _check_mapped(wl, name):
    g = gpu_run(wl, mapped=True)
    o = oracle_run(wl)
    s = compare(wl, g, o)
    _report(name, s)
    assert_parity(s)
    assert g["status"] == 0 and g["bits"] == 0
    return g, o


def _same_as_plain(wl, g):
    """Mapped and plain runs agree bit for bit in one explicit launch shape.

    A tapered statistics grid (the default on large batches) cuts a row by
    its place in the run's row order, which differs between the two entry
    points; an explicit shape cuts every row alike."""
    S, NT = g["launch"]
    m = gpu_run(wl, mapped=True, slices=S, threads=NT)
    p = gpu_run(wl, slices=S, threads=NT)
    assert p["launch"] == m["launch"] == (S, NT)
    np.testing.assert_array_equal(m["out_tokens"], p["out_tokens"])
    np.testing.assert_array_equal(m["out_num_accepted"], p["out_num_accepted"])
    for key in READBACK:
        np.testing.assert_array_equal(m[key], p[key], err_msg=key)


def test_multibranch_full_size_mapped():
    """32 sequences x 8 branches, gamma=5, V=152064, bf16: the benchmark's shared-row case."""
    wl = workloads.multibranch()
    m = wl.meta
    rows = m["target_rows"].shape[0] + m["draft_rows"].shape[0]
    assert rows < wl.batch * (2 * wl.gamma + 1)
    g, _ = _check_mapped(wl, "multibranch mapped")
    _same_as_plain(wl, g)


def test_multibranch_small_ragged_vocab():
    """V=50257: bf16 rows of 100514 bytes, not a multiple of 16 (scalar-load path)."""
    wl = workloads.multibranch(seed=5, sequences=6, branches=4, gamma=5, vocab=50257)
    g, _ = _check_mapped(wl, "multibranch small ragged")
    _same_as_plain(wl, g)


@pytest.mark.parametrize("B,G,V,nt,nd,dtype,T", [
    (24, 4, 5000, 40, 30, "f32", 1.0),      # many-to-one across sequences
    (16, 7, 32000, 9, 5, "bf16", 0.7),     # few rows, long drafts
    (8, 3, 1000, 1, 1, "f32", 1.0),        # every position reads the same row
    (40, 2, 4099, 120, 80, "f32", 1.3),    # as many rows as positions, shuffled
    (5, 40, 2048, 60, 33, "bf16", 1.0),    # gamma past one warp of positions
])
def test_random_maps(B, G, V, nt, nd, dtype, T):
    wl = workloads.random_maps(seed=B + G, batch=B, gamma=G, vocab=V, target_rows=nt,
                               draft_rows=nd, dtype=dtype, temperature=T)
    g, _ = _check_mapped(wl, f"random maps {B}x{G}x{V} {nt}/{nd} {dtype}")
    _same_as_plain(wl, g)


def test_gamma_zero_mapped():
    """gamma = 0: only the bonus draw from the mapped target row."""
    wl = workloads.random_maps(seed=11, batch=24, gamma=0, vocab=3000, target_rows=10,
                               draft_rows=0)
    g, _ = _check_mapped(wl, "gamma 0 mapped")
    _same_as_plain(wl, g)


def test_identity_maps_equal_plain_run():
    """The per-position layout with identity maps is the plain step."""
    wl = workloads.b8_g3_v32000(seed=2)
    B, G, V = wl.batch, wl.gamma, wl.vocab
    wl.meta.update({"target_rows": wl.target.reshape(B * (G + 1), V),
                    "target_map": np.arange(B * (G + 1), dtype=np.int32).reshape(B, G + 1),
                    "draft_rows": wl.draft.reshape(B * G, V),
                    "draft_map": np.arange(B * G, dtype=np.int32).reshape(B, G)})
    g, _ = _check_mapped(wl, "identity maps")
    _same_as_plain(wl, g)


def test_row_index_out_of_range():
    """A bad map entry voids its sequence only and is reported as SV_ERR_ROW_INDEX."""
    from speculative_decoding_verification_90_b200 import specverify as sv_mod
    wl = workloads.random_maps(seed=3, batch=12, gamma=4, vocab=4000, target_rows=20,
                               draft_rows=15)
    d = to_device(wl)
    d["target_map"][3, 1] = 20          # one past the last target row
    d["target_map"][7, 4] = -1          # the bonus position of sequence 7
    d["draft_map"][5, 0] = 15
    g = gpu_run(wl, inputs=d, mapped=True)
    assert g["status"] == sv_mod.SV_ERR_ROW_INDEX
    assert g["bits"] & 8
    bad = [3, 5, 7]
    for b in bad:
        assert g["out_num_accepted"][b] == 0
        assert (g["out_tokens"][b] == -1).all()
    o = oracle_run(wl)
    good = [b for b in range(wl.batch) if b not in bad]
    s = compare(wl, g, o, seqs=good)
    _report("row index error", s)
    assert_parity(s)


def test_mapped_invalid_arguments():
    """Argument errors are returned by the C entry point before anything is enqueued."""
    from speculative_decoding_verification_90_b200 import specverify as sv_mod
    wl = workloads.random_maps(seed=4, batch=6, gamma=2, vocab=2000, target_rows=7, draft_rows=5)
    d = to_device(wl)
    B, G = wl.batch, wl.gamma
    out_t = torch.empty((B, G + 1), dtype=torch.int32, device="cuda")
    out_n = torch.empty((B,), dtype=torch.int32, device="cuda")
    with sv_mod.SpecVerify(B, G, wl.vocab, wl.dtype) as sv:
        def call(nt=7, tmap=None, nd=5, dmap=None):
            tmap = d["target_map"].data_ptr() if tmap is None else tmap
            dmap = d["draft_map"].data_ptr() if dmap is None else dmap
            return sv_mod._lib.specverify_run_mapped(
                sv.handle, d["target_rows"].data_ptr(), nt, tmap, d["draft_rows"].data_ptr(), nd,
                dmap, d["tokens"].data_ptr(), d["u_accept"].data_ptr(), d["u_resample"].data_ptr(),
                ctypes.c_float(1.0), out_t.data_ptr(), out_n.data_ptr(), None)
        assert call(nt=0) == sv_mod.SV_ERR_INVALID_ARG
        assert call(nt=B * (G + 1) + 1) == sv_mod.SV_ERR_INVALID_ARG
        assert call(nd=0) == sv_mod.SV_ERR_INVALID_ARG
        assert call(nd=B * G + 1) == sv_mod.SV_ERR_INVALID_ARG
        assert call(tmap=0) == sv_mod.SV_ERR_INVALID_ARG
        assert call(dmap=0) == sv_mod.SV_ERR_INVALID_ARG
        assert call(tmap=d["target_map"].data_ptr() + 2) == sv_mod.SV_ERR_INVALID_ARG
        assert call() == sv_mod.SV_OK
        torch.cuda.synchronize()
        assert sv.status()[0] == sv_mod.SV_OK
        with pytest.raises(ValueError):
            sv.run_mapped(d["target_rows"][:, :100], d["target_map"], d["draft_rows"],
                          d["draft_map"], d["tokens"], d["u_accept"], d["u_resample"], 1.0,
                          out_t, out_n)


def test_mapped_and_plain_calls_interleaved():
    """One handle alternating between the two entry points keeps giving the same results."""
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    wl = workloads.multibranch(seed=9, sequences=4, branches=4, gamma=5, vocab=32000)
    d = to_device(wl)
    with SpecVerify(wl.batch, wl.gamma, wl.vocab, wl.dtype) as sv:
        first = None
        for i in range(6):
            r = gpu_run(wl, inputs=d, sv=sv, mapped=(i % 2 == 0), readback=False)
            key = (r["out_tokens"].tobytes(), r["out_num_accepted"].tobytes())
            first = first or key
            assert key == first
            assert r["status"] == 0
