"""GPU parity: the CUDA path against the CPU oracle on the same seeded inputs.

Every call goes through the C ABI (libspecverify.so via the ctypes binding).
Workloads follow the benchmark configurations (sizes, value distributions,
temperatures); the full-size ones run in the launch shape the benchmark times
(the handle's default).
"""
import json
import os

import numpy as np
import pytest

from speculative_decoding_verification_90_b200 import workloads

from parity import assert_parity, compare, gpu_run, oracle_run, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _report(name, s):
    print(f"\n[{name}] seqs={s['sequences']} hard={len(s['hard'])} "
          f"margin={len(s['margin_cases'])} dq={s.get('max_dq')} dp={s.get('max_dp')} "
          f"lseT={s.get('max_target_lse_abs')} lseD={s.get('max_draft_lse_abs')} dz={s.get('max_dz')}")


def _check(wl, name, **kw):
    g = gpu_run(wl, **kw)
    o = oracle_run(wl)
    s = compare(wl, g, o)
    _report(name, s)
    assert_parity(s)
    assert g["status"] == 0 and g["bits"] == 0
    return g, o, s


# ---------------------------------------------------------------------------
# benchmark configurations
# ---------------------------------------------------------------------------

def test_char_level_calls_one_by_one():
    """B=1, gamma=4, V=256, fp32: 1000 independent calls, each its own launch."""
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    wl = workloads.char_level(calls=1000, seed=0)
    o = oracle_run(wl)
    d = to_device(wl)
    outs_t = np.empty((wl.batch, wl.gamma + 1), np.int32)
    outs_n = np.empty(wl.batch, np.int32)
    with SpecVerify(1, wl.gamma, wl.vocab, "f32") as sv:
        ot = torch.empty((1, wl.gamma + 1), dtype=torch.int32, device="cuda")
        on = torch.empty((1,), dtype=torch.int32, device="cuda")
        for b in range(wl.batch):
            sv.run(d["target"][b:b + 1], d["draft"][b:b + 1], d["tokens"][b:b + 1],
                   d["u_accept"][b:b + 1], d["u_resample"][b:b + 1], 1.0, ot, on)
            outs_t[b] = ot.cpu().numpy()[0]
            outs_n[b] = on.cpu().numpy()[0]
        assert sv.status() == (0, 0)
    s = compare(wl, {"out_tokens": outs_t, "out_num_accepted": outs_n}, o, check_probs=False)
    _report("char_level x1000 calls", s)
    assert_parity(s)


def test_char_level_batched():
    wl = workloads.char_level(calls=1000, seed=0)
    _check(wl, "char_level batched")


def test_b8_g3_v32000():
    _check(workloads.b8_g3_v32000(seed=0), "b8_g3_v32000")


@pytest.mark.slow
def test_b64_g8_v128256_full_size():
    _check(workloads.b64_g8_v128256(seed=0), "b64_g8_v128256")


@pytest.mark.slow
def test_multibranch_full_size():
    wl = workloads.multibranch(seed=0)
    g, o, s = _check(wl, "multibranch")
    # branches of a sequence share the rows before the branch point: their
    # decisions there are computed from identical inputs and must agree
    K = wl.meta["branches"]
    rb = g["q_tok"].reshape(-1, K, wl.gamma)
    shared = wl.meta["shared"].reshape(-1, K, wl.gamma)
    for s_ in range(rb.shape[0]):
        cols = shared[s_, 0]
        assert (rb[s_, :, cols] == rb[s_, :1, cols]).all()


@pytest.mark.slow
def test_exactness_config_parity_and_law():
    """B=60000 rows at one position with TV(p, q) = 0.657; GPU vs oracle and vs q."""
    beta = json.load(open(os.path.join(GOLDEN, "exactness_beta.json")))["beta"]
    wl = workloads.exactness(beta, batch=60000, seed=0)
    g, o, s = _check(wl, "exactness")
    import oracle
    q0, _, _ = oracle.softmax(wl.target[0, 0], 1.0)
    N, V = wl.batch, wl.vocab
    emp = np.bincount(g["out_tokens"][:, 0], minlength=V) / N
    tv = 0.5 * np.abs(emp - q0).sum()
    rng = np.random.default_rng(1234)
    direct = [0.5 * np.abs(np.bincount(rng.choice(V, N, p=q0), minlength=V) / N - q0).sum()
              for _ in range(20)]
    print(f"\n[exactness] TV(gpu samples, q) = {tv:.4f}; direct sampling {np.mean(direct):.4f} "
          f"+- {np.std(direct):.4f}")
    assert tv <= np.mean(direct) + 3 * np.std(direct)


# ---------------------------------------------------------------------------
# launch shapes, alignment, ragged vocabularies
# ---------------------------------------------------------------------------

def _small(seed, B, G, V, dtype, T=1.0, mix=0.8, sigma=3.0):
    rng = np.random.default_rng(seed)
    tgt = (rng.standard_normal((B, G + 1, V)) * sigma).astype(np.float32)
    drf = (mix * tgt[:, :G] + (1 - mix) * rng.standard_normal((B, G, V)) * sigma).astype(np.float32)
    return workloads._finish(f"small_{B}_{G}_{V}_{dtype}", dtype, T, tgt, drf, rng)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("V", [1, 7, 64, 1000, 4099, 50257])
def test_vocab_sizes_and_ragged_tails(dtype, V):
    wl = _small(V, 24, 3, V, dtype, T=0.9)
    for slices, threads in [(1, 256), (3, 128), (8, 512), (64, 256)]:
        g = gpu_run(wl, slices=slices, threads=threads)
        s = compare(wl, g, oracle_run(wl))
        _report(f"V={V} {dtype} S={slices} NT={threads}", s)
        assert_parity(s)


@pytest.mark.parametrize("slices", [1, 2, 4, 5, 8, 13, 31])
@pytest.mark.parametrize("threads", [128, 256, 512])
def test_launch_shapes(slices, threads):
    wl = _small(11, 16, 5, 32000, "bf16", T=0.7, mix=0.9)
    g = gpu_run(wl, slices=slices, threads=threads)
    s = compare(wl, g, oracle_run(wl))
    assert_parity(s)


@pytest.mark.parametrize("draw_slices", [1, 2, 5, 31])
def test_draw_shapes(draw_slices):
    wl = _small(22, 20, 4, 32000, "bf16", T=0.9)
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    with SpecVerify(wl.batch, wl.gamma, wl.vocab, "bf16") as sv:
        s0, t0 = sv.launch()
        sv.set_launch(s0, t0, draw_slices)
        g = gpu_run(wl, sv=sv)
    assert_parity(compare(wl, g, oracle_run(wl)))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_misaligned_pointers_take_scalar_path(dtype):
    """Logit tensors offset by one element from a 16-byte boundary."""
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    wl = _small(12, 8, 2, 1024, dtype)
    d = to_device(wl)
    B, G, V = wl.batch, wl.gamma, wl.vocab
    for key, shape in (("target", (B, G + 1, V)), ("draft", (B, G, V))):
        big = torch.empty(d[key].numel() + 1, dtype=d[key].dtype, device="cuda")
        view = big[1:].view(shape)
        view.copy_(d[key])
        d[key] = view
        assert view.data_ptr() % 16 != 0
    g = gpu_run(wl, inputs=d)
    s = compare(wl, g, oracle_run(wl))
    assert_parity(s)


# ---------------------------------------------------------------------------
# edge cases of the method
# ---------------------------------------------------------------------------

def test_gamma_zero_is_plain_sampling():
    wl = _small(13, 50, 0, 300, "f32")
    g, o, s = _check(wl, "gamma=0")
    assert (g["out_num_accepted"] == 0).all()


def test_gamma_above_warp_width():
    wl = _small(14, 6, 40, 500, "bf16", mix=0.97)
    _check(wl, "gamma=40")


def test_identical_distributions_accept_all():
    rng = np.random.default_rng(15)
    B, G, V = 12, 6, 5000
    tgt = (rng.standard_normal((B, G + 1, V)) * 3).astype(np.float32)
    wl = workloads._finish("same", "bf16", 1.0, tgt, tgt[:, :G].copy(), rng)
    g, o, s = _check(wl, "p == q")
    assert (g["out_num_accepted"] == G).all()
    assert np.allclose(g["ratio"], 1.0, atol=1e-6)


def test_disjoint_supports_reject_first():
    rng = np.random.default_rng(16)
    B, G, V = 20, 3, 2048
    tgt = (rng.standard_normal((B, G + 1, V)) * 2).astype(np.float32)
    drf = (rng.standard_normal((B, G, V)) * 2).astype(np.float32)
    tgt[:, :, V // 2:] = -np.inf
    drf[:, :, : V // 2] = -np.inf
    wl = workloads._finish("disjoint", "f32", 1.0, tgt, drf, rng)
    g, o, s = _check(wl, "disjoint")
    assert (g["out_num_accepted"] == 0).all()
    assert (g["out_tokens"][:, 0] < V // 2).all()


def test_masked_vocab_entries_and_temperatures():
    for T in (0.05, 0.5, 1.0, 3.0):
        rng = np.random.default_rng(int(T * 100))
        B, G, V = 10, 4, 3000
        tgt = (rng.standard_normal((B, G + 1, V)) * 3).astype(np.float32)
        drf = (0.8 * tgt[:, :G] + 0.2 * rng.standard_normal((B, G, V)) * 3).astype(np.float32)
        mask = rng.random((B, 1, V)) < 0.3
        tgt = np.where(mask, -np.inf, tgt).astype(np.float32)
        drf = np.where(mask[:, :, :], -np.inf, drf).astype(np.float32)
        wl = workloads._finish(f"masked_T{T}", "bf16", T, tgt, drf, rng)
        _check(wl, f"masked T={T}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("V", [64, 4099, 152064])
def test_zero_residual_mass_falls_back_to_target(dtype, V):
    """Rows equal except at the drafted token t of the rejecting position, where
    the target logit is -1000 (q(t) underflows to 0) and the draft's -690
    (-688 in bf16; p(t) about 1e-300): t is rejected with ratio 0, every other
    q(i) equals p(i), so the residual max(0, q - p) has no mass.  The draw then
    comes from q at that position with the same uniform, and the ZERO_MASS
    warning is raised.  At V = 152064 the draw's recomputation of q's tile
    masses covers the whole row in one place (the rows the other draw warps
    had covered)."""
    rng = np.random.default_rng(V)
    B, G = 24, 2
    tgt = (rng.standard_normal((B, G + 1, V)) * 2).astype(np.float32)
    drf = tgt[:, :G].copy()
    n = rng.integers(0, G, size=B)
    tok = np.zeros((B, G), np.int32)
    for b in range(B):
        for j in range(G):
            tok[b, j] = int(np.argmax(tgt[b, j]))
        t = int(rng.integers(0, V))
        tok[b, n[b]] = t
        tgt[b, n[b], t] = -1000.0
        drf[b, n[b], t] = -690.0
    wl = workloads._finish(f"zero_mass_{V}_{dtype}", dtype, 1.0, tgt, drf, rng, tokens=tok)
    wl.u_accept[:] = 0.5
    g = gpu_run(wl)
    o = oracle_run(wl)
    assert (o["seq_status"] == 18).all()
    assert g["bits"] == 4 and g["status"] == 18
    np.testing.assert_array_equal(g["out_num_accepted"], n)
    s = compare(wl, g, o, check_probs=False)
    _report(f"zero mass V={V} {dtype}", s)
    assert not s["unresolved"]
    assert_parity(s)


def test_tokens_at_vocab_edges():
    wl = _small(17, 30, 3, 777, "f32", mix=0.6)
    wl.tokens[:, 0] = 0
    wl.tokens[:, 1] = wl.vocab - 1
    _check(wl, "edge tokens")


def test_data_errors_set_status_and_empty_outputs():
    wl = _small(18, 6, 3, 256, "f32")
    wl.tokens[1, 2] = 256
    wl.tokens[2, 0] = -5
    wl.target[3, 3, 17] = np.nan
    wl.draft[4, 1, :] = -np.inf
    g = gpu_run(wl)
    o = oracle_run(wl)
    assert o["seq_status"].tolist() == [0, 16, 16, 17, 17, 0]
    s = compare(wl, g, o, check_probs=False)
    assert not s["hard"], s
    for b in (1, 2, 3, 4):
        assert g["out_num_accepted"][b] == 0 and (g["out_tokens"][b] == -1).all()
    assert g["bits"] == 3
    assert g["status"] == 16


def test_repeated_calls_reset_tickets_and_are_deterministic():
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    wl = _small(19, 32, 4, 8192, "bf16")
    d = to_device(wl)
    o = oracle_run(wl)
    with SpecVerify(wl.batch, wl.gamma, wl.vocab, "bf16") as sv:
        first = None
        for _ in range(5):
            g = gpu_run(wl, inputs=d, sv=sv)
            if first is None:
                first = g
                assert_parity(compare(wl, g, o))
            else:
                assert np.array_equal(g["out_tokens"], first["out_tokens"])
                assert np.array_equal(g["out_num_accepted"], first["out_num_accepted"])
                assert np.array_equal(g["target_lse"], first["target_lse"])


def test_host_buffer_entry_point_matches_device_entry_point():
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    wl = _small(20, 16, 3, 4096, "bf16")
    g = gpu_run(wl)
    t = torch.from_numpy(wl.target.view(np.int16)).view(torch.bfloat16).pin_memory()
    dr = torch.from_numpy(wl.draft.view(np.int16)).view(torch.bfloat16).pin_memory()
    ot = torch.empty((wl.batch, wl.gamma + 1), dtype=torch.int32).pin_memory()
    on = torch.empty((wl.batch,), dtype=torch.int32).pin_memory()
    with SpecVerify(wl.batch, wl.gamma, wl.vocab, "bf16") as sv:
        sv.run_host(t, dr, torch.from_numpy(wl.tokens), torch.from_numpy(wl.u_accept),
                    torch.from_numpy(wl.u_resample), wl.temperature, ot, on)
    assert np.array_equal(ot.numpy(), g["out_tokens"])
    assert np.array_equal(on.numpy(), g["out_num_accepted"])


def test_empty_batch_is_a_no_op():
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    with SpecVerify(0, 3, 100, "f32") as sv:
        e = torch.empty(0, device="cuda")
        sv.run(e.view(0, 4, 100), e.view(0, 3, 100), e.int().view(0, 3), e.view(0, 3), e,
               1.0, e.int().view(0, 4), e.int())
        assert sv.status() == (0, 0)


def test_invalid_arguments_rejected_before_launch():
    from speculative_decoding_verification_90_b200 import specverify as S
    h = S.specverify_create(4, 2, 100, S.SV_DTYPE_F32, 0)
    try:
        x = torch.zeros(4 * 3 * 100, device="cuda")
        i = torch.zeros(16, dtype=torch.int32, device="cuda")
        for T in (0.0, -1.0, float("nan"), float("inf")):
            with pytest.raises(S.SpecVerifyError):
                S.specverify_run(h, x.data_ptr(), x.data_ptr(), i.data_ptr(), x.data_ptr(),
                                 x.data_ptr(), T, i.data_ptr(), i.data_ptr(), 0)
        with pytest.raises(S.SpecVerifyError):
            S.specverify_run(h, 0, x.data_ptr(), i.data_ptr(), x.data_ptr(), x.data_ptr(), 1.0,
                             i.data_ptr(), i.data_ptr(), 0)
        with pytest.raises(S.SpecVerifyError):
            S.specverify_run(h, x.data_ptr() + 1, x.data_ptr(), i.data_ptr(), x.data_ptr(),
                             x.data_ptr(), 1.0, i.data_ptr(), i.data_ptr(), 0)
        for c, t, d in ((0, 256, 0), (9, 256, 0), (2, 100, 0), (1, 128, 65)):
            with pytest.raises(S.SpecVerifyError):
                S.specverify_set_launch(h, c, t, d)
    finally:
        S.specverify_destroy(h)
    for args in ((-1, 2, 100), (4, -1, 100), (4, 2, 0), (4, 256, 100)):
        with pytest.raises(S.SpecVerifyError):
            S.specverify_create(*args, S.SV_DTYPE_F32, 0)
