"""GPU parity of the single-launch form of the step (specverify_set_fused).

The whole step runs in one persistent kernel whose warps take statistics
units and draw chunks from one ordered task list; every case below is checked
decision by decision against the CPU oracle, like the three-kernel form in
test_gpu_parity.py, on the same seeded workloads.  The cases cover the task
layout (unit, chunk and lag settings, including a lag of zero and a lag of
the whole batch), the control words that each launch leaves at zero
(repeated calls, graph replays, alternation with the three-kernel form),
the error outcomes and the zero-mass fallback.
"""
import numpy as np
import pytest

from speculative_decoding_verification_90_b200 import workloads

from parity import assert_parity, compare, gpu_run, oracle_run, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _small(seed, B, G, V, dtype, T=1.0, mix=0.8, sigma=3.0):
    rng = np.random.default_rng(seed)
    tgt = (rng.standard_normal((B, G + 1, V)) * sigma).astype(np.float32)
    drf = (mix * tgt[:, :G] + (1 - mix) * rng.standard_normal((B, G, V)) * sigma).astype(np.float32)
    return workloads._finish(f"fused_{B}_{G}_{V}_{dtype}", dtype, T, tgt, drf, rng)


def _check(wl, fused=True):
    g = gpu_run(wl, fused=fused)
    o = oracle_run(wl)
    s = compare(wl, g, o)
    assert_parity(s)
    assert g["status"] == 0 and g["bits"] == 0
    return g, o, s


def test_single_launch_counts_one_kernel():
    """Launch counts: one in fused mode; otherwise statistics, decide and draw
    (three) at every batch size."""
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    with SpecVerify(4, 3, 4096, "bf16") as sv:
        assert sv.kernels_per_run() == 3 and sv.fused()[0] == 0  # off by default
        sv.set_fused(True)
        assert sv.kernels_per_run() == 1 and sv.fused()[0] == 1
        assert sv.kernels_per_run(mapped=True) == 3  # the mapped form keeps the kernels
        sv.set_fused(False)
        assert sv.kernels_per_run() == 3
    for B, G, V, dt in ((60000, 1, 4096, "f32"), (64, 8, 128256, "bf16")):
        with SpecVerify(B, G, V, dt) as sv:
            assert sv.kernels_per_run() == 3 and sv.kernels_per_run(mapped=True) == 3


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("V", [64, 1000, 4099, 50257])
def test_vocab_sizes(dtype, V):
    _check(_small(V + 3, 24, 3, V, dtype, T=0.9))


def test_gamma_zero_bonus_only():
    _check(_small(31, 9, 0, 3000, "bf16"))


def test_gamma_above_warp_width():
    _check(_small(32, 6, 40, 640, "f32", mix=0.97))


def test_char_level_batched():
    _check(workloads.char_level(calls=1000, seed=0))


def test_b8_g3_v32000():
    _check(workloads.b8_g3_v32000(seed=0))


@pytest.mark.parametrize("shape", [(160, 1, 0), (256, 4, 1), (1024, 8, 3), (4096, 64, 64),
                                   (2048, 5, 10 ** 6), (1024, 4096, 2)])
def test_task_layouts(shape):
    """Statistics units of 160 .. 4096 groups, draw chunks of 1 .. 4096 tiles
    (one chunk per row), lag 0 (a sequence's draw right after its
    statistics), 1, 2, 3, 64 and beyond the batch (every draw after every
    statistics unit)."""
    wl = _small(33, 40, 4, 20000, "bf16")
    _check(wl, fused=shape)


@pytest.mark.slow
def test_b64_g8_v128256_full_size():
    _check(workloads.b64_g8_v128256(seed=0))


@pytest.mark.slow
def test_multibranch_full_size():
    _check(workloads.multibranch(seed=0))


def test_repeated_calls_graph_replays_and_alternation():
    """Each launch leaves its control words at zero: five calls in a row, two
    replays of a captured graph of two calls, and calls alternating with the
    three-kernel form all give the first call's outputs."""
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    wl = _small(34, 32, 4, 8192, "bf16")
    d = to_device(wl)
    o = oracle_run(wl)
    with SpecVerify(wl.batch, wl.gamma, wl.vocab, "bf16") as sv:
        sv.set_fused(True)
        first = gpu_run(wl, inputs=d, sv=sv)
        assert_parity(compare(wl, first, o))
        for i in range(6):
            sv.set_fused(i % 2 == 0)
            g = gpu_run(wl, inputs=d, sv=sv, readback=False)
            assert np.array_equal(g["out_tokens"], first["out_tokens"])
            assert np.array_equal(g["out_num_accepted"], first["out_num_accepted"])
        sv.set_fused(True)
        ot = torch.full((wl.batch, wl.gamma + 1), -7, dtype=torch.int32, device="cuda")
        on = torch.full((wl.batch,), -7, dtype=torch.int32, device="cuda")
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                for _ in range(2):
                    sv.run(d["target"], d["draft"], d["tokens"], d["u_accept"], d["u_resample"],
                           wl.temperature, ot, on)
        torch.cuda.synchronize()
        for _ in range(2):
            ot.fill_(-7)
            graph.replay()
            torch.cuda.synchronize()
            assert np.array_equal(ot.cpu().numpy(), first["out_tokens"])
            assert np.array_equal(on.cpu().numpy(), first["out_num_accepted"])
        del graph
        assert sv.status() == (0, 0)


def test_data_errors_set_status_and_empty_outputs():
    wl = _small(35, 6, 3, 256, "f32")
    wl.tokens[1, 2] = 256
    wl.tokens[2, 0] = -5
    wl.target[3, 3, 17] = np.nan
    wl.draft[4, 1, :] = -np.inf
    g = gpu_run(wl, fused=True)
    o = oracle_run(wl)
    assert o["seq_status"].tolist() == [0, 16, 16, 17, 17, 0]
    s = compare(wl, g, o, check_probs=False)
    assert not s["hard"], s
    for b in (1, 2, 3, 4):
        assert g["out_num_accepted"][b] == 0 and (g["out_tokens"][b] == -1).all()
    assert g["bits"] == 3 and g["status"] == 16
    # the next call on clean inputs is unaffected
    wl.tokens[1, 2], wl.tokens[2, 0] = 3, 4
    wl.target[3, 3, 17] = 0.5
    wl.draft[4, 1, :] = 0.25
    _check(wl)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zero_residual_mass_falls_back_to_target(dtype):
    """The construction of the three-kernel test: rows equal except at the
    drafted token of the rejecting position, whose target logit underflows;
    the residual has no mass, the draw comes from q at that position and the
    ZERO_MASS warning is raised."""
    V = 20000
    rng = np.random.default_rng(V + 1)
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
    wl = workloads._finish(f"fused_zero_mass_{dtype}", dtype, 1.0, tgt, drf, rng, tokens=tok)
    wl.u_accept[:] = 0.5
    g = gpu_run(wl, fused=True)
    o = oracle_run(wl)
    assert (o["seq_status"] == 18).all()
    assert g["bits"] == 4 and g["status"] == 18
    np.testing.assert_array_equal(g["out_num_accepted"], n)
    s = compare(wl, g, o, check_probs=False)
    assert not s["unresolved"]
    assert_parity(s)


def test_misaligned_pointers_keep_three_kernels():
    """With the single launch on, a run whose logit pointers are not 16-byte
    aligned takes the three-kernel (scalar-load) path and still matches."""
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    wl = _small(36, 8, 2, 1000, "f32")
    o = oracle_run(wl)
    d = to_device(wl)
    tgt = torch.empty(d["target"].numel() + 1, dtype=torch.float32, device="cuda")[1:]
    tgt.copy_(d["target"].flatten())
    drf = torch.empty(d["draft"].numel() + 1, dtype=torch.float32, device="cuda")[1:]
    drf.copy_(d["draft"].flatten())
    d["target"] = tgt.view(d["target"].shape)
    d["draft"] = drf.view(d["draft"].shape)
    with SpecVerify(wl.batch, wl.gamma, wl.vocab, "f32") as sv:
        sv.set_fused(True)
        g = gpu_run(wl, inputs=d, sv=sv)
    assert_parity(compare(wl, g, o))


def test_invalid_settings_rejected():
    from speculative_decoding_verification_90_b200.specverify import SpecVerify, SpecVerifyError
    with SpecVerify(4, 3, 152064, "bf16") as sv:
        for args in [(True, 64), (True, 1 << 21), (True, 1024, -1), (True, 1024, 8, -2),
                     (True, 128)]:
            with pytest.raises(SpecVerifyError):
                sv.set_fused(*args)
        sv.set_fused(True, 4096, 4096, 0)
        assert sv.fused() == (1, 4096, 4096, 0)
