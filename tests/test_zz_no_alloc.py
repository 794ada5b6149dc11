"""The allocation-free entry point (specverify_run_noalloc) against the handle's.

Some callers cannot allocate device memory: code inside a captured graph region
that must not call cudaMalloc, embedders whose memory belongs to a pool they
cannot reach from this library, serving paths that forbid allocation.  For them
the library keeps its workspace in one static device array.  These tests call
the entry point through the C ABI, twice in a row (the array keeps the previous
call's contents), and check the outputs against specverify_run on the same
inputs; decisions must be identical, the tolerance of every parity test here.
This file is collected last on purpose.
"""
import numpy as np
import pytest

from speculative_decoding_verification_90_b200 import workloads

from parity import gpu_run, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _workload(seed, B, G, V, dtype, T):
    rng = np.random.default_rng(seed)
    tgt = (rng.standard_normal((B, G + 1, V)) * 3).astype(np.float32)
    drf = (0.8 * tgt[:, :G] + 0.2 * rng.standard_normal((B, G, V)) * 3).astype(np.float32)
    return workloads._finish(f"noalloc_{B}_{G}_{V}_{dtype}", dtype, T, tgt, drf, rng)


@pytest.mark.parametrize("dtype,V,T", [("bf16", 32000, 0.7), ("f32", 4099, 1.0)])
def test_noalloc_matches_the_handle_entry_point_on_two_calls(dtype, V, T):
    from speculative_decoding_verification_90_b200 import specverify as S
    wl = _workload(31, 24, 4, V, dtype, T)
    d = to_device(wl)
    ref = gpu_run(wl, inputs=d, readback=False)
    code = S.SV_DTYPE_BF16 if dtype == "bf16" else S.SV_DTYPE_F32
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        out_t = torch.full((wl.batch, wl.gamma + 1), -7, dtype=torch.int32, device="cuda")
        out_n = torch.full((wl.batch,), -7, dtype=torch.int32, device="cuda")
        S.specverify_run_noalloc(wl.batch, wl.gamma, wl.vocab, code, d["target"].data_ptr(),
                                 d["draft"].data_ptr(), d["tokens"].data_ptr(),
                                 d["u_accept"].data_ptr(), d["u_resample"].data_ptr(), T,
                                 out_t.data_ptr(), out_n.data_ptr(), stream)
        torch.cuda.synchronize()
        assert np.array_equal(out_t.cpu().numpy(), ref["out_tokens"])
        assert np.array_equal(out_n.cpu().numpy(), ref["out_num_accepted"])


def _noalloc(S, wl, d, T=None):
    code = S.SV_DTYPE_BF16 if wl.dtype == "bf16" else S.SV_DTYPE_F32
    out_t = torch.full((wl.batch, wl.gamma + 1), -7, dtype=torch.int32, device="cuda")
    out_n = torch.full((wl.batch,), -7, dtype=torch.int32, device="cuda")
    S.specverify_run_noalloc(wl.batch, wl.gamma, wl.vocab, code, d["target"].data_ptr(),
                             d["draft"].data_ptr(), d["tokens"].data_ptr(),
                             d["u_accept"].data_ptr(), d["u_resample"].data_ptr(),
                             wl.temperature if T is None else T, out_t.data_ptr(),
                             out_n.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return out_t.cpu().numpy(), out_n.cpu().numpy()


def test_noalloc_calls_of_different_shapes_in_a_row():
    """What one call leaves in the shared array must not reach the next: a
    large batch and vocabulary, then a smaller one, then one whose sequence 1
    holds an out-of-range token (its error outcome), then a clean one; and a
    call rejected for its temperature in between, which must enqueue nothing.
    Each call's outputs equal the handle entry point's on the same inputs."""
    from speculative_decoding_verification_90_b200 import specverify as S
    calls = [_workload(41, 64, 6, 50257, "bf16", 1.0), _workload(42, 9, 2, 3001, "f32", 0.8),
             _workload(43, 16, 3, 8192, "bf16", 1.0), _workload(44, 16, 3, 8192, "bf16", 1.0)]
    calls[2].tokens[1, 1] = calls[2].vocab + 5
    for i, wl in enumerate(calls):
        d = to_device(wl)
        ref = gpu_run(wl, inputs=d, readback=False)
        if i == 3:
            with pytest.raises(S.SpecVerifyError) as err:
                _noalloc(S, wl, d, T=float("nan"))
            assert err.value.status == S.SV_ERR_INVALID_ARG
        got_t, got_n = _noalloc(S, wl, d)
        assert np.array_equal(got_t, ref["out_tokens"]), i
        assert np.array_equal(got_n, ref["out_num_accepted"]), i
        if i == 2:
            assert got_n[1] == 0 and (got_t[1] == -1).all()


def test_noalloc_rejects_a_batch_beyond_its_scratch():
    from speculative_decoding_verification_90_b200 import specverify as S
    B, G, V = 60000, 1, 4096  # needs more than the 16 MiB static workspace
    with pytest.raises(S.SpecVerifyError) as err:
        S.specverify_run_noalloc(B, G, V, S.SV_DTYPE_F32, 16, 16, 16, 16, 16, 1.0, 16, 16, 0)
    assert err.value.status == S.SV_ERR_INVALID_ARG
    assert "scratch" in S.specverify_last_error()
