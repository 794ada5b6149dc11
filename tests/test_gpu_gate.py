"""GPU parity of the fold gate (specfold_gate_run) against the CPU oracle.

Decision parity: the recompute flag of every row equals the oracle's except
where the oracle's relative margin |d - tau| / tau is below GATE_MARGIN (the
sums of squares are fp32 per lane on the GPU, fp64 in the oracle); packed rows,
provenance and sources are then bit-exact, and the packed batch holds exactly
the hidden rows it names.  rel_diff agrees within GATE_REL_TOL relative.
"""
import ctypes

import numpy as np
import pytest

from speculative_decoding_verification_90_b200 import workloads

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

GATE_MARGIN = 1e-5
GATE_REL_TOL = 1e-5


def _dev_hidden(h, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(h).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(h, np.float32)).cuda()


def gpu_gate(hidden, parent, tau, dtype, packed_hidden=True, optional=True, gate=None,
             dev_hidden=None):
    from speculative_decoding_verification_90_b200.specverify import FoldGate
    nb, npos, dim = hidden.shape
    own = gate is None
    g = FoldGate(nb, npos, dim, dtype) if own else gate
    try:
        H = dev_hidden if dev_hidden is not None else _dev_hidden(hidden, dtype)
        par = torch.from_numpy(np.ascontiguousarray(parent, np.int32)).cuda()
        rows = nb * npos
        packed = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
        n = torch.full((1,), -7, dtype=torch.int32, device="cuda")
        rel = torch.full((nb, npos), -7.0, dtype=torch.float32, device="cuda") if optional else None
        prov = torch.full((nb, npos), -7, dtype=torch.int32, device="cuda") if optional else None
        src = torch.full((nb, npos), -7, dtype=torch.int32, device="cuda") if optional else None
        ph = torch.zeros((rows, dim), dtype=H.dtype, device="cuda") if packed_hidden else None
        g.run(H, par, tau, packed, n, rel_diff=rel, provenance=prov, source=src,
              packed_hidden=ph)
        torch.cuda.synchronize()
        st, bits = g.status()
        k = int(n.item())
        out = {"packed": packed.cpu().numpy()[:k], "n": k, "status": st, "bits": bits}
        if optional:
            out.update(rel_diff=rel.cpu().numpy(), provenance=prov.cpu().numpy(),
                       source=src.cpu().numpy())
        if packed_hidden:
            out["packed_hidden"] = ph[:k]
            out["hidden_dev"] = H
        return out
    finally:
        if own:
            g.close()


def check(hidden, parent, tau, dtype, name, **kw):
    import oracle
    g = gpu_gate(hidden, parent, tau, dtype, **kw)
    o = oracle.gate(hidden, np.asarray(parent, np.int32), tau)
    margin = o["margin"] < GATE_MARGIN
    rec_o = o["recompute"].astype(bool)
    rec_g = np.zeros_like(rec_o).ravel()
    rec_g[g["packed"]] = True
    rec_g = rec_g.reshape(rec_o.shape)
    bad = (rec_g != rec_o) & ~margin
    print(f"\n[{name}] rows={rec_o.size} packed={g['n']} oracle={len(o['packed'])} "
          f"margin_rows={int(margin.sum())} differing={int((rec_g != rec_o).sum())}")
    assert not bad.any(), np.argwhere(bad)[:5]
    assert (np.diff(g["packed"]) > 0).all()
    if not (rec_g != rec_o).any():
        np.testing.assert_array_equal(g["packed"], o["packed"])
        if "provenance" in g:
            np.testing.assert_array_equal(g["provenance"], o["provenance"])
            np.testing.assert_array_equal(g["source"], o["source"])
    if "rel_diff" in g:
        d_o = o["rel_diff"]
        fin = np.isfinite(d_o)
        np.testing.assert_array_equal(np.isinf(g["rel_diff"]), np.isinf(d_o))
        err = np.abs(g["rel_diff"][fin] - d_o[fin]) / np.maximum(d_o[fin], 1e-30)
        assert err.size == 0 or err.max() <= GATE_REL_TOL, err.max()
    if "packed_hidden" in g and g["n"]:
        H = g["hidden_dev"].reshape(-1, hidden.shape[2])
        idx = torch.from_numpy(g["packed"].astype(np.int64)).cuda()
        assert torch.equal(g["packed_hidden"], H[idx])
    expect_status = 20 if o["status"] == oracle.GATE_ERR_PARENT else 0
    assert g["status"] == expect_status and bool(g["bits"]) == bool(expect_status)
    return g, o


def test_gate_full_size():
    """128 sequences x 8 branches, 32 positions, hidden 4096, bf16 (the benchmark case)."""
    w = workloads.gate_tree()
    g, o = check(w.hidden, w.parent, w.tau, w.dtype, w.name)
    assert 0 < g["n"] < w.rows


@pytest.mark.parametrize("seqs,branches,positions,dim,dtype,tau", [
    (3, 4, 5, 1001, "f32", 0.05),     # f32, odd hidden size: scalar loads
    (6, 5, 7, 1536, "bf16", 0.08),    # 1.5B-model hidden size, rows not a multiple of 8
    (2, 3, 3, 100, "bf16", 0.05),     # 200-byte rows: scalar loads
    (40, 8, 32, 256, "bf16", 0.05),   # 10240 rows: 1280 blocks, several scan chunks
    (1, 1, 1, 8, "f32", 0.05),        # one row, no parent
    (5, 8, 32, 4096, "f32", 0.05),    # 16 KB rows: half-row stages of the bulk-copy ring
    (2, 4, 3, 3000, "bf16", 0.05),    # 6000-byte rows: 17 whole-row stages, one warp each
    (2, 4, 3, 12800, "f32", 0.05),    # 51200-byte rows: the largest the ring takes (4 half-row stages)
    (2, 4, 3, 12804, "f32", 0.05),    # 51216-byte rows: register form
    (1, 3, 2, 2048, "bf16", 0.05),    # 6 rows: fewer rows than SMs, two blocks with nothing to read
])
def test_gate_shapes(seqs, branches, positions, dim, dtype, tau):
    w = workloads.gate_tree(seed=seqs + dim, sequences=seqs, branches=branches,
                            positions=positions, dim=dim, dtype=dtype, tau=tau)
    check(w.hidden, w.parent, w.tau, w.dtype, w.name)


@pytest.mark.parametrize("tau", [0.0, float("inf"), 0.02, 1.0])
def test_gate_tau_range(tau):
    w = workloads.gate_tree(seed=7, sequences=8, branches=6, positions=16, dim=512, tau=tau)
    g, o = check(w.hidden, w.parent, tau, w.dtype, f"tau={tau}")
    if tau == float("inf"):
        assert g["n"] == 8 * 16                    # the roots' rows only


@pytest.mark.parametrize("parent", [
    [-1, 0, 9, 1],          # out of range
    [-1, 1, 1, 0],          # self link and a child of it
    [-1, 2, 1, 0],          # two-cycle
    [-1, 2, 3, 2, 0, 4],    # a chain into a cycle
    [-5, 0, 1, 2],          # bad negative at the top
])
def test_gate_invalid_parents(parent):
    rng = np.random.default_rng(len(parent))
    nb = len(parent)
    h = rng.standard_normal((nb, 4, 64)).astype(np.float32)
    h[1:] = h[0] + np.float32(0.01) * rng.standard_normal((nb - 1, 4, 64)).astype(np.float32)
    g, o = check(h, parent, 0.05, "f32", f"parents {parent}")
    assert g["status"] == 20


def test_gate_deep_chain_max_branches():
    """16384 branches in one chain (the largest tree), each a copy of its parent:
    every row folds and its source is the root's row."""
    nb, npos, dim = 16384, 1, 16
    rng = np.random.default_rng(5)
    h = np.broadcast_to(rng.standard_normal((1, npos, dim)).astype(np.float32),
                        (nb, npos, dim)).copy()
    parent = np.arange(-1, nb - 1, dtype=np.int32)
    h[100, 0, 3] += 5.0          # one branch differs: its subtree now sources from it
    g, o = check(h, parent, 0.05, "f32", "deep chain")
    assert g["n"] == 3           # the root, branch 100 and branch 101 (differs from 100)


def test_gate_optional_outputs_absent_and_repeat():
    w = workloads.gate_tree(seed=3, sequences=4, branches=8, positions=32, dim=768)
    from speculative_decoding_verification_90_b200.specverify import FoldGate
    H = _dev_hidden(w.hidden, w.dtype)
    with FoldGate(w.branches, w.positions, w.dim, w.dtype) as gate:
        first = None
        for i in range(4):
            g = gpu_gate(w.hidden, w.parent, w.tau, w.dtype, packed_hidden=(i % 2 == 0),
                         optional=(i % 2 == 1), gate=gate, dev_hidden=H)
            assert g["status"] == 0
            first = first if first is not None else g["packed"]
            np.testing.assert_array_equal(g["packed"], first)
    import oracle
    np.testing.assert_array_equal(first, oracle.gate(w.hidden, w.parent, w.tau)["packed"])


def test_gate_invalid_arguments():
    from speculative_decoding_verification_90_b200 import specverify as m
    with pytest.raises(m.SpecVerifyError):
        m.specfold_gate_create(16385, 1, 8, m.SV_DTYPE_F32, 0)
    with pytest.raises(m.SpecVerifyError):
        m.specfold_gate_create(4, 0, 8, m.SV_DTYPE_F32, 0)
    with m.FoldGate(2, 2, 8, "f32") as gate:
        H = torch.zeros((2, 2, 8), device="cuda")
        par = torch.tensor([-1, 0], dtype=torch.int32, device="cuda")
        packed = torch.empty(4, dtype=torch.int32, device="cuda")
        n = torch.empty(1, dtype=torch.int32, device="cuda")
        for tau in (float("nan"), -1.0):
            assert m._lib.specfold_gate_run(gate.handle, H.data_ptr(), par.data_ptr(),
                                            ctypes.c_float(tau), None, None, None,
                                            packed.data_ptr(), n.data_ptr(), None,
                                            None) == m.SV_ERR_INVALID_ARG
        assert m._lib.specfold_gate_run(gate.handle, H.data_ptr(), par.data_ptr(),
                                        ctypes.c_float(0.1), None, None, None, None,
                                        n.data_ptr(), None, None) == m.SV_ERR_INVALID_ARG
        assert m._lib.specfold_gate_run(gate.handle, H.data_ptr() + 2, par.data_ptr(),
                                        ctypes.c_float(0.1), None, None, None,
                                        packed.data_ptr(), n.data_ptr(), None,
                                        None) == m.SV_ERR_INVALID_ARG
        gate.run(H, par, 0.1, packed, n)
        torch.cuda.synchronize()
        assert gate.status()[0] == 0 and int(n.item()) == 2
