"""Two-rank (gloo, CPU) checks of the multi-GPU host path: rank seeding, the
sequence split, the max-over-ranks timing reduction and the output gather.

Sequences are independent, so verifying a batch in two shards must give the
same outputs as verifying it whole; the CPU oracle stands in for the device
path here (no GPU on this host)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from speculative_decoding_verification_90_b200 import dist as svdist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        import oracle
        from speculative_decoding_verification_90_b200 import workloads
        svdist.init("gloo", timeout_s=60)
        assert svdist.env_rank() == (rank, rank, world)
        # weak scaling: every rank draws its own batch from its own seed
        seed = svdist.rank_seed(7, rank)
        mine = workloads.char_level(calls=40, seed=seed)
        # strong split of one shared batch: each rank verifies its shard
        full = workloads.char_level(calls=50, seed=3)
        lo, hi = svdist.shard(full.batch, world, rank)
        part = oracle.verify(full.target[lo:hi], full.draft[lo:hi], full.tokens[lo:hi],
                             full.u_accept[lo:hi], full.u_resample[lo:hi], 1.0)
        pad = 25  # equal shapes for all_gather: 50 sequences over 2 ranks
        toks = torch.full((pad, full.gamma + 1), -9, dtype=torch.int32)
        nums = torch.full((pad,), -9, dtype=torch.int32)
        toks[: hi - lo] = torch.from_numpy(part["out_tokens"])
        nums[: hi - lo] = torch.from_numpy(part["out_num_accepted"])
        all_t, all_n = svdist.gather_outputs(toks, nums)
        slowest = svdist.max_over_ranks(10.0 + rank)
        dist.barrier()
        result_q.put((rank, mine.tokens.sum().item(), slowest, all_t.numpy(), all_n.numpy()))
        dist.destroy_process_group()
    except Exception as e:  # report, never hang the parent
        result_q.put((rank, "error", repr(e), None, None))


def test_two_rank_gloo_path():
    import oracle
    from speculative_decoding_verification_90_b200 import workloads
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(2):
        rank, a, b, c, d = q.get(timeout=180)
        results[rank] = (a, b, c, d)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        assert results[rank][0] != "error", results[rank]
        assert results[rank][1] == 11.0  # max over ranks of 10 + rank
    assert results[0][0] != results[1][0]  # different seeds, different batches
    full = workloads.char_level(calls=50, seed=3)
    ref = oracle.verify(full.target, full.draft, full.tokens, full.u_accept, full.u_resample, 1.0)
    got_t, got_n = results[0][2], results[0][3]
    assert np.array_equal(got_t, results[1][2])
    assert np.array_equal(got_t, ref["out_tokens"])
    assert np.array_equal(got_n, ref["out_num_accepted"])


def test_shard_covers_the_batch_once():
    for batch in (0, 1, 7, 256, 60000):
        for world in (1, 2, 3, 8):
            spans = [svdist.shard(batch, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == batch
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    with pytest.raises(ValueError):
        svdist.shard(10, 2, 2)


# ---------------------------------------------------------------------------
# the sampling variants and the fold gate shard the same way: whole sequences
# per rank, no data-path collective; gathered results equal one whole run
# ---------------------------------------------------------------------------

_GATE = dict(seed=2, sequences=4, branches=8, positions=4, dim=64, dtype="f32", tau=0.2)
_LM = dict(seed=5, batch=6, gamma=3, vocab=700, hidden=128)


def _lm_verify(oracle, workloads, lm, lo, hi):
    """Sequences [lo, hi) of the LM-head workload: float64 logits of the
    output layer, then the verification on them."""
    f = workloads.bits_to_f32
    t = oracle.lm_logits(f(lm.target_hidden[lo:hi]), f(lm.target_weight))
    d = oracle.lm_logits(f(lm.draft_hidden[lo:hi]), f(lm.draft_weight))
    return oracle.verify(t, d, lm.tokens[lo:hi], lm.u_accept[lo:hi], lm.u_resample[lo:hi],
                         lm.temperature)


def _variants_worker(rank, world, port, result_q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        import oracle
        from speculative_decoding_verification_90_b200 import workloads
        svdist.init("gloo", timeout_s=60)
        # sampling variants: per-sequence temperatures travel with the shard
        wl = workloads.b8_g3_v32000(seed=21)
        temps = np.array([0.7, 0.0, 1.3, 0.9, 0.0, 2.0, 0.5, 1.0], np.float32)
        lo, hi = svdist.shard(wl.batch, world, rank)
        part = oracle.verify_sampling(wl.target[lo:hi], wl.draft[lo:hi], wl.tokens[lo:hi],
                                      wl.u_accept[lo:hi], wl.u_resample[lo:hi], temps[lo:hi],
                                      top_k=20, top_p=0.9)
        # fold gate: whole sequences (blocks of branches) per rank, parents rebased
        g = workloads.gate_tree(**_GATE)
        per = _GATE["branches"]
        s_lo, s_hi = svdist.shard(_GATE["sequences"], world, rank)
        b_lo, b_hi = s_lo * per, s_hi * per
        par = g.parent[b_lo:b_hi].copy()
        par[par >= 0] -= b_lo
        gate = oracle.gate(g.hidden[b_lo:b_hi], par, g.tau)
        # the step fused with the output layer: the batch split, the layer replicated
        lm = workloads.lmhead(**_LM)
        m_lo, m_hi = svdist.shard(lm.batch, world, rank)
        lm_part = _lm_verify(oracle, workloads, lm, m_lo, m_hi)
        mine = {"lo": lo, "tokens": part["out_tokens"], "n": part["out_num_accepted"],
                "b_lo": b_lo, "gate": gate, "lm_lo": m_lo, "lm_tokens": lm_part["out_tokens"],
                "lm_n": lm_part["out_num_accepted"]}
        everyone = [None] * world
        dist.all_gather_object(everyone, mine)
        dist.barrier()
        result_q.put((rank, everyone))
        dist.destroy_process_group()
    except Exception as e:  # report, never hang the parent
        result_q.put((rank, "error: " + repr(e)))


def test_two_rank_gloo_variants_and_gate():
    import oracle
    from speculative_decoding_verification_90_b200 import workloads
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_variants_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=240) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        assert not isinstance(results[rank], str), results[rank]
    shards = sorted(results[0], key=lambda m: m["lo"])

    wl = workloads.b8_g3_v32000(seed=21)
    temps = np.array([0.7, 0.0, 1.3, 0.9, 0.0, 2.0, 0.5, 1.0], np.float32)
    ref = oracle.verify_sampling(wl.target, wl.draft, wl.tokens, wl.u_accept, wl.u_resample,
                                 temps, top_k=20, top_p=0.9)
    np.testing.assert_array_equal(np.concatenate([m["tokens"] for m in shards]), ref["out_tokens"])
    np.testing.assert_array_equal(np.concatenate([m["n"] for m in shards]), ref["out_num_accepted"])

    g = workloads.gate_tree(**_GATE)
    per = _GATE["branches"]
    assert all(p < 0 or p // per == b // per for b, p in enumerate(g.parent))  # within a sequence
    whole = oracle.gate(g.hidden, g.parent, g.tau)
    npos = _GATE["positions"]

    def rebase(a, off):
        a = a.copy()
        a[a >= 0] += off
        return a

    for key in ("rel_diff", "recompute"):
        np.testing.assert_array_equal(np.concatenate([m["gate"][key] for m in shards]), whole[key])
    for key in ("provenance", "source"):
        np.testing.assert_array_equal(
            np.concatenate([rebase(m["gate"][key], m["b_lo"] * npos) for m in shards]), whole[key])
    np.testing.assert_array_equal(
        np.concatenate([m["gate"]["packed"] + m["b_lo"] * npos for m in shards]), whole["packed"])
    assert whole["packed"].size > 0 and whole["recompute"].sum() < whole["recompute"].size

    lm = workloads.lmhead(**_LM)
    lm_ref = _lm_verify(oracle, workloads, lm, 0, lm.batch)
    lm_shards = sorted(results[0], key=lambda m: m["lm_lo"])
    np.testing.assert_array_equal(np.concatenate([m["lm_tokens"] for m in lm_shards]),
                                  lm_ref["out_tokens"])
    np.testing.assert_array_equal(np.concatenate([m["lm_n"] for m in lm_shards]),
                                  lm_ref["out_num_accepted"])
