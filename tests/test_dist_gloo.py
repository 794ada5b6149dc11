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
