"""The multi-GPU path on CPU: world-size-2 gloo ranks (no GPU).

The mixer shards with no data exchange -- heads (and sequences) are
independent -- so N GPUs run N independent problems (weak scaling) and the
only collectives are the bench's barrier and its max-over-ranks timing.  These
tests run that host logic as two gloo processes: each rank cuts its own
contiguous head shard out of the packed inputs with the library's sharding
helpers (the tensors a caller would hand to the C ABI on that rank), computes
it with the CPU oracle, and the gathered shards equal the unsharded result bit
for bit; max_over_ranks returns the slowest rank's value; the
per-rank seeds give different problems.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outq):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from linear_attention_serving_prefill_b200.workloads import prefill_inputs
        from oracle import oracle

        from linear_attention_serving_prefill_b200.sharding import head_shard, shard_inputs

        # Head sharding: every rank builds its contiguous block of heads of the
        # same problem the way a caller of the library would (5 heads: 3 + 2).
        x = prefill_inputs([9, 0, 20], 5, 8, 6, "f32", seed=3, s0_std=0.1)
        heads = head_shard(world, rank, 5)
        sub = shard_inputs(x, heads)
        for key in ("q", "k", "v", "z", "beta", "A", "initial_state"):
            assert sub[key].is_contiguous()
        o, S = oracle.prefill(sub["q"], sub["k"], sub["v"], sub["z"], sub["A"], sub["beta"],
                              sub["cu_seqlens_host"], sub["initial_state"])
        got_o = [None] * world
        got_S = [None] * world
        dist.all_gather_object(got_o, (heads, o))
        dist.all_gather_object(got_S, (heads, S))
        # max over ranks and per-rank seeds
        slow = bench.max_over_ranks(float(10 + rank), world)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(2, rank))
        if rank == 0:
            outq.put((got_o, got_S, slow, seeds))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_heads_without_exchange():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got_o, got_S, slow, seeds = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    from linear_attention_serving_prefill_b200.workloads import prefill_inputs
    from oracle import oracle
    x = prefill_inputs([9, 0, 20], 5, 8, 6, "f32", seed=3, s0_std=0.1)
    o_ref, S_ref = oracle.prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"],
                                  x["cu_seqlens_host"], x["initial_state"])
    from linear_attention_serving_prefill_b200.sharding import gather_heads
    assert [h for h, _ in got_o] == [[0, 1, 2], [3, 4]]
    o = gather_heads([torch.from_numpy(oh) for _, oh in got_o]).numpy()
    S = gather_heads([torch.from_numpy(sh) for _, sh in got_S]).numpy()
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(S, S_ref)
    assert slow == 11.0
    assert seeds[0] != seeds[1]
