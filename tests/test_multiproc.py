"""Multi-process (world size 2, gloo, CPU) checks of the host-side N>1 logic.

The attention path shards by batch (or by key/value-head group) with no
exchange, so what runs across processes is set-up, the batch split and the
max-over-ranks timing reduction. These run here on CPU; the per-shard compute
is the oracle, which shows that splitting the batch changes no result.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from attention_gqa_b200 import shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    r, w = shard.init_from_env("gloo", timeout_s=60)
    assert (r, w) == (rank, world)
    try:
        # the batch split covers every sequence exactly once
        for batch in (0, 1, 2, 5, 64):
            spans = [None] * world
            dist.all_gather_object(spans, shard.batch_range(batch, rank, world))
            covered = [b for lo, hi in spans for b in range(lo, hi)]
            assert covered == list(range(batch)), (batch, spans)

        # max over ranks, element-wise
        got = shard.max_over_ranks([rank + 0.5, 10.0 - rank, -rank])
        assert got == [world - 0.5, 10.0, 0.0], got

        # batch-sharded attention equals the unsharded result (oracle as the compute)
        import oracle
        import synth
        x = synth.make_prefill_inputs(1, 0, 3, 16)
        q, k, v = (synth.bf16_bits_to_f64(x[n]) for n in ("q", "k", "v"))
        lo, hi = shard.batch_range(3, rank, world)
        part = oracle.prefill(q[lo:hi], k[lo:hi], v[lo:hi], x["sinks"], x["pos"][lo:hi], 5)
        parts = [None] * world
        dist.all_gather_object(parts, part)
        if rank == 0:
            full = oracle.prefill(q, k, v, x["sinks"], x["pos"], 5)
            assert np.array_equal(np.concatenate(parts, axis=0), full)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_batch_range_single_process():
    assert shard.batch_range(10, 0, 1) == (0, 10)
    assert [shard.batch_range(10, r, 4) for r in range(4)] == [(0, 3), (3, 6), (6, 8), (8, 10)]
    with pytest.raises(ValueError):
        shard.batch_range(4, 2, 2)
    assert shard.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]  # no process group: identity


def test_two_ranks_gloo():
    import oracle
    oracle._load()  # build the oracle library once, before the ranks start
    mp.spawn(_worker, args=(2, _free_port()), nprocs=2, join=True)
