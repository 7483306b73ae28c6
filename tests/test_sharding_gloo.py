"""Multi-process (gloo, world size 2) test of the library's event sharding
(``farthest_point_sampling_b200.sharding``), used when the tokenizer runs on
several GPUs: events are split over ranks with no data-path exchange; each
rank tokenizes its shard; gathering the shards must reproduce the
single-process result event by event.  The per-rank compute here is the CPU
oracle, so the test needs no GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
import workloads
from farthest_point_sampling_b200 import sharding


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        full = bench.global_batch("c1", world)
        parts = sharding.partition_events(full.sizes(), full.K, world)
        c, f, off = sharding.shard_events(full.coords, full.feats, full.offsets, parts[rank])
        mine = workloads.Batch(c, f, off, full.K, full.assign_mode, full.k, full.lloyd_iters, full.charge_col)
        out = oracle.tokenize_batch(mine)
        # timing reduction as in bench.py: max over ranks
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        gathered = [None] * world
        dist.all_gather_object(gathered, (parts[rank].tolist(), {k: v for k, v in out.items() if v is not None}))
        if rank == 0:
            q.put((float(t.item()), gathered))
    finally:
        dist.destroy_process_group()


@pytest.mark.slow
def test_two_rank_sharding_matches_single_process():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    tmax, gathered = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert tmax == 2.0
    full = bench.global_batch("c1", world)
    ref = oracle.tokenize_batch(full)
    seen = np.zeros(full.B, bool)
    for events, out in gathered:
        events = np.array(events)
        assert not seen[events].any()
        seen[events] = True
        # map shard-local packed indices back to the full batch
        sizes = full.sizes()[events]
        shard_off = np.concatenate([[0], np.cumsum(sizes)])
        for j, e in enumerate(events):
            o0 = full.offsets[e]
            idx = out["centroid_idx"][j]
            want = ref["centroid_idx"][e]
            np.testing.assert_array_equal(np.where(idx >= 0, idx - shard_off[j] + o0, -1), want)
            np.testing.assert_array_equal(out["token_id"][shard_off[j]:shard_off[j + 1]],
                                          ref["token_id"][o0:o0 + sizes[j]])
            np.testing.assert_array_equal(out["pooled"][j], ref["pooled"][e])
    assert seen.all()


def test_partition_is_balanced_and_complete():
    b = workloads.make_workload("c1", B=512)
    for world in (2, 4, 8):
        parts = sharding.partition_events(b.sizes(), b.K, world)
        allev = np.sort(np.concatenate(parts))
        assert np.array_equal(allev, np.arange(b.B))
        cost = sharding.event_cost(b.sizes(), b.K)
        loads = np.array([cost[p].sum() for p in parts])
        # LPT bound: no rank exceeds the mean by more than the largest event
        assert loads.max() <= loads.mean() + cost.max() + 1e-9


def test_shard_events_torch_matches_numpy():
    b = workloads.make_workload("c1")
    parts = sharding.partition_events(b.sizes(), b.K, 3)
    for p in parts:
        c, f, off = sharding.shard_events(b.coords, b.feats, b.offsets, p)
        tc, tf, toff = sharding.shard_events(torch.from_numpy(b.coords), torch.from_numpy(b.feats),
                                             torch.from_numpy(b.offsets), p)
        np.testing.assert_array_equal(tc.numpy(), c)
        np.testing.assert_array_equal(tf.numpy(), f)
        np.testing.assert_array_equal(toff.numpy(), off)
        assert off[-1] == b.sizes()[p].sum()
    assert bench.partition_events is not None  # bench.py delegates to the library helper
