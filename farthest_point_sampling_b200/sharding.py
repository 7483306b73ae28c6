"""Event sharding over devices (one process per GPU).

Events are independent: FPS, the assignment, Lloyd and the pooling of one
event read only that event's points (Neptune README, "How it works", step 1:
every event is tokenized on its own).  A batch therefore splits over GPUs by
whole events, with no exchange step and no collective on the data path; each
rank runs the ordinary tokenizer on its shard.

The split balances the FPS cost, N*K point-centroid evaluations per event
with more than K points (events with N <= K only copy their points), by the
longest-processing-time rule: events in decreasing cost order, each to the
rank with the least load so far.  One event never spans two ranks.

Works on numpy arrays or torch tensors (CPU or CUDA) alike; only the event
sizes are read on the host.
"""
from __future__ import annotations

from typing import List, Sequence

import numpy as np

__all__ = ["event_cost", "partition_events", "shard_events"]


def _host_sizes(offsets) -> np.ndarray:
    if hasattr(offsets, "detach"):  # torch tensor
        offsets = offsets.detach().to("cpu").numpy()
    off = np.asarray(offsets, dtype=np.int64)
    return np.diff(off)


def event_cost(sizes, K: int) -> np.ndarray:
    """Relative cost of each event: N*K for an FPS event (N > K), a small
    copy cost for a passthrough event (N <= K)."""
    sizes = np.asarray(sizes, dtype=np.int64)
    return np.where(sizes > K, sizes.astype(np.float64) * K, sizes.astype(np.float64) * 0.01 + 1.0)


def partition_events(sizes, K: int, world: int) -> List[np.ndarray]:
    """Longest-processing-time split of events over ``world`` ranks by N*K
    cost.  Returns, per rank, the sorted event ids it owns (possibly empty)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = event_cost(sizes, K)
    order = np.argsort(-cost, kind="stable")
    load = np.zeros(world)
    parts: List[list] = [[] for _ in range(world)]
    for e in order:
        r = int(np.argmin(load))
        parts[r].append(int(e))
        load[r] += cost[e]
    return [np.array(sorted(p), dtype=np.int64) for p in parts]


def shard_events(coords, feats, offsets, events: Sequence[int]):
    """The packed (coords, feats, offsets) of the given events, in the given
    order, with offsets renumbered from 0.  Inputs are numpy arrays or torch
    tensors; the outputs have the same kind and device."""
    sizes = _host_sizes(offsets)
    off_h = np.zeros(len(sizes) + 1, np.int64)
    np.cumsum(sizes, out=off_h[1:])
    events = np.asarray(events, dtype=np.int64)
    new_off = np.zeros(len(events) + 1, np.int64)
    if len(events):
        np.cumsum(sizes[events], out=new_off[1:])
    if hasattr(coords, "detach"):  # torch
        import torch

        idx = [torch.arange(int(off_h[e]), int(off_h[e + 1]), device=coords.device) for e in events]
        sel = torch.cat(idx) if idx else torch.zeros(0, dtype=torch.long, device=coords.device)
        return (coords.index_select(0, sel).contiguous(), feats.index_select(0, sel).contiguous(),
                torch.from_numpy(new_off).to(offsets.device))
    cs = [coords[off_h[e]:off_h[e + 1]] for e in events]
    fs = [feats[off_h[e]:off_h[e + 1]] for e in events]
    c = np.ascontiguousarray(np.concatenate(cs)) if cs else coords[:0]
    f = np.ascontiguousarray(np.concatenate(fs)) if fs else feats[:0]
    return c, f, new_off
