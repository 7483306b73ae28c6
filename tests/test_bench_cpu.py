"""bench.py's host-side baselines run on the CPU: the single-thread oracle rate
and the all-cores rate over cost-balanced event slices in spawned workers."""
import bench
import workloads


def test_all_cores_oracle_baseline():
    b = workloads.make_workload("c0")
    rate1, reps1, el1 = bench.cpu_oracle_rate(b, 0.2)
    assert rate1 > 0 and reps1 >= 1
    rate, w, reps, el = bench.cpu_oracle_rate_parallel(b, 0.3, rate1, max_workers=2)
    assert 1 <= w <= 2 and reps >= 1 and el > 0 and rate > 0


def test_slices_cover_every_event_once():
    b = workloads.make_workload("c1")
    for w in (1, 3, 8):
        parts = bench.partition_events(b.sizes(), b.K, w)
        got = sorted(int(e) for p in parts for e in p)
        assert got == list(range(b.B))
        assert sum(bench.shard(b, p).P for p in parts) == b.P
