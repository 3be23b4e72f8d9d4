"""The seeded workload recipes (host logic, no GPU): the sweep's covering
subset holds every value of every axis."""
from indexer_top_sparse_c4_b200 import workloads as wl


def test_sweep_cases_cover_every_axis_value():
    axes = (wl.SWEEP_CONTEXTS, wl.SWEEP_BATCHES, wl.SWEEP_HEADS, wl.SWEEP_BUDGETS, wl.SWEEP_KV, wl.SWEEP_DISTS)
    for i, values in enumerate(axes):
        assert {case[i] for case in wl.SWEEP_CASES} == set(values), i
    assert len(set(wl.SWEEP_CASES)) == len(wl.SWEEP_CASES)
