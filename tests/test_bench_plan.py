"""The bench's step planning (CPU): exactly K timed steps, no empty graph,
whole rotations per graph, and an instance count whose footprint exceeds 4x
the L2, for the step counts the bench is run with."""

import pytest

import bench


@pytest.mark.parametrize("K", [1, 2, 5, 20, 95, 96, 97, 200, 2000, 4096, 200000])
@pytest.mark.parametrize("R", [1, 12, 96, 100])
def test_plan_graphs_times_exactly_K_steps(K, R):
    per, n_full, tail = bench.plan_graphs(K, R)
    assert per >= 1 and n_full >= 1 and 0 <= tail
    assert per * n_full + tail == K
    if K >= R:
        assert per % R == 0                      # whole rotations: step j of a graph runs instance j % R
        assert tail < per
        assert per <= max(2048, R)
    else:
        assert (per, n_full, tail) == (K, 1, 0)  # K distinct instances, once each
    # the instance sequence of the timed steps is the rotation 0, 1, ..., R-1, 0, ...
    seq = [j % R for _ in range(n_full) for j in range(per)] + [j % R for j in range(tail)]
    assert seq == [i % R for i in range(K)]


def test_plan_graphs_driver_command():
    # bench.py --steps 20 at the headline workload: one graph of 20 distinct instances
    assert bench.plan_graphs(20, 96) == (20, 1, 0)
    assert bench.plan_graphs(200000, 96) == (2016, 99, 416)


@pytest.mark.parametrize("K,R", [(0, 96), (5, 0), (-1, 3)])
def test_plan_graphs_rejects_empty(K, R):
    with pytest.raises(ValueError):
        bench.plan_graphs(K, R)


def test_instances_exceed_four_l2():
    l2 = 126 * 2 ** 20
    step = bench.algorithmic_bytes(bench.get_config(bench.WORKLOAD), 16384)
    for S in (1, 7, 32):
        R = bench.instances_needed(step, l2, S)
        assert R * step >= 4 * l2 and R % S == 0
        assert (R - S) * step < 4 * l2 or R == S
    assert bench.instances_needed(step, l2, 1, minimum=500) == 500
