"""The decode bench's graph replay schedule: exactly the requested steps, in
layer order, with whole model passes only where they start on a pass."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _expand(schedule, n):
    steps = []
    for kind, i in schedule:
        steps.extend(range(n) if kind == "pass" else [i])
    return steps


@pytest.mark.parametrize("first,count,n", [(0, 64, 32), (64, 3000, 32), (3, 40, 32), (1, 2, 32),
                                           (64, 20, 32), (5, 100, 7), (0, 0, 4), (31, 33, 32), (0, 1, 1)])
def test_schedule_covers_exactly_the_steps_in_order(first, count, n):
    sched = bench.replay_schedule(first, count, n)
    assert _expand(sched, n) == [s % n for s in range(first, first + count)]


def test_schedule_uses_whole_passes_where_it_can():
    sched = bench.replay_schedule(64, 3000, 32)
    passes = sum(1 for k, _ in sched if k == "pass")
    assert passes == 3000 // 32          # 64 is a pass boundary; the last 24 steps are single layers
    assert all(k == "layer" for k, _ in sched[passes:])
    # a run that starts mid-pass finishes that pass layer by layer first
    sched = bench.replay_schedule(30, 40, 32)
    assert sched[:2] == [("layer", 30), ("layer", 31)] and sched[2] == ("pass", 0)
