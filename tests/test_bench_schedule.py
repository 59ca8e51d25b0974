"""The decode bench's step structure: which projection of a layer reads which
one's output (host logic, no GPU)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import LLAMA3_8B_DECODE, WORKLOADS, LayerShape  # noqa: E402


def test_llama3_8b_layer_dependencies():
    # q_proj on the step input; gate_proj and up_proj on q_proj's output;
    # down_proj on up_proj's output
    assert bench.chain_sources(LLAMA3_8B_DECODE) == [-1, 0, 0, 2]


def test_sweep_and_unrelated_shapes():
    assert bench.chain_sources(WORKLOADS["decode_sweep"].shapes) == [-1, 0]
    shapes = (LayerShape("a", 256, 512), LayerShape("b", 128, 1024), LayerShape("c", 64, 256))
    assert bench.chain_sources(shapes) == [-1, -1, 0]


def test_every_source_feeds_a_matching_width():
    for wl in WORKLOADS.values():
        src = bench.chain_sources(wl.shapes)
        for i, d in enumerate(src):
            assert d < i
            if d >= 0:
                assert wl.shapes[d].N == wl.shapes[i].K


def test_launches_cover_the_steps_in_order():
    m = bench.DecodeModel(None, None, [None] * 32, [None] * 32, LLAMA3_8B_DECODE, 1, 8)
    for first, count in [(0, 20), (64, 2000), (5, 3), (3, 8), (0, 1)]:
        ls = m.launches(first, count)
        steps = [s for a, k in ls for s in range(a, a + k)]
        assert steps == list(range(first, first + count))
        assert all(1 <= k <= 8 for _, k in ls)
        assert all(k == 8 for _, k in ls[:-1])
