"""Host logic of the bench's timed region, on the CPU with a stand-in for the
CUDA graph API: the steps captured and replayed are exactly the K steps the
JSON line reports, in order modulo the inputs' rotation period, and the
launch description says what runs."""
import contextlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


class _FakeGraph:
    capturing = None

    def __init__(self):
        self.steps = []
        self.log = None

    def replay(self):
        self.log.extend(self.steps)


class _FakeCuda:
    def __init__(self, log):
        self._log = log

        class Graph(_FakeGraph):
            pass

        def make():
            g = Graph()
            g.log = log
            return g

        self.CUDAGraph = make

    @contextlib.contextmanager
    def graph(self, g, stream=None):
        _FakeGraph.capturing = g
        try:
            yield
        finally:
            _FakeGraph.capturing = None

    @contextlib.contextmanager
    def stream(self, s):
        yield

    def synchronize(self):
        pass


class _FakeTorch:
    def __init__(self):
        self.replayed = []
        self.cuda = _FakeCuda(self.replayed)


def _step(i):
    assert _FakeGraph.capturing is not None, "a step ran outside a capture"
    _FakeGraph.capturing.steps.append(i)


@pytest.mark.parametrize("K,g_max,period", [(20, 1200, 3), (1200, 1200, 3), (2500, 1200, 3), (20000, 1200, 4),
                                            (7, 4, 2), (1, 1200, 3)])
def test_graph_steps_replay_exactly_k_steps(K, g_max, period):
    torch = _FakeTorch()
    gs = bench.GraphSteps(torch, None, _step, K, g_max)
    torch.replayed.clear()                    # the untimed upload replay
    gs.replays(1)                             # what the timed region runs
    got = torch.replayed
    assert len(got) == K
    if g_max % period == 0 or K <= g_max:
        # step j of the run uses the input that step j names
        assert [i % period for i in got] == [j % period for j in range(K)]
    desc = gs.launch()
    if K <= g_max:
        assert desc == f"one CUDA graph of the {K} steps, replayed once"
    else:
        assert f"exactly {K} steps" in desc and f"replayed {K // g_max} times" in desc
        assert (f"one graph of {K % g_max} steps" in desc) == (K % g_max != 0)


def test_capture_steps_records_the_named_range():
    torch = _FakeTorch()
    g = bench.capture_steps(torch, None, _step, 5, 3)
    assert g.steps == [5, 6, 7]


def test_gpu_launches_per_step_follow_the_merge_rule():
    """One launch (the decode) when no sequence can span two tiles, two (decode
    and merge) otherwise; the tile is 128 rows on tcgen05, 64 on CUDA cores."""
    from grouped_query_attention_mqa_b200.workloads import WORKLOADS
    long = WORKLOADS["long_mqa_b64_m8k"]
    paper = WORKLOADS["paper_mqa_b128_m128"]
    assert bench.launches_per_step(long, "tcgen05", 0) == 2
    assert bench.launches_per_step(long, "tcgen05", 128) == 1
    assert bench.launches_per_step(paper, "tcgen05", 0) == 1
    assert bench.launches_per_step(paper, "simt", 0) == 2
