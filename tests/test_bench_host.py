"""Host-side checks of bench.py's timing plumbing (no GPU): the timed region
replays exactly --steps steps, rotating through the weight copies without a
break, and a recorded DRAM-traffic figure is reported only while the sources it
was measured on are unchanged."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _FakeGraph:
    """Stands in for a captured CUDA graph of fn(0..n-1): replay() calls them."""

    def __init__(self, fn, n):
        self.fn, self.n = fn, n

    def replay(self):
        for i in range(self.n):
            self.fn(i)


def _plan_steps(monkeypatch, n, copies, full=None):
    monkeypatch.setattr(bench, "capture", lambda torch, fn, k: _FakeGraph(fn, k))
    seen = []
    plan = bench.StepPlan(None, lambda i: seen.append(i % copies), n, copies, full=full)
    return plan, seen


def test_step_plan_replays_exactly_n_steps_in_rotation(monkeypatch):
    copies = 32
    for n in (1, 20, bench.GRAPH_STEPS - 1, bench.GRAPH_STEPS, 2 * bench.GRAPH_STEPS + 37, 100000):
        plan, seen = _plan_steps(monkeypatch, n, copies)
        plan.replay()
        assert len(seen) == n, n
        assert seen == [i % copies for i in range(n)], n
        assert plan.nfull == n // bench.GRAPH_STEPS
        assert (plan.rem is None) == (n % bench.GRAPH_STEPS == 0)


def test_step_plan_warmup_shares_the_full_graph(monkeypatch):
    plan, _ = _plan_steps(monkeypatch, 3000, 32)
    warm, seen = _plan_steps(monkeypatch, 2000, 32, full=plan.full)
    assert warm.full is plan.full
    warm.warm()  # one replay of each graph
    assert len(seen) == 2000 - bench.GRAPH_STEPS  # the shared full graph records into the first plan's list


def test_profiled_traffic_follows_the_sources(monkeypatch, tmp_path):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    other = tmp_path / "h.h"
    other.write_text("header\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.source_digest("k.cu,h.h")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "# comment line\n"
        f"gemv_x k.cu,h.h {digest} 12345\n")
    assert bench.profiled_traffic("gemv_x") == 12345.0
    assert bench.profiled_traffic("gemv_y") is None
    other.write_text("header, edited\n")  # any listed source changing voids the figure
    assert bench.profiled_traffic("gemv_x") is None

