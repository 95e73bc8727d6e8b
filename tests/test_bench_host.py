"""Host logic of bench.py on CPU: how a step count is split into graph
replays, how many rotated input sets a workload needs to exceed L2, and when
the recorded DRAM traffic of the dominant kernel still applies."""
import hashlib
import json

import pytest

import bench


class FakeGraph:
    def __init__(self, calls, log):
        self.calls = list(calls)  # the set indices captured, in order
        self.log = log

    def replay(self):
        self.log.extend(self.calls)


@pytest.fixture
def fake_capture(monkeypatch):
    """bench.capture replaced by a recorder: each 'graph' remembers which
    input sets its steps use, and a replay appends them to a log."""
    log, captured = [], []

    def capture(fns, stream):
        g = FakeGraph([fn() for fn in fns], log)
        captured.append(g)
        return g

    monkeypatch.setattr(bench, "capture", capture)
    monkeypatch.setattr(bench.torch.cuda, "stream", lambda s: _NullCtx())
    return log, captured


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def _loop(nsets, per_graph=64):
    fns = [(lambda i=i: i) for i in range(nsets)]
    return bench.GraphLoop(fns, stream=None, per_graph=per_graph)


@pytest.mark.parametrize("nsets,steps", [(9, 40), (9, 63), (9, 64), (9, 2000), (7, 20000),
                                         (1, 5), (16, 100)])
def test_graph_loop_runs_exactly_k_steps_in_rotation(fake_capture, nsets, steps):
    log, _ = fake_capture
    lp = _loop(nsets)
    assert lp.per_graph % nsets == 0 and lp.per_graph >= nsets
    lp.prepare(steps)
    warm = len(log)  # prepare replays the tail graph once, outside timing
    assert warm == steps % lp.per_graph
    del log[:]
    lp.run(steps)
    assert len(log) == steps
    assert log == [i % nsets for i in range(steps)]


def test_graph_loop_uses_one_tail_graph_not_single_replays(fake_capture):
    log, captured = fake_capture
    lp = _loop(9)  # per_graph 63
    n_before = len(captured)
    lp.prepare(40)
    assert len(captured) == n_before + 1 and len(captured[-1].calls) == 40
    replays = []
    for g in [lp.graph] + lp.single + list(lp.tail.values()):
        g.replay = (lambda g=g: replays.append(g))
    lp.run(40 + 2 * lp.per_graph)
    assert replays == [lp.graph, lp.graph, lp.tail[40]]
    # a count that was not prepared still runs, one replay per step
    replays.clear()
    lp.run(5)
    assert replays == lp.single[:5]


def test_graph_loop_prepare_is_idempotent(fake_capture):
    _, captured = fake_capture
    lp = _loop(9)
    lp.prepare(40)
    n = len(captured)
    lp.prepare(40)
    lp.prepare(63)  # a multiple of per_graph needs no tail
    assert len(captured) == n


class FakeW8:
    def __init__(self, ws):
        self.ws = ws

    def linear_workspace_bytes(self, M, N, K):
        return self.ws


def test_sets_needed_exceeds_l2_for_every_timed_loop():
    wl = bench.WORKLOADS[bench.MAIN_WORKLOAD]
    w8 = FakeW8(ws=wl.M * wl.K + 4 * wl.M)
    n, per = bench.sets_needed(w8, wl)
    M, N, K = wl.M, wl.N, wl.K
    gemm_alone = M * K + N * K + 2 * M * N
    # the smallest timed footprint (the GEMM alone) times n exceeds 1.5 x L2 ...
    assert n * min(per, gemm_alone) > 1.5 * bench.L2_BYTES
    # ... and n is the smallest count that does
    assert (n - 1) * min(per, gemm_alone) <= 1.5 * bench.L2_BYTES
    assert per > gemm_alone


def test_sets_needed_is_capped_for_tiny_workloads():
    class WL:
        M, N, K = 16, 256, 256
    n, _ = bench.sets_needed(FakeW8(ws=0), WL)
    assert n == 16


def test_recorded_traffic_only_while_the_sources_match(tmp_path, monkeypatch):
    csrc = tmp_path / "w8a8_int8_dynamic_b200" / "csrc"
    csrc.mkdir(parents=True)
    for i, f in enumerate(bench.TRAFFIC_SOURCES):
        (csrc / f).write_bytes(f"// source {i}\n".encode())
    h = hashlib.sha256()
    for f in bench.TRAFFIC_SOURCES:
        h.update((csrc / f).read_bytes())
    (tmp_path / "profiles").mkdir()
    rec = {"square": {"gemm_bytes_per_launch": 123, "source_sha256_16": h.hexdigest()[:16]}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "HERE", str(tmp_path))
    assert bench.recorded_traffic("square") == 123
    assert bench.recorded_traffic("other") is None
    (csrc / bench.TRAFFIC_SOURCES[-1]).write_bytes(b"// changed\n")
    assert bench.recorded_traffic("square") is None

