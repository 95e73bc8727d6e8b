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


def test_sets_needed_exceeds_l2_for_every_timed_loop():
    names = bench.chain_of(bench.MAIN_WORKLOAD)
    shapes = bench.chain_shapes(names)
    ws = [M * K + 4 * M for M, N, K, _ in shapes]
    fp = bench.footprints(shapes, ws)
    # the step, both GEMMs and both quantisations are timed loops of the block
    assert set(fp) == {"step", "gemm0", "gemm1", "quant0", "quant1"}
    n = bench.sets_needed(fp)
    smallest = min(fp.values())
    # the smallest timed footprint times n exceeds 1.5 x L2 ...
    assert n * smallest > 1.5 * bench.L2_BYTES
    # ... and n is the smallest count that does
    assert (n - 1) * smallest <= 1.5 * bench.L2_BYTES
    (M0, N0, K0, _), (M1, N1, K1, _) = shapes
    assert fp["gemm0"] == M0 * K0 + N0 * K0 + 2 * M0 * N0
    assert fp["quant0"] == 3 * M0 * K0
    assert fp["step"] > fp["gemm0"] + fp["gemm1"]


def test_sets_needed_is_capped_for_tiny_workloads():
    fp = bench.footprints([(16, 256, 256, False)], [0])
    assert "quant0" not in fp  # too small to exceed L2 even over 16 sets
    assert bench.sets_needed(fp) == 16


def test_block_chain_is_the_dit_mlp_config():
    """The headline step: up-projection 3072 -> 12288 with GELU in its
    epilogue, then the row-parallel down-projection 12288 -> 3072, 4096
    tokens, each layer a full-size workload; the variant with the
    down-projection's quantisation fused into the up-projection has the same
    layers."""
    names = bench.chain_of(bench.MAIN_WORKLOAD)
    assert [a for _, a, _ in names] == [bench.ACT_GELU, bench.ACT_NONE]
    assert [f for _, _, f in names] == [False, False]
    assert [(n, a) for n, a, _ in bench.BLOCK_FUSED_QUANT] == [(n, a) for n, a, _ in names]
    assert [f for _, _, f in bench.BLOCK_FUSED_QUANT] == [True, False]
    assert bench.chain_shapes(names) == [(4096, 12288, 3072, True), (4096, 3072, 12288, True)]
    ops = sum(bench.algorithmic(*s)[0] for s in bench.chain_shapes(names))
    assert ops == 2 * 2 * 4096 * 12288 * 3072
    assert bench.chain_of("square_512x4096x4096") == (("square_512x4096x4096", bench.ACT_NONE,
                                                       False),)


def test_whole_job_value_and_compact_kernel_names():
    assert bench.whole_job_tops(1e12, 10, 2, 0.5) == pytest.approx(40.0)
    assert bench.short_kernel("gemm2sm_kernel<256, 3> (2-SM pair, 256x256 tiles)") == "pair256"
    assert bench.short_kernel("gemm_kernel<128, 3, 2> (1-SM, 128x128 tiles)") == "1sm128"
    assert bench.short_kernel("decode_kernel (swap-AB stream-K, needs a workspace)") == "decode"


def test_recorded_traffic_only_while_the_sources_match(tmp_path, monkeypatch):
    csrc = tmp_path / "w8a8_int8_dynamic_b200" / "csrc"
    csrc.mkdir(parents=True)
    fam = "gemm2sm_kernel"
    for i, f in enumerate(bench.TRAFFIC_SOURCES[fam]):
        (csrc / f).write_bytes(f"// source {i}\nint  f{i}(int x) {{ return x; }}  /* end */\n".encode())
    h = hashlib.sha256()
    for i, f in enumerate(bench.TRAFFIC_SOURCES[fam]):
        h.update(f"int f{i}(int x) {{ return x; }}\n".encode())
    (tmp_path / "profiles").mkdir()
    rec = {"mlp": {"gemm_bytes_per_launch": 123, "kernel_family": fam,
                   "source_sha256_16": h.hexdigest()[:16]},
           "odd": {"gemm_bytes_per_launch": 5, "kernel_family": "unknown",
                   "source_sha256_16": h.hexdigest()[:16]}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "HERE", str(tmp_path))
    assert bench.sources_hash(fam) == h.hexdigest()[:16]
    assert bench.recorded_traffic("mlp") == 123
    assert bench.recorded_traffic("other") is None
    assert bench.recorded_traffic("odd") is None
    # comments and layout do not count; code does
    last = csrc / bench.TRAFFIC_SOURCES[fam][-1]
    i = len(bench.TRAFFIC_SOURCES[fam]) - 1
    last.write_bytes(f"/* reworded */ int f{i}(int x)\n{{\n  return x;  // same code\n}}\n".encode())
    assert bench.recorded_traffic("mlp") == 123
    last.write_bytes(f"int f{i}(int x) {{ return x + 1; }}\n".encode())
    assert bench.recorded_traffic("mlp") is None


def test_code_text_keeps_literals_and_drops_comments():
    src = 'a = "// not a comment"; /* gone\n */ b = \'/\'; // gone\nc  =\t"x\\"y";'
    assert bench.code_text(src) == 'a = "// not a comment"; b = \'/\'; c = "x\\"y";'


def test_sweep_loops_hold_about_25_ms_of_work():
    peak, hbm = 3285.6, 6540.8
    rows = {}
    for name in bench.SWEEP:
        wl = bench.WORKLOADS[name]
        ops, gemm_bytes, _, _ = bench.algorithmic(wl.M, wl.N, wl.K, wl.bias)
        n = bench.sweep_steps(ops, gemm_bytes, peak, hbm)
        assert 100 <= n <= 2000
        t = max(ops / (peak * 1e12 * 0.6), gemm_bytes / (hbm * 1e9 * 0.8))
        if 100 < n < 2000:
            assert n * t == pytest.approx(25e-3, rel=0.01)
        rows[name] = n
    # the 4096-token MLP layers are the longest: a few hundred steps at most
    assert rows["dit_mlp_up_4096x12288x3072"] < 300
    assert rows["small_64x128x256"] == 2000
