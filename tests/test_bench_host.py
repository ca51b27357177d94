"""Host-side logic of bench.py, without a GPU: the ordering of the pipelined
end-to-end loop (copy-in / compute / copy-out on three streams, two buffer
sets) checked against fake streams and events that record what is enqueued,
and the DRAM-traffic lookup that ties a committed ncu capture to the kernel
source it was taken on."""
import importlib.util
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    saved = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    finally:
        sys.argv = saved
    return mod


class _Log:
    def __init__(self):
        self.ops = []      # (stream, kind, arg)
        self.current = None


def _fake_torch(log):
    class Event:
        n = 0

        def __init__(self):
            Event.n += 1
            self.id = Event.n

        def record(self, stream):
            log.ops.append((stream.name, "record", self.id))

    class Stream:
        made = 0

        def __init__(self, device=None, name=None):
            if name is None:
                name = ("in", "out")[Stream.made]
                Stream.made += 1
            self.name, self.device = name, device

        def wait_event(self, ev):
            log.ops.append((self.name, "wait", ev.id))

        def wait_stream(self, other):
            log.ops.append((self.name, "wait_stream", other.name))

    class StreamCtx:
        def __init__(self, s):
            self.s = s

        def __enter__(self):
            self.prev, log.current = log.current, self.s

        def __exit__(self, *exc):
            log.current = self.prev

    cuda = types.SimpleNamespace(Stream=Stream, Event=Event, stream=StreamCtx)
    return types.SimpleNamespace(cuda=cuda), Stream


def _simulate(ops):
    """Replay the enqueued operations on in-order streams where a wait blocks
    until the event's most recent record (at enqueue time) has executed;
    returns the order in which the work items ran."""
    streams = {}
    last_record = {}
    for i, (s, kind, arg) in enumerate(ops):
        if kind == "wait":
            arg = (arg, last_record.get(arg))
        if kind == "record":
            last_record[arg] = i
        streams.setdefault(s, []).append((i, kind, arg))
    done, order, pos = set(), [], {s: 0 for s in streams}
    progress = True
    while progress:
        progress = False
        for s, q in streams.items():
            while pos[s] < len(q):
                i, kind, arg = q[pos[s]]
                if kind == "wait" and arg[1] is not None and arg[1] not in done:
                    break
                if kind == "wait_stream":
                    other = streams.get(arg, [])
                    if any(j < i and j not in done for j, _, _ in other):
                        break
                done.add(i)
                if kind in ("copy_in", "compute", "copy_out"):
                    order.append((kind, arg))
                pos[s] += 1
                progress = True
    assert all(pos[s] == len(q) for s, q in streams.items()), "deadlock in the replay"
    return order


def test_pipelined_e2e_respects_buffer_reuse():
    bench = _bench()
    log = _Log()
    fake, Stream = _fake_torch(log)
    main = Stream(name="cmp")
    n, nb = 6, 2

    def work(kind):
        def f(k):
            log.ops.append((log.current.name, kind, (k, len([o for o in log.ops if o[1] == kind]))))
        return f

    bench.pipelined_e2e(fake, n, nb, work("copy_in"), work("compute"), work("copy_out"), main)
    kinds = [o for o in log.ops if o[1] in ("copy_in", "compute", "copy_out")]
    assert [o[0] for o in kinds if o[1] == "copy_in"] == ["in"] * n
    assert [o[0] for o in kinds if o[1] == "compute"] == ["cmp"] * n
    assert [o[0] for o in kinds if o[1] == "copy_out"] == ["out"] * n
    order = _simulate(log.ops)
    pos = {item: i for i, item in enumerate(order)}
    for step in range(n):
        k = step % nb
        cin, cmp, cout = ("copy_in", (k, step)), ("compute", (k, step)), ("copy_out", (k, step))
        assert pos[cin] < pos[cmp] < pos[cout]
        if step >= nb:
            # the buffer set is refilled only after the step that used it read it,
            # and overwritten by compute only after its result was copied out
            assert pos[("compute", (k, step - nb))] < pos[cin]
            assert pos[("copy_out", (k, step - nb))] < pos[cmp]
    # the end of the run waits for both copy streams
    assert log.ops[-2:] == [("cmp", "wait_stream", "in"), ("cmp", "wait_stream", "out")]


def test_traffic_lookup_follows_source_hash(tmp_path, monkeypatch):
    bench = _bench()
    csrc = tmp_path / "hstu_sequential_transduction_jagged_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cuh"
    src.write_text("kernel v1\n")
    import hashlib
    h = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles" / "k_traffic.txt").write_text(
        f"# comment\nsource = k.cuh\nsource_sha256_16 = {h}\ndram_bytes_per_launch = 1234\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profiles("k") == 1234.0
    src.write_text("kernel v2\n")
    assert bench.traffic_from_profiles("k") is None


def test_visible_pair_count_matches_the_mask():
    """bench.py's algorithmic pair count for masked workloads equals the number
    of visible (query, key) pairs of the oracle's mask."""
    import numpy as np
    from gen import make_case
    from oracle import hstu as O
    bench = _bench()
    case = make_case("small-bf16", seed=3, lengths=[300, 77, 129])
    assert bench.visible_pairs(case) == sum(n * (n + 1) // 2 for n in (300, 77, 129))
    segs = np.array([[40, 200], [0, 77], [129, 0]], dtype=np.int32)
    ts = case.timestamps.copy()
    ts[240:300] = np.sort(np.random.default_rng(0).integers(ts[40], ts[239] + 1, 60))
    case.timestamps = ts
    case.extra["segments"] = segs
    want = sum(int(O.segment_mask(ts[case.offsets[u]:case.offsets[u + 1]], a, b).sum())
               for u, (a, b) in enumerate(segs))
    got = bench.visible_pairs(case)
    assert isinstance(got, int) and got == want
