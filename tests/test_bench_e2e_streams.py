"""bench.py's end-to-end loop, on a machine without a GPU: its copies in, fused
linears and copies out run on three streams ordered by events.  Here every stream
is a queue of operations and every event wait an edge; the operations run in random
orders that respect those edges, on real (small) data, and every pair of accesses to
one buffer, at least one a write, must be ordered.  A loop with any one of its waits
removed must be caught."""
import itertools
import os
import random
import sys
import types

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

OPS = []          # dict(stream, deps, fn, reads, writes, done)


class Buf:
    ids = itertools.count()

    def __init__(self, data, dev):
        self.data, self.dev, self.id = data, dev, next(Buf.ids)


class T:
    """Fake tensor: a buffer plus a dtype tag."""

    def __init__(self, buf, dtype=None):
        self.buf, self.dtype = buf, dtype

    shape = property(lambda s: s.buf.data.shape)

    def pin_memory(self):
        return self

    def view(self, dtype):
        return T(self.buf, dtype)

    def clone(self):
        assert not self.buf.dev
        return T(Buf(self.buf.data.copy(), False), self.dtype)

    def copy_(self, src, non_blocking=False):
        dst = self

        def f():
            dst.buf.data[...] = src.buf.data
        CUR[0].enqueue(f, [src.buf], [dst.buf])
        return self


class Stream:
    ids = itertools.count()

    def __init__(self):
        self.id, self.last, self.pending = next(Stream.ids), None, set()

    def enqueue(self, fn, reads, writes):
        deps = set(self.pending)
        if self.last is not None:
            deps.add(self.last)
        self.pending = set()
        OPS.append(dict(stream=self.id, deps=deps, fn=fn, reads=reads, writes=writes, done=False))
        self.last = len(OPS) - 1
        return self.last

    def wait_event(self, ev):
        if ev.op is not None:
            self.pending.add(ev.op)


class Event:
    def __init__(self, enable_timing=False):
        self.op = None

    def record(self, stream=None):
        self.op = (stream or CUR[0]).enqueue(lambda: None, [], [])

    def elapsed_time(self, other):
        return 1.0


MAIN = Stream()
CUR = [MAIN]


class _StreamCtx:
    def __init__(self, s):
        self.s = s

    def __enter__(self):
        self.prev = CUR[0]
        CUR[0] = self.s

    def __exit__(self, *a):
        CUR[0] = self.prev


def synchronize():
    pend = [i for i, o in enumerate(OPS) if not o["done"]]
    while pend:
        ready = [i for i in pend if all(OPS[d]["done"] for d in OPS[i]["deps"])]
        assert ready, "deadlock"
        i = RNG.choice(ready)
        OPS[i]["fn"]()
        OPS[i]["done"] = True
        pend.remove(i)


def race_check():
    n = len(OPS)
    anc = [set() for _ in range(n)]
    for i, o in enumerate(OPS):
        for d in o["deps"]:
            anc[i] |= anc[d] | {d}
    acc = {}
    for i, o in enumerate(OPS):
        for b in o["reads"]:
            acc.setdefault(b.id, []).append((i, "r"))
        for b in o["writes"]:
            acc.setdefault(b.id, []).append((i, "w"))
    races = 0
    for b, lst in acc.items():
        for (i, ki), (j, kj) in itertools.combinations(lst, 2):
            if i == j or (ki == "r" and kj == "r"):
                continue
            if i not in anc[j] and j not in anc[i]:
                races += 1
    return races


cuda = types.SimpleNamespace(
    current_stream=lambda: CUR[0], Stream=Stream, Event=Event, stream=_StreamCtx,
    synchronize=synchronize)
fake_torch = types.SimpleNamespace(
    cuda=cuda, int16="int16", bfloat16="bf16",
    from_numpy=lambda a: T(Buf(a.copy(), False)),
    empty=lambda shape, dtype=None: T(Buf(np.zeros(shape, np.int64), False), dtype),
    empty_like=lambda t: T(Buf(np.zeros_like(t.buf.data), True), t.dtype),
    equal=lambda a, b: np.array_equal(a.buf.data, b.buf.data))


def linear_fn(x, cinv, sid, alpha, beta, t, qw, s_w, bias, y, ws, stream=None):
    def f():
        ws.buf.data[...] = x.buf.data[:, :1] * 3 + t       # the workspace is scratch
        y.buf.data[...] = x.buf.data[:, : y.buf.data.shape[1]] * 7 + ws.buf.data[:, :1] + t
    CUR[0].enqueue(f, [x.buf, ws.buf], [y.buf, ws.buf])


fake_wq = types.SimpleNamespace(wq_linear_w4a8=linear_fn, wq_linear_w4a4=linear_fn)


class Layer:
    def __init__(self, j, M, K, N, n_sets, T_):
        g = np.random.default_rng(j)
        self.M, self.K, self.N, self.T, self.bits = M, K, N, T_, 8
        self.host_x = [g.integers(0, 1000, (M, K)).astype(np.uint16) for _ in range(n_sets)]
        self.x = [T(Buf(np.zeros((M, K), np.int64), True)) for _ in range(n_sets)]
        self.y = T(Buf(np.zeros((M, N), np.int64), True))
        self.ws = T(Buf(np.zeros((M, 1), np.int64), True))
        self.cinv = self.sid = self.alpha = self.beta = self.qw = self.s_w = self.bias = None

    def ops(self):
        return 2 * self.M * self.N * self.K


RNG = random.Random(0)


def run(seed, steps, n_sets, T_, module=bench):
    global RNG
    RNG = random.Random(seed)
    OPS.clear()
    MAIN.last, MAIN.pending, CUR[0] = None, set(), MAIN
    layers = [Layer(j, 6, 8, 4, n_sets, T_) for j in range(4)]
    args = types.SimpleNamespace(e2e_steps=steps)
    out = module.run_e2e(args, layers, fake_wq, fake_torch, 1)
    races = race_check()
    return out, races


@pytest.mark.parametrize("steps,n_sets,T_", [(10, 2, 1), (7, 3, 10), (1, 2, 3), (2, 2, 2)])
def test_overlapped_loop_is_race_free_and_matches_serial(steps, n_sets, T_):
    for seed in range(8):
        out, races = run(seed, steps, n_sets, T_)
        assert races == 0
        assert out["overlapped_equals_serial"] and out["loop"].startswith("overlapped")


WAITS = ["            s_in.wait_event(x_read[j][r])\n",
         "            main.wait_event(x_in[j])\n",
         "            main.wait_event(y_sent[j][b])\n",
         "            s_out.wait_event(y_out[j])\n"]


@pytest.mark.parametrize("line", WAITS, ids=["x-set-free", "copied-in", "output-sent",
                                             "output-made"])
def test_a_missing_wait_is_caught(line):
    with open(os.path.join(ROOT, "bench.py")) as f:
        src = f.read()
    assert src.count(line) == 1
    mod = types.ModuleType("bench_without_one_wait")
    mod.__file__ = os.path.join(ROOT, "bench.py")
    exec(compile(src.replace(line, ""), "bench_without_one_wait", "exec"), mod.__dict__)
    caught = 0
    for seed in range(6):
        out, races = run(seed, 10, 2, 3, module=mod)
        caught += bool(races) or not out["overlapped_equals_serial"]
    assert caught == 6
