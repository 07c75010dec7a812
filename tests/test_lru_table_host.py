"""The expert cache's table code (csrc/lru_table.cuh), built for the host, against
the oracle's cache simulation (oracle/lru.py) over long random traces. CPU only.

The device runs these same functions from one thread; here g++ builds them into
a small library (tests/lru_table_host.cpp), and every call of a random sequence
of layer resolves (each followed by the prefetch of the next layer's prediction,
as the layer forward does), explicit prefetches and evictions must give the same
loads, the same CACHE_FULL outcomes, the same hit and miss counts and the same
table as the simulation. The two implementations share nothing: the table keeps
an intrusive recency list and a free bitmap, the simulation integer stamps and
linear scans."""
import ctypes as C
import os
import subprocess

import numpy as np
import pytest

from conftest import ROOT
from oracle.lru import CacheFull, LruSim

_SRC = [os.path.join(ROOT, "tests", "lru_table_host.cpp"),
        os.path.join(ROOT, "expert_ffn_layer_top_b200", "csrc", "lru_table.cuh"),
        os.path.join(ROOT, "include", "moe.h")]
_SO = os.path.join(ROOT, "_build", "lru_table_host.so")
CACHE_FULL = 6


@pytest.fixture(scope="module")
def lib():
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    if not os.path.exists(_SO) or any(os.path.getmtime(s) > os.path.getmtime(_SO) for s in _SRC):
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-Wall", "-shared", "-fPIC", _SRC[0], "-o", tmp])
        os.replace(tmp, _SO)
    L = C.CDLL(_SO)
    P, I = C.c_void_p, C.c_int
    L.lru_host_create.restype = P
    L.lru_host_create.argtypes = [I, I, I, I]
    L.lru_host_destroy.argtypes = [P]
    L.lru_host_resolve.argtypes = [P, I, P, I, I, I, P]
    L.lru_host_prefetch.argtypes = [P, I, P, I, P]
    L.lru_host_resize.restype = I
    L.lru_host_resize.argtypes = [P, I, P]
    L.lru_host_plan.restype = I
    L.lru_host_plan.argtypes = [I, I, I, I, I, C.c_double, C.c_double, C.c_double, P]
    L.lru_host_evict.argtypes = [P, I, P, I]
    L.lru_host_slot_of.restype = I
    L.lru_host_slot_of.argtypes = [P, I, I]
    L.lru_host_counts.argtypes = [P, P]
    return L


class Table:
    def __init__(self, lib, S, L, E, Smax=None):
        self.lib, self.L, self.E = lib, L, E
        self.Smax = Smax or S
        self.h = lib.lru_host_create(S, L, E, self.Smax)
        self.io = np.zeros(3 + 4 * E, np.int32)

    def _pairs(self, start, n):
        return [(int(self.io[start + 2 * i]), int(self.io[start + 2 * i + 1])) for i in range(n)]

    def resolve(self, layer, idx, prefetch_next=True, pf_mode=None, depth=-1):
        a = np.ascontiguousarray(idx, np.int32)
        mode = (1 if prefetch_next else 0) if pf_mode is None else pf_mode
        self.lib.lru_host_resolve(self.h, layer, a.ctypes.data, len(a), mode, depth, self.io.ctypes.data)
        if self.io[0] == CACHE_FULL:
            return None, None
        na, nb = int(self.io[1]), int(self.io[2])
        return self._pairs(3, na), (None if nb < 0 else self._pairs(3 + 2 * na, nb))

    def prefetch(self, layer, ids):
        a = np.ascontiguousarray(ids, np.int32)
        self.lib.lru_host_prefetch(self.h, layer, a.ctypes.data, len(a), self.io.ctypes.data)
        return None if self.io[0] == CACHE_FULL else self._pairs(3, int(self.io[1]))

    def resize(self, S_new):
        moves = np.zeros(2 * S_new + 2, np.int32)
        n = self.lib.lru_host_resize(self.h, S_new, moves.ctypes.data)
        assert n >= 0
        return [(int(moves[2 * i]), int(moves[2 * i + 1])) for i in range(n)]

    def evict(self, layer, ids):
        a = np.ascontiguousarray(ids if ids is not None else [], np.int32)
        self.lib.lru_host_evict(self.h, layer, a.ctypes.data, -1 if ids is None else len(a))

    def table(self):
        return [self.lib.lru_host_slot_of(self.h, l, e) for l in range(self.L) for e in range(self.E)]

    def counts(self):
        out = np.zeros(2, np.uint64)
        self.lib.lru_host_counts(self.h, out.ctypes.data)
        return int(out[0]), int(out[1])

    def close(self):
        self.lib.lru_host_destroy(self.h)


def _run_trace(lib, seed, n_ops, policies=False, resizes=False):
    """A random trace. With ``policies`` each resolve's next-layer prefetch is one of:
    none, the whole prediction, the first d of it by pair count, or the whole layer.
    With ``resizes`` the pool is resized now and then, up and down."""
    g = np.random.default_rng(seed)
    # small pools (frequent eviction, CACHE_FULL) and pools over several free-bitmap words
    S = int(g.integers(2, 25)) if seed % 3 else int(g.integers(33, 97))
    L = int(g.integers(1, 5))
    E = int(g.choice([5, 8, 33, 64, 100]))
    Smax = 2 * S + 40 if resizes else S
    dev, sim = Table(lib, S, L, E, Smax), LruSim(S, L, E, 1)
    full = 0
    for op in range(n_ops):
        r = g.random()
        layer = int(g.integers(0, L))
        if resizes and r > 0.93:
            S_new = int(g.integers(1, Smax + 1))
            assert dev.resize(S_new) == sim.resize(S_new), (seed, op, "resize")
        elif r < 0.7:
            k = int(g.integers(1, min(E, 8) + 1))
            T = int(g.integers(1, 6))
            # Zipf-skewed expert popularity, so that hits, misses and evictions all occur
            pop = g.zipf(1.3, size=(T, k)) % E
            pf_mode, depth = 1, -1
            if policies:
                pf_mode = int(g.integers(0, 3))
                depth = int(g.integers(-1, 6)) if pf_mode == 1 else -1
            got, got_next = dev.resolve(layer, pop.ravel(), pf_mode=pf_mode, depth=depth)
            try:
                want = sim.resolve(layer, pop.ravel())
            except CacheFull:
                want = None
            assert got == want, (seed, op, "resolve")
            if want is None:
                full += 1
            else:
                if layer + 1 < L and pf_mode != 0:
                    try:
                        want_next = sim.prefetch(layer + 1, sim.predict(layer + 1, depth, pf_mode == 2))
                    except CacheFull:
                        want_next = None
                    assert got_next == want_next, (seed, op, "prediction")
                else:
                    assert got_next is None
        elif r < 0.85:
            ids = [int(e) for e in g.choice(E, int(g.integers(1, min(E, 6) + 1)), replace=False)]
            got = dev.prefetch(layer, ids)
            try:
                want = sim.prefetch(layer, ids)
            except CacheFull:
                want = None
            assert got == want, (seed, op, "prefetch")
        else:
            kind = g.integers(0, 3)
            if kind == 0:
                dev.evict(-1, None)
                sim.evict()
            elif kind == 1:
                dev.evict(layer, None)
                sim.evict(layer)
            else:
                ids = [int(e) for e in g.choice(E, int(g.integers(0, 4)), replace=False)]
                dev.evict(layer, ids)
                sim.evict(layer, ids)
        assert dev.counts() == (sim.hits, sim.misses), (seed, op, "counts")
        assert dev.table() == sim.table(), (seed, op, "table")
    dev.close()
    return sim, full


@pytest.mark.parametrize("block", range(4))
def test_device_table_code_matches_the_simulation_on_random_traces(lib, block):
    totals = np.zeros(4, np.int64)
    for seed in range(block * 50, block * 50 + 50):
        sim, full = _run_trace(lib, seed, 150)
        totals += (sim.hits, sim.misses, sim.loads, full)
    hits, misses, loads, full = totals
    # the traces exercise every branch: hits, misses, loads beyond the misses (prefetches), CACHE_FULL
    assert hits > 0 and misses > 0 and loads > misses and full > 0


@pytest.mark.parametrize("block", range(2))
def test_prefetch_depths_full_layers_and_resizes_match_the_simulation(lib, block):
    """Next-layer prefetch of none / the whole prediction / its first d experts by pair
    count / the whole layer, and pool resizes up and down, on random traces: loads, moves,
    counts and the table agree with the simulation after every call."""
    moves = 0
    for seed in range(1000 + block * 60, 1000 + block * 60 + 60):
        sim, _ = _run_trace(lib, seed, 150, policies=True, resizes=True)
        moves += sim.moves
    assert moves > 0


def test_prefetch_plan(lib):
    """The per-call decision: fixed policies pass through; the adaptive one streams the
    whole next layer when the call is expected to reach half of the experts, else the
    number of experts the measured rate moves during the measured compute time."""
    flags = np.zeros(2, np.int32)

    def plan(policy, depth, T, k, E, bw=0.0, t=0.0, eb=1.0):
        d = lib.lru_host_plan(policy, depth, T, k, E, bw, t, eb, flags.ctypes.data)
        return d, bool(flags[0]), bool(flags[1])

    NONE, PRED, FULL, ADAPT = 0, 1, 2, 3
    assert plan(NONE, 5, 4, 8, 128) == (0, False, True)
    assert plan(PRED, -1, 4, 8, 128) == (-1, False, False)
    assert plan(PRED, 7, 4, 8, 128) == (7, False, False)
    assert plan(FULL, -1, 4, 8, 128) == (128, True, False)
    # prefill-sized: 4096 tokens x top-8 of 128 reach every expert
    assert plan(ADAPT, -1, 4096, 8, 128) == (128, True, False)
    # T = 8 with top-8 of 128: 1 - (120/128)^8 = 40% of the experts: depth from the rates
    assert plan(ADAPT, -1, 8, 8, 128) == (-1, False, False)              # nothing measured yet
    assert plan(ADAPT, -1, 8, 8, 128, bw=50e9, t=1e-3, eb=5e6) == (10, False, False)
    assert plan(ADAPT, -1, 8, 8, 128, bw=50e9, t=1.0, eb=5e6) == (128, False, False)
    # T = 11: 1 - (120/128)^11 = 50.8% >= half
    assert plan(ADAPT, -1, 11, 8, 128)[1] is True
    assert plan(ADAPT, -1, 10, 8, 128)[1] is False


def test_hand_worked_trace_through_the_table_code(lib, golden_dir):
    """The hand-worked trace of tests/golden/lru_trace.txt, replayed on the table code."""
    dev = Table(lib, 3, 2, 4)
    for line in open(os.path.join(golden_dir, "lru_trace.txt")):
        if line.startswith("#") or not line.strip():
            continue
        lhs, rhs = line.split("->")
        op, layer, ids = lhs.split()
        ids = [int(i) for i in ids.split(",")]
        before = dev.table()
        got = dev.resolve(int(layer), ids, False)[0] if op == "resolve" else dev.prefetch(int(layer), ids)
        if rhs.strip() == "FULL":
            assert got is None and dev.table() == before
            continue
        loads_s, counts = rhs.split("|")
        assert got == [tuple(int(v) for v in p.split(":")) for p in loads_s.split()]
        assert dev.counts() == tuple(int(v) for v in counts.split())
    dev.close()
