"""Pins for the oracle's expert-cache simulator.

* hand-worked event sequences (tests/golden/cache_traces.txt);
* a second simulator written here with a different data structure (a lazy
  min-heap keyed by (count, last use, id) instead of a linear scan) must give
  the identical event sequence on long random traces;
* Belady's farthest-in-future policy on the flattened trace is optimal for
  demand paging, so no policy can miss less: it bounds the oracle from below;
* a cache at least as large as the number of distinct ids only takes
  compulsory misses.
"""
import heapq
from pathlib import Path

import numpy as np
import pytest

import workloads as W

GOLDEN = Path(__file__).parent / "golden"


def _golden_traces():
    traces, cur = [], None
    for line in (GOLDEN / "cache_traces.txt").read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        f = line.split()
        if f[0] == "trace":
            cur = dict(name=f[1], experts=int(f[2]), cap=int(f[3]), decay=int(f[4]), n=int(f[5]),
                       ids=[], ev=[])
        elif f[0] == "ids":
            cur["ids"].append([int(v) for v in f[2:]])
        elif f[0] == "ev":
            cur["ev"].append(tuple(int(v) for v in f[1:]))
        elif f[0] == "end":
            traces.append(cur)
    return traces


@pytest.mark.parametrize("tr", _golden_traces(), ids=lambda t: t["name"])
def test_cache_hand_worked(oracle_lib, tr):
    ids = np.array(tr["ids"], np.int32)
    r = oracle_lib.cache_sim(ids, tr["experts"], tr["cap"], tr["decay"])
    got = []
    for s in range(ids.shape[0]):
        for j in range(ids.shape[1]):
            got.append((s, j, int(ids[s, j]), int(r["hit"][s, j]), int(r["slot"][s, j]), int(r["victim"][s, j])))
    assert got == tr["ev"]


def heap_sim(ids, n_experts, capacity, decay):
    """Independent re-implementation with a lazily invalidated heap."""
    steps, n = ids.shape
    slot_of, expert_in = {}, [None] * capacity
    free = list(range(capacity))
    heapq.heapify(free)
    cnt = [0] * n_experts
    last = [-1] * n_experts
    heap = []                       # (cnt, last, id, version)
    ver = [0] * n_experts
    out = []

    def push(e):
        ver[e] += 1
        heapq.heappush(heap, (cnt[e], last[e], e, ver[e]))

    for s in range(steps):
        if decay > 0 and s > 0 and s % decay == 0:
            cnt = [c // 2 for c in cnt]
            heap = []
            for e in slot_of:
                push(e)
        step = set(int(v) for v in ids[s])
        for j in range(n):
            e = int(ids[s, j])
            cnt[e] += 1
            last[e] = s
            if e in slot_of:
                out.append((1, slot_of[e], -1))
                push(e)
                continue
            if free:
                sl = heapq.heappop(free)
                victim = -1
            else:
                skipped = []
                while True:
                    c, l, v, vv = heapq.heappop(heap)
                    if v not in slot_of or vv != ver[v]:
                        continue
                    if v in step:
                        skipped.append((c, l, v, vv))
                        continue
                    break
                for it in skipped:
                    heapq.heappush(heap, it)
                victim = v
                sl = slot_of.pop(v)
            slot_of[e] = sl
            expert_in[sl] = e
            push(e)
            out.append((0, sl, victim))
    return out


@pytest.mark.parametrize("seed,E,cap,decay,n,steps", [
    (1, 64, 8, 16, 4, 400), (2, 300, 40, 64, 10, 600), (3, 24576, 2048, 256, 10, 300),
    (4, 50, 10, 0, 10, 200), (5, 500, 64, 7, 10, 500)])
def test_cache_matches_independent_simulator(oracle_lib, seed, E, cap, decay, n, steps):
    gen = W.paging_trace(seed, E, n, steps, drift_every=50, hot=min(cap, E // 2))
    ids = np.stack([np.argsort(-l, kind="stable")[:n] for l in gen]).astype(np.int32)
    r = oracle_lib.cache_sim(ids, E, cap, decay)
    ref = heap_sim(ids, E, cap, decay)
    got = [(int(r["hit"][s, j]), int(r["slot"][s, j]), int(r["victim"][s, j]))
           for s in range(steps) for j in range(n)]
    assert got == ref
    assert r["misses"] == sum(1 for h, _, _ in ref if h == 0)


def belady_misses(seq, capacity):
    nxt = {}
    future = [0] * len(seq)
    for i in range(len(seq) - 1, -1, -1):
        future[i] = nxt.get(seq[i], 1 << 60)
        nxt[seq[i]] = i
    cache, misses = {}, 0
    for i, e in enumerate(seq):
        if e in cache:
            cache[e] = future[i]
            continue
        misses += 1
        if len(cache) >= capacity:
            v = max(cache, key=lambda c: cache[c])
            del cache[v]
        cache[e] = future[i]
    return misses


@pytest.mark.parametrize("seed,cap", [(11, 6), (12, 12), (13, 30)])
def test_cache_not_below_belady(oracle_lib, seed, cap):
    gen = W.paging_trace(seed, 80, 4, 300, drift_every=40, hot=20)
    ids = np.stack([np.argsort(-l, kind="stable")[:4] for l in gen]).astype(np.int32)
    r = oracle_lib.cache_sim(ids, 80, cap, 32)
    assert r["misses"] >= belady_misses(ids.ravel().tolist(), cap)


def test_cache_large_enough_only_compulsory(oracle_lib):
    rng = np.random.default_rng(4)
    ids = np.stack([rng.choice(40, 5, replace=False) for _ in range(200)]).astype(np.int32)
    r = oracle_lib.cache_sim(ids, 40, 40, 8)
    assert r["misses"] == len(np.unique(ids))
    assert np.all(r["victim"] == -1)


def test_cache_rejects_bad_trace(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.cache_sim(np.array([[1, 1]], np.int32), 4, 2, 0)   # repeated id
    with pytest.raises(ValueError):
        oracle_lib.cache_sim(np.array([[1, 2, 3]], np.int32), 4, 2, 0)  # n > capacity
    with pytest.raises(ValueError):
        oracle_lib.cache_sim(np.array([[7]], np.int32), 4, 2, 0)      # id out of range


# ------------------------------------------------------------ with prefetch
def _prefetch_golden():
    rows, out = [], {}
    for line in (GOLDEN / "cache_prefetch_trace.txt").read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("stage"):
            head, rest = line.split(":", 1)
            stage, pf = rest.split("|")
            e, hit, slot, victim = (int(v) for v in stage.split())
            pfi, pfo = pf.split("->")
            pfs, pfv = pfo.split(";")
            rows.append(dict(id=e, hit=hit, slot=slot, victim=victim, pf=[int(v) for v in pfi.split()],
                             pf_slot=[int(v) for v in pfs.split()], pf_victim=[int(v) for v in pfv.split()]))
        else:
            f = line.split()
            out[f[0]] = [int(v) for v in f[1:]]
    return rows, out


def test_prefetch_sim_hand_worked_trace(oracle_lib):
    rows, out = _prefetch_golden()
    ids = np.array([[r["id"]] for r in rows], np.int32)
    pf = np.array([r["pf"] for r in rows], np.int32)
    got = oracle_lib.cache_sim_prefetch(ids, pf, 6, 3, 0)
    assert got["hit"][:, 0].astype(int).tolist() == [r["hit"] for r in rows]
    assert got["slot"][:, 0].tolist() == [r["slot"] for r in rows]
    assert got["victim"][:, 0].tolist() == [r["victim"] for r in rows]
    assert got["pf_slot"].tolist() == [r["pf_slot"] for r in rows]
    assert got["pf_victim"].tolist() == [r["pf_victim"] for r in rows]
    assert got["misses"] == out["misses"][0] and got["prefetched"] == out["prefetched"][0]
    assert got["counts"].tolist() == out["counts"]


def test_prefetch_sim_without_prefetch_is_the_plain_policy(oracle_lib):
    rng = np.random.default_rng(21)
    for E, cap, decay, n in ((40, 10, 8, 4), (300, 32, 16, 10)):
        ids = np.stack([rng.choice(E, n, replace=False) for _ in range(400)]).astype(np.int32)
        a = oracle_lib.cache_sim(ids, E, cap, decay)
        b = oracle_lib.cache_sim_prefetch(ids, np.full((400, 3), -1, np.int32), E, cap, decay)
        for key in ("slot", "hit", "victim", "counts"):
            assert np.array_equal(a[key], b[key]), key
        assert a["misses"] == b["misses"] and b["prefetched"] == 0


def _prefetch_sim_sorted(ids, pf, E, cap, decay):
    """Independent restatement: the resident set as a dict, victims picked by
    sorting the unprotected residents on (count, last use, id)."""
    slot_of, free, cnt, last = {}, list(range(cap)), [0] * E, [-1] * E
    ev, pev, misses = [], [], 0
    for s in range(ids.shape[0]):
        if decay and s and s % decay == 0:
            cnt = [c // 2 for c in cnt]
        step = [int(v) for v in ids[s]]
        prot = set(step)

        def place(e):
            if free:
                free.sort()
                return free.pop(0), -1
            cand = sorted((cnt[c], last[c], c) for c in slot_of if c not in prot)
            if not cand:
                return None, -1
            v = cand[0][2]
            return slot_of.pop(v), v
        for e in step:
            cnt[e] += 1
            last[e] = s
            if e in slot_of:
                ev.append((1, slot_of[e], -1))
                continue
            misses += 1
            sl, v = place(e)
            slot_of[e] = sl
            ev.append((0, sl, v))
        prot |= {int(v) for v in pf[s] if v >= 0}
        for e in (int(v) for v in pf[s]):
            if e < 0 or e in slot_of:
                pev.append((-1, -1))
                continue
            sl, v = place(e)
            if sl is None:
                pev.append((-1, -1))
                continue
            slot_of[e] = sl
            pev.append((sl, v))
    return ev, pev, misses, cnt


def test_prefetch_sim_matches_an_independent_simulator(oracle_lib):
    rng = np.random.default_rng(22)
    E, cap, decay, n, npf, steps = 60, 12, 16, 4, 3, 300
    ids = np.stack([rng.choice(E, n, replace=False) for _ in range(steps)]).astype(np.int32)
    pf = rng.integers(-1, E, size=(steps, npf)).astype(np.int32)
    got = oracle_lib.cache_sim_prefetch(ids, pf, E, cap, decay)
    ev, pev, misses, cnt = _prefetch_sim_sorted(ids, pf, E, cap, decay)
    assert [tuple(v) for v in zip(got["hit"].ravel().astype(int), got["slot"].ravel(), got["victim"].ravel())] == ev
    assert list(zip(got["pf_slot"].ravel().tolist(), got["pf_victim"].ravel().tolist())) == pev
    assert got["misses"] == misses and got["counts"].tolist() == cnt


def test_prefetching_the_next_step_leaves_only_the_first_misses(oracle_lib):
    """A prefetch of exactly the next step's ids (room for both steps) turns
    every later access into a hit."""
    rng = np.random.default_rng(23)
    E, cap, n, steps = 200, 24, 8, 100
    ids = np.stack([rng.choice(E, n, replace=False) for _ in range(steps)]).astype(np.int32)
    pf = np.vstack([ids[1:], np.full((1, n), -1, np.int32)])
    got = oracle_lib.cache_sim_prefetch(ids, pf, E, cap, 0)
    assert got["misses"] == n and got["hit"][1:].all()


def _admit_golden():
    rows, out = [], {}
    for line in (GOLDEN / "cache_admit_trace.txt").read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("step"):
            ev = [[int(v) for v in part.split()] for part in line.split(":", 1)[1].split(";")]
            rows.append(ev)
        else:
            f = line.split()
            out[f[0]] = [int(v) for v in f[1:]]
    return rows, out


def test_admit_sim_hand_worked_trace(oracle_lib):
    rows, out = _admit_golden()
    ids = np.array([[ev[0] for ev in r] for r in rows], np.int32)
    got = oracle_lib.cache_sim_admit(ids, 5, 2, 0, 2)
    assert got["hit"].astype(int).tolist() == [[ev[1] for ev in r] for r in rows]
    assert got["slot"].tolist() == [[ev[2] for ev in r] for r in rows]
    assert got["victim"].tolist() == [[ev[3] for ev in r] for r in rows]
    assert got["misses"] == out["misses"][0] and got["in_place"] == out["in_place"][0]
    assert got["counts"].tolist() == out["counts"]


@pytest.mark.parametrize("admit_min", [0, 1])
def test_admit_sim_without_threshold_is_the_base_policy(oracle_lib, admit_min):
    rng = np.random.default_rng(77 + admit_min)
    ids = np.stack([rng.choice(40, 4, replace=False) for _ in range(300)]).astype(np.int32)
    a = oracle_lib.cache_sim_admit(ids, 40, 9, 16, admit_min)
    b = oracle_lib.cache_sim(ids, 40, 9, 16)
    assert np.array_equal(a["slot"], b["slot"]) and np.array_equal(a["victim"], b["victim"])
    assert np.array_equal(a["hit"].astype(bool), b["hit"]) and a["misses"] == b["misses"] and a["in_place"] == 0
    assert np.array_equal(a["counts"], b["counts"])


def test_admit_sim_invariants(oracle_lib):
    """A threshold no counter reaches admits nothing.  With a cache as large
    as the pool and no decay (nothing is ever evicted), each expert is
    computed in place for its first admit_min - 1 uses, enters at use
    admit_min and hits afterwards."""
    rng = np.random.default_rng(5)
    ids = np.stack([rng.choice(30, 3, replace=False) for _ in range(200)]).astype(np.int32)
    never = oracle_lib.cache_sim_admit(ids, 30, 6, 0, 10 ** 6)
    assert (never["hit"] == 3).all() and (never["slot"] == -1).all() and (never["victim"] == -1).all()
    assert never["misses"] == ids.size == never["in_place"]
    big = oracle_lib.cache_sim_admit(ids, 30, 30, 0, 3)
    uses = np.zeros(30, int)
    for s in range(ids.shape[0]):
        for j in range(ids.shape[1]):
            e = ids[s, j]
            uses[e] += 1
            want = 3 if uses[e] < 3 else (0 if uses[e] == 3 else 1)
            assert big["hit"][s, j] == want, (s, j, e, uses[e])
    assert (big["victim"] == -1).all()
