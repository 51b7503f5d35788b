"""The static schedule validator (libamk, C++) against the brute-force
interleaving checker (oracle/interleave.py) on tiny adversarial schedules.

x-techcon AutoMegaKernel article, section 1: adversarial schedules, unsafe
ones confirmed by an independent oracle, zero false accepts.  Here every
random schedule must get the same accept/reject verdict from both, and the
same class of reason (deadlock <-> V1/V4, race <-> V5/V6, syntax rules
equal).  The pages' own 7160-schedule corpus is not available; the counts of
this corpus are reported by test_corpus_counts.
"""
import random

import pytest

import persistent_megakernel_decode_cta_b200 as amk
from persistent_megakernel_decode_cta_b200 import build
from oracle import interleave as bf

R, W, A, RP, RS, RF = bf.READ, bf.WRITE, bf.ACCUM, bf.READ_PREV, bf.RESET, bf.READ_FLAGGED


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def _same_class(v_rule, b_reason):
    if b_reason == "deadlock":
        return v_rule in ("V1", "V4")
    if b_reason == "race":
        return v_rule in ("V5", "V6")
    return v_rule == b_reason


def agree(g):
    ok_v, rule, msg = amk.validate_graph(g)
    ok_b, reason = bf.check(g)
    assert ok_v == ok_b, (rule, reason, msg, g)
    if not ok_v:
        assert _same_class(rule, reason), (rule, reason, msg, g)
    return ok_v, (rule if not ok_v else "ok")


# ---- random schedule generator ------------------------------------------------

def random_schedule(rng: random.Random):
    """A mostly valid random schedule: a random DAG, counters (some shared),
    queues in a topological order, accesses consistent with happens-before."""
    T = rng.randint(1, 9)
    S = rng.randint(1, 3)
    preds = [[j for j in range(i) if rng.random() < 0.35] for i in range(T)]
    counters = []            # list of producer-task lists
    waits = [[] for _ in range(T)]
    signals = [[] for _ in range(T)]
    own = {}
    for i in range(T):
        if len(preds[i]) >= 2 and rng.random() < 0.4:
            c = len(counters)          # one shared counter for all predecessors
            counters.append(list(preds[i]))
            for j in preds[i]:
                signals[j].append(c)
            waits[i].append((c, len(preds[i])))
        else:
            for j in preds[i]:
                if j not in own:
                    own[j] = len(counters)
                    counters.append([j])
                    signals[j].append(own[j])
                waits[i].append((own[j], 1))
    # queues: a topological order split across SMs
    order = list(range(T))
    sm_of = [rng.randrange(S) for _ in range(T)]
    queues = [[t for t in order if sm_of[t] == s] for s in range(S)]
    # happens-before (ancestor sets) of this DAG + queue order
    anc = [set() for _ in range(T)]
    for i in range(T):
        direct = set(preds[i])
        q = queues[sm_of[i]]
        k = q.index(i)
        if k > 0:
            direct.add(q[k - 1])
        for j in direct:
            anc[i] |= anc[j] | {j}
    nb = rng.randint(1, 3)
    bufs = [{"size": rng.randint(2, 6), "output": False, "pair": -1} for _ in range(nb)]
    acc = [[] for _ in range(T)]
    for b in range(nb):
        size = bufs[b]["size"]
        writer = rng.randrange(T)
        lo = rng.randrange(size)
        hi = rng.randint(lo + 1, size)
        acc[writer].append((b, W, lo, hi))
        for t in range(T):
            if writer in anc[t] and rng.random() < 0.5:
                acc[t].append((b, R, rng.randint(lo, hi - 1), hi))
            elif t != writer and rng.random() < 0.25:
                # a flagged read orders itself after the writer (a cycle or a
                # queue contradiction when t comes first: a deadlock)
                acc[t].append((b, RF, rng.randint(lo, hi - 1), hi))
    if rng.random() < 0.5:
        bufs[0]["output"] = True
    if rng.random() < 0.3:
        # a double-buffered accumulator: ACCUMs, an ordered RESET of the pair,
        # READ_PREV of the pair before the reset
        key, nxt = len(bufs), len(bufs) + 1
        bufs.append({"size": 1, "output": True, "pair": nxt})
        bufs.append({"size": 1, "output": False, "pair": -1})
        accs = rng.sample(range(T), rng.randint(1, T))
        for t in accs:
            acc[t].append((key, A, 0, 1))
        last = max(range(T), key=lambda t: len(anc[t]))
        acc[last].append((nxt, RS, 0, 1))
        for t in range(T):
            if t in anc[last] and rng.random() < 0.4:
                acc[t].append((nxt, RP, 0, 1))
    tasks = [{"sm": sm_of[t], "waits": waits[t], "signals": signals[t], "accesses": acc[t]}
             for t in range(T)]
    return {"n_counters": len(counters), "buffers": bufs, "tasks": tasks, "queues": queues}


def mutate(g, rng: random.Random):
    """One adversarial edit from the classes the pages name."""
    tasks = g["tasks"]
    T = len(tasks)
    kind = rng.randrange(12)
    t = rng.randrange(T)
    if kind == 0 and tasks[t]["waits"]:               # threshold 0 / too high
        i = rng.randrange(len(tasks[t]["waits"]))
        c, th = tasks[t]["waits"][i]
        tasks[t]["waits"][i] = (c, rng.choice([0, th + 1, th + 5]))
    elif kind == 1 and tasks[t]["waits"]:             # partial wait
        i = rng.randrange(len(tasks[t]["waits"]))
        c, th = tasks[t]["waits"][i]
        tasks[t]["waits"][i] = (c, max(1, th - 1))
    elif kind == 2 and T > 1:                         # cycle: an early task waits on a later one
        a, b = sorted(rng.sample(range(T), 2))
        c = g["n_counters"]
        g["n_counters"] += 1
        tasks[b]["signals"].append(c)
        tasks[a]["waits"].append((c, 1))
    elif kind == 3:                                   # queue order swap
        q = rng.choice(g["queues"])
        if len(q) > 1:
            i = rng.randrange(len(q) - 1)
            q[i], q[i + 1] = q[i + 1], q[i]
    elif kind == 4 and tasks[t]["waits"]:             # drop a wait (missing HB)
        tasks[t]["waits"].pop(rng.randrange(len(tasks[t]["waits"])))
    elif kind == 5:                                   # a read by an arbitrary task
        b = rng.randrange(len(g["buffers"]))
        size = g["buffers"][b]["size"]
        lo = rng.randrange(size)
        tasks[t]["accesses"].append((b, rng.choice([R, W, A, RF]), lo,
                                     rng.randint(lo + 1, size)))
    elif kind == 6:                                   # dangling references
        choice = rng.randrange(4)
        if choice == 0:
            tasks[t]["waits"].append((g["n_counters"] + 3, 1))
        elif choice == 1:
            tasks[t]["signals"].append(-1)
        elif choice == 2:
            tasks[t]["accesses"].append((len(g["buffers"]) + 1, R, 0, 1))
        else:
            b = rng.randrange(len(g["buffers"]))
            tasks[t]["accesses"].append((b, R, 0, g["buffers"][b]["size"] + 1))
    elif kind == 7:                                   # an unwritten output
        g["buffers"].append({"size": 2, "output": True, "pair": -1})
    elif kind == 8:                                   # accumulate without a reset pair covering it
        b = rng.randrange(len(g["buffers"]))
        if g["buffers"][b]["pair"] >= 0:
            tasks[t]["accesses"] = [a for a in tasks[t]["accesses"] if a[1] != RS]
        else:
            g["buffers"].append({"size": 2, "output": False, "pair": -1})
            g["buffers"][b]["pair"] = len(g["buffers"]) - 1
            tasks[t]["accesses"].append((b, A, 0, 1))
    elif kind == 9:                                   # READ_PREV / RESET out of order
        b = rng.randrange(len(g["buffers"]))
        tasks[t]["accesses"].append((b, rng.choice([RP, RS]), 0, 1))
    elif kind == 10:                                  # task placed on two queues / wrong sm
        q = rng.choice(g["queues"])
        if rng.random() < 0.5:
            q.append(t)
        else:
            tasks[t]["sm"] = (tasks[t]["sm"] + 1) % max(len(g["queues"]), 2)
    else:                                             # extra signal on a shared counter
        if g["n_counters"] > 0:
            tasks[t]["signals"].append(rng.randrange(g["n_counters"]))
    return g


def corpus(n, seed):
    rng = random.Random(seed)
    for _ in range(n):
        g = random_schedule(rng)
        for _ in range(rng.choice([0, 0, 1, 1, 2, 3])):
            g = mutate(g, rng)
        yield g


def test_validator_matches_brute_force():
    n_ok = n_bad = 0
    for g in corpus(4000, seed=7):
        ok, _ = agree(g)
        n_ok += ok
        n_bad += not ok
    assert n_ok > 400 and n_bad > 400


@pytest.mark.slow
def test_corpus_counts():
    """10^4 schedules; prints the corpus' accepted/unsafe split and checks zero
    false accepts and zero false rejects."""
    from collections import Counter
    reasons = Counter()
    for g in corpus(10000, seed=2024):
        ok, rule = agree(g)
        reasons[rule] += 1
    print("validator corpus:", dict(reasons))
    assert reasons["ok"] > 1000


# ---- hand-made cases, one per rule ------------------------------------------------

def _g(tasks, queues, n_counters, buffers=None):
    return {"n_counters": n_counters, "buffers": buffers or [], "tasks": tasks,
            "queues": queues}


def T_(sm, waits=(), signals=(), acc=()):
    return {"sm": sm, "waits": list(waits), "signals": list(signals), "accesses": list(acc)}


def test_rule_examples():
    buf = [{"size": 4, "output": False, "pair": -1}]
    # valid producer -> consumer
    assert agree(_g([T_(0, signals=[0], acc=[(0, W, 0, 4)]),
                     T_(1, waits=[(0, 1)], acc=[(0, R, 0, 4)])], [[0], [1]], 1, buf))[0]
    # V2: threshold above the producer count (deadlock)
    assert agree(_g([T_(0, signals=[0]), T_(1, waits=[(0, 2)])], [[0], [1]], 1))[1] == "V2"
    # V3: partial wait on a shared counter
    assert agree(_g([T_(0, signals=[0]), T_(1, signals=[0]), T_(2, waits=[(0, 1)])],
                    [[0], [1], [2]], 1))[1] == "V3"
    # V1: two tasks wait on each other
    assert agree(_g([T_(0, waits=[(1, 1)], signals=[0]), T_(1, waits=[(0, 1)], signals=[1])],
                    [[0], [1]], 2))[1] == "V1"
    # V4: queue order against the dependency (same SM)
    assert agree(_g([T_(0, signals=[0]), T_(0, waits=[(0, 1)])], [[1, 0]], 1))[1] == "V4"
    # V4: cross-queue cycle with an acyclic dependency graph
    assert agree(_g([T_(0, waits=[(1, 1)]), T_(0, signals=[0]),
                     T_(1, waits=[(0, 1)]), T_(1, signals=[1])],
                    [[0, 1], [2, 3]], 2))[1] == "V4"
    # V5: reader not ordered after its writer
    assert agree(_g([T_(0, acc=[(0, W, 0, 2)]), T_(1, acc=[(0, R, 1, 3)])], [[0], [1]], 0,
                    buf))[1] == "V5"
    # V6: unordered writes
    assert agree(_g([T_(0, acc=[(0, W, 0, 2)]), T_(1, acc=[(0, A, 1, 2)])], [[0], [1]], 0,
                    buf))[1] == "V6"
    # accumulators may be unordered
    assert agree(_g([T_(0, acc=[(0, A, 0, 2)]), T_(1, acc=[(0, A, 1, 2)])], [[0], [1]], 0,
                    buf))[0]
    # V6: READ_PREV after the reset of the same memory
    assert agree(_g([T_(0, signals=[0], acc=[(0, RS, 0, 1)]),
                     T_(1, waits=[(0, 1)], acc=[(0, RP, 0, 1)])], [[0], [1]], 1, buf))[1] == "V6"
    # V7: range past the end
    assert agree(_g([T_(0, acc=[(0, R, 0, 5)])], [[0]], 0, buf))[1] == "V7"
    # V8: output never written
    assert agree(_g([T_(0)], [[0]], 0, [{"size": 1, "output": True, "pair": -1}]))[1] == "V8"
    # V9: accumulator without a covering reset
    bufs = [{"size": 2, "output": False, "pair": 1}, {"size": 2, "output": False, "pair": -1}]
    assert agree(_g([T_(0, acc=[(0, A, 0, 2), (1, RS, 0, 1)])], [[0]], 0, bufs))[1] == "V9"
    assert agree(_g([T_(0, acc=[(0, A, 0, 2), (1, RS, 0, 2)])], [[0]], 0, bufs))[0]


def test_flagged_read_examples():
    """READ_FLAGGED: the reader waits for the words themselves (no counter):
    ordered after every writer or accumulator of its range; rule V10 wants
    exactly one value per element to wait for."""
    buf = [{"size": 4, "output": False, "pair": -1}]
    # valid: no counter at all, the flagged read orders the reader
    assert agree(_g([T_(0, acc=[(0, W, 0, 4)]), T_(1, acc=[(0, RF, 0, 4)])],
                    [[0], [1]], 0, buf))[0]
    # valid: two writers of disjoint halves, one reader of the whole
    assert agree(_g([T_(0, acc=[(0, W, 0, 2)]), T_(1, acc=[(0, W, 2, 4)]),
                     T_(2, acc=[(0, RF, 0, 4)])], [[0], [1], [2]], 0, buf))[0]
    # valid: accumulated elements (the flag comes when the accumulation ends)
    assert agree(_g([T_(0, acc=[(0, A, 0, 2)]), T_(1, acc=[(0, A, 0, 2)]),
                     T_(2, acc=[(0, RF, 0, 2)])], [[0], [1], [2]], 0, buf))[0]
    # V10: an element nobody writes (the reader would wait for ever)
    assert agree(_g([T_(0, acc=[(0, W, 0, 2)]), T_(1, acc=[(0, RF, 0, 3)])],
                    [[0], [1]], 0, buf))[1] == "V10"
    # V10: an element written twice (the reader could take the first value)
    assert agree(_g([T_(0, signals=[0], acc=[(0, W, 0, 2)]),
                     T_(1, waits=[(0, 1)], acc=[(0, W, 1, 2)]),
                     T_(2, acc=[(0, RF, 0, 2)])], [[0], [1], [2]], 1, buf))[1] == "V10"
    # V10: written and accumulated
    assert agree(_g([T_(0, acc=[(0, W, 0, 2)]), T_(1, acc=[(0, A, 0, 2)]),
                     T_(2, acc=[(0, RF, 0, 2)])], [[0], [1], [2]], 0, buf))[1] == "V10"
    # V1: a task that flag-reads its own output
    assert agree(_g([T_(0, acc=[(0, W, 0, 2), (0, RF, 0, 2)])], [[0]], 0, buf))[1] == "V1"
    # V1: two tasks flag-reading each other's output
    bufs = [{"size": 2, "output": False, "pair": -1}, {"size": 2, "output": False, "pair": -1}]
    assert agree(_g([T_(0, acc=[(0, W, 0, 2), (1, RF, 0, 2)]),
                     T_(1, acc=[(1, W, 0, 2), (0, RF, 0, 2)])], [[0], [1]], 0,
                    bufs))[1] == "V1"
    # V4: the reader is queued before its writer on the same SM
    assert agree(_g([T_(0, acc=[(0, W, 0, 2)]), T_(0, acc=[(0, RF, 0, 2)])], [[1, 0]], 0,
                    buf))[1] == "V4"
    # a flagged read does not order the reader against a later reset
    bufs = [{"size": 2, "output": False, "pair": -1}]
    assert agree(_g([T_(0, acc=[(0, W, 0, 2)]), T_(1, acc=[(0, RF, 0, 2)]),
                     T_(2, acc=[(0, RS, 0, 2)])], [[0], [1], [2]], 0, bufs))[1] == "V6"


def test_flagged_join_nodes_scale():
    """A level of many writers and many full-width flagged readers (the
    shape of a decode layer) validates quickly: the readers of one writer set
    share a join node."""
    n = 64
    buf = [{"size": n, "output": False, "pair": -1}]
    tasks = [T_(i, acc=[(0, W, i, i + 1)]) for i in range(n)]
    tasks += [T_(i, acc=[(0, RF, 0, n)]) for i in range(n)]
    queues = [[i, n + i] for i in range(n)]
    ok, rule, msg = amk.validate_graph(_g(tasks, queues, 0, buf))
    assert ok, (rule, msg)
