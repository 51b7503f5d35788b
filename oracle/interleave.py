"""Brute-force interleaving checker for per-SM task schedules.

TEST INFRASTRUCTURE ONLY.  This is the independent check that pins the
schedule validator (x-techcon AutoMegaKernel article, section 1: 7160
adversarial schedules, the unsafe ones confirmed by an independent oracle,
zero false accepts).  It shares no code with the validator and uses no graph
algorithm: it executes the schedule's semantics.

Semantics (tasks are atomic):
  * SM s runs its queue in order; the head task may run once, for every
    (counter, t) it waits on, the number of finished signals to that counter
    is >= t, and, for every READ_FLAGGED range it has, every task with a
    WRITE or ACCUM overlapping that range has finished (a flagged word takes
    the epoch's tag from its one writer, or when its accumulation is done; a
    task that writes what it flag-reads never runs).  Running it adds 1 per
    signal.
  * A state is the set of finished tasks.  All reachable states are
    enumerated from the empty set.
  * Deadlock: a reachable state with unfinished tasks and no runnable head.
  * "a always before b": no reachable state contains b but not a.
Verdicts, on overlapping accesses of different tasks:
  READ (and READ_FLAGGED) needs every WRITE/ACCUM always before it; WRITE/WRITE, WRITE/ACCUM and
  RESET/RESET need one fixed order; READ_PREV needs to be always before every
  WRITE/ACCUM/RESET; RESET needs every other access always before it.
The purely syntactic conditions (ids and ranges, thresholds 1 <= t <= number
of producers, full-count waits on shared counters, every element of a
READ_FLAGGED range written exactly once or only accumulated, outputs written,
reset coverage of double-buffered accumulators) are definitions, checked as
written.

Graph format (plain Python): {
  "n_counters": int,
  "buffers": [{"size": int, "output": bool, "pair": int}],
  "tasks": [{"sm": int, "waits": [(ctr, t)], "signals": [ctr],
             "accesses": [(buf, kind, begin, end)]}],
  "queues": [[task ids in order] per SM]}
kinds: 0 READ, 1 WRITE, 2 ACCUM, 3 READ_PREV, 4 RESET, 5 READ_FLAGGED.
"""
from __future__ import annotations

from typing import Dict, List, Tuple

READ, WRITE, ACCUM, READ_PREV, RESET, READ_FLAGGED = range(6)


def _syntax(g) -> str:
    T = len(g["tasks"])
    C = g["n_counters"]
    bufs = g["buffers"]
    B = len(bufs)
    for i, b in enumerate(bufs):
        if b["size"] < 0 or (b["pair"] != -1 and not (0 <= b["pair"] < B and b["pair"] != i)):
            return "V7"
    seen = []
    for s, q in enumerate(g["queues"]):
        for t in q:
            if not (0 <= t < T) or t in seen or g["tasks"][t]["sm"] != s:
                return "V7"
            seen.append(t)
    if len(seen) != T or (T > 0 and len(g["queues"]) < 1):
        return "V7"
    for task in g["tasks"]:
        for c, _ in task["waits"]:
            if not (0 <= c < C):
                return "V7"
        for c in task["signals"]:
            if not (0 <= c < C):
                return "V7"
        for (b, k, lo, hi) in task["accesses"]:
            if not (0 <= b < B) or k not in (READ, WRITE, ACCUM, READ_PREV, RESET,
                                             READ_FLAGGED):
                return "V7"
            if lo < 0 or hi <= lo or hi > bufs[b]["size"]:
                return "V7"
    nprod = [0] * C
    for task in g["tasks"]:
        for c in task["signals"]:
            nprod[c] += 1
    for task in g["tasks"]:
        for c, t in task["waits"]:
            if t < 1 or t > nprod[c]:
                return "V2"
    for task in g["tasks"]:
        for c, t in task["waits"]:
            if nprod[c] > 1 and t != nprod[c]:
                return "V3"
    # V10: each flagged-read element has exactly one value to wait for
    for task in g["tasks"]:
        for (b, k, lo, hi) in task["accesses"]:
            if k != READ_FLAGGED:
                continue
            for x in range(lo, hi):
                nw = na = 0
                for other in g["tasks"]:
                    for (b2, k2, lo2, hi2) in other["accesses"]:
                        if b2 == b and lo2 <= x < hi2:
                            nw += k2 == WRITE
                            na += k2 == ACCUM
                if not ((nw == 1 and na == 0) or (nw == 0 and na >= 1)):
                    return "V10"
    return ""


def _flag_deps(g):
    """Per task, the tasks whose WRITE/ACCUM its READ_FLAGGED ranges wait for."""
    tasks = g["tasks"]
    deps = []
    for task in tasks:
        d = set()
        for (b, k, lo, hi) in task["accesses"]:
            if k != READ_FLAGGED:
                continue
            for w, other in enumerate(tasks):
                for (b2, k2, lo2, hi2) in other["accesses"]:
                    if b2 == b and k2 in (WRITE, ACCUM) and lo2 < hi and lo < hi2:
                        d.add(w)
        deps.append(d)
    return deps


def _post_syntax(g) -> str:
    bufs = g["buffers"]
    for i, b in enumerate(bufs):
        if b["output"]:
            if not any(bb == i and k in (WRITE, ACCUM)
                       for task in g["tasks"] for (bb, k, _, _) in task["accesses"]):
                return "V8"
    for i, b in enumerate(bufs):
        p = b["pair"]
        if p < 0:
            continue
        covered = set()
        for task in g["tasks"]:
            for (bb, k, lo, hi) in task["accesses"]:
                if bb == p and k == RESET:
                    covered.update(range(lo, hi))
        for task in g["tasks"]:
            for (bb, k, lo, hi) in task["accesses"]:
                if bb == i and k == ACCUM and not set(range(lo, hi)) <= covered:
                    return "V9"
    return ""


def _reachable(g) -> Tuple[List[int], bool]:
    """All reachable finished-sets (bitmasks) and whether one deadlocks."""
    tasks, queues = g["tasks"], g["queues"]
    T = len(tasks)
    full = (1 << T) - 1
    fdeps = _flag_deps(g)
    start = 0
    seen = {start}
    stack = [start]
    deadlock = False
    while stack:
        st = stack.pop()
        counts: Dict[int, int] = {}
        for t in range(T):
            if st >> t & 1:
                for c in tasks[t]["signals"]:
                    counts[c] = counts.get(c, 0) + 1
        moved = False
        for q in queues:
            head = next((t for t in q if not st >> t & 1), None)
            if head is None:
                continue
            if (all(counts.get(c, 0) >= th for c, th in tasks[head]["waits"])
                    and all(st >> w & 1 for w in fdeps[head])):
                moved = True
                nxt = st | (1 << head)
                if nxt not in seen:
                    seen.add(nxt)
                    stack.append(nxt)
        if not moved and st != full:
            deadlock = True
    return sorted(seen), deadlock


def check(g) -> Tuple[bool, str]:
    """(accepted, reason) with reason in {"ok", "V2", "V3", "V7", "V8", "V9",
    "V10", "deadlock", "race"}."""
    r = _syntax(g)
    if r:
        return False, r
    states, deadlock = _reachable(g)
    if deadlock:
        return False, "deadlock"
    T = len(g["tasks"])
    # can_precede[a][b]: some reachable state has a finished and b not
    can_precede = [[False] * T for _ in range(T)]
    for st in states:
        done = [t for t in range(T) if st >> t & 1]
        todo = [t for t in range(T) if not st >> t & 1]
        for a in done:
            row = can_precede[a]
            for b in todo:
                row[b] = True

    def always_before(a, b):
        return not can_precede[b][a]

    accs = [(t, b, k, lo, hi) for t, task in enumerate(g["tasks"])
            for (b, k, lo, hi) in task["accesses"]]
    for i in range(len(accs)):
        for j in range(len(accs)):
            if i == j:
                continue
            ta, ba, ka, la, ha = accs[i]
            tb, bb, kb, lb, hb = accs[j]
            if ta == tb or ba != bb or not (la < hb and lb < ha):
                continue
            if ka in (READ, READ_FLAGGED) and kb in (WRITE, ACCUM) and not always_before(tb, ta):
                return False, "race"
            if (((ka == WRITE and kb in (WRITE, ACCUM)) or (ka == RESET and kb == RESET))
                    and not (always_before(ta, tb) or always_before(tb, ta))):
                return False, "race"
            if ka == READ_PREV and kb in (WRITE, ACCUM, RESET) and not always_before(ta, tb):
                return False, "race"
            if ka == RESET and kb != RESET and not always_before(tb, ta):
                return False, "race"
    r = _post_syntax(g)
    if r:
        return False, r
    return True, "ok"
