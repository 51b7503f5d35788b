"""Brute-force model of the split-K attention merge: "the last chunk task to
arrive merges the partials".

TEST INFRASTRUCTURE ONLY.  The schedule validator treats the attention tasks
of one KV head as a commutative accumulation into the layer's attention
output; the protocol that realises it at run time is a per-(layer, KV head)
arrival counter (gist.science technical summary, "De Safety Gate": every
memory access must respect happens-before; the split-K combine is an online
softmax).  This module executes that protocol's semantics on tiny cases,
over every interleaving of its events, and reports what goes wrong.  It
shares no code with the kernel or the host library: it restates the rules.

The protocol, per decode step at position pos with C chunks per KV head:
  * n = pos + 1 positions are cut into chunks of max(ceil(n / C), 32)
    positions; the nne chunks that hold a position are the step's arrivals
    (empty chunks do nothing).  With nne == 1 the single chunk writes the
    output itself and nothing arrives.
  * Each non-empty chunk task writes its partial (m, l, o), then adds one to
    the head's counter with an acquire-release read-modify-write.  The task
    that reads base + nne - 1 (the count of all earlier arrivals, this
    step's included, is then base + nne) merges: it reads every partial of
    the step and writes the output.
  * The counter is never reset; the host adds the step's nne to base after
    each step with nne > 1.

Events of one step (steps run one after another: each is one kernel launch
on one stream).  Task c: W_c (store of its partial), A_c (the atomic), and,
if it merges, R_c,j (load of partial j, for every j) in order.  Memory
visibility is modelled as a global order of "visible" events:
  * with the release half of the atomic, W_c is visible before A_c; without
    it, W_c becomes visible at some later event V_c, possibly after A_c and
    after the merger's loads;
  * with the acquire half, the merger's loads come after its A_c; without
    it, they may be satisfied early, at any point after the task's start
    (the task does not yet know it is the merger; the values stay the ones
    read then).
A step is correct when exactly one task merges and every load of the merger
sees this step's partial.  ``check`` explores every interleaving of every
step of a position sequence and returns the first violation, or None.
"""
from __future__ import annotations

from dataclasses import dataclass
from functools import lru_cache
from typing import List, Optional, Tuple

MIN_CHUNK = 32


def chunk_len(n: int, splits: int) -> int:
    c = (n + splits - 1) // splits
    return c if c > MIN_CHUNK else MIN_CHUNK


def arrivals(pos: int, splits: int) -> int:
    """Non-empty chunks of the step at position pos (0 when the step's only
    chunk writes the output itself)."""
    n = pos + 1
    nne = (n + chunk_len(n, splits) - 1) // chunk_len(n, splits)
    return nne if nne > 1 else 0


@dataclass(frozen=True)
class Protocol:
    release: bool = True      # partial stores visible before the atomic
    acquire: bool = True      # merger's loads ordered after the atomic
    threshold: int = -1       # merge when old == base + nne + threshold
    base_rule: str = "nne"    # host: "nne" (add nne when > 1), "splits" (add C), "always"


def _base_increment(proto: Protocol, pos: int, splits: int) -> int:
    n = pos + 1
    nne = (n + chunk_len(n, splits) - 1) // chunk_len(n, splits)
    if proto.base_rule == "splits":
        return splits
    if proto.base_rule == "always":
        return nne
    return nne if nne > 1 else 0


def _step(proto: Protocol, nne: int, base: int, counter: int) -> Optional[str]:
    """Explores every interleaving of one step with nne arrivals.  The
    counter holds `counter` at the start (the value the earlier steps left);
    the kernel compares against `base`.  Returns a violation or None."""
    # per task state: phase 0 = not started, 1 = stored (W done),
    # 2 = arrived (A done; merger decided), 3 = done
    # loads: for a merger-to-be without acquire, loads can happen early; we
    # model each task's loads as a tuple of values read so far (None = not yet)
    # visible[c]: partial c of this step is visible
    # state = (phases, visible, counter, loads, merger flags)
    start = (tuple([0] * nne), tuple([False] * nne), counter,
             tuple(tuple([None] * nne) for _ in range(nne)), tuple([None] * nne))

    @lru_cache(maxsize=None)
    def explore(state) -> Optional[str]:
        phases, visible, ctr, loads, merge = state
        moves = []
        for c in range(nne):
            ph = phases[c]
            if ph == 0:  # W_c
                v = list(visible)
                if proto.release:
                    v[c] = True  # visible no later than A_c: take it at once
                moves.append((c, 1, tuple(v), ctr, loads, merge))
            elif ph == 1:  # A_c
                old = ctr
                m = list(merge)
                m[c] = old == base + nne + proto.threshold
                moves.append((c, 2, visible, ctr + 1, loads, tuple(m)))
            elif ph == 2:
                if merge[c]:
                    # loads in order after the atomic (the ones already
                    # taken early stay as they were)
                    ld = list(loads[c])
                    j = next((k for k in range(nne) if ld[k] is None), None)
                    if j is None:
                        moves.append((c, 3, visible, ctr, loads, merge))
                    else:
                        ld[j] = visible[j]
                        L = list(loads)
                        L[c] = tuple(ld)
                        moves.append((c, 2, visible, ctr, tuple(L), merge))
                else:
                    moves.append((c, 3, visible, ctr, loads, merge))
            if not proto.acquire and ph in (1, 2) and merge[c] is None:
                # an early load by a task that may turn out to merge
                ld = list(loads[c])
                j = next((k for k in range(nne) if ld[k] is None), None)
                if j is not None:
                    ld[j] = visible[j]
                    L = list(loads)
                    L[c] = tuple(ld)
                    moves.append((c, ph, visible, ctr, tuple(L), merge))
        if not proto.release:
            for c in range(nne):  # late visibility of a partial already stored
                if phases[c] >= 1 and not visible[c]:
                    v = list(visible)
                    v[c] = True
                    moves.append((c, phases[c], tuple(v), ctr, loads, merge))
        if not moves:
            n_merge = sum(1 for m in merge if m)
            if n_merge != 1:
                return f"{n_merge} tasks merged"
            c = merge.index(True)
            if not all(loads[c]):
                return "the merger read a partial of an earlier step"
            return None
        for c, ph, v, ct, ld, m in moves:
            p = list(phases)
            p[c] = ph
            bad = explore((tuple(p), v, ct, ld, m))
            if bad:
                return bad
        return None

    return explore(start)


def check(proto: Protocol, positions: List[int], splits: int) -> Optional[Tuple[int, str]]:
    """Runs the steps at `positions` in order under `proto`.  Returns (the
    position of the first failing step, what failed) or None."""
    base = 0
    counter = 0
    for pos in positions:
        n = pos + 1
        nne = (n + chunk_len(n, splits) - 1) // chunk_len(n, splits)
        if nne > 1:
            bad = _step(proto, nne, base, counter)
            if bad:
                return pos, bad
            counter += nne
        base += _base_increment(proto, pos, splits)
    return None
