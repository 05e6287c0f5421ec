"""Oracle: the diagonal (wave) schedule and a brute-force dependency checker.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.

Sources (all indices 0-based, node = (segment s, layer l)):

* Dependency graph of a layer-level recurrent model (PRMT, e.g. ARMT):
  node (s, l) depends only on (s, l-1) and (s-1, l).
  -- "Diagonal Batching for Recurrent Memory Transformers" skill page,
     section "Practical Guidance" (Diagonal Dependency Analysis), and the
     Pith review of arXiv 2506.05229, section "What carries the argument".
* Schedule: wave i holds every node with s + l = i; there are S + L - 1 waves
  instead of S * L sequential steps; Lemma 3.1 says this is the minimum
  because the longest dependency path has S + L - 1 nodes.
  -- Pith review, sections "Core claim" and "Circularity Check" (Lemma 3.1).
* The original RMT (its Eq. 1) feeds the previous segment's final-layer memory
  into every layer of the next segment, which breaks the schedule.
  -- Pith review, "Load-bearing premise"; Pith verdict, skeptic critique
     ("concrete_test", L=2, S=4).  Modelled by ``rmt_dependencies``.
* Baseline schedule: S x L sequential operations.
  -- Pith review, Figure 3 caption.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

Node = Tuple[int, int]


def diagonal_waves(S: int, L: int) -> List[List[Node]]:
    """Waves i = 0 .. S+L-2; wave i lists (s, l) with s + l = i, l ascending."""
    if S <= 0 or L <= 0:
        return []
    waves = []
    for i in range(S + L - 1):
        wave = []
        for l in range(L):
            s = i - l
            if 0 <= s < S:
                wave.append((s, l))
        waves.append(wave)
    return waves


def sequential_order(S: int, L: int) -> List[Node]:
    """The baseline order: segment-major, one node at a time."""
    return [(s, l) for s in range(S) for l in range(L)]


def prmt_dependencies(S: int, L: int) -> Dict[Node, List[Node]]:
    """Layer-level recurrence: (s, l) <- (s, l-1), (s-1, l)."""
    deps = {}
    for s in range(S):
        for l in range(L):
            d = []
            if l > 0:
                d.append((s, l - 1))
            if s > 0:
                d.append((s - 1, l))
            deps[(s, l)] = d
    return deps


def rmt_dependencies(S: int, L: int) -> Dict[Node, List[Node]]:
    """Original RMT: in addition, every layer of segment s reads the memory the
    final layer (L-1) of segment s-1 produced."""
    deps = prmt_dependencies(S, L)
    for s in range(1, S):
        for l in range(L):
            if (s - 1, L - 1) not in deps[(s, l)]:
                deps[(s, l)].append((s - 1, L - 1))
    return deps


def earliest_groups(deps: Dict[Node, List[Node]]) -> Dict[Node, int]:
    """Earliest feasible group of each node = length (in nodes) of the longest
    dependency path ending at it, minus one.  Plain memoised DFS."""
    memo: Dict[Node, int] = {}

    def level(n: Node) -> int:
        if n in memo:
            return memo[n]
        stack = [(n, False)]
        while stack:
            cur, expanded = stack.pop()
            if cur in memo:
                continue
            preds = deps[cur]
            if expanded or all(p in memo for p in preds):
                memo[cur] = 1 + max((memo[p] for p in preds), default=-1)
            else:
                stack.append((cur, True))
                stack.extend((p, False) for p in preds if p not in memo)
        return memo[n]

    for n in deps:
        level(n)
    return memo


def check_schedule(groups: Sequence[Sequence[Node]], deps: Dict[Node, List[Node]]) -> List[str]:
    """Return every violation of ``groups`` as an execution schedule of ``deps``:
    a node missing or repeated, an edge inside one group, or an edge pointing
    from a later group to an earlier one.  Empty list = valid."""
    errors = []
    where: Dict[Node, int] = {}
    for gi, grp in enumerate(groups):
        for n in grp:
            if n in where:
                errors.append(f"node {n} scheduled twice (groups {where[n]} and {gi})")
            where[n] = gi
    for n in deps:
        if n not in where:
            errors.append(f"node {n} never scheduled")
    for n, preds in deps.items():
        if n not in where:
            continue
        for p in preds:
            if p not in where:
                continue
            if where[p] == where[n]:
                errors.append(f"edge {p}->{n} inside group {where[n]}")
            elif where[p] > where[n]:
                errors.append(f"edge {p}->{n} goes backwards ({where[p]} > {where[n]})")
    return errors
