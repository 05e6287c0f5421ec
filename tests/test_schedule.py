"""Pins of the wave schedule (oracle/schedule.py) by brute force.

Lemma 3.1 of the Diagonal Batching paper (Pith review of arXiv 2506.05229,
"Core claim" and "Circularity Check"): for the layer-level dependency graph
(node (s, l) <- (s, l-1), (s-1, l)), grouping by s + l gives S + L - 1
groups, the minimum, because the longest dependency path has S + L - 1 nodes.
"""
import json
import os

import pytest

from oracle import schedule as sch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _longest_path_by_enumeration(deps):
    """Nodes on the longest path of the dependency DAG, found by walking every
    path from every node (exhaustive; no use of the grid's structure)."""
    succ = {n: [] for n in deps}
    for n, preds in deps.items():
        for p in preds:
            succ[p].append(n)
    best = 0

    def walk(n, length):
        nonlocal best
        best = max(best, length)
        for m in succ[n]:
            walk(m, length + 1)

    for n in deps:
        walk(n, 1)
    return best


def test_path_enumeration_separates_the_two_graphs():
    """The enumeration is not a restatement of S + L - 1: on the original-RMT
    graph (every layer of segment s waits for the last layer of s - 1) the
    longest path is the whole S x L sequence."""
    assert _longest_path_by_enumeration(sch.prmt_dependencies(3, 4)) == 3 + 4 - 1
    assert _longest_path_by_enumeration(sch.rmt_dependencies(3, 4)) == 3 * 4


@pytest.mark.parametrize("S,L", [(S, L) for S in range(1, 13) for L in range(1, 13)])
def test_diagonal_waves_valid_and_minimal(S, L):
    waves = sch.diagonal_waves(S, L)
    deps = sch.prmt_dependencies(S, L)
    assert len(waves) == S + L - 1
    for i, wave in enumerate(waves):
        assert all(s + l == i for s, l in wave)
        assert len(wave) == min(i + 1, L, S, S + L - 1 - i)
    flat = [n for w in waves for n in w]
    assert sorted(flat) == sorted(deps)          # every node exactly once
    assert sch.check_schedule(waves, deps) == []  # no intra-wave edge, no backward edge
    levels = sch.earliest_groups(deps)
    assert max(levels.values()) + 1 == len(waves)
    assert all(levels[(s, l)] == s + l for (s, l) in deps)   # earliest feasible group = s + l
    if S + L <= 11:
        assert _longest_path_by_enumeration(deps) == S + L - 1


@pytest.mark.parametrize("S,L", [(1, 1), (3, 5), (12, 12)])
def test_sequential_order_is_a_valid_schedule(S, L):
    order = sch.sequential_order(S, L)
    assert len(order) == S * L
    assert sch.check_schedule([[n] for n in order], sch.prmt_dependencies(S, L)) == []


def test_original_rmt_rejects_diagonal_schedule():
    """Negative control: the original RMT graph (final-layer memory feeds every
    layer of the next segment) must fail the diagonal schedule, as the Pith
    verdict's concrete test states for L=2, S=4."""
    g = json.load(open(os.path.join(GOLDEN, "rmt_concrete_test.json")))
    S, L = g["S"], g["L"]
    node, dep = tuple(g["node"]), tuple(g["depends_on"])
    deps = sch.rmt_dependencies(S, L)
    assert dep in deps[node]
    waves = sch.diagonal_waves(S, L)
    wave_of = {n: i for i, w in enumerate(waves) for n in w}
    assert wave_of[node] == g["diagonal_wave_of_node"]
    errs = sch.check_schedule(waves, deps)
    assert any(f"{dep}->{node}" in e for e in errs)
    assert sch.earliest_groups(deps)[node] >= g["earliest_group_at_least"]
    # the sequential order stays valid for the original RMT
    assert sch.check_schedule([[n] for n in sch.sequential_order(S, L)], deps) == []


@pytest.mark.parametrize("S,L", [(2, 2), (4, 3), (7, 5)])
def test_rmt_rejected_for_every_multi_segment_grid(S, L):
    assert sch.check_schedule(sch.diagonal_waves(S, L), sch.rmt_dependencies(S, L)) != []


def test_checker_catches_planted_errors():
    S, L = 4, 3
    deps = sch.prmt_dependencies(S, L)
    waves = sch.diagonal_waves(S, L)
    missing = [w[:] for w in waves]
    missing[2].pop()
    assert any("never scheduled" in e for e in sch.check_schedule(missing, deps))
    swapped = [waves[1], waves[0]] + waves[2:]
    assert any("backwards" in e for e in sch.check_schedule(swapped, deps))
    merged = [waves[0] + waves[1]] + waves[2:]
    assert any("inside group" in e for e in sch.check_schedule(merged, deps))


@pytest.mark.parametrize("S,L", [(S, L) for S in range(1, 13) for L in range(1, 13)])
def test_each_wave_starts_and_finishes_at_most_one_segment(S, L):
    """A wave holds at most one layer-0 node (the segment whose embeddings it
    first needs) and at most one last-layer node (the segment whose hidden
    states it completes); segment s starts in wave s and finishes in wave
    s + L - 1.  The per-segment host copies are ordered by exactly this."""
    for i, wave in enumerate(sch.diagonal_waves(S, L)):
        starts = [s for s, l in wave if l == 0]
        ends = [s for s, l in wave if l == L - 1]
        assert len(starts) <= 1 and len(ends) <= 1
        assert starts == ([i] if i < S else [])
        assert ends == ([i - (L - 1)] if 0 <= i - (L - 1) < S else [])
