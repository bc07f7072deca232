"""Pins for the oracle's greedy tree acceptance (CPU only).

The acceptance rule follows the page "The Architecture of Diagnosis", section
"Phase 1: Custom CUDA Kernels", item 3 (after verification a device kernel
keeps the longest prefix of draft tokens the target accepts). The page gives
no formula, so each check below pins the oracle to something independent of
its own code: numpy's argmax, a brute-force enumeration of every root path,
the textbook greedy walk, closed forms for chains and stars, and a small
example worked by hand.
"""
import itertools

import numpy as np
import pytest

import oracle
from speculative_tree_verify_mla_b200 import datagen


# ----------------------------------------------------------------- argmax

def test_argmax_matches_numpy_first_occurrence():
    rng = np.random.default_rng(11)
    x = datagen.bf16_round(rng.standard_normal((37, 1000)).astype(np.float32))
    # plant ties: the row maximum repeated at a later and an earlier column
    for r in range(0, 37, 3):
        m = x[r].max()
        x[r, rng.integers(0, 1000, size=3)] = m
    np.testing.assert_array_equal(oracle.argmax(x), np.argmax(x, axis=1))


def test_argmax_special_values():
    nan, inf = np.nan, np.inf
    rows = np.array([
        [nan, 1.0, 3.0, nan, 3.0],      # NaN skipped, tie -> lowest
        [nan, nan, nan, nan, nan],      # all NaN -> 0
        [-inf, -inf, -inf, -inf, -inf], # all equal -> 0
        [-0.0, 0.0, -1.0, -0.0, -2.0],  # -0 == +0 -> lowest
        [1.0, inf, 2.0, inf, nan],      # +inf wins, first one
        [-inf, nan, -5.0, -inf, -5.0],
    ], dtype=np.float32)
    np.testing.assert_array_equal(oracle.argmax(rows), [2, 0, 0, 0, 1, 2])
    ok = ~np.all(np.isnan(rows), axis=1)
    np.testing.assert_array_equal(oracle.argmax(rows)[ok], np.nanargmax(rows[ok], axis=1))


# ------------------------------------------------------------ acceptance

def _brute_force(parent, token, target):
    """Enumerate every root path by depth-first search over child lists; keep
    the valid ones (each step's token equals the target at its parent); the
    answer is the longest, then the one ending at the lowest node index."""
    T = len(parent)
    children = {u: [v for v in range(T) if parent[v] == u] for u in range(T)}
    best = None

    def dfs(path):
        nonlocal best
        cand = (len(path), -path[-1])
        if best is None or cand > (len(best), -best[-1]):
            best = list(path)
        for v in children[path[-1]]:
            if token[v] == target[path[-1]]:
                dfs(path + [v])

    for r in range(T):
        if parent[r] == -1:
            dfs([r])
    return best


def _greedy_walk(parent, token, target):
    """Textbook greedy walk from node 0: step to the child whose token equals
    the target at the current node, until none does."""
    T = len(parent)
    path = [0]
    while True:
        u = path[-1]
        nxt = [v for v in range(T) if parent[v] == u and token[v] == target[u]]
        if not nxt:
            return path
        assert len(nxt) == 1
        path.append(nxt[0])


def _all_parent_arrays(T):
    choices = [[-1]] + [[-1] + list(range(i)) for i in range(1, T)]
    return itertools.product(*choices)


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 6])
def test_accept_brute_force_all_forests(T):
    """Every forest with parent[i] in {-1} U [0, i), tokens from a 3-letter
    alphabet so that matches and duplicate sibling tokens are frequent."""
    rng = np.random.default_rng(100 + T)
    n = 0
    for parent in _all_parent_arrays(T):
        for _ in range(3):
            token = rng.integers(0, 3, size=T).astype(np.int32)
            target = rng.integers(0, 3, size=T).astype(np.int32)
            path, ln, bonus = oracle.tree_accept(parent, token, target)
            want = _brute_force(list(parent), token, target)
            assert ln == len(want)
            assert list(path[:ln]) == want and all(path[ln:] == -1)
            assert bonus == target[want[-1]]
            n += 1
    assert n == 3 * int(np.prod([i + 1 for i in range(T)]))


def test_accept_equals_greedy_walk_with_distinct_siblings():
    for seed in range(200):
        rng = np.random.default_rng(seed)
        T = int(rng.integers(1, 17))
        parent = datagen.random_tree(T, rng)
        token = rng.permutation(40)[:T].astype(np.int32)       # all tokens distinct
        target = np.where(rng.random(T) < 0.7,
                          token[rng.integers(0, T, size=T)], 99).astype(np.int32)
        path, ln, _ = oracle.tree_accept(parent, token, target)
        assert list(path[:ln]) == _greedy_walk(parent, token, target)


def test_accept_chain_closed_form():
    """A chain accepts 1 + (number of leading draft tokens equal to the target)."""
    rng = np.random.default_rng(5)
    for _ in range(100):
        T = int(rng.integers(1, 65))
        token = rng.integers(0, 4, size=T).astype(np.int32)
        target = rng.integers(0, 4, size=T).astype(np.int32)
        k = 0
        while k + 1 < T and token[k + 1] == target[k]:
            k += 1
        path, ln, bonus = oracle.tree_accept(datagen.chain_tree(T), token, target)
        assert ln == k + 1
        assert list(path[:ln]) == list(range(k + 1))
        assert bonus == target[k]


def test_accept_star_closed_form():
    """A star accepts the root plus the lowest-index child matching target[0]."""
    token = np.array([9, 4, 7, 7, 4], dtype=np.int32)
    for t0, want in [(7, [0, 2]), (4, [0, 1]), (5, [0])]:
        target = np.array([t0, 1, 2, 3, 6], dtype=np.int32)
        path, ln, bonus = oracle.tree_accept(datagen.star_tree(5), token, target)
        assert list(path[:ln]) == want
        assert bonus == target[want[-1]]


def test_accept_hand_worked_example():
    """parent [-1,0,0,1,1], tokens [5,7,8,9,3], target [7,3,1,2,0]:
    node 1 (7 == target[0]) is accepted, node 2 (8) is not; under node 1,
    node 4 (3 == target[1]) is accepted, node 3 (9) is not. Path 0-1-4,
    bonus target[4] = 0."""
    path, ln, bonus = oracle.tree_accept([-1, 0, 0, 1, 1], [5, 7, 8, 9, 3], [7, 3, 1, 2, 0])
    assert (list(path), ln, bonus) == ([0, 1, 4, -1, -1], 3, 0)


def test_accept_rejects_malformed_parent():
    with pytest.raises(ValueError):
        oracle.tree_accept([-1, 1], [0, 0], [0, 0])       # self-parent
    with pytest.raises(ValueError):
        oracle.tree_accept([-1, 0, 3, 0], [0] * 4, [0] * 4)   # forward parent


def test_accept_commit_is_stable_partition():
    rng = np.random.default_rng(8)
    for _ in range(50):
        T = int(rng.integers(1, 20))
        L = int(rng.integers(0, 30))
        parent = datagen.random_tree(T, rng)
        token = rng.integers(0, 3, size=T).astype(np.int32)
        target = rng.integers(0, 3, size=T).astype(np.int32)
        path, ln, _ = oracle.tree_accept(parent, token, target)
        pt = rng.permutation(1000)[:L + T].astype(np.int32)
        new = oracle.accept_commit(pt, L, path, ln)
        np.testing.assert_array_equal(new[:L], pt[:L])                 # prefix untouched
        np.testing.assert_array_equal(new[L:L + ln], pt[L + path[:ln]])  # path, in order
        rest = [u for u in range(T) if u not in set(path[:ln].tolist())]
        np.testing.assert_array_equal(new[L + ln:], pt[L + np.array(rest, dtype=int)])
        assert sorted(new.tolist()) == sorted(pt.tolist())               # still a permutation


def test_accept_case_generator_plants_targets():
    """The planted maximum is found by argmax, so with p_follow = 1 and distinct
    sibling tokens the accepted path reaches a leaf of the tree."""
    parents = [datagen.random_tree(13, np.random.default_rng(3))]
    case = datagen.make_accept_case("t", parents=parents, vocab=4096, seed=2, p_follow=1.0)
    res = oracle.accept_case(case)
    end = res["path"][0, res["len"][0] - 1]
    assert not np.any(parents[0] == end)          # end is a leaf
