"""Pins for the oracle's best-first draft-tree construction (CPU only).

Page "The Architecture of Diagnosis", section "Phase 1: Custom CUDA Kernels",
item 1 says only that a GPU builder grows the draft tree best-first. The
reading (kdv_oracle.cpp): a node is a path of per-position candidate choices,
its score is the fp32 sum of the candidates' log-probabilities, and the tree
is the first T nodes in (score descending, path ascending) order. These
tests pin the oracle's expansion to an independent brute-force sort of every
path, to closed forms and to a hand-worked example.
"""
import itertools

import numpy as np
import pytest

import oracle


def _brute_force(T, root_token, cand_token, cand_logp):
    D, K = cand_token.shape
    nodes = [((), np.float32(0.0))]
    frontier = [((), np.float32(0.0))]
    for d in range(D):
        nxt = []
        for path, sc in frontier:
            for j in range(K):
                s = np.float32(sc + cand_logp[d, j])      # one float32 add, root-first
                nxt.append((path + (j,), s))
        nodes += nxt
        frontier = nxt
    # score descending; ties: the path digit by digit, a prefix first
    nodes.sort(key=lambda n: (-float(n[1]), n[0]))
    chosen = nodes[:T]
    index = {path: i for i, (path, _) in enumerate(chosen)}
    parent = [index[p[:-1]] if p else -1 for p, _ in chosen]
    token = [int(cand_token[len(p) - 1, p[-1]]) if p else root_token for p, _ in chosen]
    depth = [len(p) for p, _ in chosen]
    score = [s for _, s in chosen]
    return parent, token, depth, score


@pytest.mark.parametrize("D,K", [(1, 1), (2, 2), (3, 2), (2, 3), (4, 2), (3, 3)])
def test_build_matches_brute_force_sort(D, K):
    rng = np.random.default_rng(10 * D + K)
    total = sum(K ** d for d in range(D + 1))
    for trial in range(20):
        # quantised log-probabilities (and some zeros) make score ties common
        cand_logp = -np.round(rng.exponential(0.7, size=(D, K)) * 4) / 4
        cand_logp = cand_logp.astype(np.float32)
        cand_token = rng.integers(0, 50, size=(D, K)).astype(np.int32)
        for T in sorted({1, 2, total // 2 + 1, total}):
            got = oracle.tree_build(T, 7, cand_token, cand_logp)
            want = _brute_force(T, 7, cand_token, cand_logp)
            assert list(got[0]) == want[0]
            assert list(got[1]) == want[1]
            assert list(got[2]) == want[2]
            assert [float(x) for x in got[3]] == [float(x) for x in want[3]]


def test_build_parents_precede_children_and_scores_decrease():
    rng = np.random.default_rng(3)
    cand_logp = np.log(rng.dirichlet(np.ones(6), size=15)).astype(np.float32)[:, :6]
    cand_token = rng.integers(0, 1000, size=(15, 6)).astype(np.int32)
    parent, token, depth, score = oracle.tree_build(64, 1, cand_token, cand_logp)
    assert len(parent) == 64 and parent[0] == -1
    for i in range(1, 64):
        assert 0 <= parent[i] < i and depth[i] == depth[parent[i]] + 1
        assert score[i] <= score[parent[i]]
    assert all(score[i] >= score[i + 1] for i in range(63))


def test_build_chain_when_one_candidate():
    cand_token = np.arange(5, dtype=np.int32)[:, None] + 100
    cand_logp = np.full((5, 1), -0.5, dtype=np.float32)
    parent, token, depth, score = oracle.tree_build(4, 9, cand_token, cand_logp)
    assert list(parent) == [-1, 0, 1, 2] and list(token) == [9, 100, 101, 102]
    parent, token, depth, _ = oracle.tree_build(64, 9, cand_token, cand_logp)
    assert len(parent) == 6                       # root + 5 positions: candidates run out
    assert list(depth) == [0, 1, 2, 3, 4, 5]


def test_build_hand_worked_example():
    """Probabilities 0.6/0.4, 0.7/0.3, 0.9/0.1 at three positions: the best
    paths are () > (0) > (0,0) > (1) > (0,0,0) > (1,0) (log-probability sums
    0, -0.51, -0.87, -0.92, -0.97, -1.27)."""
    cand_token = np.array([[10, 11], [20, 21], [30, 31]], dtype=np.int32)
    cand_logp = np.log(np.array([[0.6, 0.4], [0.7, 0.3], [0.9, 0.1]], dtype=np.float32)).astype(np.float32)
    parent, token, depth, score = oracle.tree_build(6, 99, cand_token, cand_logp)
    assert list(parent) == [-1, 0, 1, 0, 2, 3]
    assert list(token) == [99, 10, 20, 11, 30, 20]
    assert list(depth) == [0, 1, 2, 1, 3, 2]


def test_build_rejects_bad_sizes():
    with pytest.raises(ValueError):
        oracle.tree_build(0, 1, np.zeros((2, 2), np.int32), np.zeros((2, 2), np.float32))
    with pytest.raises(ValueError):
        oracle.tree_build(4, 1, np.zeros((2, 9), np.int32), np.zeros((2, 9), np.float32))


def test_build_nan_logprob_reads_as_minus_inf():
    rng = np.random.default_rng(4)
    cand_logp = np.log(rng.dirichlet(np.ones(3), size=3)).astype(np.float32)
    cand_token = rng.integers(0, 9, size=(3, 3)).astype(np.int32)
    with_nan = cand_logp.copy()
    with_nan[1, 0] = np.nan
    with_inf = cand_logp.copy()
    with_inf[1, 0] = -np.inf
    a = oracle.tree_build(30, 5, cand_token, with_nan)
    b = _brute_force(30, 5, cand_token, with_inf)
    assert list(a[0]) == b[0] and list(a[1]) == b[1]


def test_build_nan_path_score_reads_as_minus_inf():
    """+inf at one position and -inf at the next make the path's fp32 sum NaN;
    that path ranks like a -inf one. With a +inf log-probability a child can
    outrank its parent, so the reference here is a plain best-first expansion
    (frontier as a Python list, best = min of (-score, path)) with NaN sums
    replaced by -inf."""
    cand_token = np.array([[10, 11], [20, 21], [30, 31]], dtype=np.int32)
    cand_logp = np.array([[np.inf, -0.5], [-np.inf, -0.25], [-1.0, -2.0]], dtype=np.float32)
    got = oracle.tree_build(15, 3, cand_token, cand_logp)

    D, K = cand_token.shape
    frontier = [((), np.float32(0.0), -1)]
    out = []
    with np.errstate(invalid="ignore"):
        while frontier and len(out) < 15:
            best = min(range(len(frontier)), key=lambda i: (-float(frontier[i][1]), frontier[i][0]))
            path, sc, par = frontier.pop(best)
            out.append((path, sc, par))
            if len(path) < D:
                for j in range(K):
                    s = np.float32(sc + cand_logp[len(path), j])
                    frontier.append((path + (j,), np.float32(-np.inf) if np.isnan(s) else s, len(out) - 1))
    assert list(got[0]) == [par for _, _, par in out]
    assert list(got[2]) == [len(p) for p, _, _ in out]
    assert [float(x) for x in got[3]] == [float(s) for _, s, _ in out]
    # the paths under (0, 0) are the NaN ones
    assert any(p[:2] == (0, 0) and np.isneginf(s) for p, s, _ in out)
