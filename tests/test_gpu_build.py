"""GPU parity of kdv_tree_build against the oracle (bit-exact: the tree is
integer output and the scores are the same float adds in the same order).

Best-first draft-tree construction (page "The Architecture of Diagnosis",
section "Phase 1: Custom CUDA Kernels", item 1).
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_tree_verify_mla_b200 import datagen, kdv

pytestmark = pytest.mark.gpu
dev = "cuda"


def _run(case, max_T=64):
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    sumT = int(case.tree_off[-1])
    out = {k: torch.full((sumT,), -7, dtype=torch.int32, device=dev) for k in ("parent", "token", "depth")}
    score = torch.full((sumT,), float("nan"), device=dev)
    d_err = torch.zeros(1, dtype=torch.int32, device=dev)
    keep = [i32(case.tree_off), i32(case.root_token), i32(case.cand_token),
            torch.from_numpy(case.cand_logp).to(dev)]
    p = kdv.make_build_params(batch=case.batch, max_T=max_T, depth=case.depth, topk=case.topk,
                              tree_off=keep[0], root_token=keep[1], cand_token=keep[2],
                              cand_logp=keep[3], parent=out["parent"], token=out["token"],
                              depth_out=out["depth"], score=score, d_err=d_err)
    kdv.kdv_tree_build(p)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res["score"] = score.cpu().numpy()
    return res, int(d_err.item())


def _check(case, max_T=64, expect_err=0):
    got, err = _run(case, max_T)
    assert err == expect_err
    for b in range(case.batch):
        t0, t1 = int(case.tree_off[b]), int(case.tree_off[b + 1])
        want = oracle.tree_build(t1 - t0, int(case.root_token[b]), case.cand_token[b], case.cand_logp[b])
        n = len(want[0])
        np.testing.assert_array_equal(got["parent"][t0:t0 + n], want[0])
        np.testing.assert_array_equal(got["token"][t0:t0 + n], want[1])
        np.testing.assert_array_equal(got["depth"][t0:t0 + n], want[2])
        np.testing.assert_array_equal(got["score"][t0:t0 + n], want[3])
        if n < t1 - t0:
            assert (got["parent"][t0 + n:t1] == -1).all() and (got["token"][t0 + n:t1] == -1).all()
    return got


@pytest.mark.parametrize("budgets", [[32], [13, 32, 64, 1, 16, 9, 48, 2]])
def test_build_block16_budgets(budgets):
    """D = 15 draft positions (block 16), K = 8 candidates, budgets up to 64."""
    _check(datagen.make_build_case(budgets, seed=len(budgets)))


@pytest.mark.parametrize("D,K", [(1, 1), (2, 3), (4, 2), (16, 8), (0, 4)])
def test_build_shapes_with_ties(D, K):
    paths = 1 + sum(K ** d for d in range(1, D + 1))
    case = datagen.make_build_case([min(64, paths), min(7, paths)], D=D, K=K, seed=D * 10 + K,
                                   quantised=True)
    _check(case)


def test_build_budget_beyond_paths_is_reported():
    case = datagen.make_build_case([10, 3], D=3, K=1, seed=2)      # only 4 paths per tree
    _check(case, expect_err=kdv.KDV_DERR_BAD_LENGTH)


def test_build_nan_logprob_reported_and_read_as_minus_inf():
    case = datagen.make_build_case([20], D=4, K=3, seed=5)
    case.cand_logp = case.cand_logp.copy()
    case.cand_logp[0, 1, 2] = np.nan
    _check(case, expect_err=kdv.KDV_DERR_BAD_SCORE)


def test_build_nan_path_score_silent_minus_inf():
    """+inf then -inf on one path: the NaN sum ranks as -inf, not reported."""
    case = datagen.make_build_case([40, 15], D=3, K=2, seed=6)
    case.cand_logp = case.cand_logp.copy()
    case.cand_logp[0, 0, 0] = np.inf
    case.cand_logp[0, 1, 0] = -np.inf
    case.cand_logp[1, 2, 1] = np.inf
    _check(case, expect_err=kdv.KDV_DERR_BAD_LENGTH)   # 15 paths < 40


@pytest.mark.parametrize("value", [0.0, -np.inf, -1.0])
def test_build_all_scores_tied_keys_decide(value):
    """Every candidate with one log-probability: depth-16, K = 8 keys exceed
    32 bits, so the path-key tie-break runs on both halves of the key."""
    case = datagen.make_build_case([64, 64, 33, 5], D=16, K=8, seed=7)
    case.cand_logp = np.full_like(case.cand_logp, value)
    _check(case)


def test_build_full_batch():
    rng = np.random.default_rng(8)
    budgets = [int(x) for x in rng.integers(1, 65, size=kdv.KDV_MAX_BATCH)]
    _check(datagen.make_build_case(budgets, seed=9))
