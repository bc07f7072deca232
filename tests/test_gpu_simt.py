"""GPU parity of the mask-build, SIMT verify and combine kernels vs the oracle.

All calls go through the C ABI (libkdv.so via the ctypes binding)."""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from speculative_tree_verify_mla_b200 import datagen, kdv
from tests.parity import assert_parity, parity_stats

pytestmark = pytest.mark.gpu


def _all_trees(T):
    ranges = [[-1]] + [list(range(-1, i)) for i in range(1, T)]
    return [np.array(c, dtype=np.int32) for c in itertools.product(*ranges)]


# ---------------------------------------------------------------------------
# mask build: bit-exact
# ---------------------------------------------------------------------------
def test_mask_build_all_small_trees_bit_exact():
    trees = [t for T in range(1, 7) for t in _all_trees(T)]
    trees += [datagen.random_tree(T, np.random.default_rng(T)) for T in (9, 13, 15, 16, 33, 64)]
    trees += [datagen.chain_tree(64), datagen.star_tree(64)]
    for start in range(0, len(trees), 120):          # batch of <= 120 trees per call
        chunk = trees[start:start + 120]
        parent = np.concatenate(chunk)
        off = np.zeros(len(chunk) + 1, dtype=np.int32)
        off[1:] = np.cumsum([len(t) for t in chunk])
        dev = torch.device("cuda")
        p = torch.from_numpy(parent).to(dev)
        o = torch.from_numpy(off).to(dev)
        mask = torch.zeros(len(parent), dtype=torch.int64, device=dev)
        depth = torch.zeros(len(parent), dtype=torch.int32, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        kdv.kdv_tree_mask_build(p, o, len(chunk), 64, mask, depth, err)
        torch.cuda.synchronize()
        assert err.item() == 0
        got = mask.cpu().numpy().view(np.uint64)
        got_d = depth.cpu().numpy()
        for i, t in enumerate(chunk):
            ref, ref_d = oracle.tree_mask(t)
            assert np.array_equal(got[off[i]:off[i + 1]], ref), t
            assert np.array_equal(got_d[off[i]:off[i + 1]], ref_d), t


def test_mask_build_flags_malformed_parent():
    dev = torch.device("cuda")
    parent = torch.tensor([-1, 0, 2, 1], dtype=torch.int32, device=dev)    # node 2 -> itself
    mask = torch.full((4,), 7, dtype=torch.int64, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    kdv.kdv_tree_mask_build(parent, None, 1, 4, mask, None, err)
    torch.cuda.synchronize()
    assert err.item() == kdv.KDV_DERR_BAD_PARENT
    m = mask.cpu().numpy()
    assert m[0] == 1 and m[1] == 3 and m[2] == 0


# ---------------------------------------------------------------------------
# SIMT verify
# ---------------------------------------------------------------------------
def test_tiny_fp32_case_simt():
    case = datagen.tiny_fp32_case()
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_SIMT, num_splits=1).run()
    o, lse = dc.results()
    o_ref, lse_ref = oracle.verify_case(case)
    st = assert_parity(o, lse, o_ref, lse_ref, max_tol=1e-5, mean_tol=1e-6, lse_tol=1e-5)
    assert dc.error_flag() == 0, st


@pytest.mark.parametrize("splits", [0, 2, 5])
def test_tiny_fp32_splits_simt(splits):
    case = datagen.tiny_fp32_case()
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_SIMT, num_splits=splits).run()
    o, lse = dc.results()
    o_ref, lse_ref = oracle.verify_case(case)
    assert_parity(o, lse, o_ref, lse_ref, max_tol=1e-5, mean_tol=1e-6, lse_tol=1e-5)


def test_partials_and_combine_simt():
    """return_partials gives the per-split (o_k, lse_k) of the documented key
    ranges; kdv_combine merges them."""
    case = datagen.make_case("p", H=3, D_c=48, D_r=16, D_n=16, D_v=16, prefix_len=[150],
                             parents=[datagen.random_tree(11, np.random.default_rng(3))],
                             dtype="f32", seed=5)
    S = 4
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_SIMT, num_splits=S, return_partials=True).run()
    o_part, lse_part = dc.results()
    n = 150 + 11
    c = 128 * math.ceil(n / (128 * S))
    for s in range(S):
        lo, hi = min(s * c, n), min((s + 1) * c, n)
        ro, rl = oracle.verify_request(H=3, L=150, parent=case.parent, D_c=48, D_r=16,
                                       scale=case.scale, q=case.q, pool=case.kv, key_lo=lo,
                                       key_hi=hi)
        if hi > lo:
            assert_parity(o_part[s], lse_part[s], ro, rl, max_tol=1e-5, mean_tol=1e-6,
                          lse_tol=1e-5)
        else:
            assert np.all(o_part[s] == 0) and np.all(np.isneginf(lse_part[s]))
    o = torch.empty(case.rows, 48, device="cuda")
    lse = torch.empty(case.rows, device="cuda")
    kdv.kdv_combine(dc.o_part, dc.lse_part, S, case.rows, 48, o, lse)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.verify_case(case)
    assert_parity(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, max_tol=1e-5,
                  mean_tol=1e-6, lse_tol=1e-5)


def test_combine_matches_oracle_combine_with_empty_parts():
    rng = np.random.default_rng(0)
    S, rows, d = 5, 37, 72
    o_part = rng.standard_normal((S, rows, d)).astype(np.float32)
    lse_part = (rng.standard_normal((S, rows)) * 3).astype(np.float32)
    lse_part[1, :] = -np.inf
    lse_part[:, 3] = -np.inf                      # a row with every part empty
    o_ref, l_ref = oracle.combine(o_part, lse_part)
    op = torch.from_numpy(o_part).cuda()
    lp = torch.from_numpy(lse_part).cuda()
    o = torch.empty(rows, d, device="cuda")
    lse = torch.empty(rows, device="cuda")
    kdv.kdv_combine(op, lp, S, rows, d, o, lse)
    torch.cuda.synchronize()
    np.testing.assert_allclose(o.cpu().numpy(), o_ref, rtol=1e-5, atol=1e-5)
    got_l = lse.cpu().numpy()
    assert np.isneginf(got_l[3]) and np.all(o.cpu().numpy()[3] == 0)
    fin = np.isfinite(l_ref)
    np.testing.assert_allclose(got_l[fin], l_ref[fin], rtol=1e-6, atol=1e-5)


def test_bf16_batched_paged_simt():
    parents = [datagen.random_tree(7, np.random.default_rng(1)), datagen.chain_tree(3),
               datagen.star_tree(9)]
    kw = dict(H=5, D_c=128, D_r=32, D_n=64, D_v=64, prefix_len=[300, 0, 77], parents=parents,
              dtype="bf16", seed=8)
    a = datagen.make_case("a", **kw, paged=False)
    b = datagen.make_case("b", **kw, paged=True)
    oa, la = kdv.DeviceCase(a, impl=kdv.KDV_IMPL_SIMT, num_splits=3).run().results()
    ob, lb = kdv.DeviceCase(b, impl=kdv.KDV_IMPL_SIMT, num_splits=3).run().results()
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)      # paging is bit-exact
    o_ref, lse_ref = oracle.verify_case(b)
    assert_parity(ob, lb, o_ref, lse_ref, max_tol=1e-4, mean_tol=1e-5, lse_tol=1e-4)


def test_bad_slot_sets_error_flag():
    case = datagen.make_case("bad", H=2, D_c=32, D_r=8, D_n=8, D_v=8, prefix_len=[20],
                             parents=[datagen.chain_tree(3)], dtype="f32", seed=1, paged=True)
    case.page_table = case.page_table.copy()
    case.page_table[4] = 10_000                   # outside the 23-slot pool
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_SIMT, num_splits=1).run()
    o, lse = dc.results()
    assert dc.error_flag() == kdv.KDV_DERR_BAD_SLOT
    assert np.all(np.isfinite(o))


def test_device_length_mismatch_sets_error_flag():
    case = datagen.make_case("len", H=2, D_c=32, D_r=8, D_n=8, D_v=8, prefix_len=[20],
                             parents=[datagen.chain_tree(3)], dtype="f32", seed=1)
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_SIMT, num_splits=1)
    dc.prefix_len.fill_(19)
    dc.run()
    dc.results()
    assert dc.error_flag() == kdv.KDV_DERR_BAD_LENGTH
