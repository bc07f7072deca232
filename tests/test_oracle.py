"""Pins for the CPU oracle: it is checked against things other than itself.

* hand-derived masks (tests/golden), and brute force over every discovery-
  ordered parent[] with T <= 6 against a transitive closure computed by
  boolean matrix products (a different algorithm from the parent walk);
* torch's scaled_dot_product_attention (fp64, CPU) with an explicit boolean
  mask built from that closure, for chain, star, forest and random trees,
  decode (T=1) and no-prefix (L=0) special cases;
* absorbed == non-absorbed MLA on tiny shapes (rel err <= 1e-12);
* closed form q = 0: o = mean of visible c_kv rows, lse = ln |V(t)|;
* perturbing node u leaves every non-descendant bit-identical;
* split invariance of the log-sum-exp combine;
* page-table addressing of a permuted pool is bit-identical to contiguous.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from speculative_tree_verify_mla_b200 import datagen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# independent helpers (no oracle code)
# --------------------------------------------------------------------------
def closure_masks(parent):
    """Ancestor-or-self relation by repeated boolean squaring of the
    child->parent adjacency matrix (reflexive-transitive closure)."""
    T = len(parent)
    A = np.eye(T, dtype=bool)
    for i, p in enumerate(parent):
        if p >= 0:
            A[i, p] = True
    R = A.copy()
    for _ in range(max(1, math.ceil(math.log2(max(T, 2)))) + 1):
        R = R | ((R.astype(np.int64) @ R.astype(np.int64)) > 0)
    masks = np.zeros(T, dtype=np.uint64)
    for t in range(T):
        for u in range(T):
            if R[t, u]:
                masks[t] |= np.uint64(1) << np.uint64(u)
    return R, masks


def all_parent_arrays(T):
    ranges = [[-1]] + [list(range(-1, i)) for i in range(1, T)]
    for combo in itertools.product(*ranges):
        yield np.array(combo, dtype=np.int32)


def sdpa_reference(case, b=0):
    """torch SDPA (float64) per head with an explicit visibility mask from
    the closure. Returns (o [T*H][D_c], lse [T*H]); lse from p and s_0."""
    H, D_c = case.H, case.D_c
    t0, t1 = int(case.tree_off[b]), int(case.tree_off[b + 1])
    T, L = t1 - t0, int(case.prefix_len[b])
    k0, k1 = int(case.kv_off[b]), int(case.kv_off[b + 1])
    idx = case.page_table[k0:k1] if case.page_table is not None else np.arange(k0, k1)
    K = torch.from_numpy(case.kv[idx].astype(np.float64))           # [L+T, D_q]
    V = K[:, :D_c]
    R, _ = closure_masks(case.parent[t0:t1])
    vis = torch.zeros(T, L + T, dtype=torch.bool)
    vis[:, :L] = True
    vis[:, L:] = torch.from_numpy(R)
    q = torch.from_numpy(case.q[t0 * H:t1 * H].astype(np.float64)).view(T, H, -1)
    o = torch.empty(T, H, D_c, dtype=torch.float64)
    lse = torch.empty(T, H, dtype=torch.float64)
    eye = torch.eye(L + T, dtype=torch.float64)
    for h in range(H):
        qh = q[:, h, :]
        o[:, h] = torch.nn.functional.scaled_dot_product_attention(
            qh[None, None], K[None, None], V[None, None], attn_mask=vis[None, None],
            scale=case.scale)[0, 0]
        p = torch.nn.functional.scaled_dot_product_attention(
            qh[None, None], K[None, None], eye[None, None], attn_mask=vis[None, None],
            scale=case.scale)[0, 0]                                      # [T, L+T]
        # key 0 is visible to every row when L > 0, else the root (key L) is
        j0 = 0 if L > 0 else L
        s0 = case.scale * (qh @ K[j0])
        lse[:, h] = s0 - torch.log(p[:, j0])
    return o.reshape(T * H, D_c).numpy(), lse.reshape(T * H).numpy()


def small_case(parents, L, H=3, D_c=16, D_r=8, seed=11, paged=False, dtype="f32"):
    return datagen.make_case("small", H=H, D_c=D_c, D_r=D_r, D_n=8, D_v=8,
                             prefix_len=L if isinstance(L, list) else [L],
                             parents=parents, dtype=dtype, seed=seed, paged=paged)


# --------------------------------------------------------------------------
# mask
# --------------------------------------------------------------------------
def test_mask_golden_tiny_tree():
    rows = np.loadtxt(os.path.join(GOLDEN, "tiny_tree_mask.txt"), dtype=np.int64, comments="#")
    parent = rows[:, 1].astype(np.int32)
    mask, depth = oracle.tree_mask(parent)
    assert mask.tolist() == rows[:, 2].tolist()
    assert depth.tolist() == rows[:, 3].tolist()


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 6])
def test_mask_brute_force_all_trees(T):
    n = 0
    for parent in all_parent_arrays(T):
        mask, depth = oracle.tree_mask(parent)
        R, ref = closure_masks(parent)
        assert np.array_equal(mask, ref), parent
        assert np.array_equal(depth, R.sum(axis=1) - 1), parent
        n += 1
    assert n == math.factorial(T)


def test_mask_rejects_malformed():
    for bad in ([0], [-1, 1], [-1, 2, 0], [-1, -5]):
        with pytest.raises(ValueError):
            oracle.tree_mask(np.array(bad, dtype=np.int32))
    # 64 nodes is the largest supported tree; 65 is rejected
    oracle.tree_mask(datagen.chain_tree(64))
    with pytest.raises(ValueError):
        oracle.tree_mask(datagen.chain_tree(65))


def test_mask_chain_64_top_bit():
    mask, depth = oracle.tree_mask(datagen.chain_tree(64))
    assert int(mask[63]) == (1 << 64) - 1
    assert depth[63] == 63


# --------------------------------------------------------------------------
# attention vs torch SDPA with an independently built mask
# --------------------------------------------------------------------------
@pytest.mark.parametrize("name,parent,L", [
    ("chain", datagen.chain_tree(6), 9),
    ("star", datagen.star_tree(5), 7),
    ("forest", np.array([-1, 0, -1, 2, 1, 3], dtype=np.int32), 4),
    ("decode_T1", np.array([-1], dtype=np.int32), 12),
    ("no_prefix", np.array([-1, 0, 1, 0], dtype=np.int32), 0),
    ("random", datagen.random_tree(9, np.random.default_rng(5)), 13),
])
def test_oracle_matches_sdpa(name, parent, L):
    case = small_case([parent], L)
    o, lse = oracle.verify_case(case)
    o_ref, lse_ref = sdpa_reference(case)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-11, atol=1e-11)


def test_chain_equals_causal_attention():
    """A chain tree is ordinary causal attention over L+T keys with queries
    at positions L..L+T-1 (is_causal with the prefix prepended)."""
    L, T, H = 10, 7, 2
    case = small_case([datagen.chain_tree(T)], L, H=H)
    o, _ = oracle.verify_case(case)
    K = torch.from_numpy(case.kv[:L + T].astype(np.float64))
    q = torch.from_numpy(case.q.astype(np.float64)).view(T, H, -1)
    for h in range(H):
        causal = torch.ones(T, L + T, dtype=torch.bool).tril(diagonal=L)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[None, None, :, h], K[None, None], K[None, None, :, :case.D_c],
            attn_mask=causal[None, None], scale=case.scale)[0, 0]
        np.testing.assert_allclose(o.reshape(T, H, -1)[:, h], ref.numpy(), rtol=1e-11, atol=1e-12)


def test_batched_requests_are_independent():
    parents = [datagen.random_tree(5, np.random.default_rng(1)), datagen.chain_tree(3)]
    case = small_case(parents, [6, 11], seed=3)
    o, lse = oracle.verify_case(case)
    for b in range(2):
        o_ref, lse_ref = sdpa_reference(case, b)
        rows = list(case.request_rows(b))
        np.testing.assert_allclose(o[rows], o_ref, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[rows], lse_ref, rtol=1e-11, atol=1e-11)


# --------------------------------------------------------------------------
# absorption
# --------------------------------------------------------------------------
@pytest.mark.parametrize("dims", [dict(H=4, D_c=64, D_r=16, D_n=32, D_v=32),
                                  dict(H=2, D_c=512, D_r=64, D_n=128, D_v=128)])
def test_absorbed_equals_non_absorbed(dims):
    rng = np.random.default_rng(7)
    H, D_c, D_r, D_n, D_v = dims["H"], dims["D_c"], dims["D_r"], dims["D_n"], dims["D_v"]
    T, L = 5, 9
    parent = np.array([-1, 0, 0, 1, 1], dtype=np.int32)
    c_kv = rng.standard_normal((L + T, D_c)).astype(np.float32)
    k_rope = rng.standard_normal((L + T, D_r)).astype(np.float32)
    q_nope = rng.standard_normal((T * H, D_n)).astype(np.float32)
    q_rope = rng.standard_normal((T * H, D_r)).astype(np.float32)
    w_uk = (rng.standard_normal((H, D_c, D_n)) / math.sqrt(D_c)).astype(np.float32)
    w_uv = (rng.standard_normal((H, D_c, D_v)) / math.sqrt(D_c)).astype(np.float32)
    scale = 1 / math.sqrt(D_n + D_r)
    out_ref, lse_ref = oracle.verify_mla(H=H, L=L, parent=parent, D_c=D_c, D_r=D_r, D_n=D_n,
                                         D_v=D_v, scale=scale, q_nope=q_nope, q_rope=q_rope,
                                         c_kv=c_kv, k_rope=k_rope, w_uk=w_uk, w_uv=w_uv)
    # absorbed route: the kernel-level routine reads float32 storage, so
    # q_lat is rounded to float32 (relative 6e-8) before it; the exact-fp64
    # comparison is the next test.
    q_lat = oracle.absorb_q(H, q_nope, w_uk)
    q_lat32 = q_lat.astype(np.float32)
    q = np.concatenate([q_lat32, q_rope], axis=1)
    pool = np.concatenate([c_kv, k_rope], axis=1)
    o_lat, lse = oracle.verify_request(H=H, L=L, parent=parent, D_c=D_c, D_r=D_r, scale=scale,
                                       q=q, pool=pool)
    out = oracle.unabsorb_o(H, o_lat, w_uv)
    np.testing.assert_allclose(out, out_ref, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-5, atol=1e-6)


def test_absorbed_equals_non_absorbed_exact():
    """With W_UK chosen so that q_lat is exactly representable in float32
    (small-integer weights and queries), both routes agree to 1e-12."""
    rng = np.random.default_rng(8)
    H, D_c, D_r, D_n, D_v, T, L = 3, 32, 8, 16, 12, 4, 6
    parent = np.array([-1, 0, 1, 0], dtype=np.int32)
    c_kv = (rng.integers(-4, 5, (L + T, D_c)) / 8).astype(np.float32)
    k_rope = (rng.integers(-4, 5, (L + T, D_r)) / 8).astype(np.float32)
    q_nope = (rng.integers(-3, 4, (T * H, D_n)) / 4).astype(np.float32)
    q_rope = (rng.integers(-3, 4, (T * H, D_r)) / 4).astype(np.float32)
    w_uk = (rng.integers(-2, 3, (H, D_c, D_n)) / 16).astype(np.float32)
    w_uv = (rng.integers(-2, 3, (H, D_c, D_v)) / 16).astype(np.float32)
    scale = 1 / math.sqrt(D_n + D_r)
    out_ref, lse_ref = oracle.verify_mla(H=H, L=L, parent=parent, D_c=D_c, D_r=D_r, D_n=D_n,
                                         D_v=D_v, scale=scale, q_nope=q_nope, q_rope=q_rope,
                                         c_kv=c_kv, k_rope=k_rope, w_uk=w_uk, w_uv=w_uv)
    q_lat = oracle.absorb_q(H, q_nope, w_uk)
    assert np.array_equal(q_lat, q_lat.astype(np.float32).astype(np.float64))
    q = np.concatenate([q_lat.astype(np.float32), q_rope], axis=1)
    pool = np.concatenate([c_kv, k_rope], axis=1)
    o_lat, lse = oracle.verify_request(H=H, L=L, parent=parent, D_c=D_c, D_r=D_r, scale=scale,
                                       q=q, pool=pool)
    out = oracle.unabsorb_o(H, o_lat, w_uv)
    np.testing.assert_allclose(out, out_ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_absorb_unabsorb_match_einsum():
    rng = np.random.default_rng(9)
    H, D_c, D_n, D_v, rows = 4, 24, 8, 6, 4 * 3
    q_nope = rng.standard_normal((rows, D_n)).astype(np.float32)
    w_uk = rng.standard_normal((H, D_c, D_n)).astype(np.float32)
    w_uv = rng.standard_normal((H, D_c, D_v)).astype(np.float32)
    o_lat = rng.standard_normal((rows, D_c))
    ql = oracle.absorb_q(H, q_nope, w_uk)
    ref = np.einsum("thn,hcn->thc", q_nope.astype(np.float64).reshape(-1, H, D_n),
                    w_uk.astype(np.float64)).reshape(rows, D_c)
    np.testing.assert_allclose(ql, ref, rtol=1e-12, atol=1e-12)
    out = oracle.unabsorb_o(H, o_lat, w_uv)
    ref2 = np.einsum("thc,hcv->thv", o_lat.reshape(-1, H, D_c),
                     w_uv.astype(np.float64)).reshape(rows, D_v)
    np.testing.assert_allclose(out, ref2, rtol=1e-12, atol=1e-12)


def test_projections_one_hot_select_weight_columns():
    """Closed forms of the per-head projections (node-major rows, head =
    row % H): a one-hot q_nope at k makes q_lat the k-th column of W_UK[h];
    a one-hot o_lat at d makes the output the d-th row of W_UV[h]. A
    transposed weight or a node-major/head-major mix-up fails this."""
    rng = np.random.default_rng(11)
    H, D_c, D_n, D_v, T = 3, 10, 4, 5, 4
    rows = T * H
    w_uk = rng.standard_normal((H, D_c, D_n)).astype(np.float32)
    w_uv = rng.standard_normal((H, D_c, D_v)).astype(np.float32)
    ks = rng.integers(0, D_n, rows)
    ds = rng.integers(0, D_c, rows)
    q_nope = np.zeros((rows, D_n), np.float32)
    q_nope[np.arange(rows), ks] = 1.0
    o_lat = np.zeros((rows, D_c))
    o_lat[np.arange(rows), ds] = 1.0
    ql = oracle.absorb_q(H, q_nope, w_uk)
    out = oracle.unabsorb_o(H, o_lat, w_uv)
    for row in range(rows):
        t, h = divmod(row, H)
        assert np.array_equal(ql[row], w_uk[h][:, ks[row]].astype(np.float64))
        assert np.array_equal(out[row], w_uv[h][ds[row], :].astype(np.float64))


# --------------------------------------------------------------------------
# closed forms and invariants
# --------------------------------------------------------------------------
def test_zero_query_is_uniform_average():
    parent = np.array([-1, 0, 0, 2, 3, 1], dtype=np.int32)
    case = small_case([parent], 17, H=2)
    case.q[:] = 0
    o, lse = oracle.verify_case(case)
    R, _ = closure_masks(parent)
    L, D_c = 17, case.D_c
    for t in range(len(parent)):
        vis = list(range(L)) + [L + u for u in range(len(parent)) if R[t, u]]
        mean = case.kv[vis, :D_c].astype(np.float64).mean(axis=0)
        for h in range(2):
            np.testing.assert_allclose(o[t * 2 + h], mean, rtol=1e-13, atol=1e-14)
            assert abs(lse[t * 2 + h] - math.log(len(vis))) < 1e-13


def test_perturbing_a_node_leaves_non_descendants_bit_identical():
    parent = datagen.random_tree(10, np.random.default_rng(21))
    case = small_case([parent], 8, H=2, seed=4)
    o0, l0 = oracle.verify_case(case)
    R, _ = closure_masks(parent)
    L, H = 8, 2
    for u in range(10):
        c2 = small_case([parent], 8, H=2, seed=4)
        c2.q[u * H:(u + 1) * H] += 3.0
        c2.kv[L + u] *= -2.0
        o1, l1 = oracle.verify_case(c2)
        for t in range(10):
            rows = slice(t * H, (t + 1) * H)
            if not R[t, u]:     # u is not t and not an ancestor of t
                assert np.array_equal(o0[rows], o1[rows]) and np.array_equal(l0[rows], l1[rows])
            else:
                assert not np.array_equal(o0[rows], o1[rows])


@pytest.mark.parametrize("cuts", [[5], [1, 2, 3], [0, 10, 10, 22], [24]])
def test_split_invariance(cuts):
    parent = datagen.random_tree(7, np.random.default_rng(2))
    L = 17
    case = small_case([parent], L, H=2, seed=9)
    o, lse = oracle.verify_case(case)
    bounds = [0] + cuts + [L + 7]
    parts_o, parts_l = [], []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        po, pl = oracle.verify_request(H=2, L=L, parent=parent, D_c=case.D_c, D_r=case.D_r,
                                       scale=case.scale, q=case.q, pool=case.kv,
                                       key_lo=lo, key_hi=hi)
        parts_o.append(po)
        parts_l.append(pl)
    oc, lc = oracle.combine(np.stack(parts_o), np.stack(parts_l))
    np.testing.assert_allclose(oc, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lc, lse, rtol=1e-12, atol=1e-12)


def test_combine_special_cases():
    rng = np.random.default_rng(3)
    o1 = rng.standard_normal((1, 4, 5))
    l1 = rng.standard_normal((1, 4))
    o, l = oracle.combine(o1, l1)
    assert np.array_equal(o, o1[0]) and np.allclose(l, l1[0], rtol=0, atol=1e-15)
    # an empty part (-inf) weighs nothing; all-empty rows give zeros / -inf
    o2 = np.stack([o1[0], np.full((4, 5), 7.0)])
    l2 = np.stack([l1[0], np.full(4, -np.inf)])
    o, l = oracle.combine(o2, l2)
    np.testing.assert_allclose(o, o1[0], rtol=1e-15)
    o, l = oracle.combine(np.zeros((3, 2, 5)), np.full((3, 2), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(l))
    # two equal parts: LSE = lse + ln 2, o = average
    o, l = oracle.combine(np.stack([o1[0], 3 * o1[0]]), np.stack([l1[0], l1[0]]))
    np.testing.assert_allclose(o, 2 * o1[0], rtol=1e-14)
    np.testing.assert_allclose(l, l1[0] + math.log(2), rtol=1e-14)


def test_empty_split_gives_zero_and_neg_inf():
    parent = np.array([-1, 0, 0], dtype=np.int32)
    case = small_case([parent], 4, H=1)
    # keys [5, 6) = tree node 1 only: node 2 does not see it
    o, l = oracle.verify_request(H=1, L=4, parent=parent, D_c=case.D_c, D_r=case.D_r,
                                 scale=case.scale, q=case.q, pool=case.kv, key_lo=5, key_hi=6)
    assert np.all(o[2] == 0) and np.isneginf(l[2])
    assert np.isfinite(l[1]) and np.isneginf(l[0])


def test_paged_pool_bit_identical_to_contiguous():
    parents = [datagen.random_tree(6, np.random.default_rng(4)), datagen.chain_tree(4)]
    a = small_case(parents, [9, 5], seed=6, paged=False)
    b = small_case(parents, [9, 5], seed=6, paged=True)
    assert b.page_table is not None and not np.array_equal(b.kv, a.kv)
    oa, la = oracle.verify_case(a)
    ob, lb = oracle.verify_case(b)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)


def test_row_selection_matches_full():
    case = datagen.make_case("sel", H=4, D_c=32, D_r=8, D_n=8, D_v=8, prefix_len=[20, 3],
                             parents=[datagen.chain_tree(5), datagen.star_tree(4)], seed=2)
    o, l = oracle.verify_case(case)
    rows = np.array([0, 3, 7, 19, 20, 35], dtype=np.int64)
    os_, ls = oracle.verify_case(case, rows=rows)
    assert np.array_equal(os_, o[rows]) and np.array_equal(ls, l[rows])


def test_datagen_bf16_values_are_bf16():
    case = datagen.make_case("b", H=2, D_c=16, D_r=8, D_n=8, D_v=8, prefix_len=[5],
                             parents=[datagen.chain_tree(3)], dtype="bf16", seed=1)
    bits = case.kv.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0)
    bits = case.q.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0)


def test_tree_generator_respects_depth_and_order():
    for s in range(20):
        p = datagen.random_tree(16, np.random.default_rng(s))
        _, depth = oracle.tree_mask(p)
        assert p[0] == -1 and all(p[i] < i for i in range(1, 16))
        assert depth.max() <= 6
