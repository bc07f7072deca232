"""The seeded input recipe (speculative_tree_verify_mla_b200/datagen.py):
shapes, value distributions, determinism and the structure of each workload,
on the CPU. The module holds none of the method's arithmetic; these tests
check that the inputs are what the workloads state."""
import math

import numpy as np
import pytest

import oracle
from speculative_tree_verify_mla_b200 import datagen


def _bf16_exact(a):
    return np.all((np.ascontiguousarray(a, dtype=np.float32).view(np.uint32) & 0xFFFF) == 0)


def test_kimi_layer_shapes_scale_and_distributions():
    c = datagen.kimi_layer_case()
    assert (c.H, c.D_c, c.D_r, c.D_n, c.D_v) == (64, 512, 64, 128, 128)
    assert c.prefix_len.tolist() == [5553] and c.tree_T.tolist() == [13]
    assert c.q.shape == (13 * 64, 576) and c.kv.shape == (5553 + 13, 576)
    assert c.scale == pytest.approx(1 / math.sqrt(192))
    assert c.dtype == "bf16" and _bf16_exact(c.q) and _bf16_exact(c.kv)
    assert c.page_table is None and c.kv_off.tolist() == [0, 5566]
    # c_kv, k_rope ~ N(0,1); q_lat ~ N(0, D_n/D_c); q_rope ~ N(0,1)
    assert np.std(c.kv[:, :512]) == pytest.approx(1.0, rel=0.02)
    assert np.std(c.kv[:, 512:]) == pytest.approx(1.0, rel=0.02)
    assert np.std(c.q[:, :512]) == pytest.approx(math.sqrt(128 / 512), rel=0.02)
    assert np.std(c.q[:, 512:]) == pytest.approx(1.0, rel=0.03)
    assert abs(np.mean(c.kv)) < 0.01
    _, depth = oracle.tree_mask(c.parent)
    assert c.parent[0] == -1 and all(c.parent[i] < i for i in range(1, 13)) and depth.max() <= 6


def test_inputs_are_deterministic_per_seed():
    a = datagen.kimi_layer_case(L=300, T=9)
    b = datagen.kimi_layer_case(L=300, T=9)
    c = datagen.kimi_layer_case(L=300, T=9, seed=2)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.kv, b.kv) and np.array_equal(a.parent, b.parent)
    assert not np.array_equal(a.kv, c.kv) and not np.array_equal(a.q, c.q)


def test_context_sweep_layers_share_the_tree_not_the_kv():
    l0 = datagen.context_sweep_case(1663, 0)
    l1 = datagen.context_sweep_case(1663, 1)
    assert l0.tree_T.tolist() == [15] and l0.prefix_len.tolist() == [1663]
    assert np.array_equal(l0.parent, l1.parent)
    assert not np.array_equal(l0.kv, l1.kv) and not np.array_equal(l0.q, l1.q)
    assert l0.seed == 2000 and l1.seed == 2001


def test_tiny_fp32_case_matches_its_statement():
    c = datagen.tiny_fp32_case()
    assert (c.H, c.D_c, c.D_r, c.D_n, c.D_v) == (4, 64, 16, 32, 32)
    assert c.parent.tolist() == [-1, 0, 0, 1, 1] and c.prefix_len.tolist() == [128]
    assert c.dtype == "f32" and c.scale == pytest.approx(1 / math.sqrt(48))
    assert np.std(c.kv[:, :64]) == pytest.approx(1 / 8, rel=0.1)


def test_paged_pool_is_a_permutation_of_the_logical_rows():
    """Small prefixes so the pool stays tiny; the structure is the one the
    8-request batch uses."""
    c = datagen.batched_paged_case(B=8, lo=16, hi=64)
    n_keys = int(c.kv_off[-1])
    assert np.array_equal(np.sort(c.page_table), np.arange(n_keys))
    assert all(16 <= l <= 64 for l in c.prefix_len) and all(9 <= t <= 16 for t in c.tree_T)
    assert c.kv_off.tolist() == [0] + np.cumsum(c.prefix_len + c.tree_T).tolist()
    # the same requests unpaged: logical key i sits at slot page_table[i]
    flat = datagen.make_case("flat", **datagen.KIMI, prefix_len=c.prefix_len.tolist(),
                             parents=[c.parent[c.tree_off[b]:c.tree_off[b + 1]] for b in range(8)],
                             dtype="bf16", seed=c.seed)
    assert np.array_equal(c.kv[c.page_table], flat.kv)
    assert np.array_equal(c.q, flat.q)


def test_build_case_candidates_are_sorted_log_probabilities():
    c = datagen.make_build_case([32, 5, 64], D=15, K=8, seed=3)
    assert c.tree_off.tolist() == [0, 32, 37, 101] and c.cand_logp.shape == (3, 15, 8)
    assert np.all(c.cand_logp <= 0)
    assert np.all(np.diff(c.cand_logp, axis=2) <= 0)            # descending per position
    assert np.all(np.exp(c.cand_logp.astype(np.float64)).sum(axis=2) < 1.0)
    for b in range(3):
        for d in range(15):
            assert len(set(c.cand_token[b, d].tolist())) == 8
    q = datagen.make_build_case([8], D=4, K=3, seed=1, quantised=True)
    assert np.all(q.cand_logp * 4 == np.round(q.cand_logp * 4))


def test_accept_case_plants_the_target_above_every_draw():
    c = datagen.make_accept_case("a", parents=[datagen.random_tree(13, np.random.default_rng(0))],
                                 vocab=4096, seed=5)
    assert c.logits.shape == (13, 4096) and _bf16_exact(c.logits)
    top = c.logits.max(axis=1)
    assert np.all(top == 16.0) and np.all((c.logits == 16.0).sum(axis=1) == 1)
    # siblings carry distinct draft tokens
    for p in range(13):
        kids = [u for u in range(13) if c.parent[u] == p]
        assert len({int(c.token[u]) for u in kids}) == len(kids)


def test_accept_batch_uses_the_paged_batch_structure():
    a = datagen.batched_accept_case()
    assert a.batch == 8 and a.vocab == datagen.KIMI_VOCAB
    assert all(1024 <= l <= 32768 for l in a.prefix_len)
    assert np.array_equal(np.sort(a.page_table), np.arange(int(a.kv_off[-1])))
