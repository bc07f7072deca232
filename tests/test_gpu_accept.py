"""GPU parity of kdv_tree_accept against the oracle (bit-exact: integer work).

Greedy tree acceptance (page "The Architecture of Diagnosis", section
"Phase 1: Custom CUDA Kernels", item 3): argmax of the target logits at every
node, the longest accepted path, the bonus token and the in-place page-table
commit. Every output is an integer, so the CUDA path must equal the oracle
exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_tree_verify_mla_b200 import datagen, kdv

pytestmark = pytest.mark.gpu


def _check(case, dc, expect_err=0):
    dc.run()
    got = dc.results()
    want = oracle.accept_case(case)
    assert dc.error_flag() == expect_err
    np.testing.assert_array_equal(got["target"], want["target"])
    np.testing.assert_array_equal(got["len"], want["len"])
    np.testing.assert_array_equal(got["path"], want["path"])
    np.testing.assert_array_equal(got["bonus"], want["bonus"])
    np.testing.assert_array_equal(got["prefix_len_out"], case.prefix_len + want["len"])
    if "page_table" in want:
        np.testing.assert_array_equal(got["page_table"], want["page_table"])
    return got, want


def test_accept_kimi_full_vocab():
    """One Kimi-shape tree (T=13) over the full 163,840-entry vocabulary, bf16."""
    case = datagen.kimi_accept_case()
    _, want = _check(case, kdv.DeviceAcceptCase(case))
    assert want["len"][0] >= 2          # the planted targets make the path non-trivial


def test_accept_batched_paged_commit():
    """Eight requests with the batched verify's trees and page table; commit in place."""
    case = datagen.batched_accept_case()
    got, want = _check(case, kdv.DeviceAcceptCase(case))
    # the committed table is still a permutation of the pool
    assert sorted(got["page_table"].tolist()) == list(range(case.page_table.shape[0]))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("vocab", [1, 37, 8192, 8200, 50021])
def test_accept_vocab_edges(dtype, vocab):
    """Vocabulary sizes around the 8-wide vector groups and the 8192-logit chunks."""
    rng = np.random.default_rng(vocab)
    parents = [datagen.random_tree(int(rng.integers(1, 17)), rng) for _ in range(3)]
    case = datagen.make_accept_case("edge", parents=parents, vocab=vocab, seed=vocab, dtype=dtype,
                                    prefix_len=[3, 0, 11], paged=True)
    _check(case, kdv.DeviceAcceptCase(case))


def test_accept_ties_nan_and_duplicate_siblings():
    rng = np.random.default_rng(21)
    parents = [datagen.random_tree(16, rng) for _ in range(6)] + [datagen.star_tree(9),
                                                                 datagen.chain_tree(12)]
    case = datagen.make_accept_case("ties", parents=parents, vocab=4099, seed=21, ties=True,
                                    nan_rows=5, sibling_dups=True, prefix_len=list(range(8)),
                                    paged=True)
    assert np.isnan(case.logits).all(axis=1).any()      # one row is all NaN -> target 0
    _check(case, kdv.DeviceAcceptCase(case))


def test_accept_given_targets_and_forests():
    """target_in instead of logits; forests (several roots), T=1 and T=64 trees."""
    rng = np.random.default_rng(5)
    forest = datagen.random_tree(20, rng)
    forest[[4, 9, 15]] = -1
    parents = [forest, np.array([-1], dtype=np.int32), datagen.random_tree(64, rng, max_depth=63)]
    case = datagen.make_accept_case("given", parents=parents, vocab=300, seed=5,
                                    with_logits=False, p_follow=0.95, prefix_len=[7, 1, 40],
                                    paged=True)
    assert case.logits is None and case.max_T == 64
    _check(case, kdv.DeviceAcceptCase(case))


def test_accept_scalar_path_for_unaligned_rows():
    """Logits rows that are not 16-byte multiples take the scalar path."""
    case = datagen.make_accept_case("pad", parents=[datagen.random_tree(13, np.random.default_rng(2))],
                                    vocab=1001, seed=2)
    dc = kdv.DeviceAcceptCase(case)
    padded = torch.zeros(case.total_nodes, 1003, dtype=torch.bfloat16, device="cuda")
    padded[:, :1001] = dc.logits
    dc.logits_padded = padded
    dc.params.logits = padded.data_ptr()
    dc.params.logits_ld = 1003
    _check(case, dc)


def test_accept_bad_parent_flags_only_that_request():
    parents = [datagen.random_tree(8, np.random.default_rng(1)), datagen.chain_tree(6)]
    case = datagen.make_accept_case("bad", parents=parents, vocab=512, seed=3, prefix_len=[2, 4],
                                    paged=True)
    good = datagen.make_accept_case("bad", parents=parents, vocab=512, seed=3, prefix_len=[2, 4],
                                    paged=True)
    case.parent = case.parent.copy()
    case.parent[8 + 3] = 5                       # request 1, node 3: parent after itself
    dc = kdv.DeviceAcceptCase(case)
    dc.run()
    got = dc.results()
    assert dc.error_flag() == kdv.KDV_DERR_BAD_PARENT
    assert got["len"][1] == 0 and got["bonus"][1] == -1 and (got["path"][1] == -1).all()
    np.testing.assert_array_equal(got["page_table"][good.kv_off[1]:], good.page_table[good.kv_off[1]:])
    want = oracle.accept_case(good)
    assert got["len"][0] == want["len"][0]
    np.testing.assert_array_equal(got["path"][0], want["path"][0])
    np.testing.assert_array_equal(got["page_table"][:good.kv_off[1]], want["page_table"][:good.kv_off[1]])
