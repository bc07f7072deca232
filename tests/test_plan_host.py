"""Host-side invariants of the split-L planner (kdv_verify_attn_plan reads
only host fields, so it runs without a GPU; with no device it plans for the
SM-count fallback). The planner's choice of chunk is a cost model, so these
tests check what every plan must satisfy rather than particular values."""
import ctypes

import pytest

from speculative_tree_verify_mla_b200 import kdv

ROWS_PER_ITEM = {kdv.KDV_IMPL_TC: 256, kdv.KDV_IMPL_TC_STAGED: 256, kdv.KDV_IMPL_SIMT: 8}


def _plan(L, T, H=64, impl=kdv.KDV_IMPL_AUTO, splits=0, dtype=kdv.KDV_BF16):
    B = len(L)
    p = kdv.VerifyParams()
    p.batch, p.num_heads, p.d_latent, p.d_rope, p.scale = B, H, 512, 64, 0.1
    p.dtype, p.impl, p.num_splits = dtype, impl, splits
    hp, ht = (ctypes.c_int32 * B)(*L), (ctypes.c_int32 * B)(*T)
    p.h_prefix_len, p.h_tree_T = hp, ht
    return kdv.kdv_verify_attn_plan(p)


CASES = [([5553], [13]), ([200000], [16]), ([0], [1]), ([13], [15]),
         ([1000, 30000, 5000, 1024, 32768, 7, 0, 12345], [9, 16, 12, 1, 64, 3, 2, 13])]


@pytest.mark.parametrize("impl", sorted(ROWS_PER_ITEM))
@pytest.mark.parametrize("L,T", CASES)
def test_items_are_row_tiles_times_splits(L, T, impl):
    splits, items = _plan(L, T, impl=impl)
    r = ROWS_PER_ITEM[impl]
    assert items == sum(-(-t * 64 // r) * s for t, s in zip(T, splits))


@pytest.mark.parametrize("impl", [kdv.KDV_IMPL_TC, kdv.KDV_IMPL_TC_STAGED])
@pytest.mark.parametrize("L,T", CASES)
def test_splits_bounded_by_two_key_tiles_per_split(L, T, impl):
    """Every split of the tensor-core kernel spans at least two 128-key
    tiles (one request's keys n = L + T), so 1 <= S <= ceil(n / 256)."""
    splits, _ = _plan(L, T, impl=impl)
    for l, t, s in zip(L, T, splits):
        assert 1 <= s <= max(1, -(-(l + t) // 256))


@pytest.mark.parametrize("forced", [1, 3, 17])
def test_forced_split_count_is_used_for_every_request(forced):
    splits, _ = _plan([5553, 100, 40000], [13, 4, 16], splits=forced)
    assert splits == [forced] * 3


def test_splits_never_fall_as_the_prefix_grows():
    prev = 0
    for L in range(0, 300_000, 4999):
        (s,), _ = _plan([L], [16])
        assert s >= prev
        prev = s


def test_plan_rejects_oversized_trees():
    with pytest.raises(RuntimeError):
        _plan([100], [65])


def test_retired_one_sm_variant_is_rejected():
    with pytest.raises(kdv.KdvError) as e:
        _plan([100], [5], impl=kdv.KDV_IMPL_TC_1SM)
    assert e.value.status == kdv.KDV_ERR_UNSUPPORTED
