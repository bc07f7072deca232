"""GPU parity of the tensor-core (tcgen05/TMEM/TMA) verify kernel vs the oracle,
through the C ABI. Kimi/DeepSeekV3 latent dims (512 + 64), bf16 inputs, the
2-SM-MMA kernel on 4-CTA clusters."""
import dataclasses
import math

import numpy as np
import pytest

import oracle
from speculative_tree_verify_mla_b200 import datagen, kdv
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


@pytest.fixture
def impl():
    return kdv.KDV_IMPL_TC


def _run(case, impl, splits=1, partials=False):
    dc = kdv.DeviceCase(case, impl=impl, num_splits=splits, return_partials=partials).run()
    out = dc.results()
    assert dc.error_flag() == 0
    return out


@pytest.mark.parametrize("L,T,H", [(700, 13, 64), (0, 5, 64), (1, 1, 64), (63, 2, 64),
                                   (64, 3, 8), (65, 16, 8), (130, 64, 4), (257, 7, 3)])
def test_tc_single_split(L, T, H, impl):
    parents = [datagen.random_tree(T, np.random.default_rng(L + T))]
    case = datagen.make_case("tc", **dict(datagen.KIMI, H=H), prefix_len=[L], parents=parents,
                             seed=L * 7 + T)
    o, lse = _run(case, impl, splits=1)
    o_ref, lse_ref = oracle.verify_case(case)
    assert_parity(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("splits", [0, 3, 7])
def test_tc_splits_merged(splits, impl):
    case = datagen.kimi_layer_case(L=1500, T=13, seed=11)
    o, lse = _run(case, impl, splits=splits)
    o_ref, lse_ref = oracle.verify_case(case)
    assert_parity(o, lse, o_ref, lse_ref)


def test_tc_partials_match_oracle_ranges(impl):
    case = datagen.kimi_layer_case(L=300, T=9, seed=12)
    S = 4
    o_part, lse_part = _run(case, impl, splits=S, partials=True)
    n = 300 + 9
    c = 128 * math.ceil(n / (128 * S))
    for s in range(S):
        lo, hi = min(s * c, n), min((s + 1) * c, n)
        if hi <= lo:
            assert np.all(o_part[s] == 0) and np.all(np.isneginf(lse_part[s]))
            continue
        ro, rl = oracle.verify_request(H=64, L=300, parent=case.parent, D_c=512, D_r=64,
                                       scale=case.scale, q=case.q, pool=case.kv, key_lo=lo,
                                       key_hi=hi)
        assert_parity(o_part[s], lse_part[s], ro, rl)


def test_tc_batched_contiguous(impl):
    parents = [datagen.random_tree(T, np.random.default_rng(T)) for T in (9, 16, 12)]
    case = datagen.make_case("b3", **datagen.KIMI, prefix_len=[1030, 77, 400], parents=parents,
                             seed=21)
    o, lse = _run(case, impl, splits=0)
    o_ref, lse_ref = oracle.verify_case(case)
    assert_parity(o, lse, o_ref, lse_ref)


def test_tc_lazy_rescale_growing_logits(impl):
    """Logits that grow along the keys force the running max up by far more
    than the lazy-rescale threshold several times within one split."""
    case = datagen.kimi_layer_case(L=900, T=6, seed=13)
    ramp = np.linspace(0.2, 3.0, case.kv.shape[0], dtype=np.float32)[:, None]
    case.kv = datagen.bf16_round(case.kv * ramp)
    case = datagen.scaled_case(case, 3.0)
    o, lse = _run(case, impl, splits=1)
    o_ref, lse_ref = oracle.verify_case(case)
    # a sharp softmax: the max error is set by the rounding of the few
    # dominant weights, ~2^-11 * max|v| / RMS(o) ~ 1.5e-3 normalised here
    assert_parity(o, lse, o_ref, lse_ref)


def test_tc_matches_simt_on_same_inputs(impl):
    case = datagen.kimi_layer_case(L=513, T=13, seed=14)
    o1, l1 = _run(case, impl, splits=2)
    o2, l2 = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_SIMT, num_splits=2).run().results()
    assert_parity(o1, l1, o2, l2)


# ---------------------------------------------------------------------------
# Paged KV (page_size 1) on the 2-SM kernel: TMA four-row gathers through the
# page table.

def test_tc_paged_bit_identical_to_contiguous():
    """A random-permutation page table over a permuted pool gives exactly the
    output of the identity layout (same logical key order, same arithmetic)."""
    parents = [datagen.random_tree(T, np.random.default_rng(T + 3)) for T in (13, 9, 16)]
    kw = dict(**datagen.KIMI, prefix_len=[1500, 70, 2049], parents=parents, seed=31)
    a = datagen.make_case("a", **kw, paged=False)
    b = datagen.make_case("b", **kw, paged=True)
    for splits in (1, 0):
        oa, la = _run(a, kdv.KDV_IMPL_TC, splits=splits)
        ob, lb = _run(b, kdv.KDV_IMPL_TC, splits=splits)
        np.testing.assert_array_equal(oa, ob)
        np.testing.assert_array_equal(la, lb)
    o_ref, lse_ref = oracle.verify_case(b)
    assert_parity(ob, lb, o_ref, lse_ref)


@pytest.mark.parametrize("L,T", [(0, 3), (5, 1), (127, 13), (300, 64)])
def test_tc_paged_edges(L, T):
    case = datagen.make_case("pe", **datagen.KIMI, prefix_len=[L],
                             parents=[datagen.random_tree(T, np.random.default_rng(L))], seed=L + 5,
                             paged=True)
    o, lse = _run(case, kdv.KDV_IMPL_TC, splits=0)
    o_ref, lse_ref = oracle.verify_case(case)
    assert_parity(o, lse, o_ref, lse_ref)


def test_tc_paged_bad_slot_reported():
    case = datagen.make_case("bs", **datagen.KIMI, prefix_len=[200],
                             parents=[datagen.chain_tree(4)], seed=9, paged=True)
    case.page_table = case.page_table.copy()
    case.page_table[17] = case.kv.shape[0] + 5          # outside the pool
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_TC, num_splits=1).run()
    dc.results()
    assert dc.error_flag() == kdv.KDV_DERR_BAD_SLOT


def test_tc_auto_stages_a_paged_pool():
    """AUTO reads a paged pool through the staged contiguous copy (its
    workspace covers it), and gives the bits the in-place gathers give."""
    case = datagen.make_case("ap", **datagen.KIMI, prefix_len=[1000],
                             parents=[datagen.chain_tree(3)], seed=2, paged=True)
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_AUTO, num_splits=0)
    dc_st = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_TC_STAGED, num_splits=0)
    dc_tc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_TC, num_splits=0)
    assert dc.ws_bytes == dc_st.ws_bytes > dc_tc.ws_bytes
    o, lse = dc.run().results()
    o2, lse2 = dc_tc.run().results()
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)




# ---------------------------------------------------------------------------
# Paged KV through a staged contiguous copy (KDV_IMPL_TC_STAGED).

def test_tc_staged_equals_gather():
    """Staging in logical order and reading with tiled boxes gives what the
    four-row gathers give, up to the staged path's fp16 Q.K^T over the
    latent dims: exact except for inputs below 2^-14 in magnitude, which fp16
    holds as subnormals (a few fp32 ulps on a small fraction of outputs)."""
    parents = [datagen.random_tree(T, np.random.default_rng(T + 7)) for T in (13, 16, 9)]
    case = datagen.make_case("st", **datagen.KIMI, prefix_len=[2100, 333, 4097], parents=parents,
                             seed=41, paged=True)
    for splits in (0, 1, 3):
        og, lg = _run(case, kdv.KDV_IMPL_TC, splits=splits)
        os_, ls_ = _run(case, kdv.KDV_IMPL_TC_STAGED, splits=splits)
        diff = np.abs(og - os_)
        assert np.count_nonzero(diff) <= 2e-3 * diff.size
        assert diff.max() <= 1e-4 * float(np.sqrt(np.mean(og.astype(np.float64) ** 2)))
        assert np.abs(lg - ls_).max() <= 1e-5
    o_ref, lse_ref = oracle.verify_case(case)
    assert_parity(os_, ls_, o_ref, lse_ref)


def test_tc_staged_bad_slot_reported():
    case = datagen.make_case("sb", **datagen.KIMI, prefix_len=[300], parents=[datagen.chain_tree(5)],
                             seed=3, paged=True)
    case.page_table = case.page_table.copy()
    case.page_table[40] = -3
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_TC_STAGED, num_splits=0).run()
    dc.results()
    assert dc.error_flag() == kdv.KDV_DERR_BAD_SLOT


@pytest.mark.parametrize("value,err", [(-65536.0, kdv.KDV_DERR_RANGE), (65280.0, 0)])
def test_tc_staged_q_lat_range(value, err):
    """The staged path reads q_lat in fp16: a value fp16 cannot hold is
    reported; the largest bf16 magnitude below it is accepted."""
    case = datagen.make_case("sq", **datagen.KIMI, prefix_len=[300], parents=[datagen.chain_tree(5)],
                             seed=4, paged=True)
    q = case.q.copy()
    q[7, 100] = value
    case = dataclasses.replace(case, q=q)
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_TC_STAGED, num_splits=0).run()
    dc.results()
    assert dc.error_flag() == err


def test_tc_staged_without_page_table_is_tc():
    case = datagen.kimi_layer_case(L=900, T=13, seed=5)
    a = _run(case, kdv.KDV_IMPL_TC, splits=0)
    b = _run(case, kdv.KDV_IMPL_TC_STAGED, splits=0)
    np.testing.assert_array_equal(a[0], b[0])
