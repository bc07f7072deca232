"""GPU invariants of kdv_verify_attn that need no tolerance.

1. Perturbation: changing node u's query rows and its own KV row leaves the
   output of every node that does not see u (every non-descendant of u)
   bit-identical. A node's visible keys are the prefix plus its ancestors
   and itself (page "The Architecture of Diagnosis", section "Phase 1: Custom
   CUDA Kernels", item 2: the mask follows the tree), so node t's result
   cannot depend on a key it does not see or on another node's query.
2. Rows outside a request: in a contiguous pool, the rows between and after
   the requests' key ranges are never part of any result -- filling them
   with NaN and +-Inf changes no output bit.
3. The fp16 range of the P.V operand: a c_kv value with |x| >= 65536 is
   reported as KDV_DERR_RANGE; the largest bf16 value below it is exact.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from speculative_tree_verify_mla_b200 import datagen, kdv
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


def _sees(parent, t, u):
    """True when node u is node t or one of t's ancestors."""
    while t >= 0:
        if t == u:
            return True
        t = int(parent[t])
    return False


def _results(case, impl, splits):
    dc = kdv.DeviceCase(case, impl=impl, num_splits=splits).run()
    o, lse = dc.results()
    assert dc.error_flag() == 0
    return o, lse


def _perturbed(case, u, rng):
    """Copy of a single-request case with node u's H query rows and its own KV
    row (logical key L + u) replaced by fresh bf16 values."""
    H, L = case.H, int(case.prefix_len[0])
    q = case.q.copy()
    q[u * H:(u + 1) * H] = datagen.bf16_round(rng.standard_normal(q[u * H:(u + 1) * H].shape).astype(np.float32))
    kv = case.kv.copy()
    slot = L + u if case.page_table is None else int(case.page_table[L + u])
    kv[slot] = datagen.bf16_round(rng.standard_normal(kv.shape[1]).astype(np.float32) * 2)
    return dataclasses.replace(case, q=q, kv=kv)


@pytest.mark.parametrize("impl,paged,splits", [
    (kdv.KDV_IMPL_TC, False, 0), (kdv.KDV_IMPL_TC, False, 3), (kdv.KDV_IMPL_TC, True, 0),
    (kdv.KDV_IMPL_TC_STAGED, True, 2), (kdv.KDV_IMPL_SIMT, False, 0)])
def test_perturbing_a_node_leaves_non_descendants_bit_identical(impl, paged, splits):
    T, L, H = 13, 1500, 64
    parent = datagen.random_tree(T, np.random.default_rng(77))
    case = datagen.make_case("pert", **datagen.KIMI, prefix_len=[L], parents=[parent], seed=78, paged=paged)
    o0, l0 = _results(case, impl, splits)
    rng = np.random.default_rng(79)
    checked = 0
    for u in range(T):
        o1, l1 = _results(_perturbed(case, u, rng), impl, splits)
        for t in range(T):
            rows = slice(t * H, (t + 1) * H)
            if _sees(parent, t, u):
                # u's own rows and its descendants' rows do change
                assert not np.array_equal(o0[rows], o1[rows])
                continue
            np.testing.assert_array_equal(o0[rows], o1[rows], err_msg=f"u={u} t={t}")
            np.testing.assert_array_equal(l0[rows], l1[rows], err_msg=f"u={u} t={t}")
            checked += 1
    assert checked > 0


@pytest.mark.parametrize("fill", [np.nan, np.inf, -np.inf])
@pytest.mark.parametrize("splits", [1, 0])
def test_rows_outside_the_requests_never_reach_an_output(fill, splits):
    """Three requests in one contiguous pool with gaps of 1..300 rows between
    and after their key ranges. Gaps of zeros and gaps of `fill` give the
    same bits, finite and at parity with the oracle."""
    parents = [datagen.random_tree(T, np.random.default_rng(T + 40)) for T in (13, 5, 16)]
    base = datagen.make_case("gap", **datagen.KIMI, prefix_len=[700, 129, 2000], parents=parents, seed=41)
    gaps = [1, 131, 300]              # rows after each request (the last one ends the pool)
    n = (base.prefix_len + base.tree_T).astype(np.int64)
    kv_off = np.zeros(4, dtype=np.int32)
    for b in range(3):
        kv_off[b + 1] = kv_off[b] + n[b] + gaps[b]

    def pool(value):
        kv = np.full((int(kv_off[-1]), base.D_q), value, dtype=np.float32)
        for b in range(3):
            kv[kv_off[b]:kv_off[b] + n[b]] = base.kv[base.kv_off[b]:base.kv_off[b] + n[b]]
        return dataclasses.replace(base, kv=kv, kv_off=kv_off)

    clean, dirty = pool(0.0), pool(fill)
    oc, lc = _results(clean, kdv.KDV_IMPL_TC, splits)
    od, ld = _results(dirty, kdv.KDV_IMPL_TC, splits)
    assert np.all(np.isfinite(od)) and np.all(np.isfinite(ld))
    np.testing.assert_array_equal(oc, od)
    np.testing.assert_array_equal(lc, ld)
    o_ref, lse_ref = oracle.verify_case(base)
    assert_parity(od, ld, o_ref, lse_ref)


def test_latent_values_beyond_fp16_are_reported():
    case = datagen.kimi_layer_case(L=600, T=5, seed=17)
    kv = case.kv.copy()
    kv[123, 77] = 65536.0               # first bf16 value fp16 cannot hold
    dc = kdv.DeviceCase(dataclasses.replace(case, kv=kv), impl=kdv.KDV_IMPL_TC, num_splits=0).run()
    dc.results()
    assert dc.error_flag() == kdv.KDV_DERR_RANGE


def test_largest_in_range_latent_value_is_exact():
    """+-65280 (the largest bf16 magnitude below 65536) pass P.V unchanged.
    The queries' q_lat entries on those two dims are zero, so the values
    reach only P.V (Q.K^T is unchanged) and dominate those output columns."""
    case = datagen.kimi_layer_case(L=600, T=5, seed=18)
    kv = case.kv.copy()
    kv[200, 3] = 65280.0
    kv[201, 300] = -65280.0
    q = case.q.copy()
    q[:, [3, 300]] = 0.0
    case = dataclasses.replace(case, kv=kv, q=q)
    o, lse = _results(case, kdv.KDV_IMPL_TC, 0)
    o_ref, lse_ref = oracle.verify_case(case)
    big = [3, 300]
    rest = [c for c in range(case.D_c) if c not in big]
    assert_parity(o[:, rest], lse, o_ref[:, rest], lse_ref)
    # the two large columns: each weight's fp16 rounding (2^-11 relative)
    # bounds the relative error; 1e-3 absolute covers the unit-scale rest
    np.testing.assert_allclose(o[:, big], o_ref[:, big], rtol=2e-3, atol=1e-3)
    assert np.abs(o_ref[:, big]).max() > 1e3
