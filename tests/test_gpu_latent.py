"""The fp16 latent rows that the tensor-core kernel's P.V reads (kdv_latent_f16).

The kernel runs P.V in fp16 (P rounded to fp16, V re-encoded from the bf16
pool), so every call first writes, for each key it reads, the c_kv part of
the pool row as fp16, in logical key order per request. bf16 -> fp16 is a
plain value conversion (exact for 2^-14 <= |x| < 65536), so the rows must
equal torch's cast of the same bf16 values bit for bit, for a contiguous pool
and through a page table. A caller that already holds those rows passes them
(params.v16) and gets the same bits as a call that converts them itself.
"""
import numpy as np
import pytest
import torch

from speculative_tree_verify_mla_b200 import datagen, kdv

pytestmark = pytest.mark.gpu


def _logical_rows(case):
    """The pool rows each request reads, in logical key order."""
    rows = []
    for b in range(case.batch):
        n = int(case.prefix_len[b]) + int(case.tree_T[b])
        k0 = int(case.kv_off[b])
        idx = np.arange(k0, k0 + n)
        if case.page_table is not None:
            idx = case.page_table[idx]
        rows.append(idx)
    return np.concatenate(rows)


@pytest.mark.parametrize("paged", [False, True])
def test_latent_f16_rows_equal_the_cast(paged):
    parents = [datagen.random_tree(T, np.random.default_rng(T + 60)) for T in (13, 9, 16)]
    case = datagen.make_case("lf", **datagen.KIMI, prefix_len=[1500, 77, 2049], parents=parents, seed=61,
                             paged=paged)
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_TC, num_splits=0)
    n_keys = int((case.prefix_len + case.tree_T).sum())
    v16 = torch.full((n_keys, 512), float("nan"), dtype=torch.float16, device="cuda")
    kdv.kdv_latent_f16(dc.params, v16)
    torch.cuda.synchronize()
    assert dc.error_flag() == 0
    want = dc.kv[torch.from_numpy(_logical_rows(case)).cuda(), :512].to(torch.float16)
    assert torch.equal(v16.view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("impl", [kdv.KDV_IMPL_TC, kdv.KDV_IMPL_TC_STAGED])
@pytest.mark.parametrize("splits", [0, 1])
def test_caller_rows_give_the_same_bits(splits, impl):
    """Also for the staged path, whose Q.K^T then reads the caller's rows for
    the keys' latent dims (the pass still stages k_rope and q_lat)."""
    case = datagen.make_case("lc", **datagen.KIMI, prefix_len=[2300], parents=[datagen.random_tree(13, np.random.default_rng(5))],
                             seed=62, paged=True)
    own = kdv.DeviceCase(case, impl=impl, num_splits=splits).run()
    o1, l1 = own.results()
    mirror = kdv.DeviceCase(case, impl=impl, num_splits=splits)
    v16 = torch.empty(2300 + 13, 512, dtype=torch.float16, device="cuda")
    kdv.kdv_latent_f16(mirror.params, v16)
    mirror.params.v16 = v16.data_ptr()
    assert kdv.kdv_verify_attn_workspace(mirror.params) < own.ws_bytes
    o2, l2 = mirror.run().results()
    assert own.error_flag() == 0 and mirror.error_flag() == 0
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
