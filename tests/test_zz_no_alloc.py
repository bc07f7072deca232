"""kdv_verify_attn_noalloc: verify attention without caller scratch memory.

Callers such as a serving engine that reserved all free device memory for its
KV cache at start-up, or a plug-in whose host framework owns every device
allocation, cannot hand the library a workspace. This entry point keeps the
split partials in a scratch array built into the library instead. These tests
call it through the C ABI and check that it gives what kdv_verify_attn gives
(with a caller workspace) on two calls in a row, the second on different data
so that stale scratch contents from the first call would show up.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from speculative_tree_verify_mla_b200 import datagen, kdv
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


def _noalloc_outputs(dc):
    """Run the no-allocation entry point on a prepared DeviceCase; returns (o, lse)."""
    p = kdv.VerifyParams.from_buffer_copy(dc.params)   # host length arrays stay alive in dc
    p.workspace = None           # the entry point must not need the caller's workspace
    p.workspace_bytes = 0
    o = torch.full_like(dc.o, float("nan"))
    lse = torch.full_like(dc.lse, float("nan"))
    p.o = o.data_ptr()
    p.lse = lse.data_ptr()
    status = kdv.load().kdv_verify_attn_noalloc(ctypes.byref(p), kdv._stream(None))
    assert status == kdv.KDV_OK, kdv.status_string(status)
    torch.cuda.synchronize()
    return o.cpu().numpy(), lse.cpu().numpy()


def test_noalloc_matches_workspace_path_twice():
    cases = [datagen.kimi_layer_case(L=5553, T=13, seed=1),
             datagen.kimi_layer_case(L=3001, T=9, seed=77)]
    for case in cases:
        dc = kdv.DeviceCase(case, num_splits=0)
        assert 0 < dc.ws_bytes <= kdv.KDV_NOALLOC_SCRATCH_BYTES   # the path really uses scratch
        o_ref, lse_ref = dc.run().results()
        assert dc.error_flag() == 0
        o, lse = _noalloc_outputs(dc)
        assert dc.error_flag() == 0
        assert_parity(o, lse, o_ref, lse_ref, max_tol=1e-6, mean_tol=1e-7, lse_tol=1e-6,
                      rel_max_tol=1e-5, rel_mean_tol=1e-6)


def test_noalloc_rejects_plans_beyond_its_scratch():
    case = datagen.kimi_layer_case(L=5553, T=13, seed=1)
    dc = kdv.DeviceCase(case, num_splits=64)        # 64 splits x 832 rows x 2 KB > 16 MiB
    assert dc.ws_bytes > kdv.KDV_NOALLOC_SCRATCH_BYTES
    status = kdv.load().kdv_verify_attn_noalloc(ctypes.byref(dc.params), kdv._stream(None))
    assert status == kdv.KDV_ERR_WORKSPACE
