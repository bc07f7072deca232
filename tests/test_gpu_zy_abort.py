"""The bounded-wait abort path of the tensor-core verify kernel.

Every wait inside the kernel is bounded; when one runs out the kernel records
KDV_DERR_TIMEOUT, retires the copies and MMAs it has in flight, keeps the
cluster resident until the P tiles still travelling toward an O CTA have
landed, and exits normally. The caller's `wait_limit_ns` shortens the bound
so that legitimate waits run out: here 1 ns, so nearly every wait that does
not succeed on its first probe gives up. The call must end (within seconds),
report the timeout, and leave the context usable: a normal call on the same
stream right after it must pass parity.

(The file name sorts after the other GPU tests and before the no-allocation
test, so a run that stops at the first failure has run the others first.)
"""
import time

import numpy as np
import pytest
import torch

import oracle
from speculative_tree_verify_mla_b200 import datagen, kdv
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("paged", [False, True])
def test_short_wait_limit_times_out_and_context_stays_usable(paged):
    case = datagen.kimi_layer_case(L=1200, T=13, seed=91, paged=paged)
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_TC, num_splits=0)
    dc.params.wait_limit_ns = 1
    t0 = time.time()
    dc.run()
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert dc.error_flag() == kdv.KDV_DERR_TIMEOUT
    assert elapsed < 30.0
    # the same problem again with the default bound, on the same stream
    dc.d_err.zero_()
    dc.params.wait_limit_ns = 0
    o, lse = dc.run().results()
    assert dc.error_flag() == 0
    o_ref, lse_ref = oracle.verify_case(case)
    assert_parity(o, lse, o_ref, lse_ref)
