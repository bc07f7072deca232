"""Stream ordering through the chain of programmatic-dependent launches.

A verify call launches the fp16 latent-row pass as a programmatic dependent
of whatever kernel precedes it on the stream (it waits for that kernel
before any access), the attention kernel as a dependent of that pass, and
the split merge as a dependent of the attention kernel. A caller's kernel
that writes the pool or the queries right before the call, on the same
stream and with no synchronisation, must therefore be seen by the call:
here torch kernels rewrite q and kv between calls, and every call's output
must equal the oracle on the values just written (and differ from the
previous call's output).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from speculative_tree_verify_mla_b200 import datagen, kdv
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("splits,paged", [(0, False), (1, False), (0, True)])
def test_writes_just_before_a_call_are_seen(splits, paged):
    parents = [datagen.random_tree(13, np.random.default_rng(55))]
    case = datagen.make_case("ord", **datagen.KIMI, prefix_len=[1900], parents=parents, seed=56, paged=paged)
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_AUTO, num_splits=splits)
    dc.build_mask()
    prev = None
    for step in range(3):
        # new inputs written by torch kernels on the call's stream, no sync
        gen = torch.Generator(device="cuda").manual_seed(100 + step)
        dc.q.copy_(torch.randn(dc.q.shape, generator=gen, device="cuda").to(dc.q.dtype))
        dc.kv.copy_(torch.randn(dc.kv.shape, generator=gen, device="cuda").to(dc.kv.dtype))
        kdv.kdv_verify_attn(dc.params)          # the legacy default stream, as torch's kernels
        torch.cuda.synchronize()
        o, lse = dc.results()
        assert dc.error_flag() == 0
        step_case = dataclasses.replace(case, q=dc.q.float().cpu().numpy(), kv=dc.kv.float().cpu().numpy())
        o_ref, lse_ref = oracle.verify_case(step_case)
        assert_parity(o, lse, o_ref, lse_ref)
        if prev is not None:
            assert not np.array_equal(o, prev)
        prev = o.copy()
