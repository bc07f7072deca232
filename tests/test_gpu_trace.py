"""The tracing build of the library (include/kdv_trace.h, libkdv_trace.so).

It must compute the same bits as libkdv.so -- the stamps are extra stores,
nothing else -- and its stamps must respect the pipeline's causal order:
within a CTA the stages follow the program, and across the CTAs of a work
item a stage never precedes the one it waits for (the O pair sees a P tile
only after the S pair's softmax saw the S tile it comes from). The tracing
build runs in a child process, since one process loads one of the two
libraries.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

from speculative_tree_verify_mla_b200 import build, datagen, kdv

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
import numpy as np
sys.path.insert(0, {root!r})
from speculative_tree_verify_mla_b200 import datagen, kdv
kdv.use_trace_library()
import torch
case = datagen.kimi_layer_case(L={L}, T=13, seed=5)
dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_AUTO, num_splits={S})
dc.run()
torch.cuda.synchronize()
kdv.kdv_trace_clear()
dc.verify()
o, lse = dc.results()
_, items = kdv.kdv_verify_attn_plan(dc.params)
np.savez({out!r}, o=o, lse=lse, st=kdv.kdv_trace_read(4 * items), err=dc.error_flag())
"""

ST = {name: i for i, name in enumerate(kdv.KDV_TRACE_STAGES)}


@pytest.mark.parametrize("L,S", [(2000, 0), (700, 1)])
def test_trace_build_same_bits_and_causal_stamps(tmp_path, L, S):
    build.build_trace()
    out = str(tmp_path / "trace.npz")
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT, L=L, S=S, out=out)],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    z = np.load(out)
    assert int(z["err"]) == 0
    case = datagen.kimi_layer_case(L=L, T=13, seed=5)
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_AUTO, num_splits=S).run()
    o, lse = dc.results()
    assert dc.error_flag() == 0
    np.testing.assert_array_equal(o.view(np.uint32), z["o"].view(np.uint32))
    np.testing.assert_array_equal(lse.view(np.uint32), z["lse"].view(np.uint32))

    st = z["st"].astype(np.int64)
    n_items = st.shape[0] // 4
    assert n_items >= 1

    def ordered(row, stages):
        seq = [int(row[ST[x]]) for x in stages]
        return all(v > 0 for v in seq) and all(a <= b for a, b in zip(seq, seq[1:]))

    for it in range(n_items):
        s0, s1, o0, o1 = st[4 * it:4 * it + 4]        # S pair (leader first), O pair (leader first)
        for row in (s0, s1):
            assert ordered(row, ["setup", "softmax0 sees S t0", "softmax0 pushed t0", "softmax0 done",
                                 "teardown"]), (it, row)
            assert row[ST["softmax1 done"]] > 0
        assert ordered(s0, ["setup", "S mma t0 issued", "S mma last issued", "teardown"]), (it, s0)
        for row in (o0, o1):
            assert ordered(row, ["setup", "V rows ready"]), (it, row)
            assert ordered(row, ["setup", "O sees P t0", "epilogue start", "epilogue stored", "teardown"]), (it, row)
        assert ordered(o0, ["setup", "PV t0 issued", "PV last issued", "epilogue start", "teardown"]), (it, o0)
        # across the cluster: P tile 0 reaches an O CTA only after its S
        # partner's softmax warp that stamps saw S tile 0 (it pushes after)
        assert s0[ST["softmax0 sees S t0"]] <= o0[ST["O sees P t0"]]
        assert s1[ST["softmax0 sees S t0"]] <= o1[ST["O sees P t0"]]
