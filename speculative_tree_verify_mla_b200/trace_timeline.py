"""Stage timeline of the tensor-core verify kernel, from its tracing build.

    python -m speculative_tree_verify_mla_b200.trace_timeline [--workload kimi|long|paged] [--L N]

Loads ``libkdv_trace.so`` (``python speculative_tree_verify_mla_b200/build.py
--trace``, or ``__graft_entry__.build()``), which computes exactly what
``libkdv.so`` computes and in addition has every CTA of the verify kernel
write the global timer at the pipeline stages listed in
``include/kdv_trace.h``. The tool runs one ``kdv_verify_attn`` call of the
chosen workload a few times, clears the stamps, runs it once more and prints,
for every stage, the minimum, median and maximum over the CTAs that reached
it, in microseconds after the earliest setup stamp, and the spread of the
work items' durations. Workloads are the seeded synthetic inputs of the
benchmark: the Kimi-shape layer (H=64, T=13, L=5553 unless --L), the
200,000-key layer, and the 8-request paged batch.
"""
from __future__ import annotations

import argparse
import sys

import numpy as np


def _case(workload: str, L: int):
    from speculative_tree_verify_mla_b200 import datagen
    if workload == "kimi":
        return f"kimi_layer_L{L}_T13", datagen.kimi_layer_case(L=L, T=13, seed=1)
    if workload == "long":
        return "long_context_L200000_T16", datagen.long_context_case()
    if workload == "paged":
        return "batched_paged_B8", datagen.batched_paged_case(seed=4)
    raise ValueError(workload)


def timeline(workload: str = "kimi", L: int = 5553, warm: int = 3) -> str:
    import torch
    from speculative_tree_verify_mla_b200 import kdv
    kdv.use_trace_library()
    kdv.load()
    name, case = _case(workload, L)
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_AUTO, num_splits=0)
    dc.run()
    for _ in range(warm):
        dc.verify()
    torch.cuda.synchronize()
    splits, items = kdv.kdv_verify_attn_plan(dc.params)
    n_ctas = 4 * items
    kdv.kdv_trace_clear()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    dc.verify()
    e1.record()
    torch.cuda.synchronize()
    if dc.error_flag() != 0:
        raise RuntimeError(f"device error flag {dc.error_flag()}")
    st = kdv.kdv_trace_read(n_ctas).astype(np.int64)
    setup = st[:, 0]
    t0 = setup[setup > 0].min()
    lines = [f"workload {name}: {items} work items (splits {splits}), {n_ctas} CTAs "
             f"({min(n_ctas, kdv.KDV_TRACE_CTAS)} traced); call {e0.elapsed_time(e1) * 1e3:.1f} us "
             "(CUDA events around the traced call)",
             f"{'stage':22s} {'CTAs':>5s} {'min':>8s} {'median':>8s} {'max':>8s}   us after the first setup stamp"]
    for slot, stage in enumerate(kdv.KDV_TRACE_STAGES):
        v = st[:, slot]
        v = v[v > 0]
        if len(v) == 0:
            continue
        r = (v - t0) / 1000.0
        lines.append(f"{stage:22s} {len(r):5d} {r.min():8.2f} {np.median(r):8.2f} {r.max():8.2f}")
    n_items = min(items, kdv.KDV_TRACE_CTAS // 4)
    per = st[:4 * n_items].reshape(n_items, 4, kdv.KDV_TRACE_SLOTS)
    start = per[:, :, 0].min(axis=1)
    end = per[:, :, 14].max(axis=1)
    ok = (start > 0) & (end > 0)
    dur = (end[ok] - start[ok]) / 1000.0
    lines.append(f"item duration (first setup -> last teardown stamp of its 4 CTAs): min {dur.min():.2f} "
                 f"median {np.median(dur):.2f} max {dur.max():.2f} us")
    return "\n".join(lines)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", choices=("kimi", "long", "paged"), default="kimi")
    ap.add_argument("--L", type=int, default=5553, help="prefix length of the kimi workload")
    args = ap.parse_args(argv)
    print(timeline(args.workload, args.L))
    return 0


if __name__ == "__main__":
    sys.exit(main())
