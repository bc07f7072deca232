#!/usr/bin/env python
"""Benchmark of tree-verify MLA attention (absorbed form) on B200.

Workload: one Kimi/DeepSeekV3-shape attention layer (H=64, kv_lora_rank=512,
qk_rope=64, qk_nope=128, v=128) at prefix L=5553 with a T=13 random
best-first draft tree (depth <= 6), bf16 inputs, fp32 accumulation. One
benchmark step is one verify step over NL independent layers (default 61,
each with its own seeded queries and latent KV cache, all sharing the step's
draft tree): kdv_tree_mask_build once, then kdv_verify_attn per layer
(tensor-core kernel + split merge). The 61 KV caches (391 MB) exceed the
126 MB L2, so each layer reads its KV from HBM. The timed steps replay a CUDA
graph of the step; the metric is microseconds per layer.

Also reported: the dominant kernel's roofline (tensor bound), an end-to-end
number through the C ABI with host buffers, and the CPU oracle as a baseline.

Launch: python bench.py [--gpus N --steps K --warmup W]; for N > 1 under
torchrun, each rank runs its own layers (weak scaling, no collective on the
data path). ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "tree-verify MLA attn µs/layer @5.5k ctx; TFLOP/s and % of roofline"
UNIT = "us"
L_PREFIX, T_TREE, N_LAYERS_DEFAULT = 5553, 13, 61
FLOP_PER_ROW_KEY = 2 * 576 + 2 * 512        # QK^T over 576 dims + PV over 512
KV_ROW_BYTES = 576 * 2
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "verify_tc_traffic.json")
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}


def workload_case(layer: int):
    from speculative_tree_verify_mla_b200 import datagen
    seed = 1 if layer == 0 else 1000 + layer
    return datagen.kimi_layer_case(L=L_PREFIX, T=T_TREE, seed=seed, tree_seed=1)


def layer_flops_bytes(case):
    T, H, L = int(case.tree_T[0]), case.H, int(case.prefix_len[0])
    # |Anc*(t)| = depth(t) + 1, from parent[] (parents precede children)
    depth = np.zeros(T, dtype=np.int64)
    for t in range(1, T):
        depth[t] = depth[case.parent[t]] + 1 if case.parent[t] >= 0 else 0
    visible = H * (T * L + int((depth + 1).sum()))
    return float(visible * FLOP_PER_ROW_KEY), float((L + T) * KV_ROW_BYTES)


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return {"bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "hbm_gbs": float(pk["hbm_gbs"]), "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=FALLBACK_PEAKS["bf16_tflops"], source="fallback")


TC_KERNEL = {2: ("verify_tc2_kernel", "verify_tc2.cu"), 3: ("verify_tc_kernel", "verify_tc.cu")}


def kernel_source_hash(src="verify_tc2.cu"):
    h = hashlib.sha256()
    for fn in (src, "sm100_ptx.cuh", "kdv_internal.cuh"):
        with open(os.path.join(ROOT, "speculative_tree_verify_mla_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel, src):
    """Per-launch DRAM bytes of the TC kernel from the committed ncu summary,
    or None when it was taken on a different kernel or kernel source."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        if t.get("kernel") == kernel and t.get("kernel_source_hash") == kernel_source_hash(src):
            return float(t["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the GPU is busy."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# --------------------------------------------------------------------------
# CPU oracle timing (the baseline leg and the --impl reference arm)
# --------------------------------------------------------------------------
def time_oracle(case, n_rows: int):
    import oracle
    rows = np.linspace(0, case.rows - 1, n_rows).astype(np.int64)
    t0 = time.perf_counter()
    o, lse = oracle.verify_case(case, rows=rows)
    dt = time.perf_counter() - t0
    return dt, rows, o, lse


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    cores = os.cpu_count()
    case = workload_case(0)
    rows_total = case.rows
    # size the per-step sample so the whole run stays within ~2 minutes
    dt1, *_ = time_oracle(case, 32)
    per_row = dt1 / 32
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_rows = int(max(8, min(rows_total, budget / max(per_row, 1e-6))))
    for _ in range(args.warmup):
        time_oracle(case, n_rows)
    times = []
    for _ in range(args.steps):
        dt, *_ = time_oracle(case, n_rows)
        times.append(dt)
    us_per_layer = (sum(times) / len(times)) / n_rows * rows_total * 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": us_per_layer, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": us_per_layer / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"kimi_layer_L{L_PREFIX}_T{T_TREE}", "H": 64, "d_latent": 512,
                   "d_rope": 64, "prefix_len": L_PREFIX, "tree_nodes": T_TREE},
        "cpu_baseline": {"value": us_per_layer, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n_rows} of {rows_total} query rows of layer 0 per step, "
                                   "scaled to a full layer"},
        "e2e": {"value": us_per_layer, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------
def run_gpu(args):
    import torch
    from speculative_tree_verify_mla_b200 import kdv
    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    kdv.load()
    NL = args.layers
    stream = torch.cuda.Stream(device=dev)

    # ---- inputs (resident in HBM before timing) ----
    cases = [workload_case(rank * 10_000 + l if world > 1 else l) for l in range(NL)]
    c0 = cases[0]
    T, H = int(c0.tree_T[0]), c0.H
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    parent = i32(c0.parent)
    tree_off = i32(c0.tree_off)
    kv_off = i32(c0.kv_off)
    prefix_len = i32(c0.prefix_len)
    mask = torch.zeros(T, dtype=torch.int64, device=dev)
    d_err = torch.zeros(1, dtype=torch.int32, device=dev)
    qs, kvs, outs, lses, wss, params, tc_params = [], [], [], [], [], [], []
    common = dict(batch=1, num_heads=H, d_latent=512, d_rope=64, scale=c0.scale, dtype=kdv.KDV_BF16,
                  q_row_stride=576, page_table=None, kv_off=kv_off, tree_off=tree_off,
                  prefix_len=prefix_len, h_prefix_len=[L_PREFIX], h_tree_T=[T], mask=mask,
                  d_err=d_err)
    for c in cases:
        q = torch.from_numpy(c.q).to(torch.bfloat16).to(dev)
        kv = torch.from_numpy(c.kv).to(torch.bfloat16).to(dev)
        o = torch.empty(c.rows, 512, dtype=torch.float32, device=dev)
        lse = torch.empty(c.rows, dtype=torch.float32, device=dev)
        p = kdv.make_params(**common, impl=args.impl_code, q=q, kv=kv, num_slots=kv.shape[0],
                            num_splits=0, return_partials=0, o=o, lse=lse, o_part=None,
                            lse_part=None, workspace=None, workspace_bytes=0)
        nbytes = kdv.kdv_verify_attn_workspace(p)
        ws = torch.empty(max(16, nbytes), dtype=torch.uint8, device=dev)
        p.workspace, p.workspace_bytes = ws.data_ptr(), nbytes
        qs.append(q); kvs.append(kv); outs.append(o); lses.append(lse); wss.append(ws); params.append(p)
    splits, items = kdv.kdv_verify_attn_plan(params[0])
    S = splits[0]
    o_part = torch.empty(S, c0.rows, 512, dtype=torch.float32, device=dev)
    lse_part = torch.empty(S, c0.rows, dtype=torch.float32, device=dev)
    for l, c in enumerate(cases):
        tc_params.append(kdv.make_params(**common, impl=args.impl_code, q=qs[l], kv=kvs[l],
                                         num_slots=kvs[l].shape[0], num_splits=S, return_partials=1,
                                         o=None, lse=None, o_part=o_part, lse_part=lse_part,
                                         workspace=None, workspace_bytes=0))

    def step(s):
        kdv.kdv_tree_mask_build(parent, tree_off, 1, T, mask, None, d_err, s)
        for p in params:
            kdv.kdv_verify_attn(p, s)

    def tc_only(s):
        for p in tc_params:
            kdv.kdv_verify_attn(p, s)

    # eager warm-up (sets kernel attributes), then capture graphs
    with torch.cuda.stream(stream):
        step(stream)
        tc_only(stream)
    stream.synchronize()
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        step(stream)
    g_tc = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_tc, stream=stream):
        tc_only(stream)
    torch.cuda.synchronize()

    sampler = ClockSampler(dev.index if world == 1 else local)
    sampler.start()
    time.sleep(0.3)
    # graph replays and the timing events all go on `stream`
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g_step.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            g_step.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    ms_total = ev0.elapsed_time(ev1)
    if world > 1:
        t = torch.tensor([ms_total], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        torch.distributed.barrier()
        ms_total = float(t.item())
    ms_per_step = ms_total / args.steps

    # dominant kernel alone (same grid, partials out): per-launch duration
    reps = max(3, min(50, args.steps // 4))
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(2):
            g_tc.replay()
        e2.record(stream)
        for _ in range(reps):
            g_tc.replay()
        e3.record(stream)
    torch.cuda.synchronize()
    tc_us = e2.elapsed_time(e3) * 1e3 / (reps * NL)
    clocks = sampler.stop()
    assert int(d_err.item()) == 0, f"device error flag {int(d_err.item())}"

    # eager (stream-ordered, no graph) per-layer time, for reference
    with torch.cuda.stream(stream):
        e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e4.record(stream)
        for _ in range(3):
            step(stream)
        e5.record(stream)
    torch.cuda.synchronize()
    eager_us = e4.elapsed_time(e5) * 1e3 / (3 * NL)

    # ---- end to end through the C ABI with host buffers ----
    pin = lambda t: t.cpu().pin_memory()
    h_parent = pin(parent)
    h_q = [pin(q) for q in qs]
    h_tree_kv = [pin(kv[L_PREFIX:L_PREFIX + T]) for kv in kvs]
    h_o = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    h_l = [torch.empty(l.shape, dtype=l.dtype).pin_memory() for l in lses]
    h2d = h_parent.numel() * 4 + sum(x.numel() * 2 for x in h_q) + sum(x.numel() * 2 for x in h_tree_kv)
    d2h = sum(x.numel() * 4 for x in h_o) + sum(x.numel() * 4 for x in h_l)

    def e2e_step():
        with torch.cuda.stream(stream):
            parent.copy_(h_parent, non_blocking=True)
            for l in range(NL):
                qs[l].copy_(h_q[l], non_blocking=True)
                kvs[l][L_PREFIX:L_PREFIX + T].copy_(h_tree_kv[l], non_blocking=True)
            step(stream)
            for l in range(NL):
                h_o[l].copy_(outs[l], non_blocking=True)
                h_l[l].copy_(lses[l], non_blocking=True)
        stream.synchronize()

    e2e_steps = max(2, min(10, args.steps))
    e2e_step()
    if world > 1:
        torch.distributed.barrier()
    e6, e7 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e6.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e7.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e6.elapsed_time(e7) / e2e_steps
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())

    flops, kv_bytes = layer_flops_bytes(c0)
    peaks = load_peaks()
    us_per_layer = ms_per_step * 1e3 / (NL * world)
    tc_tflops = flops / (tc_us * 1e-6) / 1e12
    kname, ksrc = TC_KERNEL.get(args.impl_code, TC_KERNEL[2])
    traffic = load_traffic(kname, ksrc)
    roof_us = max(flops / (peaks["bf16_tflops"] * 1e12), kv_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e6
    result = {
        "metric": METRIC, "value": us_per_layer, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"kimi_layer_L{L_PREFIX}_T{T_TREE}", "H": H, "d_latent": 512,
                   "d_rope": 64, "d_nope": 128, "d_v": 128, "prefix_len": L_PREFIX,
                   "tree_nodes": T, "layers_per_step": NL, "splits": S, "grid_items": items,
                   "l2": f"{NL} distinct KV caches ({NL * kv_bytes / 1e6:.0f} MB) per step > 126 MB L2",
                   "timing": "CUDA graph replay of the step, CUDA events on the launch stream",
                   "parallelism": f"replica{world}" if world > 1 else "single"},
        "tflops_per_layer": flops / (us_per_layer * 1e-6) / 1e12,
        "roofline_us_per_layer": roof_us,
        "frac_of_roofline": roof_us / us_per_layer,
        "eager_us_per_layer": eager_us,
        "roofline": {"bound": "tensor", "kernel": kname, "achieved": tc_tflops,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tc_tflops / peaks["bf16_tflops"], "traffic": traffic,
                     "us_per_launch": tc_us, "flops_per_launch": flops,
                     "kv_bytes_per_launch": kv_bytes, "peak_source": peaks["source"] + " burst bf16"},
        "e2e": {"value": e2e_ms * 1e3 / NL, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": args.steps * (1 + 2 * NL) if S > 1 else args.steps * (1 + NL),
        "clocks": clocks,
    }

    # ---- CPU oracle on the host cores (rank 0, N=1 only): baseline + spot parity ----
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        dt1, *_ = time_oracle(c0, 64)
        n_rows = int(min(c0.rows, max(64, 15.0 / max(dt1 / 64, 1e-6))))
        dt, rows, o_ref, l_ref = time_oracle(c0, n_rows)
        cpu_us = dt / n_rows * c0.rows * 1e6
        result["cpu_baseline"] = {"value": cpu_us, "unit": UNIT, "cores": os.cpu_count(),
                                  "kind": "oracle",
                                  "sample": f"{n_rows} of {c0.rows} query rows of layer 0 "
                                            "(fp64, all keys), scaled to a full layer"}
        from tests.parity import parity_stats
        got_o = outs[0].cpu().numpy()[rows]
        got_l = lses[0].cpu().numpy()[rows]
        st = parity_stats(got_o, got_l, o_ref, l_ref)
        result["parity_layer0"] = {k: float(f"{v:.3g}") for k, v in st.items()}
    if rank == 0:
        print(json.dumps(result))
    if world > 1:
        del g_step, g_tc
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--layers", type=int, default=N_LAYERS_DEFAULT)
    ap.add_argument("--impl", choices=["kdv", "reference"], default="kdv")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=["tc2", "tc1"], default="tc2",
                    help="tensor-core kernel: 2-SM MMAs (default) or 1-SM MMAs")
    args = ap.parse_args()
    args.impl_code = 2 if args.kernel == "tc2" else 3
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
