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
number through the C ABI with host buffers, the CPU oracle as a baseline, and
sub-records for the other configurations -- the 200k-key long context, the
8-request paged batch and the context sweep (L = 13, 1663, 3333, 5553), each
with its own roofline -- plus greedy acceptance, the two projections and the
tree builder.

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
# an earlier measurement on B200s of the same kind: burst bf16 GEMM, the same
# GEMM held for seconds under the 1 kW power cap, and a STREAM-style copy
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
# NVIDIA's dense (no 2:4 sparsity) B200 figures, reported beside the measured ones
DATASHEET_PEAKS = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}


def workload_case(layer: int):
    from speculative_tree_verify_mla_b200 import datagen
    seed = 1 if layer == 0 else 1000 + layer
    return datagen.kimi_layer_case(L=L_PREFIX, T=T_TREE, seed=seed, tree_seed=1)


SWEEP_L = (13, 1663, 3333, 5553)
WORKLOADS = {
    "kimi": "Kimi-shape layer, L=5553, T=13 random tree, NL layers per step",
    "sweep": "context sweep, T=15 shared tree, L in {13, 1663, 3333, 5553}, NL layers per step",
    "long": "L=200,000, T=16, KV ~ N(0,1), one layer per step",
    "paged": "8 requests, L_b ~ U[1024, 32768], T_b ~ U[9, 16], page_size-1 pool through a "
             "random-permutation page table, one batch per step",
}


def workload_cases(name: str, layers: int, rank: int = 0, world: int = 1, L: int = L_PREFIX):
    """The list of verify problems one step runs (one kdv_verify_attn call each)."""
    from speculative_tree_verify_mla_b200 import datagen
    if name == "kimi":
        return [workload_case(rank * 10_000 + l if world > 1 else l) for l in range(layers)]
    if name == "sweep":
        return [datagen.context_sweep_case(L, l + 100 * rank) for l in range(layers)]
    if name == "long":
        return [datagen.long_context_case()]
    if name == "paged":
        return [datagen.batched_paged_case(seed=4 + 1000 * rank)]
    raise ValueError(name)


def workload_name(name: str, L: int = L_PREFIX) -> str:
    return {"kimi": f"kimi_layer_L{L_PREFIX}_T{T_TREE}", "sweep": f"context_sweep_L{L}_T15",
            "long": "long_context_L200000_T16", "paged": "batched_paged_B8"}[name]


def case_flops_bytes(case):
    """Algorithmic work of one verify call: 2176 FLOPs per (row, visible key),
    tree keys counted at their true visible count; 1152 B per KV row read once."""
    flops, kv_bytes = 0.0, 0.0
    for b in range(case.batch):
        t0, t1 = int(case.tree_off[b]), int(case.tree_off[b + 1])
        par, T, L = case.parent[t0:t1], t1 - t0, int(case.prefix_len[b])
        depth = np.zeros(T, dtype=np.int64)      # |Anc*(t)| = depth(t) + 1
        for t in range(1, T):
            depth[t] = depth[par[t]] + 1 if par[t] >= 0 else 0
        flops += case.H * (T * L + int((depth + 1).sum())) * FLOP_PER_ROW_KEY
        kv_bytes += (L + T) * KV_ROW_BYTES
    return float(flops), float(kv_bytes)


def layer_flops_bytes(case):
    return case_flops_bytes(case)


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return {"bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "hbm_gbs": float(pk["hbm_gbs"]), "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


def tensor_fracs(tflops: float, peaks) -> dict:
    """A tensor-bound kernel's rate against the sustained (power-capped)
    measured bf16 peak and against the datasheet's dense bf16 peak."""
    return {"frac_of_sustained": tflops / peaks["bf16_tflops_sustained"],
            "peak_sustained": peaks["bf16_tflops_sustained"],
            "frac_of_datasheet": tflops / DATASHEET_PEAKS["bf16_tflops"],
            "peak_datasheet": DATASHEET_PEAKS["bf16_tflops"]}


TC_KERNEL = {0: ("verify_tc2_kernel", "verify_tc2.cu"), 2: ("verify_tc2_kernel", "verify_tc2.cu"),
             4: ("verify_tc2_kernel", "verify_tc2.cu")}


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


def max_over_ranks(x: float, device) -> float:
    """The largest of every rank's x (device time of the slowest rank); the
    identity on one process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_us_per_call(ms_per_step: float, calls_per_rank: int, world: int) -> float:
    """Whole-job time per verify call: every rank runs calls_per_rank calls in
    a step (weak scaling), the step lasts as long as the slowest rank."""
    return ms_per_step * 1e3 / (calls_per_rank * world)


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
    L_main = args.sweep_L if args.workload == "sweep" else L_PREFIX
    case = workload_cases(args.workload, 1, 0, 1, L_main)[0]
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
        "config": {"workload": workload_name(args.workload, L_main), "H": 64, "d_latent": 512,
                   "d_rope": 64, "prefix_len": [int(x) for x in case.prefix_len],
                   "tree_nodes": [int(x) for x in case.tree_T]},
        "cpu_baseline": {"value": us_per_layer, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n_rows} of {rows_total} query rows of the first call per "
                                   "step, scaled to the whole call"},
        "e2e": {"value": us_per_layer, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------
class Problems:
    """The step's verify problems, resident on the device: one kdv_verify_attn
    call per case (inputs, outputs, workspace), masks shared by cases whose
    trees are identical, and a partials-out twin of every call for timing the
    tensor-core kernel alone (given its fp16 latent rows, prepared once, so
    that the twin launches only the attention kernel)."""

    def __init__(self, cases, impl_code, dev):
        import torch
        from speculative_tree_verify_mla_b200 import kdv
        self.cases = cases
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
        self.d_err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.trees = {}          # tree bytes -> (parent, tree_off, batch, max_T, mask)
        self.q, self.kv, self.o, self.lse, self.ws, self.params, self.tc_params = [], [], [], [], [], [], []
        self.out = []
        self.page_table, self.kv_off, self.tree_off, self.keep = [], [], [], []
        self.splits, self.items = [], []
        self.v16, self.n_keys = [], []
        self.tc = impl_code in (kdv.KDV_IMPL_TC, kdv.KDV_IMPL_TC_STAGED, kdv.KDV_IMPL_AUTO)
        for c in cases:
            key = c.parent.tobytes() + c.tree_off.tobytes()
            if key not in self.trees:
                sumT = int(c.tree_off[-1])
                self.trees[key] = (i32(c.parent), i32(c.tree_off), c.batch, int(max(c.tree_T)),
                                   torch.zeros(sumT, dtype=torch.int64, device=dev))
            mask = self.trees[key][4]
            q = torch.from_numpy(c.q).to(torch.bfloat16).to(dev)
            kv = torch.from_numpy(c.kv).to(torch.bfloat16).to(dev)
            pt = i32(c.page_table) if c.page_table is not None else None
            kv_off, tree_off, plen = i32(c.kv_off), i32(c.tree_off), i32(c.prefix_len)
            # o and lse of a call in one allocation, so that a caller reading
            # its results back to the host needs one copy, not two
            out = torch.empty(c.rows * 513, dtype=torch.float32, device=dev)
            o, lse = out[:c.rows * 512].view(c.rows, 512), out[c.rows * 512:]
            self.out.append(out)
            common = dict(batch=c.batch, num_heads=c.H, d_latent=512, d_rope=64, scale=c.scale,
                          dtype=kdv.KDV_BF16, impl=impl_code, q=q, q_row_stride=576, kv=kv,
                          num_slots=kv.shape[0], page_table=pt, kv_off=kv_off, tree_off=tree_off,
                          prefix_len=plen, h_prefix_len=[int(x) for x in c.prefix_len],
                          h_tree_T=[int(x) for x in c.tree_T], mask=mask, d_err=self.d_err)
            p = kdv.make_params(**common, num_splits=0, return_partials=0, o=o, lse=lse,
                                o_part=None, lse_part=None, workspace=None, workspace_bytes=0)
            nbytes = kdv.kdv_verify_attn_workspace(p)
            ws = torch.empty(max(16, nbytes), dtype=torch.uint8, device=dev)
            p.workspace, p.workspace_bytes = ws.data_ptr(), nbytes
            splits, items = kdv.kdv_verify_attn_plan(p)
            # partials-out twin (uniform S = the largest planned split count)
            S = max(splits)
            o_part = torch.empty(S, c.rows, 512, dtype=torch.float32, device=dev)
            lse_part = torch.empty(S, c.rows, dtype=torch.float32, device=dev)
            tp = kdv.make_params(**common, num_splits=S, return_partials=1, o=None, lse=None,
                                 o_part=o_part, lse_part=lse_part, workspace=None,
                                 workspace_bytes=0)
            n_keys = int((c.prefix_len + c.tree_T).sum())
            v16 = torch.empty(n_keys, 512, dtype=torch.float16, device=dev)
            kdv.kdv_latent_f16(tp, v16)
            tp.v16 = v16.data_ptr()
            self.v16.append(v16)
            self.n_keys.append(n_keys)
            tbytes = kdv.kdv_verify_attn_workspace(tp)       # staged paged rows, if any
            tws = torch.empty(max(16, tbytes), dtype=torch.uint8, device=dev)
            tp.workspace, tp.workspace_bytes = tws.data_ptr(), tbytes
            self.keep += [o_part, lse_part, plen, tws]
            self.q.append(q); self.kv.append(kv); self.o.append(o); self.lse.append(lse)
            self.ws.append(ws); self.params.append(p); self.tc_params.append(tp)
            self.page_table.append(pt); self.kv_off.append(kv_off); self.tree_off.append(tree_off)
            self.splits.append(splits); self.items.append(items)

    def step(self, s):
        from speculative_tree_verify_mla_b200 import kdv
        for parent, tree_off, B, max_T, mask in self.trees.values():
            kdv.kdv_tree_mask_build(parent, tree_off, B, max_T, mask, None, self.d_err, s)
        for p in self.params:
            kdv.kdv_verify_attn(p, s)

    def tc_only(self, s):
        from speculative_tree_verify_mla_b200 import kdv
        for p in self.tc_params:
            kdv.kdv_verify_attn(p, s)

    def latent_only(self, s):
        """The fp16 latent-row pass of every call alone."""
        from speculative_tree_verify_mla_b200 import kdv
        for p, v in zip(self.tc_params, self.v16):
            kdv.kdv_latent_f16(p, v, s)

    def launches_per_step(self):
        # mask builds, then per call: the fp16 latent rows, the attention
        # kernel and, unless that kernel merges its own splits, the merge
        from speculative_tree_verify_mla_b200 import kdv
        return len(self.trees) + sum(kdv.kdv_verify_attn_launches(p) for p in self.params)


def graph_of(fn, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn(stream)
    return g


def replay_us(g, stream, reps):
    """Mean device time of one replay of graph g (CUDA events on `stream`)."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(2):
            g.replay()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / reps


def time_tree_accept(dev, stream, peaks, n_bufs: int = 40, reps: int = 20):
    """Greedy tree acceptance after the Kimi-shape verify (T=13, V=163,840 bf16
    logits): n_bufs distinct cases (n_bufs x 4.26 MB > L2) replayed round
    robin in a CUDA graph; HBM-bound, so reported against the copy bandwidth."""
    import torch
    from speculative_tree_verify_mla_b200 import datagen, kdv
    base = datagen.kimi_accept_case()
    dcs = []
    for i in range(n_bufs):
        dc = kdv.DeviceAcceptCase(base, device=dev, commit=False, update_prefix=False)
        if i:   # a distinct logits buffer per case, same values
            dc.logits = dc.logits.clone()
            dc.params.logits = dc.logits.data_ptr()
        dcs.append(dc)

    def run(s):
        for dc in dcs:
            kdv.kdv_tree_accept(dc.params, s)

    with torch.cuda.stream(stream):
        run(stream)
    stream.synchronize()
    g = graph_of(run, stream)
    us = replay_us(g, stream, reps) / n_bufs
    res = dcs[0].results()
    bytes_ = float(base.total_nodes * base.vocab * 2)
    gbs = bytes_ / (us * 1e-6) / 1e9
    del g
    return {"workload": "kimi_accept_T13_V163840", "us_per_call": us, "launches_per_call": 2,
            "bound": "hbm", "algorithmic_bytes": bytes_, "achieved_gbs": gbs,
            "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
            "accept_len": int(res["len"][0]),
            "timing": f"{n_bufs} distinct logits buffers ({n_bufs * bytes_ / 1e6:.0f} MB > L2), graph replay"}


def time_projections(dev, stream, peaks, n_layers: int = 61, reps: int = 10):
    """q_lat = W_UK q_nope and out = W_UV^T o_lat for the Kimi-shape layer
    (H=64, 512/128/128, T=13): n_layers distinct bf16 weight sets (n_layers x
    16.8 MB > L2), graph-replayed; HBM-bound on the weights."""
    import torch
    from speculative_tree_verify_mla_b200 import datagen, kdv
    case = datagen.kimi_layer_case(L=16, T=T_TREE, seed=1)
    q_nope, w_uk, w_uv = datagen.layer_weights(case)
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16).to(dev)
    qn = bf(q_nope)
    wk0, wv0 = bf(w_uk), bf(w_uv)
    wks = [wk0] + [wk0.clone() for _ in range(n_layers - 1)]
    wvs = [wv0] + [wv0.clone() for _ in range(n_layers - 1)]
    q = torch.zeros(case.rows, 576, dtype=torch.bfloat16, device=dev)
    o_lat = torch.randn(case.rows, 512, device=dev) * 0.05
    out = torch.empty(case.rows, 128, device=dev)

    flag = [0]

    def absorb(s):
        for wk in wks:
            kdv.kdv_absorb_q(case.H, qn, wk, q[:, :512], s, flags=flag[0])

    def unabsorb(s):
        for wv in wvs:
            kdv.kdv_unabsorb_o(case.H, o_lat, wv, out, s, flags=flag[0])

    res = {}
    # the headline figure passes KDV_PROJ_STATIC_WEIGHTS (weights are constant
    # over a step, so each call's weight copies may start while the previous
    # kernel finishes); the plain calls are kept beside it
    for name, fn, wbytes in (("absorb_q_plain", absorb, wk0.numel() * 2),
                             ("unabsorb_o_plain", unabsorb, wv0.numel() * 2),
                             ("absorb_q", absorb, wk0.numel() * 2), ("unabsorb_o", unabsorb, wv0.numel() * 2)):
        flag[0] = 0 if name.endswith("_plain") else kdv.KDV_PROJ_STATIC_WEIGHTS
        with torch.cuda.stream(stream):
            fn(stream)
        stream.synchronize()
        g = graph_of(fn, stream)
        us = replay_us(g, stream, reps) / n_layers
        del g
        gbs = wbytes / (us * 1e-6) / 1e9
        res[name] = {"us_per_layer": us, "weight_bytes": wbytes, "achieved_gbs": gbs,
                     "frac": gbs / peaks["hbm_gbs"]}
    res.update({"bound": "hbm", "peak_gbs": peaks["hbm_gbs"], "workload": f"kimi_proj_T{T_TREE}",
                "flags": "KDV_PROJ_STATIC_WEIGHTS (the _plain records: none)",
                "timing": f"{n_layers} distinct weight sets ({n_layers * 16.8:.0f} MB > L2), graph replay"})
    return res


def time_tree_build(dev, stream, budget: int = 32, n_calls: int = 64, reps: int = 20):
    """Best-first draft-tree construction: D = 15 positions x K = 8 candidates,
    budget 32 (block 16, budget 32), for one request and for a full batch of
    128. n_calls back-to-back launches are captured in one graph so that the
    host's launch rate does not bound the figure; latency-bound."""
    import torch
    from speculative_tree_verify_mla_b200 import datagen, kdv
    res = {"workload": f"build_T{budget}_D15_K8", "bound": "latency", "launches_per_call": 1,
           "timing": f"{n_calls} launches in one graph, graph replay"}
    for batch, key in ((1, "us_per_call"), (kdv.KDV_MAX_BATCH, f"us_per_call_B{kdv.KDV_MAX_BATCH}")):
        case = datagen.make_build_case([budget] * batch, D=15, K=8, seed=3)
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
        keep = [i32(case.tree_off), i32(case.root_token), i32(case.cand_token),
                torch.from_numpy(case.cand_logp).to(dev),
                torch.empty(budget * batch, dtype=torch.int32, device=dev),
                torch.empty(budget * batch, dtype=torch.int32, device=dev)]
        p = kdv.make_build_params(batch=batch, max_T=64, depth=15, topk=8, tree_off=keep[0],
                                  root_token=keep[1], cand_token=keep[2], cand_logp=keep[3],
                                  parent=keep[4], token=keep[5], depth_out=None, score=None, d_err=None)

        def fn(s):
            for _ in range(n_calls):
                kdv.kdv_tree_build(p, s)

        with torch.cuda.stream(stream):
            fn(stream)
        stream.synchronize()
        g = graph_of(fn, stream)
        res[key] = replay_us(g, stream, reps) / n_calls
        del g
    return res


def time_config(name: str, dev, stream, peaks, impl_code: int = 0, reps: int = 20):
    """One of the other verify configurations as a sub-record of the headline
    line: the whole kdv_verify_attn call (kernel + split merge) and the
    tensor-core kernel alone (the partials-out twin, same grid), each from a
    CUDA graph replayed `reps` times, against the roofline of that call.
    Their KV (230 MB for the 200k layer, ~156 MB for the paged batch) exceeds
    the 126 MB L2, so back-to-back replays read it from HBM."""
    import torch
    prob = Problems(workload_cases(name, 1), impl_code, dev)
    with torch.cuda.stream(stream):
        prob.step(stream)
        prob.tc_only(stream)
    stream.synchronize()
    g_step, g_tc = graph_of(prob.step, stream), graph_of(prob.tc_only, stream)
    call_us = replay_us(g_step, stream, reps)
    tc_us = replay_us(g_tc, stream, reps)
    del g_step, g_tc
    err = int(prob.d_err.item())
    c = prob.cases[0]
    flops, kv_bytes = case_flops_bytes(c)
    roof_us = max(flops / (peaks["bf16_tflops"] * 1e12), kv_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e6
    tc_tflops = flops / (tc_us * 1e-6) / 1e12
    return {"workload": workload_name(name), "description": WORKLOADS[name],
            "us_per_call": call_us, "roofline_us": roof_us, "frac_of_roofline": roof_us / call_us,
            "kernel": {"name": TC_KERNEL[impl_code][0], "us_per_launch": tc_us, "achieved_tflops": tc_tflops,
                       "peak_tflops": peaks["bf16_tflops"], "frac": tc_tflops / peaks["bf16_tflops"]},
            "flops_per_call": flops, "kv_bytes_per_call": kv_bytes, "splits": prob.splits[0],
            "grid_items": prob.items[0], "d_err": err,
            "timing": f"CUDA graph of one call, {reps} replays, CUDA events on the launch stream"}


def time_sweep(dev, stream, peaks, n_layers: int = 61, reps: int = 5):
    """The context sweep (T=15, 61 distinct layers per step) at every swept
    prefix length: µs per layer of the whole step from a CUDA graph replay,
    against that layer's roofline."""
    import torch
    res = {"workload": "context_sweep_T15", "layers_per_step": n_layers,
           "timing": f"CUDA graph of the {n_layers}-layer step, {reps} replays"}
    for L in SWEEP_L:
        prob = Problems(workload_cases("sweep", n_layers, L=L), 0, dev)
        with torch.cuda.stream(stream):
            prob.step(stream)
        stream.synchronize()
        g = graph_of(prob.step, stream)
        us = replay_us(g, stream, reps) / n_layers
        del g
        flops, kv_bytes = case_flops_bytes(prob.cases[0])
        roof_us = max(flops / (peaks["bf16_tflops"] * 1e12), kv_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e6
        res[f"L{L}"] = {"us_per_layer": us, "roofline_us": roof_us, "frac_of_roofline": roof_us / us,
                        "splits": prob.splits[0], "d_err": int(prob.d_err.item())}
        del prob
        torch.cuda.empty_cache()
    return res


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
    stream = torch.cuda.Stream(device=dev)
    NL = args.layers if args.workload in ("kimi", "sweep") else 1
    L_main = args.sweep_L if args.workload == "sweep" else L_PREFIX

    # ---- inputs (resident in HBM before timing) ----
    prob = Problems(workload_cases(args.workload, NL, rank, world, L_main), args.impl_code, dev)
    c0 = prob.cases[0]
    with torch.cuda.stream(stream):        # eager warm-up sets kernel attributes
        prob.step(stream)
        prob.tc_only(stream)
    stream.synchronize()
    g_step = graph_of(prob.step, stream)
    g_tc = graph_of(prob.tc_only, stream)
    g_lat = graph_of(prob.latent_only, stream)
    torch.cuda.synchronize()

    sampler = ClockSampler(dev.index if world == 1 else local)
    sampler.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):        # graph replays and events all go on `stream`
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
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), dev)
    if world > 1:
        torch.distributed.barrier()
    ms_per_step = ms_total / args.steps

    # dominant kernel alone (same grid, partials out): per-launch duration
    tc_us = replay_us(g_tc, stream, max(3, min(50, args.steps // 4))) / len(prob.params)
    lat_us = replay_us(g_lat, stream, max(3, min(50, args.steps // 4))) / len(prob.params)
    clocks = sampler.stop()
    assert int(prob.d_err.item()) == 0, f"device error flag {int(prob.d_err.item())}"

    # eager (stream-ordered, no graph) per-call time, for reference
    with torch.cuda.stream(stream):
        e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e4.record(stream)
        for _ in range(3):
            prob.step(stream)
        e5.record(stream)
    torch.cuda.synchronize()
    eager_us = e4.elapsed_time(e5) * 1e3 / (3 * len(prob.params))

    # ---- end to end through the C ABI with host buffers: the step's tree
    # (parent[]), every query row and the tree nodes' own KV rows go up, o and
    # lse come back ----
    pin = lambda t: t.cpu().pin_memory()
    h_parent = [pin(tr[0]) for tr in prob.trees.values()]
    h_q = [pin(q) for q in prob.q]
    up_rows = []                 # per call: (device row view, pinned host copy) of the tree-node KV rows
    for c, kv, pt in zip(prob.cases, prob.kv, prob.page_table):
        rows_c = []
        for b in range(c.batch):
            L, T, k0 = int(c.prefix_len[b]), int(c.tree_T[b]), int(c.kv_off[b])
            if c.page_table is None:
                rows_c.append((kv[k0 + L:k0 + L + T], pin(kv[k0 + L:k0 + L + T])))
            else:
                for u in range(T):
                    slot = int(c.page_table[k0 + L + u])
                    rows_c.append((kv[slot:slot + 1], pin(kv[slot:slot + 1])))
        up_rows.append(rows_c)
    h_out = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in prob.out]   # o then lse
    h2d = (sum(x.numel() * 4 for x in h_parent) + sum(x.numel() * 2 for x in h_q)
           + sum(h.numel() * 2 for rows_c in up_rows for _, h in rows_c))
    d2h = sum(x.numel() * 4 for x in h_out)

    # The step pipelines its copies with the compute the way a serving loop
    # would: every call's inputs go up on a copy stream, each call starts once
    # its own inputs have landed, and its o and lse (one allocation, so one
    # copy) come back on another copy stream while the next call runs. All
    # copies stay inside the timed step.
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_tree = torch.cuda.Event()
    ev_in = [torch.cuda.Event() for _ in prob.params]
    ev_out = [torch.cuda.Event() for _ in prob.params]

    def e2e_step():
        s_in.wait_stream(stream)
        with torch.cuda.stream(s_in):
            for tr, hp in zip(prob.trees.values(), h_parent):
                tr[0].copy_(hp, non_blocking=True)
            ev_tree.record(s_in)
            for l, (q, hq) in enumerate(zip(prob.q, h_q)):
                q.copy_(hq, non_blocking=True)
                for d, h in up_rows[l]:
                    d.copy_(h, non_blocking=True)
                ev_in[l].record(s_in)
        stream.wait_event(ev_tree)
        for parent, tree_off, B, max_T, mask in prob.trees.values():
            kdv.kdv_tree_mask_build(parent, tree_off, B, max_T, mask, None, prob.d_err, stream)
        for l, p in enumerate(prob.params):
            stream.wait_event(ev_in[l])
            kdv.kdv_verify_attn(p, stream)
            ev_out[l].record(stream)
            s_out.wait_event(ev_out[l])
            with torch.cuda.stream(s_out):
                h_out[l].copy_(prob.out[l], non_blocking=True)
        stream.wait_stream(s_out)
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
    e2e_ms = max_over_ranks(e6.elapsed_time(e7) / e2e_steps, dev)

    flops, kv_bytes = case_flops_bytes(c0)
    peaks = load_peaks()
    n_calls = len(prob.params)
    us_per_call = job_us_per_call(ms_per_step, n_calls, world)
    tc_tflops = flops / (tc_us * 1e-6) / 1e12
    kname, ksrc = TC_KERNEL.get(args.impl_code, TC_KERNEL[2])
    traffic = load_traffic(kname, ksrc) if args.workload == "kimi" else None
    roof_us = max(flops / (peaks["bf16_tflops"] * 1e12), kv_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e6
    workload = workload_name(args.workload, L_main)
    if args.workload == "kimi":
        cfg = {"workload": workload, "H": c0.H, "d_latent": 512, "d_rope": 64, "d_nope": 128,
               "d_v": 128, "prefix_len": L_PREFIX, "tree_nodes": int(c0.tree_T[0]),
               "layers_per_step": NL}
    else:
        cfg = {"workload": workload, "description": WORKLOADS[args.workload], "H": c0.H,
               "d_latent": 512, "d_rope": 64, "prefix_len": [int(x) for x in c0.prefix_len],
               "tree_nodes": [int(x) for x in c0.tree_T], "calls_per_step": n_calls}
    step_bytes = n_calls * kv_bytes
    cfg.update({"splits": prob.splits[0], "grid_items": prob.items[0],
                "l2": (f"{n_calls} distinct KV caches ({step_bytes / 1e6:.0f} MB) per step > 126 MB L2"
                       if step_bytes > 126e6 else
                       f"KV {step_bytes / 1e6:.0f} MB per step fits L2: warm-L2 number"),
                "timing": "CUDA graph replay of the step, CUDA events on the launch stream",
                "parallelism": f"replica{world}" if world > 1 else "single"})
    result = {
        "metric": METRIC, "value": us_per_call, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": cfg,
        "tflops_per_layer": flops / (us_per_call * 1e-6) / 1e12,
        "roofline_us_per_layer": roof_us,
        "frac_of_roofline": roof_us / us_per_call,
        "eager_us_per_layer": eager_us,
        "roofline": {"bound": "tensor", "kernel": kname, "achieved": tc_tflops,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tc_tflops / peaks["bf16_tflops"], "traffic": traffic,
                     "us_per_launch": tc_us, "flops_per_launch": flops,
                     "kv_bytes_per_launch": kv_bytes,
                     # what the kernel itself must read: the bf16 rows (its QK^T), the fp16
                     # latent rows (its P.V) and the query rows -- compare with traffic
                     "read_bytes_per_launch": kv_bytes + prob.n_keys[0] * 1024.0 + c0.rows * 1152.0,
                     "peak_source": peaks["source"] + " burst bf16",
                     **tensor_fracs(tc_tflops, peaks)},
        "latent_f16": {"kernel": "latent_f16_kernel", "us_per_call": lat_us, "bound": "hbm",
                       "bytes_per_call": prob.n_keys[0] * 2048.0,
                       "achieved_gbs": prob.n_keys[0] * 2048.0 / (lat_us * 1e-6) / 1e9,
                       "frac": prob.n_keys[0] * 2048.0 / (lat_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                       "note": "bf16 c_kv -> fp16 rows read by the attention kernel's P.V; "
                               "1 KB read + 1 KB written per key; included in value"},
        "e2e": {"value": e2e_ms * 1e3 / n_calls, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": args.steps * prob.launches_per_step(),
        "clocks": clocks,
    }

    # single-GPU sub-records: at N=1 only (under torchrun the other ranks
    # would sit idle in teardown while rank 0 measures them)
    if args.workload == "kimi" and rank == 0 and world == 1 and not args.headline_only:
        result["long_context"] = time_config("long", dev, stream, peaks)
        result["paged"] = time_config("paged", dev, stream, peaks)
        result["context_sweep"] = time_sweep(dev, stream, peaks)
        result["tree_accept"] = time_tree_accept(dev, stream, peaks)
        result["projections"] = time_projections(dev, stream, peaks)
        result["tree_build"] = time_tree_build(dev, stream)

    # ---- CPU oracle on the host cores (rank 0, N=1 only): baseline + spot parity ----
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        dt1, *_ = time_oracle(c0, 16)
        n_rows = int(min(c0.rows, max(16, 15.0 / max(dt1 / 16, 1e-6))))
        dt, rows, o_ref, l_ref = time_oracle(c0, n_rows)
        cpu_us = dt / n_rows * c0.rows * 1e6
        result["cpu_baseline"] = {"value": cpu_us, "unit": UNIT, "cores": os.cpu_count(),
                                  "kind": "oracle",
                                  "sample": f"{n_rows} of {c0.rows} query rows of the first call "
                                            "(fp64, all keys), scaled to the whole call"}
        from tests.parity import parity_stats
        got_o = prob.o[0].cpu().numpy()[rows]
        got_l = prob.lse[0].cpu().numpy()[rows]
        st = parity_stats(got_o, got_l, o_ref, l_ref)
        result["parity_layer0"] = {k: float(f"{v:.3g}") for k, v in st.items()}
    if rank == 0:
        print(json.dumps(result))
    if world > 1:
        del g_step, g_tc, g_lat
        torch.distributed.destroy_process_group()
    return 0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--layers", type=int, default=N_LAYERS_DEFAULT)
    ap.add_argument("--impl", choices=["kdv", "reference"], default="kdv")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=["auto", "tc2", "tc2s", "simt"], default="auto",
                    help="auto (default: what KDV_IMPL_AUTO picks -- the tensor-core kernel, over a "
                         "staged contiguous copy when the pool is paged), tc2 (the tensor-core "
                         "kernel, gathering a paged pool through its page table), tc2s (staged), "
                         "simt (the CUDA-core kernel)")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="kimi",
                    help="kimi (default, the headline): " + WORKLOADS["kimi"] + "; sweep: "
                         + WORKLOADS["sweep"] + " (--sweep-L picks L); long: " + WORKLOADS["long"]
                         + "; paged: " + WORKLOADS["paged"])
    ap.add_argument("--sweep-L", type=int, choices=SWEEP_L, default=5553)
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the sub-records (other configurations, acceptance, projections, builder)")
    args = ap.parse_args(argv)
    args.impl_code = {"auto": 0, "tc2": 2, "tc2s": 4, "simt": 1}[args.kernel]
    args.warmup = max(3, args.warmup)
    return args


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
