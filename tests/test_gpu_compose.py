"""On-device composition: tree build -> mask -> verify -> accept (+ page
commit), one stream, captured once in a CUDA graph and replayed with no host
round trip between the steps -- the composition the pages validated with a
chained test (page "The Architecture of Diagnosis", section "Phase 1: Custom
CUDA Kernels": an on-device composition test chained build -> verify ->
accept). Checked against the oracle run step by step on the same inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_tree_verify_mla_b200 import datagen, kdv
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu
dev = "cuda"


def test_build_verify_accept_on_device():
    budgets, prefixes, H = [32, 16], [3000, 1200], 64
    build = datagen.make_build_case(budgets, D=15, K=8, seed=11)
    # verify inputs for the tree slots; they do not depend on the tree's shape
    placeholder = [datagen.chain_tree(T) for T in budgets]
    vcase = datagen.make_case("compose", **datagen.KIMI, prefix_len=prefixes, parents=placeholder,
                              dtype="bf16", seed=12, paged=True)
    # the target model's next token at every node slot: the best candidate at
    # the position numbered like the slot, except every fourth slot, which
    # gets a token no candidate has (an input fixed here, independent of the
    # built tree; best-first builders usually place the top path in the first
    # slots, so some of it is accepted)
    target = np.zeros(sum(budgets), dtype=np.int32)
    for b, T in enumerate(budgets):
        t0 = int(vcase.tree_off[b])
        for t in range(T):
            target[t0 + t] = build.cand_token[b, min(t, 14), 0] if t % 4 != 3 else datagen.KIMI_VOCAB - 1

    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    sumT, B = sum(budgets), len(budgets)
    tree_off, root_token = i32(build.tree_off), i32(build.root_token)
    cand_token, cand_logp = i32(build.cand_token), torch.from_numpy(build.cand_logp).to(dev)
    parent = torch.full((sumT,), -7, dtype=torch.int32, device=dev)
    token = torch.full((sumT,), -7, dtype=torch.int32, device=dev)
    d_err = torch.zeros(1, dtype=torch.int32, device=dev)
    bp = kdv.make_build_params(batch=B, max_T=64, depth=15, topk=8, tree_off=tree_off,
                               root_token=root_token, cand_token=cand_token, cand_logp=cand_logp,
                               parent=parent, token=token, depth_out=None, score=None, d_err=d_err)
    dc = kdv.DeviceCase(vcase, num_splits=0)          # q, paged KV, mask, outputs
    dc.parent = parent                                 # the mask is built from the built tree
    dc.params.d_err = d_err.data_ptr()
    page_table0 = dc.page_table.clone()
    target_d = i32(target)
    acc = {k: torch.full((B,), -7, dtype=torch.int32, device=dev) for k in ("len", "bonus", "plen")}
    path = torch.full((B, 64), -7, dtype=torch.int32, device=dev)
    ap = kdv.make_accept_params(batch=B, max_T=64, total_nodes=sumT, vocab=datagen.KIMI_VOCAB,
                                dtype=kdv.KDV_BF16, logits=None, logits_ld=0, target_in=target_d,
                                token=token, parent=parent, tree_off=dc.tree_off, target_out=None,
                                accept_len=acc["len"], accept_path=path, bonus=acc["bonus"],
                                page_table=dc.page_table, kv_off=dc.kv_off, prefix_len=dc.prefix_len,
                                prefix_len_out=acc["plen"], workspace=None, workspace_bytes=0,
                                d_err=d_err)
    stream = torch.cuda.Stream()

    def step(s):
        kdv.kdv_tree_build(bp, s)
        kdv.kdv_tree_mask_build(parent, dc.tree_off, B, 64, dc.mask, None, d_err, s)
        kdv.kdv_verify_attn(dc.params, s)
        kdv.kdv_tree_accept(ap, s)

    with torch.cuda.stream(stream):
        step(stream)                                   # eager pass: kernel attributes
    stream.synchronize()
    dc.page_table.copy_(page_table0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step(stream)
    dc.page_table.copy_(page_table0)
    parent.fill_(-7)
    dc.o.fill_(float("nan"))
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    assert int(d_err.item()) == 0

    # ---- the oracle, step by step
    want_parent, want_token = [], []
    for b, T in enumerate(budgets):
        p_, t_, _, _ = oracle.tree_build(T, int(build.root_token[b]), build.cand_token[b], build.cand_logp[b])
        want_parent.append(p_)
        want_token.append(t_)
    np.testing.assert_array_equal(parent.cpu().numpy(), np.concatenate(want_parent))
    np.testing.assert_array_equal(token.cpu().numpy(), np.concatenate(want_token))
    for b in range(B):
        m, _ = oracle.tree_mask(want_parent[b])
        t0 = int(vcase.tree_off[b])
        np.testing.assert_array_equal(dc.mask.cpu().numpy()[t0:t0 + budgets[b]].view(np.uint64), m)
    vcase.parent = np.concatenate(want_parent).astype(np.int32)
    o_ref, lse_ref = oracle.verify_case(vcase)
    assert_parity(dc.o.cpu().numpy(), dc.lse.cpu().numpy(), o_ref, lse_ref)
    acase = datagen.AcceptCase(name="compose", vocab=datagen.KIMI_VOCAB, max_T=64, parent=vcase.parent,
                               tree_off=vcase.tree_off, token=np.concatenate(want_token), logits=None,
                               target_in=target, dtype="bf16", prefix_len=vcase.prefix_len,
                               kv_off=vcase.kv_off, page_table=vcase.page_table)
    want = oracle.accept_case(acase)
    np.testing.assert_array_equal(acc["len"].cpu().numpy(), want["len"])
    np.testing.assert_array_equal(acc["bonus"].cpu().numpy(), want["bonus"])
    np.testing.assert_array_equal(path.cpu().numpy()[:, :64], np.pad(want["path"], ((0, 0), (0, 64 - want["path"].shape[1])), constant_values=-1))
    np.testing.assert_array_equal(dc.page_table.cpu().numpy(), want["page_table"])
    np.testing.assert_array_equal(acc["plen"].cpu().numpy(), vcase.prefix_len + want["len"])
    assert want["len"].max() >= 2                       # the chain accepted something
