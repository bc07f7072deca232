"""Seeded synthetic inputs for tree-verify MLA attention.

This module only draws inputs: random trees (``parent[]`` arrays), latent KV
rows, queries, projection weights, prefix lengths and page tables. It does no
part of the attention arithmetic. Both the CUDA path's tests/bench and the
CPU oracle read the same arrays from here, so the two sides see bit-identical
inputs.

Recipe (all draws use numpy's PCG64 ``default_rng`` on a per-tensor seed
sequence ``[seed, tensor_id, extra...]`` so adding a tensor never shifts
another tensor's values):

* Trees: node 0 is the root (``parent[0] = -1``); node ``i > 0`` picks its
  parent uniformly among earlier nodes whose depth is at most ``max_depth-1``,
  so nodes are in discovery (topological) order and depth <= ``max_depth``.
  This is the plainest reading of a best-first draft tree: the page
  "Architecture of Diagnosis", section "Phase 1: Custom CUDA Kernels", item 1,
  only says the tree is built best-first on the device.
* Latent KV rows are ``c_kv[512] || k_rope[64]`` (576 elements per token; the
  page "From Diagnosis to Deployment", section "The Second Thread", gives
  kv_lora_rank=512 and qk_rope_head_dim=64).
* Activations ~ N(0,1); weights ~ N(0,1)/sqrt(fan_in) with fan_in = D_c.
  The kernel-level query ``q = q_lat || q_rope`` draws q_lat directly from
  N(0, D_n/D_c), the distribution the absorption W_UK . q_nope gives for
  q_nope ~ N(0,1) and W_UK ~ N(0, 1/D_c).
* bf16 configurations round every floating-point input to bf16 with
  round-to-nearest-even; arrays are returned as float32 holding bf16-exact
  values, so fp64 readers and bf16 device copies agree bit for bit.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

# Stable per-tensor stream ids (never renumber: stored fixtures depend on them).
_IDS = {
    "tree": 1, "ckv": 2, "krope": 3, "qlat": 4, "qrope": 5, "qnope": 6,
    "wuk": 7, "wuv": 8, "prefix": 9, "treeT": 10, "perm": 11, "tokens": 12,
    "logits": 13, "misc": 14, "cands": 15,
}


def rng_for(seed: int, name: str, *extra: int) -> np.random.Generator:
    """Independent PCG64 stream for (seed, tensor name, extra ints)."""
    return np.random.default_rng([int(seed), _IDS[name], *[int(e) for e in extra]])


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float data to the bf16 grid (round-to-nearest-even), as float32.

    Uses torch's float32 -> bfloat16 conversion, which rounds to nearest even.
    """
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def random_tree(T: int, rng: np.random.Generator, max_depth: int = 6) -> np.ndarray:
    """parent[] of a random discovery-ordered tree with depth <= max_depth."""
    parent = np.full(T, -1, dtype=np.int32)
    depth = np.zeros(T, dtype=np.int32)
    for i in range(1, T):
        cands = [j for j in range(i) if depth[j] <= max_depth - 1]
        j = int(cands[int(rng.integers(0, len(cands)))])
        parent[i] = j
        depth[i] = depth[j] + 1
    return parent


def chain_tree(T: int) -> np.ndarray:
    """parent = [-1, 0, 1, ..., T-2]: a single draft sequence."""
    return np.arange(-1, T - 1, dtype=np.int32)


def star_tree(T: int) -> np.ndarray:
    """Every non-root node hangs off the root."""
    p = np.zeros(T, dtype=np.int32)
    p[0] = -1
    return p


@dataclasses.dataclass
class VerifyCase:
    """One batched tree-verify problem (kernel-level inputs).

    Rows are node-major: row = (tree_off[b] + t) * H + h.
    Logical key j of request b (0 <= j < L_b + T_b) lives in pool row
    ``page_table[kv_off[b] + j]`` (or ``kv_off[b] + j`` when unpaged);
    key L_b + u holds tree node u's own latent KV row.
    """
    name: str
    H: int
    D_c: int
    D_r: int
    D_n: int
    D_v: int
    scale: float
    dtype: str                      # "bf16" or "f32"
    prefix_len: np.ndarray          # int32 [B]
    tree_T: np.ndarray              # int32 [B]
    parent: np.ndarray              # int32 [sumT], per-request local indices
    tree_off: np.ndarray            # int32 [B+1]
    kv_off: np.ndarray              # int32 [B+1]
    q: np.ndarray                   # float32 [sumT*H, D_c+D_r]
    kv: np.ndarray                  # float32 [num_slots, D_c+D_r]
    page_table: Optional[np.ndarray] = None   # int32 [sum(L+T)] or None
    seed: int = 0

    @property
    def batch(self) -> int:
        return int(self.prefix_len.shape[0])

    @property
    def D_q(self) -> int:
        return self.D_c + self.D_r

    @property
    def rows(self) -> int:
        return int(self.q.shape[0])

    def request_rows(self, b: int) -> range:
        return range(int(self.tree_off[b]) * self.H, int(self.tree_off[b + 1]) * self.H)


def _draw(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return (rng.standard_normal(shape, dtype=np.float64) * std).astype(np.float32)


def make_case(name: str, *, H: int, D_c: int, D_r: int, D_n: int, D_v: int,
              prefix_len: List[int], parents: List[np.ndarray], dtype: str = "bf16",
              seed: int = 0, paged: bool = False, scale: Optional[float] = None,
              kv_std: float = 1.0, krope_std: Optional[float] = None,
              qlat_std: Optional[float] = None, qrope_std: float = 1.0) -> VerifyCase:
    """Build a batched case from explicit prefix lengths and trees."""
    B = len(prefix_len)
    assert len(parents) == B
    tree_T = np.array([len(p) for p in parents], dtype=np.int32)
    plen = np.array(prefix_len, dtype=np.int32)
    tree_off = np.zeros(B + 1, dtype=np.int32)
    tree_off[1:] = np.cumsum(tree_T)
    kv_off = np.zeros(B + 1, dtype=np.int32)
    kv_off[1:] = np.cumsum(plen + tree_T)
    D_q = D_c + D_r
    if scale is None:
        scale = 1.0 / math.sqrt(D_n + D_r)
    if krope_std is None:
        krope_std = kv_std
    if qlat_std is None:
        qlat_std = math.sqrt(D_n / D_c)
    n_keys = int(kv_off[-1])
    sumT = int(tree_off[-1])
    logical = np.empty((n_keys, D_q), dtype=np.float32)
    logical[:, :D_c] = _draw(rng_for(seed, "ckv", n_keys, D_c), (n_keys, D_c), kv_std)
    logical[:, D_c:] = _draw(rng_for(seed, "krope", n_keys, D_r), (n_keys, D_r), krope_std)
    q = np.empty((sumT * H, D_q), dtype=np.float32)
    q[:, :D_c] = _draw(rng_for(seed, "qlat", sumT, H, D_c), (sumT * H, D_c), qlat_std)
    q[:, D_c:] = _draw(rng_for(seed, "qrope", sumT, H, D_r), (sumT * H, D_r), qrope_std)
    if dtype == "bf16":
        logical = bf16_round(logical)
        q = bf16_round(q)
    elif dtype != "f32":
        raise ValueError(dtype)
    page_table = None
    kv = logical
    if paged:
        perm = rng_for(seed, "perm", n_keys).permutation(n_keys).astype(np.int32)
        page_table = perm
        kv = np.empty_like(logical)
        kv[perm] = logical          # logical key i is stored at slot perm[i]
    return VerifyCase(name=name, H=H, D_c=D_c, D_r=D_r, D_n=D_n, D_v=D_v, scale=float(scale),
                      dtype=dtype, prefix_len=plen, tree_T=tree_T,
                      parent=np.concatenate(parents).astype(np.int32), tree_off=tree_off,
                      kv_off=kv_off, q=q, kv=kv, page_table=page_table, seed=seed)


# ---------------------------------------------------------------------------
# The five named workloads.
# ---------------------------------------------------------------------------
KIMI = dict(H=64, D_c=512, D_r=64, D_n=128, D_v=128)
TINY = dict(H=4, D_c=64, D_r=16, D_n=32, D_v=32)
CONTEXT_SWEEP = (13, 1663, 3333, 5553)
N_LAYERS = 61


def tiny_fp32_case() -> VerifyCase:
    """Tiny fp32 case: H=4, D_c=64, D_r=16, D_n=D_v=32, L=128, T=5,
    parent=[-1,0,0,1,1], seed 0; every tensor ~ N(0,1)/sqrt(its own last dim)."""
    D = TINY
    parents = [np.array([-1, 0, 0, 1, 1], dtype=np.int32)]
    # q_lat = W_UK . q_nope with q_nope ~ N(0,1/D_n), W_UK ~ N(0,1/D_c): var 1/D_c.
    return make_case("tiny_fp32", **D, prefix_len=[128], parents=parents, dtype="f32", seed=0,
                     kv_std=1 / math.sqrt(D["D_c"]), krope_std=1 / math.sqrt(D["D_r"]),
                     qlat_std=1 / math.sqrt(D["D_c"]), qrope_std=1 / math.sqrt(D["D_r"]))


def tiny_fp32_layer(case: VerifyCase):
    """q_nope, W_UK, W_UV for the tiny case (non-absorbed inputs), float32."""
    H, D_c, D_n, D_v = case.H, case.D_c, case.D_n, case.D_v
    sumT = int(case.tree_off[-1])
    q_nope = _draw(rng_for(case.seed, "qnope", sumT, H, D_n), (sumT * H, D_n), 1 / math.sqrt(D_n))
    w_uk = _draw(rng_for(case.seed, "wuk", H, D_c, D_n), (H, D_c, D_n), 1 / math.sqrt(D_c))
    w_uv = _draw(rng_for(case.seed, "wuv", H, D_c, D_v), (H, D_c, D_v), 1 / math.sqrt(D_c))
    return q_nope, w_uk, w_uv


def layer_weights(case: VerifyCase, bf16: bool = True):
    """q_nope ~ N(0,1), W_UK, W_UV ~ N(0,1)/sqrt(D_c) for a Kimi-shape layer."""
    H, D_c, D_n, D_v = case.H, case.D_c, case.D_n, case.D_v
    sumT = int(case.tree_off[-1])
    q_nope = _draw(rng_for(case.seed, "qnope", sumT, H, D_n), (sumT * H, D_n), 1.0)
    w_uk = _draw(rng_for(case.seed, "wuk", H, D_c, D_n), (H, D_c, D_n), 1 / math.sqrt(D_c))
    w_uv = _draw(rng_for(case.seed, "wuv", H, D_c, D_v), (H, D_c, D_v), 1 / math.sqrt(D_c))
    if bf16:
        q_nope, w_uk, w_uv = bf16_round(q_nope), bf16_round(w_uk), bf16_round(w_uv)
    return q_nope, w_uk, w_uv


def kimi_layer_case(L: int = 5553, T: int = 13, seed: int = 1, paged: bool = False,
                    tree_seed: Optional[int] = None) -> VerifyCase:
    """One Kimi/DeepSeekV3-shape layer: H=64, 512/64/128/128, bf16, random tree."""
    ts = seed if tree_seed is None else tree_seed
    parents = [random_tree(T, rng_for(ts, "tree", T))]
    return make_case(f"kimi_L{L}_T{T}", **KIMI, prefix_len=[L], parents=parents,
                     dtype="bf16", seed=seed, paged=paged)


def context_sweep_case(L: int, layer: int, T: int = 15) -> VerifyCase:
    """Layer ``layer`` (0..60) of the context sweep at prefix L, T=15.

    The draft tree belongs to the verify step, so all 61 layers share it
    (tree seed 2000); each layer has its own KV and queries (seed 2000+layer).
    """
    parents = [random_tree(T, rng_for(2000, "tree", T))]
    return make_case(f"sweep_L{L}_layer{layer}", **KIMI, prefix_len=[L], parents=parents,
                     dtype="bf16", seed=2000 + layer)


def long_context_case(L: int = 200_000, T: int = 16) -> VerifyCase:
    """One layer at 200k context, T=16, KV ~ N(0,1), seed 3."""
    return kimi_layer_case(L=L, T=T, seed=3)


def batched_paged_case(B: int = 8, lo: int = 1024, hi: int = 32768,
                       t_lo: int = 9, t_hi: int = 16, seed: int = 4) -> VerifyCase:
    """B requests, prefixes ~ U{lo..hi}, trees of U{t_lo..t_hi} nodes, paged
    at page_size=1 through a random permutation of the pool."""
    plen = rng_for(seed, "prefix", B).integers(lo, hi + 1, size=B)
    tT = rng_for(seed, "treeT", B).integers(t_lo, t_hi + 1, size=B)
    parents = [random_tree(int(tT[b]), rng_for(seed, "tree", b, int(tT[b]))) for b in range(B)]
    return make_case(f"paged_B{B}", **KIMI, prefix_len=[int(x) for x in plen], parents=parents,
                     dtype="bf16", seed=seed, paged=True)


def scaled_case(case: VerifyCase, rows_scale: float) -> VerifyCase:
    """Copy of ``case`` with q multiplied by ``rows_scale`` (re-rounded to the
    case's dtype): sharpens or flattens the softmax for edge-case tests."""
    q = case.q * np.float32(rows_scale)
    if case.dtype == "bf16":
        q = bf16_round(q)
    return dataclasses.replace(case, q=q, name=f"{case.name}_qx{rows_scale}")


# ---------------------------------------------------------------------------
# Greedy tree acceptance inputs.
#
# The pages give no vocabulary size; the synthetic logits use 163,840 columns,
# the vocabulary of the Kimi K2 tokenizer that the Kimi-shape layer belongs to.
KIMI_VOCAB = 163_840


@dataclasses.dataclass
class AcceptCase:
    """One batched greedy-acceptance problem.

    ``logits`` rows are the target model's outputs at each tree node (node-major,
    request after request); ``token[u]`` is the draft token of node u. Logical
    key j of request b has slot ``page_table[kv_off[b] + j]`` (when paged).
    """
    name: str
    vocab: int
    max_T: int
    parent: np.ndarray              # int32 [sumT]
    tree_off: np.ndarray            # int32 [B+1]
    token: np.ndarray               # int32 [sumT]
    logits: Optional[np.ndarray]    # float32 [sumT, vocab] (bf16-exact when dtype bf16)
    target_in: Optional[np.ndarray] # int32 [sumT] when logits is None
    dtype: str                      # "bf16" or "f32"
    prefix_len: np.ndarray          # int32 [B]
    kv_off: np.ndarray              # int32 [B+1]
    page_table: Optional[np.ndarray] = None
    seed: int = 0

    @property
    def batch(self) -> int:
        return int(self.tree_off.shape[0] - 1)

    @property
    def total_nodes(self) -> int:
        return int(self.tree_off[-1])


def make_accept_case(name: str, *, parents: List[np.ndarray], vocab: int, seed: int,
                     p_follow: float = 0.8, dtype: str = "bf16", with_logits: bool = True,
                     prefix_len: Optional[List[int]] = None, paged: bool = False,
                     sibling_dups: bool = False, ties: bool = False,
                     nan_rows: int = 0) -> AcceptCase:
    """Draft tokens and target logits for a batch of trees.

    Siblings get distinct tokens while the vocabulary allows it (and unless
    ``sibling_dups``, which copies a sibling's token now and then). At every node the planted target token is,
    with probability ``p_follow``, the token of one of its children, else a
    random token; the planted logit is 16.0, above every N(0,1) draw. ``ties``
    plants the same 16.0 at a second random column; ``nan_rows`` rows get NaN
    at random columns (one row entirely NaN when nan_rows > 0).
    """
    B = len(parents)
    tree_T = np.array([len(p) for p in parents], dtype=np.int32)
    tree_off = np.zeros(B + 1, dtype=np.int32)
    tree_off[1:] = np.cumsum(tree_T)
    sumT = int(tree_off[-1])
    parent = np.concatenate([np.asarray(p, dtype=np.int32) for p in parents])
    token = np.zeros(sumT, dtype=np.int32)
    target = np.zeros(sumT, dtype=np.int32)
    rt = rng_for(seed, "tokens")
    for b in range(B):
        t0, T = int(tree_off[b]), int(tree_T[b])
        par = parent[t0:t0 + T]
        token[t0] = int(rt.integers(0, vocab))
        children = [[] for _ in range(T)]
        for u in range(1, T):
            if par[u] >= 0:
                children[par[u]].append(u)
        for p_ in range(T):
            kids = children[p_]
            if kids:
                draw = rt.choice(vocab, size=len(kids), replace=len(kids) > vocab)
                for k, u in enumerate(kids):
                    token[t0 + u] = int(draw[k])
                if sibling_dups and len(kids) > 1 and rt.random() < 0.5:
                    token[t0 + kids[-1]] = token[t0 + kids[0]]
            if kids and rt.random() < p_follow:
                target[t0 + p_] = token[t0 + kids[int(rt.integers(0, len(kids)))]]
            else:
                target[t0 + p_] = int(rt.integers(0, vocab))
    logits = None
    if with_logits:
        rl = rng_for(seed, "logits")
        logits = rl.standard_normal((sumT, vocab), dtype=np.float32)
        if dtype == "bf16":
            logits = bf16_round(logits)
        logits[np.arange(sumT), target] = 16.0
        if ties:
            logits[np.arange(sumT), rl.integers(0, vocab, size=sumT)] = 16.0
        for i in range(min(nan_rows, sumT)):
            r = int(rl.integers(0, sumT))
            logits[r, rl.integers(0, vocab, size=16)] = np.nan
        if nan_rows > 0:
            logits[int(rl.integers(0, sumT))] = np.nan
    if prefix_len is None:
        prefix_len = [0] * B
    plen = np.asarray(prefix_len, dtype=np.int32)
    kv_off = np.zeros(B + 1, dtype=np.int32)
    kv_off[1:] = np.cumsum(plen + tree_T)
    page_table = None
    if paged:
        n_keys = int(kv_off[-1])
        page_table = rng_for(seed, "perm", n_keys).permutation(n_keys).astype(np.int32)
    return AcceptCase(name=name, vocab=vocab, max_T=int(tree_T.max()), parent=parent,
                      tree_off=tree_off, token=token, logits=logits,
                      target_in=None if with_logits else target, dtype=dtype,
                      prefix_len=plen, kv_off=kv_off, page_table=page_table, seed=seed)


def kimi_accept_case(T: int = 13, seed: int = 1, vocab: int = KIMI_VOCAB) -> AcceptCase:
    """Acceptance after one Kimi-shape verify: one tree of T nodes (the same
    tree draw as ``kimi_layer_case``), bf16 logits over the full vocabulary."""
    parent = random_tree(T, rng_for(seed, "tree", T))
    return make_accept_case(f"kimi_accept_T{T}", parents=[parent], vocab=vocab, seed=seed,
                            prefix_len=[5553])


def batched_accept_case(B: int = 8, seed: int = 4, vocab: int = KIMI_VOCAB) -> AcceptCase:
    """Acceptance for the batched paged verify: the same prefixes, trees and
    page-table permutation as ``batched_paged_case(B, seed=seed)``."""
    plen = rng_for(seed, "prefix", B).integers(1024, 32768 + 1, size=B)
    tT = rng_for(seed, "treeT", B).integers(9, 16 + 1, size=B)
    parents = [random_tree(int(tT[b]), rng_for(seed, "tree", b, int(tT[b]))) for b in range(B)]
    return make_accept_case(f"paged_accept_B{B}", parents=parents, vocab=vocab, seed=seed,
                            prefix_len=[int(x) for x in plen], paged=True)



# ---------------------------------------------------------------------------
# Draft-tree construction inputs: a block drafter's per-position candidates.
#
# The pages name a block size of 16 and a node budget of 32 for the drafter
# (page "The Three Acts of Engineering", section "Act III", "The Reproducible
# Estimator"); a block of 16 positions after the root gives D = 15 draft
# positions here. K = 8 candidates per position is this library's choice (the
# builder's limit).

@dataclasses.dataclass
class BuildCase:
    """Per request: root token, K candidate tokens and log-probabilities for
    each of D positions, and the node budget (tree_off CSR)."""
    depth: int
    topk: int
    tree_off: np.ndarray        # int32 [B+1]
    root_token: np.ndarray      # int32 [B]
    cand_token: np.ndarray      # int32 [B][D][K]
    cand_logp: np.ndarray       # float32 [B][D][K]

    @property
    def batch(self) -> int:
        return int(self.tree_off.shape[0] - 1)


def make_build_case(budgets: List[int], D: int = 15, K: int = 8, seed: int = 0,
                    vocab: int = KIMI_VOCAB, quantised: bool = False) -> BuildCase:
    """Candidates: per position, K distinct random tokens whose log-probabilities
    are the K largest entries of a log-softmax over K+8 N(0, 2) logits (sorted
    descending). ``quantised`` rounds them to multiples of 1/4 so that score
    ties are common."""
    B = len(budgets)
    rng = rng_for(seed, "cands", B, D, K)
    toks = np.zeros((B, D, K), dtype=np.int32)
    logp = np.zeros((B, D, K), dtype=np.float32)
    for b in range(B):
        for d in range(D):
            toks[b, d] = rng.choice(vocab, size=K, replace=False)
            z = rng.standard_normal(K + 8) * 2.0
            ls = z - (np.log(np.exp(z - z.max()).sum()) + z.max())
            top = np.sort(ls)[::-1][:K]
            if quantised:
                top = np.round(top * 4) / 4
            logp[b, d] = top.astype(np.float32)
    off = np.zeros(B + 1, dtype=np.int32)
    off[1:] = np.cumsum(budgets)
    root = rng.integers(0, vocab, size=B).astype(np.int32)
    return BuildCase(depth=D, topk=K, tree_off=off, root_token=root, cand_token=toks, cand_logp=logp)
