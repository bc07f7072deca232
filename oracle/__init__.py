"""CPU oracle for tree-verify MLA attention (fp64, plain loops).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg use this package; the product path never imports it. It
shares no code with the CUDA library. The arithmetic lives in
``kdv_oracle.cpp``; this module compiles it with g++ and marshals numpy arrays.

Every function cites what it follows in ``kdv_oracle.cpp``'s header: the
multi-head latent attention named on the page "The Architecture of
Diagnosis" (section "Phase 1: Custom CUDA Kernels", item 2) with the latent
dims of the page "From Diagnosis to Deployment" (section "The Second Thread").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kdv_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libkdv_oracle.so")
_lib = None
_lock = threading.Lock()

_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u64p = np.ctypeslib.ndpointer(dtype=np.uint64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the oracle to ``oracle/libkdv_oracle.so`` (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            c = ctypes
            lib.oracle_tree_mask.argtypes = [_i32p, c.c_int32, _u64p, _i32p]
            lib.oracle_tree_mask.restype = c.c_int
            lib.oracle_verify_absorbed.argtypes = [
                c.c_int32, c.c_int32, c.c_int32, c.c_int32, c.c_int32, c.c_double,
                _f32p, _f32p, c.c_int64, c.c_void_p, c.c_int64, _i32p,
                c.c_int32, c.c_int32, c.c_void_p, c.c_int64, _f64p, _f64p, c.c_int]
            lib.oracle_verify_absorbed.restype = c.c_int
            lib.oracle_verify_mla.argtypes = [
                c.c_int32, c.c_int32, c.c_int32, c.c_int32, c.c_int32, c.c_int32, c.c_int32,
                c.c_double, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _i32p, _f64p, _f64p, c.c_int]
            lib.oracle_verify_mla.restype = c.c_int
            lib.oracle_absorb_q.argtypes = [c.c_int32, c.c_int64, c.c_int32, c.c_int32,
                                            _f32p, _f32p, _f64p, c.c_int]
            lib.oracle_absorb_q.restype = None
            lib.oracle_unabsorb_o.argtypes = [c.c_int32, c.c_int64, c.c_int32, c.c_int32,
                                              _f64p, _f32p, _f64p, c.c_int]
            lib.oracle_unabsorb_o.restype = None
            lib.oracle_combine.argtypes = [c.c_int32, c.c_int64, c.c_int32, _f64p, _f64p,
                                           _f64p, _f64p]
            lib.oracle_combine.restype = None
            lib.oracle_argmax.argtypes = [c.c_int64, c.c_int64, _f32p, c.c_int64, _i32p]
            lib.oracle_argmax.restype = None
            lib.oracle_tree_accept.argtypes = [c.c_int32, _i32p, _i32p, _i32p, _i32p,
                                               c.POINTER(c.c_int32), c.POINTER(c.c_int32)]
            lib.oracle_tree_accept.restype = c.c_int
            lib.oracle_accept_commit.argtypes = [c.c_int32, c.c_int32, c.c_int32, _i32p, _i32p]
            lib.oracle_accept_commit.restype = None
            _f32p_ = _f32p
            lib.oracle_tree_build.argtypes = [c.c_int32, c.c_int32, c.c_int32, c.c_int32, _i32p, _f32p_,
                                              _i32p, _i32p, _i32p, _f32p_]
            lib.oracle_tree_build.restype = c.c_int
            _lib = lib
    return _lib


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def tree_mask(parent: Sequence[int]):
    """Ancestor bitmask (self included) and depth of one tree, by walking parent[]."""
    p = np.ascontiguousarray(parent, dtype=np.int32)
    T = p.shape[0]
    mask = np.zeros(T, dtype=np.uint64)
    depth = np.zeros(T, dtype=np.int32)
    rc = _load().oracle_tree_mask(p, T, mask, depth)
    if rc != 0:
        raise ValueError("malformed parent[]")
    return mask, depth


def verify_request(*, H: int, L: int, parent, D_c: int, D_r: int, scale: float, q, pool,
                   page_table=None, kv_base: int = 0, key_lo: int = 0,
                   key_hi: Optional[int] = None, rows=None, n_threads: int = 0):
    """Absorbed-form verify attention of one request (see kdv_oracle.cpp).

    q: [T*H][D_c+D_r] rows of this request; pool: [num_slots][D_c+D_r];
    page_table: [L+T] pool rows of logical keys, or None (rows kv_base + j).
    Returns (o_lat [n_rows][D_c] float64, lse [n_rows] float64).
    """
    lib = _load()
    p = np.ascontiguousarray(parent, dtype=np.int32)
    T = int(p.shape[0])
    q = _f32(q)
    pool = _f32(pool)
    assert q.shape == (T * H, D_c + D_r), q.shape
    if key_hi is None:
        key_hi = L + T
    pt_arr = None
    if page_table is not None:
        pt_arr = np.ascontiguousarray(page_table, dtype=np.int32)
        assert pt_arr.shape[0] == L + T
    rows_arr = None
    n_rows = T * H
    if rows is not None:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int32)
        n_rows = int(rows_arr.shape[0])
    o = np.zeros((n_rows, D_c), dtype=np.float64)
    lse = np.zeros(n_rows, dtype=np.float64)
    rc = lib.oracle_verify_absorbed(
        H, T, L, D_c, D_r, float(scale), q, pool, pool.shape[0],
        pt_arr.ctypes.data if pt_arr is not None else None, kv_base, p,
        int(key_lo), int(key_hi), rows_arr.ctypes.data if rows_arr is not None else None,
        n_rows, o, lse, n_threads)
    if rc != 0:
        raise ValueError("malformed input to oracle_verify_absorbed")
    return o, lse


def verify_case(case, rows=None, n_threads: int = 0):
    """Oracle output for a whole ``datagen.VerifyCase`` (all requests).

    rows: optional sorted global row indices to evaluate. Returns (o, lse)
    for those rows in that order (all rows when None).
    """
    H = case.H
    outs_o, outs_l = [], []
    for b in range(case.batch):
        t0, t1 = int(case.tree_off[b]), int(case.tree_off[b + 1])
        r0, r1 = t0 * H, t1 * H
        if rows is None:
            sel = None
        else:
            rr = np.asarray(rows)
            sel = rr[(rr >= r0) & (rr < r1)] - r0
            if sel.size == 0:
                continue
        L = int(case.prefix_len[b])
        k0, k1 = int(case.kv_off[b]), int(case.kv_off[b + 1])
        pt = case.page_table[k0:k1] if case.page_table is not None else None
        o, l = verify_request(H=H, L=L, parent=case.parent[t0:t1], D_c=case.D_c, D_r=case.D_r,
                              scale=case.scale, q=case.q[r0:r1], pool=case.kv, page_table=pt,
                              kv_base=k0, rows=sel, n_threads=n_threads)
        outs_o.append(o)
        outs_l.append(l)
    return np.concatenate(outs_o), np.concatenate(outs_l)


def verify_mla(*, H, L, parent, D_c, D_r, D_n, D_v, scale, q_nope, q_rope, c_kv, k_rope,
               w_uk, w_uv, n_threads: int = 0):
    """Non-absorbed MLA (explicit K = c_kv W_UK, V = c_kv W_UV) of one request."""
    p = np.ascontiguousarray(parent, dtype=np.int32)
    T = int(p.shape[0])
    out = np.zeros((T * H, D_v), dtype=np.float64)
    lse = np.zeros(T * H, dtype=np.float64)
    rc = _load().oracle_verify_mla(H, T, L, D_c, D_r, D_n, D_v, float(scale), _f32(q_nope),
                                   _f32(q_rope), _f32(c_kv), _f32(k_rope), _f32(w_uk),
                                   _f32(w_uv), p, out, lse, n_threads)
    if rc != 0:
        raise ValueError("malformed parent[]")
    return out, lse


def absorb_q(H: int, q_nope, w_uk, n_threads: int = 0) -> np.ndarray:
    """q_lat[t*H+h] = W_UK[h] q_nope[t*H+h]  (W_UK stored [H][D_c][D_n])."""
    q_nope = _f32(q_nope)
    w_uk = _f32(w_uk)
    rows, D_n = q_nope.shape
    D_c = w_uk.shape[1]
    out = np.zeros((rows, D_c), dtype=np.float64)
    _load().oracle_absorb_q(H, rows, D_c, D_n, q_nope, w_uk, out, n_threads)
    return out


def unabsorb_o(H: int, o_lat, w_uv, n_threads: int = 0) -> np.ndarray:
    """out[t*H+h] = W_UV[h]^T o_lat[t*H+h]  (W_UV stored [H][D_c][D_v])."""
    o_lat = np.ascontiguousarray(o_lat, dtype=np.float64)
    w_uv = _f32(w_uv)
    rows, D_c = o_lat.shape
    D_v = w_uv.shape[2]
    out = np.zeros((rows, D_v), dtype=np.float64)
    _load().oracle_unabsorb_o(H, rows, D_c, D_v, o_lat, w_uv, out, n_threads)
    return out


def combine(o_part, lse_part):
    """Log-sum-exp merge of split partials: o_part [S][rows][d], lse_part [S][rows]."""
    o_part = np.ascontiguousarray(o_part, dtype=np.float64)
    lse_part = np.ascontiguousarray(lse_part, dtype=np.float64)
    S, rows, d = o_part.shape
    o = np.zeros((rows, d), dtype=np.float64)
    lse = np.zeros(rows, dtype=np.float64)
    _load().oracle_combine(S, rows, d, o_part, lse_part, o, lse)
    return o, lse


# ---------------------------------------------------------------------------
# Greedy tree acceptance (kdv_oracle.cpp: "Greedy tree acceptance"; page "The
# Architecture of Diagnosis", section "Phase 1: Custom CUDA Kernels", item 3).

def argmax(logits) -> np.ndarray:
    """Per-row argmax (lowest index among equal maxima, NaN never wins, all-NaN -> 0)."""
    x = _f32(logits)
    if x.ndim == 1:
        x = x[None, :]
    rows, vocab = x.shape
    out = np.zeros(rows, dtype=np.int32)
    _load().oracle_argmax(rows, vocab, x, vocab, out)
    return out


def tree_accept(parent, token, target):
    """Greedy acceptance of one tree: (path [T] root-first, -1 padded; len; bonus)."""
    p = np.ascontiguousarray(parent, dtype=np.int32)
    T = int(p.shape[0])
    tok = np.ascontiguousarray(token, dtype=np.int32)
    tgt = np.ascontiguousarray(target, dtype=np.int32)
    assert tok.shape == (T,) and tgt.shape == (T,)
    path = np.zeros(T, dtype=np.int32)
    n = ctypes.c_int32(0)
    bonus = ctypes.c_int32(0)
    rc = _load().oracle_tree_accept(T, p, tok, tgt, path, ctypes.byref(n), ctypes.byref(bonus))
    if rc != 0:
        raise ValueError("malformed parent[]")
    return path, int(n.value), int(bonus.value)


def accept_commit(page_table, L: int, path, n: int) -> np.ndarray:
    """Page table of one request ([L+T] slots) after committing the accepted path."""
    pt = np.array(page_table, dtype=np.int32, copy=True)
    pa = np.ascontiguousarray(path, dtype=np.int32)
    T = int(pt.shape[0]) - int(L)
    _load().oracle_accept_commit(int(L), T, int(n), pa, pt)
    return pt


def accept_case(case):
    """Oracle acceptance of a whole ``datagen.AcceptCase``.

    Returns dict with target [sumT], path [B][max_T] (-1 padded), len [B],
    bonus [B], and page_table (committed copy) when the case has one.
    """
    target = argmax(case.logits) if case.logits is not None else np.asarray(case.target_in,
                                                                            dtype=np.int32)
    B = case.batch
    path = np.full((B, case.max_T), -1, dtype=np.int32)
    lens = np.zeros(B, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    pt = None if case.page_table is None else np.array(case.page_table, dtype=np.int32)
    for b in range(B):
        t0, t1 = int(case.tree_off[b]), int(case.tree_off[b + 1])
        pb, n, bo = tree_accept(case.parent[t0:t1], case.token[t0:t1], target[t0:t1])
        path[b, :t1 - t0] = pb
        lens[b] = n
        bonus[b] = bo
        if pt is not None:
            k0, k1 = int(case.kv_off[b]), int(case.kv_off[b + 1])
            pt[k0:k1] = accept_commit(pt[k0:k1], int(case.prefix_len[b]), pb, n)
    out = {"target": target, "path": path, "len": lens, "bonus": bonus}
    if pt is not None:
        out["page_table"] = pt
    return out


# ---------------------------------------------------------------------------
# Best-first draft-tree construction (kdv_oracle.cpp: "Best-first draft-tree
# construction"; page "The Architecture of Diagnosis", section "Phase 1:
# Custom CUDA Kernels", item 1).

def tree_build(T: int, root_token: int, cand_token, cand_logp):
    """First T nodes in (score desc, candidate path asc) order.

    cand_token int32 [D][K], cand_logp float32 [D][K] (log-probabilities).
    Returns (parent, token, depth, score) of the emitted nodes.
    """
    ct = np.ascontiguousarray(cand_token, dtype=np.int32)
    cl = np.ascontiguousarray(cand_logp, dtype=np.float32)
    D, K = ct.shape
    parent = np.zeros(T, dtype=np.int32)
    token = np.zeros(T, dtype=np.int32)
    depth = np.zeros(T, dtype=np.int32)
    score = np.zeros(T, dtype=np.float32)
    n = _load().oracle_tree_build(int(T), int(D), int(K), int(root_token), ct, cl, parent, token, depth,
                                  score)
    if n < 0:
        raise ValueError("bad sizes")
    return parent[:n], token[:n], depth[:n], score[:n]
