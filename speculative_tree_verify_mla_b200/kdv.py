"""Thin Python binding of the C-ABI library ``libkdv.so`` (include/kdv.h).

Argument marshalling only: each ``kdv_*`` function here takes torch tensors
(device memory, allocated by the caller) and host lists, passes raw pointers
and sizes to the C entry point of the same name, and raises ``KdvError`` on a
non-zero status. Every step of the computation runs in the library's CUDA
kernels. There is no fallback: if ``libkdv.so`` is missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkdv.so")
# the same library with the verify kernel's stage stamps (include/kdv_trace.h)
TRACE_LIB_PATH = os.path.join(_PKG, "libkdv_trace.so")
TRACE_EXPORTED = ("kdv_trace_clear", "kdv_trace_read")
KDV_TRACE_CTAS = 1024
KDV_TRACE_SLOTS = 16
# stage slots, in kdv_trace.h order
KDV_TRACE_STAGES = ("setup", "S mma t0 issued", "S mma t1 issued", "S mma last issued",
                    "softmax0 sees S t0", "softmax0 pushed t0", "softmax0 done", "softmax1 done",
                    "V rows ready", "PV t0 issued", "PV last issued", "O sees P t0",
                    "epilogue start", "epilogue stored", "teardown")

KDV_OK = 0
KDV_ERR_INVALID_ARG = -1
KDV_ERR_UNSUPPORTED = -2
KDV_ERR_WORKSPACE = -3
KDV_ERR_CUDA = -4

KDV_DERR_BAD_PARENT = 1
KDV_DERR_BAD_SLOT = 2
KDV_DERR_BAD_LENGTH = 3
KDV_DERR_BAD_TOKEN = 4
KDV_DERR_TIMEOUT = 5
KDV_DERR_BAD_SCORE = 6
KDV_DERR_RANGE = 7

KDV_BF16 = 0
KDV_F32 = 1
KDV_PROJ_STATIC_WEIGHTS = 1     # kdv_absorb_q_ex / kdv_unabsorb_o_ex flag: weights not written by the previous kernel
KDV_IMPL_AUTO = 0
KDV_IMPL_SIMT = 1
KDV_IMPL_TC = 2
KDV_IMPL_TC_1SM = 3          # retired: kdv_verify_attn returns KDV_ERR_UNSUPPORTED
KDV_IMPL_TC_STAGED = 4
KDV_MAX_TREE = 64
KDV_MAX_BATCH = 128

# Every entry point include/kdv.h declares (checked by the CPU tests).
EXPORTED = ("kdv_status_string", "kdv_version", "kdv_tree_mask_build",
            "kdv_verify_attn_workspace", "kdv_verify_attn_plan", "kdv_verify_attn",
            "kdv_verify_attn_noalloc", "kdv_latent_f16", "kdv_combine", "kdv_tree_accept_workspace",
            "kdv_tree_accept", "kdv_absorb_q", "kdv_unabsorb_o", "kdv_tree_build",
            "kdv_absorb_q_ex", "kdv_unabsorb_o_ex", "kdv_verify_attn_launches")
KDV_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class KdvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class VerifyParams(ctypes.Structure):
    """Mirror of ``kdv_verify_params`` (field order and types must match kdv.h)."""
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_heads", ctypes.c_int32),
        ("d_latent", ctypes.c_int32), ("d_rope", ctypes.c_int32),
        ("scale", ctypes.c_float), ("dtype", ctypes.c_int32), ("impl", ctypes.c_int32),
        ("q", ctypes.c_void_p), ("q_row_stride", ctypes.c_int64),
        ("kv", ctypes.c_void_p), ("num_slots", ctypes.c_int64),
        ("page_table", ctypes.c_void_p), ("kv_off", ctypes.c_void_p),
        ("tree_off", ctypes.c_void_p), ("prefix_len", ctypes.c_void_p),
        ("h_prefix_len", ctypes.POINTER(ctypes.c_int32)),
        ("h_tree_T", ctypes.POINTER(ctypes.c_int32)),
        ("mask", ctypes.c_void_p), ("num_splits", ctypes.c_int32),
        ("return_partials", ctypes.c_int32),
        ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("o_part", ctypes.c_void_p), ("lse_part", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("d_err", ctypes.c_void_p), ("wait_limit_ns", ctypes.c_uint64), ("v16", ctypes.c_void_p),
    ]


class AcceptParams(ctypes.Structure):
    """Mirror of ``kdv_accept_params`` (field order and types must match kdv.h)."""
    _fields_ = [
        ("batch", ctypes.c_int32), ("max_T", ctypes.c_int32),
        ("total_nodes", ctypes.c_int32), ("vocab", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("logits", ctypes.c_void_p), ("logits_ld", ctypes.c_int64),
        ("target_in", ctypes.c_void_p), ("token", ctypes.c_void_p),
        ("parent", ctypes.c_void_p), ("tree_off", ctypes.c_void_p),
        ("target_out", ctypes.c_void_p), ("accept_len", ctypes.c_void_p),
        ("accept_path", ctypes.c_void_p), ("bonus", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p), ("kv_off", ctypes.c_void_p),
        ("prefix_len", ctypes.c_void_p), ("prefix_len_out", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("d_err", ctypes.c_void_p),
    ]


class BuildParams(ctypes.Structure):
    """Mirror of ``kdv_tree_build_params`` (field order and types must match kdv.h)."""
    _fields_ = [
        ("batch", ctypes.c_int32), ("max_T", ctypes.c_int32), ("depth", ctypes.c_int32),
        ("topk", ctypes.c_int32), ("tree_off", ctypes.c_void_p), ("root_token", ctypes.c_void_p),
        ("cand_token", ctypes.c_void_p), ("cand_logp", ctypes.c_void_p),
        ("parent", ctypes.c_void_p), ("token", ctypes.c_void_p), ("depth_out", ctypes.c_void_p),
        ("score", ctypes.c_void_p), ("d_err", ctypes.c_void_p),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Load libkdv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                               "or speculative_tree_verify_mla_b200/build.py")
        lib = ctypes.CDLL(LIB_PATH)
        c = ctypes
        lib.kdv_status_string.argtypes = [c.c_int]
        lib.kdv_status_string.restype = c.c_char_p
        lib.kdv_version.argtypes = []
        lib.kdv_version.restype = c.c_int32
        lib.kdv_tree_mask_build.argtypes = [c.c_void_p, c.c_void_p, c.c_int32, c.c_int32,
                                            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p]
        lib.kdv_tree_mask_build.restype = c.c_int
        lib.kdv_verify_attn_workspace.argtypes = [c.POINTER(VerifyParams), c.POINTER(c.c_size_t)]
        lib.kdv_verify_attn_workspace.restype = c.c_int
        lib.kdv_verify_attn_plan.argtypes = [c.POINTER(VerifyParams), c.c_void_p, c.c_void_p]
        lib.kdv_verify_attn_plan.restype = c.c_int
        lib.kdv_verify_attn_launches.argtypes = [c.POINTER(VerifyParams), c.POINTER(c.c_int32)]
        lib.kdv_verify_attn_launches.restype = c.c_int
        lib.kdv_verify_attn.argtypes = [c.POINTER(VerifyParams), c.c_void_p]
        lib.kdv_verify_attn.restype = c.c_int
        lib.kdv_verify_attn_noalloc.argtypes = [c.POINTER(VerifyParams), c.c_void_p]
        lib.kdv_verify_attn_noalloc.restype = c.c_int
        lib.kdv_latent_f16.argtypes = [c.POINTER(VerifyParams), c.c_void_p, c.c_void_p]
        lib.kdv_latent_f16.restype = c.c_int
        lib.kdv_combine.argtypes = [c.c_void_p, c.c_void_p, c.c_int32, c.c_int64, c.c_int32,
                                    c.c_void_p, c.c_void_p, c.c_void_p]
        lib.kdv_combine.restype = c.c_int
        lib.kdv_tree_accept_workspace.argtypes = [c.POINTER(AcceptParams), c.POINTER(c.c_size_t)]
        lib.kdv_tree_accept_workspace.restype = c.c_int
        lib.kdv_tree_accept.argtypes = [c.POINTER(AcceptParams), c.c_void_p]
        lib.kdv_tree_accept.restype = c.c_int
        lib.kdv_absorb_q.argtypes = [c.c_int32, c.c_int32, c.c_int32, c.c_int32, c.c_void_p, c.c_int64,
                                     c.c_int32, c.c_void_p, c.c_int32, c.c_void_p, c.c_int64, c.c_int32,
                                     c.c_void_p]
        lib.kdv_absorb_q.restype = c.c_int
        lib.kdv_unabsorb_o.argtypes = [c.c_int32, c.c_int32, c.c_int32, c.c_int32, c.c_void_p, c.c_int64,
                                       c.c_void_p, c.c_int32, c.c_void_p, c.c_int64, c.c_int32, c.c_void_p]
        lib.kdv_unabsorb_o.restype = c.c_int
        lib.kdv_absorb_q_ex.argtypes = list(lib.kdv_absorb_q.argtypes[:-1]) + [c.c_uint32, c.c_void_p]
        lib.kdv_absorb_q_ex.restype = c.c_int
        lib.kdv_unabsorb_o_ex.argtypes = list(lib.kdv_unabsorb_o.argtypes[:-1]) + [c.c_uint32, c.c_void_p]
        lib.kdv_unabsorb_o_ex.restype = c.c_int
        lib.kdv_tree_build.argtypes = [c.POINTER(BuildParams), c.c_void_p]
        lib.kdv_tree_build.restype = c.c_int
        if hasattr(lib, "kdv_trace_read"):          # the tracing build
            lib.kdv_trace_clear.argtypes = [c.c_void_p]
            lib.kdv_trace_clear.restype = c.c_int
            lib.kdv_trace_read.argtypes = [c.c_void_p, c.c_int64]
            lib.kdv_trace_read.restype = c.c_int
        _lib = lib
    return _lib


def use_trace_library() -> None:
    """Make ``load()`` open libkdv_trace.so (call before the first load)."""
    global LIB_PATH
    if _lib is not None and LIB_PATH != TRACE_LIB_PATH:
        raise RuntimeError("libkdv.so is already loaded in this process")
    LIB_PATH = TRACE_LIB_PATH


def kdv_trace_clear(stream=None) -> None:
    _check(load().kdv_trace_clear(_stream(stream)), "kdv_trace_clear")


def kdv_trace_read(n_ctas: int) -> np.ndarray:
    """Stage stamps of the first n_ctas CTAs of the last traced launch:
    uint64 [n_ctas][KDV_TRACE_SLOTS] global-timer ns (0 = stage not reached)."""
    n_ctas = min(int(n_ctas), KDV_TRACE_CTAS)
    out = np.zeros((n_ctas, KDV_TRACE_SLOTS), dtype=np.uint64)
    _check(load().kdv_trace_read(out.ctypes.data, out.size), "kdv_trace_read")
    return out


def status_string(status: int) -> str:
    return load().kdv_status_string(int(status)).decode()


def kdv_version() -> int:
    return int(load().kdv_version())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    return int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        if torch.cuda.is_available():
            return int(torch.cuda.current_stream().cuda_stream) or None
        return None
    if isinstance(stream, torch.cuda.Stream):
        return int(stream.cuda_stream) or None
    return int(stream) or None


def _check(status: int, where: str):
    if status != KDV_OK:
        raise KdvError(status, where)


def kdv_tree_mask_build(parent: torch.Tensor, tree_off: Optional[torch.Tensor], batch: int,
                        max_T: int, mask: torch.Tensor, depth: Optional[torch.Tensor] = None,
                        d_err: Optional[torch.Tensor] = None, stream=None) -> None:
    """parent[] -> ancestor bitmask (int64 tensor holding the uint64 bits)."""
    _check(load().kdv_tree_mask_build(_ptr(parent), _ptr(tree_off), int(batch), int(max_T),
                                      _ptr(mask), _ptr(depth), _ptr(d_err), _stream(stream)),
           "kdv_tree_mask_build")


def make_params(**kw) -> VerifyParams:
    """Build a VerifyParams from keyword arguments (tensors become pointers)."""
    p = VerifyParams()
    keep = []
    for k, v in kw.items():
        if k in ("h_prefix_len", "h_tree_T"):
            arr = (ctypes.c_int32 * len(v))(*[int(x) for x in v])
            keep.append(arr)
            setattr(p, k, ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32)))
        elif isinstance(v, torch.Tensor):
            setattr(p, k, int(v.data_ptr()))
        elif v is None:
            setattr(p, k, None)
        else:
            setattr(p, k, v)
    p._keep = keep          # keep host arrays alive with the struct
    return p


def kdv_verify_attn_workspace(params: VerifyParams) -> int:
    n = ctypes.c_size_t(0)
    _check(load().kdv_verify_attn_workspace(ctypes.byref(params), ctypes.byref(n)),
           "kdv_verify_attn_workspace")
    return int(n.value)


def kdv_verify_attn_plan(params: VerifyParams):
    """(splits per request, grid work items) that kdv_verify_attn would use."""
    splits = (ctypes.c_int32 * max(1, params.batch))()
    items = ctypes.c_int32(0)
    _check(load().kdv_verify_attn_plan(ctypes.byref(params), splits, ctypes.byref(items)),
           "kdv_verify_attn_plan")
    return [int(splits[i]) for i in range(params.batch)], int(items.value)


def kdv_verify_attn_launches(params: VerifyParams) -> int:
    """How many kernels kdv_verify_attn launches for these parameters."""
    n = ctypes.c_int32(0)
    _check(load().kdv_verify_attn_launches(ctypes.byref(params), ctypes.byref(n)),
           "kdv_verify_attn_launches")
    return int(n.value)


def kdv_verify_attn(params: VerifyParams, stream=None) -> None:
    _check(load().kdv_verify_attn(ctypes.byref(params), _stream(stream)), "kdv_verify_attn")


def kdv_verify_attn_noalloc(params: VerifyParams, stream=None) -> None:
    """kdv_verify_attn with the library's built-in scratch instead of params.workspace."""
    _check(load().kdv_verify_attn_noalloc(ctypes.byref(params), _stream(stream)),
           "kdv_verify_attn_noalloc")


def kdv_latent_f16(params: VerifyParams, v16: torch.Tensor, stream=None) -> None:
    """The fp16 latent rows [sum(L+T)][512] of a call (see kdv.h)."""
    _check(load().kdv_latent_f16(ctypes.byref(params), _ptr(v16), _stream(stream)), "kdv_latent_f16")


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDV_BF16
    if t.dtype == torch.float32:
        return KDV_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def kdv_absorb_q(num_heads: int, q_nope: torch.Tensor, w_uk: torch.Tensor, q_lat: torch.Tensor,
                 stream=None, flags: int = 0) -> None:
    """q_lat[row, :D_c] = W_UK[row % H] q_nope[row] (2-D row-strided tensors).
    flags != 0 calls kdv_absorb_q_ex (KDV_PROJ_STATIC_WEIGHTS)."""
    rows, d_nope = q_nope.shape
    d_latent = w_uk.shape[1]
    args = (int(rows), int(num_heads), int(d_latent), int(d_nope), _ptr(q_nope), int(q_nope.stride(0)),
            _dt(q_nope), _ptr(w_uk), _dt(w_uk), _ptr(q_lat), int(q_lat.stride(0)), _dt(q_lat))
    if flags:
        _check(load().kdv_absorb_q_ex(*args, int(flags), _stream(stream)), "kdv_absorb_q_ex")
    else:
        _check(load().kdv_absorb_q(*args, _stream(stream)), "kdv_absorb_q")


def kdv_unabsorb_o(num_heads: int, o_lat: torch.Tensor, w_uv: torch.Tensor, out: torch.Tensor,
                   stream=None, flags: int = 0) -> None:
    """out[row] = W_UV[row % H]^T o_lat[row] (o_lat fp32).
    flags != 0 calls kdv_unabsorb_o_ex (KDV_PROJ_STATIC_WEIGHTS)."""
    rows, d_latent = o_lat.shape
    d_v = w_uv.shape[2]
    args = (int(rows), int(num_heads), int(d_latent), int(d_v), _ptr(o_lat), int(o_lat.stride(0)), _ptr(w_uv),
            _dt(w_uv), _ptr(out), int(out.stride(0)), _dt(out))
    if flags:
        _check(load().kdv_unabsorb_o_ex(*args, int(flags), _stream(stream)), "kdv_unabsorb_o_ex")
    else:
        _check(load().kdv_unabsorb_o(*args, _stream(stream)), "kdv_unabsorb_o")


def kdv_combine(o_part: torch.Tensor, lse_part: torch.Tensor, S: int, rows: int, d: int,
                o: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(load().kdv_combine(_ptr(o_part), _ptr(lse_part), int(S), int(rows), int(d), _ptr(o),
                              _ptr(lse), _stream(stream)), "kdv_combine")


# ---------------------------------------------------------------------------
# Device-resident problem (upload once, call many times).
# ---------------------------------------------------------------------------
class DeviceCase:
    """A ``datagen.VerifyCase`` uploaded to the GPU, plus output buffers.

    ``run()`` calls kdv_tree_mask_build then kdv_verify_attn through the C ABI.
    """

    def __init__(self, case, device="cuda", impl: int = KDV_IMPL_AUTO, num_splits: int = 0,
                 return_partials: bool = False):
        dev = torch.device(device)
        self.case = case
        self.impl = impl
        self.num_splits = num_splits
        self.return_partials = return_partials
        tdt = torch.bfloat16 if case.dtype == "bf16" else torch.float32
        self.dtype = KDV_BF16 if case.dtype == "bf16" else KDV_F32
        self.q = torch.from_numpy(case.q).to(tdt).to(dev)
        self.kv = torch.from_numpy(case.kv).to(tdt).to(dev)
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
        self.parent = i32(case.parent)
        self.tree_off = i32(case.tree_off)
        self.kv_off = i32(case.kv_off)
        self.prefix_len = i32(case.prefix_len)
        self.page_table = i32(case.page_table) if case.page_table is not None else None
        sumT = int(case.tree_off[-1])
        self.mask = torch.zeros(sumT, dtype=torch.int64, device=dev)
        self.depth = torch.zeros(sumT, dtype=torch.int32, device=dev)
        self.d_err = torch.zeros(1, dtype=torch.int32, device=dev)
        rows = case.rows
        self.o = torch.empty(rows, case.D_c, dtype=torch.float32, device=dev)
        self.lse = torch.empty(rows, dtype=torch.float32, device=dev)
        S = max(1, num_splits)
        self.o_part = self.lse_part = None
        if return_partials:
            self.o_part = torch.empty(S, rows, case.D_c, dtype=torch.float32, device=dev)
            self.lse_part = torch.empty(S, rows, dtype=torch.float32, device=dev)
        self.params = self._params()
        self.ws_bytes = kdv_verify_attn_workspace(self.params)
        self.workspace = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.params.workspace = int(self.workspace.data_ptr())
        self.params.workspace_bytes = self.ws_bytes

    def _params(self) -> VerifyParams:
        c = self.case
        return make_params(
            batch=c.batch, num_heads=c.H, d_latent=c.D_c, d_rope=c.D_r, scale=c.scale,
            dtype=self.dtype, impl=self.impl, q=self.q, q_row_stride=c.D_q, kv=self.kv,
            num_slots=int(c.kv.shape[0]), page_table=self.page_table, kv_off=self.kv_off,
            tree_off=self.tree_off, prefix_len=self.prefix_len,
            h_prefix_len=[int(x) for x in c.prefix_len], h_tree_T=[int(x) for x in c.tree_T],
            mask=self.mask, num_splits=self.num_splits,
            return_partials=1 if self.return_partials else 0, o=self.o, lse=self.lse,
            o_part=self.o_part, lse_part=self.lse_part, workspace=None, workspace_bytes=0,
            d_err=self.d_err)

    def build_mask(self, stream=None):
        c = self.case
        kdv_tree_mask_build(self.parent, self.tree_off, c.batch, int(max(c.tree_T)), self.mask,
                            self.depth, self.d_err, stream)

    def verify(self, stream=None):
        kdv_verify_attn(self.params, stream)

    def run(self, stream=None):
        self.build_mask(stream)
        self.verify(stream)
        return self

    def results(self):
        """(o, lse) or (o_part, lse_part) as numpy arrays, after a sync."""
        torch.cuda.synchronize()
        if self.return_partials:
            return self.o_part.cpu().numpy(), self.lse_part.cpu().numpy()
        return self.o.cpu().numpy(), self.lse.cpu().numpy()

    def error_flag(self) -> int:
        torch.cuda.synchronize()
        return int(self.d_err.item())


# ---------------------------------------------------------------------------
# Greedy tree acceptance.
# ---------------------------------------------------------------------------
def make_accept_params(**kw) -> AcceptParams:
    """Build an AcceptParams from keyword arguments (tensors become pointers)."""
    p = AcceptParams()
    for k, v in kw.items():
        if isinstance(v, torch.Tensor):
            setattr(p, k, int(v.data_ptr()))
        else:
            setattr(p, k, v)
    return p


def kdv_tree_build(params: BuildParams, stream=None) -> None:
    _check(load().kdv_tree_build(ctypes.byref(params), _stream(stream)), "kdv_tree_build")


def make_build_params(**kw) -> BuildParams:
    p = BuildParams()
    for k, v in kw.items():
        setattr(p, k, int(v.data_ptr()) if isinstance(v, torch.Tensor) else v)
    return p


def kdv_tree_accept_workspace(params: AcceptParams) -> int:
    n = ctypes.c_size_t(0)
    _check(load().kdv_tree_accept_workspace(ctypes.byref(params), ctypes.byref(n)),
           "kdv_tree_accept_workspace")
    return int(n.value)


def kdv_tree_accept(params: AcceptParams, stream=None) -> None:
    _check(load().kdv_tree_accept(ctypes.byref(params), _stream(stream)), "kdv_tree_accept")


class DeviceAcceptCase:
    """A ``datagen.AcceptCase`` uploaded to the GPU, plus output buffers.

    ``run()`` calls kdv_tree_accept through the C ABI; the page table (when
    the case has one) is committed in place, so ``run()`` restores it first.
    """

    def __init__(self, case, device="cuda", commit: bool = True, update_prefix: bool = True):
        dev = torch.device(device)
        self.case = case
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
        self.logits = None
        self.dtype = KDV_BF16 if case.dtype == "bf16" else KDV_F32
        if case.logits is not None:
            tdt = torch.bfloat16 if case.dtype == "bf16" else torch.float32
            self.logits = torch.from_numpy(case.logits).to(tdt).to(dev)
        self.target_in = i32(case.target_in) if case.target_in is not None else None
        self.token = i32(case.token)
        self.parent = i32(case.parent)
        self.tree_off = i32(case.tree_off)
        self.kv_off = i32(case.kv_off)
        self.prefix_len = i32(case.prefix_len)
        self.page_table0 = i32(case.page_table) if (case.page_table is not None and commit) else None
        self.page_table = self.page_table0.clone() if self.page_table0 is not None else None
        sumT, B = case.total_nodes, case.batch
        self.target_out = torch.full((sumT,), -7, dtype=torch.int32, device=dev)
        self.accept_len = torch.full((B,), -7, dtype=torch.int32, device=dev)
        self.accept_path = torch.full((B, case.max_T), -7, dtype=torch.int32, device=dev)
        self.bonus = torch.full((B,), -7, dtype=torch.int32, device=dev)
        self.prefix_len_out = torch.full((B,), -7, dtype=torch.int32, device=dev) if update_prefix else None
        self.d_err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.params = make_accept_params(
            batch=B, max_T=case.max_T, total_nodes=sumT, vocab=case.vocab, dtype=self.dtype,
            logits=self.logits, logits_ld=case.vocab, target_in=self.target_in, token=self.token,
            parent=self.parent, tree_off=self.tree_off, target_out=self.target_out,
            accept_len=self.accept_len, accept_path=self.accept_path, bonus=self.bonus,
            page_table=self.page_table, kv_off=self.kv_off, prefix_len=self.prefix_len,
            prefix_len_out=self.prefix_len_out, workspace=None, workspace_bytes=0,
            d_err=self.d_err)
        self.ws_bytes = kdv_tree_accept_workspace(self.params)
        self.workspace = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.params.workspace = int(self.workspace.data_ptr())
        self.params.workspace_bytes = self.ws_bytes

    def run(self, stream=None):
        if self.page_table is not None:
            self.page_table.copy_(self.page_table0)
        kdv_tree_accept(self.params, stream)
        return self

    def results(self) -> dict:
        torch.cuda.synchronize()
        out = {"target": self.target_out.cpu().numpy(), "path": self.accept_path.cpu().numpy(),
               "len": self.accept_len.cpu().numpy(), "bonus": self.bonus.cpu().numpy()}
        if self.page_table is not None:
            out["page_table"] = self.page_table.cpu().numpy()
        if self.prefix_len_out is not None:
            out["prefix_len_out"] = self.prefix_len_out.cpu().numpy()
        return out

    def error_flag(self) -> int:
        torch.cuda.synchronize()
        return int(self.d_err.item())
