"""CPU checks of the C-ABI library: it loads, exports every declared entry
point, and rejects bad arguments on the host before touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

from speculative_tree_verify_mla_b200 import build, kdv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return kdv.load()


def declared_symbols(header="kdv.h"):
    txt = open(os.path.join(ROOT, "include", header)).read()
    return set(re.findall(r"KDV_API[^;(]*?\b(kdv_\w+)\s*\(", txt))


def test_exports_every_declared_symbol(lib):
    assert sorted(fn for fn in os.listdir(os.path.join(ROOT, "include")) if fn.endswith(".h")) == \
        ["kdv.h", "kdv_trace.h"]
    names = declared_symbols()
    assert names == set(kdv.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n
    # the product library has none of the tracing build's entry points
    for n in kdv.TRACE_EXPORTED:
        assert not hasattr(lib, n), n


def test_trace_build_exports_its_symbols():
    """libkdv_trace.so exports everything kdv.h declares plus kdv_trace.h's."""
    import ctypes as c
    path = build.build_trace()
    tlib = c.CDLL(path)
    names = declared_symbols("kdv_trace.h")
    assert names == set(kdv.TRACE_EXPORTED), names
    for n in names | declared_symbols():
        assert hasattr(tlib, n), n
    txt = open(os.path.join(ROOT, "include", "kdv_trace.h")).read()
    assert int(re.search(r"#define KDV_TRACE_CTAS (\d+)", txt).group(1)) == kdv.KDV_TRACE_CTAS
    assert int(re.search(r"#define KDV_TRACE_SLOTS (\d+)", txt).group(1)) == kdv.KDV_TRACE_SLOTS
    stages = re.findall(r"KDV_TRACE_\w+ = (\d+),?", txt)
    assert [int(x) for x in stages] == list(range(len(kdv.KDV_TRACE_STAGES)))
    # host-side argument checks need no GPU
    assert tlib.kdv_trace_read(None, c.c_int64(-1)) == kdv.KDV_ERR_INVALID_ARG
    assert tlib.kdv_trace_read(None, c.c_int64(kdv.KDV_TRACE_CTAS * kdv.KDV_TRACE_SLOTS + 1)) == \
        kdv.KDV_ERR_INVALID_ARG
    assert tlib.kdv_trace_read(None, c.c_int64(0)) == kdv.KDV_OK


def test_status_strings(lib):
    for s in (0, -1, -2, -3, -4):
        assert kdv.status_string(s).startswith("KDV_")
    assert kdv.status_string(-99) == "KDV_ERR_UNKNOWN"
    assert kdv.kdv_version() == 123


@pytest.mark.parametrize("cls,cname", [(kdv.VerifyParams, "kdv_verify_params"),
                                       (kdv.AcceptParams, "kdv_accept_params"),
                                       (kdv.BuildParams, "kdv_tree_build_params")])
def test_params_struct_layout(tmp_path, cls, cname):
    """ctypes mirror matches the C struct: compile a probe against kdv.h."""
    fields = [f[0] for f in cls._fields_]
    src = tmp_path / "probe.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "kdv.h"\nint main(void){'
                   + "".join(f'printf("%zu\\n", offsetof({cname}, {f}));' for f in fields)
                   + f'printf("%zu\\n", sizeof({cname})); return 0;}}')
    exe = tmp_path / "probe"
    import subprocess
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = [int(x) for x in subprocess.check_output([str(exe)]).split()]
    want = [getattr(cls, f).offset for f in fields] + [ctypes.sizeof(cls)]
    assert got == want


def _params(**over):
    base = dict(batch=1, num_heads=4, d_latent=64, d_rope=16, scale=0.1, dtype=kdv.KDV_F32,
                impl=kdv.KDV_IMPL_SIMT, q=None, q_row_stride=0, kv=None, num_slots=10,
                page_table=None, kv_off=None, tree_off=None, prefix_len=None,
                h_prefix_len=[5], h_tree_T=[3], mask=None, num_splits=0, return_partials=0,
                o=None, lse=None, o_part=None, lse_part=None, workspace=None,
                workspace_bytes=0, d_err=None, v16=None)
    base.update(over)
    return kdv.make_params(**base)


@pytest.mark.parametrize("over,status", [
    (dict(batch=0), kdv.KDV_ERR_INVALID_ARG),
    (dict(batch=129, h_prefix_len=[1] * 129, h_tree_T=[1] * 129), kdv.KDV_ERR_UNSUPPORTED),
    (dict(num_heads=0), kdv.KDV_ERR_INVALID_ARG),
    (dict(h_tree_T=[65]), kdv.KDV_ERR_UNSUPPORTED),
    (dict(h_tree_T=[0]), kdv.KDV_ERR_INVALID_ARG),
    (dict(h_prefix_len=[-1]), kdv.KDV_ERR_INVALID_ARG),
    (dict(dtype=7), kdv.KDV_ERR_INVALID_ARG),
    (dict(impl=kdv.KDV_IMPL_TC), kdv.KDV_ERR_UNSUPPORTED),          # f32, 64/16 dims
    (dict(d_latent=513), kdv.KDV_ERR_UNSUPPORTED),
    (dict(d_rope=65), kdv.KDV_ERR_UNSUPPORTED),
    (dict(num_splits=-1), kdv.KDV_ERR_INVALID_ARG),
    (dict(return_partials=1, num_splits=0), kdv.KDV_ERR_INVALID_ARG),
    (dict(scale=float("nan")), kdv.KDV_ERR_INVALID_ARG),
])
def test_host_validation(lib, over, status):
    p = _params(**over)
    n = ctypes.c_size_t(0)
    assert lib.kdv_verify_attn_workspace(ctypes.byref(p), ctypes.byref(n)) == status
    assert lib.kdv_verify_attn(ctypes.byref(p), None) == status


def test_null_pointers_rejected_before_launch(lib):
    p = _params()
    assert lib.kdv_verify_attn(ctypes.byref(p), None) == kdv.KDV_ERR_INVALID_ARG


def test_tc_alignment_rejected(lib):
    p = _params(dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, impl=kdv.KDV_IMPL_TC,
                q=0x1002, kv=0x2000, kv_off=0x3000, tree_off=0x4000, mask=0x5000, o=0x6000)
    assert lib.kdv_verify_attn(ctypes.byref(p), None) == kdv.KDV_ERR_INVALID_ARG
    p = _params(dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, impl=kdv.KDV_IMPL_TC,
                q=0x1000, kv=0x2000, kv_off=0x3000, tree_off=0x4000, mask=0x5000, o=0x6000,
                q_row_stride=577)
    assert lib.kdv_verify_attn(ctypes.byref(p), None) == kdv.KDV_ERR_INVALID_ARG
    # outputs are written in 16-byte vectors: a 4-byte aligned o is refused
    p = _params(dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, impl=kdv.KDV_IMPL_TC,
                q=0x1000, kv=0x2000, kv_off=0x3000, tree_off=0x4000, mask=0x5000, o=0x6004)
    assert lib.kdv_verify_attn(ctypes.byref(p), None) == kdv.KDV_ERR_INVALID_ARG


def test_workspace_sizes(lib):
    # forced single split: direct output, no workspace
    assert kdv.kdv_verify_attn_workspace(_params(num_splits=1)) == 0
    # forced 3 splits, merged by the library (SIMT kernel): 3 * T*H partial
    # rows of D_c fp32 values, then one fp32 lse each
    n = kdv.kdv_verify_attn_workspace(_params(num_splits=3))
    parts = 3 * 3 * 4
    assert n == ((parts * 64 * 4 + 255) // 256) * 256 + parts * 4
    # the tensor-core kernel keeps its merge partials o_k in fp16, then the
    # fp16 latent rows of every key the call reads (L + T = 8 here, 1 KB each)
    al = lambda x: ((x + 255) // 256) * 256
    p = _params(num_splits=3, dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, impl=kdv.KDV_IMPL_TC)
    n = kdv.kdv_verify_attn_workspace(p)
    assert n == al(al(parts * 512 * 2) + parts * 4) + al(8 * 1024)
    # ... unless the caller passes those rows
    p = _params(num_splits=3, dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, impl=kdv.KDV_IMPL_TC, v16=0x10000)
    assert kdv.kdv_verify_attn_workspace(p) == al(parts * 512 * 2) + parts * 4
    # a single split: only the fp16 rows
    p = _params(num_splits=1, dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, impl=kdv.KDV_IMPL_TC)
    assert kdv.kdv_verify_attn_workspace(p) == al(8 * 1024)
    # partials returned to the caller: no workspace
    assert kdv.kdv_verify_attn_workspace(_params(num_splits=3, return_partials=1)) == 0


def test_tensor_core_path_takes_positive_scales_only(lib):
    """The TC kernel takes its row maxima over unscaled logits, so it needs
    scale > 0: forced, a non-positive scale is refused; AUTO sends it to the
    SIMT kernel (one launch, no fp16 latent pass)."""
    tc = dict(dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, num_splits=1)
    for scale in (0.0, -0.1):
        n = ctypes.c_size_t(0)
        p = _params(impl=kdv.KDV_IMPL_TC, scale=scale, **tc)
        assert lib.kdv_verify_attn_workspace(ctypes.byref(p), ctypes.byref(n)) == kdv.KDV_ERR_UNSUPPORTED
        assert kdv.kdv_verify_attn_launches(_params(impl=kdv.KDV_IMPL_AUTO, scale=scale, **tc)) == 1
    assert kdv.kdv_verify_attn_launches(_params(impl=kdv.KDV_IMPL_AUTO, scale=0.1, **tc)) == 2


def test_launch_counts(lib):
    """Kernels one kdv_verify_attn call launches (host planning only)."""
    tc = dict(dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, impl=kdv.KDV_IMPL_TC)
    assert kdv.kdv_verify_attn_launches(_params(num_splits=1)) == 1                  # SIMT, direct
    assert kdv.kdv_verify_attn_launches(_params(num_splits=3)) == 2                  # SIMT + merge
    assert kdv.kdv_verify_attn_launches(_params(num_splits=3, return_partials=1)) == 1
    assert kdv.kdv_verify_attn_launches(_params(num_splits=1, **tc)) == 2            # latent + TC
    assert kdv.kdv_verify_attn_launches(_params(num_splits=1, v16=0x10000, **tc)) == 1
    assert kdv.kdv_verify_attn_launches(_params(num_splits=3, v16=0x10000, **tc)) == 2
    assert kdv.kdv_verify_attn_launches(_params(num_splits=3, **tc)) == 3              # + merge
    st = dict(tc, impl=kdv.KDV_IMPL_TC_STAGED, page_table=0x7000)
    assert kdv.kdv_verify_attn_launches(_params(num_splits=1, v16=0x10000, **st)) == 2
    n = ctypes.c_int32(0)
    assert lib.kdv_verify_attn_launches(None, ctypes.byref(n)) == kdv.KDV_ERR_INVALID_ARG
    assert lib.kdv_verify_attn_launches(ctypes.byref(_params()), None) == kdv.KDV_ERR_INVALID_ARG


def test_mask_build_validation(lib):
    f = lib.kdv_tree_mask_build
    assert f(None, None, 1, 4, 0x1000, None, None, None) == kdv.KDV_ERR_INVALID_ARG
    assert f(0x1000, None, 1, 65, 0x2000, None, None, None) == kdv.KDV_ERR_UNSUPPORTED
    assert f(0x1000, None, 2, 4, 0x2000, None, None, None) == kdv.KDV_ERR_INVALID_ARG
    assert f(0x1000, None, 1, 0, 0x2000, None, None, None) == kdv.KDV_ERR_INVALID_ARG
    assert f(0x1000, None, 1, 4, 0x2004, None, None, None) == kdv.KDV_ERR_INVALID_ARG


def test_combine_validation(lib):
    f = lib.kdv_combine
    assert f(None, None, 0, 4, 8, None, None, None) == kdv.KDV_ERR_INVALID_ARG
    assert f(None, None, 2, 4, 8, None, None, None) == kdv.KDV_ERR_INVALID_ARG
    assert f(None, None, 2, -1, 8, None, None, None) == kdv.KDV_ERR_INVALID_ARG


def _accept(**over):
    base = dict(batch=2, max_T=8, total_nodes=10, vocab=1000, dtype=kdv.KDV_BF16, logits=0x1000,
                logits_ld=1000, target_in=None, token=0x2000, parent=0x3000, tree_off=0x4000,
                target_out=None, accept_len=0x5000, accept_path=0x6000, bonus=None,
                page_table=None, kv_off=None, prefix_len=None, prefix_len_out=None,
                workspace=None, workspace_bytes=0, d_err=None)
    base.update(over)
    return kdv.make_accept_params(**base)


@pytest.mark.parametrize("over,status", [
    (dict(batch=0), kdv.KDV_ERR_UNSUPPORTED),
    (dict(batch=129, total_nodes=129), kdv.KDV_ERR_UNSUPPORTED),
    (dict(max_T=65), kdv.KDV_ERR_UNSUPPORTED),
    (dict(total_nodes=17), kdv.KDV_ERR_INVALID_ARG),          # > batch * max_T
    (dict(total_nodes=1), kdv.KDV_ERR_INVALID_ARG),           # < batch
    (dict(vocab=0), kdv.KDV_ERR_INVALID_ARG),
    (dict(dtype=5), kdv.KDV_ERR_INVALID_ARG),
    (dict(logits_ld=999), kdv.KDV_ERR_INVALID_ARG),
    (dict(logits=None), kdv.KDV_ERR_INVALID_ARG),             # neither logits nor target_in
    (dict(token=None), kdv.KDV_ERR_INVALID_ARG),
    (dict(accept_path=None), kdv.KDV_ERR_INVALID_ARG),
    (dict(page_table=0x7000), kdv.KDV_ERR_INVALID_ARG),       # no kv_off / prefix_len
    (dict(prefix_len_out=0x7000), kdv.KDV_ERR_INVALID_ARG),   # no prefix_len
])
def test_accept_host_validation(lib, over, status):
    p = _accept(**over)
    n = ctypes.c_size_t(0)
    assert lib.kdv_tree_accept_workspace(ctypes.byref(p), ctypes.byref(n)) == status
    assert lib.kdv_tree_accept(ctypes.byref(p), None) == status


def test_accept_workspace(lib):
    # one 64-bit key per (node, 8192-logit chunk)
    assert kdv.kdv_tree_accept_workspace(_accept()) == 10 * 1 * 8
    assert kdv.kdv_tree_accept_workspace(_accept(vocab=163840, logits_ld=163840)) == 10 * 20 * 8
    assert kdv.kdv_tree_accept_workspace(_accept(logits=None, target_in=0x1000)) == 0
    # a missing workspace is refused before any launch
    assert lib.kdv_tree_accept(ctypes.byref(_accept()), None) == kdv.KDV_ERR_WORKSPACE


def test_library_has_no_oracle_dependency():
    """The CUDA library and its binding never reference the oracle."""
    pkg = os.path.join(ROOT, "speculative_tree_verify_mla_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, fn
                assert "kdv_oracle" not in txt, fn


def test_oracle_has_no_cuda_path_dependency():
    """The oracle shares no code with the CUDA path: its sources never import
    the package, load libkdv or include the library's headers."""
    odir = os.path.join(ROOT, "oracle")
    for fn in os.listdir(odir):
        if fn.endswith((".py", ".cpp", ".c", ".h")):
            txt = open(os.path.join(odir, fn)).read()
            assert "speculative_tree_verify_mla_b200" not in txt, fn
            assert "libkdv.so" not in txt and "kdv.h" not in txt and "csrc" not in txt, fn


def test_projection_validation(lib):
    fa, fu = lib.kdv_absorb_q, lib.kdv_unabsorb_o
    B, F = kdv.KDV_BF16, kdv.KDV_F32
    # rows not a multiple of H; null pointers; strides shorter than rows; dtypes; limits
    assert fa(13, 4, 512, 128, 0x1000, 128, B, 0x2000, B, 0x3000, 576, B, None) == kdv.KDV_ERR_INVALID_ARG
    assert fa(16, 4, 512, 128, None, 128, B, 0x2000, B, 0x3000, 576, B, None) == kdv.KDV_ERR_INVALID_ARG
    assert fa(16, 4, 512, 128, 0x1000, 100, B, 0x2000, B, 0x3000, 576, B, None) == kdv.KDV_ERR_INVALID_ARG
    assert fa(16, 4, 512, 128, 0x1000, 128, 9, 0x2000, B, 0x3000, 576, B, None) == kdv.KDV_ERR_INVALID_ARG
    assert fa(16, 4, 512, 600, 0x1000, 600, B, 0x2000, B, 0x3000, 576, B, None) == kdv.KDV_ERR_UNSUPPORTED
    assert fa(0, 4, 512, 128, None, 128, B, None, B, None, 576, B, None) == kdv.KDV_OK
    assert fu(13, 4, 512, 128, 0x1000, 512, 0x2000, B, 0x3000, 128, F, None) == kdv.KDV_ERR_INVALID_ARG
    assert fu(16, 4, 513, 128, 0x1000, 513, 0x2000, B, 0x3000, 128, F, None) == kdv.KDV_ERR_UNSUPPORTED
    assert fu(16, 4, 512, 128, 0x1000, 512, 0x2000, B, 0x3000, 100, F, None) == kdv.KDV_ERR_INVALID_ARG
    # the flagged forms validate the same way and refuse unknown flag bits
    fax, fux = lib.kdv_absorb_q_ex, lib.kdv_unabsorb_o_ex
    S = kdv.KDV_PROJ_STATIC_WEIGHTS
    assert fax(13, 4, 512, 128, 0x1000, 128, B, 0x2000, B, 0x3000, 576, B, S, None) == kdv.KDV_ERR_INVALID_ARG
    assert fax(0, 4, 512, 128, None, 128, B, None, B, None, 576, B, S, None) == kdv.KDV_OK
    assert fax(0, 4, 512, 128, None, 128, B, None, B, None, 576, B, 2, None) == kdv.KDV_ERR_INVALID_ARG
    assert fux(16, 4, 513, 128, 0x1000, 513, 0x2000, B, 0x3000, 128, F, S, None) == kdv.KDV_ERR_UNSUPPORTED
    assert fux(16, 4, 512, 128, 0x1000, 512, 0x2000, B, 0x3000, 128, F, 4, None) == kdv.KDV_ERR_INVALID_ARG


def test_tree_build_validation(lib):
    def bp(**over):
        base = dict(batch=2, max_T=32, depth=15, topk=8, tree_off=0x1000, root_token=0x2000,
                    cand_token=0x3000, cand_logp=0x4000, parent=0x5000, token=0x6000, depth_out=None,
                    score=None, d_err=None)
        base.update(over)
        return kdv.make_build_params(**base)
    f = lambda **o: lib.kdv_tree_build(ctypes.byref(bp(**o)), None)
    assert f(batch=0) == kdv.KDV_ERR_UNSUPPORTED
    assert f(max_T=65) == kdv.KDV_ERR_UNSUPPORTED
    assert f(depth=17) == kdv.KDV_ERR_UNSUPPORTED
    assert f(topk=9) == kdv.KDV_ERR_UNSUPPORTED
    assert f(topk=0) == kdv.KDV_ERR_UNSUPPORTED
    assert f(parent=None) == kdv.KDV_ERR_INVALID_ARG
    assert f(cand_logp=None) == kdv.KDV_ERR_INVALID_ARG
    assert lib.kdv_tree_build(None, None) == kdv.KDV_ERR_INVALID_ARG


def test_staged_workspace_size(lib):
    al = lambda x: ((x + 255) // 256) * 256
    # forced single split (no merge region): the fp16 latent rows, then the
    # staged offsets [B+1], the staged k_rope rows, then q_lat in fp16
    # (T * H = 3 * 4 rows)
    p = _params(dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, impl=kdv.KDV_IMPL_TC_STAGED,
                page_table=0x7000, num_splits=1, h_prefix_len=[100], h_tree_T=[3])
    assert kdv.kdv_verify_attn_workspace(p) == al(103 * 1024) + 256 + al(103 * 64 * 2) + 3 * 4 * 512 * 2
    # the caller's fp16 rows: the staged region starts the workspace ...
    p.v16 = 0x10000
    assert kdv.kdv_verify_attn_workspace(p) == 256 + al(103 * 64 * 2) + 3 * 4 * 512 * 2
    # ... or follows the merge region (3 splits: 3 * 12 partial rows)
    p = _params(dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, impl=kdv.KDV_IMPL_TC_STAGED,
                page_table=0x7000, num_splits=3, h_prefix_len=[100], h_tree_T=[3], v16=0x10000)
    parts = 3 * 3 * 4
    assert kdv.kdv_verify_attn_workspace(p) == \
        al(al(parts * 512 * 2) + parts * 4) + 256 + al(103 * 64 * 2) + 3 * 4 * 512 * 2
    # reading the pool through the page table needs only the fp16 rows
    p = _params(dtype=kdv.KDV_BF16, d_latent=512, d_rope=64, impl=kdv.KDV_IMPL_TC,
                page_table=0x7000, num_splits=1, h_prefix_len=[100], h_tree_T=[3])
    assert kdv.kdv_verify_attn_workspace(p) == al(103 * 1024)
    # impl codes past the last one are rejected
    n = ctypes.c_size_t(0)
    assert lib.kdv_verify_attn_workspace(ctypes.byref(_params(impl=5)), ctypes.byref(n)) == \
        kdv.KDV_ERR_INVALID_ARG
