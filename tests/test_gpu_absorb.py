"""GPU parity of kdv_absorb_q / kdv_unabsorb_o against the oracle, and the
whole absorbed layer (absorb -> verify -> up-project) against the oracle's
non-absorbed MLA.

The projections are the latent projection the verify kernel absorbs (page
"The Architecture of Diagnosis", section "Phase 1: Custom CUDA Kernels",
item 2). Accumulation is fp32 on every GPU kernel (the tensor-core forms take
bf16 weights and bf16 q_nope; the up-projection feeds its fp32 o_lat to them as
a bf16 hi + lo pair), so fp32 outputs are held to a relative 2e-5 and bf16
outputs to one bf16 unit in the last place. Node counts of 40 and 70 take
several passes of the tensor-core kernels (64 and 32 nodes per pass).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from speculative_tree_verify_mla_b200 import datagen, kdv
from tests.parity import LSE_TOL, REL_MAX_TOL, REL_MEAN_TOL, assert_parity, parity_stats

pytestmark = pytest.mark.gpu
dev = "cuda"


def _t(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dtype).to(dev)


def _rel_err(got, want):
    return np.abs(got - want).max() / np.abs(want).max()


@pytest.mark.parametrize("T,wdt", [(13, torch.bfloat16), (1, torch.bfloat16), (40, torch.bfloat16),
                                   (70, torch.bfloat16), (13, torch.float32)])
def test_absorb_q_kimi(T, wdt):
    case = datagen.kimi_layer_case(L=64, T=T, seed=5)
    q_nope, w_uk, _ = datagen.layer_weights(case)
    ref = oracle.absorb_q(case.H, q_nope, w_uk)
    out = torch.full((case.rows, 512), float("nan"), device=dev)
    kdv.kdv_absorb_q(case.H, _t(q_nope, wdt), _t(w_uk, wdt), out)
    torch.cuda.synchronize()
    assert _rel_err(out.cpu().numpy(), ref) < 2e-5


def test_absorb_q_into_verify_rows_bf16():
    """q_lat written as bf16 straight into the first 512 columns of 576-wide
    q rows; the q_rope columns stay untouched."""
    case = datagen.kimi_layer_case(L=64, T=13, seed=6)
    q_nope, w_uk, _ = datagen.layer_weights(case)
    ref = oracle.absorb_q(case.H, q_nope, w_uk)
    q = torch.full((case.rows, 576), 3.0, dtype=torch.bfloat16, device=dev)
    kdv.kdv_absorb_q(case.H, _t(q_nope, torch.bfloat16), _t(w_uk, torch.bfloat16), q[:, :512])
    torch.cuda.synchronize()
    got = q.float().cpu().numpy()
    assert np.all(got[:, 512:] == 3.0)
    # round-to-nearest-even of the fp32 sum: within one bf16 ulp of the exact
    # value, plus the fp32 accumulation error of a 128-term sum (for entries
    # near zero, where one ulp is tiny)
    assert np.all(np.abs(got[:, :512] - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-6)


@pytest.mark.parametrize("T,out_dt", [(13, torch.float32), (40, torch.float32), (70, torch.float32),
                                      (13, torch.bfloat16)])
def test_unabsorb_o_kimi(T, out_dt):
    case = datagen.kimi_layer_case(L=64, T=T, seed=7)
    _, _, w_uv = datagen.layer_weights(case)
    o_lat = np.random.default_rng(T).standard_normal((case.rows, 512)).astype(np.float32) * 0.05
    ref = oracle.unabsorb_o(case.H, o_lat, w_uv)
    out = torch.full((case.rows, 128), float("nan"), dtype=out_dt, device=dev)
    kdv.kdv_unabsorb_o(case.H, _t(o_lat), _t(w_uv, torch.bfloat16), out)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    if out_dt == torch.float32:
        assert _rel_err(got, ref) < 2e-5
    else:
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-6)


def _bf16_exact(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).bfloat16().float().numpy()


@pytest.mark.parametrize("H,T,D_c,D_n,D_v,pad", [(3, 5, 200, 72, 40, 0), (2, 17, 136, 8, 8, 0),
                                                 (1, 33, 512, 512, 96, 0), (2, 3, 100, 16, 24, 3)])
def test_projections_ragged_shapes_bf16_weights(H, T, D_c, D_n, D_v, pad):
    """bf16 weights with shapes that leave every tile ragged: weight rows not
    a multiple of the 128-row tile, k not a multiple of the 64-wide box, d not
    a multiple of the 8-way phase split, columns not a multiple of 32, and node
    counts across several 16-node passes; pad > 0 gives the input rows a
    stride that is not a multiple of 8 elements (element-wise staging)."""
    rng = np.random.default_rng(H * 1000 + T)
    rows = H * T
    q_nope = _bf16_exact(rng.standard_normal((rows, D_n)))
    w_uk = _bf16_exact(rng.standard_normal((H, D_c, D_n)) * D_n ** -0.5)
    w_uv = _bf16_exact(rng.standard_normal((H, D_c, D_v)) * D_c ** -0.5)
    o_lat = rng.standard_normal((rows, D_c)).astype(np.float32)
    q_in = torch.zeros(rows, D_n + pad, dtype=torch.bfloat16, device=dev)
    q_in[:, :D_n] = _t(q_nope, torch.bfloat16)
    o_in = torch.zeros(rows, D_c + pad, device=dev)
    o_in[:, :D_c] = _t(o_lat)
    q_lat = torch.full((rows, D_c), float("nan"), device=dev)
    kdv.kdv_absorb_q(H, q_in[:, :D_n], _t(w_uk, torch.bfloat16), q_lat)
    out = torch.full((rows, D_v), float("nan"), device=dev)
    kdv.kdv_unabsorb_o(H, o_in[:, :D_c], _t(w_uv, torch.bfloat16), out)
    torch.cuda.synchronize()
    assert _rel_err(q_lat.cpu().numpy(), oracle.absorb_q(H, q_nope, w_uk)) < 2e-5
    assert _rel_err(out.cpu().numpy(), oracle.unabsorb_o(H, o_lat, w_uv)) < 2e-5


def test_tiny_layer_end_to_end_fp32():
    """The tiny fp32 layer through the GPU: absorb, verify (SIMT), up-project,
    against the oracle's non-absorbed MLA (explicit K = c_kv W_UK, V = c_kv W_UV)."""
    case = datagen.tiny_fp32_case()
    q_nope, w_uk, w_uv = datagen.tiny_fp32_layer(case)
    D_c, D_r, H = case.D_c, case.D_r, case.H
    L, T = int(case.prefix_len[0]), int(case.tree_T[0])
    out_ref, lse_ref = oracle.verify_mla(H=H, L=L, parent=case.parent, D_c=D_c, D_r=D_r, D_n=case.D_n,
                                         D_v=case.D_v, scale=case.scale, q_nope=q_nope,
                                         q_rope=case.q[:, D_c:], c_kv=case.kv[:, :D_c],
                                         k_rope=case.kv[:, D_c:], w_uk=w_uk, w_uv=w_uv)
    dc = kdv.DeviceCase(case, impl=kdv.KDV_IMPL_SIMT, num_splits=2)
    dc.q[:, :D_c] = float("nan")                           # the absorb must fill these
    kdv.kdv_absorb_q(H, _t(q_nope), _t(w_uk), dc.q[:, :D_c])
    dc.run()
    out = torch.empty(case.rows, case.D_v, device=dev)
    kdv.kdv_unabsorb_o(H, dc.o, _t(w_uv), out)
    torch.cuda.synchronize()
    assert dc.error_flag() == 0
    np.testing.assert_allclose(out.cpu().numpy(), out_ref, rtol=2e-5, atol=2e-6)
    np.testing.assert_allclose(dc.lse.cpu().numpy(), lse_ref, rtol=2e-5, atol=2e-6)


def test_kimi_layer_end_to_end_bf16():
    """Kimi shape at L=1500: bf16 absorb written into the bf16 q rows, the
    tensor-core verify, fp32 up-projection.

    Two checks. (1) The attention kernel against the oracle on the very q
    rows the GPU absorb produced (read back from the device): the standard
    bars. (2) The whole layer against the oracle's non-absorbed MLA in fp64.
    Here the q rows' bf16 storage of q_lat (the kernel's input type) adds an
    error no kernel can remove; the oracle itself, run in fp64 on the same
    rounded q_lat and up-projected, measures that floor, and the layer must
    stay within floor + the standard bars."""
    case = datagen.kimi_layer_case(L=1500, T=13, seed=8)
    q_nope, w_uk, w_uv = datagen.layer_weights(case)
    L, T = 1500, 13
    out_ref, lse_ref = oracle.verify_mla(H=64, L=L, parent=case.parent, D_c=512, D_r=64, D_n=128,
                                         D_v=128, scale=case.scale, q_nope=q_nope,
                                         q_rope=case.q[:, 512:], c_kv=case.kv[:, :512],
                                         k_rope=case.kv[:, 512:], w_uk=w_uk, w_uv=w_uv)
    dc = kdv.DeviceCase(case, num_splits=0)
    kdv.kdv_absorb_q(64, _t(q_nope, torch.bfloat16), _t(w_uk, torch.bfloat16), dc.q[:, :512])
    dc.run()
    out = torch.empty(case.rows, 128, device=dev)
    kdv.kdv_unabsorb_o(64, dc.o, _t(w_uv, torch.bfloat16), out)
    torch.cuda.synchronize()
    assert dc.error_flag() == 0
    # (1) the kernel on its actual inputs
    q_gpu = dc.q.float().cpu().numpy()
    case_gpu = dataclasses.replace(case, q=q_gpu)
    o_abs, lse_abs = oracle.verify_case(case_gpu)
    assert_parity(dc.o.cpu().numpy(), dc.lse.cpu().numpy(), o_abs, lse_abs)
    # (2) the layer: the fp64 floor of bf16 q_lat, then floor + bars
    floor = parity_stats(oracle.unabsorb_o(64, o_abs, w_uv), lse_abs, out_ref, lse_ref)
    st = parity_stats(out.cpu().numpy(), dc.lse.cpu().numpy(), out_ref, lse_ref)
    assert st["rel_max"] <= floor["rel_max"] + REL_MAX_TOL, (st, floor)
    assert st["rel_mean"] <= floor["rel_mean"] + REL_MEAN_TOL, (st, floor)
    assert st["lse"] <= floor["lse"] + LSE_TOL, (st, floor)


@pytest.mark.parametrize("T", [13, 70])
def test_static_weights_flag_gives_the_same_bits(T):
    """KDV_PROJ_STATIC_WEIGHTS only changes when the weight copies may start
    (programmatic dependent launch), not what is computed: a chain of flagged
    calls -- each a dependent of the one before, the outputs of one call the
    inputs of the next -- must give the plain calls' bits."""
    case = datagen.kimi_layer_case(L=64, T=T, seed=7)
    q_nope, w_uk, w_uv = datagen.layer_weights(case)
    qn, wk, wv = _t(q_nope, torch.bfloat16), _t(w_uk, torch.bfloat16), _t(w_uv, torch.bfloat16)
    outs = []
    for flags in (0, kdv.KDV_PROJ_STATIC_WEIGHTS):
        q = torch.zeros(case.rows, 576, dtype=torch.bfloat16, device=dev)
        o_lat = torch.empty(case.rows, 512, device=dev)
        out = torch.empty(case.rows, 128, device=dev)
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            for _ in range(3):
                kdv.kdv_absorb_q(case.H, qn, wk, q[:, :512], s, flags=flags)
                o_lat.copy_(q[:, :512].float() * 0.01)          # a kernel between that reads the output
                kdv.kdv_unabsorb_o(case.H, o_lat, wv, out, s, flags=flags)
                kdv.kdv_unabsorb_o(case.H, o_lat, wv, out, s, flags=flags)   # back to back
        s.synchronize()
        outs.append((q.cpu(), out.cpu()))
    assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16))
    assert torch.equal(outs[0][1].view(torch.int32), outs[1][1].view(torch.int32))
