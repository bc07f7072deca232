"""Parity metric shared by the GPU tests.

Bars (the stated tolerance, read on unit-scale outputs): errors of o_lat are
divided by the RMS of the oracle's o_lat over the tensor, because o_lat
entries shrink like 1/sqrt(L) with context while the inputs stay N(0,1):

    normalised max |err| <= 1e-2, normalised mean |err| <= 1e-3,
    |lse err| <= 1e-3 (absolute, natural log).

The absolute errors are held to the same 1e-2 / 1e-3 as well (they are the
looser pair whenever RMS(o_ref) < 1).

What the bf16 tensor-core path is expected to give: its only rounding beyond
fp32 accumulation is that of the softmax numerators P, which it rounds to
fp16 before P.V (unit roundoff 2^-11). Weight j then carries a relative
error delta_j, uniform within +-2^-11/m_j for mantissa m_j in [1, 2), and
o's error is sum_j w_j delta_j v_j: normal with standard deviation
std(delta) * RMS(o), std(delta) = 2^-11 * sqrt(E[1/m^2] / 3) ~ 2.1e-4 for
log-uniform mantissas. That puts the normalised mean error near
sqrt(2/pi) * 2.1e-4 ~ 1.7e-4 and the max over ~1e5..1e6 elements at 4-5
standard deviations, ~1e-3. A CPU emulation of the kernel's arithmetic
gives 1.3e-4 and 0.6e-3..1.0e-3 on the Kimi-shape cases. fp32 paths pass
far tighter bars, set per test.
"""
import numpy as np

MAX_TOL = 1e-2       # absolute, stated
MEAN_TOL = 1e-3      # absolute, stated
LSE_TOL = 1e-3       # absolute, stated
REL_MAX_TOL = 1e-2   # normalised by RMS(o_ref)
REL_MEAN_TOL = 1e-3


def parity_stats(o, lse, o_ref, lse_ref):
    o = np.asarray(o, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(o_ref ** 2))) if o_ref.size else 1.0
    rms = rms or 1.0
    err = np.abs(o - o_ref)
    lse = np.asarray(lse, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin), "lse finiteness differs"
    lse_err = np.abs(lse[fin] - lse_ref[fin])
    mx = float(err.max()) if err.size else 0.0
    mn = float(err.mean()) if err.size else 0.0
    return dict(max=mx, mean=mn, rel_max=mx / rms, rel_mean=mn / rms,
                lse=float(lse_err.max()) if lse_err.size else 0.0, rms=rms)


def assert_parity(o, lse, o_ref, lse_ref, max_tol=MAX_TOL, mean_tol=MEAN_TOL, lse_tol=LSE_TOL,
                  rel_max_tol=REL_MAX_TOL, rel_mean_tol=REL_MEAN_TOL):
    assert np.all(np.isfinite(o)), "non-finite output"
    st = parity_stats(o, lse, o_ref, lse_ref)
    ok = (st["max"] <= max_tol and st["mean"] <= mean_tol and st["lse"] <= lse_tol
          and st["rel_max"] <= rel_max_tol and st["rel_mean"] <= rel_mean_tol)
    assert ok, st
    return st


def assert_parity_fp32(o, lse, o_ref, lse_ref, tol=1e-5):
    """fp32 inputs and arithmetic: every bar at ``tol`` (relative ones too)."""
    return assert_parity(o, lse, o_ref, lse_ref, max_tol=tol, mean_tol=tol / 10, lse_tol=tol,
                         rel_max_tol=tol * 100, rel_mean_tol=tol * 10)
