"""Parity metric shared by the GPU tests.

Two sets of bars, both checked:

1. The stated tolerance, on absolute errors of o_lat and lse. Every workload
   draws its activations from N(0,1) (unit scale), so absolute errors are the
   errors "on unit-scale outputs": max |err| <= 1e-2, mean |err| <= 1e-3,
   |lse err| <= 1e-3.

2. Relative bars, which keep the check sharp at long context where o_lat
   entries shrink like 1/sqrt(L). Errors are divided by the RMS of the
   oracle's o_lat. The tensor-core path rounds the softmax numerators P to
   bf16 before P.V. The unit roundoff is u = 2^-9, so each weight carries a
   relative error up to u. That alone gives a normalised mean error of about
   sqrt(2/pi) * u/sqrt(3) ~ 0.9e-3, and a max a few times larger. The bars
   are mean <= 2e-3 (~2x the bf16 floor) and max <= 3e-2. fp32 paths pass
   far tighter bars, set per test.
"""
import numpy as np

MAX_TOL = 1e-2       # absolute, stated
MEAN_TOL = 1e-3      # absolute, stated
LSE_TOL = 1e-3       # absolute, stated
REL_MAX_TOL = 3e-2   # normalised by RMS(o_ref), derived from bf16 P rounding
REL_MEAN_TOL = 2e-3


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
