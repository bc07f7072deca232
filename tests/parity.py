"""Parity metric shared by the GPU tests.

Errors on o_lat are divided by the RMS of the oracle's o_lat over the compared
tensor ("unit-scale outputs"): o_lat is an average of ~L latent rows, so its
entries shrink like 1/sqrt(L) and a raw 1e-2 bar would say nothing at long
context. Bars (fp: bf16 inputs, fp32 accumulation): normalised max |err| <=
1e-2, normalised mean |err| <= 1e-3, LSE absolute error <= 1e-3.
"""
import numpy as np

MAX_TOL = 1e-2
MEAN_TOL = 1e-3
LSE_TOL = 1e-3


def parity_stats(o, lse, o_ref, lse_ref):
    o = np.asarray(o, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(o_ref ** 2))) or 1.0
    err = np.abs(o - o_ref) / rms
    lse = np.asarray(lse, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin), "lse finiteness differs"
    lse_err = np.abs(lse[fin] - lse_ref[fin])
    return dict(max=float(err.max()) if err.size else 0.0,
                mean=float(err.mean()) if err.size else 0.0,
                lse=float(lse_err.max()) if lse_err.size else 0.0,
                rms=rms, raw_max=float(np.abs(o - o_ref).max()) if err.size else 0.0)


def assert_parity(o, lse, o_ref, lse_ref, max_tol=MAX_TOL, mean_tol=MEAN_TOL, lse_tol=LSE_TOL):
    st = parity_stats(o, lse, o_ref, lse_ref)
    assert np.all(np.isfinite(o)), "non-finite output"
    assert st["max"] <= max_tol and st["mean"] <= mean_tol and st["lse"] <= lse_tol, st
    return st
