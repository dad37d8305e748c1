"""Comparison helpers: GPU outputs against the oracle, with the bands the
stated tolerances allow (each band's reading is on its constant in oracle/tq_oracle.py)."""

from __future__ import annotations

import numpy as np

from oracle import tq_oracle as O


def tables_of(ctx) -> O.Tables:
    """Oracle tables for a library context (built by the oracle from the seed)."""
    return O.make_tables(ctx.d, ctx.bits, ctx.seed, m=ctx.m)


def check_quantize(payload, norms, K64, tb: O.Tables, report=None):
    """payload (N, row_bytes) uint8 and norms (N, 2) fp16 from the GPU against
    the oracle's quantisation of the exact inputs K64 (N, d) float64.

    Codes must be equal except within CODE_BAND of a boundary; sign bits equal
    except within SIGN_BAND of 0 or in a key with an excused code difference;
    fp16 norms equal except within NORM_BAND of a rounding midpoint (then one
    ulp either way).  Mismatching coordinates must stay below 1e-4.
    """
    payload = np.asarray(payload)
    norms = np.asarray(norms).view(np.float16).reshape(-1, 2)
    qz = O.quantize(K64, tb)
    codes, bits = O.unpack_rows(payload, tb.d, tb.m, tb.bmse)
    pad_c, pad_b = O.unpack_padding(payload, tb.d, tb.m, tb.bmse)
    assert not pad_c.any() and not pad_b.any(), "layout padding slots must be zero"
    code_mis = codes != qz.codes
    code_band = O.code_boundary_distance(qz.u, tb.t) <= O.CODE_BAND
    bad_codes = code_mis & ~code_band
    assert not bad_codes.any(), f"{bad_codes.sum()} codes differ outside the band, e.g. {np.argwhere(bad_codes)[:5]}"
    frac_code = code_mis.mean()
    assert frac_code < 1e-4, frac_code
    key_exc = code_mis.any(axis=1)
    sign_mis = bits != qz.bits
    sign_band = O.sign_boundary_distance(qz.z, qz.n, tb.m) <= O.SIGN_BAND
    bad_signs = sign_mis & ~sign_band & ~key_exc[:, None]
    assert not bad_signs.any(), f"{bad_signs.sum()} sign bits differ outside the band, e.g. {np.argwhere(bad_signs)[:5]}"
    frac_sign = float((sign_mis & ~key_exc[:, None]).mean()) if sign_mis.size else 0.0   # m = 0: no sign bits
    assert frac_sign < 1e-4, frac_sign

    def norm_ok(gpu16, exact, excused):
        want = exact.astype(np.float16)
        same = gpu16 == want
        near = O.fp16_midpoint_distance(exact) <= O.NORM_BAND
        one_ulp = np.abs(gpu16.astype(np.float64) - want.astype(np.float64)) <= \
            np.abs(np.spacing(want).astype(np.float64)) * 1.0001
        ok = same | (near & one_ulp) | excused
        return ok

    nk_ok = norm_ok(norms[:, 0], qz.n, np.zeros(len(qz.n), bool))
    assert nk_ok.all(), f"||k|| differs: {np.argwhere(~nk_ok)[:5].ravel()}"
    nr_ok = norm_ok(norms[:, 1], qz.rho, key_exc)
    assert nr_ok.all(), f"||r|| differs: {np.argwhere(~nr_ok)[:5].ravel()}"
    stats = dict(code_mismatch=float(frac_code), sign_mismatch=float(frac_sign),
                 code_near_boundary=float(code_band.mean()) if code_band.size else 0.0,
                 sign_near_boundary=float(sign_band.mean()) if sign_band.size else 0.0,   # m = 0: no sign bits
                 keys=int(len(qz.n)))
    if report is not None:
        report.update(stats)
    return stats, qz


def oracle_estimates(payload, norms, Q64, tb: O.Tables):
    """Estimator values (and abs-sum A) computed by the oracle from packed rows."""
    codes, bits = O.unpack_rows(np.asarray(payload), tb.d, tb.m, tb.bmse)
    nr = np.asarray(norms).view(np.float16).reshape(-1, 2)
    return O.estimate(Q64, codes, bits, nr[:, 0], nr[:, 1], tb)


def check_close(gpu, ref, A, tol=1e-3):
    """|gpu - ref| <= tol * A elementwise (the logits tolerance)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    worst = float(np.max(err / np.maximum(A, 1e-30)))
    assert np.all(err <= tol * A), f"worst relative-to-A error {worst}"
    return worst
