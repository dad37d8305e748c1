"""Comparison helpers: GPU outputs against the oracle, with the bands the
stated tolerances allow (each band's reading is on its constant in oracle/tq_oracle.py)."""

from __future__ import annotations

import numpy as np

from oracle import tq_oracle as O

# The limit on the fraction of mismatching coordinates (codes or sign bits).
MISMATCH_LIMIT = 1e-4


def tables_of(ctx) -> O.Tables:
    """Oracle tables for a library context (built by the oracle from the seed)."""
    return O.make_tables(ctx.d, ctx.bits, ctx.seed, m=ctx.m)


def check_quantize(payload, norms, K64, tb: O.Tables, report=None):
    """payload (N, row_bytes) uint8 and norms (N, 2) fp16 from the GPU against
    the oracle's quantisation of the exact inputs K64 (N, d) float64.

    Codes must be equal except within CODE_BAND of a boundary; sign bits equal
    except within SIGN_BAND of 0 (cosine of the JL row and the residual) or in
    a key with an excused code difference; fp16 norms equal except near a
    rounding midpoint (O.norm_band: 1e-5 on the unit-sphere scale; then one
    ulp either way).  Mismatching coordinates must stay below 1e-4.

    Returns (stats, quantized): stats holds the reported fractions
    (mismatching codes and sign bits, coordinates near a boundary) plus the
    sign mismatches that the literal narrower band |(S r)_i| <= 1e-5 ||r||
    would not excuse (diagnostic, not asserted).  With `report` (a dict),
    the stats are also merged into it.
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
    frac_code = float(code_mis.mean()) if code_mis.size else 0.0
    assert frac_code < MISMATCH_LIMIT, frac_code
    key_exc = code_mis.any(axis=1)
    sign_mis = bits != qz.bits
    sdist = O.sign_boundary_distance(qz.z, qz.rho, tb.S)
    sign_band = sdist <= O.SIGN_BAND
    bad_signs = sign_mis & ~sign_band & ~key_exc[:, None]
    assert not bad_signs.any(), f"{bad_signs.sum()} sign bits differ outside the band, e.g. {np.argwhere(bad_signs)[:5]}"
    own_sign_mis = sign_mis & ~key_exc[:, None]
    frac_sign = float(own_sign_mis.mean()) if sign_mis.size else 0.0   # m = 0: no sign bits
    assert frac_sign < MISMATCH_LIMIT, frac_sign
    narrow = np.abs(qz.z) <= 1e-5 * qz.rho[:, None]

    band_n, band_rho = O.norm_band(qz.n, qz.rho)

    def norm_ok(gpu16, exact, excused, band):
        want = exact.astype(np.float16)
        same = gpu16 == want
        near = O.fp16_midpoint_distance(exact) <= band
        one_ulp = np.abs(gpu16.astype(np.float64) - want.astype(np.float64)) <= \
            np.abs(np.spacing(want).astype(np.float64)) * 1.0001
        ok = same | (near & one_ulp) | excused
        return ok, same

    nk_ok, nk_same = norm_ok(norms[:, 0], qz.n, np.zeros(len(qz.n), bool), band_n)
    assert nk_ok.all(), f"||k|| differs: {np.argwhere(~nk_ok)[:5].ravel()}"
    nr_ok, nr_same = norm_ok(norms[:, 1], qz.rho, key_exc, band_rho)
    assert nr_ok.all(), f"||r|| differs: {np.argwhere(~nr_ok)[:5].ravel()}"
    stats = dict(keys=int(len(qz.n)), coords=int(code_mis.size), sign_bits=int(sign_mis.size),
                 code_mismatch=frac_code, sign_mismatch=frac_sign,
                 code_near_boundary=float(code_band.mean()) if code_band.size else 0.0,
                 sign_near_boundary=float(sign_band.mean()) if sign_band.size else 0.0,   # m = 0: no sign bits
                 sign_mismatch_outside_narrow_band=float((own_sign_mis & ~narrow).mean()) if sign_mis.size else 0.0,
                 keys_with_code_mismatch=int(key_exc.sum()),
                 norm_k_ulp_diffs=int((~nk_same).sum()), norm_r_ulp_diffs=int((~nr_same & ~key_exc).sum()))
    if report is not None:
        merge_stats(report, stats)
    return stats, qz


def merge_stats(acc: dict, stats: dict):
    """Accumulate check_quantize stats (fractions weighted by their counts)."""
    if not acc:
        acc.update(stats)
        return acc
    for key, w in (("code_mismatch", "coords"), ("code_near_boundary", "coords"), ("sign_mismatch", "sign_bits"),
                   ("sign_near_boundary", "sign_bits"), ("sign_mismatch_outside_narrow_band", "sign_bits")):
        tot = acc[w] + stats[w]
        acc[key] = (acc[key] * acc[w] + stats[key] * stats[w]) / tot if tot else 0.0
    for key in ("keys", "coords", "sign_bits", "keys_with_code_mismatch", "norm_k_ulp_diffs", "norm_r_ulp_diffs"):
        acc[key] += stats[key]
    return acc


def format_stats(stats: dict) -> str:
    return (f"{stats['keys']} keys: codes mismatching {stats['code_mismatch']:.2e} "
            f"(near a boundary {stats['code_near_boundary']:.2e}), sign bits mismatching "
            f"{stats['sign_mismatch']:.2e} (near 0 {stats['sign_near_boundary']:.2e}; outside |z| <= 1e-5 ||r||: "
            f"{stats['sign_mismatch_outside_narrow_band']:.2e})")


def oracle_estimates(payload, norms, Q64, tb: O.Tables):
    """Estimator values (and abs-sum A) computed by the oracle from packed rows."""
    codes, bits = O.unpack_rows(np.asarray(payload), tb.d, tb.m, tb.bmse)
    nr = np.asarray(norms).view(np.float16).reshape(-1, 2)
    return O.estimate(Q64, codes, bits, nr[:, 0], nr[:, 1], tb)


# Plain relative error is asserted (besides the A-scaled bound) where the
# estimate is at least this fraction of its term scale A.
REL_FLOOR = 0.05


def check_close(gpu, ref, A, tol=1e-3, rel_floor=None, report=None):
    """|gpu - ref| <= tol * A elementwise (the logits tolerance: A is the sum
    of the absolute values of the estimator's terms, since logits cross 0).
    With rel_floor, also |gpu - ref| <= tol * |ref| wherever |ref| >=
    rel_floor * A (the plain relative error, away from 0).
    Returns the worst A-relative error; with `report`, records both worsts."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    err = np.abs(gpu - ref)
    worst = float(np.max(err / np.maximum(A, 1e-30))) if err.size else 0.0
    assert np.all(err <= tol * A), f"worst relative-to-A error {worst}"
    if rel_floor is not None:
        big = np.abs(ref) >= rel_floor * A
        rel = err[big] / np.abs(ref[big])
        worst_rel = float(rel.max()) if rel.size else 0.0
        assert worst_rel <= tol, f"worst plain relative error {worst_rel} (|ref| >= {rel_floor} A)"
        if report is not None:
            report["logits_worst_rel"] = max(report.get("logits_worst_rel", 0.0), worst_rel)
            report["logits_rel_checked"] = report.get("logits_rel_checked", 0) + int(big.sum())
    if report is not None:
        report["logits_worst_of_A"] = max(report.get("logits_worst_of_A", 0.0), worst)
    return worst
