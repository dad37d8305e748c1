"""Pins for the CPU oracle: checks against facts fixed outside the oracle.

Each test pins one oracle function to something it does not compute itself:
published known-answer vectors, closed forms, textbook special cases,
invariants, brute force on tiny inputs and Monte-Carlo statistics with their
exact standard errors.  A plausible mistake in the oracle (a dropped term, a
wrong sign or index, a transposed operand) fails at least one of them.
"""

import math
import os

import numpy as np
import pytest
from scipy import integrate, special, stats

from oracle import tq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# Generator
# --------------------------------------------------------------------------


def _read_kat():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append([int(x, 16) for x in line.split()])
    return rows


def test_philox_known_answers():
    for row in _read_kat():
        out = O.philox4x32_10(np.array([row[:4]], dtype=np.uint64), row[4:6])[0]
        assert [int(x) for x in out] == row[6:10]


def test_gaussian_stream_is_standard_normal():
    z = O.gaussian_stream(seed=7, stream=3, count=400_001)
    assert z.shape == (400_001,)
    assert abs(z.mean()) < 4 / math.sqrt(z.size)
    assert abs(z.var() - 1) < 4 * math.sqrt(2 / z.size)
    assert stats.kstest(z, "norm").pvalue > 1e-3


def test_gaussian_streams_are_distinct_and_prefix_stable():
    a = O.gaussian_stream(1, 0, 1000)
    b = O.gaussian_stream(1, 1, 1000)
    c = O.gaussian_stream(2, 0, 1000)
    assert np.corrcoef(a, b)[0, 1] < 0.15 and np.corrcoef(a, c)[0, 1] < 0.15
    # counter-based: a prefix does not depend on how many values follow
    np.testing.assert_array_equal(O.gaussian_stream(1, 0, 17), a[:17])


# --------------------------------------------------------------------------
# Rotation
# --------------------------------------------------------------------------


@pytest.mark.parametrize("d", [8, 64, 128])
def test_rotation_orthogonal_and_norm_preserving(d):
    tb = O.make_tables(d, 3, seed=42)
    assert np.max(np.abs(tb.R.T @ tb.R - np.eye(d))) < 1e-12
    k = np.random.default_rng(0).standard_normal((20, d))
    np.testing.assert_allclose(np.linalg.norm(k @ tb.R.T, axis=1), np.linalg.norm(k, axis=1), rtol=1e-13)


def test_rotation_is_qr_factor_with_positive_diagonal():
    d = 16
    G = O.gaussian_stream(5, 0, d * d).reshape(d, d)
    R = O.haar_rotation(G)
    T = R.T @ G                               # must be upper triangular, positive diagonal
    assert np.max(np.abs(np.tril(T, -1))) < 1e-12
    assert np.all(np.diag(T) > 0)


def test_rotated_coordinates_follow_the_beta_law():
    # For a fixed unit vector and Haar R, each coordinate of R k follows f_d.
    d, nseed = 16, 4000
    k = np.zeros(d)
    k[0] = 1.0
    u = np.array([O.make_tables(d, 2, seed=s).R @ k for s in range(nseed)])
    assert abs(u[:, 3].mean()) < 4 / math.sqrt(d * nseed)
    assert abs(u.var() - 1 / d) < 0.05 / d
    cdf = lambda x: O.coord_cdf(x, d)
    assert stats.kstest(u[:, 5], cdf).pvalue > 1e-3


# --------------------------------------------------------------------------
# Coordinate law
# --------------------------------------------------------------------------


@pytest.mark.parametrize("d", [3, 4, 9, 64, 128])
def test_density_normalised_and_cdf_consistent(d):
    tot, _ = integrate.quad(lambda x: float(O.coord_density(x, d)), -1, 1, limit=200)
    assert abs(tot - 1) < 1e-9
    for x in (-0.3, 0.05, 0.2):
        part, _ = integrate.quad(lambda s: float(O.coord_density(s, d)), -1, x, limit=200)
        assert abs(part - float(O.coord_cdf(x, d))) < 1e-9
        mom, _ = integrate.quad(lambda s: s * float(O.coord_density(s, d)), x, 0.9, limit=200)
        assert abs(mom - float(O.coord_first_moment(x, 0.9, d))) < 1e-10


def test_large_d_law_tends_to_gaussian():
    d = 20000
    x = np.linspace(-3, 3, 13) / math.sqrt(d)
    np.testing.assert_allclose(O.coord_cdf(x, d), stats.norm.cdf(x * math.sqrt(d)), atol=2e-4)


# --------------------------------------------------------------------------
# Lloyd-Max codebook
# --------------------------------------------------------------------------


@pytest.mark.parametrize("bmse", [1, 2, 3, 4])
def test_codebook_d3_is_the_uniform_quantizer(bmse):
    # d = 3: f_3 is uniform on [-1, 1]; the optimal quantizer is uniform.
    c, t = O.lloyd_max_codebook(3, bmse)
    L = 1 << bmse
    np.testing.assert_allclose(c, -1 + (2 * np.arange(L) + 1) / L, atol=1e-12)
    np.testing.assert_allclose(t, -1 + 2 * np.arange(1, L) / L, atol=1e-12)


@pytest.mark.parametrize("d", [3, 8, 64, 128, 200])
def test_codebook_one_bit_closed_form(d):
    c, t = O.lloyd_max_codebook(d, 1)
    c1 = math.exp(special.gammaln(d / 2) - special.gammaln((d + 1) / 2)) / math.sqrt(math.pi)
    np.testing.assert_allclose(c, [-c1, c1], rtol=1e-12)
    assert t[0] == 0.0


def test_codebook_one_bit_value_at_d128():
    c, _ = O.lloyd_max_codebook(128, 1)
    assert abs(math.sqrt(128) * c[1] - 0.79944) < 1e-5


def _max_table():
    out = {}
    with open(os.path.join(GOLDEN, "gaussian_lloyd_max_levels.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                L, vals = line.split(":")
                out[int(L)] = [float(v) for v in vals.split()]
    return out


@pytest.mark.parametrize("bmse", [1, 2, 3])
def test_codebook_tends_to_max_gaussian_levels(bmse):
    ref = _max_table()[1 << bmse]
    d = 200000
    c, _ = O.lloyd_max_codebook(d, bmse)
    pos = math.sqrt(d) * c[len(c) // 2:]
    np.testing.assert_allclose(pos, ref, atol=1.5e-3)


@pytest.mark.parametrize("d,bmse", [(8, 2), (64, 3), (128, 2), (128, 3), (128, 4), (200, 1)])
def test_codebook_is_a_lloyd_fixed_point(d, bmse):
    c, t = O.lloyd_max_codebook(d, bmse)
    assert np.all(np.diff(c) > 0)
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), atol=1e-15)
    # centroid condition, checked with quadrature rather than the closed form
    edges = np.concatenate([[-1.0], t, [1.0]])
    for i in range(len(c)):
        num, _ = integrate.quad(lambda x: x * float(O.coord_density(x, d)), edges[i], edges[i + 1],
                                epsabs=1e-14, epsrel=1e-12, limit=200)
        den, _ = integrate.quad(lambda x: float(O.coord_density(x, d)), edges[i], edges[i + 1],
                                epsabs=1e-14, epsrel=1e-12, limit=200)
        assert abs(num / den - c[i]) < 1e-10
    np.testing.assert_allclose(c, -c[::-1], atol=0)


@pytest.mark.parametrize("d", [3, 5, 8])
@pytest.mark.parametrize("bmse", [1, 2])
def test_codebook_matches_exhaustive_boundary_search(d, bmse):
    # Minimise the MSE over all symmetric boundary sets on a grid (L <= 4).
    c, t = O.lloyd_max_codebook(d, bmse)

    def mse_for_bounds(tb):
        cc = O.lloyd_centroids(np.asarray(tb), d)
        return O.mse_distortion(cc, np.asarray(tb), d)

    if bmse == 1:
        grid = np.arange(-300, 301) * 1e-3
        best = min(grid, key=lambda a: mse_for_bounds([a]))
        fine = np.arange(-10, 11) * 1e-4 + best
        best = min(fine, key=lambda a: mse_for_bounds([a]))
        assert abs(best - t[0]) < 1.5e-4
        return
    grid = np.arange(1, 1000) * 1e-3
    best = min(grid, key=lambda a: mse_for_bounds([-a, 0.0, a]))
    fine = np.arange(-10, 11) * 1e-4 + best
    best = min(fine, key=lambda a: mse_for_bounds([-a, 0.0, a]))
    assert abs(best - t[2]) < 1.5e-4


def test_mse_decreases_and_sits_between_the_bounds():
    d = 128
    D = []
    for bmse in (1, 2, 3, 4):
        c, t = O.lloyd_max_codebook(d, bmse)
        D.append(O.mse_distortion(c, t, d))
    assert all(a > b for a, b in zip(D, D[1:]))
    for b, v in enumerate(D, start=1):
        # information-theoretic lower bound 4^-b; the pages quote a factor of about 2.7 above it
        assert 4.0 ** -b <= v <= 2.72 * 4.0 ** -b


@pytest.mark.parametrize("d", [8, 128])
def test_one_bit_distortion_closed_form(d):
    c, t = O.lloyd_max_codebook(d, 1)
    assert abs(O.mse_distortion(c, t, d) - (1 - d * c[1] ** 2)) < 1e-9


def test_quantize_mse_matches_the_distortion_integral():
    d, bits = 128, 3
    tb = O.make_tables(d, bits, seed=3)
    K = np.random.default_rng(1).standard_normal((20000, d))
    q = O.quantize(K, tb)
    err = np.sum((q.u - tb.c[q.codes]) ** 2, axis=1).mean()
    ref = O.mse_distortion(tb.c, tb.t, d)
    assert abs(err - ref) < 4 * 0.01 * ref


# --------------------------------------------------------------------------
# Quantize: brute force on tiny inputs, edge cases
# --------------------------------------------------------------------------


@pytest.mark.parametrize("d,bits", [(4, 3), (6, 2), (8, 2)])
def test_cell_search_equals_exhaustive_nearest_codeword(d, bits):
    import itertools

    tb = O.make_tables(d, bits, seed=11, m=4)
    K = np.random.default_rng(2).standard_normal((40, d))
    q = O.quantize(K, tb)
    L = len(tb.c)
    combos = np.array(list(itertools.product(range(L), repeat=d)))
    recon = tb.c[combos]                                      # (L^d, d)
    u = (K @ tb.R.T) / np.linalg.norm(K, axis=1, keepdims=True)
    best = combos[np.argmin(((u[:, None, :] - recon[None]) ** 2).sum(-1), axis=1)]
    np.testing.assert_array_equal(q.codes, best)


def test_quantize_residual_and_signs_by_definition():
    d, bits = 8, 3
    tb = O.make_tables(d, bits, seed=4, m=16)
    k = np.random.default_rng(3).standard_normal(d) * 3.0
    q = O.quantize(k[None], tb)
    n = np.linalg.norm(k)
    khat = n * sum(tb.c[q.codes[0, j]] * tb.R[j] for j in range(d))   # sum_j c_j R_j. (rows of R)
    r = k - khat
    np.testing.assert_allclose(q.rho[0], np.linalg.norm(r), rtol=1e-13)
    z = np.array([sum(tb.S[i, j] * r[j] for j in range(d)) for i in range(16)])
    np.testing.assert_array_equal(q.bits[0], z >= 0)
    # S = P R has the distribution of a Gaussian: its rows are P's rows rotated
    np.testing.assert_allclose(tb.S @ tb.R.T, tb.P, atol=1e-12)


def test_zero_key_and_boundary_ties():
    d = 64
    tb = O.make_tables(d, 3, seed=9)
    q = O.quantize(np.zeros((2, d)), tb)
    assert np.all(q.codes == 0) and np.all(q.bits) and np.all(q.n16 == 0) and np.all(q.rho16 == 0)
    # a coordinate exactly on a boundary takes the lower cell: move boundary t_i onto a computed u_j
    k = np.random.default_rng(5).standard_normal(d)
    u = O.quantize(k[None], tb).u[0]
    j = int(np.argmin(np.abs(u - tb.t[1])))
    t = tb.t.copy()
    t[1] = u[j]
    assert t[0] < t[1] < t[2]
    tb2 = O.Tables(d=d, bits=3, m=d, R=tb.R, P=tb.P, S=tb.S, c=tb.c, t=t)
    assert O.quantize(k[None], tb2).codes[0, j] == 1
    t[1] = np.nextafter(u[j], -1)
    assert O.quantize(k[None], tb2).codes[0, j] == 2


def test_fp16_norm_rounding_is_single_rounding_to_nearest_even():
    one = 1.0
    assert np.float64(one + 2.0 ** -11).astype(np.float16) == np.float16(1.0)            # tie -> even
    assert np.float64(one + 3 * 2.0 ** -11).astype(np.float16) == np.float16(1 + 2.0 ** -9)
    # just above a midpoint: a double rounding through fp32 would give 1.0
    v = np.float64(one + 2.0 ** -11 + 2.0 ** -40)
    assert v.astype(np.float16) == np.float16(1 + 2.0 ** -10)
    assert np.float64(70000.0).astype(np.float16) == np.float16(np.inf)


# --------------------------------------------------------------------------
# Estimator: unbiasedness (QJL), the 2/pi bias of the 1-bit MSE quantizer,
# and the exact dequantisation identity
# --------------------------------------------------------------------------


def test_qjl_two_dim_expectation_matches_quadrature():
    # d = 2, m = 1: E[sign(s.r) (s.q)] = sqrt(2/pi) <r, q> / ||r|| for s ~ N(0, I2).
    r = np.array([0.6, -0.2])
    q = np.array([0.3, 0.9])
    f = lambda b, a: np.sign(a * r[0] + b * r[1]) * (a * q[0] + b * q[1]) * math.exp(-(a * a + b * b) / 2) / (2 * math.pi)
    val, _ = integrate.dblquad(f, -9, 9, -9, 9, epsabs=1e-10)
    assert abs(val - math.sqrt(2 / math.pi) * r @ q / np.linalg.norm(r)) < 1e-6


def test_qjl_term_unbiased_over_1e5_seeds_d128():
    """Mean QJL estimate of <r, q> over 10^5 independent Gaussian S (R fixed).

    The 10^5 seeds of m = 128 rows are evaluated as batches of 1000 seeds,
    i.e. one oracle call with 128 000 rows per batch: the estimator's
    average over all rows equals the average of the per-seed estimates.
    Standard error from the closed-form variance
    rho^2 / m ((pi/2) ||q||^2 - <r/||r||, q>^2).
    """
    d, m, nseed, per = 128, 128, 100_000, 1000
    rng = np.random.default_rng(123)
    base = O.make_tables(d, 3, seed=1)
    k = rng.standard_normal(d) * (1 + 5 * (np.arange(d) < 4))
    qv = rng.standard_normal(d)
    total = 0.0
    for b in range(nseed // per):
        # the JL samples are stored as fp16 values (the method's matrix as stored)
        P = rng.standard_normal((m * per, d)).astype(np.float16).astype(np.float64)
        tb = O.Tables(d=d, bits=3, m=m * per, R=base.R, P=P, S=P @ base.R, c=base.c, t=base.t)
        qz = O.quantize(k[None], tb)
        # the QJL term of the estimator alone: feed codes whose levels are zero
        tb0 = O.Tables(d=d, bits=3, m=m * per, R=base.R, P=P, S=tb.S, c=np.zeros_like(base.c), t=base.t)
        s, _ = O.estimate(qv[None], qz.codes, qz.bits, qz.n, qz.rho, tb0)
        total += s[0, 0]
    mean = total / (nseed // per)
    r = k - qz.n[0] * (base.c[qz.codes[0]] @ base.R)
    rho = np.linalg.norm(r)
    var = rho ** 2 / m * ((math.pi / 2) * qv @ qv - (r @ qv / rho) ** 2)
    se = math.sqrt(var / nseed)
    assert abs(mean - r @ qv) < 3 * se


def test_jl_samples_are_stored_fp16_gaussians():
    tb = O.make_tables(128, 3, seed=12)
    raw = O.gaussian_stream(12, 1, 128 * 128).reshape(128, 128)
    np.testing.assert_array_equal(tb.P, raw.astype(np.float16).astype(np.float64))
    assert np.max(np.abs(tb.P - raw) / np.maximum(np.abs(raw), 1e-30)) <= 2.0 ** -11
    np.testing.assert_allclose(tb.S, tb.P @ tb.R, atol=1e-12)


def test_fp16_stored_jl_samples_keep_the_qjl_constant():
    """The JL samples are stored as their nearest fp16 values.  With R Haar and
    independent of P, a row s_i = R^T p_i points in a uniformly random
    direction, and the QJL term's expectation is E||p_i|| c_d <r/||r||, q> with
    c_d the mean |coordinate| of a random unit vector; for Gaussian rows
    E||p|| c_d = sqrt(2 / pi) exactly.  Rounding to fp16 changes E||p|| only
    through the moments of one rounded sample, computed here exactly from the
    normal law over every fp16 rounding cell (no sampling):
    E[fp16(g)^2] = 1 - 4.4e-8 and E[fp16(g)^4] = 3 (1 + O(1e-7)), so E||p||
    moves by well under 1e-7 relative at any d."""
    from scipy import special

    v = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)   # fp16 values >= 0
    cut = np.concatenate([(v[:-1] + v[1:]) / 2, [65520.0]])                         # upper edge of each cell
    lo = np.concatenate([[0.0], cut[:-1]])
    prob = 2.0 * (special.ndtr(cut) - special.ndtr(lo))
    prob[0] = special.ndtr(cut[0]) - special.ndtr(-cut[0])                          # the cell of 0 is two-sided
    assert abs(prob.sum() - 1.0) < 1e-15
    m2, m4 = np.sum(v ** 2 * prob), np.sum(v ** 4 * prob)
    assert abs(m2 - 1.0) < 1e-7 and abs(m4 / 3.0 - 1.0) < 1e-6
    # E||p|| = sqrt(d m2) (1 - (m4 - m2^2) / (8 d m2^2) + O(d^-2)) for d iid coordinates:
    # the leading factor moves by |sqrt(m2) - 1| and the correction by O(|m4 - 3| / d)
    for d in (64, 128, 200, 256):
        ratio = np.sqrt(m2) * (1 - (m4 - m2 ** 2) / (8 * d * m2 ** 2)) / (1 - 2.0 / (8 * d))
        assert abs(ratio - 1.0) < 1e-7, (d, ratio)


def test_full_estimator_unbiased_with_r_and_s_redrawn():
    d, bits, nseed = 32, 3, 4000
    rng = np.random.default_rng(5)
    k = rng.standard_normal(d) * 2
    qv = rng.standard_normal(d)
    est = []
    for s in range(nseed):
        tb = O.make_tables(d, bits, seed=1000 + s)
        qz = O.quantize(k[None], tb)
        v, _ = O.estimate(qv[None], qz.codes, qz.bits, qz.n, qz.rho, tb)
        est.append(v[0, 0])
    est = np.array(est)
    se = est.std(ddof=1) / math.sqrt(nseed)
    assert abs(est.mean() - k @ qv) < 3 * se


def test_one_bit_mse_estimator_bias_factor():
    """The MSE-only 1-bit estimator is biased: E = d c1(d)^2 <q, k>, -> 2/pi.

    Derivation: with u = R k/||k||, c[idx] = c1 sign(u); Rq = <q,k/||k||> u + w,
    E[w | u] = 0, so E[<c[idx], Rq>] = c1 E|u|_1 <q, k>/||k|| and E|u_j| = c1.
    """
    d, nseed = 16, 20000
    rng = np.random.default_rng(8)
    k = rng.standard_normal(d)
    qv = rng.standard_normal(d)
    c, _ = O.lloyd_max_codebook(d, 1)
    factor = d * c[1] ** 2
    est = []
    for s in range(nseed):
        G = rng.standard_normal((d, d))
        R = O.haar_rotation(G)
        tb = O.Tables(d=d, bits=2, m=d, R=R, P=np.zeros((d, d)), S=np.zeros((d, d)), c=c, t=np.array([0.0]))
        qz = O.quantize(k[None], tb)
        v, _ = O.estimate(qv[None], qz.codes, qz.bits, qz.n, qz.rho * 0, tb)
        est.append(v[0, 0])
    est = np.array(est)
    se = est.std(ddof=1) / math.sqrt(nseed)
    assert abs(est.mean() - factor * (k @ qv)) < 3.5 * se
    c128, _ = O.lloyd_max_codebook(128, 1)
    assert abs(128 * c128[1] ** 2 - 0.6391) < 1e-4
    cbig, _ = O.lloyd_max_codebook(10 ** 6, 1)
    assert abs(10 ** 6 * cbig[1] ** 2 - 2 / math.pi) < 1e-6


def test_dequantize_full_reproduces_the_estimator_exactly():
    d, bits = 64, 4
    tb = O.make_tables(d, bits, seed=21)
    rng = np.random.default_rng(6)
    K = rng.standard_normal((50, d))
    Q = rng.standard_normal((7, d))
    qz = O.quantize(K, tb)
    s, A = O.estimate(Q, qz.codes, qz.bits, qz.n16, qz.rho16, tb)
    xh = O.dequantize(qz.codes, qz.bits, qz.n16, qz.rho16, tb, full=True)
    np.testing.assert_allclose(Q @ xh.T, s, atol=1e-12 * A.max())
    # MSE-only reconstruction is the first term alone
    xm = O.dequantize(qz.codes, qz.bits, qz.n16, qz.rho16, tb, full=False)
    tb0 = O.Tables(d=d, bits=bits, m=d, R=tb.R, P=tb.P, S=tb.S * 0, c=tb.c, t=tb.t)
    s0, _ = O.estimate(Q, qz.codes, qz.bits, qz.n16, qz.rho16, tb0)
    np.testing.assert_allclose(Q @ xm.T, s0, atol=1e-12 * A.max())


def test_estimator_with_zero_residual_is_the_mse_term():
    d = 64
    tb = O.make_tables(d, 3, seed=2)
    codes = np.random.default_rng(0).integers(0, 4, (5, d))
    K = 2.5 * (tb.c[codes] @ tb.R)            # keys that sit exactly on reconstruction points
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    K *= 2.5
    qz = O.quantize(K * 1.0, tb)
    qv = np.random.default_rng(1).standard_normal((3, d))
    s, _ = O.estimate(qv, qz.codes, qz.bits, qz.n, qz.rho, tb)
    n = np.linalg.norm(K, axis=1)
    exact = qv @ (n[:, None] * (tb.c[qz.codes] @ tb.R)).T
    assert np.all(qz.rho < 1e-12 * n + 0.3 * n)   # residual small relative to the key
    np.testing.assert_allclose(s, exact + (O.QJL_CONST / d) * qz.rho * ((qv @ tb.S.T) @ (2.0 * qz.bits - 1).T),
                               rtol=1e-12, atol=1e-12)


def test_estimator_error_shrinks_with_bits():
    d = 128
    rng = np.random.default_rng(9)
    K = rng.standard_normal((400, d))
    Q = rng.standard_normal((8, d))
    exact = Q @ K.T
    errs = []
    for bits in (2, 3, 4, 5):
        tb = O.make_tables(d, bits, seed=31)
        qz = O.quantize(K, tb)
        s, _ = O.estimate(Q, qz.codes, qz.bits, qz.n16, qz.rho16, tb)
        errs.append(np.sqrt(np.mean((s - exact) ** 2)))
    assert all(a > b for a, b in zip(errs, errs[1:]))


def test_topk_order_and_tie_rule():
    d = 64
    tb = O.make_tables(d, 3, seed=2)
    rng = np.random.default_rng(4)
    K = rng.standard_normal((300, d))
    K[200] = K[17]                            # exact duplicate -> identical score, lower id first
    qz = O.quantize(K, tb)
    Q = K[17:18] + 0.01 * rng.standard_normal((1, d))
    ids, sc, s, _ = O.topk(Q, qz.codes, qz.bits, qz.n16, qz.rho16, tb, k=10)
    assert ids[0, 0] == 17 and list(ids[0]).index(200) == list(ids[0]).index(17) + 1
    assert np.all(np.diff(sc[0]) <= 0)
    np.testing.assert_array_equal(np.sort(s[0])[::-1][:10], sc[0])


def test_gqa_logits_head_mapping():
    d, B, Hkv, G, S = 64, 2, 2, 3, 20
    tb = O.make_tables(d, 3, seed=2)
    rng = np.random.default_rng(4)
    K = rng.standard_normal((B, Hkv, S, d))
    q = rng.standard_normal((B, Hkv * G, d))
    qz = O.quantize(K.reshape(-1, d), tb)
    sh = (B, Hkv, S)
    out, _ = O.gqa_logits(q, qz.codes.reshape(*sh, d), qz.bits.reshape(*sh, d),
                          qz.n16.reshape(sh), qz.rho16.reshape(sh), tb, scale=0.5)
    b, h, s = 1, 4, 7
    ref, _ = O.estimate(q[b, h][None], qz.codes.reshape(*sh, d)[b, h // G, s][None],
                        qz.bits.reshape(*sh, d)[b, h // G, s][None], qz.n16.reshape(sh)[b, h // G, s][None],
                        qz.rho16.reshape(sh)[b, h // G, s][None], tb)
    assert abs(out[b, h, s] - 0.5 * ref[0, 0]) < 1e-12


# --------------------------------------------------------------------------
# Packed layout
# --------------------------------------------------------------------------


@pytest.mark.parametrize("d,m,bmse", [(64, 64, 1), (64, 64, 2), (128, 128, 3), (128, 128, 2),
                                      (128, 64, 4), (256, 128, 3), (200, 200, 1), (200, 200, 3), (72, 136, 2)])
def test_pack_unpack_round_trip(d, m, bmse):
    rng = np.random.default_rng(d + m + bmse)
    codes = rng.integers(0, 1 << bmse, (33, d))
    bits = rng.integers(0, 2, (33, m)).astype(bool)
    p = O.pack_rows(codes, bits, bmse)
    assert p.shape == (33, O.row_bytes(d, m, bmse))
    c2, b2 = O.unpack_rows(p, d, m, bmse)
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(b2, bits)
    # slots past d and m (layout rounded up to multiples of 64) stay empty
    pc, pb = O.unpack_padding(p, d, m, bmse)
    assert pc.shape == (33, -(-d // 64) * 64 - d) and not pc.any()
    assert pb.shape == (33, -(-m // 64) * 64 - m) and not pb.any()


def test_padded_layout_is_the_next_multiple_of_64():
    # d = 200 codes occupy the first 200 of 256 slots: a row packed at d = 200
    # equals the d = 256 row of the same codes followed by zero codes.
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 8, (7, 200))
    bits = rng.integers(0, 2, (7, 200)).astype(bool)
    p200 = O.pack_rows(codes, bits, 3)
    codes256 = np.concatenate([codes, np.zeros((7, 56), dtype=codes.dtype)], axis=1)
    bits256 = np.concatenate([bits, np.zeros((7, 56), dtype=bool)], axis=1)
    np.testing.assert_array_equal(p200, O.pack_rows(codes256, bits256, 3))
    assert O.row_bytes(200, 200, 3) == 256 * 3 // 8 + 256 // 8 == 128
    assert O.row_bytes(200, 200, 1) == 64


def test_pack_layout_hand_example():
    # d = m = 64, b' = 3: chunk q has 3 code halfwords and 1 sign halfword (8 bytes).
    d = m = 64
    codes = np.zeros((1, d), dtype=np.int64)
    bits = np.zeros((1, m), dtype=bool)
    codes[0, 16 + 4 * 1 + 2] = 5        # quarter 1, register 1, nibble 2 -> H1 of chunk 1, bits 8..10 = 101
    codes[0, 4 * 3 + 1] = 6             # quarter 0, register 3, nibble 1: bit i of 6 -> H_i bit 7
    bits[0, 48 + 4 * 2 + 3] = True      # quarter 3, sign register 2, nibble 3 -> bit 14 of chunk 3's sign halfword
    p = O.pack_rows(codes, bits, 3)[0].view("<u2")
    want = np.zeros(16, dtype=np.uint16)
    want[4 + 1] = 0b101 << 8
    want[0 + 1] |= 1 << 7
    want[0 + 2] |= 1 << 7
    want[12 + 3] = 1 << 14
    np.testing.assert_array_equal(p, want)


def test_pack_layout_hand_example_one_bit_codes_more_sign_rows():
    # d = 64, m = 128, b' = 1: chunk q = 1 code halfword (unit 0) + 2 sign
    # halfwords (units 0, 1) = 3 halfwords; the row is 12 halfwords.
    d, m = 64, 128
    codes = np.zeros((1, d), dtype=np.int64)
    bits = np.zeros((1, m), dtype=bool)
    codes[0, 16 * 2 + 4 * 3 + 1] = 1   # quarter 2, register 3, nibble 1 -> chunk 2's H0, bit 4*1+3 = 7
    codes[0, 0] = 1                    # quarter 0, register 0, nibble 0 -> bit 0 of halfword 0
    bits[0, 32 * 1 + 4 * 6 + 0] = True  # quarter 1, sign register 6 = unit 1, i = 2, nibble 0 -> bit 2
    bits[0, 127] = True                # quarter 3, register 7 = unit 1, i = 3, nibble 3 -> bit 15
    p = O.pack_rows(codes, bits, 1)[0].view("<u2")
    assert p.shape == (12,) and O.row_bytes(d, m, 1) == 24
    want = np.zeros(12, dtype=np.uint16)
    want[0] = 0x0001
    want[2 * 3 + 0] = 0x0080
    want[1 * 3 + 1 + 1] = 0x0004
    want[3 * 3 + 1 + 1] = 0x8000
    np.testing.assert_array_equal(p, want)
    c2, b2 = O.unpack_rows(O.pack_rows(codes, bits, 1), d, m, 1)
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(b2, bits)


def test_pack_layout_hand_example_two_bit_codes_fewer_sign_rows():
    # d = 128, m = 64, b' = 2: chunk q = 2 units x 2 code halfwords + 1 sign
    # halfword = 5 halfwords; the row is 20 halfwords.
    d, m = 128, 64
    codes = np.zeros((1, d), dtype=np.int64)
    bits = np.zeros((1, m), dtype=bool)
    codes[0, 32 * 1 + 4 * 5 + 2] = 3   # quarter 1, register 5 = unit 1, pair i = 0, second code,
    #                                    nibble 2 -> bits 10-11 of chunk 1's halfword 2 * 1 + 0
    codes[0, 4 * 2 + 3] = 2            # quarter 0, register 2 = unit 0, pair 1, first code, nibble 3
    #                                    -> bits 12-13 of halfword 1
    codes[0, 127] = 1                  # quarter 3, register 7 = unit 1, pair 1, second code, nibble 3
    #                                    -> bits 14-15 of chunk 3's halfword 2 + 1
    bits[0, 16 * 2 + 4 * 1 + 3] = True  # quarter 2, sign register 1, nibble 3 -> bit 13 of chunk 2's sign halfword
    p = O.pack_rows(codes, bits, 2)[0].view("<u2")
    assert p.shape == (20,) and O.row_bytes(d, m, 2) == 40
    want = np.zeros(20, dtype=np.uint16)
    want[5 * 1 + 2] = 3 << 10
    want[0 + 1] = 2 << 12
    want[5 * 3 + 2 + 1] = 1 << 14
    want[5 * 2 + 4] = 1 << 13
    np.testing.assert_array_equal(p, want)
    c2, b2 = O.unpack_rows(O.pack_rows(codes, bits, 2), d, m, 2)
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(b2, bits)


def test_sign_boundary_distance_is_the_cosine():
    # rows s_0 = (3, 4) (norm 5) and s_1 = (0, 2); r = (1, 0): z = (3, 0)
    S = np.array([[3.0, 4.0], [0.0, 2.0]])
    r = np.array([[1.0, 0.0], [0.0, -0.5], [0.0, 0.0]])
    z = r @ S.T
    rho = np.linalg.norm(r, axis=1)
    dist = O.sign_boundary_distance(z, rho, S)
    np.testing.assert_allclose(dist[0], [3 / 5, 0.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(dist[1], [4 / 5, 1.0], rtol=0, atol=1e-15)
    assert np.all(np.isinf(dist[2]))   # zero residual: never excused


def test_norm_band_is_one_unit_sphere_band():
    # ||k|| = 10, ||r|| = 2: ||r|| / ||k|| = 0.2 on the unit sphere; a 1e-5 band
    # there is 1e-5 * 10 / 2 = 5e-5 relative to ||r||; a zero residual has none
    bn, br = O.norm_band(np.array([10.0, 3.0]), np.array([2.0, 0.0]))
    np.testing.assert_allclose(bn, [1e-5, 1e-5], rtol=0, atol=0)
    np.testing.assert_allclose(br, [5e-5, 0.0], rtol=1e-15, atol=0)


def test_fp16_midpoint_distance_hand_values():
    f = O.fp16_midpoint_distance
    # exact midpoints: 1 + 2^-11 (between 1 and 1 + 2^-10), 2049 (between 2048
    # and 2050), 2^-25 (between 0 and the smallest subnormal 2^-24), 1.5 2^-24
    # (between the first two subnormals), 65520 (the overflow threshold)
    for v in [1 + 2.0**-11, 2049.0, 2.0**-25, 1.5 * 2.0**-24, 65520.0, -(1 + 2.0**-11)]:
        assert f(np.array([v]))[0] == 0.0, v
    # 1.0: spacing 2^-11 below 1, so the nearest midpoint is 1 - 2^-12
    assert f(np.array([1.0]))[0] == 2.0**-12
    # 65504 (largest finite): midpoints 65488 below and 65520 above, both 16 away
    assert f(np.array([65504.0]))[0] == 16.0 / 65504.0
    # 1e5 rounds to inf: the nearest midpoint is the overflow threshold
    assert f(np.array([1e5]))[0] == (1e5 - 65520.0) / 1e5
    # 3.0 is representable with spacing 2^-9 on both sides
    assert f(np.array([3.0]))[0] == 2.0**-10 / 3.0
    assert np.isinf(f(np.array([0.0]))[0])


def test_fp16_midpoint_distance_against_all_midpoints():
    # every rounding midpoint of fp16, from the list of all finite non-negative
    # fp16 values; the helper's distance equals the brute-force nearest one
    allh = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = np.concatenate([(allh[:-1] + allh[1:]) / 2, [65520.0]])
    rng = np.random.default_rng(3)
    v = np.concatenate([np.exp(rng.uniform(np.log(1e-8), np.log(2e5), 20000)),
                        mids[rng.integers(0, len(mids), 200)],
                        allh[rng.integers(1, len(allh), 200)]])
    pos = np.searchsorted(mids, v)
    lo = mids[np.clip(pos - 1, 0, len(mids) - 1)]
    hi = mids[np.clip(pos, 0, len(mids) - 1)]
    want = np.minimum(np.abs(v - lo), np.abs(v - hi)) / v
    np.testing.assert_array_equal(O.fp16_midpoint_distance(v), want)


# --------------------------------------------------------------------------
# MSE-only variant (m = 0: stage 1 alone)
# --------------------------------------------------------------------------


@pytest.mark.parametrize("d,bits", [(64, 2), (128, 4), (200, 3)])
def test_mse_only_estimator_is_the_first_term(d, bits):
    """m = 0 uses the same rotation and codebook (stream 0) as m = d, stores no
    sign bits, and estimates <q, k> by n16 sum_j c[idx_j] (Rq)_j, which is also
    <q, x_hat> of the stage-1 reconstruction."""
    rng = np.random.default_rng(d + bits)
    K = rng.standard_normal((40, d))
    Q = rng.standard_normal((3, d))
    t0, t1 = O.make_tables(d, bits, 11, m=0), O.make_tables(d, bits, 11, m=d)
    np.testing.assert_array_equal(t0.R, t1.R)
    np.testing.assert_array_equal(t0.c, t1.c)
    q0, q1 = O.quantize(K, t0), O.quantize(K, t1)
    np.testing.assert_array_equal(q0.codes, q1.codes)
    assert q0.bits.shape == (40, 0)
    s0, A0 = O.estimate(Q, q0.codes, q0.bits, q0.n16, q0.rho16, t0)
    first = q1.n16.astype(np.float64)[None, :] * ((Q @ t1.R.T) @ t1.c[q1.codes].T)
    np.testing.assert_allclose(s0, first, rtol=1e-12, atol=1e-12)
    xh = O.dequantize(q0.codes, q0.bits, q0.n16, q0.rho16, t0, full=True)
    np.testing.assert_allclose(s0, Q @ xh.T, rtol=1e-10, atol=1e-10)
    p = O.pack_rows(q0.codes, q0.bits, t0.bmse)
    assert p.shape == (40, O.row_bytes(d, 0, t0.bmse)) and O.row_bytes(d, 0, t0.bmse) == -(-d // 64) * 64 * t0.bmse // 8
    c2, b2 = O.unpack_rows(p, d, 0, t0.bmse)
    np.testing.assert_array_equal(c2, q0.codes)
    assert b2.shape == (40, 0)


# --------------------------------------------------------------------------
# Channel split (fractional bit rates)
# --------------------------------------------------------------------------


def test_split_plan_orders_by_variance_with_ties_to_lower_channel():
    # channel c of head h alternates +a, -a around an offset mu over the B*S
    # rows, so its variance is exactly a^2 whatever mu is; the expected order
    # is written out by hand from the amplitudes
    B, S, d = 2, 3, 8
    amp = np.array([[1, 5, 2, 5, 0.5, 3, 4, 0.25],      # head 0: 1 and 3 tie at 5
                    [7, 1, 1, 1, 6, 2, 9, 8]], float)   # head 1: 1, 2, 3 tie at 1
    mu = np.array([100.0, -3.0, 0.0, 7.0, -50.0, 2.0, 1.0, 9.0])
    signs = np.array([1, -1, 1, -1, 1, -1], float).reshape(B, S)
    K = np.empty((B, 2, S, d))
    for h in range(2):
        K[:, h] = mu + signs[:, :, None] * amp[h]
    perm = O.split_plan(K, 4)
    # head 0 by amplitude: 5 (ch 1), 5 (ch 3), 4 (ch 6), 3 (ch 5) | the rest
    assert perm[0].tolist() == [1, 3, 5, 6, 0, 2, 4, 7]
    # head 1: 9 (ch 6), 8 (ch 7), 7 (ch 0), 6 (ch 4) | 2 (ch 5) and the three 1s
    assert perm[1].tolist() == [0, 4, 6, 7, 1, 2, 3, 5]
    # three-way tie at the cut: head 1 with 6 high channels takes the lowest tied one
    perm6 = O.split_plan(K, 6)
    assert perm6[1].tolist() == [0, 1, 4, 5, 6, 7, 2, 3]


def test_split_plan_of_no_keys_keeps_channel_order():
    perm = O.split_plan(np.zeros((1, 2, 0, 8)), 3)
    assert perm.tolist() == [[0, 1, 2, 3, 4, 5, 6, 7]] * 2


def test_split_estimator_unbiased_with_both_groups_redrawn():
    # each group's estimate is unbiased for its part of <q, k>, and the parts
    # add up to <q, k> under any split of the channels
    d, nseed = 16, 2000
    rng = np.random.default_rng(11)
    k = rng.standard_normal((1, 1, 1, d)) * np.linspace(0.5, 4.0, d)
    qv = rng.standard_normal((1, 1, d))
    perm = O.split_plan(np.concatenate([k, -k], axis=2), 8)
    est = []
    for s in range(nseed):
        thi = O.make_tables(8, 3, seed=5000 + 2 * s)
        tlo = O.make_tables(8, 2, seed=5001 + 2 * s)
        a, b = O.split_quantize(k, perm, thi, tlo)
        v, _ = O.split_gqa_logits(qv, perm, a, b, thi, tlo, 1, 1, 1)
        est.append(v[0, 0, 0])
    est = np.array(est)
    se = est.std(ddof=1) / math.sqrt(nseed)
    assert abs(est.mean() - float(k[0, 0, 0] @ qv[0, 0])) < 3 * se


def test_split_dequantize_reproduces_the_split_estimator():
    rng = np.random.default_rng(12)
    B, Hkv, S, d, G = 2, 3, 5, 16, 2
    K = rng.standard_normal((B, Hkv, S, d)) * rng.uniform(0.2, 5.0, (1, Hkv, 1, d))
    q = rng.standard_normal((B, Hkv * G, d))
    perm = O.split_plan(K, 8)
    thi, tlo = O.make_tables(8, 3, 42), O.make_tables(8, 2, 43)
    a, b = O.split_quantize(K, perm, thi, tlo)
    s, _ = O.split_gqa_logits(q, perm, a, b, thi, tlo, B, Hkv, S)
    xh = O.split_dequantize(perm, a, b, thi, tlo, B, Hkv, S, full=True)
    for h in range(Hkv * G):
        np.testing.assert_allclose(s[:, h], np.einsum("bd,bsd->bs", q[:, h], xh[:, h // G]), atol=1e-11)


def test_split_gives_the_high_variance_channels_the_finer_code():
    # with strongly unequal channel scales (different per head), the planned
    # split reconstructs the keys better than the same split with the two
    # groups' bit widths exchanged
    rng = np.random.default_rng(13)
    B, Hkv, S, d = 1, 3, 400, 16
    scales = np.exp(2.0 * rng.standard_normal((Hkv, d)))
    K = rng.standard_normal((B, Hkv, S, d)) * scales[None, :, None, :]
    perm = O.split_plan(K, 8)
    swapped = np.concatenate([perm[:, 8:], perm[:, :8]], axis=1)
    thi, tlo = O.make_tables(8, 4, 42), O.make_tables(8, 2, 43)
    for p, worse in ((perm, False), (swapped, True)):
        a, b = O.split_quantize(K, p, thi, tlo)
        x = O.split_dequantize(p, a, b, thi, tlo, B, Hkv, S, full=False)
        err = np.sum((x - K) ** 2, axis=(0, 2, 3))
        if not worse:
            planned = err
        else:
            assert np.all(planned < err)


# --------------------------------------------------------------------------
# Value path: attention output over a quantised value cache
# --------------------------------------------------------------------------


def _value_cache(B, Hkv, S, d, bits, seed, m=None):
    rng = np.random.default_rng(seed)
    V = rng.standard_normal((B * Hkv * S, d)) * rng.uniform(0.5, 3.0, d)
    tb = O.make_tables(d, bits, 40 + seed, m=m)
    return V, tb, O.quantize(V, tb)


def test_softmax_closed_form():
    p = O.softmax(np.array([[0.0, math.log(3.0)], [5.0, 5.0]]))
    np.testing.assert_allclose(p, [[0.25, 0.75], [0.5, 0.5]], rtol=0, atol=1e-15)
    # large logits do not overflow
    np.testing.assert_allclose(O.softmax(np.array([1000.0, 1000.0 + math.log(3.0)])), [0.25, 0.75], atol=1e-15)


def test_attention_of_two_keys_is_the_weighted_reconstruction():
    V, tb, qz = _value_cache(1, 1, 2, 16, 3, 1)
    o, _ = O.attention_output(np.array([[[0.0, math.log(3.0)]]]), qz.codes, qz.bits, qz.n16, qz.rho16, tb, 1)
    xh = O.dequantize(qz.codes, qz.bits, qz.n16, qz.rho16, tb, full=True)
    np.testing.assert_allclose(o[0, 0], 0.25 * xh[0] + 0.75 * xh[1], atol=1e-12)


def test_attention_with_equal_logits_is_the_mean_and_shift_invariant():
    B, Hkv, S, d = 1, 1, 7, 16
    V, tb, qz = _value_cache(B, Hkv, S, d, 4, 2)
    xh = O.dequantize(qz.codes, qz.bits, qz.n16, qz.rho16, tb, full=True)
    o, _ = O.attention_output(np.full((1, 1, S), 2.5), qz.codes, qz.bits, qz.n16, qz.rho16, tb, Hkv)
    np.testing.assert_allclose(o[0, 0], xh.mean(axis=0), atol=1e-12)
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((1, 1, S)) * 3
    o1, _ = O.attention_output(lg, qz.codes, qz.bits, qz.n16, qz.rho16, tb, Hkv)
    o2, _ = O.attention_output(lg + 40.0, qz.codes, qz.bits, qz.n16, qz.rho16, tb, Hkv)
    np.testing.assert_allclose(o1, o2, atol=1e-12)


def test_attention_head_mapping_and_single_key():
    # S = 1: every head of KV head k returns that key's reconstruction
    B, Hkv, G, d = 2, 3, 2, 16
    V, tb, qz = _value_cache(B, Hkv, 1, d, 3, 4)
    xh = O.dequantize(qz.codes, qz.bits, qz.n16, qz.rho16, tb, full=True).reshape(B, Hkv, d)
    lg = np.random.default_rng(5).standard_normal((B, Hkv * G, 1))
    o, A = O.attention_output(lg, qz.codes, qz.bits, qz.n16, qz.rho16, tb, Hkv)
    for b in range(B):
        for h in range(Hkv * G):
            np.testing.assert_allclose(o[b, h], xh[b, h // G], atol=1e-12)
            assert np.all(A[b, h] >= np.abs(o[b, h]) - 1e-12)


def test_attention_output_unbiased_over_value_tables():
    # given the weights, E over the value quantizer's R and S of the output is
    # the exact weighted sum of the values (each reconstruction is unbiased)
    d, S, nseed = 16, 3, 3000
    rng = np.random.default_rng(6)
    V = rng.standard_normal((S, d)) * 2
    lg = np.array([[[0.3, -1.0, 1.2]]])
    u = rng.standard_normal(d)
    want = float(O.softmax(lg)[0, 0] @ V @ u)
    got = []
    for s in range(nseed):
        tb = O.make_tables(d, 3, seed=9000 + s)
        qz = O.quantize(V, tb)
        o, _ = O.attention_output(lg, qz.codes, qz.bits, qz.n, qz.rho, tb, 1)
        got.append(o[0, 0] @ u)
    got = np.array(got)
    se = got.std(ddof=1) / math.sqrt(nseed)
    assert abs(got.mean() - want) < 3 * se


def test_attention_mse_only_uses_stage_one():
    V, tb, qz = _value_cache(1, 1, 4, 16, 3, 7, m=0)
    lg = np.array([[[0.1, 0.2, -0.3, 0.0]]])
    o, _ = O.attention_output(lg, qz.codes, qz.bits, qz.n16, qz.rho16, tb, 1)
    xh = qz.n16.astype(np.float64)[:, None] * (tb.c[qz.codes] @ tb.R)
    np.testing.assert_allclose(o[0, 0], O.softmax(lg)[0, 0] @ xh, atol=1e-12)
