"""Properties of the oracle that hold at every supported shape, checked on
randomly drawn (d, m, bits, seed) with hypothesis: d and m multiples of 8
from 64 to 256 (m = 0: the MSE-only variant), bits 2..4.

- the cell index is the nearest codeword (Lloyd-Max boundaries are the
  midpoints of neighbouring levels, so the cell search is a nearest-neighbour
  search, airosetta.com stage 1);
- the sign bits are [S r >= 0] of the residual r = k - n R^T c[idx];
- the full reconstruction reproduces the estimator (<q, x_hat> = s_hat);
- packing the quantised rows and unpacking them gives the codes and bits back."""

import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import tq_oracle as O

dims = st.integers(8, 32).map(lambda v: 8 * v)
shapes = st.tuples(dims, st.one_of(st.just(0), dims), st.integers(2, 4), st.integers(0, 2**32 - 1))


@settings(max_examples=25, deadline=None)
@given(shapes)
def test_quantize_estimate_pack_properties(shape):
    d, m, bits, seed = shape
    tb = O.make_tables(d, bits, seed, m=m)
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((40, d)) * np.exp(rng.standard_normal(d))
    K[3] = 0.0
    qz = O.quantize(K, tb)
    n = np.linalg.norm(K, axis=1)
    live = n > 0
    # nearest codeword (ties, which have probability zero here, aside)
    u = (K[live] @ tb.R.T) / n[live, None]
    nearest = np.argmin(np.abs(u[:, :, None] - tb.c[None, None, :]), axis=2)
    np.testing.assert_array_equal(qz.codes[live], nearest)
    # zero key: codes 0, all sign bits 1, zero norms
    assert not qz.codes[3].any() and qz.bits[3].all() and qz.n16[3] == 0 and qz.rho16[3] == 0
    if m:
        r = K - n[:, None] * (tb.c[qz.codes] @ tb.R)
        np.testing.assert_array_equal(qz.bits[live], (r[live] @ tb.S.T) >= 0)
    # the full reconstruction reproduces the estimator
    Q = rng.standard_normal((5, d))
    s, A = O.estimate(Q, qz.codes, qz.bits, qz.n16, qz.rho16, tb)
    xh = O.dequantize(qz.codes, qz.bits, qz.n16, qz.rho16, tb, full=True)
    np.testing.assert_allclose(Q @ xh.T, s, rtol=0, atol=1e-11 * A.max())
    # pack / unpack round trip
    p = O.pack_rows(qz.codes, qz.bits, bits - 1)
    assert p.shape == (40, O.row_bytes(d, m, bits - 1))
    c2, b2 = O.unpack_rows(p, d, m, bits - 1)
    np.testing.assert_array_equal(c2, qz.codes)
    np.testing.assert_array_equal(b2, qz.bits)
