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


split_shapes = st.tuples(dims, dims, st.integers(2, 4), st.integers(2, 4), st.integers(1, 3), st.integers(1, 3),
                         st.integers(1, 20), st.integers(0, 2**32 - 1))


@settings(max_examples=15, deadline=None)
@given(split_shapes)
def test_split_properties(shape):
    """Channel split: the plan is a permutation per KV head whose high group
    holds channels of variance at least that of every low-group channel; the
    split reconstruction reproduces the split logits; the high group's
    quantisation is that of the gathered channels."""
    d_hi, d_lo, b_hi, b_lo, B, Hkv, S, seed = shape
    d = d_hi + d_lo
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((B, Hkv, S, d)) * np.exp(rng.standard_normal((1, Hkv, 1, d)))
    perm = O.split_plan(K, d_hi)
    for h in range(Hkv):
        assert sorted(perm[h]) == list(range(d))
        X = K[:, h].reshape(-1, d)
        var = X.var(axis=0)
        assert var[perm[h, :d_hi]].min() >= var[perm[h, d_hi:]].max() - 1e-12 * var.max()
    tb_hi = O.make_tables(d_hi, b_hi, seed, m=d_hi)
    tb_lo = O.make_tables(d_lo, b_lo, seed + 1, m=d_lo)
    a, c = O.split_quantize(K, perm, tb_hi, tb_lo)
    G = 2
    q = rng.standard_normal((B, Hkv * G, d))
    s, A = O.split_gqa_logits(q, perm, a, c, tb_hi, tb_lo, B, Hkv, S)
    xh = O.split_dequantize(perm, a, c, tb_hi, tb_lo, B, Hkv, S, full=True)
    for h in range(Hkv * G):
        ref = np.einsum("bd,bsd->bs", q[:, h], xh[:, h // G])
        np.testing.assert_allclose(s[:, h], ref, rtol=0, atol=1e-11 * A.max())
    hi_keys = np.stack([K[:, h][..., perm[h, :d_hi]] for h in range(Hkv)], axis=1).reshape(-1, d_hi)
    np.testing.assert_array_equal(a.codes, O.quantize(hi_keys, tb_hi).codes)
