"""Plain fp64 CPU oracle for the TurboQuant hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import this module.  It
shares no code, tables or constants with the CUDA library in
``compressed_kv_cache_tq_b200/``; neither side imports the other.  Inputs
are passed in as arrays; nothing here comes from the GPU path.

What it computes, step by step, and where the pages say so:

* Random rotation R: QR factorisation of a seeded Gaussian matrix
  (airosetta.com "Google TurboQuant", section "第一階段：PolarQuant").
  The pages give no generator, no sign rule and no Q-vs-Q^T choice; the
  readings used here are listed on each function.
* Coordinate law of a rotated unit vector: a Beta-type law on [-1, 1]
  with density proportional to (1 - x^2)^((d-3)/2) (same section: the
  coordinates "follow a known, concentrated Beta distribution").
* Per-coordinate Lloyd-Max scalar quantizer with a precomputed codebook
  (same section: "Lloyd-Max ... precomputed codebook").
* 1-bit QJL sketch of the residual, sign(S r), S a seeded Gaussian
  (section "第二階段：QJL——1比特殘差校正").
* Unbiased inner-product estimator
  <q,k> ~ ||k|| sum_j c[idx_j] (Rq)_j + sqrt(pi/2)/m ||r|| <Sq, sigma>.
  The pages' formula was lost in extraction (the sentence ending in
  "保證 / 。"); the estimator used is the standard QJL one the surrounding
  text describes (unbiased, one sign bit per projected residual row).
* m = 0 selects stage 1 alone (the MSE variant, TurboQuant_mse): no sign
  sketch, and the estimator is its first term, which the same page notes is
  biased for inner products (factor 2/pi at one bit).
* Dequantisation "look up the table and rotate back" (same page, stage 1).
* Value path: the decode attention output, softmax of the logits times the
  values' unbiased reconstructions (reading in the section "Value path").
* Fractional rates (2.5 bits per channel): a per-KV-head channel split
  into a high-variance group and a low-variance group, each quantised on
  its own (readings in the section "Channel split" below).

Every function below is fp64 and follows the definitions literally: no
blocking, fusion or reordering beyond vectorising over keys.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
from scipy import special

# ---------------------------------------------------------------------------
# Counter-based generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
# "Parallel random numbers: as easy as 1, 2, 3", SC'11).  The pages name no
# generator; a published counter-based one lets the oracle and the library
# draw the same R and S independently from the seed.
# ---------------------------------------------------------------------------

_MASK32 = np.uint64(0xFFFFFFFF)
_PHILOX_M0 = np.uint64(0xD2511F53)
_PHILOX_M1 = np.uint64(0xCD9E8D57)
_PHILOX_W0 = np.uint64(0x9E3779B9)
_PHILOX_W1 = np.uint64(0xBB67AE85)


def philox4x32_10(counter: np.ndarray, key) -> np.ndarray:
    """Philox4x32 with 10 rounds.

    counter: (N, 4) array of 32-bit words; key: two 32-bit words.
    Returns (N, 4) uint32.  Each round multiplies words 0 and 2 by the two
    Philox constants, mixes the high halves with words 1, 3 and the key, and
    the key is bumped by the Weyl constants between rounds.
    """
    ctr = np.asarray(counter, dtype=np.uint64).reshape(-1, 4)
    c0, c1, c2, c3 = (ctr[:, i].copy() for i in range(4))
    k0 = np.uint64(int(key[0]) & 0xFFFFFFFF)
    k1 = np.uint64(int(key[1]) & 0xFFFFFFFF)
    for _ in range(10):
        p0 = _PHILOX_M0 * c0
        p1 = _PHILOX_M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0) & _MASK32, lo1, (hi0 ^ c3 ^ k1) & _MASK32, lo0
        k0 = (k0 + _PHILOX_W0) & _MASK32
        k1 = (k1 + _PHILOX_W1) & _MASK32
    return np.stack([c0, c1, c2, c3], axis=1).astype(np.uint32)


def gaussian_stream(seed: int, stream: int, count: int) -> np.ndarray:
    """``count`` standard normals from stream ``stream`` of generator ``seed``.

    Reading (pages silent): block i of the stream is Philox4x32-10 with
    counter (i mod 2^32, i div 2^32, stream, 0) and key (seed mod 2^32,
    seed div 2^32).  Its four words give two 53-bit uniforms
    u1 = (a + 1) 2^-53 in (0, 1] and u2 = b 2^-53 in [0, 1), where a is built
    from words 0, 1 and b from words 2, 3 as (hi >> 5) 2^26 + (lo >> 6).
    Box-Muller then yields normals 2i (cosine) and 2i+1 (sine).
    """
    nblk = (count + 1) // 2
    i = np.arange(nblk, dtype=np.uint64)
    ctr = np.zeros((nblk, 4), dtype=np.uint64)
    ctr[:, 0] = i & _MASK32
    ctr[:, 1] = i >> np.uint64(32)
    ctr[:, 2] = np.uint64(stream)
    seed = int(seed)
    w = philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)).astype(np.uint64)
    a = (w[:, 0] >> np.uint64(5)) * np.uint64(1 << 26) + (w[:, 1] >> np.uint64(6))
    b = (w[:, 2] >> np.uint64(5)) * np.uint64(1 << 26) + (w[:, 3] >> np.uint64(6))
    u1 = (a.astype(np.float64) + 1.0) * 2.0**-53
    u2 = b.astype(np.float64) * 2.0**-53
    rad = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * nblk, dtype=np.float64)
    out[0::2] = rad * np.cos(2.0 * math.pi * u2)
    out[1::2] = rad * np.sin(2.0 * math.pi * u2)
    return out[:count]


# ---------------------------------------------------------------------------
# Rotation R and JL matrix S
# ---------------------------------------------------------------------------


def haar_rotation(G: np.ndarray) -> np.ndarray:
    """Orthogonal factor of G = Q T with diag(T) > 0 (Haar distributed).

    The pages say only "QR decomposition of a Gaussian matrix".  Reading:
    R := Q with the columns of Q flipped so that diag(T) is positive, which
    makes the factorisation unique and Q Haar-distributed; the rotation is
    applied as u = R k / ||k||.
    """
    Q, T = np.linalg.qr(np.asarray(G, dtype=np.float64))
    s = np.sign(np.diag(T))
    s[s == 0] = 1.0
    return Q * s[None, :]


@dataclass
class Tables:
    """Data-oblivious parameters of one quantizer (d, b' = bits - 1, m)."""

    d: int
    bits: int          # total bits per coordinate, b
    m: int             # QJL rows
    R: np.ndarray      # (d, d) rotation
    P: np.ndarray      # (m, d) Gaussian drawn from the seed
    S: np.ndarray      # (m, d) JL matrix applied to the residual, S = P R
    c: np.ndarray      # (L,) Lloyd-Max levels on the unit-sphere scale
    t: np.ndarray      # (L-1,) decision boundaries

    @property
    def bmse(self) -> int:
        return self.bits - 1


def make_tables(d: int, bits: int, seed: int, m: int | None = None, stream_base: int = 0) -> Tables:
    """R, S and the codebook from (d, bits, seed), as tq_init builds them.

    Reading (pages silent on layout and precision): G is d x d, row-major,
    from stream ``stream_base``; P is m x d, row-major, from stream
    ``stream_base + 1``, each Gaussian sample stored as the nearest fp16
    value (the JL matrix as stored).  The JL matrix applied to the residual is
    S = P R.  Because R is Haar and independent of P, each row of S points in
    a uniformly random direction; the estimator's constant sqrt(pi/2) is then
    exact up to E||p_i|| of the stored rows, which differs from the Gaussian
    value by less than 1e-7 relative (pinned by the exact moments of an
    fp16-rounded normal sample, computed over every rounding cell).
    """
    m = d if m is None else m
    if bits < 2:
        raise ValueError("bits >= 2 (one Lloyd-Max bit plus the QJL bit)")
    G = gaussian_stream(seed, stream_base, d * d).reshape(d, d)
    P = gaussian_stream(seed, stream_base + 1, m * d).reshape(m, d).astype(np.float16).astype(np.float64)
    R = haar_rotation(G)
    S = P @ R
    c, t = lloyd_max_codebook(d, bits - 1)
    return Tables(d=d, bits=bits, m=m, R=R, P=P, S=S, c=c, t=t)


# ---------------------------------------------------------------------------
# Coordinate law and Lloyd-Max codebook
# ---------------------------------------------------------------------------


def coord_density_const(d: int) -> float:
    """C_d with f_d(x) = C_d (1 - x^2)^((d-3)/2) on [-1, 1] (d >= 2)."""
    return math.exp(special.gammaln(d / 2) - special.gammaln((d - 1) / 2) - 0.5 * math.log(math.pi))


def coord_density(x, d: int):
    """Density of one coordinate of a uniformly random unit vector in R^d."""
    x = np.asarray(x, dtype=np.float64)
    return coord_density_const(d) * (1.0 - x * x) ** ((d - 3) / 2)


def coord_cdf(x, d: int):
    """CDF of f_d: (1 + x) / 2 is Beta((d-1)/2, (d-1)/2) distributed."""
    a = (d - 1) / 2
    return special.betainc(a, a, (1.0 + np.asarray(x, dtype=np.float64)) / 2.0)


def coord_first_moment(lo, hi, d: int):
    """Integral of x f_d(x) over [lo, hi], in closed form.

    The antiderivative of x (1 - x^2)^alpha is -(1 - x^2)^(alpha+1) / (2 (alpha+1));
    with alpha = (d-3)/2, 2 (alpha + 1) = d - 1.
    """
    e = (d - 1) / 2
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    return coord_density_const(d) / (d - 1) * ((1.0 - lo * lo) ** e - (1.0 - hi * hi) ** e)


def lloyd_centroids(t: np.ndarray, d: int) -> np.ndarray:
    """Conditional means of f_d over the cells cut by boundaries t."""
    edges = np.concatenate([[-1.0], np.asarray(t, dtype=np.float64), [1.0]])
    mass = np.diff(coord_cdf(edges, d))
    return coord_first_moment(edges[:-1], edges[1:], d) / mass


def lloyd_max_codebook(d: int, bmse: int, tol: float = 1e-15, max_iter: int = 200000):
    """Lloyd-Max quantizer with L = 2^bmse levels for the law f_d.

    Alternates the two optimality conditions (boundaries at midpoints,
    levels at cell centroids) from the quantile start until the levels stop
    moving, then symmetrises (f_d is even).  For d >= 3 f_d is log-concave,
    so the fixed point is unique.
    Returns (c, t): L levels and L-1 boundaries, ascending.
    """
    L = 1 << bmse
    a = (d - 1) / 2
    c = 2.0 * special.betaincinv(a, a, (np.arange(L) + 0.5) / L) - 1.0
    best = np.inf
    stall = 0
    for _ in range(max_iter):
        t = 0.5 * (c[:-1] + c[1:])
        c_new = lloyd_centroids(t, d)
        delta = float(np.max(np.abs(c_new - c)))
        c = c_new
        if delta < tol:
            break
        if delta < best:
            best, stall = delta, 0
        else:
            stall += 1
            if stall > 50 and delta < 1e-13:
                break  # rounding noise floor
    c = 0.5 * (c - c[::-1])
    t = 0.5 * (c[:-1] + c[1:])
    return c, t


def mse_distortion(c: np.ndarray, t: np.ndarray, d: int) -> float:
    """E over one coordinate of (u_j - c[idx_j])^2, times d: E||u - c[idx]||^2.

    Computed from the cell masses and the first two moments; the second
    moment of f_d over a cell is integrated with adaptive quadrature.
    """
    from scipy import integrate

    edges = np.concatenate([[-1.0], t, [1.0]])
    total = 0.0
    for i in range(len(c)):
        lo, hi = edges[i], edges[i + 1]
        val, _ = integrate.quad(lambda x: (x - c[i]) ** 2 * float(coord_density(x, d)), lo, hi,
                                epsabs=1e-15, epsrel=1e-12, limit=200)
        total += val
    return d * total


# ---------------------------------------------------------------------------
# Quantisation (stage 1 + stage 2) and the estimator
# ---------------------------------------------------------------------------


@dataclass
class Quantized:
    codes: np.ndarray        # (N, d) int, Lloyd-Max cell index per rotated coordinate
    bits: np.ndarray         # (N, m) bool, QJL sign bit (True = +1)
    n: np.ndarray            # (N,) ||k||, fp64
    rho: np.ndarray          # (N,) ||r||, fp64
    n16: np.ndarray          # (N,) fp16 of n (round to nearest even)
    rho16: np.ndarray        # (N,) fp16 of rho
    u: np.ndarray            # (N, d) R k / ||k|| (diagnostic: distance to boundaries)
    z: np.ndarray            # (N, m) S r (diagnostic: distance to the sign boundary)


def quantize(K: np.ndarray, tb: Tables) -> Quantized:
    """Quantise rows k of K.

    1. n = ||k||; u = R k / n (rotation onto the unit sphere).
    2. idx_j = #{i : t_i < u_j}; a value exactly on a boundary takes the
       lower cell (reading).
    3. k_hat = n R^T c[idx] (look up and rotate back); r = k - k_hat.
    4. z = S r; sign bit = [z_i >= 0], so sign(0) = +1 (reading: a 1-bit
       code cannot store torch.sign's 0).
    5. Store fp16(n) and fp16(||r||).
    A zero key (n = 0) gets codes 0, all sign bits 1 and zero norms
    (reading: its direction is undefined).
    """
    K = np.asarray(K, dtype=np.float64)
    n = np.sqrt(np.sum(K * K, axis=1))
    zero = n == 0
    y = K @ tb.R.T
    u = y / np.where(zero, 1.0, n)[:, None]
    u[zero] = 0.0
    codes = np.sum(u[:, :, None] > tb.t[None, None, :], axis=2)
    codes[zero] = 0
    khat = n[:, None] * (tb.c[codes] @ tb.R)
    r = K - khat
    rho = np.sqrt(np.sum(r * r, axis=1))
    z = r @ tb.S.T
    bits = z >= 0
    return Quantized(codes=codes, bits=bits, n=n, rho=rho, n16=n.astype(np.float16),
                     rho16=rho.astype(np.float16), u=u, z=z)


QJL_CONST = math.sqrt(math.pi / 2.0)


def estimate(Q: np.ndarray, codes, bits, n16, rho16, tb: Tables):
    """Estimated inner products between queries Q (nq, d) and packed keys.

    s = n16 sum_j c[idx_j] (Rq)_j + sqrt(pi/2)/m rho16 sum_i sigma_i (Sq)_i
    with sigma_i = 2 bit_i - 1.  Also returns A, the sum of the absolute
    values of all terms (the scale the tolerance is measured against).
    Returns (s, A), each (nq, N).
    """
    Q = np.atleast_2d(np.asarray(Q, dtype=np.float64))
    x = Q @ tb.R.T                       # rows: R q
    cv = tb.c[np.asarray(codes)]         # (N, d)
    n16 = np.asarray(n16, dtype=np.float64)
    k1 = n16[None, :] * (x @ cv.T)
    a1 = n16[None, :] * (np.abs(x) @ np.abs(cv).T)
    if tb.m == 0:
        # m = 0: stage 1 alone (TurboQuant_mse), the first term
        return k1, a1
    y = Q @ tb.S.T                       # rows: S q
    sig = 2.0 * np.asarray(bits, dtype=np.float64) - 1.0
    rho16 = np.asarray(rho16, dtype=np.float64)
    k2 = (QJL_CONST / tb.m) * rho16[None, :] * (y @ sig.T)
    a2 = (QJL_CONST / tb.m) * rho16[None, :] * np.sum(np.abs(y), axis=1)[:, None]
    return k1 + k2, a1 + a2


def dequantize(codes, bits, n16, rho16, tb: Tables, full: bool = True):
    """Reconstruct x_hat = n16 R^T c[idx] (+ sqrt(pi/2)/m rho16 S^T sigma).

    Stage 1 alone ("full=False") is the MSE reconstruction ("look up the
    codebook and rotate back").  With the QJL term, <q, x_hat> equals the
    estimator exactly, so this is the vector the estimator implicitly uses.
    """
    n16 = np.asarray(n16, dtype=np.float64)
    rho16 = np.asarray(rho16, dtype=np.float64)
    xh = n16[:, None] * (tb.c[np.asarray(codes)] @ tb.R)
    if full and tb.m > 0:
        sig = 2.0 * np.asarray(bits, dtype=np.float64) - 1.0
        xh = xh + (QJL_CONST / tb.m) * rho16[:, None] * (sig @ tb.S)
    return xh


def gqa_logits(q: np.ndarray, codes, bits, n16, rho16, tb: Tables, scale: float = 1.0):
    """Attention logits for GQA decode.

    q: (B, Hq, d); codes (B, Hkv, S, d), bits (B, Hkv, S, m), norms (B, Hkv, S).
    Query head h reads KV head h // (Hq / Hkv).  Returns (logits, A),
    each (B, Hq, S).
    """
    B, Hq, _ = q.shape
    Hkv = codes.shape[1]
    G = Hq // Hkv
    S = codes.shape[2]
    out = np.empty((B, Hq, S))
    absum = np.empty((B, Hq, S))
    for b in range(B):
        for hk in range(Hkv):
            s, a = estimate(q[b, hk * G:(hk + 1) * G], codes[b, hk], bits[b, hk],
                            n16[b, hk], rho16[b, hk], tb)
            out[b, hk * G:(hk + 1) * G] = scale * s
            absum[b, hk * G:(hk + 1) * G] = abs(scale) * a
    return out, absum


def topk(Q: np.ndarray, codes, bits, n16, rho16, tb: Tables, k: int):
    """Inner-product top-k over a quantised database.

    Order: estimated score descending, ties to the lower id (reading).
    Returns (ids (nq, k) int64, scores (nq, k), A (nq, N)).
    """
    s, A = estimate(Q, codes, bits, n16, rho16, tb)
    N = s.shape[1]
    ids = np.empty((s.shape[0], k), dtype=np.int64)
    sc = np.empty((s.shape[0], k))
    idx = np.arange(N)
    for i in range(s.shape[0]):
        order = np.lexsort((idx, -s[i]))[:k]
        ids[i] = order
        sc[i] = s[i, order]
    return ids, sc, s, A


# ---------------------------------------------------------------------------
# Value path: decode attention output over a quantised value cache
#
# mooersco.com sections 1.2 and 1.3: the keys set the attention weights
# (softmax of the logits), the values are summed with those weights, and the
# values are compressed with a JL projection kept as sign bits, the output
# being recovered by an estimator.  The other pages describe one two-stage
# quantizer for the whole KV cache.  Reading: values are quantised with the
# same quantizer as keys (tables of their own), and each value enters the
# output through its unbiased reconstruction
#   v_hat = n16 R^T c[idx] + sqrt(pi/2)/m rho16 S^T sigma
# (stage 1 alone when m = 0), so that
#   o = sum_s softmax(l)_s v_hat_s,
# with l the (already scaled) logits of the query head against the keys.
# ---------------------------------------------------------------------------


def softmax(logits: np.ndarray) -> np.ndarray:
    """Softmax over the last axis in fp64 (shifted by the maximum)."""
    x = np.asarray(logits, dtype=np.float64)
    e = np.exp(x - np.max(x, axis=-1, keepdims=True))
    return e / np.sum(e, axis=-1, keepdims=True)


def attention_output(logits: np.ndarray, codes, bits, n16, rho16, tb: Tables, Hkv: int):
    """Attention output of every query head over a quantised value cache.

    logits: (B, Hq, S), already scaled; value rows ordered (B, Hkv, S), query
    head h reads KV head h // (Hq / Hkv).  Returns (o, A), each (B, Hq, d):
    o[b, h] = sum_s softmax(logits[b, h])_s v_hat[b, h // G, s], and A the
    same weighted sum of the absolute values of every term of v_hat (the
    scale the tolerance is measured against).
    """
    B, Hq, S = logits.shape
    G = Hq // Hkv
    p = softmax(logits) if S > 0 else np.zeros((B, Hq, 0))
    vh = dequantize(codes, bits, n16, rho16, tb, full=True).reshape(B, Hkv, S, tb.d)
    n16 = np.asarray(n16, dtype=np.float64).reshape(B, Hkv, S)
    cv = np.abs(tb.c[np.asarray(codes)]).reshape(B, Hkv, S, tb.d)
    # |terms| of coordinate i: n16 sum_j |R_ji| |c_j| (+ the QJL term's)
    absv = n16[..., None] * (cv @ np.abs(tb.R))
    if tb.m > 0:
        rho16 = np.asarray(rho16, dtype=np.float64).reshape(B, Hkv, S)
        absv = absv + (QJL_CONST / tb.m) * rho16[..., None] * np.sum(np.abs(tb.S), axis=0)[None, None, None, :]
    o = np.zeros((B, Hq, tb.d))
    A = np.zeros((B, Hq, tb.d))
    for b in range(B):
        for h in range(Hq):
            o[b, h] = p[b, h] @ vh[b, h // G]
            A[b, h] = p[b, h] @ absv[b, h // G]
    return o, A


# ---------------------------------------------------------------------------
# Channel split: fractional bit rates such as 2.5 bits per channel
#
# The pages give 3.5- and 2.5-bit settings (the rom4ai.github.io note
# "TurboQuant: Online Vector Quantization with Near-Optimal Distortion Rate"
# sizes the cache at 3.5 bits per channel; mooersco.com section 2.1 lists a
# 2.5-bit setting with at least 7x less memory; zhengruan.com reports a small
# quality loss at 2.5 bits) without saying how a fractional rate is reached,
# and mooersco.com's FAQ notes that the unrotated channels' variances differ
# by two orders of magnitude.  Reading:
# per KV head, the d_hi channels of largest variance form a high group and
# the rest a low group; each group is quantised as its own vector with its
# own tables (rotation, JL matrix, codebook) and bit width, and the inner
# product estimate is the sum of the two groups' estimates, since
# <q, k> = <q_hi, k_hi> + <q_lo, k_lo> for the same channel split of q and k.
# ---------------------------------------------------------------------------


def split_plan(K: np.ndarray, d_hi: int) -> np.ndarray:
    """Channel order per KV head for keys K (B, Hkv, S, d).

    For head h, the variance of channel c over all B x S keys of that head
    is sum_rows (x - mean)^2 / (B S) (the 1 / (B S - 1) of the sample
    variance would not change the order).  The d_hi channels of largest
    variance, ties to the lower channel index, come first in ascending
    channel order, then the other channels in ascending order (reading).
    Returns perm (Hkv, d) int64: group coordinate p of head h is channel
    perm[h, p]; coordinates p < d_hi form the high group.
    """
    K = np.asarray(K, dtype=np.float64)
    B, Hkv, S, d = K.shape
    perm = np.empty((Hkv, d), dtype=np.int64)
    for h in range(Hkv):
        X = K[:, h].reshape(B * S, d)
        if X.shape[0] > 0:
            mean = X.mean(axis=0)
            var = np.sum((X - mean) ** 2, axis=0) / X.shape[0]
        else:
            var = np.zeros(d)
        order = sorted(range(d), key=lambda c: (-var[c], c))
        hi = sorted(order[:d_hi])
        lo = sorted(order[d_hi:])
        perm[h] = hi + lo
    return perm


def split_groups(X: np.ndarray, perm: np.ndarray, d_hi: int):
    """Gather the two channel groups of X (B, H, S, d) or (B, H, d) by perm (H, d):
    returns (X_hi, X_lo) with the channel axis last."""
    X = np.asarray(X, dtype=np.float64)
    H = perm.shape[0]
    hi = np.stack([X[:, h][..., perm[h, :d_hi]] for h in range(H)], axis=1)
    lo = np.stack([X[:, h][..., perm[h, d_hi:]] for h in range(H)], axis=1)
    return hi, lo


def split_quantize(K: np.ndarray, perm: np.ndarray, tb_hi: Tables, tb_lo: Tables):
    """Quantise keys K (B, Hkv, S, d) group by group: the high group (the
    first tb_hi.d coordinates of perm) with tb_hi, the rest with tb_lo.
    Returns (Quantized hi, Quantized lo), rows in [B][Hkv][S] order."""
    B, Hkv, S, d = K.shape
    assert tb_hi.d + tb_lo.d == d
    Khi, Klo = split_groups(K, perm, tb_hi.d)
    return quantize(Khi.reshape(-1, tb_hi.d), tb_hi), quantize(Klo.reshape(-1, tb_lo.d), tb_lo)


def split_gqa_logits(q: np.ndarray, perm: np.ndarray, qz_hi: Quantized, qz_lo: Quantized, tb_hi: Tables,
                     tb_lo: Tables, B: int, Hkv: int, S: int, scale: float = 1.0):
    """Split-cache attention logits: for query head h (KV head hk = h // G)
    the estimate of <q_hi, k_hi> with tb_hi plus that of <q_lo, k_lo> with
    tb_lo, both groups gathered by perm[hk].  Returns (logits, A), each
    (B, Hq, S), A the sum of both groups' absolute-term sums."""
    Bq, Hq, d = q.shape
    G = Hq // Hkv
    # each query head takes the channel split of the KV head it reads
    qperm = np.repeat(perm, G, axis=0)
    q_hi, q_lo = split_groups(q[:, :, None, :], qperm, tb_hi.d)
    q_hi, q_lo = q_hi[:, :, 0], q_lo[:, :, 0]

    def view(qz, tb):
        return (qz.codes.reshape(B, Hkv, S, tb.d), qz.bits.reshape(B, Hkv, S, tb.m),
                qz.n16.reshape(B, Hkv, S), qz.rho16.reshape(B, Hkv, S))

    s_hi, a_hi = gqa_logits(q_hi, *view(qz_hi, tb_hi), tb_hi, scale)
    s_lo, a_lo = gqa_logits(q_lo, *view(qz_lo, tb_lo), tb_lo, scale)
    return s_hi + s_lo, a_hi + a_lo


def split_dequantize(perm: np.ndarray, qz_hi: Quantized, qz_lo: Quantized, tb_hi: Tables, tb_lo: Tables,
                     B: int, Hkv: int, S: int, full: bool = True) -> np.ndarray:
    """Reconstruct keys (B, Hkv, S, d) in the original channel order: each
    group's reconstruction scattered back to the channels perm names."""
    xh = dequantize(qz_hi.codes, qz_hi.bits, qz_hi.n16, qz_hi.rho16, tb_hi, full).reshape(B, Hkv, S, tb_hi.d)
    xl = dequantize(qz_lo.codes, qz_lo.bits, qz_lo.n16, qz_lo.rho16, tb_lo, full).reshape(B, Hkv, S, tb_lo.d)
    out = np.empty((B, Hkv, S, tb_hi.d + tb_lo.d))
    for h in range(Hkv):
        out[:, h][..., perm[h, :tb_hi.d]] = xh[:, h]
        out[:, h][..., perm[h, tb_hi.d:]] = xl[:, h]
    return out


# ---------------------------------------------------------------------------
# Packed row layout (the library's documented storage format)
#
# The pages fix no storage layout (they only say that no constants are stored
# per block, i.e. the codebook is global).  This is the format the C ABI documents, restated
# here from its definition so that packed bytes can be compared exactly.
#
# d and m are multiples of 64.  A row holds one key: four "quarter" chunks
# q = 0..3, each 2 (b' d/64 + m/64) bytes, chunk q holding coordinates
# j = q d/4 + 4 r + e (r = 0 .. d/16 - 1, e = 0..3) as little-endian 16-bit
# halfwords: first the code halfwords of units u = 0 .. d/64 - 1 (b' each),
# then the sign halfwords (one per 16 sign coordinates).  Unit u covers
# r = 4u .. 4u+3; "nibble e" of a halfword is bits 4e .. 4e+3.
#   b' = 1: H0 nibble e bit i       = code(r = 4u+i, e)
#   b' = 2: Hi nibble e bits 0-1    = code(4u+2i, e), bits 2-3 = code(4u+2i+1, e)
#   b' = 3: Hi nibble e bits 0-2    = code(4u+i, e) (i < 3); bit 3 = bit i of code(4u+3, e)
#   b' = 4: Hi nibble e             = code(4u+i, e)
#   signs: H nibble e bit i         = sign bit of coordinate q m/4 + 4(4u+i) + e
# Norms are stored apart: per key two fp16 values (||k||, ||r||).
# ---------------------------------------------------------------------------


def layout_dims(d: int, m: int) -> tuple:
    """Slots of the packed layout: d and m rounded up to multiples of 64.

    Reading (the pages fix no storage format): a dimension that is not a
    multiple of 64 (d = 200 for the vector-search workload) is stored in the
    quarter-chunk layout of the next multiple of 64; the slots past d (codes)
    and past m (sign bits) hold zeros and carry no information.
    """
    return -(-d // 64) * 64, -(-m // 64) * 64


def row_bytes(d: int, m: int, bmse: int) -> int:
    dp, mp = layout_dims(d, m)
    return dp * bmse // 8 + mp // 8


def _check_layout_dims(d: int, m: int, bmse: int):
    if d % 8 or m % 8 or d < 8 or m < 0:
        raise ValueError("packed layout needs d and m multiples of 8 (m = 0: no sign bits)")
    if not 1 <= bmse <= 4:
        raise ValueError("1 <= b' <= 4")


def _code_halfwords(cq: np.ndarray, bmse: int) -> list:
    """cq: (N, d/4) codes of one quarter -> list of (N,) uint16 halfwords."""
    N, qd = cq.shape
    out = []
    for u in range(qd // 16):
        def code(r, e):
            return cq[:, 4 * r + e].astype(np.uint32)
        if bmse == 1:
            h = np.zeros(N, dtype=np.uint32)
            for e in range(4):
                for i in range(4):
                    h |= (code(4 * u + i, e) & 1) << (4 * e + i)
            out.append(h)
        elif bmse == 2:
            for i in range(2):
                h = np.zeros(N, dtype=np.uint32)
                for e in range(4):
                    h |= (code(4 * u + 2 * i, e) & 3) << (4 * e)
                    h |= (code(4 * u + 2 * i + 1, e) & 3) << (4 * e + 2)
                out.append(h)
        elif bmse == 3:
            for i in range(3):
                h = np.zeros(N, dtype=np.uint32)
                for e in range(4):
                    h |= (code(4 * u + i, e) & 7) << (4 * e)
                    h |= ((code(4 * u + 3, e) >> i) & 1) << (4 * e + 3)
                out.append(h)
        else:
            for i in range(4):
                h = np.zeros(N, dtype=np.uint32)
                for e in range(4):
                    h |= (code(4 * u + i, e) & 15) << (4 * e)
                out.append(h)
    return out


def _sign_halfwords(bq: np.ndarray) -> list:
    N, qm = bq.shape
    out = []
    for u in range(qm // 16):
        h = np.zeros(N, dtype=np.uint32)
        for e in range(4):
            for i in range(4):
                h |= bq[:, 4 * (4 * u + i) + e].astype(np.uint32) << (4 * e + i)
        out.append(h)
    return out


def pack_rows(codes: np.ndarray, bits: np.ndarray, bmse: int) -> np.ndarray:
    """(N, d) codes and (N, m) sign bits -> (N, row_bytes) uint8."""
    codes = np.asarray(codes)
    bits = np.asarray(bits)
    N, d = codes.shape
    m = bits.shape[1]
    _check_layout_dims(d, m, bmse)
    dp, mp = layout_dims(d, m)
    codes = np.concatenate([codes, np.zeros((N, dp - d), dtype=codes.dtype)], axis=1)
    bits = np.concatenate([bits, np.zeros((N, mp - m), dtype=bits.dtype)], axis=1)
    halves = []
    for q in range(4):
        halves += _code_halfwords(codes[:, q * dp // 4:(q + 1) * dp // 4], bmse)
        halves += _sign_halfwords(bits[:, q * mp // 4:(q + 1) * mp // 4])
    hw = np.stack(halves, axis=1).astype(np.uint16)
    out = hw.astype("<u2").view(np.uint8).reshape(N, -1)
    assert out.shape[1] == row_bytes(d, m, bmse)
    return out


def unpack_rows(payload: np.ndarray, d: int, m: int, bmse: int):
    """Inverse of pack_rows: (N, row_bytes) uint8 -> (codes (N, d), bits (N, m)).

    The padding slots (past d and m) are read too and returned separately by
    ``unpack_padding`` so that tests can check they are zero."""
    codes, bits = _unpack_slots(payload, d, m, bmse)
    return codes[:, :d], bits[:, :m]


def unpack_padding(payload: np.ndarray, d: int, m: int, bmse: int):
    """The code and sign slots past d and m (all zero in a valid row)."""
    codes, bits = _unpack_slots(payload, d, m, bmse)
    return codes[:, d:], bits[:, m:]


def _unpack_slots(payload: np.ndarray, d: int, m: int, bmse: int):
    _check_layout_dims(d, m, bmse)
    d, m = layout_dims(d, m)
    payload = np.ascontiguousarray(payload, dtype=np.uint8)
    N = payload.shape[0]
    hw = payload.reshape(N, -1).view("<u2").astype(np.uint32)
    ud, um = d // 64, m // 64
    per_q = bmse * ud + um
    codes = np.zeros((N, d), dtype=np.int64)
    bits = np.zeros((N, m), dtype=bool)
    for q in range(4):
        base = q * per_q
        for u in range(ud):
            H = [hw[:, base + u * bmse + i] for i in range(bmse)]
            for e in range(4):
                def put(r, val):
                    codes[:, q * d // 4 + 4 * r + e] = val
                if bmse == 1:
                    for i in range(4):
                        put(4 * u + i, (H[0] >> (4 * e + i)) & 1)
                elif bmse == 2:
                    for i in range(2):
                        put(4 * u + 2 * i, (H[i] >> (4 * e)) & 3)
                        put(4 * u + 2 * i + 1, (H[i] >> (4 * e + 2)) & 3)
                elif bmse == 3:
                    hi = np.zeros(N, dtype=np.uint32)
                    for i in range(3):
                        put(4 * u + i, (H[i] >> (4 * e)) & 7)
                        hi |= ((H[i] >> (4 * e + 3)) & 1) << i
                    put(4 * u + 3, hi)
                else:
                    for i in range(4):
                        put(4 * u + i, (H[i] >> (4 * e)) & 15)
        for u in range(um):
            h = hw[:, base + ud * bmse + u]
            for e in range(4):
                for i in range(4):
                    bits[:, q * m // 4 + 4 * (4 * u + i) + e] = ((h >> (4 * e + i)) & 1).astype(bool)
    return codes, bits


def pack_norms(n16: np.ndarray, rho16: np.ndarray) -> np.ndarray:
    """(N,) fp16 pairs -> (N, 2) fp16: [||k||, ||r||] per key."""
    return np.stack([np.asarray(n16, np.float16), np.asarray(rho16, np.float16)], axis=1)


# ---------------------------------------------------------------------------
# Parity bands (the readings of the stated tolerances that the parity tests apply)
#
# The stated tolerance: codes and sign bits bit-exact except where the rotated
# value lies within 1e-5 of a decision boundary.  The code decision variable
# u_j = (R k)_j / ||k|| is one coordinate of the unit vector k / ||k|| in an
# orthonormal basis, so its band is |u_j - t_i| <= 1e-5 as it stands.  The
# sign decision variable is (S r)_i = <s_i, r>; read on the same unit-sphere
# scale it is the coordinate of the unit residual r / ||r|| along the unit JL
# direction s_i / ||s_i||, i.e. the cosine of the angle between them, and the
# band is |(S r)_i| <= 1e-5 ||s_i|| ||r||.
# ---------------------------------------------------------------------------

CODE_BAND = 1e-5     # |u_j - t_i| on the unit-sphere scale
SIGN_BAND = 1e-5     # |(S r)_i| / (||s_i|| ||r||): cosine between the JL row and the residual
NORM_BAND = 1e-5     # distance of the exact norm to an fp16 rounding midpoint, on the unit-sphere scale


def norm_band(n: np.ndarray, rho: np.ndarray):
    """Relative bands of the two stored norms (reading of the same 1e-5 on
    the unit-sphere scale as the code band): ||k|| / ||k|| = 1 is the scale of
    ||k||, so its band is 1e-5 relative; ||r|| / ||k|| is the length of the
    residual on the unit sphere, so a band of 1e-5 there is 1e-5 ||k|| / ||r||
    relative to ||r||.  Returns (band_n, band_rho) per key."""
    n = np.asarray(n, dtype=np.float64)
    rho = np.asarray(rho, dtype=np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        band_rho = np.where(rho > 0, NORM_BAND * n / np.where(rho > 0, rho, 1.0), 0.0)
    return np.full(n.shape, NORM_BAND), band_rho


def code_boundary_distance(u: np.ndarray, t: np.ndarray) -> np.ndarray:
    """min_i |u_j - t_i| for every coordinate."""
    return np.min(np.abs(u[..., None] - t), axis=-1)


def sign_boundary_distance(z: np.ndarray, rho: np.ndarray, S: np.ndarray) -> np.ndarray:
    """|z_i| / (||s_i|| ||r||) for z = S r (rows of z: keys, columns: JL rows).

    A key with a zero residual (rho = 0, e.g. the zero key) has z = 0 and sign
    bits fixed by the reading [0 >= 0]; it gets distance inf (never excused)."""
    rho = np.asarray(rho, dtype=np.float64)
    rn = np.sqrt(np.sum(np.asarray(S, dtype=np.float64) ** 2, axis=1))
    den = rho[:, None] * rn[None, :]
    with np.errstate(divide="ignore", invalid="ignore"):
        out = np.abs(z) / np.where(den > 0, den, 1.0)
    out[np.broadcast_to(den <= 0, out.shape)] = np.inf
    return out


FP16_MAX = 65504.0
FP16_OVERFLOW = 65520.0   # the rounding midpoint above the largest fp16: values >= it round to inf


def fp16_midpoint_distance(v: np.ndarray) -> np.ndarray:
    """Relative distance of |v| to the nearest fp16 rounding midpoint.

    The rounding midpoints of round-to-nearest fp16 are the means of two
    adjacent representable values: (h + next_up(h)) / 2 and
    (h + next_down(h)) / 2 around h = fp16(|v|); h = 0 has only the one
    above it (0 is a value, not a midpoint).  Above the largest finite value
    65504 the midpoint is the overflow threshold 65520 (values from there on
    round to inf).  v = 0 gets inf."""
    v = np.abs(np.asarray(v, dtype=np.float64))
    with np.errstate(over="ignore"):
        h16 = v.astype(np.float16)
        h = h16.astype(np.float64)
        up = np.nextafter(h16, np.float16(np.inf)).astype(np.float64)
        dn = np.nextafter(h16, np.float16(0)).astype(np.float64)
    with np.errstate(invalid="ignore"):
        mid_up = np.where(h >= FP16_MAX, FP16_OVERFLOW, (h + up) / 2)
        mid_dn = np.where(np.isinf(h), FP16_OVERFLOW, np.where(h == 0, np.inf, (h + dn) / 2))
        dist = np.minimum(np.abs(mid_up - v), np.abs(mid_dn - v))
    with np.errstate(divide="ignore", invalid="ignore"):
        rel = dist / np.where(v == 0, 1.0, v)
    rel = np.where(v == 0, np.inf, rel)
    return rel
