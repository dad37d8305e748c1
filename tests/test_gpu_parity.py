"""GPU parity: libtq's kernels (through the C ABI) against the CPU oracle.

Small cases span several 128-key tiles with ragged tails; the full-size
decode and long-context workloads are checked on sampled rows in the launch
configuration bench.py times.  Bands and tolerances: tests/parity.py."""

import math

import numpy as np
import pytest
import torch

from compressed_kv_cache_tq_b200 import workloads as W
from oracle import tq_oracle as O

from tests.parity import REL_FLOOR, check_close, check_quantize, format_stats, oracle_estimates, tables_of

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _ctx(lib, d=128, bits=3, seed=42, m=None):
    return lib.tq_init(d, bits, seed, m=m)


def _status_clean(lib, ctx):
    torch.cuda.synchronize()
    assert lib.tq_check_device_status(ctx) == 0


def test_device_tables_match_oracle(lib):
    ctx = _ctx(lib, bits=4, seed=11)
    R, P, c, t = ctx.export_tables()
    tb = tables_of(ctx)
    assert np.max(np.abs(R - tb.R)) < 1e-12 and np.max(np.abs(P - tb.P)) < 1e-13
    assert np.max(np.abs(c - tb.c)) < 1e-12 and np.max(np.abs(t - tb.t)) < 1e-12


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("m", [128, 0])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("n", [1, 127, 441, 4133])
def test_quantize_tensor_core_path(lib, bits, n, m, dtype):
    """d = 128 keys on the tensor-core quantizer, bf16 keys and fp32 keys (split
    into bf16 hi + lo on the way in), with the sign sketch (m = 128) and
    without it (m = 0, the MSE-only variant)."""
    ctx = _ctx(lib, bits=bits, seed=7 + bits, m=m)
    scales = W.head_channel_scales(1, 128, seed=3)
    k32 = W.decode_keys_pair(0, 0, n, 128, scales, seed=3 + n)
    kb = torch.from_numpy(k32).to(dtype)
    payload, norms = lib.tq_quantize(ctx, kb.to(DEV))
    _status_clean(lib, ctx)
    rep = {}
    check_quantize(payload.cpu().numpy(), norms.cpu().numpy(), kb.to(torch.float64).numpy(), tables_of(ctx), rep)


@pytest.mark.parametrize("bits", [3, 4])
def test_quantize_fp32_strided_and_ragged(lib, bits):
    """fp32 keys with a leading dimension above d (TMA rows 544 bytes apart)
    and a ragged last tile, against the oracle; equal to the rows quantised
    from a contiguous copy."""
    ctx = _ctx(lib, bits=bits, seed=9)
    n, ld = 3 * 128 + 77, 136
    k = W.toy_keys(n, 128, seed=21)
    wide = torch.zeros((n, ld), dtype=torch.float32)
    wide[:, :128] = torch.from_numpy(k)
    dev = wide.to(DEV)
    payload = torch.empty((n, ctx.row_bytes), dtype=torch.uint8, device=DEV)
    norms = torch.empty((n, 2), dtype=torch.float16, device=DEV)
    import ctypes

    st = lib.lib().tq_quantize(ctx.handle, ctypes.c_void_p(dev.data_ptr()), 0, n, ld,
                               ctypes.c_void_p(payload.data_ptr()), ctypes.c_void_p(norms.data_ptr()),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    _status_clean(lib, ctx)
    check_quantize(payload.cpu().numpy(), norms.cpu().numpy(), k.astype(np.float64), tables_of(ctx))
    p2, n2 = lib.tq_quantize(ctx, torch.from_numpy(k).to(DEV))
    assert torch.equal(p2, payload) and torch.equal(n2.view(torch.int16), norms.view(torch.int16))


def test_quantize_toy_fp32(lib):
    """toy workload: 4096 fp32 keys (+ a ragged tail), b = 3."""
    ctx = _ctx(lib, bits=3, seed=42)
    k = W.toy_keys(4096 + 37, 128, seed=1000)
    payload, norms = lib.tq_quantize(ctx, torch.from_numpy(k).to(DEV))
    _status_clean(lib, ctx)
    check_quantize(payload.cpu().numpy(), norms.cpu().numpy(), k.astype(np.float64), tables_of(ctx))


@pytest.mark.parametrize("d,m,bits,dtype", [(64, 64, 3, torch.bfloat16), (64, 64, 2, torch.float32),
                                            (256, 256, 3, torch.bfloat16), (128, 64, 4, torch.float32),
                                            (192, 128, 2, torch.bfloat16), (200, 200, 2, torch.float32),
                                            (200, 200, 4, torch.float32), (72, 136, 3, torch.bfloat16)])
def test_quantize_other_shapes(lib, d, m, bits, dtype):
    ctx = _ctx(lib, d=d, bits=bits, seed=5, m=m)
    k = W.toy_keys(777, d, seed=d + m)
    kt = torch.from_numpy(k).to(dtype)
    payload, norms = lib.tq_quantize(ctx, kt.to(DEV))
    _status_clean(lib, ctx)
    check_quantize(payload.cpu().numpy(), norms.cpu().numpy(), kt.to(torch.float64).numpy(), tables_of(ctx))


@pytest.mark.parametrize("d,bits", [(200, 2), (200, 3), (200, 4), (208, 3), (256, 2), (232, 4)])
def test_quantize_wide_tensor_core_path(lib, d, bits):
    """fp32 keys with 192 < d <= 256 (a layout of 256 slots) and m = d on the wide tensor-core
    quantizer (operands streamed from L2, one tile in tensor memory): several
    tiles with a ragged tail, a leading dimension above d, layout padding
    slots zero; equal to the rows quantised from a contiguous copy."""
    import ctypes

    ctx = _ctx(lib, d=d, bits=bits, seed=5)
    n = 3 * 128 + 45
    ld = d + 8
    k = W.search_vectors(n, d, seed=d + bits, which=0) * np.float32(7.0)
    k[7] = 0.0                                    # zero key
    wide = torch.zeros((n, ld), dtype=torch.float32)
    wide[:, :d] = torch.from_numpy(k)
    dev = wide.to(DEV)
    payload = torch.empty((n, ctx.row_bytes), dtype=torch.uint8, device=DEV)
    norms = torch.empty((n, 2), dtype=torch.float16, device=DEV)
    st = lib.lib().tq_quantize(ctx.handle, ctypes.c_void_p(dev.data_ptr()), 0, n, ld,
                               ctypes.c_void_p(payload.data_ptr()), ctypes.c_void_p(norms.data_ptr()),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    _status_clean(lib, ctx)
    check_quantize(payload.cpu().numpy(), norms.cpu().numpy(), k.astype(np.float64), tables_of(ctx))
    p2, n2 = lib.tq_quantize(ctx, torch.from_numpy(k).to(DEV))
    assert torch.equal(p2, payload) and torch.equal(n2.view(torch.int16), norms.view(torch.int16))
    codes, bits_ = O.unpack_rows(payload.cpu().numpy()[7:8], d, d, bits - 1)
    assert not codes.any() and bits_.all()


def test_quantize_edge_cases(lib):
    ctx = _ctx(lib, bits=4, seed=3)
    k = W.toy_keys(300, 128, seed=9)
    k[5] = 0.0                       # zero key
    k[17] *= 1e4                     # ||k|| above the fp16 range -> +inf norms
    k[40] = 0.0
    k[40][3] = 1.0                   # a basis vector
    wide = torch.zeros((300, 256), dtype=torch.bfloat16)
    wide[:, :128] = torch.from_numpy(k).to(torch.bfloat16)
    keys = wide.to(DEV)[:, :128]     # leading dimension 256
    payload = torch.empty((300, ctx.row_bytes), dtype=torch.uint8, device=DEV)
    norms = torch.empty((300, 2), dtype=torch.float16, device=DEV)
    import ctypes

    st = lib.lib().tq_quantize(ctx.handle, ctypes.c_void_p(keys.data_ptr()), 1, 300, 256,
                               ctypes.c_void_p(payload.data_ptr()), ctypes.c_void_p(norms.data_ptr()),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    # key 17's norm overflows fp16: the range bit is set, and the read clears it
    w = ctypes.c_uint32()
    assert lib.lib().tq_check_device_status(ctx.handle, None, ctypes.byref(w)) == 7   # TQ_ERR_RANGE
    assert w.value == lib.STATUS_RANGE
    _status_clean(lib, ctx)
    kk = wide[:, :128].to(torch.float64).numpy()
    nr = norms.cpu().numpy()
    assert np.all(nr[5] == 0) and np.isinf(nr[17, 0])
    codes, bits = O.unpack_rows(payload.cpu().numpy(), 128, 128, 3)
    assert np.all(codes[5] == 0) and np.all(bits[5])
    ok = np.ones(300, bool)
    ok[17] = False
    check_quantize(payload.cpu().numpy()[ok], nr[ok], kk[ok], tables_of(ctx))
    # n == 0 is a no-op; bad leading dimension is rejected
    assert lib.lib().tq_quantize(ctx.handle, ctypes.c_void_p(keys.data_ptr()), 1, 0, 256, None, None, None) == 0
    assert lib.lib().tq_quantize(ctx.handle, ctypes.c_void_p(keys.data_ptr()), 1, 10, 100,
                                 ctypes.c_void_p(payload.data_ptr()), ctypes.c_void_p(norms.data_ptr()),
                                 None) == 1


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d,m", [(128, 128), (128, 0), (64, 64)])
def test_quantize_flags_norms_out_of_fp16_range(lib, dtype, d, m):
    """Every quantizer path reports a norm that does not fit in fp16 through
    the context's status word; keys in range leave it clean."""
    ctx = _ctx(lib, d=d, bits=4, seed=3, m=m)
    k = torch.from_numpy(W.toy_keys(500, d, seed=2)).to(dtype)
    lib.tq_quantize(ctx, k.to(DEV))
    _status_clean(lib, ctx)
    k[333] *= 3e4
    _, norms = lib.tq_quantize(ctx, k.to(DEV))
    torch.cuda.synchronize()
    assert lib.tq_check_device_status(ctx) == lib.STATUS_RANGE
    nr = norms.cpu().numpy().view(np.float16)
    assert np.isinf(nr[333, 0]) and np.all(np.isfinite(np.delete(nr, 333, axis=0)))
    assert lib.tq_check_device_status(ctx) == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_bounded_wait_gives_up_and_context_recovers(lib, dtype):
    """The failure path of the tensor-core quantizer's bounded waits, forced
    with the test hook: with a wait budget of a few cycles the first wait that
    is not satisfied at once gives up, every role leaves its loop, the kernel
    returns, and the status word reports it (TQ_ERR_DEVICE); with the default
    budget restored the next call on the same context is complete and equal
    to the oracle."""
    import ctypes

    L = lib.lib()
    ctx = _ctx(lib, bits=4, seed=12)
    kt = torch.from_numpy(W.toy_keys(4133, 128, seed=31)).to(dtype)
    assert L.tq_set_wait_budget(ctx.handle, -1) == 1
    assert L.tq_set_wait_budget(ctx.handle, 4) == 0
    lib.tq_quantize(ctx, kt.to(DEV))
    torch.cuda.synchronize()
    w = ctypes.c_uint32()
    assert L.tq_check_device_status(ctx.handle, None, ctypes.byref(w)) == 6   # TQ_ERR_DEVICE
    assert w.value & lib.STATUS_QUANTIZE_WAIT
    assert L.tq_set_wait_budget(ctx.handle, 0) == 0
    payload, norms = lib.tq_quantize(ctx, kt.to(DEV))
    _status_clean(lib, ctx)
    check_quantize(payload.cpu().numpy(), norms.cpu().numpy(), kt.to(torch.float64).numpy(), tables_of(ctx))


def test_quantize_is_deterministic(lib):
    ctx = _ctx(lib, bits=3, seed=1)
    kb = torch.from_numpy(W.toy_keys(3000, 128, seed=4)).to(torch.bfloat16).to(DEV)
    p1, n1 = lib.tq_quantize(ctx, kb)
    p2, n2 = lib.tq_quantize(ctx, kb)
    assert torch.equal(p1, p2) and torch.equal(n1.view(torch.int16), n2.view(torch.int16))


def _cache(lib, ctx, B, Hkv, S, seed):
    scales = W.head_channel_scales(Hkv, ctx.d, seed)
    k = np.stack([np.stack([W.decode_keys_pair(b, h, S, ctx.d, scales, seed) for h in range(Hkv)])
                  for b in range(B)])
    kb = torch.from_numpy(k).to(torch.bfloat16).to(DEV).reshape(-1, ctx.d)
    return lib.tq_quantize(ctx, kb)


@pytest.mark.parametrize("m", [128, 0])
@pytest.mark.parametrize("bits,B,Hkv,G,S", [(3, 2, 2, 4, 1037), (4, 1, 3, 4, 515), (4, 2, 2, 1, 200),
                                            (3, 1, 2, 2, 333), (2, 2, 1, 8, 129), (4, 1, 1, 12, 100),
                                            (4, 1, 2, 3, 16), (3, 1, 1, 64, 300), (4, 2, 1, 16, 257),
                                            (2, 1, 2, 12, 100), (4, 1, 1, 9, 77)])
def test_logits_against_oracle(lib, bits, B, Hkv, G, S, m):
    """With the sign term (m = 128) and without it (m = 0, MSE-only), on the
    int8 MMA kernel; G > 8 (9, 12, 16 and the toy batch's 64) runs as chunks
    of 8 query heads that each stream the rows again."""
    ctx = _ctx(lib, bits=bits, seed=21, m=m)
    payload, norms = _cache(lib, ctx, B, Hkv, S, seed=31)
    Hq = Hkv * G
    q = W.queries((B, Hq, 128), seed=41)
    scale = 1.0 / math.sqrt(128)
    out = lib.tq_logits(ctx, torch.from_numpy(q).to(DEV), payload, norms, Hkv, scale=scale)
    _status_clean(lib, ctx)
    tb = tables_of(ctx)
    pl, nr, o = payload.cpu().numpy(), norms.cpu().numpy(), out.cpu().numpy()
    for b in range(B):
        for hk in range(Hkv):
            rows = slice((b * Hkv + hk) * S, (b * Hkv + hk + 1) * S)
            s, A = oracle_estimates(pl[rows], nr[rows], q[b, hk * G:(hk + 1) * G].astype(np.float64), tb)
            check_close(o[b, hk * G:(hk + 1) * G], scale * s, scale * A, rel_floor=REL_FLOOR)


@pytest.mark.parametrize("d,bits", [(200, 2), (200, 4), (72, 3)])
def test_logits_padded_layout_against_oracle(lib, d, bits):
    """d not a multiple of 64 (vector-search d = 200): the CUDA-core estimator
    on the padded layout."""
    ctx = _ctx(lib, d=d, bits=bits, seed=23)
    B, Hkv, G, S = 1, 2, 3, 301
    k = W.search_vectors(B * Hkv * S, d, seed=7, which=0)
    payload, norms = lib.tq_quantize(ctx, torch.from_numpy(k).to(DEV))
    q = W.search_vectors(B * Hkv * G, d, seed=7, which=1).reshape(B, Hkv * G, d)
    out = lib.tq_logits(ctx, torch.from_numpy(q).to(DEV), payload, norms, Hkv)
    _status_clean(lib, ctx)
    tb = tables_of(ctx)
    pl, nr, o = payload.cpu().numpy(), norms.cpu().numpy(), out.cpu().numpy()
    for hk in range(Hkv):
        rows = slice(hk * S, (hk + 1) * S)
        s_, A = oracle_estimates(pl[rows], nr[rows], q[0, hk * G:(hk + 1) * G].astype(np.float64), tb)
        check_close(o[0, hk * G:(hk + 1) * G], s_, A)


def test_toy_logits_all_pairs(lib):
    """toy workload: 64 queries x 4096 keys, all pairs (one GQA group of 64)."""
    ctx = _ctx(lib, bits=3, seed=42)
    k = W.toy_keys(4096, 128, seed=1000)
    payload, norms = lib.tq_quantize(ctx, torch.from_numpy(k).to(DEV))
    q = W.queries((1, 64, 128), seed=1001)
    out = lib.tq_logits(ctx, torch.from_numpy(q).to(DEV), payload, norms, 1)
    _status_clean(lib, ctx)
    s, A = oracle_estimates(payload.cpu().numpy(), norms.cpu().numpy(), q[0].astype(np.float64), tables_of(ctx))
    check_close(out.cpu().numpy()[0], s, A, rel_floor=REL_FLOOR)


@pytest.mark.parametrize("full", [True, False])
@pytest.mark.parametrize("d,bits", [(128, 4), (64, 2), (200, 4)])
def test_dequantize_against_oracle(lib, full, d, bits):
    ctx = _ctx(lib, d=d, bits=bits, seed=13)
    k = W.toy_keys(555, d, seed=8)
    payload, norms = lib.tq_quantize(ctx, torch.from_numpy(k).to(DEV))
    xh = lib.tq_dequantize(ctx, payload, norms, full=full)
    _status_clean(lib, ctx)
    tb = tables_of(ctx)
    codes, bits_ = O.unpack_rows(payload.cpu().numpy(), d, d, tb.bmse)
    nr = norms.cpu().numpy().astype(np.float64)
    ref = O.dequantize(codes, bits_, nr[:, 0], nr[:, 1], tb, full=full)
    # fp32 accumulation over d + m terms: bound by the sum of the magnitudes
    v = nr[:, :1] * np.abs(tb.c[codes]).sum(1, keepdims=True)
    if full:
        v = v + O.QJL_CONST / tb.m * nr[:, 1:2] * np.abs(tb.P).sum()
    err = np.abs(xh.cpu().numpy() - ref)
    assert np.all(err <= 2e-5 * v), float(np.max(err / v))


def test_dequantize_full_matches_logits(lib):
    ctx = _ctx(lib, bits=3, seed=2)
    payload, norms = _cache(lib, ctx, 1, 1, 300, seed=5)
    xh = lib.tq_dequantize(ctx, payload, norms, full=True)
    q = torch.from_numpy(W.queries((1, 4, 128), seed=6)).to(DEV)
    out = lib.tq_logits(ctx, q, payload, norms, 1)
    ref = (q[0].double() @ xh.double().T).cpu().numpy()
    _, A = oracle_estimates(payload.cpu().numpy(), norms.cpu().numpy(), q[0].cpu().double().numpy(), tables_of(ctx))
    check_close(out[0].cpu().numpy(), ref, A)


@pytest.mark.parametrize("d,bits,n,nq,k", [(128, 3, 5000, 16, 10), (128, 4, 3001, 9, 1), (128, 2, 700, 5, 64),
                                           (128, 3, 100, 3, 10), (200, 2, 3000, 7, 10), (200, 4, 2000, 5, 10),
                                           (104, 3, 3000, 6, 10), (72, 2, 1500, 4, 5)])
def test_topk_against_oracle(lib, d, bits, n, nq, k):
    ctx = _ctx(lib, d=d, bits=bits, seed=17)
    db = W.search_vectors(n, d, seed=100 + bits, which=0)
    qs = W.search_vectors(nq, d, seed=100 + bits, which=1)
    payload, norms = lib.tq_quantize(ctx, torch.from_numpy(db).to(DEV))
    ids, scores = lib.tq_topk(ctx, torch.from_numpy(qs).to(DEV), payload, norms, k)
    _status_clean(lib, ctx)
    s, A = oracle_estimates(payload.cpu().numpy(), norms.cpu().numpy(), qs.astype(np.float64), tables_of(ctx))
    ids = ids.cpu().numpy()
    order = np.array([np.lexsort((np.arange(n), -s[i]))[:k + 1] for i in range(nq)])
    near_tie = 0
    for i in range(nq):
        kth, nxt = s[i, order[i, k - 1]], s[i, order[i, min(k, n - 1)]] if k < n else -np.inf
        if k < n and kth - nxt < 1e-6 * A[i].max():
            near_tie += 1
            assert set(ids[i][:k - 1]) <= set(order[i][:k + 1])
            continue
        np.testing.assert_array_equal(ids[i], order[i, :k])
    assert near_tie <= max(1, nq // 10)
    np.testing.assert_allclose(scores.cpu().numpy(), np.take_along_axis(s, ids, 1), rtol=1e-6,
                               atol=1e-6 * A.max())


@pytest.mark.parametrize("d,bits,n,nq", [(200, 2, 20000, 500), (128, 4, 20000, 500), (200, 4, 12000, 2100)])
def test_topk_many_query_tiles(lib, d, bits, n, nq):
    """More (query tile, row tile) units than SMs: CTAs switch query tiles
    inside their range of the tensor-core search.  With 2100 queries (17 tiles)
    the CTAs work in groups of four over the same row tiles, and three members
    of the last group have no query tile."""
    ctx = _ctx(lib, d=d, bits=bits, seed=19)
    k = 10
    db = W.search_vectors(n, d, seed=300 + bits, which=0)
    qs = W.search_vectors(nq, d, seed=300 + bits, which=1)
    payload, norms = lib.tq_quantize(ctx, torch.from_numpy(db).to(DEV))
    ids, scores = lib.tq_topk(ctx, torch.from_numpy(qs).to(DEV), payload, norms, k)
    _status_clean(lib, ctx)
    s, A = oracle_estimates(payload.cpu().numpy(), norms.cpu().numpy(), qs.astype(np.float64), tables_of(ctx))
    ids = ids.cpu().numpy()
    near_tie = 0
    for i in range(nq):
        order = np.lexsort((np.arange(n), -s[i]))[:k + 1]
        if s[i, order[k - 1]] - s[i, order[k]] < 1e-6 * A[i].max():
            near_tie += 1
            assert set(ids[i][:k - 1]) <= set(order)
            continue
        np.testing.assert_array_equal(ids[i], order[:k])
    assert near_tie <= nq // 20
    np.testing.assert_allclose(scores.cpu().numpy(), np.take_along_axis(s, ids, 1), rtol=1e-6, atol=1e-6 * A.max())


def _oracle_scores_chunked(payload, norms, Q64, tb: O.Tables, chunk: int = 131072):
    """Oracle estimates (and abs-term sums) of every (query, row) pair, taken
    over row chunks so that host memory stays bounded at 10^6 rows."""
    n = payload.shape[0]
    s = np.empty((Q64.shape[0], n))
    A = np.empty_like(s)
    for r0 in range(0, n, chunk):
        r1 = min(n, r0 + chunk)
        s[:, r0:r1], A[:, r0:r1] = oracle_estimates(payload[r0:r1], norms[r0:r1], Q64, tb)
    return s, A


def _oracle_topk_order(si: np.ndarray, k: int) -> np.ndarray:
    """The oracle's first k + 1 rows of one query: score descending, ties to the lower id."""
    n = si.shape[0]
    if n <= k + 1:
        cand = np.arange(n)
    else:
        thr = np.partition(si, n - (k + 1))[n - (k + 1)]
        cand = np.nonzero(si >= thr)[0]
    return cand[np.lexsort((cand, -si[cand]))][:k + 1]


def _search_sampled(lib, n, nq, bits, k=10, d=200, n_sample=8, chunk=131072, max_near_tie=2):
    ctx = _ctx(lib, d=d, bits=bits, seed=42)
    db = W.search_vectors(n, d, seed=1004, which=0)
    qs = W.search_vectors(nq, d, seed=1004, which=1)
    payload, norms = lib.tq_quantize(ctx, torch.from_numpy(db).to(DEV))
    ids, scores = lib.tq_topk(ctx, torch.from_numpy(qs).to(DEV), payload, norms, k)
    _status_clean(lib, ctx)
    tb = tables_of(ctx)
    pay, nrm = payload.cpu().numpy(), norms.cpu().numpy()
    rng = np.random.default_rng(100 + bits)
    rows = np.sort(rng.choice(n, min(n, 2000), replace=False))
    rows[-1] = n - 1
    check_quantize(pay[rows], nrm[rows], db[rows].astype(np.float64), tb)
    sample = np.concatenate([[0, nq - 1], rng.choice(np.arange(1, nq - 1), n_sample - 2, replace=False)])
    s, A = _oracle_scores_chunked(pay, nrm, qs[sample].astype(np.float64), tb, chunk)
    got_ids, got_scores = ids.cpu().numpy()[sample], scores.cpu().numpy()[sample]
    near_tie = 0
    for i in range(len(sample)):
        order = _oracle_topk_order(s[i], k)
        if k < n and s[i, order[k - 1]] - s[i, order[k]] < 1e-6 * A[i].max():
            near_tie += 1
            assert set(got_ids[i][:k - 1]) <= set(order)
            continue
        np.testing.assert_array_equal(got_ids[i], order[:k])
    assert near_tie <= max_near_tie
    np.testing.assert_allclose(got_scores, np.take_along_axis(s, got_ids, 1), rtol=1e-6, atol=1e-6 * A.max())


@pytest.mark.parametrize("bits", [2, 4])
def test_search_full_size_sampled(lib, bits):
    """The search workload in the launch configuration bench.py times: 10^6
    unit vectors in d = 200 indexed, 10^4 queries, k = 10, tables seed 42.
    2000 sampled rows of the index against the oracle's quantisation, and the
    answers of eight queries (the first, the last, six seeded) against the
    oracle's top-k over all 10^6 rows."""
    _search_sampled(lib, 1_000_000, 10_000, bits)


def test_topk_identical_rows_take_lowest_ids(lib):
    """3000 copies of one vector: every row ties, the candidate list overflows
    and the exact scan returns ids 0 .. k-1 (ties go to the lower id)."""
    ctx = _ctx(lib, d=200, bits=4, seed=3)
    v = W.search_vectors(1, 200, seed=9, which=0)
    db = np.repeat(v, 3000, axis=0)
    qs = W.search_vectors(4, 200, seed=9, which=1)
    payload, norms = lib.tq_quantize(ctx, torch.from_numpy(db).to(DEV))
    ids, scores = lib.tq_topk(ctx, torch.from_numpy(qs).to(DEV), payload, norms, 10)
    _status_clean(lib, ctx)
    np.testing.assert_array_equal(ids.cpu().numpy(), np.tile(np.arange(10), (4, 1)))
    s, A = oracle_estimates(payload.cpu().numpy()[:1], norms.cpu().numpy()[:1], qs.astype(np.float64), tables_of(ctx))
    np.testing.assert_allclose(scores.cpu().numpy(), np.repeat(s, 10, axis=1), rtol=1e-6, atol=1e-6 * A.max())


def test_logits_rejects_bad_workspace(lib):
    ctx = _ctx(lib, bits=3, seed=1)
    payload, norms = _cache(lib, ctx, 1, 1, 64, seed=1)
    q = torch.zeros((1, 4, 128), device=DEV)
    small = torch.empty(256, dtype=torch.uint8, device=DEV)
    with pytest.raises(lib.TQError) as e:
        lib.tq_logits(ctx, q, payload, norms, 1, workspace=small)
    assert e.value.status == 5


# --------------------------------------------------------------------------
# Full-size workloads, sampled (the configuration bench.py times)
# --------------------------------------------------------------------------


@pytest.mark.parametrize("name,B,Hkv,G,S,bits,m", [("decode", 8, 8, 4, 32768, 4, 128),
                                                   ("longctx", 1, 8, 4, 131072, 3, 128),
                                                   ("decode_mse_only", 8, 8, 4, 32768, 4, 0)])
def test_full_size_sampled(lib, name, B, Hkv, G, S, bits, m):
    seed = 1002 if name == "longctx" else 1001
    ctx = _ctx(lib, bits=bits, seed=42, m=m)
    keys = W.decode_keys(B, Hkv, S, 128, seed, device=DEV).reshape(-1, 128)
    payload, norms = lib.tq_quantize(ctx, keys)
    Hq = Hkv * G
    q = W.queries((B, Hq, 128), seed=seed + 7)
    out = lib.tq_logits(ctx, torch.from_numpy(q).to(DEV), payload, norms, Hkv, scale=1.0 / math.sqrt(128))
    _status_clean(lib, ctx)
    tb = tables_of(ctx)
    rng = np.random.default_rng(0)
    pairs = [(0, 0), (B - 1, Hkv - 1), (B // 2, 3)]
    rep = {}
    for b, h in pairs:
        s_idx = np.sort(rng.choice(S, 1500, replace=False))
        s_idx[-1] = S - 1
        rows = (b * Hkv + h) * S + s_idx
        k64 = W.decode_keys_rows(b, h, s_idx, S, 128, Hkv, seed)
        check_quantize(payload[rows].cpu().numpy(), norms[rows].cpu().numpy(), k64, tb, rep)
        est, A = oracle_estimates(payload[rows].cpu().numpy(), norms[rows].cpu().numpy(),
                                  q[b, h * G:(h + 1) * G].astype(np.float64), tb)
        got = out[b, h * G:(h + 1) * G][:, torch.from_numpy(s_idx).to(DEV)].cpu().numpy()
        check_close(got, est / math.sqrt(128), A / math.sqrt(128), rel_floor=REL_FLOOR, report=rep)
    print(f"{name}: {format_stats(rep)}; logits worst {rep['logits_worst_of_A']:.2e} of A, "
          f"{rep['logits_worst_rel']:.2e} relative where |s| >= {REL_FLOOR} A")


# --------------------------------------------------------------------------
# MSE-only variant (m = 0) and decode-time append
# --------------------------------------------------------------------------


@pytest.mark.parametrize("d,bits,dtype", [(128, 4, torch.bfloat16), (64, 2, torch.float32), (200, 3, torch.float32)])
def test_mse_only_quantize_logits_dequantize(lib, d, bits, dtype):
    ctx = _ctx(lib, d=d, bits=bits, seed=27, m=0)
    assert ctx.m == 0 and ctx.row_bytes == -(-d // 64) * 64 * (bits - 1) // 8
    k = W.toy_keys(900, d, seed=4)
    kt = torch.from_numpy(k).to(dtype)
    payload, norms = lib.tq_quantize(ctx, kt.to(DEV))
    _status_clean(lib, ctx)
    tb = tables_of(ctx)
    check_quantize(payload.cpu().numpy(), norms.cpu().numpy(), kt.to(torch.float64).numpy(), tb)
    q = W.queries((1, 3, d), seed=5)
    out = lib.tq_logits(ctx, torch.from_numpy(q).to(DEV), payload, norms, 1)
    _status_clean(lib, ctx)
    s, A = oracle_estimates(payload.cpu().numpy(), norms.cpu().numpy(), q[0].astype(np.float64), tb)
    check_close(out.cpu().numpy()[0], s, A)
    xh = lib.tq_dequantize(ctx, payload, norms, full=True).cpu().numpy()
    codes, bits_ = O.unpack_rows(payload.cpu().numpy(), d, 0, tb.bmse)
    nr = norms.cpu().numpy().astype(np.float64)
    ref = O.dequantize(codes, bits_, nr[:, 0], nr[:, 1], tb, full=True)
    v = nr[:, :1] * np.abs(tb.c[codes]).sum(1, keepdims=True)
    assert np.all(np.abs(xh - ref) <= 2e-5 * v)


def test_mse_only_topk(lib):
    ctx = _ctx(lib, d=200, bits=4, seed=31, m=0)
    n, nq, k = 4000, 20, 10
    db = W.search_vectors(n, 200, seed=77, which=0)
    qs = W.search_vectors(nq, 200, seed=77, which=1)
    payload, norms = lib.tq_quantize(ctx, torch.from_numpy(db).to(DEV))
    ids, scores = lib.tq_topk(ctx, torch.from_numpy(qs).to(DEV), payload, norms, k)
    _status_clean(lib, ctx)
    s, A = oracle_estimates(payload.cpu().numpy(), norms.cpu().numpy(), qs.astype(np.float64), tables_of(ctx))
    ids = ids.cpu().numpy()
    for i in range(nq):
        order = np.lexsort((np.arange(n), -s[i]))[:k + 1]
        if s[i, order[k - 1]] - s[i, order[k]] < 1e-6 * A[i].max():
            assert set(ids[i][:k - 1]) <= set(order)
            continue
        np.testing.assert_array_equal(ids[i], order[:k])


@pytest.mark.parametrize("m", [128, 0])
def test_decode_time_append_matches_batch(lib, m):
    """A decode loop quantizes one new key per step into the next cache row;
    the rows equal those of one batched call (tensor-core path for m = 128 at
    n = 1, CUDA-core path for m = 0)."""
    ctx = _ctx(lib, d=128, bits=4, seed=8, m=m)
    keys = torch.from_numpy(W.toy_keys(40, 128, seed=12)).to(torch.bfloat16).to(DEV)
    batch_p, batch_n = lib.tq_quantize(ctx, keys)
    cache_p = torch.zeros_like(batch_p)
    cache_n = torch.zeros_like(batch_n)
    for s in range(keys.shape[0]):
        lib.tq_quantize(ctx, keys[s:s + 1], cache_p[s:s + 1], cache_n[s:s + 1])
    _status_clean(lib, ctx)
    assert torch.equal(cache_p, batch_p)
    assert torch.equal(cache_n, batch_n)
