"""GPU parity of the value path (tq_attend) against the oracle.

Given identical logits (seeded synthetic arrays) and the same packed value
cache, the attention output must satisfy |o_gpu - o_oracle| <= 1e-3 A, A the
oracle's softmax-weighted sum of the absolute values of every term of the
reconstructions.  The end-to-end test (tq_logits, then tq_attend, against the
oracle's logits and attention from the same packed caches) widens the band by
the logits' own deviation: a logit error dl changes each softmax weight by a
factor within exp(+-2 max|dl|), so the output moves by at most
(exp(2 max|dl|) - 1) A."""

import math

import numpy as np
import pytest
import torch

from compressed_kv_cache_tq_b200 import workloads as W
from oracle import tq_oracle as O

from tests.parity import check_close, check_quantize, oracle_estimates, tables_of

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _values(B, Hkv, S, d, seed):
    k = W.decode_keys(B, Hkv, S, d, seed, device="cpu").reshape(-1, d)
    return k.to(DEV), k.to(torch.float64).numpy()


def _oracle_attention(logits, payload, norms, tb, Hkv):
    codes, bits = O.unpack_rows(np.asarray(payload), tb.d, tb.m, tb.bmse)
    nr = np.asarray(norms).view(np.float16).reshape(-1, 2)
    return O.attention_output(logits, codes, bits, nr[:, 0], nr[:, 1], tb, Hkv)


@pytest.mark.parametrize("B,Hkv,G,S,d,bits,m", [(2, 2, 4, 517, 128, 4, 128), (1, 3, 2, 64, 128, 3, 128),
                                                (2, 1, 8, 1000, 128, 2, 128), (1, 2, 1, 33, 64, 3, 64),
                                                (1, 1, 4, 300, 200, 3, 200), (1, 2, 4, 257, 128, 4, 0),
                                                (2, 2, 4, 1, 128, 4, 128), (1, 2, 3, 190, 128, 3, 128),
                                                (1, 2, 1, 300, 128, 4, 128), (2, 1, 2, 700, 128, 2, 128),
                                                (1, 1, 4, 600, 128, 2, 0), (1, 1, 4, 3000, 128, 3, 0)])
def test_attend_against_oracle(lib, B, Hkv, G, S, d, bits, m):
    """d = m = 128 (or m = 0) with up to 4 query heads per KV head runs on the
    tensor-core kernel, the other shapes on CUDA cores; S up to 3000 gives
    several key tiles per chunk."""
    ctx = lib.tq_init(d, bits, 77, m=m)
    v, V64 = _values(B, Hkv, S, d, seed=2001 + S)
    payload, norms = lib.tq_quantize(ctx, v)
    tb = tables_of(ctx)
    check_quantize(payload.cpu().numpy(), norms.cpu().numpy(), V64, tb)
    logits = 3.0 * W.queries((B, Hkv * G, S), seed=31 + S)
    out = lib.tq_attend(ctx, torch.from_numpy(logits).to(DEV), payload, norms, Hkv)
    torch.cuda.synchronize()
    ref, A = _oracle_attention(logits.astype(np.float64), payload.cpu().numpy(), norms.cpu().numpy(), tb, Hkv)
    check_close(out.cpu().numpy(), ref, A)


def test_attend_running_maximum_and_masked_keys(lib):
    """Logits whose maximum keeps rising along the keys (each warp's running
    maximum, and with it every partial sum, is rescaled many times), falling
    ones, a wide range (most weights underflow), and masked keys (-inf): a
    random 30 % of the keys, and the whole first half of one head's keys, so
    that some chunks of that head have no weight at all."""
    B, Hkv, G, S, d = 1, 2, 4, 3000, 128
    ctx = lib.tq_init(d, 4, 91)
    v, V64 = _values(B, Hkv, S, d, seed=4401)
    payload, norms = lib.tq_quantize(ctx, v)
    tb = tables_of(ctx)
    logits = W.queries((B, Hkv * G, S), seed=4402).astype(np.float64)
    ramp = np.arange(S) / S
    logits[0, 0] += 40.0 * ramp            # rising
    logits[0, 1] -= 40.0 * ramp            # falling
    logits[0, 2] *= 20.0                   # wide range
    logits[0, 3] += 8.0 * np.sin(ramp * 37.0)
    rng = np.random.default_rng(4403)
    logits[0, 4:8][:, rng.random(S) < 0.3] = -np.inf
    logits[0, 5, : S // 2] = -np.inf
    out = lib.tq_attend(ctx, torch.from_numpy(logits.astype(np.float32)).to(DEV), payload, norms, Hkv)
    torch.cuda.synchronize()
    ref, A = _oracle_attention(logits.astype(np.float32).astype(np.float64), payload.cpu().numpy(),
                               norms.cpu().numpy(), tb, Hkv)
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    check_close(got, ref, A)


def test_attend_without_keys_is_zero(lib):
    ctx = lib.tq_init(128, 4, 77)
    payload = torch.empty((0, ctx.row_bytes), dtype=torch.uint8, device=DEV)
    norms = torch.empty((0, 2), dtype=torch.float16, device=DEV)
    out = lib.tq_attend(ctx, torch.empty((2, 8, 0), device=DEV), payload, norms, 2)
    torch.cuda.synchronize()
    assert out.shape == (2, 8, 128) and not out.abs().any()


def test_attend_rejects_more_than_eight_heads_per_kv_head(lib):
    ctx = lib.tq_init(128, 4, 77)
    v, _ = _values(1, 1, 10, 128, seed=5)
    payload, norms = lib.tq_quantize(ctx, v)
    with pytest.raises(lib.TQError):
        lib.tq_attend(ctx, torch.zeros((1, 16, 10), device=DEV), payload, norms, 1)


def test_decode_attention_end_to_end(lib):
    """keys -> tq_quantize -> tq_logits -> tq_attend over values -> output."""
    B, Hkv, G, S, d = 2, 2, 4, 700, 128
    kctx, vctx = lib.tq_init(d, 4, 42), lib.tq_init(d, 4, 142)
    k, K64 = _values(B, Hkv, S, d, seed=3001)
    v, V64 = _values(B, Hkv, S, d, seed=3002)
    kp, kn = lib.tq_quantize(kctx, k)
    vp, vn = lib.tq_quantize(vctx, v)
    q = W.queries((B, Hkv * G, d), seed=3003)
    scale = 1.0 / math.sqrt(d)
    lg = lib.tq_logits(kctx, torch.from_numpy(q).to(DEV), kp, kn, Hkv, scale=scale)
    out = lib.tq_attend(vctx, lg, vp, vn, Hkv)
    torch.cuda.synchronize()
    tk, tv = tables_of(kctx), tables_of(vctx)
    # the oracle's logits from the same packed keys
    ref_lg = np.empty((B, Hkv * G, S))
    absl = np.empty_like(ref_lg)
    kpn, knn = kp.cpu().numpy().reshape(B, Hkv, S, -1), kn.cpu().numpy().reshape(B, Hkv, S, 2)
    for b in range(B):
        for h in range(Hkv):
            est, A = oracle_estimates(kpn[b, h], knn[b, h], q[b, h * G:(h + 1) * G].astype(np.float64), tk)
            ref_lg[b, h * G:(h + 1) * G] = scale * est
            absl[b, h * G:(h + 1) * G] = scale * A
    check_close(lg.cpu().numpy(), ref_lg, absl)
    dl = float(np.max(np.abs(lg.cpu().numpy().astype(np.float64) - ref_lg)))
    ref, A = _oracle_attention(ref_lg, vp.cpu().numpy(), vn.cpu().numpy(), tv, Hkv)
    widen = math.expm1(2.0 * dl)
    check_close(out.cpu().numpy(), ref, A, tol=1e-3 + widen)


def test_attend_full_size_sampled(lib):
    """The decode workload's shape (batch 8, 8 KV heads, 32 query heads, seq
    32768, b = 4, several key tiles per chunk and several chunks per group):
    every output of six (batch, KV head) groups."""
    B, Hkv, G, S, d = 8, 8, 4, 32768, 128
    ctx = lib.tq_init(d, 4, 142)
    v = W.decode_keys(B, Hkv, S, d, 2002, device=DEV).reshape(-1, d)
    payload, norms = lib.tq_quantize(ctx, v)
    logits = torch.from_numpy(3.0 * W.queries((B, Hkv * G, S), seed=2003)).to(DEV)
    out = lib.tq_attend(ctx, logits, payload, norms, Hkv)
    torch.cuda.synchronize()
    assert lib.tq_check_device_status(ctx) == 0
    tb = tables_of(ctx)
    lg = logits.cpu().numpy().astype(np.float64)
    for b, h in [(0, 0), (B - 1, Hkv - 1), (3, 5), (4, 6), (2, 0), (5, 1)]:
        rows = slice((b * Hkv + h) * S, (b * Hkv + h + 1) * S)
        ref, A = _oracle_attention(lg[b:b + 1, h * G:(h + 1) * G], payload[rows].cpu().numpy(),
                                   norms[rows].cpu().numpy(), tb, 1)
        check_close(out[b, h * G:(h + 1) * G].cpu().numpy(), ref[0], A[0])


def test_attend_argument_errors(lib):
    """A short workspace and misaligned rows are refused before any launch."""
    import ctypes

    ctx = lib.tq_init(128, 4, 77)
    v, _ = _values(1, 2, 64, 128, seed=6)
    payload, norms = lib.tq_quantize(ctx, v)
    logits = torch.zeros((1, 8, 64), device=DEV)
    out = torch.empty((1, 8, 128), device=DEV)
    L = lib.lib()
    need = lib.tq_attend_workspace_bytes(ctx, 1, 8, 2, 64)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    vp = ctypes.c_void_p
    assert L.tq_attend(ctx.handle, vp(logits.data_ptr()), 1, 8, 2, 64, vp(payload.data_ptr()), vp(norms.data_ptr()),
                       vp(out.data_ptr()), vp(ws.data_ptr()), need - 1, None) == 5
    assert L.tq_attend(ctx.handle, vp(logits.data_ptr()), 1, 8, 2, 64, vp(payload.data_ptr() + 8),
                       vp(norms.data_ptr()), vp(out.data_ptr()), vp(ws.data_ptr()), need, None) == 1
    assert L.tq_attend(ctx.handle, vp(logits.data_ptr()), 1, 8, 3, 64, vp(payload.data_ptr()), vp(norms.data_ptr()),
                       vp(out.data_ptr()), vp(ws.data_ptr()), need, None) == 1
