"""GPU parity of the channel split (fractional bit rates) against the oracle.

The plan (channel order per KV head) is compared with the oracle's exactly,
except at a near-tie of two variances at the cut, where any valid order is
accepted.  Quantisation and logits run on the oracle's plan, set into the
split from the host, so both sides quantise the same groups; each group is
then held to the single-quantizer bands of tests/parity.py."""

import math

import numpy as np
import pytest
import torch

from compressed_kv_cache_tq_b200 import workloads as W
from oracle import tq_oracle as O

from tests.parity import check_close, check_quantize, tables_of

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _status_clean(lib, *ctxs):
    torch.cuda.synchronize()
    for c in ctxs:
        assert lib.tq_check_device_status(c) == 0


def _keys(B, Hkv, S, d, seed, dtype=torch.bfloat16, offset=0.0):
    """Keys drawn like the decode workload (per-head channel scales, outlier
    channels), optionally shifted by a per-channel offset; returns the device
    tensor and its exact values as float64 on the host."""
    scales = W.head_channel_scales(Hkv, d, seed)
    k = np.stack([np.stack([W.decode_keys_pair(b, h, S, d, scales, seed) for h in range(Hkv)]) for b in range(B)])
    if offset:
        k = k + offset * np.arange(d, dtype=np.float32)[None, None, None, :]
    t = torch.from_numpy(k.astype(np.float32)).to(dtype)
    return t.to(DEV), t.to(torch.float64).numpy()


def check_plan(perm_gpu, K64, d_hi):
    """The GPU's channel order equals the oracle's; at a near-tie of the
    variances at the cut (relative 1e-9) any split that respects the
    variances and keeps both groups in ascending order is accepted."""
    perm_ora = O.split_plan(K64, d_hi)
    B, Hkv, S, d = K64.shape
    ties = 0
    for h in range(Hkv):
        if np.array_equal(perm_gpu[h], perm_ora[h]):
            continue
        X = K64[:, h].reshape(-1, d)
        var = X.var(axis=0) if X.shape[0] else np.zeros(d)
        hi, lo = perm_gpu[h, :d_hi], perm_gpu[h, d_hi:]
        assert sorted(perm_gpu[h].tolist()) == list(range(d))
        assert np.all(np.diff(hi) > 0) and np.all(np.diff(lo) > 0)
        cut_hi, cut_lo = var[hi].min(), var[lo].max()
        assert cut_hi >= cut_lo * (1 - 1e-9), f"head {h}: plan differs from the oracle's away from a tie"
        ties += 1
    return ties


@pytest.mark.parametrize("dtype,offset", [(torch.bfloat16, 0.0), (torch.float32, 0.0), (torch.float32, 300.0)])
def test_split_plan_matches_oracle(lib, dtype, offset):
    hi, lo = lib.tq_init(64, 3, 42), lib.tq_init(64, 2, 43)
    sp = lib.tq_split_create(hi, lo, 3)
    keys, K64 = _keys(2, 3, 301, 128, seed=1003, dtype=dtype, offset=offset)
    sp.plan(keys)
    check_plan(sp.get_plan(), K64, 64)


def test_split_plan_without_keys_is_identity(lib):
    hi, lo = lib.tq_init(64, 3, 42), lib.tq_init(64, 2, 43)
    sp = lib.tq_split_create(hi, lo, 2)
    sp.set_plan(np.tile(np.arange(128)[::-1], (2, 1)))
    sp.plan(torch.empty((1, 2, 0, 128), dtype=torch.bfloat16, device=DEV))
    assert sp.get_plan().tolist() == [list(range(128))] * 2


def test_split_set_plan_rejects_non_permutations(lib):
    hi, lo = lib.tq_init(64, 3, 42), lib.tq_init(64, 2, 43)
    sp = lib.tq_split_create(hi, lo, 1)
    bad = np.arange(128)[None].copy()
    bad[0, 5] = 4
    with pytest.raises(lib.TQError):
        sp.set_plan(bad)


def _quantize_and_check(lib, sp, keys, K64, perm, rep=None):
    hi, lo = sp.hi, sp.lo
    sp.set_plan(perm)
    ph, nh, pl, nl = lib.tq_split_quantize(sp, keys)
    _status_clean(lib, hi, lo)
    Khi, Klo = O.split_groups(K64, perm, hi.d)
    check_quantize(ph.cpu().numpy(), nh.cpu().numpy(), Khi.reshape(-1, hi.d), tables_of(hi), rep)
    check_quantize(pl.cpu().numpy(), nl.cpu().numpy(), Klo.reshape(-1, lo.d), tables_of(lo), rep)
    return ph, nh, pl, nl


@pytest.mark.parametrize("bits_hi,bits_lo", [(3, 2), (4, 3), (2, 4), (3, 3), (4, 2), (2, 2)])
@pytest.mark.parametrize("B,Hkv,S", [(2, 3, 301), (1, 2, 128), (3, 1, 5)])
def test_split_quantize_tensor_core_path(lib, bits_hi, bits_lo, B, Hkv, S):
    hi, lo = lib.tq_init(64, bits_hi, 42), lib.tq_init(64, bits_lo, 43)
    sp = lib.tq_split_create(hi, lo, Hkv)
    keys, K64 = _keys(B, Hkv, S, 128, seed=1003 + S)
    _quantize_and_check(lib, sp, keys, K64, O.split_plan(K64, 64))


def test_split_quantize_arbitrary_order(lib):
    """Any channel order (not just the plan's ascending groups) gathers correctly."""
    hi, lo = lib.tq_init(64, 3, 42), lib.tq_init(64, 2, 43)
    sp = lib.tq_split_create(hi, lo, 3)
    keys, K64 = _keys(2, 3, 200, 128, seed=77)
    rng = np.random.default_rng(5)
    perm = np.stack([rng.permutation(128) for _ in range(3)])
    _quantize_and_check(lib, sp, keys, K64, perm)


@pytest.mark.parametrize("d_hi,d_lo,bits_hi,bits_lo,dtype", [(64, 64, 3, 2, torch.float32),
                                                             (72, 64, 3, 2, torch.bfloat16),
                                                             (128, 64, 4, 2, torch.float32)])
def test_split_quantize_cuda_core_path(lib, d_hi, d_lo, bits_hi, bits_lo, dtype):
    hi, lo = lib.tq_init(d_hi, bits_hi, 42), lib.tq_init(d_lo, bits_lo, 43)
    d = d_hi + d_lo
    sp = lib.tq_split_create(hi, lo, 2)
    keys, K64 = _keys(2, 2, 173, d, seed=91, dtype=dtype)
    sp.plan(keys)
    check_plan(sp.get_plan(), K64, d_hi)
    _quantize_and_check(lib, sp, keys, K64, O.split_plan(K64, d_hi))


def _oracle_split_logits(q64, perm, ph, nh, pl, nl, tb_hi, tb_lo, B, Hkv, S, scale):
    """The split estimator computed by the oracle from the packed rows."""
    qz = []
    for pay, nrm, tb in ((ph, nh, tb_hi), (pl, nl, tb_lo)):
        codes, bits = O.unpack_rows(pay, tb.d, tb.m, tb.bmse)
        nr = np.asarray(nrm).view(np.float16).reshape(-1, 2)
        qz.append(O.Quantized(codes=codes, bits=bits, n=None, rho=None, n16=nr[:, 0], rho16=nr[:, 1], u=None, z=None))
    return O.split_gqa_logits(q64, perm, qz[0], qz[1], tb_hi, tb_lo, B, Hkv, S, scale)


@pytest.mark.parametrize("B,Hkv,G,S,bits_hi,bits_lo", [(2, 2, 4, 517, 3, 2), (1, 3, 2, 64, 4, 3),
                                                        (2, 1, 8, 200, 2, 2), (1, 2, 1, 33, 3, 2)])
def test_split_logits_against_oracle(lib, B, Hkv, G, S, bits_hi, bits_lo):
    hi, lo = lib.tq_init(64, bits_hi, 42), lib.tq_init(64, bits_lo, 43)
    sp = lib.tq_split_create(hi, lo, Hkv)
    keys, K64 = _keys(B, Hkv, S, 128, seed=500 + S)
    perm = O.split_plan(K64, 64)
    sp.set_plan(perm)
    ph, nh, pl, nl = lib.tq_split_quantize(sp, keys)
    q = W.queries((B, Hkv * G, 128), seed=9)
    scale = 1.0 / math.sqrt(128)
    out = lib.tq_split_logits(sp, torch.from_numpy(q).to(DEV), ph, nh, pl, nl, scale=scale)
    _status_clean(lib, hi, lo)
    ref, A = _oracle_split_logits(q.astype(np.float64), perm, ph.cpu().numpy(), nh.cpu().numpy(), pl.cpu().numpy(),
                                  nl.cpu().numpy(), tables_of(hi), tables_of(lo), B, Hkv, S, scale)
    check_close(out.cpu().numpy(), ref, A)


def test_split_full_size_sampled(lib):
    """The 2.5-bit split workload (batch 32, 8 KV heads, seq 16384, 64 channels
    at b = 3 and 64 at b = 2): plan over all keys, quantize, logits; the plan
    is compared in full, rows and logits on samples."""
    B, Hkv, G, S, d = 32, 8, 4, 16384, 128
    seed = 1003
    hi, lo = lib.tq_init(64, 3, 42), lib.tq_init(64, 2, 43)
    sp = lib.tq_split_create(hi, lo, Hkv)
    keys = W.decode_keys(B, Hkv, S, d, seed, device=DEV)
    sp.plan(keys)
    perm_gpu = sp.get_plan()
    # the oracle's plan, head by head over the bf16 values
    kcpu = keys.cpu()
    perm = np.empty((Hkv, d), dtype=np.int64)
    for h in range(Hkv):
        Kh = kcpu[:, h:h + 1].to(torch.float64).numpy()
        perm[h] = O.split_plan(Kh, 64)[0]
        check_plan(perm_gpu[h:h + 1], Kh, 64)
    del kcpu
    sp.set_plan(perm)
    ph, nh, pl, nl = lib.tq_split_quantize(sp, keys)
    q = W.queries((B, Hkv * G, d), seed=seed + 7)
    scale = 1.0 / math.sqrt(d)
    out = lib.tq_split_logits(sp, torch.from_numpy(q).to(DEV), ph, nh, pl, nl, scale=scale)
    _status_clean(lib, hi, lo)
    tb_hi, tb_lo = tables_of(hi), tables_of(lo)
    rng = np.random.default_rng(0)
    rep = {}
    for b, h in [(0, 0), (B - 1, Hkv - 1), (B // 2, 3)]:
        s_idx = np.sort(rng.choice(S, 1000, replace=False))
        s_idx[-1] = S - 1
        rows = (b * Hkv + h) * S + s_idx
        k64 = W.decode_keys_rows(b, h, s_idx, S, d, Hkv, seed)
        check_quantize(ph[rows].cpu().numpy(), nh[rows].cpu().numpy(), k64[:, perm[h, :64]], tb_hi, rep)
        check_quantize(pl[rows].cpu().numpy(), nl[rows].cpu().numpy(), k64[:, perm[h, 64:]], tb_lo, rep)
        sel = lambda t: t[rows].cpu().numpy()  # noqa: E731
        ref, A = _oracle_split_logits(q[b:b + 1, h * G:(h + 1) * G].astype(np.float64), perm[h:h + 1],
                                      sel(ph), sel(nh), sel(pl), sel(nl), tb_hi, tb_lo, 1, 1, len(s_idx), scale)
        got = out[b, h * G:(h + 1) * G][:, torch.from_numpy(s_idx).to(DEV)].cpu().numpy()
        check_close(got, ref[0], A[0])


@pytest.mark.parametrize("d_hi,d_lo,bits_hi,bits_lo,G", [(72, 64, 3, 2, 4), (64, 64, 3, 2, 16), (64, 128, 2, 4, 2)])
def test_split_logits_cuda_core_path(lib, d_hi, d_lo, bits_hi, bits_lo, G):
    """Shapes outside the int8-MMA split kernel (groups other than 64 + 64, more
    than 8 query heads per KV head) run on CUDA cores."""
    B, Hkv, S = 2, 2, 150
    hi, lo = lib.tq_init(d_hi, bits_hi, 42), lib.tq_init(d_lo, bits_lo, 43)
    sp = lib.tq_split_create(hi, lo, Hkv)
    keys, K64 = _keys(B, Hkv, S, d_hi + d_lo, seed=321, dtype=torch.float32)
    perm = O.split_plan(K64, d_hi)
    sp.set_plan(perm)
    ph, nh, pl, nl = lib.tq_split_quantize(sp, keys)
    q = W.queries((B, Hkv * G, d_hi + d_lo), seed=10)
    out = lib.tq_split_logits(sp, torch.from_numpy(q).to(DEV), ph, nh, pl, nl, scale=0.5)
    _status_clean(lib, hi, lo)
    ref, A = _oracle_split_logits(q.astype(np.float64), perm, ph.cpu().numpy(), nh.cpu().numpy(), pl.cpu().numpy(),
                                  nl.cpu().numpy(), tables_of(hi), tables_of(lo), B, Hkv, S, 0.5)
    check_close(out.cpu().numpy(), ref, A)


def test_split_argument_errors(lib):
    """Misaligned buffers, a short workspace and mismatched shapes are refused
    with an error status before any launch."""
    import ctypes

    hi, lo = lib.tq_init(64, 3, 42), lib.tq_init(64, 2, 43)
    sp = lib.tq_split_create(hi, lo, 2)
    keys = torch.zeros((1, 2, 16, 128), dtype=torch.bfloat16, device=DEV)
    L = lib.lib()
    ph = torch.empty((32, hi.row_bytes + 16), dtype=torch.uint8, device=DEV)
    nh = torch.empty((32, 2), dtype=torch.float16, device=DEV)
    pl = torch.empty((32, lo.row_bytes), dtype=torch.uint8, device=DEV)
    nl = torch.empty((32, 2), dtype=torch.float16, device=DEV)
    vp = ctypes.c_void_p
    # keys pointer off 16-byte alignment
    st = L.tq_split_quantize(sp.handle, vp(keys.data_ptr() + 2), 1, 1, 16, vp(ph.data_ptr()), vp(nh.data_ptr()),
                             vp(pl.data_ptr()), vp(nl.data_ptr()), None)
    assert st == 1
    # plan workspace too small
    ws = torch.empty(64, dtype=torch.uint8, device=DEV)
    assert L.tq_split_plan(sp.handle, vp(keys.data_ptr()), 1, 1, 16, vp(ws.data_ptr()), 64, None) == 5
    # query heads not a multiple of the KV heads
    q = torch.zeros((1, 3, 128), device=DEV)
    out = torch.empty((1, 3, 16), device=DEV)
    ws2 = torch.empty(1 << 16, dtype=torch.uint8, device=DEV)
    assert L.tq_split_logits(sp.handle, vp(q.data_ptr()), 1, 3, 16, vp(ph.data_ptr()), vp(nh.data_ptr()),
                             vp(pl.data_ptr()), vp(nl.data_ptr()), 1.0, vp(out.data_ptr()), vp(ws2.data_ptr()),
                             ws2.numel(), None) == 1
    # a split of 512 channels (the largest: two 256-channel contexts) is accepted
    sp2 = lib.tq_split_create(lib.tq_init(256, 3, 3), lib.tq_init(256, 2, 4), 1)
    sp2.close()
