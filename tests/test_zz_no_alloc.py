"""tq_logits_noalloc: the logits call for callers that cannot allocate device
memory where they compute logits (an engine that gives its whole device-memory
budget to its own pool, or a decode loop in which a cudaMalloc, which may
synchronise the device, is not acceptable).  Its scratch is a static device
array inside libtq.  The test calls it through the C ABI twice in a row and
checks each result against the oracle's estimates and against tq_logits, the
call that takes a workspace."""

import ctypes
import math

import numpy as np
import pytest
import torch

from compressed_kv_cache_tq_b200 import workloads as W
from tests.parity import REL_FLOOR, check_close, oracle_estimates, tables_of

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_oracle_and_tq_logits_on_two_calls(lib):
    L = lib.lib()
    ctx = lib.tq_init(128, 4, 42)
    stream = torch.cuda.current_stream()
    scale = 1.0 / math.sqrt(128)
    tb = tables_of(ctx)
    for B, Hkv, G, S, seed in [(2, 4, 4, 1000, 1), (1, 3, 8, 777, 2)]:
        Hq = Hkv * G
        scales = W.head_channel_scales(Hkv, 128, seed)
        k = np.stack([np.stack([W.decode_keys_pair(b, h, S, 128, scales, seed) for h in range(Hkv)])
                      for b in range(B)])
        keys = torch.from_numpy(k).to(torch.bfloat16).cuda().reshape(-1, 128)
        payload, norms = lib.tq_quantize(ctx, keys)
        q = torch.from_numpy(W.queries((B, Hq, 128), seed=seed + 10)).cuda()
        ref = lib.tq_logits(ctx, q, payload, norms, Hkv, scale=scale)
        out = torch.full((B, Hq, S), float("nan"), device="cuda")
        st = L.tq_logits_noalloc(ctx.handle, _ptr(q), B, Hq, Hkv, S, _ptr(payload), _ptr(norms), scale, _ptr(out),
                                 ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, L.tq_strerror(st)
        torch.cuda.synchronize()
        assert lib.tq_check_device_status(ctx) == 0
        pl, nr = payload.cpu().numpy(), norms.cpu().numpy()
        o, r = out.cpu().numpy(), ref.cpu().numpy()
        qh = q.cpu().double().numpy()
        for b in range(B):
            for hk in range(Hkv):
                rows = slice((b * Hkv + hk) * S, (b * Hkv + hk + 1) * S)
                s, A = oracle_estimates(pl[rows], nr[rows], qh[b, hk * G:(hk + 1) * G], tb)
                heads = slice(hk * G, (hk + 1) * G)
                check_close(o[b, heads], scale * s, scale * A, rel_floor=REL_FLOOR)
                check_close(o[b, heads], r[b, heads], scale * A)


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    L = lib.lib()
    ctx = lib.tq_init(128, 4, 42)
    B, Hkv, Hq, S = 1024, 1, 4, 16
    need = L.tq_logits_workspace_bytes(ctx.handle, B, Hq, Hkv)
    assert need > (1 << 20)
    q = torch.zeros((B, Hq, 128), device="cuda")
    payload = torch.zeros((B * Hkv * S, ctx.row_bytes), dtype=torch.uint8, device="cuda")
    norms = torch.zeros((B * Hkv * S, 2), dtype=torch.float16, device="cuda")
    out = torch.zeros((B, Hq, S), device="cuda")
    st = L.tq_logits_noalloc(ctx.handle, _ptr(q), B, Hq, Hkv, S, _ptr(payload), _ptr(norms), 1.0, _ptr(out), None)
    assert st == 5   # TQ_ERR_WORKSPACE


def test_noalloc_argument_errors(lib):
    L = lib.lib()
    ctx = lib.tq_init(128, 4, 42)
    B, Hkv, Hq, S = 1, 2, 8, 64
    q = torch.zeros((B, Hq, 128), device="cuda")
    payload = torch.zeros((B * Hkv * S + 1, ctx.row_bytes), dtype=torch.uint8, device="cuda")
    norms = torch.zeros((B * Hkv * S + 1, 2), dtype=torch.float16, device="cuda")
    out = torch.zeros((B, Hq, S), device="cuda")
    h = ctx.handle

    def call(q_=q, B_=B, Hq_=Hq, Hkv_=Hkv, S_=S, p_=None, n_=None, o_=out):
        p_ = _ptr(payload) if p_ is None else p_
        n_ = _ptr(norms) if n_ is None else n_
        return L.tq_logits_noalloc(h, None if q_ is None else _ptr(q_), B_, Hq_, Hkv_, S_, p_, n_, 1.0,
                                   None if o_ is None else _ptr(o_), None)

    assert call() == 0
    assert call(B_=0) == 0 and call(Hq_=0) == 0          # no-ops
    assert call(B_=-1) == 1 and call(S_=-1) == 1
    assert call(Hkv_=0) == 1 and call(Hkv_=3) == 1       # Hq not a multiple of Hkv
    assert call(q_=None) == 1 and call(o_=None) == 1
    assert call(p_=ctypes.c_void_p(payload.data_ptr() + 8)) == 1    # payload not 16-byte aligned
    assert call(n_=ctypes.c_void_p(norms.data_ptr() + 2)) == 1      # norms not 4-byte aligned
    torch.cuda.synchronize()
    assert lib.tq_check_device_status(ctx) == 0
