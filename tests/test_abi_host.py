"""Host-side checks of libtq (no GPU): the library loads, exports every
symbol include/tq.h declares, its host-built tables agree with the oracle's,
and argument validation fails cleanly before any device work."""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import tq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from compressed_kv_cache_tq_b200 import build, tq

    if not os.path.exists(tq.LIB_PATH):
        build.build()
    return tq


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    lib = L.lib()
    names = declared_symbols()
    assert len(names) >= 14
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(L.EXPORTED) == names


@pytest.mark.parametrize("d,bits,m,seed,base", [(128, 3, 128, 42, 0), (128, 4, 128, 7, 0), (64, 2, 64, 5, 2),
                                                (256, 3, 128, 9, 0), (64, 4, 192, 1, 4), (200, 2, 200, 42, 0),
                                                (200, 4, 200, 42, 0)])
def test_host_tables_match_oracle(L, d, bits, m, seed, base):
    R, P, c, t = L.tq_host_tables(d, bits, seed, m=m, stream_base=base)
    tb = O.make_tables(d, bits, seed, m=m, stream_base=base)
    assert np.max(np.abs(R - tb.R)) < 1e-12
    assert np.max(np.abs(P - tb.P)) < 1e-13
    np.testing.assert_allclose(c, tb.c, atol=1e-12, rtol=0)
    np.testing.assert_allclose(t, tb.t, atol=1e-12, rtol=0)


def test_host_tables_reject_unsupported(L):
    lib = L.lib()
    # d, m: multiples of 8 from 64 to 256; bits 2..4
    for d, bits, m in [(100, 3, 100), (128, 5, 128), (128, 1, 128), (512, 3, 512), (128, 3, 36), (56, 3, 56),
                       (264, 3, 264)]:
        assert lib.tq_host_tables(d, bits, m, 1, 0, None, None, None, None) == 2


def test_argument_validation_without_device(L):
    lib = L.lib()
    assert lib.tq_init(128, 3, 1, None) == 1
    assert lib.tq_quantize(None, None, 0, 10, 128, None, None, None) == 1
    assert lib.tq_logits_workspace_bytes(None, 1, 4, 1) == 0
    assert lib.tq_topk_workspace_bytes(None, 1, 4, 1) == 0
    assert lib.tq_logits(None, None, 1, 4, 1, 10, None, None, 1.0, None, None, 0, None) == 1
    assert lib.tq_logits_noalloc(None, None, 1, 4, 1, 10, None, None, 1.0, None, None) == 1
    assert lib.tq_check_device_status(None, None, None) == 1
    assert lib.tq_set_wait_budget(None, 0) == 1
    assert lib.tq_strerror(7) == b"a norm exceeded the fp16 range"
    assert lib.tq_info(None, None, None, None, None) == 1
    assert lib.tq_strerror(5) == b"workspace too small"
    lib.tq_free(None)
    # channel split
    import ctypes
    h = ctypes.c_void_p()
    assert lib.tq_split_create(None, None, 8, ctypes.byref(h)) == 1 and not h.value
    assert lib.tq_split_create(None, None, 8, None) == 1
    assert lib.tq_split_plan_workspace_bytes(None) == 0
    assert lib.tq_split_logits_workspace_bytes(None, 1, 4) == 0
    assert lib.tq_split_plan(None, None, 1, 1, 1, None, 0, None) == 1
    assert lib.tq_split_set_plan(None, None) == 1
    assert lib.tq_split_get_plan(None, None) == 1
    assert lib.tq_split_quantize(None, None, 1, 1, 1, None, None, None, None, None) == 1
    assert lib.tq_split_logits(None, None, 1, 4, 1, None, None, None, None, 1.0, None, None, 0, None) == 1
    lib.tq_split_free(None)
    # value path
    assert lib.tq_attend_workspace_bytes(None, 1, 8, 2, 64) == 0
    assert lib.tq_attend(None, None, 1, 8, 2, 64, None, None, None, None, 0, None) == 1


def test_topk_merge_validation_without_device(L):
    """tq_topk_merge refuses bad counts, pointers and shard offsets on the
    host; nothing is dereferenced on the device before these checks pass
    (the fake device addresses below are never touched)."""
    lib = L.lib()
    dev = ctypes.c_void_p(1 << 20)           # aligned, never dereferenced
    odd = ctypes.c_void_p((1 << 20) + 2)     # misaligned for 4- and 8-byte elements
    first = (ctypes.c_int64 * 64)(*range(0, 6400, 100))
    fp = ctypes.cast(first, ctypes.c_void_p)
    assert lib.tq_topk_merge(dev, dev, fp, 0, 4, 10, dev, dev, None) == 1          # no parts
    assert lib.tq_topk_merge(dev, dev, fp, 65, 4, 10, dev, dev, None) == 1         # more than 64 parts
    assert lib.tq_topk_merge(dev, dev, fp, 2, -1, 10, dev, dev, None) == 1         # negative query count
    assert lib.tq_topk_merge(dev, dev, fp, 2, 4, 0, dev, dev, None) == 1           # k = 0
    assert lib.tq_topk_merge(dev, dev, fp, 64, 4, 65, dev, dev, None) == 2         # 4160 candidates > 4096
    assert lib.tq_topk_merge(None, None, None, 2, 0, 10, None, None, None) == 0    # no queries: nothing to do
    assert lib.tq_topk_merge(None, dev, fp, 2, 4, 10, dev, dev, None) == 1         # null scores
    assert lib.tq_topk_merge(dev, dev, None, 2, 4, 10, dev, dev, None) == 1        # null offsets
    assert lib.tq_topk_merge(odd, dev, fp, 2, 4, 10, dev, dev, None) == 1          # scores misaligned
    assert lib.tq_topk_merge(dev, odd, fp, 2, 4, 10, dev, dev, None) == 1          # ids misaligned
    assert lib.tq_topk_merge(dev, dev, fp, 2, 4, 10, odd, dev, None) == 1          # out ids misaligned
    first[1] = -5
    assert lib.tq_topk_merge(dev, dev, fp, 2, 4, 10, dev, dev, None) == 1          # negative first row


def test_row_bytes_formula():
    for d, m, b in [(128, 128, 3), (128, 128, 2), (64, 64, 1), (256, 256, 3)]:
        assert O.row_bytes(d, m, b) == d * b // 8 + m // 8
    # dimensions that are not multiples of 64 are stored in the next multiple of 64
    for d, m, b in [(200, 200, 1), (200, 200, 3), (72, 136, 2)]:
        dp, mp = -(-d // 64) * 64, -(-m // 64) * 64
        assert O.row_bytes(d, m, b) == dp * b // 8 + mp // 8


def test_binding_refuses_buffers_that_disagree_with_the_sizes(L):
    """The binding checks dtype, shape, contiguity and device of every buffer
    before it hands bare pointers to the C ABI (CPU tensors stand in here)."""
    import types

    import torch

    ctx = types.SimpleNamespace(row_bytes=64, d=128)
    pay = torch.zeros((10, 64), dtype=torch.uint8)
    nrm = torch.zeros((10, 2), dtype=torch.float16)
    L._need_rows(ctx, pay, nrm, 10, pay.device)
    L._need_rows(ctx, pay, nrm, None, None)
    bad = [
        (torch.zeros((9, 64), dtype=torch.uint8), nrm, 10),           # fewer rows than keys
        (torch.zeros((10, 48), dtype=torch.uint8), nrm, 10),          # another layout's row size
        (torch.zeros((10, 64), dtype=torch.int8), nrm, 10),           # wrong dtype
        (torch.zeros((640,), dtype=torch.uint8), nrm, 10),            # flat
        (torch.zeros((64, 10), dtype=torch.uint8).t(), nrm, 10),      # not contiguous
        (pay, torch.zeros((10, 2), dtype=torch.float32), 10),         # norms not fp16
        (pay, torch.zeros((9, 2), dtype=torch.float16), None),        # norms for fewer rows
        (pay, torch.zeros((20,), dtype=torch.float16), None),         # norms flat
    ]
    for p, n_, rows in bad:
        with pytest.raises(ValueError):
            L._need_rows(ctx, p, n_, rows, None)
    with pytest.raises(ValueError):
        L._need_rows(ctx, pay, nrm, 10, torch.device("meta"))         # another device
    with pytest.raises(TypeError):
        L._need_tensor(None, "out", torch.float32, (1,))
    L._need_tensor(torch.zeros((2, 8, 5)), "out", torch.float32, (2, 8, 5))
    with pytest.raises(ValueError):
        L._need_tensor(torch.zeros((2, 8, 4)), "out", torch.float32, (2, 8, 5))
    L._need_workspace(torch.zeros(300, dtype=torch.uint8), None)
    for ws in (torch.zeros(300, dtype=torch.float32), torch.zeros((2, 150), dtype=torch.uint8)):
        with pytest.raises(ValueError):
            L._need_workspace(ws, None)
