"""Thin ctypes binding of libtq (include/tq.h): argument marshalling only.

Every step of the path runs in libtq's CUDA kernels.  torch provides device
memory and the current stream.  There is no fallback: if libtq.so is missing
or no CUDA device is present, the calls raise.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_F32, TQ_BF16 = 0, 1

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape or type", 3: "CUDA error",
           4: "out of memory", 5: "workspace too small", 6: "device-side error",
           7: "a norm exceeded the fp16 range"}

# Bits of the context status word (tq_check_device_status).
STATUS_QUANTIZE_WAIT, STATUS_SEARCH_WAIT, STATUS_RANGE = 0x1, 0x2, 0x4


class TQError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, status)} {detail}".strip())


_lib = None


def lib() -> ctypes.CDLL:
    """Load libtq.so (built in-tree by compressed_kv_cache_tq_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m compressed_kv_cache_tq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, u32, u64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint32,
                                           ctypes.c_uint64, ctypes.c_float, ctypes.c_size_t)
        sig = {
            "tq_init": (i32, [i32, i32, u64, ctypes.POINTER(vp)]),
            "tq_init_ex": (i32, [i32, i32, i32, u64, u32, ctypes.POINTER(vp)]),
            "tq_free": (None, [vp]),
            "tq_host_tables": (i32, [i32, i32, i32, u64, u32, vp, vp, vp, vp]),
            "tq_info": (i32, [vp, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32),
                              ctypes.POINTER(i32)]),
            "tq_export_tables": (i32, [vp, vp, vp, vp, vp]),
            "tq_quantize": (i32, [vp, vp, i32, i64, i64, vp, vp, vp]),
            "tq_dequantize": (i32, [vp, vp, vp, i64, i32, vp, vp]),
            "tq_logits_workspace_bytes": (sz, [vp, i32, i32, i32]),
            "tq_logits": (i32, [vp, vp, i32, i32, i32, i64, vp, vp, f32, vp, vp, sz, vp]),
            "tq_logits_noalloc": (i32, [vp, vp, i32, i32, i32, i64, vp, vp, f32, vp, vp]),
            "tq_topk_workspace_bytes": (sz, [vp, i64, i64, i32]),
            "tq_topk": (i32, [vp, vp, i64, vp, vp, i64, i32, vp, vp, vp, sz, vp]),
            "tq_check_device_status": (i32, [vp, vp, ctypes.POINTER(u32)]),
            "tq_set_wait_budget": (i32, [vp, i64]),
            "tq_topk_merge": (i32, [vp, vp, vp, i32, i64, i32, vp, vp, vp]),
            "tq_attend_workspace_bytes": (sz, [vp, i32, i32, i32, i64]),
            "tq_attend": (i32, [vp, vp, i32, i32, i32, i64, vp, vp, vp, vp, sz, vp]),
            "tq_split_create": (i32, [vp, vp, i32, ctypes.POINTER(vp)]),
            "tq_split_free": (None, [vp]),
            "tq_split_plan_workspace_bytes": (sz, [vp]),
            "tq_split_plan": (i32, [vp, vp, i32, i32, i64, vp, sz, vp]),
            "tq_split_set_plan": (i32, [vp, vp]),
            "tq_split_get_plan": (i32, [vp, vp]),
            "tq_split_quantize": (i32, [vp, vp, i32, i32, i64, vp, vp, vp, vp, vp]),
            "tq_split_logits_workspace_bytes": (sz, [vp, i32, i32]),
            "tq_split_logits": (i32, [vp, vp, i32, i32, i64, vp, vp, vp, vp, f32, vp, vp, sz, vp]),
            "tq_strerror": (ctypes.c_char_p, [i32]),
            "tq_last_cuda_error": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


EXPORTED = ["tq_init", "tq_init_ex", "tq_host_tables", "tq_free", "tq_info", "tq_export_tables", "tq_quantize", "tq_dequantize",
            "tq_logits_workspace_bytes", "tq_logits", "tq_logits_noalloc", "tq_topk_workspace_bytes", "tq_topk",
            "tq_check_device_status", "tq_set_wait_budget", "tq_strerror", "tq_last_cuda_error", "tq_topk_merge",
            "tq_attend_workspace_bytes", "tq_attend",
            "tq_split_create", "tq_split_free",
            "tq_split_plan_workspace_bytes", "tq_split_plan", "tq_split_set_plan", "tq_split_get_plan",
            "tq_split_quantize", "tq_split_logits_workspace_bytes", "tq_split_logits"]


def _check(status: int, what: str):
    if status != 0:
        detail = ""
        if status == 3:
            detail = lib().tq_last_cuda_error().decode()
        raise TQError(status, what, detail)


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need_cuda(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _need_tensor(t, name: str, dtype: torch.dtype, shape: tuple, device=None):
    """t must be a contiguous tensor of `dtype` with `shape` (a None entry
    matches any size), on `device` when one is given.  The C ABI receives bare
    pointers and derives every extent from the sizes passed beside them, so a
    buffer that disagrees with them would be read or written out of bounds:
    it is refused here, before any launch."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != len(shape) or any(w is not None and g != w for g, w in zip(t.shape, shape)):
        want = "(" + ", ".join("*" if w is None else str(w) for w in shape) + ")"
        raise ValueError(f"{name} must have shape {want}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def _need_rows(ctx, payload, norms, rows, device, suffix=""):
    """Packed rows of ctx's layout: payload uint8 (rows, row_bytes), norms fp16 (rows, 2)."""
    _need_tensor(payload, "payload" + suffix, torch.uint8, (rows, ctx.row_bytes), device)
    _need_tensor(norms, "norms" + suffix, torch.float16, (payload.shape[0], 2), device)


def _need_workspace(ws, device):
    _need_tensor(ws, "workspace", torch.uint8, (None,), device)


class Context:
    """A quantizer: R, S, codebook for (d, bits, m, seed) on the current device."""

    def __init__(self, d: int, bits: int, seed: int, m: int | None = None, stream_base: int = 0):
        if not torch.cuda.is_available():
            raise RuntimeError("libtq needs a CUDA device")
        torch.cuda.current_device()            # make the device's primary context current
        h = ctypes.c_void_p()
        _check(lib().tq_init_ex(d, bits, d if m is None else m, seed, stream_base, ctypes.byref(h)), "tq_init")
        self._h = h
        self.d, self.bits, self.m, self.row_bytes = self.info()
        self.seed = seed

    @property
    def handle(self):
        return self._h

    def info(self):
        d, b, m, rb = (ctypes.c_int() for _ in range(4))
        _check(lib().tq_info(self._h, ctypes.byref(d), ctypes.byref(b), ctypes.byref(m), ctypes.byref(rb)),
               "tq_info")
        return d.value, b.value, m.value, rb.value

    def export_tables(self):
        import numpy as np

        L = 1 << (self.bits - 1)
        R = np.empty((self.d, self.d))
        P = np.empty((self.m, self.d))
        c = np.empty(L)
        t = np.empty(L - 1)
        _check(lib().tq_export_tables(self._h, R.ctypes.data, P.ctypes.data, c.ctypes.data, t.ctypes.data),
               "tq_export_tables")
        return R, P, c, t

    def close(self):
        if getattr(self, "_h", None):
            lib().tq_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def tq_host_tables(d: int, bits: int, seed: int, m: int | None = None, stream_base: int = 0):
    """fp64 (R, P, c, t) exactly as tq_init builds them; runs on the host only."""
    import numpy as np

    m = d if m is None else m
    L = 1 << (bits - 1)
    R, P, c, t = np.empty((d, d)), np.empty((m, d)), np.empty(L), np.empty(L - 1)
    _check(lib().tq_host_tables(d, bits, m, seed, stream_base, R.ctypes.data, P.ctypes.data, c.ctypes.data,
                                t.ctypes.data), "tq_host_tables")
    return R, P, c, t


def tq_init(d: int, bits: int, seed: int, m: int | None = None, stream_base: int = 0) -> Context:
    return Context(d, bits, seed, m, stream_base)


def tq_quantize(ctx: Context, keys: torch.Tensor, payload: torch.Tensor | None = None,
                norms: torch.Tensor | None = None, stream=None):
    """keys (n, d) fp32/bf16 on the device -> (payload uint8 (n, row_bytes), norms fp16 (n, 2))."""
    _need_cuda(keys, "keys")
    if keys.dim() != 2 or keys.shape[1] != ctx.d:
        raise ValueError("keys must be (n, d)")
    dtype = {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16}.get(keys.dtype)
    if dtype is None:
        raise ValueError("keys must be float32 or bfloat16")
    n = keys.shape[0]
    if payload is None:
        payload = torch.empty((n, ctx.row_bytes), dtype=torch.uint8, device=keys.device)
    if norms is None:
        norms = torch.empty((n, 2), dtype=torch.float16, device=keys.device)
    _need_rows(ctx, payload, norms, n, keys.device)
    _check(lib().tq_quantize(ctx.handle, _ptr(keys), dtype, n, keys.stride(0), _ptr(payload), _ptr(norms),
                             ctypes.c_void_p(_stream(stream))), "tq_quantize")
    return payload, norms


def tq_dequantize(ctx: Context, payload: torch.Tensor, norms: torch.Tensor, full: bool = True,
                  out: torch.Tensor | None = None, stream=None):
    _need_cuda(payload, "payload")
    _need_rows(ctx, payload, norms, None, payload.device)
    n = payload.shape[0]
    if out is None:
        out = torch.empty((n, ctx.d), dtype=torch.float32, device=payload.device)
    _need_tensor(out, "out", torch.float32, (n, ctx.d), payload.device)
    _check(lib().tq_dequantize(ctx.handle, _ptr(payload), _ptr(norms), n, int(full), _ptr(out),
                               ctypes.c_void_p(_stream(stream))), "tq_dequantize")
    return out


def tq_logits_workspace_bytes(ctx: Context, B: int, Hq: int, Hkv: int) -> int:
    return int(lib().tq_logits_workspace_bytes(ctx.handle, B, Hq, Hkv))


def tq_logits(ctx: Context, q: torch.Tensor, payload: torch.Tensor, norms: torch.Tensor, Hkv: int,
              scale: float = 1.0, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
              stream=None):
    """q (B, Hq, d) fp32; payload/norms rows ordered (B, Hkv, S) -> logits (B, Hq, S) fp32."""
    _need_cuda(q, "q")
    _need_cuda(payload, "payload")
    _need_cuda(norms, "norms")
    if q.dtype != torch.float32 or q.dim() != 3 or q.shape[2] != ctx.d:
        raise ValueError("q must be float32 (B, Hq, d)")
    B, Hq, _ = q.shape
    if payload.shape[0] % (B * Hkv):
        raise ValueError("payload rows must be B * Hkv * S")
    S = payload.shape[0] // (B * Hkv)
    _need_rows(ctx, payload, norms, None, q.device)
    if out is None:
        out = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    _need_tensor(out, "out", torch.float32, (B, Hq, S), q.device)
    ws_bytes = tq_logits_workspace_bytes(ctx, B, Hq, Hkv)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=q.device)
    _need_workspace(workspace, q.device)
    _check(lib().tq_logits(ctx.handle, _ptr(q), B, Hq, Hkv, S, _ptr(payload), _ptr(norms), float(scale), _ptr(out),
                           _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream))), "tq_logits")
    return out


def tq_logits_noalloc(ctx: Context, q: torch.Tensor, payload: torch.Tensor, norms: torch.Tensor, Hkv: int,
                      scale: float = 1.0, out: torch.Tensor | None = None, stream=None):
    """tq_logits with the library's static scratch array instead of a workspace."""
    _need_cuda(q, "q")
    _need_cuda(payload, "payload")
    _need_cuda(norms, "norms")
    if q.dtype != torch.float32 or q.dim() != 3 or q.shape[2] != ctx.d:
        raise ValueError("q must be float32 (B, Hq, d)")
    B, Hq, _ = q.shape
    if Hkv < 1 or B * Hkv == 0 or payload.shape[0] % (B * Hkv):
        raise ValueError("payload rows must be B * Hkv * S")
    S = payload.shape[0] // (B * Hkv)
    _need_rows(ctx, payload, norms, None, q.device)
    if out is None:
        out = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    _need_tensor(out, "out", torch.float32, (B, Hq, S), q.device)
    _check(lib().tq_logits_noalloc(ctx.handle, _ptr(q), B, Hq, Hkv, S, _ptr(payload), _ptr(norms), float(scale),
                                   _ptr(out), ctypes.c_void_p(_stream(stream))), "tq_logits_noalloc")
    return out


def tq_attend_workspace_bytes(ctx: Context, B: int, Hq: int, Hkv: int, S: int) -> int:
    return int(lib().tq_attend_workspace_bytes(ctx.handle, B, Hq, Hkv, S))


def tq_attend(ctx: Context, logits: torch.Tensor, payload: torch.Tensor, norms: torch.Tensor, Hkv: int,
              out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """logits (B, Hq, S) fp32 against a value cache (rows (B, Hkv, S)) -> out (B, Hq, d) fp32."""
    _need_cuda(logits, "logits")
    _need_cuda(payload, "payload")
    _need_cuda(norms, "norms")
    if logits.dtype != torch.float32 or logits.dim() != 3:
        raise ValueError("logits must be float32 (B, Hq, S)")
    B, Hq, S = logits.shape
    if payload.shape[0] != B * Hkv * S:
        raise ValueError("payload rows must be B * Hkv * S")
    _need_rows(ctx, payload, norms, B * Hkv * S, logits.device)
    if out is None:
        out = torch.empty((B, Hq, ctx.d), dtype=torch.float32, device=logits.device)
    _need_tensor(out, "out", torch.float32, (B, Hq, ctx.d), logits.device)
    ws_bytes = tq_attend_workspace_bytes(ctx, B, Hq, Hkv, S)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=logits.device)
    _need_workspace(workspace, logits.device)
    _check(lib().tq_attend(ctx.handle, _ptr(logits), B, Hq, Hkv, S, _ptr(payload), _ptr(norms), _ptr(out),
                           _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream))), "tq_attend")
    return out


def tq_topk_workspace_bytes(ctx: Context, nq: int, n: int, k: int) -> int:
    return int(lib().tq_topk_workspace_bytes(ctx.handle, nq, n, k))


def tq_topk(ctx: Context, q: torch.Tensor, payload: torch.Tensor, norms: torch.Tensor, k: int,
            workspace: torch.Tensor | None = None, stream=None):
    """q (nq, d) fp32 -> (ids int64 (nq, k), scores fp32 (nq, k))."""
    _need_cuda(q, "q")
    _need_cuda(payload, "payload")
    _need_cuda(norms, "norms")
    _need_tensor(q, "q", torch.float32, (None, ctx.d), q.device)
    _need_rows(ctx, payload, norms, None, q.device)
    nq, n = q.shape[0], payload.shape[0]
    ids = torch.empty((nq, k), dtype=torch.int64, device=q.device)
    scores = torch.empty((nq, k), dtype=torch.float32, device=q.device)
    ws_bytes = tq_topk_workspace_bytes(ctx, nq, n, k)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=q.device)
    _need_workspace(workspace, q.device)
    _check(lib().tq_topk(ctx.handle, _ptr(q), nq, _ptr(payload), _ptr(norms), n, k, _ptr(ids), _ptr(scores),
                         _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream))), "tq_topk")
    return ids, scores


def tq_topk_merge(scores: torch.Tensor, ids: torch.Tensor, first_rows, k: int, stream=None):
    """scores fp32 / ids int64 [parts, nq, k] (shard-local ids), first_rows: one int per shard
    -> (ids int64 (nq, k) global, scores fp32 (nq, k))."""
    import numpy as np

    _need_cuda(scores, "scores")
    _need_cuda(ids, "ids")
    if scores.dim() != 3 or scores.shape != ids.shape or scores.dtype != torch.float32 or ids.dtype != torch.int64:
        raise ValueError("scores (fp32) and ids (int64) must both be (parts, nq, k)")
    if ids.device != scores.device:
        raise ValueError("scores and ids must be on the same device")
    parts, nq, kk = scores.shape
    fr = np.ascontiguousarray(np.asarray(first_rows, dtype=np.int64))
    if fr.shape != (parts,):
        raise ValueError("first_rows must hold one row offset per part")
    out_ids = torch.empty((nq, k), dtype=torch.int64, device=scores.device)
    out_sc = torch.empty((nq, k), dtype=torch.float32, device=scores.device)
    if kk != k:
        raise ValueError("each part must hold k candidates per query")
    _check(lib().tq_topk_merge(_ptr(scores), _ptr(ids), fr.ctypes.data, parts, nq, k, _ptr(out_ids), _ptr(out_sc),
                               ctypes.c_void_p(_stream(stream))), "tq_topk_merge")
    return out_ids, out_sc


def tq_check_device_status(ctx: Context, stream=None) -> int:
    """The context's status word (0: clean; STATUS_* bits otherwise), cleared by the read."""
    w = ctypes.c_uint32()
    st = lib().tq_check_device_status(ctx.handle, ctypes.c_void_p(_stream(stream)), ctypes.byref(w))
    if st not in (0, 6, 7):
        _check(st, "tq_check_device_status")
    return w.value


class Split:
    """A per-KV-head channel split between two contexts (high group: hi, low group: lo)."""

    def __init__(self, hi: Context, lo: Context, Hkv: int):
        h = ctypes.c_void_p()
        _check(lib().tq_split_create(hi.handle, lo.handle, Hkv, ctypes.byref(h)), "tq_split_create")
        self._h = h
        self.hi, self.lo, self.Hkv, self.d = hi, lo, Hkv, hi.d + lo.d

    @property
    def handle(self):
        return self._h

    def plan(self, keys: torch.Tensor, workspace: torch.Tensor | None = None, stream=None):
        """Choose the channel order from keys (B, Hkv, S, d) on the device."""
        _need_cuda(keys, "keys")
        if keys.dim() != 4 or keys.shape[1] != self.Hkv or keys.shape[3] != self.d:
            raise ValueError("keys must be (B, Hkv, S, d)")
        dtype = {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16}.get(keys.dtype)
        if dtype is None:
            raise ValueError("keys must be float32 or bfloat16")
        ws_bytes = int(lib().tq_split_plan_workspace_bytes(self._h))
        if workspace is None:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=keys.device)
        _need_workspace(workspace, keys.device)
        _check(lib().tq_split_plan(self._h, _ptr(keys), dtype, keys.shape[0], keys.shape[2], _ptr(workspace),
                                   workspace.numel(), ctypes.c_void_p(_stream(stream))), "tq_split_plan")

    def set_plan(self, perm):
        import numpy as np

        p = np.ascontiguousarray(perm, dtype=np.int32)
        if p.shape != (self.Hkv, self.d):
            raise ValueError("perm must be (Hkv, d)")
        _check(lib().tq_split_set_plan(self._h, p.ctypes.data), "tq_split_set_plan")

    def get_plan(self):
        import numpy as np

        p = np.empty((self.Hkv, self.d), dtype=np.int32)
        _check(lib().tq_split_get_plan(self._h, p.ctypes.data), "tq_split_get_plan")
        return p

    def close(self):
        if getattr(self, "_h", None):
            lib().tq_split_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def tq_split_create(hi: Context, lo: Context, Hkv: int) -> Split:
    return Split(hi, lo, Hkv)


def tq_split_quantize(sp: Split, keys: torch.Tensor, payload_hi=None, norms_hi=None, payload_lo=None, norms_lo=None,
                      stream=None):
    """keys (B, Hkv, S, d) -> (payload_hi, norms_hi, payload_lo, norms_lo), rows (B, Hkv, S)."""
    _need_cuda(keys, "keys")
    if keys.dim() != 4 or keys.shape[1] != sp.Hkv or keys.shape[3] != sp.d:
        raise ValueError("keys must be (B, Hkv, S, d)")
    dtype = {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16}.get(keys.dtype)
    if dtype is None:
        raise ValueError("keys must be float32 or bfloat16")
    B, _, S, _ = keys.shape
    n = B * sp.Hkv * S
    dev = keys.device
    if payload_hi is None:
        payload_hi = torch.empty((n, sp.hi.row_bytes), dtype=torch.uint8, device=dev)
    if norms_hi is None:
        norms_hi = torch.empty((n, 2), dtype=torch.float16, device=dev)
    if payload_lo is None:
        payload_lo = torch.empty((n, sp.lo.row_bytes), dtype=torch.uint8, device=dev)
    if norms_lo is None:
        norms_lo = torch.empty((n, 2), dtype=torch.float16, device=dev)
    _need_rows(sp.hi, payload_hi, norms_hi, n, dev, "_hi")
    _need_rows(sp.lo, payload_lo, norms_lo, n, dev, "_lo")
    _check(lib().tq_split_quantize(sp.handle, _ptr(keys), dtype, B, S, _ptr(payload_hi), _ptr(norms_hi),
                                   _ptr(payload_lo), _ptr(norms_lo), ctypes.c_void_p(_stream(stream))),
           "tq_split_quantize")
    return payload_hi, norms_hi, payload_lo, norms_lo


def tq_split_logits(sp: Split, q: torch.Tensor, payload_hi, norms_hi, payload_lo, norms_lo, scale: float = 1.0,
                    out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """q (B, Hq, d) fp32 against a split cache -> logits (B, Hq, S) fp32."""
    _need_cuda(q, "q")
    for t, nm in ((payload_hi, "payload_hi"), (norms_hi, "norms_hi"), (payload_lo, "payload_lo"),
                  (norms_lo, "norms_lo")):
        _need_cuda(t, nm)
    if q.dtype != torch.float32 or q.dim() != 3 or q.shape[2] != sp.d:
        raise ValueError("q must be float32 (B, Hq, d)")
    B, Hq, _ = q.shape
    if payload_hi.shape[0] % (B * sp.Hkv) or payload_lo.shape[0] != payload_hi.shape[0]:
        raise ValueError("payload rows must be B * Hkv * S")
    S = payload_hi.shape[0] // (B * sp.Hkv)
    _need_rows(sp.hi, payload_hi, norms_hi, None, q.device, "_hi")
    _need_rows(sp.lo, payload_lo, norms_lo, payload_hi.shape[0], q.device, "_lo")
    if out is None:
        out = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    _need_tensor(out, "out", torch.float32, (B, Hq, S), q.device)
    ws_bytes = int(lib().tq_split_logits_workspace_bytes(sp.handle, B, Hq))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=q.device)
    _need_workspace(workspace, q.device)
    _check(lib().tq_split_logits(sp.handle, _ptr(q), B, Hq, S, _ptr(payload_hi), _ptr(norms_hi), _ptr(payload_lo),
                                 _ptr(norms_lo), float(scale), _ptr(out), _ptr(workspace), workspace.numel(),
                                 ctypes.c_void_p(_stream(stream))), "tq_split_logits")
    return out
