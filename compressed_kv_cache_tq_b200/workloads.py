"""Seeded synthetic inputs shaped like the workloads on the TurboQuant pages.

This module holds no part of the method's arithmetic: it only draws keys,
queries and database vectors.  The tests feed the same arrays to the CUDA
library and to the CPU oracle; bench.py uses it for its inputs.

Workloads (sizes from the decode / long-context / split / search settings):
  toy      N = 4096 keys, d = 128, fp32 N(0, 1) with 4 seeded channels x10;
           64 fp32 N(0, 1) queries; b = 3.
  decode   Llama-3.1-8B-shaped decode layer: batch 8, 8 KV heads, 32 query
           heads, head_dim 128, seq 32768; bf16 keys = N(0, 1) x per-(KV head,
           channel) lognormal(0, 1) scale, 2% of channels (3 per head) x20; b = 4.
  longctx  batch 1, 8 KV heads, seq 131072, keys as in decode; b = 3.
  search   unit-normalised mixture of 100 Gaussian clusters in d = 200.
Every draw is a function of (seed, block indices) only, so any block can be
regenerated on its own (the tests rebuild sampled rows on the CPU).
"""

from __future__ import annotations

import numpy as np


def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def toy_keys(n: int = 4096, d: int = 128, seed: int = 1000) -> np.ndarray:
    """fp32 N(0, 1) keys with 4 seeded channels scaled by 10."""
    g = _rng(seed, 0)
    k = g.standard_normal((n, d), dtype=np.float32)
    ch = g.choice(d, size=4, replace=False)
    k[:, ch] *= 10.0
    return k


def queries(shape, seed: int) -> np.ndarray:
    """fp32 N(0, 1) queries of the given shape."""
    return _rng(seed, 1).standard_normal(shape, dtype=np.float32)


def head_channel_scales(Hkv: int, d: int, seed: int, outlier_frac: float = 0.02, outlier_mult: float = 20.0):
    """Per-(KV head, channel) scale: lognormal(0, 1) times 20 on round(2% d) channels per head."""
    g = _rng(seed, 2)
    s = np.exp(g.standard_normal((Hkv, d))).astype(np.float32)
    n_out = int(round(outlier_frac * d))
    for h in range(Hkv):
        s[h, g.choice(d, size=n_out, replace=False)] *= outlier_mult
    return s


def decode_keys_pair(b: int, h: int, S: int, d: int, scales: np.ndarray, seed: int) -> np.ndarray:
    """fp32 keys of one (batch, KV head) pair before rounding to bf16: (S, d)."""
    g = _rng(seed, 3, b, h)
    return g.standard_normal((S, d), dtype=np.float32) * scales[h][None, :]


def decode_keys(B: int, Hkv: int, S: int, d: int, seed: int, device="cpu", rows=None):
    """bf16 keys [B, Hkv, S, d] as a torch tensor (generated pair by pair)."""
    import torch

    scales = head_channel_scales(Hkv, d, seed)
    out = torch.empty((B, Hkv, S, d), dtype=torch.bfloat16, device=device)
    for b in range(B):
        for h in range(Hkv):
            out[b, h] = torch.from_numpy(decode_keys_pair(b, h, S, d, scales, seed)).to(device).to(torch.bfloat16)
    return out


def decode_keys_rows(b: int, h: int, s_idx: np.ndarray, S: int, d: int, Hkv: int, seed: int) -> np.ndarray:
    """The bf16 values (as float64) of selected rows s_idx of pair (b, h)."""
    import torch

    scales = head_channel_scales(Hkv, d, seed)
    k = torch.from_numpy(decode_keys_pair(b, h, S, d, scales, seed)[s_idx]).to(torch.bfloat16)
    return k.to(torch.float64).numpy()


def search_vectors(n: int, d: int = 200, clusters: int = 100, spread: float = 0.3, seed: int = 1004,
                   which: int = 0) -> np.ndarray:
    """Unit-normalised points of a 100-cluster Gaussian mixture (which = 0 database, 1 queries)."""
    centers = _rng(seed, 5).standard_normal((clusters, d))
    g = _rng(seed, 6, which)
    lab = g.integers(0, clusters, n)
    x = centers[lab] + spread * g.standard_normal((n, d))
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    return x.astype(np.float32)
