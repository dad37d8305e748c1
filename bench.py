"""Benchmark of the TurboQuant hot path on B200 (one JSON line on rank 0).

Workload (the decode configuration the headline metric is quoted on):
  Llama-3.1-8B-shaped decode layer: batch 8, 8 KV heads, 32 query heads
  (GQA 4), head_dim 128, seq 32768; bf16 keys N(0,1) x per-(KV head, channel)
  lognormal(0,1) scales with 2% of channels x20; b = 4 (3 Lloyd-Max bits + 1
  QJL bit, m = 128); one fp32 query token per sequence.

A step is one pass of the whole path over one batch: quantize all
8 x 8 x 32768 keys into a packed cache (tq_quantize) and score the 32 query
heads against a packed cache (tq_logits: query preparation + logits).  The
logits of step i read the cache written in step i-1, so neither kernel reads
data it wrote itself in the same step; the keys (537 MB) and the packed cache
(143 MB) are larger than L2, and 680 MB of other traffic separate a cache's
write from its read.  Per-GPU work is fixed (weak scaling): with --gpus N each
rank runs the full workload; there is no data-path collective.

--impl reference runs the CPU oracle (test infrastructure) on a bounded sample
of the same workload on the host cores, on rank 0 only.

--workload longctx runs the same step on the long-context configuration: one
sequence of 131072 keys for each of 8 KV heads (keys drawn as above), b = 3
(2 Lloyd-Max bits + 1 QJL bit), 32 query heads.

--workload split runs the 2.5-bit channel split: 32 x 8 x 16384 keys, per KV
head the 64 channels of largest variance at b = 3 and the other 64 at b = 2
(each group its own d = 64 quantizer); a step is tq_split_quantize plus
tq_split_logits (the channel plan is computed once, before the steps).

--workload attend adds a quantised value cache to the decode layer: a step
quantizes keys and values, computes the logits and the attention output
(tq_attend).

--workload mse runs the decode layer with the MSE-only variant (m = 0: no
sign sketch).

--workload search times the vector-search configuration instead (one JSON
line): 1 000 000 unit vectors of a 100-cluster Gaussian mixture, d = 200 fp32,
10 000 queries drawn the same way, b = 2 and b = 4, top-10 by the estimator
(tq_topk); a step is the index build (tq_quantize of every row) plus the
search of every query; recall@1@10 against the exact fp32 inner products.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "tq_logits keys scored/s & HBM GB/s (% of 8 TB/s); tq_quantize vectors/s"

B, HKV, HQ, D, S, BITS = 8, 8, 32, 128, 32768, 4
SEED_KEYS, SEED_TABLES = 1001, 42
WORKLOAD = "decode_llama31_8b_layer_b8_hkv8_hq32_d128_s32768_b4"

# The key-cache workloads a step can run: (B, Hkv, Hq, d, S, bits, key seed, name).
# decode: the Llama-3.1-8B-shaped decode layer above.  longctx: one sequence of
# 131072 keys per KV head, keys drawn as in decode, b = 3 (2 Lloyd-Max bits +
# 1 QJL bit): quantize every key on append, then the 32 query heads' logits.
KV_WORKLOADS = {
    "decode": (8, 8, 32, 128, 32768, 4, 1001, "decode_llama31_8b_layer_b8_hkv8_hq32_d128_s32768_b4"),
    "longctx": (1, 8, 32, 128, 131072, 3, 1002, "longctx_prefill_decode_b1_hkv8_hq32_d128_s131072_b3"),
    # 2.5 bits per channel: per KV head the 64 channels of largest variance at
    # b = 3, the other 64 at b = 2, each group its own d = m = 64 quantizer
    "split": (32, 8, 32, 128, 16384, (3, 2), 1003, "split25_b32_hkv8_hq32_d128_s16384_b3x64_b2x64"),
    # the decode layer with a quantised value cache as well (values b = 4,
    # tables of their own): quantize keys and values, logits, attention output
    "attend": (8, 8, 32, 128, 32768, 4, 1001, "decode_attention_llama31_8b_layer_b8_hkv8_hq32_d128_s32768_b4"),
    # the MSE-only variant (stage 1 alone, no sign sketch) on the decode layer:
    # b = 4 gives 3 Lloyd-Max bits per coordinate, 48-byte rows
    "mse": (8, 8, 32, 128, 32768, 4, 1001, "decode_mse_only_llama31_8b_layer_b8_hkv8_hq32_d128_s32768_b4_m0"),
    # the toy configuration: 4096 fp32 keys (N(0,1), 4 seeded channels x10),
    # 64 fp32 queries scoring all 64 x 4096 pairs (one GQA group of 64), b = 3;
    # one batch is launch-latency bound (about 2 MB), so the batch of the step
    # replicates it 256 times (B = 256 copies of the same keys and queries)
    "toy": (256, 1, 64, 128, 4096, 3, 1000, "toy_n4096_d128_fp32_b3_q64_all_pairs_x256_replicas"),
}
SEED_VALUES = 2002
ATTEND = False
JL_ROWS = None   # m of the key quantizer (None: m = d; 0: the MSE-only variant)
KEY_DTYPE = "bf16"   # storage type of the keys fed to the quantizer
TOY = False
KV_NAME = "decode"


def set_workload(name: str, seq: int | None = None, batch: int | None = None):
    """Point the module's shape globals at one of KV_WORKLOADS (seq overrides S,
    batch overrides B)."""
    global B, HKV, HQ, D, S, BITS, SEED_KEYS, WORKLOAD, ATTEND, JL_ROWS, KEY_DTYPE, TOY, KV_NAME
    B, HKV, HQ, D, S, BITS, SEED_KEYS, WORKLOAD = KV_WORKLOADS[name]
    KV_NAME = name
    ATTEND = name == "attend"
    JL_ROWS = 0 if name == "mse" else None
    TOY = name == "toy"
    KEY_DTYPE = "fp32" if TOY else "bf16"
    if seq is not None and seq != S:
        WORKLOAD = WORKLOAD.replace(f"_s{S}_", f"_s{seq}_")
        S = seq
    if batch is not None and batch != B:
        WORKLOAD = (WORKLOAD.replace(f"_x{B}_replicas", f"_x{batch}_replicas") if TOY
                    else WORKLOAD.replace(f"_b{B}_", f"_b{batch}_"))
        B = batch


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return j["hbm_gbs"], j["bf16_tflops"], j.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """SM clocks and throttle reasons sampled while the timed region runs.

    NVML is polled every 2 ms from a thread (so that even a timed region of a
    few milliseconds gets samples); without NVML, nvidia-smi is sampled every
    20 ms instead."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.samples = []        # (sm_mhz, max_mhz, reasons) from NVML
        self.stop = False
        self.nvml = None

    def _nvml_open(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
        h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
        return pynvml, h, bits

    def _poll(self):
        pynvml, h, bits = self.nvml
        mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop:
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), [n for n, b in bits.items() if r & b]))
            except Exception:
                break
            time.sleep(0.002)

    def __enter__(self):
        try:
            self.nvml = self._nvml_open()
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 2.0 and self.t.is_alive():
                time.sleep(0.001)
            if self.samples:
                self.first = len(self.samples)
                return self
        except Exception:
            self.nvml = None
        self.stop = True
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # nvidia-smi takes a moment to start: wait for its first sample, so
            # that the samples from here on fall inside the timed region
            t0 = time.time()
            while not self.lines and time.time() - t0 < 5.0 and self.proc.poll() is None:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        self.first = len(self.lines)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.nvml is not None and not self.stop:
            t0 = time.time()
            while len(self.samples) <= self.first and time.time() - t0 < 0.1:
                time.sleep(0.001)
            self.stop = True
            self.t.join(timeout=1.0)
            return
        # a short timed region may end before the next sample: wait for one
        t0 = time.time()
        while self.proc and len(self.lines) <= self.first and time.time() - t0 < 0.5:
            time.sleep(0.005)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        if self.nvml is not None:
            for v, m, r in (self.samples[self.first:] or self.samples):
                sm.append(v)
                mx = m
                reasons.update(r)
            src = "nvml, 2 ms"
        else:
            for ln in (self.lines[self.first:] or self.lines):
                f = [x.strip() for x in ln.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm.append(float(f[1]))
                    mx = float(f[2])
                except ValueError:
                    continue
                for nm, v in zip(self.NAMES, f[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
            src = "nvidia-smi, 20 ms"
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "source": src}


def bytes_per_key():
    """Algorithmic bytes per key: bf16 key in; packed row(s) and fp16 norm pairs out;
    the logits read those and write one fp32 logit per query head of the group."""
    if isinstance(BITS, tuple):   # split: two groups of D / 2 channels
        g = D // 2
        row = sum(g * (b - 1) // 8 + g // 8 + 4 for b in BITS)
    else:
        m = D if JL_ROWS is None else JL_ROWS
        row = D * (BITS - 1) // 8 + m // 8 + 4
    kin = (4 if KEY_DTYPE == "fp32" else 2) * D
    bpk = {"quantize_in": kin, "quantize_out": row, "logits_in": row, "logits_out": 4 * (HQ // HKV)}
    if ATTEND:
        # keys and values are both quantised; the attention reads the value
        # rows and the logits of the group's query heads
        bpk.update(quantize_in=4 * D, quantize_out=2 * row, attend_in=row + 4 * (HQ // HKV))
    return bpk


def quantize_flops_per_key():
    """Rotation and JL products: 2 d^2 + 2 m d per quantizer (per group for the split)."""
    if isinstance(BITS, tuple):
        g = D // 2
        return 2 * (2 * g * g + 2 * g * g)
    m = D if JL_ROWS is None else JL_ROWS
    return 2 * D * D + 2 * m * D


def kv_config(world: int) -> dict:
    """The `config` of a key-cache workload's JSON line (both arms)."""
    n = B * HKV * S
    bpk = bytes_per_key()
    return {"workload": WORKLOAD, "global_batch": B * world, "seq_len": S, "kv_heads": HKV,
            "q_heads": HQ, "head_dim": D,
            "bits": ({"high_64_channels": BITS[0], "low_64_channels": BITS[1]} if isinstance(BITS, tuple)
                     else BITS),
            "jl_rows": D if JL_ROWS is None else JL_ROWS, "key_dtype": KEY_DTYPE,
            "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2: keys {n * bpk['quantize_in'] / 1e6:.0f} MB, packed caches "
                  f"{n * (bpk['quantize_out']) / 1e6:.0f} MB each; logits read the cache written one step "
                  "earlier, with the keys' traffic in between"}


def search_config(n: int, nq: int, d: int, k: int, world: int) -> dict:
    """The `config` of the vector-search JSON line (both arms)."""
    return {"workload": f"vector_search_{n}_d200_nq{nq}_top10", "rows": n, "queries": nq, "d": d, "m": d,
            "k": k, "bits": [2, 4], "parallelism": f"rows sharded x{world}",
            "l2": f"the fp16 row matrix ({n * 896 / 1e6:.0f} MB) "
                  + ("exceeds L2" if n * 896 > 126e6 else "fits in L2 (profiling size)")}


SEARCH_METRIC = "tq_topk queries/s (10^6 rows, d=200, top-10) and recall@1@10; index build ms"


def search_cpu_index(db, bits: int = 4):
    """The oracle's index of db (fp64 numpy rows): (tables, quantised rows, seconds)."""
    from oracle import tq_oracle as O

    tb = O.make_tables(db.shape[1], bits, SEED_TABLES, m=db.shape[1])
    t0 = time.perf_counter()
    qz = O.quantize(db, tb)
    return tb, qz, time.perf_counter() - t0


def search_cpu_score(tb, qz, rows: slice, qs, k: int) -> float:
    """Seconds the oracle takes for the top-k of queries qs over rows `rows` of an index."""
    from oracle import tq_oracle as O

    t0 = time.perf_counter()
    O.topk(qs, qz.codes[rows], qz.bits[rows], qz.n16[rows], qz.rho16[rows], tb, k)
    return time.perf_counter() - t0


def _threads() -> int:
    from threadpoolctl import threadpool_info

    return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])


def search_cpu_baseline(db, qs, n: int, k: int, bits: int = 4) -> dict:
    """The oracle, as it stands, on a bounded sample of the search workload:
    db (the first rows of the database, fp64 numpy) indexed, then the queries
    qs scored against them; queries/s scaled to n rows (the index build is
    reported, not counted, as on the GPU)."""
    tb, qz, t_index = search_cpu_index(db, bits)
    t_score = search_cpu_score(tb, qz, slice(None), qs, k)
    return {"value": qs.shape[0] / (t_score * n / db.shape[0]), "unit": "queries/s", "cores": _threads(),
            "kind": "oracle",
            "sample": f"b={bits}: {db.shape[0]} rows indexed in {t_index:.1f} s, {qs.shape[0]} queries scored "
                      f"against them in {t_score:.1f} s, scaled to {n} rows; fp64 numpy"}


def host_queries():
    """The step's queries [B, Hq, d] (fp32 numpy): N(0, 1); the toy batch
    repeats its 64 queries in every replica."""
    from compressed_kv_cache_tq_b200 import workloads as W

    if TOY:
        import numpy as np

        return np.repeat(W.queries((1, HQ, D), seed=SEED_KEYS + 1), B, axis=0)
    return W.queries((B, HQ, D), seed=SEED_KEYS + 7)


def device_keys(dev):
    """The step's keys [B, Hkv, S, d] on the device (bf16, or fp32 for the toy batch)."""
    import torch

    from compressed_kv_cache_tq_b200 import workloads as W

    if TOY:
        k = torch.from_numpy(W.toy_keys(S, D, SEED_KEYS)).to(dev)
        return k.expand(B, HKV, S, D).contiguous()
    return W.decode_keys(B, HKV, S, D, SEED_KEYS, device=dev)


def cpu_baseline(budget_s: float = 12.0, max_keys: int = 1 << 19, chunk: int = 8192):
    """The oracle, as it stands, on a bounded sample of the workload (host cores).

    Timed: quantisation of the sampled keys and the estimates of their group's
    query heads.  For the split, the channel plan of each sampled pair is
    taken from the sample itself, outside the timed part (it is a one-time
    calibration, not part of a step)."""
    import numpy as np
    import torch
    from threadpoolctl import threadpool_info

    from compressed_kv_cache_tq_b200 import workloads as W
    from oracle import tq_oracle as O

    split = isinstance(BITS, tuple)
    if split:
        tb_hi = O.make_tables(D // 2, BITS[0], SEED_TABLES)
        tb_lo = O.make_tables(D // 2, BITS[1], SEED_TABLES + 1)
    else:
        tb = O.make_tables(D, BITS, SEED_TABLES, m=JL_ROWS)
    scales = None if TOY else W.head_channel_scales(HKV, D, SEED_KEYS)
    if ATTEND:
        tbv = O.make_tables(D, BITS, SEED_TABLES + 100)
        vscales = W.head_channel_scales(HKV, D, SEED_VALUES)
    q = host_queries()
    G = HQ // HKV
    chunk = min(chunk, S)
    done, busy = 0, 0.0
    for b in range(B):
        for h in range(HKV):
            if TOY:   # every replica holds the same fp32 keys
                kb = W.toy_keys(S, D, SEED_KEYS).astype(np.float64)
            else:
                keys = W.decode_keys_pair(b, h, S, D, scales, SEED_KEYS)
                kb = torch.from_numpy(keys).to(torch.bfloat16).to(torch.float64).numpy()
            if ATTEND:
                vb = torch.from_numpy(W.decode_keys_pair(b, h, S, D, vscales, SEED_VALUES)).to(
                    torch.bfloat16).to(torch.float64).numpy()
            qh = q[b, h * G:(h + 1) * G].astype(np.float64)
            for s0 in range(0, S, chunk):
                kc = kb[s0:s0 + chunk]
                if ATTEND:
                    # keys and values of the chunk, logits, attention over the chunk
                    t0 = time.perf_counter()
                    qz = O.quantize(kc, tb)
                    lg, _ = O.estimate(qh, qz.codes, qz.bits, qz.n16, qz.rho16, tb)
                    vz = O.quantize(vb[s0:s0 + chunk], tbv)
                    O.attention_output(lg[None] / math.sqrt(D), vz.codes, vz.bits, vz.n16, vz.rho16, tbv, 1)
                elif split:
                    perm = O.split_plan(kc[None, None], D // 2)
                    t0 = time.perf_counter()
                    a, c = O.split_quantize(kc[None, None], perm, tb_hi, tb_lo)
                    O.split_gqa_logits(qh[None], perm, a, c, tb_hi, tb_lo, 1, 1, len(kc))
                else:
                    t0 = time.perf_counter()
                    qz = O.quantize(kc, tb)
                    O.estimate(qh, qz.codes, qz.bits, qz.n16, qz.rho16, tb)
                busy += time.perf_counter() - t0
                done += len(kc)
                if busy > budget_s or done >= max_keys:
                    break
            if busy > budget_s or done >= max_keys:
                break
        if busy > budget_s or done >= max_keys:
            break
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": done / busy, "unit": "keys/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} of {B * HKV * S} keys (quantize + {G}-head estimates"
                      f"{'; values quantised and attended over each 8192-key chunk' if ATTEND else ''}), "
                      f"{busy:.1f} s, fp64 numpy"}


def measure_search(n: int, nq: int, steps: int, warmup: int, local: int = 0, dist=None, rank: int = 0,
                   world: int = 1, bits_list=(2, 4)) -> dict:
    """Vector-search workload: index build + top-10 of nq queries over n rows
    (d = 200), per bit rate.  With a process group the database is split by
    rows over the ranks: each rank indexes and searches its block, and the
    per-rank top-10 lists are all-gathered and merged on the device
    (compressed_kv_cache_tq_b200.sharded).  Times are the slowest rank's."""
    import torch

    from compressed_kv_cache_tq_b200 import sharded, tq, workloads as W

    d, k = 200, 10
    dev = torch.device("cuda", local)
    first, count = sharded.shard_rows(n, world, rank)
    firsts = [sharded.shard_rows(n, world, r)[0] for r in range(world)]
    db = torch.from_numpy(W.search_vectors(n, d, seed=1004, which=0)).to(dev)
    shard = db[first:first + count]
    qs = torch.from_numpy(W.search_vectors(nq, d, seed=1004, which=1)).to(dev)
    # exact top-1 of every query by the plain inner product (fp32, on the device)
    top1 = torch.empty(nq, dtype=torch.int64, device=dev)
    for q0 in range(0, nq, 500):
        top1[q0:q0 + 500] = (qs[q0:q0 + 500] @ db.T).argmax(1)
    stream = torch.cuda.current_stream()
    per_bits = {}
    hbm, tf, tf_sus, src = peaks()

    def search(ctx, qv, payload, norms, ws):
        ids, scores = tq.tq_topk(ctx, qv, payload, norms, k, workspace=ws)
        if world > 1:
            ids, scores = sharded.gather_topk(ids, scores, firsts, k)
        return ids, scores

    with ClockSampler(local) as clocks:
        for bits in bits_list:
            ctx = tq.tq_init(d, bits, SEED_TABLES)
            payload = torch.empty((count, ctx.row_bytes), dtype=torch.uint8, device=dev)
            norms = torch.empty((count, 2), dtype=torch.float16, device=dev)
            ws = torch.empty(tq.tq_topk_workspace_bytes(ctx, nq, count, k), dtype=torch.uint8, device=dev)
            ids = scores = None
            for _ in range(warmup):
                tq.tq_quantize(ctx, shard, payload, norms)
                ids, scores = search(ctx, qs, payload, norms, ws)
            torch.cuda.synchronize()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            t_build, t_search = [], []
            for _ in range(steps):
                if dist is not None:
                    dist.barrier()
                ev[0].record(stream)
                tq.tq_quantize(ctx, shard, payload, norms)
                ev[1].record(stream)
                ids, scores = search(ctx, qs, payload, norms, ws)
                ev[2].record(stream)
                torch.cuda.synchronize()
                t_build.append(ev[0].elapsed_time(ev[1]))
                t_search.append(ev[1].elapsed_time(ev[2]))
            assert tq.tq_check_device_status(ctx) == 0, "a kernel reported a device-side error"
            recall = float((ids == top1[:, None]).any(1).float().mean())
            # end to end through the public API: queries from pinned host memory, ids and scores back
            hq = qs.cpu().pin_memory()
            hid = torch.empty((nq, k), dtype=torch.int64, pin_memory=True)
            hsc = torch.empty((nq, k), dtype=torch.float32, pin_memory=True)
            dq = torch.empty_like(qs)
            if dist is not None:
                dist.barrier()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            dq.copy_(hq, non_blocking=True)
            i2, s2 = search(ctx, dq, payload, norms, ws)
            hid.copy_(i2, non_blocking=True)
            hsc.copy_(s2, non_blocking=True)
            b_.record(stream)
            torch.cuda.synchronize()
            ms_b = max_over_ranks(sorted(t_build)[len(t_build) // 2], dist, dev)
            ms_s = max_over_ranks(sorted(t_search)[len(t_search) // 2], dist, dev)
            e2e = max_over_ranks(a.elapsed_time(b_), dist, dev)
            flops = 2.0 * (d + d) * count * nq   # this rank's share of the contraction
            # index build: fp32 rows in, packed rows + norms out
            b_bytes = count * (4 * d + ctx.row_bytes + 4)
            per_bits[f"b{bits}"] = {
                "index_build_ms": ms_b, "search_ms": ms_s,
                "queries_per_s": nq / ms_s * 1e3, "recall_at_1_at_10": recall,
                "search_TFLOP_s_per_gpu": flops / ms_s / 1e9, "search_frac_of_measured_tensor": flops / ms_s / 1e9 / tf,
                "index_build_GB_s": b_bytes / ms_b / 1e6, "index_build_frac_of_measured_hbm": b_bytes / ms_b / 1e6 / hbm,
                "e2e_ms": e2e}
            del ws
    return {"per_bits": per_bits, "clocks": clocks.summary(), "db": db, "qs": qs, "n": n, "nq": nq, "d": d, "k": k}


def run_search(args):
    """The vector-search JSON line (--workload search)."""
    import torch

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    res = measure_search(args.rows, args.queries, args.steps, args.warmup, local, dist, rank, world)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    n, nq, d, k = res["n"], res["nq"], res["d"], res["k"]
    hbm, tf, tf_sus, src = peaks()
    # the oracle on a bounded sample: up to 200 000 rows indexed, 128 queries scored against them
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        n_cpu = min(n, 200_000)
        cpu = search_cpu_baseline(res["db"][:n_cpu].double().cpu().numpy(), res["qs"][:128].double().cpu().numpy(),
                                  n, k)
    b4 = res["per_bits"]["b4"]
    line = {
        "metric": SEARCH_METRIC,
        "value": b4["queries_per_s"], "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": b4["index_build_ms"] + b4["search_ms"],
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": search_config(n, nq, d, k, world),
        "per_bits": res["per_bits"],
        "roofline": {"bound": "tensor", "kernel": "tq_topk (decode + scoring + re-scoring), per GPU",
                     "achieved": b4["search_TFLOP_s_per_gpu"], "peak": tf, "unit": "TFLOP/s",
                     "frac": b4["search_TFLOP_s_per_gpu"] / tf,
                     "peak_source": src + " (bf16 GEMM; fp16 has the same rate)", "traffic": None},
        "e2e": {"value": nq / b4["e2e_ms"] * 1e3, "unit": "queries/s", "h2d_bytes_per_step": nq * d * 4,
                "d2h_bytes_per_step": nq * k * 12},
        "gpu_launches": 4 + (1 if world > 1 else 0),
        "clocks": res["clocks"],
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)
    return 0


def run_reference_search(args):
    """The search workload's reference arm: the oracle indexes a bounded
    sample of the database once (setup), then each step scores a batch of
    queries against it; queries/s scaled to the full database."""
    import numpy as np

    from compressed_kv_cache_tq_b200 import workloads as W

    n, nq, d, k = args.rows, args.queries, 200, 10
    n_cpu = min(n, 200_000)
    db = W.search_vectors(n, d, seed=1004, which=0)[:n_cpu].astype(np.float64)
    qs = W.search_vectors(nq, d, seed=1004, which=1).astype(np.float64)
    tb, qz, t_index = search_cpu_index(db)      # setup, as the index build is on the GPU
    # each step: a batch of queries against a rotating slice of the index
    per_step, rows_step = 32, min(n_cpu, 20_000)
    nslices = max(1, n_cpu // rows_step)

    def step(i):
        r0 = (i % nslices) * rows_step
        sel = np.arange(i * per_step, (i + 1) * per_step) % nq
        return search_cpu_score(tb, qz, slice(r0, r0 + rows_step), qs[sel], k)

    for i in range(args.warmup):
        step(i)
    busy = 0.0
    t0 = time.perf_counter()
    for i in range(args.steps):
        busy += step(i)
    dt = time.perf_counter() - t0
    v = per_step * args.steps / (busy * n / rows_step)
    sample = (f"b=4: {n_cpu} rows indexed once in {t_index:.1f} s (setup); each step scores {per_step} queries "
              f"against a {rows_step}-row slice of the index, scaled to {n} rows; fp64 numpy")
    line = {"impl": "reference", "metric": SEARCH_METRIC, "value": v, "unit": "queries/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": search_config(n, nq, d, k, args.gpus),
            "cpu_baseline": {"value": v, "unit": "queries/s", "cores": _threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args, rank):
    if rank != 0:
        return 0
    if args.workload == "search":
        return run_reference_search(args)
    # each step a bounded sample, sized so that all steps take about a minute
    budget = min(2.0, max(0.005, 60.0 / max(1, args.steps + args.warmup)))
    chunk = 8192 if budget >= 0.5 else (2048 if budget >= 0.05 else 256)
    for _ in range(args.warmup):
        cpu_baseline(budget_s=min(budget, 3.0), max_keys=chunk, chunk=chunk)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(cpu_baseline(budget_s=budget, max_keys=max(chunk, 1 << 16 if budget >= 0.5 else chunk),
                                 chunk=chunk))
    dt = time.perf_counter() - t0
    v = sum(x["value"] for x in vals) / len(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "keys/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": kv_config(args.gpus),
            "cpu_baseline": {"value": v, "unit": "keys/s", "cores": vals[0]["cores"], "kind": "oracle",
                             "sample": vals[-1]["sample"]},
            "e2e": {"value": v, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per key of the
# current kernels, from one ncu capture at S = 16384 (1 048 576 keys); per
# launch it scales with the keys processed.  Summary with the command:
# profiles/traffic_decode_s16384.md.  Set to None when a kernel changes.
DRAM_BYTES_PER_KEY = {"decode": {"tq_quantize": (268.719872e6 + 47.794176e6) / 1048576,
                                  "tq_logits": (71.457536e6 + 0.553472e6) / 1048576}}


def dense_logits_context(keys4, q, reps: int = 20) -> dict:
    """Context for the pages' comparison of 4-bit logits with 32-bit ones: the
    same logits as a dense torch matmul (cuBLAS) of the queries with the
    unquantised keys, in fp32 and bf16, timed with CUDA events like the
    kernels.  Not part of the path; any failure only drops the field."""
    import torch

    res = {"what": "torch.matmul(q, K^T) over unquantised keys [B, Hkv, S, d] per GQA group (cuBLAS), "
                   "keys larger than L2"}
    try:
        Bk, Hk, Sk, Dk = keys4.shape
        G = q.shape[1] // Hk
        for name, dt in (("fp32", torch.float32), ("bf16", torch.bfloat16)):
            K = keys4.to(dt)
            qq = q.to(dt).reshape(Bk, Hk, G, Dk)
            for _ in range(3):
                torch.matmul(qq, K.transpose(-1, -2))
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(reps):
                torch.matmul(qq, K.transpose(-1, -2))
            b.record()
            torch.cuda.synchronize()
            res[f"{name}_ms"] = a.elapsed_time(b) / reps
            del K, qq
    except Exception as e:   # context only
        res["error"] = type(e).__name__
    return res


def max_over_ranks(x: float, dist, device) -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return float(x)
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def result_line(*, world, n, steps, warmup, ms, q_ms, l_ms, e2e_ms, h2d, d2h, clocks, a_ms=None) -> dict:
    """The JSON result: whole-job rates over all ranks (each rank processes n keys
    per step; ms and e2e_ms are the slowest rank's), the per-kernel breakdown and
    the roofline of the dominant kernel."""
    ms_step = ms / steps
    hbm, tf, tf_sus, src = peaks()
    bpk = bytes_per_key()
    q_bytes = n * (bpk["quantize_in"] + bpk["quantize_out"])
    l_bytes = n * (bpk["logits_in"] + bpk["logits_out"])
    kq, kl = ("tq_split_quantize", "tq_split_logits") if isinstance(BITS, tuple) else ("tq_quantize", "tq_logits")
    fl = n * quantize_flops_per_key() * (2 if ATTEND else 1)
    kernels = {
        kq: {"ms": q_ms, "bytes": q_bytes, "GB/s": q_bytes / q_ms / 1e6, "vectors_per_s": n / q_ms * 1e3,
             "flops": fl, "TFLOP/s": fl / q_ms / 1e9},
        kl: {"ms": l_ms, "bytes": l_bytes, "GB/s": l_bytes / l_ms / 1e6, "keys_per_s": n / l_ms * 1e3,
             "pct_of_8TBs": 100 * l_bytes / l_ms / 1e6 / 8000.0},
    }
    if a_ms is not None:
        a_bytes = n * bpk["attend_in"]
        kernels["tq_attend"] = {"ms": a_ms, "bytes": a_bytes, "GB/s": a_bytes / a_ms / 1e6,
                                "keys_per_s": n / a_ms * 1e3}
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    ach = kernels[dom]["GB/s"]
    dram = DRAM_BYTES_PER_KEY.get(WORKLOAD.split("_")[0], {}).get(dom)
    return {
        "metric": METRIC,
        "value": world * n / ms_step * 1e3,
        "unit": "keys/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if KEY_DTYPE == "bf16" else "f32",
        "data": "synthetic",
        "config": kv_config(world),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": hbm, "unit": "GB/s",
                     "frac": ach / hbm, "peak_source": src,
                     "traffic": None if dram is None else dram * n,
                     "traffic_source": "ncu capture at S=16384 scaled by keys (bytes per launch)"},
        "kernels": kernels,
        "logits_keys_per_s": world * n / l_ms * 1e3,
        "quantize_vectors_per_s": world * n / q_ms * 1e3,
        "e2e": {"value": world * n / e2e_ms * 1e3, "unit": "keys/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": (6 if a_ms is not None else 3) * steps,
        "clocks": clocks,
    }


def measure_kv(steps: int, warmup: int, local: int, dist=None, target_s: float | None = None,
               e2e: bool = True, keep: bool = False) -> dict:
    """One key-cache workload (the module's current shape globals) on this rank's GPU.

    A step quantizes the step's keys into one of two packed caches and scores
    the queries against the other (written one step earlier); with ATTEND it
    also quantizes values and computes the attention output.  Times: CUDA
    events on the launching stream, max over ranks.  With target_s, the step
    count is chosen from the warm-up time so that the timed loop lasts about
    target_s seconds.  keep: return the device tensors too (parity checks)."""
    import torch

    from compressed_kv_cache_tq_b200 import tq, workloads as W

    dev = torch.device("cuda", local)
    keys4 = device_keys(dev)
    keys = keys4.reshape(-1, D)
    n = keys.shape[0]
    q = torch.from_numpy(host_queries()).to(dev)
    out = torch.empty((B, HQ, S), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(D)
    stream = torch.cuda.current_stream()
    extra = {}
    if isinstance(BITS, tuple):
        # split: plan the channel groups once from the keys (calibration, timed on its own)
        hi, lo = tq.tq_init(D // 2, BITS[0], SEED_TABLES), tq.tq_init(D // 2, BITS[1], SEED_TABLES + 1)
        ctx = hi
        sp = tq.tq_split_create(hi, lo, HKV)
        pws = torch.empty(max(1, int(tq.lib().tq_split_plan_workspace_bytes(sp.handle))), dtype=torch.uint8,
                          device=dev)
        sp.plan(keys4, workspace=pws)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        sp.plan(keys4, workspace=pws)
        b_.record(stream)
        torch.cuda.synchronize()
        extra["split_plan_ms"] = a.elapsed_time(b_)
        caches = [(torch.empty((n, hi.row_bytes), dtype=torch.uint8, device=dev),
                   torch.empty((n, 2), dtype=torch.float16, device=dev),
                   torch.empty((n, lo.row_bytes), dtype=torch.uint8, device=dev),
                   torch.empty((n, 2), dtype=torch.float16, device=dev)) for _ in range(2)]
        ws = torch.empty(max(256, int(tq.lib().tq_split_logits_workspace_bytes(sp.handle, B, HQ))),
                         dtype=torch.uint8, device=dev)

        def quantize(k4, c):
            tq.tq_split_quantize(sp, k4, *c)

        def logits(qq, c):
            tq.tq_split_logits(sp, qq, *c, scale=scale, out=out, workspace=ws)
    else:
        ctx = tq.tq_init(D, BITS, SEED_TABLES, m=JL_ROWS)
        caches = [(torch.empty((n, ctx.row_bytes), dtype=torch.uint8, device=dev),
                   torch.empty((n, 2), dtype=torch.float16, device=dev)) for _ in range(2)]
        ws = torch.empty(tq.tq_logits_workspace_bytes(ctx, B, HQ, HKV), dtype=torch.uint8, device=dev)

        def quantize(k4, c):
            tq.tq_quantize(ctx, k4.reshape(-1, D), c[0], c[1])

        def logits(qq, c):
            tq.tq_logits(ctx, qq, c[0], c[1], HKV, scale=scale, out=out, workspace=ws)

    # fill both caches once so the first logits read valid data
    for c in caches:
        quantize(keys4, c)
    attend = None
    vals4 = dvals = None
    if ATTEND:
        vctx = tq.tq_init(D, BITS, SEED_TABLES + 100)
        vals4 = W.decode_keys(B, HKV, S, D, SEED_VALUES, device=dev)
        vcaches = [(torch.empty((n, vctx.row_bytes), dtype=torch.uint8, device=dev),
                    torch.empty((n, 2), dtype=torch.float16, device=dev)) for _ in range(2)]
        o_att = torch.empty((B, HQ, D), dtype=torch.float32, device=dev)
        aws = torch.empty(max(256, tq.tq_attend_workspace_bytes(vctx, B, HQ, HKV, S)), dtype=torch.uint8,
                          device=dev)
        for c in vcaches:
            tq.tq_quantize(vctx, vals4.reshape(-1, D), c[0], c[1])
        kq_only = quantize

        def quantize(k4, c):
            kq_only(k4, c)
            vc = vcaches[0 if c is caches[0] else 1]
            tq.tq_quantize(vctx, (vals4 if k4 is keys4 else dvals).reshape(-1, D), vc[0], vc[1])

        def attend(c):
            vc = vcaches[0 if c is caches[0] else 1]
            tq.tq_attend(vctx, out, vc[0], vc[1], HKV, out=o_att, workspace=aws)

    ev = []

    def step(i, record):
        cw, cr = caches[i % 2], caches[(i + 1) % 2]
        if record:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4 if attend else 3)]
            e[0].record(stream)
        quantize(keys4, cw)
        if record:
            e[1].record(stream)
        logits(q, cr)
        if record:
            e[2].record(stream)
        if attend:
            attend(cr)
            if record:
                e[3].record(stream)
        if record:
            ev.append(e)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(warmup):
        step(i, False)
    barrier()
    if target_s is not None:
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(3):
            step(i, False)
        b_.record(stream)
        torch.cuda.synchronize()
        per = a.elapsed_time(b_) / 3
        steps = int(max(10, min(20000, target_s * 1e3 / max(per, 1e-3))))
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        t_start.record(stream)
        for i in range(steps):
            step(i, True)
        t_end.record(stream)
        barrier()
    ms = max_over_ranks(t_start.elapsed_time(t_end), dist, dev)
    assert tq.tq_check_device_status(ctx) == 0, "a kernel reported a device-side error"
    q_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / len(ev)
    l_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / len(ev)
    a_ms = sum(e[2].elapsed_time(e[3]) for e in ev) / len(ev) if attend else None
    res = {"steps": steps, "ms": ms, "q_ms": q_ms, "l_ms": l_ms, "a_ms": a_ms, "n": n, "clocks": clocks.summary(),
           "extra": extra, "h2d": int(keys.numel() * keys.element_size() * (2 if ATTEND else 1) + q.numel() * 4),
           "d2h": int((B * HQ * D if ATTEND else out.numel()) * 4)}

    if e2e:
        # end to end through the public API: pinned host keys in, logits (or attention output) out
        host_keys = torch.empty(keys4.shape, dtype=keys4.dtype, pin_memory=True)
        host_keys.copy_(keys4)
        if ATTEND:
            host_vals = torch.empty(vals4.shape, dtype=vals4.dtype, pin_memory=True)
            host_vals.copy_(vals4)
            dvals = torch.empty_like(vals4)
            host_att = torch.empty(o_att.shape, dtype=o_att.dtype, pin_memory=True)
        host_q = q.cpu().pin_memory()
        host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        dkeys = torch.empty_like(keys4)
        dq = torch.empty_like(q)

        def e2e_step(i):
            cw, cr = caches[i % 2], caches[(i + 1) % 2]
            dkeys.copy_(host_keys, non_blocking=True)
            if ATTEND:
                dvals.copy_(host_vals, non_blocking=True)
            dq.copy_(host_q, non_blocking=True)
            quantize(dkeys, cw)
            logits(dq, cr)
            if attend:
                attend(cr)
                host_att.copy_(o_att, non_blocking=True)
            else:
                host_out.copy_(out, non_blocking=True)

        e2e_steps = max(3, min(steps, 10))
        for i in range(3):
            e2e_step(i)
        barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        b_.record(stream)
        barrier()
        res["e2e_ms"] = max_over_ranks(a.elapsed_time(b_) / e2e_steps, dist, dev)
    if keep:
        res.update(keys4=keys4, q=q, out=out, cache=caches[0], ctx=ctx, scale=scale)
    return res


def kv_entry(res: dict, cpu: dict | None) -> dict:
    """A `configs` entry: the workload's step and kernels, each kernel's
    algorithmic bytes per second against the measured HBM bandwidth."""
    line = result_line(world=1, n=res["n"], steps=res["steps"], warmup=3, ms=res["ms"], q_ms=res["q_ms"],
                       l_ms=res["l_ms"], e2e_ms=res.get("e2e_ms", res["ms"] / res["steps"]), a_ms=res["a_ms"],
                       h2d=res["h2d"], d2h=res["d2h"], clocks=res["clocks"])
    hbm = peaks()[0]
    for kern in line["kernels"].values():
        kern["frac_of_measured_hbm"] = kern["GB/s"] / hbm
    ent = {"workload": WORKLOAD, "steps": res["steps"], "ms_per_step": line["ms_per_step"],
           "keys_per_s": line["value"], "kernels": line["kernels"], "roofline": line["roofline"],
           "clocks": res["clocks"], **res["extra"]}
    if cpu is not None:
        ent["cpu_baseline"] = cpu
    return ent


def oracle_parity(res: dict, n_keys: int = 102400) -> dict:
    """The oracle check of the run's own outputs (test infrastructure, CPU):
    about n_keys sampled rows of the packed cache the timed steps wrote, from
    every (batch, KV head) pair, against the oracle's quantisation of the same
    keys, and the logits of those rows against the oracle's estimates from the
    packed rows.  Reports the fractions of mismatching codes and sign bits and
    of coordinates near a decision boundary."""
    import numpy as np
    import torch

    from tests.parity import REL_FLOOR, check_close, check_quantize, merge_stats, oracle_estimates, tables_of

    rep, lrep = {}, {}
    t0 = time.perf_counter()
    try:
        tb = tables_of(res["ctx"])
        G = HQ // HKV
        per = max(1, n_keys // (B * HKV))
        rng = np.random.default_rng(7)
        payload, norms = res["cache"][0], res["cache"][1]
        for b in range(B):
            for h in range(HKV):
                s_idx = np.sort(rng.choice(S, min(S, per), replace=False))
                rows = torch.from_numpy((b * HKV + h) * S + s_idx).to(payload.device)
                k64 = res["keys4"][b, h][rows - (b * HKV + h) * S].to(torch.float64).cpu().numpy()
                pl, nr = payload[rows].cpu().numpy(), norms[rows].cpu().numpy()
                st, _ = check_quantize(pl, nr, k64, tb)
                merge_stats(rep, st)
                est, A = oracle_estimates(pl, nr, res["q"][b, h * G:(h + 1) * G].cpu().double().numpy(), tb)
                got = res["out"][b, h * G:(h + 1) * G][:, rows - (b * HKV + h) * S].cpu().numpy()
                check_close(got, res["scale"] * est, res["scale"] * A, rel_floor=REL_FLOOR, report=lrep)
        ok, err = True, None
    except AssertionError as e:
        ok, err = False, str(e)[:300]
    out = {"ok": ok, "checked_against": "oracle (fp64 numpy)", **rep,
           "logits_worst_err_of_term_scale": lrep.get("logits_worst_of_A"),
           "logits_worst_rel_err": lrep.get("logits_worst_rel"), "logits_rel_floor": REL_FLOOR,
           "seconds": time.perf_counter() - t0}
    if err:
        out["error"] = err
    return out


def configs_block(local: int, no_cpu: bool, search_rows: int, search_queries: int) -> dict:
    """Every other configuration of the workload table, measured in this
    process after the headline workload (about a second of timed steps each),
    with its own oracle baseline on a bounded sample of the same workload."""
    import torch

    block = {}
    hbm, tf, _, src = peaks()
    for name, batch in (("toy", 1), ("toy", None), ("longctx", None), ("split", None), ("mse", None),
                        ("attend", None)):
        set_workload(name, batch=batch)
        key = name if batch is None else f"{name}_single_batch"
        try:
            res = measure_kv(10, 3, local, target_s=0.5 if batch == 1 else 1.0, e2e=False)
            cpu = None if no_cpu else cpu_baseline(budget_s=6.0, max_keys=1 << 17)
            block[key] = kv_entry(res, cpu)
        except Exception as e:   # one config failing must not hide the others
            block[key] = {"workload": WORKLOAD, "error": f"{type(e).__name__}: {str(e)[:200]}"}
        torch.cuda.empty_cache()
    set_workload("decode")
    try:
        res = measure_search(search_rows, search_queries, 3, 3, local)
        ent = {"workload": search_config(search_rows, search_queries, 200, 10, 1)["workload"],
               "per_bits": res["per_bits"], "clocks": res["clocks"],
               "peaks": {"hbm_GB_s": hbm, "tensor_TFLOP_s": tf, "source": src}}
        if not no_cpu:
            n_cpu = min(search_rows, 50_000)
            ent["cpu_baseline"] = search_cpu_baseline(res["db"][:n_cpu].double().cpu().numpy(),
                                                      res["qs"][:32].double().cpu().numpy(), search_rows, 10)
        block["search"] = ent
        del res
    except Exception as e:
        block["search"] = {"error": f"{type(e).__name__}: {str(e)[:200]}"}
    torch.cuda.empty_cache()
    return block


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other configurations measured after the headline workload")
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "longctx", "split", "attend", "mse", "toy", "search"])
    ap.add_argument("--rows", type=int, default=1_000_000, help="search: database rows")
    ap.add_argument("--queries", type=int, default=10_000, help="search: queries")
    ap.add_argument("--seq", type=int, default=None,
                    help="sequence length (default: the workload's own; smaller values for profiling)")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in KV_WORKLOADS:
        set_workload(args.workload, args.seq)
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.warmup < 3:
        args.warmup = 3
    if args.workload == "search":
        if args.steps == 1000:
            args.steps = 5
        return run_search(args)

    import torch

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    solo = world == 1 and rank == 0
    res = measure_kv(args.steps, args.warmup, local, dist, keep=solo and not args.no_cpu_baseline)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    line = result_line(world=world, n=res["n"], steps=args.steps, warmup=args.warmup, ms=res["ms"], q_ms=res["q_ms"],
                       l_ms=res["l_ms"], e2e_ms=res["e2e_ms"], a_ms=res["a_ms"], h2d=res["h2d"], d2h=res["d2h"],
                       clocks=res["clocks"])
    line.update(res["extra"])
    if solo:
        ctx_d = dense_logits_context(device_keys(torch.device("cuda", local)), res.get("q", torch.from_numpy(
            host_queries()).cuda(local)))
        for name in ("fp32", "bf16"):
            if f"{name}_ms" in ctx_d:
                ctx_d[f"logits_speedup_vs_{name}"] = ctx_d[f"{name}_ms"] / res["l_ms"]
        line["context_dense_logits"] = ctx_d
    if solo and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
        if not isinstance(BITS, tuple):
            # the oracle check of what the timed steps wrote (test infrastructure, host cores)
            line["parity"] = oracle_parity(res)
    for kk in ("keys4", "q", "out", "cache", "ctx"):
        res.pop(kk, None)
    torch.cuda.empty_cache()
    if solo and not args.no_configs and args.workload == "decode" and args.seq is None:
        line["configs"] = configs_block(local, args.no_cpu_baseline, args.rows, args.queries)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
