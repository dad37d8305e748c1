"""bench.py's workload table and algorithmic byte counts (host logic, no GPU).

The roofline numbers divide these per-key byte counts by measured kernel
times, so they are checked here against the packed layout's sizes
(include/tq.h: row bytes = dp b'/8 + mp/8, plus two fp16 norms)."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from oracle import tq_oracle as O  # noqa: E402


@pytest.fixture(autouse=True)
def _restore():
    yield
    bench.set_workload("decode")


def test_decode_bytes_per_key():
    bench.set_workload("decode")
    bpk = bench.bytes_per_key()
    assert bpk == {"quantize_in": 256, "quantize_out": O.row_bytes(128, 128, 3) + 4,
                   "logits_in": O.row_bytes(128, 128, 3) + 4, "logits_out": 16}
    assert bench.quantize_flops_per_key() == 2 * 128 * 128 + 2 * 128 * 128


def test_longctx_workload():
    bench.set_workload("longctx")
    assert (bench.B, bench.HKV, bench.S, bench.BITS) == (1, 8, 131072, 3)
    assert bench.bytes_per_key()["quantize_out"] == O.row_bytes(128, 128, 2) + 4


def test_split_bytes_per_key():
    bench.set_workload("split")
    bpk = bench.bytes_per_key()
    # two groups of 64 channels: b = 3 (2 code bits) and b = 2 (1 code bit), each with its sign bits and norms
    rows = O.row_bytes(64, 64, 2) + O.row_bytes(64, 64, 1) + 8
    assert bpk["quantize_out"] == bpk["logits_in"] == rows == 48
    assert bench.quantize_flops_per_key() == 2 * (2 * 64 * 64 + 2 * 64 * 64)


def test_mse_only_bytes_per_key():
    bench.set_workload("mse")
    bpk = bench.bytes_per_key()
    assert bpk["quantize_out"] == O.row_bytes(128, 0, 3) + 4 == 52
    assert bench.quantize_flops_per_key() == 2 * 128 * 128


def test_attend_bytes_per_key():
    bench.set_workload("attend")
    bpk = bench.bytes_per_key()
    row = O.row_bytes(128, 128, 3) + 4
    assert bpk["quantize_in"] == 512 and bpk["quantize_out"] == 2 * row
    assert bpk["attend_in"] == row + 16


def test_seq_override_renames_the_workload():
    bench.set_workload("split", 2048)
    assert bench.S == 2048 and "_s2048_" in bench.WORKLOAD


def test_result_line_names_the_dominant_kernel():
    bench.set_workload("attend")
    line = bench.result_line(world=1, n=1000, steps=10, warmup=3, ms=20.0, q_ms=1.0, l_ms=0.2, a_ms=1.5, e2e_ms=5.0,
                             h2d=1, d2h=1, clocks={})
    assert line["roofline"]["kernel"] == "tq_attend"
    assert line["gpu_launches"] == 60
    assert set(line["kernels"]) == {"tq_quantize", "tq_logits", "tq_attend"}


def test_toy_workload_fp32_keys_and_replicas():
    bench.set_workload("toy")
    assert (bench.B, bench.HKV, bench.HQ, bench.S, bench.BITS, bench.KEY_DTYPE) == (256, 1, 64, 4096, 3, "fp32")
    bpk = bench.bytes_per_key()
    # fp32 keys in; 64 fp32 logits out per key (all 64 x 4096 pairs)
    assert bpk == {"quantize_in": 512, "quantize_out": O.row_bytes(128, 128, 2) + 4,
                   "logits_in": O.row_bytes(128, 128, 2) + 4, "logits_out": 256}
    assert bench.kv_config(1)["key_dtype"] == "fp32"
    bench.set_workload("toy", batch=1)
    assert bench.B == 1 and bench.WORKLOAD.endswith("_x1_replicas")
    q = bench.host_queries()
    assert q.shape == (1, 64, 128) and q.dtype.name == "float32"
