"""Host check of the value path's chunk plan (csrc/attend_plan.h): for many
(batch, KV heads, keys, SM count) shapes and both kernels, the chunks are
whole tiles, cover every key, none is empty, and there are at most as many
as the merge kernel holds factors for (it keeps one per chunk in shared
memory).  The decode-layer shape gets several chunks per (batch, KV head),
enough to fill the SMs.  The header is compiled alone with the host C++
compiler."""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "compressed_kv_cache_tq_b200", "csrc")

HARNESS = r"""
#include <cstdio>
#include "attend_plan.h"
using namespace tq;
int main() {
  const int Bs[] = {1, 2, 8, 32};
  const int Hs[] = {1, 8};
  const long long Ss[] = {0, 1, 127, 128, 129, 3000, 32768, 131072, 1000000, 4000000};
  const int smss[] = {148, 132, 1};
  for (int B : Bs) for (int H : Hs) for (long long S : Ss) for (int sms : smss) for (int mma = 0; mma < 2; ++mma) {
    const AttPlan p = att_plan_for(B, H, S, mma != 0, sms, 128);
    printf("%d %d %lld %d %d %d %lld %d\n", B, H, S, sms, mma, p.nsplit, (long long)p.chunk, kAttMaxSplits);
  }
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_attend_plan_chunks_cover_keys_within_merge_limit():
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "p.cpp")
        exe = os.path.join(td, "p")
        with open(src, "w") as f:
            f.write(HARNESS)
        subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, src, "-o", exe], check=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n")
    rows = [list(map(int, ln.split())) for ln in out if ln]
    assert len(rows) == 4 * 2 * 10 * 3 * 2
    plans = {}
    for B, H, S, sms, mma, ns, chunk, cap in rows:
        assert cap == 1024
        assert 1 <= ns <= cap, (B, H, S, sms, mma, ns)
        assert chunk >= 128 and chunk % 128 == 0
        assert ns * chunk >= S                         # every key in a chunk
        assert S == 0 or (ns - 1) * chunk < S          # no empty chunk
        plans[(B, H, S, sms, mma)] = ns
    # decode layer (8 x 8 groups of 32 768 keys, tensor-core kernel, 148 SMs):
    # several chunks per group, at least one full wave of two blocks per SM
    ns = plans[(8, 8, 32768, 148, 1)]
    assert ns > 1 and 64 * ns >= 2 * 148
    # a single short sequence stays one chunk
    assert plans[(1, 1, 127, 148, 1)] == 1 and plans[(1, 1, 0, 148, 0)] == 1
