"""Host check of the tensor-core search's work schedule (csrc/search_units.h):
for many (query tiles, row tiles, SM count) shapes, the CTAs of the launch
grid the launcher would pick together score every (query tile, row tile)
unit exactly once, the members of a group walk the same row tiles in the
same order, and no CTA gets much more than its share.  The header is
compiled alone with the host C++ compiler."""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "compressed_kv_cache_tq_b200", "csrc")

HARNESS = r"""
#include <cstdio>
#include <vector>
#include "search_units.h"
using namespace tq;
int main() {
  const long long qts[] = {1, 2, 3, 7, 8, 9, 15, 16, 17, 31, 32, 33, 79, 80, 200};
  const long long rts[] = {1, 2, 5, 61, 391, 7813};
  const int smss[] = {148, 132, 7, 4, 1};
  for (long long qt : qts)
    for (long long rt : rts)
      for (int sms : smss) {
        const long long G = search_group(qt, sms);
        const long long units = ((qt + G - 1) / G) * rt;   // as the launcher computes them
        const long long groups = units < sms / G ? units : sms / G;
        const long long grid = groups * G;
        std::vector<int> seen(qt * rt, 0);
        long long mx = 0;
        bool lockstep = true;
        for (long long g = 0; g < groups; ++g) {
          // members of one group: the same row tile at the same step
          std::vector<std::vector<long long>> rows(G);
          for (long long r = 0; r < G; ++r) {
            Units w(qt, rt, g * G + r, grid, G);
            long long c = 0;
            while (w.next()) {
              if (w.qt < 0 || w.qt >= qt || w.t < 0 || w.t >= rt || w.qt % G != r) {
                printf("BAD %lld %lld %d\n", qt, rt, sms);
                return 1;
              }
              ++seen[w.qt * rt + w.t];
              rows[r].push_back(w.qt / G * rt + w.t);
              ++c;
            }
            if (c > mx) mx = c;
          }
          for (long long r = 1; r < G; ++r)
            for (size_t i = 0; i < rows[r].size() && i < rows[0].size(); ++i)
              if (rows[r][i] != rows[0][i]) lockstep = false;
        }
        int once = 1;
        for (int x : seen) once &= (x == 1);
        const long long share = (units + groups - 1) / groups;
        printf("%lld %lld %d G=%lld grid=%lld once=%d lockstep=%d max=%lld share=%lld\n", qt, rt, sms, G, grid, once,
               lockstep ? 1 : 0, mx, share);
      }
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_search_schedule_covers_every_unit_once():
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "h.cpp")
        exe = os.path.join(td, "h")
        with open(src, "w") as f:
            f.write(HARNESS)
        subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, src, "-o", exe], check=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n")
    lines = [ln for ln in out if ln]
    assert len(lines) == 15 * 6 * 5
    for ln in lines:
        f = ln.split()
        qt, rt, sms = int(f[0]), int(f[1]), int(f[2])
        kv = dict(x.split("=") for x in f[3:])
        G, grid = int(kv["G"]), int(kv["grid"])
        assert kv["once"] == "1", ln
        assert kv["lockstep"] == "1", ln
        assert 1 <= grid <= sms and grid % G == 0, ln
        assert G <= max(1, qt), ln
        # a member's units are its group's share of (query-tile group, row tile) pairs
        assert int(kv["max"]) <= int(kv["share"]), ln
    # the vector-search workload (10^4 queries, 10^6 rows): 79 query tiles on
    # 148 SMs run in groups of eight on 144 CTAs
    big = [ln for ln in lines if ln.startswith("79 7813 148 ")]
    assert big and "G=8" in big[0] and "grid=144" in big[0]
