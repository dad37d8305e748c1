// Chunk plan of the value path (k_attend.cu): into how many chunks of keys
// the partial-sum kernels split each (batch, KV head), and their length.
// Host code; the host test compiles it alone.
#pragma once

#include <stdint.h>

namespace tq {

struct AttPlan {
  int nsplit;      // chunks per (batch, KV head), 1 .. kAttMaxSplits
  int64_t chunk;   // keys per chunk, a multiple of the tile
};

// The merge kernel holds one factor per chunk in shared memory.
constexpr int kAttMaxSplits = 1024;

// The time is the number of waves of resident blocks (two per SM) times a
// block's time, taken as a fixed part plus the chunk length.  The
// tensor-core kernel's fixed part (ring fill, the merge of its warps' partial
// sums) was measured at the cost of about 180 keys; the CUDA-core kernel's is
// charged as a small cost per split.  Chunks are whole tiles of `tile` keys;
// the last chunk may be short, none is empty.
inline AttPlan att_plan_for(int B, int Hkv, int64_t S, bool mma, int sms, int tile) {
  const int64_t groups = int64_t(B) * Hkv;
  const int64_t cap = int64_t(sms) * 2;
  int64_t max_ns = (S + tile - 1) / tile;
  if (max_ns > kAttMaxSplits) max_ns = kAttMaxSplits;
  if (max_ns < 1) max_ns = 1;
  int64_t best = 1;
  double best_cost = 1e300;
  for (int64_t ns = 1; ns <= max_ns; ++ns) {
    const double waves = double((groups * ns + cap - 1) / cap);
    const double cost = mma ? waves * (180.0 + double(S) / double(ns))
                            : waves / double(ns) + 0.0002 * double(ns);
    if (cost < best_cost) {
      best_cost = cost;
      best = ns;
    }
  }
  int64_t chunk = (S + best - 1) / best;
  chunk = (chunk + tile - 1) / tile * tile;
  if (chunk < tile) chunk = tile;
  int64_t ns = (S + chunk - 1) / chunk;
  if (ns < 1) ns = 1;
  return AttPlan{int(ns), chunk};
}

}  // namespace tq
