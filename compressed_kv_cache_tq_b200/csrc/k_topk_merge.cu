// Merge of per-shard top-k lists: a database split by rows over several
// devices (or several calls) is searched shard by shard with tq_topk, the
// (score, shard-local id) lists are gathered, and this kernel keeps, per
// query, the k best by score descending and global id ascending (the order
// tq_topk itself uses; airosetta.com "Google TurboQuant" on vector search).
//
// One block per query: the parts * k candidates (<= 4096) are loaded into
// shared memory with their global ids (local id + the shard's first row),
// padded to a power of two with entries that sort last, and ordered by a
// bitonic sort on (order key of the score, id).
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kMergeThreads = 256;

// Monotone unsigned key of a float score; -0 and +0 map to the same key, so
// that they tie (and fall back to the id order) as equal scores do in tq_topk.
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = f == 0.f ? 0u : __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// true when candidate (ka, ia) goes after (kb, ib): lower score, or equal score and higher id
__device__ __forceinline__ bool after(uint32_t ka, int64_t ia, uint32_t kb, int64_t ib) {
  return ka < kb || (ka == kb && ia > ib);
}

__global__ void __launch_bounds__(kMergeThreads) topk_merge_kernel(const float* __restrict__ scores,
                                                                   const int64_t* __restrict__ ids,
                                                                   MergeOffsets off, int64_t nq, int parts, int k,
                                                                   int n2, int64_t* __restrict__ out_ids,
                                                                   float* __restrict__ out_scores) {
  extern __shared__ __align__(8) uint8_t smraw[];
  int64_t* sid = reinterpret_cast<int64_t*>(smraw);          // [n2]
  uint32_t* skey = reinterpret_cast<uint32_t*>(sid + n2);    // [n2]
  float* ssc = reinterpret_cast<float*>(skey + n2);          // [n2]
  const int64_t qi = blockIdx.x;
  const int nc = parts * k;
  for (int i = threadIdx.x; i < n2; i += kMergeThreads) {
    if (i < nc) {
      const int p = i / k, j = i - p * k;
      const size_t src = (size_t(p) * nq + qi) * k + j;
      const float s = scores[src];
      ssc[i] = s;
      skey[i] = order_key(s);
      sid[i] = ids[src] + off.first_row[p];
    } else {
      ssc[i] = 0.f;
      skey[i] = 0u;          // below every real score's key
      sid[i] = INT64_MAX;
    }
  }
  __syncthreads();
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < n2 / 2; t += kMergeThreads) {
        const int lo = 2 * t - (t & (stride - 1)), hi = lo + stride;
        const bool descending_block = (lo & size) == 0;   // this run sorts best-first
        const bool swap = descending_block ? after(skey[lo], sid[lo], skey[hi], sid[hi])
                                           : after(skey[hi], sid[hi], skey[lo], sid[lo]);
        if (swap) {
          const uint32_t tk = skey[lo];
          skey[lo] = skey[hi];
          skey[hi] = tk;
          const int64_t ti = sid[lo];
          sid[lo] = sid[hi];
          sid[hi] = ti;
          const float ts = ssc[lo];
          ssc[lo] = ssc[hi];
          ssc[hi] = ts;
        }
      }
      __syncthreads();
    }
  }
  for (int j = threadIdx.x; j < k; j += kMergeThreads) {
    out_ids[qi * k + j] = sid[j];
    out_scores[qi * k + j] = ssc[j];
  }
}

}  // namespace

cudaError_t launch_topk_merge(const float* scores, const int64_t* ids, const MergeOffsets& off, int64_t nq, int parts,
                              int k, int64_t* out_ids, float* out_scores, cudaStream_t st) {
  int n2 = 1;
  while (n2 < parts * k) n2 <<= 1;
  const size_t smem = size_t(n2) * (8 + 4 + 4);
  auto kern = topk_merge_kernel;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  kern<<<unsigned(nq), kMergeThreads, smem, st>>>(scores, ids, off, nq, parts, k, n2, out_ids, out_scores);
  return cudaGetLastError();
}

}  // namespace tq
