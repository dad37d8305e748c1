// Inner-product top-k over a packed database (vector search; airosetta.com
// "Google TurboQuant" names GloVe recall@1@k with near-zero indexing time).
//
// The tensor-core path (k_search_tc.cu) serves sm_100a and k <= 32; this file
// is the general path.  Three kernels per block of queries:
//   1. estimator scores for all (query, row) pairs (the logits kernels with
//      scale 1, one "KV head" holding the whole database);
//   2. per query, an exact radix select of the KC-th largest fp32 score and a
//      gather of the KC best candidate rows (KC = max(4k, 128) <= 1024);
//   3. per query, fp64 re-scoring of the candidates from the fp64 tables and a
//      bitonic sort by (score descending, id ascending); the first k are kept.
#include <cuda_fp16.h>

#include <algorithm>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kSelThreads = 1024;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One block per query.  Writes exactly KC candidate ids (n >= KC).
__global__ void __launch_bounds__(kSelThreads) select_kernel(const float* __restrict__ scores, int64_t n, int KC,
                                                             int64_t* __restrict__ cand) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_remaining, s_count_gt, s_count_eq;
  const float* sc = scores + size_t(blockIdx.x) * n;
  const int tid = threadIdx.x;
  uint32_t prefix = 0, mask = 0, remaining = uint32_t(KC);
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int64_t i = tid; i < n; i += kSelThreads) {
      const uint32_t k = order_key(sc[i]);
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t cum = 0;
      int bin = 255;
      for (; bin > 0; --bin) {
        if (cum + hist[bin] >= remaining) break;
        cum += hist[bin];
      }
      s_prefix = prefix | (uint32_t(bin) << shift);
      s_remaining = remaining - cum;
    }
    __syncthreads();
    prefix = s_prefix;
    remaining = s_remaining;
    mask |= 255u << shift;
    __syncthreads();
  }
  // prefix is now the KC-th largest key; take every key above it, then keys
  // equal to it until KC are taken.
  if (tid == 0) {
    s_count_gt = 0;
    s_count_eq = 0;
  }
  __syncthreads();
  const uint32_t thr = prefix;
  const uint32_t n_gt = uint32_t(KC) - remaining;    // keys strictly above thr
  int64_t* out = cand + size_t(blockIdx.x) * KC;
  for (int64_t i = tid; i < n; i += kSelThreads) {
    const uint32_t k = order_key(sc[i]);
    if (k > thr) {
      out[atomicAdd(&s_count_gt, 1u)] = i;
    } else if (k == thr) {
      const uint32_t slot = atomicAdd(&s_count_eq, 1u);
      if (slot < remaining) out[n_gt + slot] = i;
    }
  }
}

// One block per query: fp64 re-scoring and the final order.
__global__ void __launch_bounds__(512) rescore_kernel(const float* __restrict__ q, const int64_t* __restrict__ cand,
                                                      int KC, int SP, int k, const uint8_t* __restrict__ payload,
                                                      const uint16_t* __restrict__ norms,
                                                      const double* __restrict__ R, const double* __restrict__ P,
                                                      const double* __restrict__ c, int d, int m, int bmse,
                                                      int64_t* __restrict__ ids, float* __restrict__ out_scores) {
  extern __shared__ double smd[];
  double* sq = smd;              // d
  double* sx = sq + d;           // d: R q
  double* sy = sx + d;           // m: P (R q) = S q
  double* ssc = sy + m;          // SP scores (KC candidates, padded to a power of two)
  int64_t* sid = reinterpret_cast<int64_t*>(ssc + SP);  // SP ids
  const int tid = threadIdx.x, nth = blockDim.x;
  const int qi = blockIdx.x;
  for (int i = tid; i < d; i += nth) sq[i] = double(q[size_t(qi) * d + i]);
  __syncthreads();
  for (int j = tid; j < d; j += nth) {
    double s = 0.0;
    for (int i = 0; i < d; ++i) s += R[size_t(j) * d + i] * sq[i];
    sx[j] = s;
  }
  __syncthreads();
  for (int i = tid; i < m; i += nth) {
    double s = 0.0;
    for (int j = 0; j < d; ++j) s += P[size_t(i) * d + j] * sx[j];
    sy[i] = s;
  }
  __syncthreads();
  const RowGeom g = make_geom(d, m, bmse);
  const double qc = m > 0 ? kQjlConst / double(m) : 0.0;   // m = 0: no sign term
  for (int ci = tid; ci < KC; ci += nth) {
    const int64_t row = cand[size_t(qi) * KC + ci];
    const uint16_t* hw = reinterpret_cast<const uint16_t*>(payload + row * g.row_bytes);
    double a = 0.0, b = 0.0;
    for (int j = 0; j < d; ++j) a += c[unpack_code(hw, g, j)] * sx[j];
    for (int i = 0; i < m; ++i) b += unpack_sign(hw, g, i) ? sy[i] : -sy[i];
    const double n16 = double(half_bits_to_float(norms[2 * row]));
    const double r16 = double(half_bits_to_float(norms[2 * row + 1]));
    ssc[ci] = n16 * a + qc * r16 * b;
    sid[ci] = row;
  }
  for (int ci = KC + tid; ci < SP; ci += nth) {
    ssc[ci] = -__longlong_as_double(0x7ff0000000000000LL);
    sid[ci] = INT64_MAX;
  }
  __syncthreads();
  // bitonic sort, descending score, ascending id on ties
  for (int size = 2; size <= SP; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < SP; i += nth) {
        const int jx = i ^ stride;
        if (jx > i) {
          const bool up = (i & size) == 0;
          const double si = ssc[i], sj = ssc[jx];
          const int64_t ii = sid[i], ij = sid[jx];
          const bool i_first = (si > sj) || (si == sj && ii < ij);
          if (up ? !i_first : i_first) {
            ssc[i] = sj;
            ssc[jx] = si;
            sid[i] = ij;
            sid[jx] = ii;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < k; i += nth) {
    ids[size_t(qi) * k + i] = sid[i];
    out_scores[size_t(qi) * k + i] = float(ssc[i]);
  }
}

// Candidates kept per query: max(4k, 128), at most 1024 and at most n (then
// every row is re-scored).
int candidates(int64_t n, int k) {
  int64_t kc = std::max<int64_t>(4 * int64_t(k), 128);
  kc = std::min<int64_t>(kc, 1024);
  return int(std::min<int64_t>(kc, n));
}

int pow2_at_least(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

int64_t query_block(int64_t nq, int64_t n) {
  const int64_t cap = std::max<int64_t>(1, (int64_t(1) << 30) / std::max<int64_t>(n * 4, 1));
  return std::min(nq, cap);
}

}  // namespace

size_t topk_ws_bytes(const tq_ctx* ctx, int64_t nq, int64_t n, int k) {
  if (search_tc_supported(ctx, nq, n, k)) return search_ws_bytes(ctx, nq, n);
  const int64_t qb = query_block(nq, n);
  const int kc = candidates(n, k);
  const size_t scores = ((size_t(qb) * n * 4 + 255) / 256) * 256;
  const size_t cand = ((size_t(qb) * kc * 8 + 255) / 256) * 256;
  const size_t lws = qprep_bytes(ctx, 1, int(std::min<int64_t>(qb, 1 << 20)));
  return scores + cand + lws;
}

cudaError_t launch_topk(const tq_ctx* ctx, const float* q, int64_t nq, const uint8_t* payload,
                        const uint16_t* norms, int64_t n, int k, int64_t* ids, float* scores, void* ws,
                        cudaStream_t st) {
  // tensor-core scoring with exact re-scoring of the candidates (sm_100a, k <= 32)
  if (search_tc_supported(ctx, nq, n, k))
    return launch_search_tc(ctx, q, nq, payload, norms, n, k, ids, scores, ws, st);
  const int64_t qb = query_block(nq, n);
  const int kc = candidates(n, k);
  const int sp = pow2_at_least(kc);
  float* sc = static_cast<float*>(ws);
  const size_t scores_bytes = ((size_t(qb) * n * 4 + 255) / 256) * 256;
  int64_t* cand = reinterpret_cast<int64_t*>(static_cast<uint8_t*>(ws) + scores_bytes);
  const size_t cand_bytes = ((size_t(qb) * kc * 8 + 255) / 256) * 256;
  void* lws = static_cast<uint8_t*>(ws) + scores_bytes + cand_bytes;
  const size_t rs_smem = size_t(2 * ctx->d + ctx->m + sp) * 8 + size_t(sp) * 8;
  cudaFuncSetAttribute(rescore_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(rs_smem));
  for (int64_t q0 = 0; q0 < nq; q0 += qb) {
    const int64_t nb = std::min(qb, nq - q0);
    // all nb queries against the whole database as one GQA group
    cudaError_t e = launch_logits(ctx, q + q0 * ctx->d, 1, int(nb), 1, n, payload, norms, 1.0f, sc, lws, st);
    if (e != cudaSuccess) return e;
    select_kernel<<<unsigned(nb), kSelThreads, 0, st>>>(sc, n, kc, cand);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    rescore_kernel<<<unsigned(nb), 512, rs_smem, st>>>(q + q0 * ctx->d, cand, kc, sp, k, payload, norms, ctx->dR64,
                                                        ctx->dP64, ctx->dc64, ctx->d, ctx->m, ctx->bmse,
                                                        ids + q0 * k, scores + q0 * k);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tq
