// Inner-product top-k on the tensor cores (sm_100a): the vector-search use of
// airosetta.com "Google TurboQuant" (recall@1@k over GloVe-like vectors with
// near-zero indexing time).  The estimator of one (query, row) pair,
//   s = n16 sum_j c[idx_j] (Rq)_j + sqrt(pi/2)/m rho16 sum_i sigma_i (Sq)_i,
// is one inner product s = <Kw, Qw> of a per-row weight vector
//   Kw = [n16 c[idx_0 .. d-1], sqrt(pi/2)/m rho16 sigma_0 .. m-1, 0 ...]
// and a per-query vector Qw = [Rq, Sq, 0 ...], both KP = round-up(d + m, 64)
// long.  Five kernels:
//   1. decode_rows_kernel: packed rows -> Kw in fp16 (one warp per row), and
//      the largest code-part norm ||Kw_code|| and sign weight |w| over rows.
//   2. query_tables_kernel: x = R q and y = P R q = S q in fp64 (kept for the
//      exact re-scoring).
//   3. prep_queries_kernel: Qw = [x, y] rounded to fp16 and the per-query
//      error bound E_q.
//   4. search_tc_kernel: tcgen05 MMA of 128-query tiles (resident in tensor
//      memory, the A operand) against 128-row tiles (a twelve-stage TMA ring
//      of 16 KB K-blocks: shared memory holds only row tiles, so that about
//      190 KB of them are in flight per SM), scores in TMEM; the epilogue
//      keeps each query's running k best scores and appends every row whose
//      score is at least (k-th best - 2 E_q) to the query's candidate list.
//   5. finish_kernel: per query, the k-th largest approximate score among the candidates (by
//      bisection), the candidates within 2 E_q of it re-scored exactly in fp64
//      and ordered by (score descending, id ascending); the first k are the
//      answer.
// Completeness: every approximate score is within E_q of the exact one.  The
// k-th largest approximate score A_k is then at most T + E_q (T: the exact
// k-th largest; otherwise k rows would have exact scores above T), and every
// row of the exact top k has approximate score >= T - E_q >= A_k - 2 E_q, so
// it is a candidate.  A CTA that scans only part of the rows uses its own,
// lower, A_k: its cut keeps a superset.  Segments of the same query share the
// largest local A_k published so far (each is at most the global one, so the
// argument holds for their maximum).  A query whose candidate list
// overflows is answered by an exact scan of all rows in the finishing kernel.
// Error bound: Kw (from fp32 arithmetic) and Qw (from the fp64 tables) are
// rounded to fp16 (relative 2^-11 each; the bound below also leaves 2e-4 of
// ||Kw|| ||q|| for fp32 arithmetic before the rounding), and the tensor cores accumulate KP <= 512 exact products in
// fp32 (below KP 2^-23 of sum |Kw_j Qw_j|).  With
//   sum_j |Kw_j Qw_j| <= max ||Kw_code|| ||Rq||_2 + max |w| ||Sq||_1
// (Cauchy-Schwarz on the code part; the sign part has |sigma_i| = 1),
//   E_q = 1.5e-3 (max ||Kw_code|| ||Rq||_2 + max |w| ||Sq||_1) + an absolute
// term for fp16 subnormals bounds |s_approx - s| (1.5e-3 > 2^-10 + 512 2^-23
// + 2e-4).
#include <cuda_fp16.h>

#include <algorithm>

#include "search_units.h"
#include "tc_sm100.cuh"
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

using namespace tc;

constexpr int kQT = 128;                 // queries per tile (MMA M)
constexpr int kRT = 128;                 // database rows per tile (MMA N)
constexpr int kBStages = 12;             // row-tile K-block ring (16 KB stages)
constexpr int kSearchThreads = 192;      // TMA warp, MMA warp, 4 epilogue warps
constexpr int kMaxK = 32;                // k handled by the epilogue's running top-k
constexpr int kCap = 2048;               // candidates kept per query
constexpr float kErrRel = 1.5e-3f;       // relative error bound (see above)
constexpr float kErrAbs = 0x1p-20f;      // absolute term (fp16 subnormals)
constexpr uint32_t kIdescSearch = idesc_f16(0, kQT, kRT);   // fp16 x fp16 -> fp32, 128 x 128
// TMEM: the query tile (A operand, K-major, two fp16 per column) in columns
// 0 .. KP / 2 - 1 (at most 256), two score accumulators of 128 columns above.
constexpr uint32_t kTmemD = 256;

struct SearchSmem {
  static constexpr uint32_t kOffB = 0;                           // kBStages blocks of 128 rows x 128 B
  static constexpr uint32_t kOffBar = kOffB + kBStages * 16384u;
  static constexpr uint32_t kBytes = kOffBar + 256 + 1024;       // + slack for 1024-byte alignment
};

enum SBar {
  kSAFull = 0,                 // query tile written to TMEM (128 epilogue arrivals)
  kSBFull = 1,
  kSBEmpty = kSBFull + kBStages,
  kSDFull = kSBEmpty + kBStages,
  kSDEmpty = kSDFull + 2,
  kSDone = kSDEmpty + 2,       // final commit of the MMA thread (tracks every MMA it issued)
  kSNumBars = kSDone + 1
};

// Waits test the phase without a suspend-time hint: the pipeline's waits often
// find the phase incomplete, and a suspended thread resumed far too late.
__device__ __forceinline__ bool swait(uint32_t bar, uint32_t parity, volatile int* abort_flag, uint32_t* status) {
  return tc::mbar_wait<false>(bar, parity, abort_flag, status, kStatusSearchTc);
}
__device__ __forceinline__ bool swait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           uint32_t* status) {
  return tc::mbar_wait_warp<false>(bar, parity, abort_flag, status, kStatusSearchTc);
}
__device__ __forceinline__ void sdrain(uint32_t bar, uint32_t parity, volatile int* abort_flag, uint32_t* status) {
  tc::mbar_drain<false>(bar, parity, abort_flag, status, kStatusSearchTc);
}

// One warp per row: Kw in fp16, rows n .. n_pad - 1 all zero.  maxk_bits[0]
// gets the largest ||Kw_code|| and maxk_bits[1] the largest |w| (of the
// rounded values, as float bits).
// Kw entries 8 c .. 8 c + 7 of one row (lv: the levels, n16: the row's norm,
// w: its sign weight).  A chunk of codes lies in one quarter and one
// 16-coordinate unit of the packed layout (a quarter holds dp / 4 codes, a
// multiple of 16), so its codes come from at most three halfwords; so do a
// chunk's signs when it starts at a multiple of 8 past d.  Other chunks take
// the general unpack per entry (with d and m multiples of 8, only the zero
// padding past d + m).
__device__ __forceinline__ void decode_chunk(const uint16_t* __restrict__ hw, const RowGeom& g, int c,
                                             const float* lv, float n16, float w, float (&v)[8]) {
  const int j0 = 8 * c;
  if (j0 + 8 <= g.d) {
    const int qd = g.dp >> 2;
    const int q = (j0 >= qd) + (j0 >= 2 * qd) + (j0 >= 3 * qd);
    const int r0 = (j0 - q * qd) >> 2;   // register of entries 0..3; entries 4..7 are in r0 + 1
    const int i0 = r0 & 3;               // 0 or 2
    const uint16_t* base = hw + q * g.per_q + (r0 >> 2) * g.bmse;
    if (g.bmse == 3) {
      const uint32_t h0 = __ldg(base), h1 = __ldg(base + 1), h2 = __ldg(base + 2);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (i0 == 0) {
          v[e] = n16 * lv[(h0 >> (4 * e)) & 7u];
          v[4 + e] = n16 * lv[(h1 >> (4 * e)) & 7u];
        } else {
          v[e] = n16 * lv[(h2 >> (4 * e)) & 7u];
          v[4 + e] = n16 * lv[((h0 >> (4 * e + 3)) & 1u) | (((h1 >> (4 * e + 3)) & 1u) << 1) |
                              (((h2 >> (4 * e + 3)) & 1u) << 2)];
        }
      }
    } else if (g.bmse == 2) {
      const uint32_t h = __ldg(base + (i0 >> 1));
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[e] = n16 * lv[(h >> (4 * e)) & 3u];
        v[4 + e] = n16 * lv[(h >> (4 * e + 2)) & 3u];
      }
    } else {
      const uint32_t h = __ldg(base);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[e] = n16 * lv[(h >> (4 * e + i0)) & 1u];
        v[4 + e] = n16 * lv[(h >> (4 * e + i0 + 1)) & 1u];
      }
    }
    return;
  }
  const int s0 = j0 - g.d;
  if (s0 >= 0 && j0 + 8 <= g.d + g.m && (s0 & 7) == 0) {
    const int qm = g.mp >> 2;
    const int q = (s0 >= qm) + (s0 >= 2 * qm) + (s0 >= 3 * qm);
    const int r0 = (s0 - q * qm) >> 2, i0 = r0 & 3;
    const uint32_t h = __ldg(hw + q * g.per_q + g.bmse * g.uq + (r0 >> 2));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[e] = (h >> (4 * e + i0)) & 1u ? w : -w;
      v[4 + e] = (h >> (4 * e + i0 + 1)) & 1u ? w : -w;
    }
    return;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int j = j0 + e;
    v[e] = j < g.d ? n16 * lv[unpack_code(hw, g, j)] : j < g.d + g.m ? (unpack_sign(hw, g, j - g.d) ? w : -w) : 0.f;
  }
}

// One warp per row, the rows taken in a grid-stride loop: Kw in fp16, and the
// largest code-part norm and sign weight over the rows (reduced in the block,
// one atomic per block and quantity).
__global__ void __launch_bounds__(256) decode_rows_kernel(const uint8_t* __restrict__ payload,
                                                          const uint16_t* __restrict__ norms, int64_t n,
                                                          int64_t n_pad, int d, int m, int bmse, int kp,
                                                          CodebookParams cb, __half* __restrict__ kw,
                                                          uint32_t* __restrict__ maxk_bits) {
  __shared__ float lv[kMaxLevels];
  __shared__ float red[2][8];
  if (threadIdx.x < kMaxLevels) lv[threadIdx.x] = cb.c[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const RowGeom g = make_geom(d, m, bmse);
  const int64_t nwarps = int64_t(gridDim.x) * (blockDim.x >> 5);
  float mk = 0.f, mw = 0.f;
  for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + wib; r < n_pad; r += nwarps) {
    __half* out = kw + r * kp;
    if (r >= n) {   // padding rows
      for (int c = lane; c < kp / 8; c += 32) *reinterpret_cast<uint4*>(out + 8 * c) = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint16_t* hw = reinterpret_cast<const uint16_t*>(payload + r * g.row_bytes);
    const float n16 = half_bits_to_float(__ldg(norms + 2 * r));
    const float w = m > 0 ? float(kQjlConst) / float(m) * half_bits_to_float(__ldg(norms + 2 * r + 1)) : 0.f;
    float ss = 0.f;
    for (int c = lane; c < kp / 8; c += 32) {
      float v[8];
      decode_chunk(hw, g, c, lv, n16, w, v);
      __align__(16) __half h[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        h[e] = __float2half_rn(v[e]);
        const float hv = __half2float(h[e]);
        if (8 * c + e < d) ss = fmaf(hv, hv, ss);
      }
      *reinterpret_cast<uint4*>(out + 8 * c) = *reinterpret_cast<const uint4*>(h);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    mk = fmaxf(mk, sqrtf(ss));
    mw = fmaxf(mw, fabsf(__half2float(__float2half_rn(w))));
  }
  if (lane == 0) {
    red[0][wib] = mk;
    red[1][wib] = mw;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < int(blockDim.x >> 5); ++i) {
      mk = fmaxf(mk, red[0][i]);
      mw = fmaxf(mw, red[1][i]);
    }
    if (mk > 0.f) atomicMax(maxk_bits, __float_as_uint(mk));   // non-negative floats order as their bits
    if (mw > 0.f) atomicMax(maxk_bits + 1, __float_as_uint(mw));
  }
}

// One warp per query: Qw = [R q, P R q] rounded to fp16 from the query's
// fp64 tables xy = [x, y] (the rest of the row was zeroed by the caller), and
// the error bound E_q (see the top of this file) from the rounded values.
__global__ void __launch_bounds__(256) prep_queries_kernel(const double* __restrict__ xy, int64_t nq, int d, int m,
                                                           int kp, const uint32_t* __restrict__ maxk_bits,
                                                           __half* __restrict__ qw, float* __restrict__ qerr) {
  const int lane = threadIdx.x & 31;
  const int64_t qi = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (qi >= nq) return;
  const double* src = xy + qi * (d + m);
  float ss = 0.f, s1 = 0.f;   // ||Rq||_2^2 and ||Sq||_1 of the rounded values
  for (int i = lane; i < d + m; i += 32) {
    const __half h = __double2half(src[i]);
    qw[qi * kp + i] = h;
    const float hv = __half2float(h);
    if (i < d)
      ss = fmaf(hv, hv, ss);
    else
      s1 += fabsf(hv);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
  }
  if (lane == 0) {
    const float rq = sqrtf(ss), kc = __uint_as_float(maxk_bits[0]), kw1 = __uint_as_float(maxk_bits[1]);
    qerr[qi] = kErrRel * (kc * rq + kw1 * s1) + kErrAbs * (kc + float(m) * kw1 + rq + s1);
  }
}

// float -> uint32 with the same order
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int KB>
__global__ void __launch_bounds__(kSearchThreads, 1) search_tc_kernel(
    const __grid_constant__ CUtensorMap kmap, const __half* __restrict__ qw, int64_t nq, int64_t n,
    int64_t qtiles, int64_t row_tiles, int64_t group, int k, const float* __restrict__ qerr,
    uint32_t* __restrict__ gkth, uint32_t* __restrict__ cnt,
    uint2* __restrict__ cand, uint32_t* __restrict__ status) {
  using L = SearchSmem;
  constexpr int kp = 64 * KB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + L::kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::kOffBar + 8 * kSNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + L::kOffBar + 8 * kSNumBars + 4);
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar(kSAFull), 128);
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(bar(kSBFull + s), 1);
      mbar_init(bar(kSBEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kSDFull + s), 1);
      mbar_init(bar(kSDEmpty + s), 128);
    }
    mbar_init(bar(kSDone), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // (row tiles only: the epilogue writes each query tile into TMEM)
    if (lane == 0) {
      int64_t it = 0;
      bool ok = true;
      Units w(qtiles, row_tiles, blockIdx.x, gridDim.x, group);
      while (ok && w.next()) {
        const int64_t t = w.t;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = int(it % kBStages);
          if (it >= kBStages && !swait(bar(kSBEmpty + s), uint32_t((it / kBStages - 1) & 1), abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar(kSBFull + s), 16384u);
          tma_load_2d(base + L::kOffB + 16384u * s, &kmap, 64 * kb, int(t * kRT), bar(kSBFull + s));
        }
      }
      // leave no copy in flight
      for (int64_t j = (it >= kBStages ? it - kBStages : 0); j < it; ++j)
        sdrain(bar(kSBFull + int(j % kBStages)), uint32_t((j / kBStages) & 1), abort_flag, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      int64_t qt_prev = -1, it = 0, j = 0;
      int na = 0;
      bool ok = true;
      Units w(qtiles, row_tiles, blockIdx.x, gridDim.x, group);
      for (; ok && w.next(); ++j) {
        const int64_t qt = w.qt;
        if (qt != qt_prev) {
          // the epilogue has written this query tile into TMEM (it does so
          // only after the scores of every unit of the previous tile, so no
          // MMA still reads the old one)
          if (!swait(bar(kSAFull), uint32_t(na & 1), abort_flag, status)) break;
          ++na;
          qt_prev = qt;
        }
        const int slot = int(j & 1);
        if (j >= 2 && !swait(bar(kSDEmpty + slot), uint32_t(((j >> 1) - 1) & 1), abort_flag, status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + kTmemD + 128u * slot;
        uint32_t acc = 0;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = int(it % kBStages);
          if (!swait(bar(kSBFull + s), uint32_t((it / kBStages) & 1), abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int ks = 0; ks < 4; ++ks) {
            // query coordinates 64 kb + 16 ks .. +15: TMEM columns 32 kb + 8 ks .. +7
            mma_f16_ts(d_tmem, tmem + 32u * kb + 8u * ks, smem_desc(base + L::kOffB + 16384u * s + 32u * ks),
                       kIdescSearch, acc);
            acc = 1;
          }
          mma_commit(bar(kSBEmpty + s));
        }
        if (!ok) break;
        mma_commit(bar(kSDFull + slot));
      }
      // one more commit tracks every MMA issued, on every exit path
      mma_commit(bar(kSDone));
      sdrain(bar(kSDone), 0u, abort_flag, status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // thread = query row of the tile (TMEM lane (warp & 3) * 32 + lane).  The
    // hot path is one compare per score into a 32-bit mask; the rare hits go
    // through a short loop (code kept small: the MMA issuer shares the
    // instruction cache).
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    int64_t qt_prev = -1, q = -1;
    float E2 = 0.f, kth = -INFINITY;
    float topv[kMaxK];     // the k best scores so far (unordered; dynamic index, local memory)
    float vl[32];          // a chunk with hits
    // candidates of the current tile, staged per thread (at most one per
    // score) and appended with one atomic per tile
    uint2 stage[kRT];
    int64_t j = 0;
    Units w(qtiles, row_tiles, blockIdx.x, gridDim.x, group);
    for (; w.next(); ++j) {
      const int64_t qt = w.qt, t = w.t;
      if (qt != qt_prev) {
        qt_prev = qt;
        q = qt * kQT + row;
        E2 = q < nq ? 2.f * qerr[q] : 0.f;
        // this thread's query row (zero past nq) into TMEM lane `row`, columns
        // 0 .. kp / 2 - 1.  Every MMA on the previous query tile has completed:
        // the scores of its last unit were waited for above.
        const uint4* src = reinterpret_cast<const uint4*>(qw + size_t(q) * kp);
#pragma unroll 4
        for (int c = 0; c < kp / 16; ++c) {
          const uint4 lo = __ldg(src + 2 * c), hi = __ldg(src + 2 * c + 1);
          const uint32_t r[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
          tmem_st8(tmem + lane_base + 8u * c, r);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        mbar_arrive(bar(kSAFull));
#pragma unroll 1
        for (int i = 0; i < k; ++i) topv[i] = -INFINITY;
        kth = -INFINITY;
      }
      const int slot = int(j & 1);
      if (!swait_warp(bar(kSDFull + slot), uint32_t((j >> 1) & 1), abort_flag, status)) break;
      tc_fence_after();
      const int64_t r0 = t * kRT;
      int ns = 0;
      // the best k-th score any segment of this query has published (0: none)
      float gk = -INFINITY;
      if (q < nq) {
        const uint32_t gkey = *reinterpret_cast<volatile uint32_t*>(gkth + q);
        if (gkey) gk = key_float(gkey);
      }
#pragma unroll 1
      for (int c = 0; c < kRT / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_base + kTmemD + 128u * slot + 32u * c, v);
        tmem_wait32(v);
        if (q >= nq) continue;
        const float thr = fmaxf(kth, gk) - E2;
        uint32_t mask = 0;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) mask |= (v[jj] >= thr ? 1u : 0u) << jj;
        const int64_t valid = n - (r0 + 32 * c);   // rows past n are padding
        if (valid < 32) mask &= valid > 0 ? (1u << valid) - 1u : 0u;
        if (mask == 0) continue;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) vl[jj] = v[jj];
#pragma unroll 1
        while (mask) {
          const int jj = __ffs(mask) - 1;
          mask &= mask - 1;
          const float a = vl[jj];
          if (!(a >= fmaxf(kth, gk) - E2)) continue;   // kth may have risen within the chunk
          stage[ns++] = make_uint2(__float_as_uint(a), uint32_t(r0 + 32 * c + jj));
          if (a > kth) {
            // replace one of the k kept scores equal to kth, then find the new smallest
            int im = 0;
#pragma unroll 1
            for (int i = 0; i < k; ++i)
              if (topv[i] == kth) {
                im = i;
                break;
              }
            topv[im] = a;
            float mn = INFINITY;
#pragma unroll 1
            for (int i = 0; i < k; ++i) mn = fminf(mn, topv[i]);
            kth = mn;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(kSDEmpty + slot));
      if (q < nq && kth > gk) atomicMax(gkth + q, order_key(kth));   // publish this segment's k-th best
      if (ns > 0) {
        const uint32_t pos = atomicAdd(&cnt[q], uint32_t(ns));
#pragma unroll 1
        for (int i = 0; i < ns; ++i)
          if (pos + uint32_t(i) < uint32_t(kCap)) cand[size_t(q) * kCap + pos + i] = stage[i];
      }
    }
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");   // none in flight on an early exit
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// Exact (fp64) estimate of one packed row against x = R q, y = P R q.
__device__ double exact_score(const uint8_t* __restrict__ payload, const uint16_t* __restrict__ norms, int64_t row,
                              const RowGeom& g, const double* __restrict__ c, const double* x, const double* y,
                              double qc) {
  const uint16_t* hw = reinterpret_cast<const uint16_t*>(payload + row * g.row_bytes);
  double a = 0.0, b = 0.0;
  for (int j = 0; j < g.d; ++j) a += c[unpack_code(hw, g, j)] * x[j];
  for (int i = 0; i < g.m; ++i) b += unpack_sign(hw, g, i) ? y[i] : -y[i];
  const double n16 = double(half_bits_to_float(norms[2 * row]));
  const double r16 = double(half_bits_to_float(norms[2 * row + 1]));
  return n16 * a + qc * r16 * b;
}

// The same estimate, its terms split over the 32 lanes of a warp (lane `ln`
// takes coordinates ln, ln + 32, ...) and summed by a butterfly: every lane
// returns the same value, and equal rows get equal scores.
__device__ double exact_score_warp(const uint8_t* __restrict__ payload, const uint16_t* __restrict__ norms,
                                   int64_t row, const RowGeom& g, const double* __restrict__ c, const double* x,
                                   const double* y, double qc, int ln) {
  const uint16_t* hw = reinterpret_cast<const uint16_t*>(payload + row * g.row_bytes);
  double a = 0.0, b = 0.0;
  for (int j = ln; j < g.d; j += 32) a += c[unpack_code(hw, g, j)] * x[j];
  for (int i = ln; i < g.m; i += 32) b += unpack_sign(hw, g, i) ? y[i] : -y[i];
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
    b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
  }
  const double n16 = double(half_bits_to_float(norms[2 * row]));
  const double r16 = double(half_bits_to_float(norms[2 * row + 1]));
  return n16 * a + qc * r16 * b;
}

// (score descending, id ascending): true when (sa, ia) comes first
__device__ __forceinline__ bool first(double sa, int64_t ia, double sb, int64_t ib) {
  return sa > sb || (sa == sb && ia < ib);
}

constexpr int kFinishThreads = 256;
constexpr int kTabQueries = 8;      // queries per block of query_tables_kernel

// x = R q and y = P x in fp64 for kTabQueries queries per block (the tables
// are read once per block): xy[q] = [x (d), y (m)].
__global__ void __launch_bounds__(256) query_tables_kernel(const float* __restrict__ q, int64_t nq, int d, int m,
                                                           const double* __restrict__ R,
                                                           const double* __restrict__ P,
                                                           double* __restrict__ xy) {
  __shared__ double sq[kTabQueries][256];
  __shared__ double sx[kTabQueries][256];
  const int64_t q0 = int64_t(blockIdx.x) * kTabQueries;
  const int nb = int(nq - q0 < kTabQueries ? nq - q0 : kTabQueries);
  const int tid = threadIdx.x;
  for (int idx = tid; idx < kTabQueries * d; idx += blockDim.x) {
    const int qq = idx / d, i = idx - qq * d;
    sq[qq][i] = qq < nb ? double(q[(q0 + qq) * d + i]) : 0.0;
  }
  __syncthreads();
  for (int j = tid; j < d; j += blockDim.x) {
    double acc[kTabQueries];
#pragma unroll
    for (int qq = 0; qq < kTabQueries; ++qq) acc[qq] = 0.0;
    for (int i = 0; i < d; ++i) {
      const double r = R[size_t(j) * d + i];
#pragma unroll
      for (int qq = 0; qq < kTabQueries; ++qq) acc[qq] += r * sq[qq][i];
    }
#pragma unroll
    for (int qq = 0; qq < kTabQueries; ++qq) {
      sx[qq][j] = acc[qq];
      if (qq < nb) xy[(q0 + qq) * (d + m) + j] = acc[qq];
    }
  }
  __syncthreads();
  for (int i = tid; i < m; i += blockDim.x) {
    double acc[kTabQueries];
#pragma unroll
    for (int qq = 0; qq < kTabQueries; ++qq) acc[qq] = 0.0;
    for (int j = 0; j < d; ++j) {
      const double pv = P[size_t(i) * d + j];
#pragma unroll
      for (int qq = 0; qq < kTabQueries; ++qq) acc[qq] += pv * sx[qq][j];
    }
#pragma unroll
    for (int qq = 0; qq < kTabQueries; ++qq)
      if (qq < nb) xy[(q0 + qq) * (d + m) + d + i] = acc[qq];
  }
}

// Block-wide sum of one int per thread.
__device__ __forceinline__ int block_sum(int v, int* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  int t = 0;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

// One block per query.  Shared memory: x (d) and y (m) in fp64, then kCap
// (score, id) pairs for the final sort.
__global__ void __launch_bounds__(kFinishThreads) finish_kernel(
    int d, int m, int bmse, int k, int64_t n, const uint8_t* __restrict__ payload,
    const uint16_t* __restrict__ norms, const double* __restrict__ xy, const double* __restrict__ c,
    const float* __restrict__ qerr, const uint32_t* __restrict__ cnt, const uint2* __restrict__ cand,
    int64_t* __restrict__ ids, float* __restrict__ out_scores) {
  extern __shared__ double smd[];
  double* sx = smd;                 // d
  double* sy = sx + 256;            // m
  double* ssc = sy + 256;           // kCap scores
  int64_t* sid = reinterpret_cast<int64_t*>(ssc + kCap);   // kCap ids
  __shared__ int red[kFinishThreads / 32];
  __shared__ double rs[kFinishThreads / 32];
  __shared__ int64_t ri[kFinishThreads / 32];
  __shared__ int rw[kFinishThreads / 32];
  __shared__ int s_mc;
  const int tid = threadIdx.x, nth = blockDim.x;
  const int qi = blockIdx.x;
  const RowGeom g = make_geom(d, m, bmse);
  const double qc = m > 0 ? kQjlConst / double(m) : 0.0;   // m = 0: no sign term
  for (int i = tid; i < d + m; i += nth) (i < d ? sx[i] : sy[i - d]) = xy[size_t(qi) * (d + m) + i];
  __syncthreads();
  const uint32_t total = cnt[qi];
  if (total > uint32_t(kCap)) {
    // the candidate list overflowed: exact scan of every row.  Each thread
    // keeps its best k in local memory; k rounds of a block-wide argmax.
    double best_s[kMaxK];
    int64_t best_i[kMaxK];
    for (int i = 0; i < k; ++i) {
      best_s[i] = -INFINITY;
      best_i[i] = INT64_MAX;
    }
    for (int64_t r = tid; r < n; r += nth) {
      const double sc = exact_score(payload, norms, r, g, c, sx, sy, qc);
      if (first(sc, r, best_s[k - 1], best_i[k - 1])) {
        int p = k - 1;
        while (p > 0 && first(sc, r, best_s[p - 1], best_i[p - 1])) {
          best_s[p] = best_s[p - 1];
          best_i[p] = best_i[p - 1];
          --p;
        }
        best_s[p] = sc;
        best_i[p] = r;
      }
    }
    int head = 0;
    for (int out = 0; out < k; ++out) {
      double sc = head < k ? best_s[head] : -INFINITY;
      int64_t id = head < k ? best_i[head] : INT64_MAX;
      int who = tid;
      for (int o = 16; o; o >>= 1) {
        const double s2 = __shfl_xor_sync(0xFFFFFFFFu, sc, o);
        const int64_t i2 = __shfl_xor_sync(0xFFFFFFFFu, id, o);
        const int w2 = __shfl_xor_sync(0xFFFFFFFFu, who, o);
        if (first(s2, i2, sc, id)) {
          sc = s2;
          id = i2;
          who = w2;
        }
      }
      if ((tid & 31) == 0) {
        rs[tid >> 5] = sc;
        ri[tid >> 5] = id;
        rw[tid >> 5] = who;
      }
      __syncthreads();
      if (tid == 0) {
        for (int w = 1; w < nth / 32; ++w)
          if (first(rs[w], ri[w], rs[0], ri[0])) {
            rs[0] = rs[w];
            ri[0] = ri[w];
            rw[0] = rw[w];
          }
        ids[size_t(qi) * k + out] = ri[0];
        out_scores[size_t(qi) * k + out] = float(rs[0]);
      }
      __syncthreads();
      if (tid == rw[0]) ++head;
      __syncthreads();
    }
    return;
  }
  // 1. the k-th largest approximate score, by bisection over the order keys
  constexpr int kPer = kCap / kFinishThreads;
  const int cn = int(total);
  uint32_t key[kPer];
#pragma unroll
  for (int t = 0; t < kPer; ++t) {
    const int i = tid + t * nth;
    key[t] = i < cn ? order_key(__uint_as_float(cand[size_t(qi) * kCap + i].x)) : 0u;
  }
  const int kk = cn < k ? cn : k;
  uint32_t T = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t trial = T | (1u << bit);
    int ge = 0;
#pragma unroll
    for (int t = 0; t < kPer; ++t) ge += (key[t] >= trial) ? 1 : 0;
    if (block_sum(ge, red) >= kk) T = trial;
  }
  // 2. keep the candidates within 2 E_q of it
  const float cutf = kk > 0 ? key_float(T) - 2.f * qerr[qi] : -INFINITY;
  if (tid == 0) s_mc = 0;
  __syncthreads();
#pragma unroll
  for (int t = 0; t < kPer; ++t) {
    const int i = tid + t * nth;
    if (i < cn && key_float(key[t]) >= cutf) {
      const int slot = atomicAdd(&s_mc, 1);
      sid[slot] = int64_t(cand[size_t(qi) * kCap + i].y);
    }
  }
  __syncthreads();
  const int mc = s_mc;
  // 3. exact scores (one warp per candidate), then (score descending, id ascending)
  for (int i = tid >> 5; i < mc; i += nth >> 5) {
    const double sc = exact_score_warp(payload, norms, sid[i], g, c, sx, sy, qc, tid & 31);
    if ((tid & 31) == 0) ssc[i] = sc;
  }
  int sp2 = 1;
  while (sp2 < mc) sp2 <<= 1;
  for (int i = mc + tid; i < sp2; i += nth) {
    ssc[i] = -INFINITY;
    sid[i] = INT64_MAX;
  }
  __syncthreads();
  for (int size = 2; size <= sp2; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < sp2; i += nth) {
        const int jx = i ^ stride;
        if (jx > i) {
          const bool up = (i & size) == 0;
          const bool i_first = first(ssc[i], sid[i], ssc[jx], sid[jx]);
          if (up ? !i_first : i_first) {
            const double ts = ssc[i];
            ssc[i] = ssc[jx];
            ssc[jx] = ts;
            const int64_t ti = sid[i];
            sid[i] = sid[jx];
            sid[jx] = ti;
          }
        }
      }
      __syncthreads();
    }
  for (int i = tid; i < k; i += nth) {
    ids[size_t(qi) * k + i] = i < mc ? sid[i] : INT64_MAX;
    out_scores[size_t(qi) * k + i] = i < mc ? float(ssc[i]) : -INFINITY;
  }
}

int key_blocks(const tq_ctx* ctx) { return (ctx->d + ctx->m + 63) / 64; }

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

struct SearchWs {
  __half* kw;
  __half* qw;
  float* qerr;
  uint32_t* maxk;
  uint32_t* cnt;
  uint32_t* gkth;
  uint2* cand;
  double* xy;
  size_t kw_bytes, qw_bytes, total;
};

SearchWs search_ws(const tq_ctx* ctx, int64_t nq, int64_t n, void* base) {
  const int kp = 64 * key_blocks(ctx);
  const int64_t n_pad = (n + kRT - 1) / kRT * kRT, nq_pad = (nq + kQT - 1) / kQT * kQT;
  SearchWs w{};
  size_t off = 0;
  uint8_t* b = static_cast<uint8_t*>(base);
  auto take = [&](size_t bytes) {
    uint8_t* p = b ? b + off : nullptr;
    off += align256(bytes);
    return p;
  };
  w.kw_bytes = size_t(n_pad) * kp * 2;
  w.qw_bytes = size_t(nq_pad) * kp * 2;
  w.kw = reinterpret_cast<__half*>(take(w.kw_bytes));
  w.qw = reinterpret_cast<__half*>(take(w.qw_bytes));
  w.qerr = reinterpret_cast<float*>(take(size_t(nq_pad) * 4));
  w.maxk = reinterpret_cast<uint32_t*>(take(8));
  w.cnt = reinterpret_cast<uint32_t*>(take(size_t(nq_pad) * 4));
  w.gkth = reinterpret_cast<uint32_t*>(take(size_t(nq_pad) * 4));
  w.cand = reinterpret_cast<uint2*>(take(size_t(nq) * kCap * 8));
  w.xy = reinterpret_cast<double*>(take(size_t(nq) * (ctx->d + ctx->m) * 8));
  w.total = off;
  return w;
}

template <int KB>
cudaError_t launch_search_kernel(const CUtensorMap& kmap, const __half* qw, int64_t nq, int64_t n,
                                 int64_t qtiles, int64_t row_tiles, int k, const SearchWs& w, uint32_t* status,
                                 cudaStream_t st) {
  using L = SearchSmem;
  static_assert(L::kBytes <= 232448, "shared memory per block");
  static_assert(8 * kSNumBars + 8 <= 256, "barrier area");
  static_assert(32 * KB <= int(kTmemD), "query tile columns");
  auto kern = search_tc_kernel<KB>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(L::kBytes));
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t group = search_group(qtiles, sms);
  const int64_t units = ((qtiles + group - 1) / group) * row_tiles;   // per member of a group
  const int64_t groups = units < sms / group ? units : sms / group;
  const int grid = int(groups * group);
  kern<<<grid, kSearchThreads, L::kBytes, st>>>(kmap, qw, nq, n, qtiles, row_tiles, group, k, w.qerr, w.gkth,
                                                w.cnt, w.cand, status);
  return cudaGetLastError();
}

bool encode_fp16_map(CUtensorMap* map, const void* ptr, int kp, int64_t rows, uint32_t box_rows) {
  const cuuint64_t dims[2] = {cuuint64_t(kp), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(kp) * 2};
  const cuuint32_t box[2] = {64u, box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return get_encode()(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool search_tc_supported(const tq_ctx* ctx, int64_t nq, int64_t n, int k) {
  const int kb = key_blocks(ctx);
  return k >= 1 && k <= kMaxK && kb >= 1 && kb <= 8 && n >= 1 && n < (int64_t(1) << 31) && nq >= 1 &&
         device_is_sm100() && get_encode() != nullptr;
}

size_t search_ws_bytes(const tq_ctx* ctx, int64_t nq, int64_t n) { return search_ws(ctx, nq, n, nullptr).total; }

cudaError_t launch_search_tc(const tq_ctx* ctx, const float* q, int64_t nq, const uint8_t* payload,
                             const uint16_t* norms, int64_t n, int k, int64_t* ids, float* scores, void* ws,
                             cudaStream_t st) {
  const int kb = key_blocks(ctx), kp = 64 * kb;
  const int64_t n_pad = (n + kRT - 1) / kRT * kRT, nq_pad = (nq + kQT - 1) / kQT * kQT;
  const SearchWs w = search_ws(ctx, nq, n, ws);
  cudaError_t e;
  if ((e = cudaMemsetAsync(w.qw, 0, w.qw_bytes, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(w.maxk, 0, 8, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(w.cnt, 0, size_t(nq_pad) * 4, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(w.gkth, 0, size_t(nq_pad) * 4, st)) != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int dec_per_sm = 0;   // resident blocks per SM (one wave of the grid-stride loop)
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&dec_per_sm, decode_rows_kernel, 256, 0);
  if (dec_per_sm < 1) dec_per_sm = 1;
  const int64_t row_blocks = (n_pad + 7) / 8;   // eight warps (rows) per block and pass
  const int64_t dec_blocks = row_blocks < int64_t(sms) * dec_per_sm ? row_blocks : int64_t(sms) * dec_per_sm;
  decode_rows_kernel<<<unsigned(dec_blocks), 256, 0, st>>>(
      payload, norms, n, n_pad, ctx->d, ctx->m, ctx->bmse, kp, ctx->cb, w.kw, w.maxk);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  query_tables_kernel<<<unsigned((nq + kTabQueries - 1) / kTabQueries), 256, 0, st>>>(q, nq, ctx->d, ctx->m,
                                                                                       ctx->dR64, ctx->dP64, w.xy);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  prep_queries_kernel<<<unsigned((nq + 7) / 8), 256, 0, st>>>(w.xy, nq, ctx->d, ctx->m, kp, w.maxk, w.qw, w.qerr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  CUtensorMap kmap;
  if (!encode_fp16_map(&kmap, w.kw, kp, n_pad, kRT)) return cudaErrorInvalidValue;
  const int64_t row_tiles = n_pad / kRT, qtiles = nq_pad / kQT;
  switch (kb) {
    case 1: e = launch_search_kernel<1>(kmap, w.qw, nq, n, qtiles, row_tiles, k, w, ctx->dstatus, st); break;
    case 2: e = launch_search_kernel<2>(kmap, w.qw, nq, n, qtiles, row_tiles, k, w, ctx->dstatus, st); break;
    case 3: e = launch_search_kernel<3>(kmap, w.qw, nq, n, qtiles, row_tiles, k, w, ctx->dstatus, st); break;
    case 4: e = launch_search_kernel<4>(kmap, w.qw, nq, n, qtiles, row_tiles, k, w, ctx->dstatus, st); break;
    case 5: e = launch_search_kernel<5>(kmap, w.qw, nq, n, qtiles, row_tiles, k, w, ctx->dstatus, st); break;
    case 6: e = launch_search_kernel<6>(kmap, w.qw, nq, n, qtiles, row_tiles, k, w, ctx->dstatus, st); break;
    case 7: e = launch_search_kernel<7>(kmap, w.qw, nq, n, qtiles, row_tiles, k, w, ctx->dstatus, st); break;
    default: e = launch_search_kernel<8>(kmap, w.qw, nq, n, qtiles, row_tiles, k, w, ctx->dstatus, st); break;
  }
  if (e != cudaSuccess) return e;
  const size_t fsmem = size_t(2 * 256 + kCap) * 8 + size_t(kCap) * 8;
  cudaFuncSetAttribute(finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(fsmem));
  finish_kernel<<<unsigned(nq), kFinishThreads, fsmem, st>>>(ctx->d, ctx->m, ctx->bmse, k, n, payload, norms, w.xy,
                                                             ctx->dc64, w.qerr, w.cnt, w.cand, ids, scores);
  return cudaGetLastError();
}

}  // namespace tq
