// Decode attention output over a quantised value cache (the value path).
//
// mooersco.com sections 1.2-1.3: the keys set the attention weights through
// the softmax of the logits, the values are summed with those weights, and
// the output is recovered from the compressed values by an estimator.  Values
// are quantised here with the same quantizer as keys (their own context), and
// each value enters through its unbiased reconstruction
//   v_hat = n16 R^T c[idx] + sqrt(pi/2)/m rho16 S^T sigma      (S = P R)
// so for one query head with weights w_s = exp(l_s - max l):
//   o = R^T (a + sqrt(pi/2)/m P^T b) / sum_s w_s,
//   a = sum_s w_s n16_s c[idx_s]   (rotated domain, d),
//   b = sum_s w_s rho16_s sigma_s  (sign domain, m).
// The rotations are applied once per head, after the sums, not once per key.
//
// Partial sums: one block per (batch, KV head, key chunk) computes, for every
// query head of the group, the chunk's maximum logit, the sum of its weights
// and its a, b (flash-decoding style partials), by one of two kernels:
//   attend_mma_kernel (d = m = 128 or m = 0, up to 4 query heads per KV
//     head): fp16 tensor-core MMAs over 16-key steps; each warp takes a
//     contiguous share of the chunk with its own running maximum, and the
//     block merges its eight warps' partials (described above the kernel);
//   attend_partial_kernel (every other shape): key tiles of 128 rows staged
//     in shared memory (prefetched into registers one tile ahead); warp w
//     takes the key pairs (k, k + 64) for k = w, w + 8, ...; lane L decodes
//     one "slot" of the packed layout of both keys (4 coordinates: register
//     r = 4u + i of quarter q, nibbles e = 0..3) and accumulates each head
//     with packed two-wide FMAs over the key pair.
// attend_combine_kernel: one block per query head merges the partials and
// applies P^T and R^T.
#include <cuda_fp16.h>
#include <math.h>

#include "tq_device.cuh"
#include "attend_plan.h"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kAttThreads = 256;
constexpr int kAttWarps = kAttThreads / 32;
constexpr int kAttTile = 128;         // keys per staged tile
constexpr int kAttMaxLd = 8;          // 8-byte words per thread per tile (rows of up to 128 bytes)
constexpr int kAttMaxHeads = 8;
constexpr int kAttStages = 2;         // row tiles in flight per block (cp.async ring)
constexpr int kWStages = 4;           // 16-key steps in flight per warp (tensor-core kernel)

// The slot's 4 codes (r = 4u + i, e = 0..3) as nibbles e of one word, from the
// unit's code halfwords h[0 .. BM-1] (layout in include/tq.h): code e is
// (v >> 4e) & (2^BM - 1).  For b' = 3, register 3's code bits sit in bit 3 of
// the nibbles of h0, h1, h2 and are gathered first.
template <int BM>
__device__ __forceinline__ uint32_t slot_word(const uint32_t (&h)[BM], int i) {
  if constexpr (BM == 1) {
    return (h[0] >> i) & 0x1111u;
  } else if constexpr (BM == 2) {
    return (((i >> 1) ? h[1] : h[0]) >> (2 * (i & 1))) & 0x3333u;
  } else {
    const uint32_t r3 = ((h[0] >> 3) & 0x1111u) | ((h[1] >> 2) & 0x2222u) | ((h[2] >> 1) & 0x4444u);
    return i == 3 ? r3 : ((i == 0 ? h[0] : (i == 1 ? h[1] : h[2])) & 0x7777u);
  }
}

// Partials: part[((grp * nsplit + split) * G + h) * (2 + dp + mp)] = {max, sum, a[dp], b[mp]}.
template <int BM, int GP, int NS>
__global__ void __launch_bounds__(kAttThreads, GP * NS <= 2 ? 3 : (GP * NS <= 4 ? 2 : 1)) attend_partial_kernel(
    const float* __restrict__ logits, int Hq, int Hkv, int64_t S, int64_t chunk, int nsplit,
    const uint8_t* __restrict__ payload, const uint16_t* __restrict__ norms, RowGeom g, CodebookParams cb,
    float* __restrict__ part) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int rb = g.row_bytes;
  uint8_t* srows = sm;                                                        // [kAttTile][rb]
  float* swn = reinterpret_cast<float*>(sm + kAttTile * rb);                  // [kAttTile][GP]  w n16
  float* swr = swn + kAttTile * GP;                                           // [kAttTile][GP]  w rho16
  float* sacc = swr + kAttTile * GP;                                          // [GP][dp + mp]
  float* sred = sacc + GP * (g.dp + g.mp);                                    // [GP][kAttWarps] maxima
  float* smx = sred + GP * kAttWarps;                                         // [GP] chunk maximum
  float* sl = smx + GP;                                                       // [GP] sum of weights
  float* sc = sl + GP;                                                        // [8] codebook

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = Hq / Hkv;
  const int grp = blockIdx.x / nsplit, split = blockIdx.x - grp * nsplit;
  const int b = grp / Hkv, hkv = grp - b * Hkv;
  const int64_t s_begin = int64_t(split) * chunk;
  const int64_t s_end = s_begin + chunk < S ? s_begin + chunk : S;
  const float* lg = logits + (size_t(b) * Hq + size_t(hkv) * G) * S;   // head h at lg + h S
  const uint8_t* rows = payload + (size_t(grp) * S) * rb;
  const uint32_t* nrm = reinterpret_cast<const uint32_t*>(norms) + size_t(grp) * S;

  for (int i = tid; i < GP * (g.dp + g.mp); i += kAttThreads) sacc[i] = 0.f;
  if (tid < 8) sc[tid] = cb.c[tid];
  if (tid < GP) sl[tid] = 0.f;

  // pass 1: the chunk's maximum logit per head
  float mx[GP];
#pragma unroll
  for (int h = 0; h < GP; ++h) mx[h] = -INFINITY;
  // eight independent loads in flight per thread and head
  for (int64_t s = s_begin + tid; s < s_end; s += 8 * kAttThreads) {
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      if (h < G) {
        float v[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const int64_t sx = s + int64_t(x) * kAttThreads;
          v[x] = sx < s_end ? __ldg(lg + size_t(h) * S + sx) : -INFINITY;
        }
#pragma unroll
        for (int x = 0; x < 8; ++x) mx[h] = fmaxf(mx[h], v[x]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    float v = mx[h];
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) sred[h * kAttWarps + warp] = v;
  }
  __syncthreads();
  if (tid < GP) {
    float v = sred[tid * kAttWarps];
    for (int w = 1; w < kAttWarps; ++w) v = fmaxf(v, sred[tid * kAttWarps + w]);
    smx[tid] = v;
  }
  __syncthreads();

  // this lane's slots: code slot t -> quarter, unit, register i; sign slot likewise
  const int nslot_c = g.dp / 4, nslot_s = g.mp / 4;
  int c_off[NS], c_i[NS], c_j[NS], s_off[NS], s_i[NS], s_k[NS];
#pragma unroll
  for (int ns = 0; ns < NS; ++ns) {
    const int t = lane + 32 * ns;
    const int q = t / (4 * g.uq), rem = t - q * 4 * g.uq, u = rem >> 2;
    c_i[ns] = rem & 3;
    c_off[ns] = q * g.per_q + u * BM;                       // halfword index of the unit's codes
    c_j[ns] = q * (g.dp / 4) + 4 * (4 * u + c_i[ns]);       // first coordinate (e = 0)
    const int qs = g.uqm > 0 ? t / (4 * g.uqm) : 0, rs = t - qs * 4 * (g.uqm > 0 ? g.uqm : 1), us = rs >> 2;
    s_i[ns] = rs & 3;
    s_off[ns] = qs * g.per_q + BM * g.uq + us;
    s_k[ns] = qs * (g.mp / 4) + 4 * (4 * us + s_i[ns]);
  }
  // per head and coordinate, two partial sums: keys k (x) and k + kAttTile / 2 (y) of each tile
  float2 accC[NS][GP][4], accS[NS][GP][4];
#pragma unroll
  for (int ns = 0; ns < NS; ++ns)
#pragma unroll
    for (int h = 0; h < GP; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        accC[ns][h][e] = make_float2(0.f, 0.f);
        accS[ns][h][e] = make_float2(0.f, 0.f);
      }
  // weights: thread (key k = tid % kAttTile, head tid / kAttTile + 2 it) of each tile
  constexpr int kWIt = (kAttTile * GP + kAttThreads - 1) / kAttThreads;
  float lsum[kWIt];
#pragma unroll
  for (int it = 0; it < kWIt; ++it) lsum[it] = 0.f;

  // pass 2: tiles of keys, staged one ahead in registers
  const int words = kAttTile * rb / 8;
  uint2 ld[kAttMaxLd];
  float lgv[kWIt];      // logit of this thread's (key, head) pairs in the next tile
  uint32_t nnv[kWIt];   // and the key's norms
  auto fetch = [&](int64_t s0) {
    const int nk = int(s_end - s0 < kAttTile ? s_end - s0 : kAttTile);
    const int nw = nk * rb / 8;
    const uint2* src = reinterpret_cast<const uint2*>(rows + size_t(s0) * rb);
#pragma unroll
    for (int k = 0; k < kAttMaxLd; ++k) {
      const int w = tid + k * kAttThreads;
      ld[k] = (w < nw) ? __ldg(src + w) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int it = 0; it < kWIt; ++it) {
      const int idx = tid + it * kAttThreads;
      const int k = idx % kAttTile, h = idx / kAttTile;
      const bool ok = k < nk && h < G;
      lgv[it] = ok ? __ldg(lg + size_t(h) * S + s0 + k) : 0.f;
      nnv[it] = ok ? __ldg(nrm + s0 + k) : 0u;
    }
  };
  const bool have = s_begin < s_end;
  if (have) fetch(s_begin);
  for (int64_t s0 = s_begin; s0 < s_end; s0 += kAttTile) {
    const int nk = int(s_end - s0 < kAttTile ? s_end - s0 : kAttTile);
    // stage this tile: rows, then the weights w n16 and w rho16 of every (key, head)
#pragma unroll
    for (int k = 0; k < kAttMaxLd; ++k) {
      const int w = tid + k * kAttThreads;
      if (w < words) reinterpret_cast<uint2*>(srows)[w] = ld[k];
    }
#pragma unroll
    for (int it = 0; it < kWIt; ++it) {
      const int idx = tid + it * kAttThreads;
      if (idx < kAttTile * GP) {
        const int k = idx % kAttTile, h = idx / kAttTile;
        float wn = 0.f, wr = 0.f;
        if (k < nk && h < G) {
          const float w = expf(lgv[it] - smx[h]);
          const uint32_t nn = nnv[it];
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&nn));
          wn = w * f.x;
          wr = w * f.y;
          lsum[it] += w;
        }
        // key pairs (kp, kp + kAttTile / 2) side by side: [kp][h][2]
        const int kp = k % (kAttTile / 2), half = k / (kAttTile / 2);
        swn[(kp * GP + h) * 2 + half] = wn;
        swr[(kp * GP + h) * 2 + half] = wr;
      }
    }
    __syncthreads();
    if (s0 + kAttTile < s_end) fetch(s0 + kAttTile);   // next tile in flight during the math
    const int npair = nk < kAttTile / 2 ? nk : kAttTile / 2;   // rows past nk are zero with zero weight
    for (int kp = warp; kp < npair; kp += kAttWarps) {
      const uint16_t* hwA = reinterpret_cast<const uint16_t*>(srows + kp * rb);
      const uint16_t* hwB = reinterpret_cast<const uint16_t*>(srows + (kp + kAttTile / 2) * rb);
      float2 wn2[GP], wr2[GP];
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        wn2[h] = *reinterpret_cast<const float2*>(swn + (kp * GP + h) * 2);
        wr2[h] = *reinterpret_cast<const float2*>(swr + (kp * GP + h) * 2);
      }
#pragma unroll
      for (int ns = 0; ns < NS; ++ns) {
        const int t = lane + 32 * ns;
        if (t < nslot_c) {
          uint32_t ha[BM], hb[BM];
#pragma unroll
          for (int x = 0; x < BM; ++x) {
            ha[x] = hwA[c_off[ns] + x];
            hb[x] = hwB[c_off[ns] + x];
          }
          const uint32_t va = slot_word<BM>(ha, c_i[ns]), vb = slot_word<BM>(hb, c_i[ns]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 cv = make_float2(sc[(va >> (4 * e)) & 7u], sc[(vb >> (4 * e)) & 7u]);
#pragma unroll
            for (int h = 0; h < GP; ++h) accC[ns][h][e] = __ffma2_rn(cv, wn2[h], accC[ns][h][e]);
          }
        }
        if (t < nslot_s) {
          // sign bit 4e + i of the halfword moved to bit 31 and inverted: +1.0f for a set bit, -1.0f otherwise
          const uint32_t sa = hwA[s_off[ns]], sb = hwB[s_off[ns]];
          const int sh0 = 31 - s_i[ns];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t xa = sa << (sh0 - 4 * e), xb = sb << (sh0 - 4 * e);
            const float2 sg = make_float2(__uint_as_float((~xa & 0x80000000u) | 0x3f800000u),
                                          __uint_as_float((~xb & 0x80000000u) | 0x3f800000u));
#pragma unroll
            for (int h = 0; h < GP; ++h) accS[ns][h][e] = __ffma2_rn(sg, wr2[h], accS[ns][h][e]);
          }
        }
      }
    }
    __syncthreads();
  }

  // merge the warps' sums into shared memory, then write the block's partial
#pragma unroll
  for (int ns = 0; ns < NS; ++ns) {
    const int t = lane + 32 * ns;
#pragma unroll
    for (int h = 0; h < GP; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (t < nslot_c) atomicAdd(sacc + h * (g.dp + g.mp) + c_j[ns] + e, accC[ns][h][e].x + accC[ns][h][e].y);
        if (t < nslot_s)
          atomicAdd(sacc + h * (g.dp + g.mp) + g.dp + s_k[ns] + e, accS[ns][h][e].x + accS[ns][h][e].y);
      }
  }
  // every lane of a warp holds the same head in lsum[it] (32 consecutive keys of one head)
#pragma unroll
  for (int it = 0; it < kWIt; ++it) {
    float v = lsum[it];
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int h = (tid + it * kAttThreads) / kAttTile;
    if (lane == 0 && h < GP) atomicAdd(sl + h, v);
  }
  __syncthreads();
  const int rec = 2 + g.dp + g.mp;
  for (int h = 0; h < G; ++h) {
    float* out = part + (size_t(blockIdx.x) * G + h) * rec;
    for (int i = tid; i < g.dp + g.mp; i += kAttThreads) out[2 + i] = sacc[h * (g.dp + g.mp) + i];
    if (tid == 0) {
      out[0] = smx[h];
      out[1] = sl[h];
    }
  }
}

// ---------------------------------------------------------------------------
// Tensor-core partial sums (d = m = 128, up to 4 query heads per KV head).
// The sums contract over keys: for a 16-key step, D[coordinate][column] +=
// A[coordinate][key] B[key][column] with the fp16 m16n8k16 MMA, columns =
// (head, hi / lo limb of the weight).  Thread (g, tig) of a warp builds the A
// operand of unit g of the packed rows (16 coordinates: register i, nibble e)
// for its four keys 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9 of the step:
// codes -> fp16 codebook values by byte permutes over the two byte planes of
// the fp16 levels, then a byte transpose from (key, 4 coordinates) to
// (coordinate, 2 keys); sign bits -> fp16 +-1 by one shift and one
// logic op per register.  Row mapping: m-tile 2 i + (e >> 1), row g + 8 (e & 1).
// B holds the weights w n16 (codes) and w rho16 (signs) of the same keys as
// fp16 hi + lo limbs.  Precision: each product carries the fp16 rounding of
// its codebook level (<= 2^-11 relative) and of the weight's hi + lo split
// (<= 2^-22); sums are fp32.
// Schedule: a warp streams its share of the block's chunk in 16-key steps
// through a private four-stage cp.async ring (rows, logits, norms), with no
// block-wide barrier until the end.  Weights are exp(l - M) against the
// warp's running maximum M per head (flash-decoding's online softmax): when a
// step raises M, the warp's accumulators and weight sum are scaled by
// exp(M_old - M_new) first.  At the end the eight warps' partial sums meet in
// shared memory, each scaled to the block's maximum.
// ---------------------------------------------------------------------------

// fp16 bits of the codebook levels as two byte planes (level v: lo byte v, hi byte v).
struct HalfLut {
  uint32_t lo[2], hi[2];
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte-permute selector of register i (coordinates (i, e = 0..3) in its nibbles)
// from the unit's code halfwords.
template <int BM>
__device__ __forceinline__ uint32_t reg_selector(const uint32_t (&h)[BM], int i) {
  if constexpr (BM == 3) {
    if (i < 3) return h[i] & 0x7777u;
    return ((h[0] >> 3) & 0x1111u) | ((h[1] >> 2) & 0x2222u) | ((h[2] >> 1) & 0x4444u);
  } else if constexpr (BM == 2) {
    return (h[i >> 1] >> (2 * (i & 1))) & 0x3333u;
  } else {
    return (h[0] >> i) & 0x1111u;
  }
}

// Per-warp staging ring of the tensor-core kernel: kWStages 16-key steps, each
// the packed rows (padded stride), the logits of the GP heads and the norms.
template <int BM, bool JL>
struct WarpRing {
  static constexpr int kPerQ = 2 * BM + (JL ? 2 : 0);    // halfwords per quarter chunk (d = m = 128)
  static constexpr int rb = 8 * kPerQ;                    // row bytes (a multiple of 16)
  // row stride: an odd number of 16-byte chunks, so that the rows two apart
  // read by the four lanes of a quad fall in different banks
  static constexpr int rs = (rb / 16) % 2 ? rb : rb + 16;
  static constexpr int kRows = 16 * rs;                   // bytes of one step's rows
  static constexpr int kStep = kRows + 4 * 16 * 4 + 16 * 4;   // + logits [4][16] + norms [16]
  static constexpr int kWarp = kWStages * kStep;
};

template <int BM, bool JL>
__global__ void __launch_bounds__(kAttThreads, 2) attend_mma_kernel(
    const float* __restrict__ logits, int Hq, int Hkv, int64_t S, int64_t chunk, int nsplit,
    const uint8_t* __restrict__ payload, const uint16_t* __restrict__ norms, HalfLut lut,
    float* __restrict__ part) {
  using WR = WarpRing<BM, JL>;
  constexpr int GP = 4;
  constexpr int kPerQ = WR::kPerQ, rb = WR::rb, rs = WR::rs;
  constexpr int kRed = (JL ? 256 : 128) + 4;   // a row of the reduction buffer: a (128), b (128 or none), padding
  constexpr float kL2e = 1.4426950408889634f;
  // b' = 3 with signs: a quarter chunk is 16 bytes (halfwords 0-2 unit 0
  // codes, 3-5 unit 1 codes, 6 / 7 the units' signs); unit g & 1's halfwords
  // come out of one 16-byte load
  constexpr bool kQuad16 = (BM == 3 && JL && rb == 64);
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ float wmax[kAttWarps][GP], wsum[kAttWarps][GP], wfac[kAttWarps][GP];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int G = Hq / Hkv;
  const int grp = blockIdx.x / nsplit, split = blockIdx.x - grp * nsplit;
  const int b = grp / Hkv, hkv = grp - b * Hkv;
  const int64_t s_begin = int64_t(split) * chunk;
  const int64_t s_end = s_begin + chunk < S ? s_begin + chunk : S;
  const float* lg = logits + (size_t(b) * Hq + size_t(hkv) * G) * S;   // head h at lg + h S
  const uint8_t* rows = payload + (size_t(grp) * S) * rb;
  const uint32_t* nrm = reinterpret_cast<const uint32_t*>(norms) + size_t(grp) * S;
  uint8_t* ring = sm + warp * WR::kWarp;

  // this warp's 16-key steps: a contiguous share of the block's chunk
  const int64_t nsteps = s_end > s_begin ? (s_end - s_begin + 15) / 16 : 0;
  const int64_t st0 = nsteps * warp / kAttWarps, st1 = nsteps * (warp + 1) / kAttWarps;

  // step st into its ring stage: rows by 16-byte copies, logits and norms by
  // 4-byte copies; entries past the chunk get logit -inf (weight 0) and keep
  // stale row bytes (finite levels times weight 0)
  auto stage = [&](int64_t st) {
    if (st < st1) {
      uint8_t* dst = ring + int(st % kWStages) * WR::kStep;
      const int64_t s0 = s_begin + 16 * st;
      const int nk = int(s_end - s0 < 16 ? s_end - s0 : 16);
      constexpr int kc = rb / 16;
      for (int c = lane; c < 16 * kc; c += 32) {
        const int r = c / kc, cc = c - r * kc;
        if (r < nk)
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                           uint32_t(__cvta_generic_to_shared(dst + r * rs + 16 * cc))),
                       "l"(rows + size_t(s0 + r) * rb + 16 * cc)
                       : "memory");
      }
      float* sl = reinterpret_cast<float*>(dst + WR::kRows);   // [GP][16]
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int e = lane + 32 * t, h = e >> 4, k = e & 15;
        if (h < G && k < nk)
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(uint32_t(__cvta_generic_to_shared(sl + e))),
                       "l"(lg + size_t(h) * S + s0 + k)
                       : "memory");
        else
          sl[e] = -INFINITY;
      }
      uint32_t* sn = reinterpret_cast<uint32_t*>(dst + WR::kRows + 4 * 16 * 4);   // [16]
      if (lane < 16) {
        if (lane < nk)
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(uint32_t(__cvta_generic_to_shared(sn + lane))),
                       "l"(nrm + s0 + lane)
                       : "memory");
        else
          sn[lane] = 0u;
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");   // one group per step, empty past the range
  };

  // unit g of every row (quarter g >> 1, unit g & 1): code and sign halfwords
  const int code_off = (g >> 1) * kPerQ + (g & 1) * BM;
  const int sign_off = (g >> 1) * kPerQ + 2 * BM + (g & 1);
  // byte-permute selector of the unit's halfwords: (x, y) -> hw 0 or hw 3,
  // (y, z) -> hw 2 or hw 5, (w, w) -> hw 6 or hw 7; with ^ 0x2222,
  // (x, z) -> hw 1 or hw 4 (the upper halves of the results are don't-cares)
  const uint32_t sel_u = (g & 1) ? 0x7676u : 0x1010u;
  // B column g: head hb = g / 2, limb g % 2 of the weight
  const int hb = g >> 1;
  float accC[8][4], accS[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      accC[mt][c] = 0.f;
      accS[mt][c] = 0.f;
    }
  // running maximum of head hb's logits over this warp's keys so far (the
  // accumulators and the weight sum are kept relative to it) and the weight sum
  float mrun = -INFINITY, lsum = 0.f;

#pragma unroll
  for (int j = 0; j < kWStages - 1; ++j) stage(st0 + j);
  for (int64_t st = st0; st < st1; ++st) {
    stage(st + kWStages - 1);   // into the stage the previous step used (all lanes are past it)
    asm volatile("cp.async.wait_group %0;" ::"n"(kWStages - 1) : "memory");
    __syncwarp();
    const uint8_t* srows = ring + int(st % kWStages) * WR::kStep;
    const float* sl = reinterpret_cast<const float*>(srows + WR::kRows) + hb * 16;
    const uint32_t* sn = reinterpret_cast<const uint32_t*>(srows + WR::kRows + 4 * 16 * 4);
    // keys 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9 of the step
    const float2 l01 = *reinterpret_cast<const float2*>(sl + 2 * tig);
    const float2 l89 = *reinterpret_cast<const float2*>(sl + 2 * tig + 8);
    const uint2 n01 = *reinterpret_cast<const uint2*>(sn + 2 * tig);
    const uint2 n89 = *reinterpret_cast<const uint2*>(sn + 2 * tig + 8);
    const float lv[4] = {l01.x, l01.y, l89.x, l89.y};
    const uint32_t nv[4] = {n01.x, n01.y, n89.x, n89.y};
    // the step's maximum of head hb (the 8 lanes of the head), then rescale
    // what was summed against the old maximum if it rose
    float lm = fmaxf(fmaxf(lv[0], lv[1]), fmaxf(lv[2], lv[3]));
    lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 1));
    lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 2));
    lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 4));
    const bool rise = lm > mrun;
    if (__any_sync(0xffffffffu, rise)) {
      const float f = rise ? exp2f((mrun - lm) * kL2e) : 1.f;   // 0 while nothing was summed (mrun = -inf)
      const float fa = __shfl_sync(0xffffffffu, f, 8 * tig);      // lane 8 tig has head tig: this lane's accumulators
      lsum *= f;
      if (rise) mrun = lm;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          accC[mt][c] *= fa;
          if constexpr (JL) accS[mt][c] *= fa;
        }
    }
    // weights exp(l - mrun) times the norms, as this lane's fp16 limb of key pairs
    float wn[4], wr[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float w = lv[x] > -INFINITY ? exp2f((lv[x] - mrun) * kL2e) : 0.f;
      lsum += w;
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&nv[x]));
      wn[x] = w * f.x;
      wr[x] = w * f.y;
    }
    auto limb2 = [&](float a, float c) -> uint32_t {
      const __half2 hi = __floats2half2_rn(a, c);
      const float2 hf = __half22float2(hi);
      const __half2 lo = __floats2half2_rn(a - hf.x, c - hf.y);
      const __half2 r = (g & 1) ? lo : hi;
      return *reinterpret_cast<const uint32_t*>(&r);
    };
    const uint32_t bC0 = limb2(wn[0], wn[1]), bC1 = limb2(wn[2], wn[3]);
    const int kk[4] = {2 * tig, 2 * tig + 1, 2 * tig + 8, 2 * tig + 9};
    uint32_t hc[4][BM];
    uint32_t hsg[4];
    if constexpr (kQuad16) {
      // one 16-byte load of the key's quarter chunk; this thread's unit's
      // halfwords picked by byte permutes (upper halves are don't-cares for
      // the code selectors, zero for the sign halfword)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const uint4 rw = *reinterpret_cast<const uint4*>(srows + kk[x] * rs + (g >> 1) * 16);
        hc[x][0] = prmt(rw.x, rw.y, sel_u);
        hc[x][1] = prmt(rw.x, rw.z, sel_u ^ 0x2222u);
        hc[x][2] = prmt(rw.y, rw.z, sel_u);
        hsg[x] = prmt(rw.w, rw.w, sel_u);
      }
    } else {
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const uint16_t* hw = reinterpret_cast<const uint16_t*>(srows + kk[x] * rs);
#pragma unroll
        for (int y = 0; y < BM; ++y) hc[x][y] = hw[code_off + y];
        if constexpr (JL) hsg[x] = hw[sign_off];
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t lo[4], hi[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const uint32_t sel = reg_selector<BM>(hc[x], i);
        lo[x] = prmt(lut.lo[0], lut.lo[1], sel);
        hi[x] = prmt(lut.hi[0], lut.hi[1], sel);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // bytes (key a, e = 2h), (key b, 2h), (a, 2h + 1), (b, 2h + 1) of each plane
        const uint32_t ps = h ? 0x7362u : 0x5140u;
        const uint32_t p01 = prmt(lo[0], lo[1], ps), q01 = prmt(hi[0], hi[1], ps);
        const uint32_t p23 = prmt(lo[2], lo[3], ps), q23 = prmt(hi[2], hi[3], ps);
        // fp16 pairs: row g (e = 2h) and row g + 8 (e = 2h + 1), keys (2 tig, 2 tig + 1) / (+8, +9)
        const uint32_t a0 = prmt(p01, q01, 0x5140u), a1 = prmt(p01, q01, 0x7362u);
        const uint32_t a2 = prmt(p23, q23, 0x5140u), a3 = prmt(p23, q23, 0x7362u);
        mma_16816(accC[2 * i + h], a0, a1, a2, a3, bC0, bC1);
      }
    }
    if constexpr (JL) {
      const uint32_t bS0 = limb2(wr[0], wr[1]), bS1 = limb2(wr[2], wr[3]);
      // inverted sign bits of a key pair in the two halves: bit 4e + i of the
      // halfword goes to bit 15 (key a) and bit 31 (key b) after a left shift
      // by 15 - 4e - i; set means -1 (fp16 sign bit) over 1.0 (0x3C00)
      const uint32_t w01 = ~prmt(hsg[0], hsg[1], 0x5410u), w23 = ~prmt(hsg[2], hsg[3], 0x5410u);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int e0 = 2 * h, e1 = 2 * h + 1;
          const uint32_t a0 = ((w01 << (15 - 4 * e0 - i)) & 0x80008000u) | 0x3C003C00u;
          const uint32_t a1 = ((w01 << (15 - 4 * e1 - i)) & 0x80008000u) | 0x3C003C00u;
          const uint32_t a2 = ((w23 << (15 - 4 * e0 - i)) & 0x80008000u) | 0x3C003C00u;
          const uint32_t a3 = ((w23 << (15 - 4 * e1 - i)) & 0x80008000u) | 0x3C003C00u;
          mma_16816(accS[2 * i + h], a0, a1, a2, a3, bS0, bS1);
        }
    }
    __syncwarp();   // every lane is done with this stage before it is refilled
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  // head hb's weight sum over this warp's keys: the lanes of one limb cover
  // the step's keys once (the two limb lanes computed the same weights)
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
  if (tig == 0 && (g & 1) == 0) {
    wmax[warp][hb] = mrun;
    wsum[warp][hb] = lsum;
  }
  __syncthreads();   // every warp is done with its ring: the reduction buffer reuses it

  // the warps' accumulators meet in shared memory: warp w writes its sums for
  // head tig to red[w][tig][.], relative to its own maximum; the block's
  // record takes them relative to the block's maximum
  static_assert(kAttWarps * GP * kRed * 4 <= kAttWarps * WR::kWarp, "reduction buffer");
  float* red = reinterpret_cast<float*>(sm);
  {
    // the rows of this thread's accumulators: unit g, register i, nibble e; head tig
    float* rw = red + (warp * GP + tig) * kRed;
    const int q = g >> 1, u = g & 1;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j0 = q * 32 + 4 * (4 * u + i) + 2 * h;   // e = 2h (row g) and 2h + 1 (row g + 8)
        *reinterpret_cast<float2*>(rw + j0) =
            make_float2(accC[2 * i + h][0] + accC[2 * i + h][1], accC[2 * i + h][2] + accC[2 * i + h][3]);
        if constexpr (JL)
          *reinterpret_cast<float2*>(rw + 128 + j0) =
              make_float2(accS[2 * i + h][0] + accS[2 * i + h][1], accS[2 * i + h][2] + accS[2 * i + h][3]);
      }
  }
  if (tid < kAttWarps * GP) {
    const int w = tid / GP, h = tid - w * GP;
    float M = wmax[0][h];
    for (int v = 1; v < kAttWarps; ++v) M = fmaxf(M, wmax[v][h]);
    wfac[w][h] = wmax[w][h] == -INFINITY ? 0.f : exp2f((wmax[w][h] - M) * kL2e);
  }
  __syncthreads();
  // partial record {max, sum, a[128], b[128 or 0]} in the generic layout (dp + mp slots)
  constexpr int rec = 2 + 128 + (JL ? 128 : 0);
  for (int o = tid; o < G * (rec - 2); o += kAttThreads) {
    const int h = o / (rec - 2), j = o - h * (rec - 2);
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kAttWarps; ++w) v = fmaf(wfac[w][h], red[(w * GP + h) * kRed + j], v);
    part[(size_t(blockIdx.x) * G + h) * rec + 2 + j] = v;
  }
  if (tid < G) {
    float M = wmax[0][tid], L = 0.f;
    for (int w = 1; w < kAttWarps; ++w) M = fmaxf(M, wmax[w][tid]);
    for (int w = 0; w < kAttWarps; ++w) L = fmaf(wfac[w][tid], wsum[w][tid], L);
    float* out = part + (size_t(blockIdx.x) * G + tid) * rec;
    out[0] = M;
    out[1] = L;
  }
  // the merge kernel may be scheduled once every block has written its record
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// sum over k in [k0, k1) of M[k][j] v[k], M row-major with rows of length d
// (threads of consecutive j read consecutive addresses): sixteen loads are
// issued before their products, four accumulators.
__device__ __forceinline__ float colsum(const float* __restrict__ M, int d, int j, const float* v, int k0, int k1) {
  float t[4] = {0.f, 0.f, 0.f, 0.f};
  int k = k0;
  for (; k + 16 <= k1; k += 16) {
    float mv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) mv[u] = __ldg(M + size_t(k + u) * d + j);
#pragma unroll
    for (int u = 0; u < 16; ++u) t[u & 3] = fmaf(mv[u], v[k + u], t[u & 3]);
  }
  for (; k < k1; ++k) t[0] = fmaf(__ldg(M + size_t(k) * d + j), v[k], t[0]);
  return (t[0] + t[1]) + (t[2] + t[3]);
}

// One block per query head: merge the chunk partials, then
// o = R^T (a + sqrt(pi/2)/m P^T b) / L.
__global__ void __launch_bounds__(256) attend_combine_kernel(const float* __restrict__ part, int Hq, int Hkv,
                                                             int nsplit, const float* __restrict__ R,
                                                             const float* __restrict__ P, int d, int m, RowGeom g,
                                                             float* __restrict__ out) {
  // launched as a programmatic dependent of the partial sums: wait for their records
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ float sv[];
  float* sa = sv;          // [dp] merged a, then u
  float* sb = sa + g.dp;   // [mp] merged b
  __shared__ float sf[kAttMaxSplits];   // per-split factors exp(m_i - M)
  __shared__ float sL;
  const int bh = blockIdx.x, b = bh / Hq, h = bh - b * Hq;
  const int G = Hq / Hkv, hkv = h / G, hl = h - hkv * G;
  const int grp = b * Hkv + hkv;
  const int rec = 2 + g.dp + g.mp;
  const float* p0 = part + (size_t(grp) * nsplit * G + hl) * rec;   // split i at p0 + i G rec
  // M = max_i m_i and L = sum_i exp(m_i - M) l_i over the splits, in parallel
  __shared__ float sr[8];
  float mloc = -INFINITY;
  for (int i = threadIdx.x; i < nsplit; i += blockDim.x) mloc = fmaxf(mloc, p0[size_t(i) * G * rec]);
  for (int o = 16; o; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
  if ((threadIdx.x & 31) == 0) sr[threadIdx.x >> 5] = mloc;
  __syncthreads();
  float M = sr[0];
  for (int w = 1; w < int(blockDim.x >> 5); ++w) M = fmaxf(M, sr[w]);
  __syncthreads();
  float lloc = 0.f;
  for (int i = threadIdx.x; i < nsplit; i += blockDim.x) {
    const float mi = p0[size_t(i) * G * rec];
    const float f = (M == -INFINITY || mi == -INFINITY) ? 0.f : expf(mi - M);
    sf[i] = f;
    lloc = fmaf(f, p0[size_t(i) * G * rec + 1], lloc);
  }
  for (int o = 16; o; o >>= 1) lloc += __shfl_xor_sync(0xffffffffu, lloc, o);
  if ((threadIdx.x & 31) == 0) sr[threadIdx.x >> 5] = lloc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float L = 0.f;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) L += sr[w];
    sL = L;
  }
  __syncthreads();
  const float L = sL;
  for (int j = threadIdx.x; j < g.dp + g.mp; j += blockDim.x) {
    float acc = 0.f;
#pragma unroll 4
    for (int i = 0; i < nsplit; ++i) acc = fmaf(sf[i], p0[size_t(i) * G * rec + 2 + j], acc);
    sv[j] = acc;
  }
  __syncthreads();
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const float qc = m > 0 ? float(kQjlConst) / float(m) : 0.f;
  // the two products run two threads per output when d <= 128 (each half of
  // the sum); each thread loads 16 matrix entries before it multiplies, so
  // that the L2 latency is paid once per 16 terms
  __shared__ float sp[2][256];
  const int nh = 2 * d <= int(blockDim.x) ? 2 : 1;
  const int jt = int(threadIdx.x) % d, ht = int(threadIdx.x) / d;
  if (ht < nh) sp[ht][jt] = colsum(P, d, jt, sb, m * ht / nh, m * (ht + 1) / nh);   // (P^T b)_j, part ht
  __syncthreads();
  float u_own = 0.f;
  if (threadIdx.x < d) {
    const int j = threadIdx.x;
    const float t = nh == 2 ? sp[0][j] + sp[1][j] : sp[0][j];
    u_own = (sa[j] + qc * t) * inv;
  }
  __syncthreads();
  if (threadIdx.x < d) sa[threadIdx.x] = u_own;
  __syncthreads();
  if (ht < nh) sp[ht][jt] = colsum(R, d, jt, sa, d * ht / nh, d * (ht + 1) / nh);   // (R^T u)_i, part ht
  __syncthreads();
  if (threadIdx.x < d) out[size_t(bh) * d + threadIdx.x] = nh == 2 ? sp[0][threadIdx.x] + sp[1][threadIdx.x]
                                                                 : sp[0][threadIdx.x];
}

// Key chunks per (batch, KV head): att_plan_for in attend_plan.h, with this
// device's SM count.
AttPlan att_plan(int B, int Hkv, int64_t S, bool mma) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return att_plan_for(B, Hkv, S, mma, sms, kAttTile);
}

// The tensor-core kernel serves d = m = 128 (or m = 0) with up to 4 query
// heads per KV head.
bool attend_uses_mma(const tq_ctx* ctx, int Hq, int Hkv) {
  return ctx->d == 128 && (ctx->m == 128 || ctx->m == 0) && Hq / Hkv <= 4;
}

template <int BM, int GP, int NS>
cudaError_t launch_partial(const tq_ctx* ctx, const float* logits, int B, int Hq, int Hkv, int64_t S, AttPlan ap,
                           const uint8_t* payload, const uint16_t* norms, float* part, cudaStream_t st) {
  const RowGeom g = make_geom(ctx->d, ctx->m, ctx->bmse);
  const size_t smem = size_t(kAttTile) * g.row_bytes + size_t(2 * kAttTile * GP) * 4 +
                      size_t(GP) * (g.dp + g.mp) * 4 + size_t(GP * kAttWarps + 2 * GP + 8) * 4;
  auto kern = attend_partial_kernel<BM, GP, NS>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  kern<<<unsigned(int64_t(B) * Hkv * ap.nsplit), kAttThreads, smem, st>>>(logits, Hq, Hkv, S, ap.chunk, ap.nsplit,
                                                                          payload, norms, g, ctx->cb, part);
  return cudaGetLastError();
}

template <int BM, int NS>
cudaError_t dispatch_heads(const tq_ctx* ctx, const float* logits, int B, int Hq, int Hkv, int64_t S, AttPlan ap,
                           const uint8_t* payload, const uint16_t* norms, float* part, cudaStream_t st) {
  const int G = Hq / Hkv;
  if (G <= 2) return launch_partial<BM, 2, NS>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st);
  if (G <= 4) return launch_partial<BM, 4, NS>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st);
  return launch_partial<BM, 8, NS>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st);
}

template <int BM, bool JL>
cudaError_t launch_mma_partial(const tq_ctx* ctx, const float* logits, int B, int Hq, int Hkv, int64_t S,
                               AttPlan ap, const uint8_t* payload, const uint16_t* norms, float* part,
                               cudaStream_t st) {
  HalfLut lut{};
  for (int v = 0; v < ctx->levels; ++v) {
    const uint16_t bits = __half_as_ushort(__double2half(ctx->c[v]));
    lut.lo[v / 4] |= uint32_t(bits & 0xFF) << (8 * (v % 4));
    lut.hi[v / 4] |= uint32_t(bits >> 8) << (8 * (v % 4));
  }
  const size_t smem = size_t(kAttWarps) * WarpRing<BM, JL>::kWarp;   // the warps' rings (then the reduction buffer)
  auto kern = attend_mma_kernel<BM, JL>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  kern<<<unsigned(int64_t(B) * Hkv * ap.nsplit), kAttThreads, smem, st>>>(logits, Hq, Hkv, S, ap.chunk, ap.nsplit,
                                                                          payload, norms, lut, part);
  return cudaGetLastError();
}

template <int NS>
cudaError_t dispatch_bits(const tq_ctx* ctx, const float* logits, int B, int Hq, int Hkv, int64_t S, AttPlan ap,
                          const uint8_t* payload, const uint16_t* norms, float* part, cudaStream_t st) {
  switch (ctx->bmse) {
    case 1: return dispatch_heads<1, NS>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st);
    case 2: return dispatch_heads<2, NS>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st);
    default: return dispatch_heads<3, NS>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st);
  }
}

}  // namespace

bool attend_supported(const tq_ctx* ctx, int Hq, int Hkv) {
  return Hq / Hkv <= kAttMaxHeads && ctx->bmse >= 1 && ctx->bmse <= 3 && ctx->d <= 256 && ctx->m <= 256;
}

size_t attend_ws_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int64_t S) {
  const AttPlan ap = att_plan(B, Hkv, S, attend_uses_mma(ctx, Hq, Hkv));
  const RowGeom g = make_geom(ctx->d, ctx->m, ctx->bmse);
  const size_t rec = size_t(2 + g.dp + g.mp);
  const size_t bytes = size_t(B) * Hkv * ap.nsplit * size_t(Hq / Hkv) * rec * 4;
  return (bytes + 255) / 256 * 256;
}

cudaError_t launch_attend(const tq_ctx* ctx, const float* logits, int B, int Hq, int Hkv, int64_t S,
                          const uint8_t* payload, const uint16_t* norms, float* out, void* ws, cudaStream_t st) {
  const AttPlan ap = att_plan(B, Hkv, S, attend_uses_mma(ctx, Hq, Hkv));
  const RowGeom g = make_geom(ctx->d, ctx->m, ctx->bmse);
  float* part = static_cast<float*>(ws);
  const bool two = g.dp > 128 || g.mp > 128;
  cudaError_t e;
  if (attend_uses_mma(ctx, Hq, Hkv)) {
    // tensor-core partial sums
    switch (ctx->bmse * 2 + (ctx->m > 0 ? 1 : 0)) {
      case 2: e = launch_mma_partial<1, false>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st); break;
      case 3: e = launch_mma_partial<1, true>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st); break;
      case 4: e = launch_mma_partial<2, false>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st); break;
      case 5: e = launch_mma_partial<2, true>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st); break;
      case 6: e = launch_mma_partial<3, false>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st); break;
      default: e = launch_mma_partial<3, true>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st); break;
    }
  } else {
    e = two ? dispatch_bits<2>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st)
            : dispatch_bits<1>(ctx, logits, B, Hq, Hkv, S, ap, payload, norms, part, st);
  }
  if (e != cudaSuccess) return e;
  // the merge overlaps its launch with the end of the partial sums
  // (programmatic dependent launch; it waits for their completion first)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(B * Hq));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = size_t(g.dp + g.mp) * 4;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attend_combine_kernel, static_cast<const float*>(part), Hq, Hkv, ap.nsplit,
                            static_cast<const float*>(ctx->dR), static_cast<const float*>(ctx->dP), ctx->d, ctx->m, g,
                            out);
}

}  // namespace tq
