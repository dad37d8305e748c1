// Decode attention logits against the packed cache: the TurboQuant
// inner-product estimator (airosetta.com "Google TurboQuant", stage 2)
//   s = n16 sum_j c[idx_j] (R q)_j + sqrt(pi/2)/m rho16 sum_i sigma_i (S q)_i
// for every (query head, key) of a GQA decode step.  The work is HBM bound
// (mooersco.com section 2.2): 4 query heads share each key of a KV head.
//
// Fast path (d = m = 128, b' = 1..3, this file's logits_mma_kernel):
//   * one warp streams 16-key tiles; thread (g, tig) loads chunk tig of keys
//     g and g + 8 with coalesced 32/128-bit loads (the packed layout puts a
//     quarter of every key's codes and signs in one contiguous chunk);
//   * codes are expanded to int8 MMA fragments with byte permutes: a 3-bit
//     code nibble indexes an 8-entry byte table holding one byte plane of the
//     int16 fixed-point codebook (two planes, hi and lo); sign bits index a
//     two-entry table {-1, +1};
//   * the products with the 4 query heads (two int8 limbs of an int16
//     fixed-point Rq / Sq each) run on the int8 tensor-core MMA
//     m16n8k32 with exact int32 accumulation;
//   * the epilogue combines limbs in fp32, applies the two norms and writes
//     the logits (fp32, [B, Hq, S]).
// Query preparation (Rq, Sq = P (Rq), int16 split, fragment order) is a
// separate small kernel writing to the caller's workspace.
#include <cuda_fp16.h>

#include <algorithm>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int D = 128;          // head dimension of the fast path (d = m)
constexpr int KS = D / 32;      // MMA k-steps
constexpr int HPT = 4;          // heads per N-tile of the MMA (2 limbs each)
constexpr int kLogitThreads = 256;

// Workspace for one (batch, kv head) group and one N-tile: B fragments of the
// code term (x = R q) and of the sign term (y = S q): [2][KS][2][32] uint32.
constexpr int kFragWords = 2 * KS * 2 * 32;

struct HeadScale {
  float code;   // multiplies the int32 code dot product
  float sign;   // multiplies the int32 sign dot product
};

// ---------------------------------------------------------------------------
// Query preparation: x = R q, y = P x (= S q), int16 fixed point per head,
// split into two signed int8 limbs, written in MMA B-fragment order.
// One block per (batch, kv head, head slot); slots >= G write zeros.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) qprep_kernel(const float* __restrict__ q, int Hq, int Hkv, int nt_per_group,
                                                    const float* __restrict__ Rt, const float* __restrict__ Pt,
                                                    float code_inv_scale, float scale, float qjl_over_m,
                                                    uint32_t* __restrict__ frags, HeadScale* __restrict__ hscale) {
  __shared__ float sq[D], sx[D], sy[D];
  __shared__ int8_t limbs[2][2][D];     // [x/y][hi/lo][coordinate]
  __shared__ float red[2][4];
  const int G = Hq / Hkv;
  const int slots = nt_per_group * HPT;
  const int blk = blockIdx.x;
  const int slot = blk % slots, grp = blk / slots;      // grp = b * Hkv + hkv
  const int b = grp / Hkv, hkv = grp % Hkv;
  const bool live = slot < G;
  const int h = hkv * G + slot;
  const int tid = threadIdx.x;
  sq[tid] = live ? q[(size_t(b) * Hq + h) * D + tid] : 0.f;
  __syncthreads();
  float x = 0.f;
  for (int i = 0; i < D; ++i) x = fmaf(Rt[i * D + tid], sq[i], x);
  sx[tid] = x;
  __syncthreads();
  float y = 0.f;
  for (int j = 0; j < D; ++j) y = fmaf(Pt[j * D + tid], sx[j], y);
  sy[tid] = y;
  float ax = fabsf(x), ay = fabsf(y);
  for (int o = 16; o; o >>= 1) {
    ax = fmaxf(ax, __shfl_xor_sync(0xffffffffu, ax, o));
    ay = fmaxf(ay, __shfl_xor_sync(0xffffffffu, ay, o));
  }
  if ((tid & 31) == 0) {
    red[0][tid >> 5] = ax;
    red[1][tid >> 5] = ay;
  }
  __syncthreads();
  const float mx = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
  const float my = fmaxf(fmaxf(red[1][0], red[1][1]), fmaxf(red[1][2], red[1][3]));
  const float kx = mx > 0.f ? 32000.f / mx : 0.f;
  const float ky = my > 0.f ? 32000.f / my : 0.f;
  const int xi = __float2int_rn(sx[tid] * kx);
  const int yi = __float2int_rn(sy[tid] * ky);
  const int xh = (xi + 128) >> 8, yh = (yi + 128) >> 8;
  limbs[0][0][tid] = int8_t(xh);
  limbs[0][1][tid] = int8_t(xi - 256 * xh);
  limbs[1][0][tid] = int8_t(yh);
  limbs[1][1][tid] = int8_t(yi - 256 * yh);
  if (tid == 0 && live) {
    hscale[size_t(b) * Hq + h].code = mx > 0.f ? scale * code_inv_scale / kx : 0.f;
    hscale[size_t(b) * Hq + h].sign = my > 0.f ? scale * qjl_over_m / ky : 0.f;
  }
  __syncthreads();
  // Fragment words of this head: lanes L with L/4 = 2 (slot % 4) + limb.
  // Word (xy, s, reg, lane) holds B[k = 16 reg + 4 tig + e][n = L/4], e = 0..3,
  // with K position k of step s mapped to coordinate tig * D/4 + 4 (2s + reg) + e.
  const int nt = slot / HPT, col = slot % HPT;
  uint32_t* fr = frags + (size_t(grp) * nt_per_group + nt) * kFragWords;
  {
    const int w = tid;                      // 128 words per head: [xy][s][reg][limb][tig]
    const int tig = w & 3, limb = (w >> 2) & 1, reg = (w >> 3) & 1, s = (w >> 4) & 3, xy = (w >> 6) & 1;
    const int lane = (2 * col + limb) * 4 + tig;
    uint32_t word = 0;
    for (int e = 0; e < 4; ++e) {
      const int j = tig * (D / 4) + 4 * (2 * s + reg) + e;
      word |= uint32_t(uint8_t(limbs[xy][limb][j])) << (8 * e);
    }
    fr[((xy * KS + s) * 2 + reg) * 32 + lane] = word;
  }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Chunk of one key for one quarter: BMSE * 2 halfwords of codes (two units)
// and 2 halfwords of signs, as 32-bit words.
template <int BMSE>
struct Chunk {
  static constexpr int kWords = BMSE + 1;
  uint32_t w[kWords];
};

template <int BMSE>
__device__ __forceinline__ void load_chunk(Chunk<BMSE>& c, const uint8_t* row, int tig, bool ok) {
  const uint32_t* p = reinterpret_cast<const uint32_t*>(row + tig * 4 * (BMSE + 1));
  if constexpr (BMSE == 3) {
    uint4 v = ok ? __ldg(reinterpret_cast<const uint4*>(p)) : make_uint4(0, 0, 0, 0);
    c.w[0] = v.x;
    c.w[1] = v.y;
    c.w[2] = v.z;
    c.w[3] = v.w;
  } else if constexpr (BMSE == 1) {
    uint2 v = ok ? __ldg(reinterpret_cast<const uint2*>(p)) : make_uint2(0, 0);
    c.w[0] = v.x;
    c.w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < BMSE + 1; ++i) c.w[i] = ok ? __ldg(p + i) : 0u;
  }
}

// Halfword h of the chunk (h = 0 .. 2 BMSE + 1) in the low 16 bits.
template <int BMSE>
__device__ __forceinline__ uint32_t chunk_half(const Chunk<BMSE>& c, int h) {
  return (h & 1) ? (c.w[h >> 1] >> 16) : c.w[h >> 1];
}

// Byte-permute selectors (4 nibbles, mode bit clear) for the 8 registers of a
// quarter: codes of register r, nibble e = coordinate (r, e).
template <int BMSE>
__device__ __forceinline__ void code_selectors(const Chunk<BMSE>& c, uint32_t (&sel)[8]) {
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    if constexpr (BMSE == 3) {
      const uint32_t h0 = chunk_half(c, 3 * u), h1 = chunk_half(c, 3 * u + 1), h2 = chunk_half(c, 3 * u + 2);
      sel[4 * u + 0] = h0 & 0x7777u;
      sel[4 * u + 1] = h1 & 0x7777u;
      sel[4 * u + 2] = h2 & 0x7777u;
      sel[4 * u + 3] = ((h0 >> 3) & 0x1111u) | ((h1 >> 2) & 0x2222u) | ((h2 >> 1) & 0x4444u);
    } else if constexpr (BMSE == 2) {
      const uint32_t h0 = chunk_half(c, 2 * u), h1 = chunk_half(c, 2 * u + 1);
      sel[4 * u + 0] = h0 & 0x3333u;
      sel[4 * u + 1] = (h0 >> 2) & 0x3333u;
      sel[4 * u + 2] = h1 & 0x3333u;
      sel[4 * u + 3] = (h1 >> 2) & 0x3333u;
    } else {
      const uint32_t h0 = chunk_half(c, u);
      sel[4 * u + 0] = h0 & 0x1111u;
      sel[4 * u + 1] = (h0 >> 1) & 0x1111u;
      sel[4 * u + 2] = (h0 >> 2) & 0x1111u;
      sel[4 * u + 3] = (h0 >> 3) & 0x1111u;
    }
  }
}

// Sign selectors for the 8 registers: one bit per nibble.
template <int BMSE>
__device__ __forceinline__ void sign_selectors(const Chunk<BMSE>& c, uint32_t (&sel)[8]) {
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const uint32_t h = chunk_half(c, 2 * BMSE + u);
#pragma unroll
    for (int i = 0; i < 4; ++i) sel[4 * u + i] = (h >> i) & 0x1111u;
  }
}

template <int BMSE, int NT>
__global__ void __launch_bounds__(kLogitThreads) logits_mma_kernel(
    const uint8_t* __restrict__ payload, const uint16_t* __restrict__ norms, int64_t S, int Hq, int Hkv,
    int64_t total_tiles, const uint32_t* __restrict__ frags, const HeadScale* __restrict__ hscale, CodeLut lut,
    float* __restrict__ out) {
  constexpr int kRowBytes = D * BMSE / 8 + D / 8;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int64_t nwarps = int64_t(gridDim.x) * (kLogitThreads / 32);
  const int64_t gw = int64_t(blockIdx.x) * (kLogitThreads / 32) + (threadIdx.x >> 5);
  const int64_t t_begin = gw * total_tiles / nwarps, t_end = (gw + 1) * total_tiles / nwarps;
  if (t_begin >= t_end) return;
  const int G = Hq / Hkv;
  const int64_t tpp = (S + 15) / 16;

  uint32_t bx[NT][KS][2], by[NT][KS][2];
  float sc_code[NT], sc_sign[NT];
  int64_t cur_grp = -1;

  for (int64_t t = t_begin; t < t_end; ++t) {
    const int64_t grp = t / tpp;
    const int64_t s0 = (t - grp * tpp) * 16;
    if (grp != cur_grp) {
      cur_grp = grp;
      const int b = int(grp / Hkv), hkv = int(grp % Hkv);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t* fr = frags + (size_t(grp) * NT + nt) * kFragWords;
#pragma unroll
        for (int s = 0; s < KS; ++s)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            bx[nt][s][r] = __ldg(fr + ((0 * KS + s) * 2 + r) * 32 + lane);
            by[nt][s][r] = __ldg(fr + ((1 * KS + s) * 2 + r) * 32 + lane);
          }
        const int hg = nt * HPT + tig;
        if (hg < G) {
          const HeadScale hs = hscale[size_t(b) * Hq + hkv * G + hg];
          sc_code[nt] = hs.code;
          sc_sign[nt] = hs.sign;
        } else {
          sc_code[nt] = 0.f;
          sc_sign[nt] = 0.f;
        }
      }
    }
    const int64_t rowA = grp * S + s0 + g, rowB = rowA + 8;
    const bool okA = s0 + g < S, okB = s0 + g + 8 < S;
    Chunk<BMSE> ca, cb;
    load_chunk<BMSE>(ca, payload + rowA * kRowBytes, tig, okA);
    load_chunk<BMSE>(cb, payload + rowB * kRowBytes, tig, okB);
    const uint32_t na = okA ? __ldg(reinterpret_cast<const uint32_t*>(norms) + rowA) : 0u;
    const uint32_t nb = okB ? __ldg(reinterpret_cast<const uint32_t*>(norms) + rowB) : 0u;

    uint32_t sa[8], sb[8];
    int acc_hi[NT][4], acc_lo[NT][4], acc_sg[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc_hi[nt][i] = acc_lo[nt][i] = acc_sg[nt][i] = 0;

    code_selectors<BMSE>(ca, sa);
    code_selectors<BMSE>(cb, sb);
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      const uint32_t ah0 = prmt(lut.hi[0], lut.hi[1], sa[2 * s]), ah1 = prmt(lut.hi[0], lut.hi[1], sb[2 * s]);
      const uint32_t ah2 = prmt(lut.hi[0], lut.hi[1], sa[2 * s + 1]),
                     ah3 = prmt(lut.hi[0], lut.hi[1], sb[2 * s + 1]);
      const uint32_t al0 = prmt(lut.lo[0], lut.lo[1], sa[2 * s]), al1 = prmt(lut.lo[0], lut.lo[1], sb[2 * s]);
      const uint32_t al2 = prmt(lut.lo[0], lut.lo[1], sa[2 * s + 1]),
                     al3 = prmt(lut.lo[0], lut.lo[1], sb[2 * s + 1]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_s8(acc_hi[nt], ah0, ah1, ah2, ah3, bx[nt][s][0], bx[nt][s][1]);
        mma_s8(acc_lo[nt], al0, al1, al2, al3, bx[nt][s][0], bx[nt][s][1]);
      }
    }
    sign_selectors<BMSE>(ca, sa);
    sign_selectors<BMSE>(cb, sb);
    constexpr uint32_t kSignLut = 0x000001FFu;   // byte 0 = -1, byte 1 = +1
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      const uint32_t a0 = prmt(kSignLut, 0u, sa[2 * s]), a1 = prmt(kSignLut, 0u, sb[2 * s]);
      const uint32_t a2 = prmt(kSignLut, 0u, sa[2 * s + 1]), a3 = prmt(kSignLut, 0u, sb[2 * s + 1]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_s8(acc_sg[nt], a0, a1, a2, a3, by[nt][s][0], by[nt][s][1]);
    }
    // epilogue: C[row][2 tig + limb] -> head tig of each N-tile
    const float kna = __half2float(__ushort_as_half(uint16_t(na))), kra = __half2float(__ushort_as_half(uint16_t(na >> 16)));
    const float knb = __half2float(__ushort_as_half(uint16_t(nb))), krb = __half2float(__ushort_as_half(uint16_t(nb >> 16)));
    const int b = int(grp / Hkv), hkv = int(grp % Hkv);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hg = nt * HPT + tig;
      if (hg >= G) continue;
      const float codeA = float(acc_hi[nt][0]) * 65536.f + float(acc_hi[nt][1] + acc_lo[nt][0]) * 256.f +
                          float(acc_lo[nt][1]);
      const float codeB = float(acc_hi[nt][2]) * 65536.f + float(acc_hi[nt][3] + acc_lo[nt][2]) * 256.f +
                          float(acc_lo[nt][3]);
      const float signA = float(acc_sg[nt][0]) * 256.f + float(acc_sg[nt][1]);
      const float signB = float(acc_sg[nt][2]) * 256.f + float(acc_sg[nt][3]);
      float* o = out + (size_t(b) * Hq + hkv * G + hg) * S + s0;
      if (okA) o[g] = kna * codeA * sc_code[nt] + kra * signA * sc_sign[nt];
      if (okB) o[g + 8] = knb * codeB * sc_code[nt] + krb * signB * sc_sign[nt];
    }
  }
}

// Generic CUDA-core estimator for shapes the MMA path does not cover.
// One block per (batch, query head); x = R q and y = S q in shared memory.
__global__ void __launch_bounds__(256) logits_simt_kernel(const float* __restrict__ q, int Hq, int Hkv, int64_t S,
                                                          const float* __restrict__ Rt,
                                                          const float* __restrict__ Pt, int d, int m, int bmse,
                                                          CodebookParams cb, const uint8_t* __restrict__ payload,
                                                          const uint16_t* __restrict__ norms, float scale,
                                                          float* __restrict__ out) {
  extern __shared__ float sm[];
  float* sq = sm;
  float* sx = sq + d;
  float* sy = sx + d;
  const int bh = blockIdx.x;
  const int b = bh / Hq, h = bh % Hq, G = Hq / Hkv, hkv = h / G;
  for (int i = threadIdx.x; i < d; i += blockDim.x) sq[i] = q[size_t(bh) * d + i];
  __syncthreads();
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float x = 0.f;
    for (int i = 0; i < d; ++i) x = fmaf(Rt[i * d + j], sq[i], x);
    sx[j] = x;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    float y = 0.f;
    for (int j = 0; j < d; ++j) y = fmaf(Pt[j * m + i], sx[j], y);
    sy[i] = y;
  }
  __syncthreads();
  const RowGeom gm = make_geom(d, m, bmse);
  const float qc = float(kQjlConst) / float(m);
  const int64_t base_row = (int64_t(b) * Hkv + hkv) * S;
  for (int64_t s = blockIdx.y * blockDim.x + threadIdx.x; s < S; s += int64_t(gridDim.y) * blockDim.x) {
    const uint16_t* hw = reinterpret_cast<const uint16_t*>(payload + (base_row + s) * gm.row_bytes);
    float a = 0.f, c = 0.f;
    for (int j = 0; j < d; ++j) a = fmaf(cb.c[unpack_code(hw, gm, j)], sx[j], a);
    for (int i = 0; i < m; ++i) c += unpack_sign(hw, gm, i) ? sy[i] : -sy[i];
    const float n16 = half_bits_to_float(norms[2 * (base_row + s)]);
    const float r16 = half_bits_to_float(norms[2 * (base_row + s) + 1]);
    out[size_t(bh) * S + s] = scale * (n16 * a + qc * r16 * c);
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

bool fast_path(const tq_ctx* ctx) { return ctx->d == D && ctx->m == D && ctx->bmse >= 1 && ctx->bmse <= 3; }

template <int BMSE, int NT>
cudaError_t launch_mma(const tq_ctx* ctx, int B, int Hq, int Hkv, int64_t S, const uint8_t* payload,
                       const uint16_t* norms, float* out, const uint32_t* frags, const HeadScale* hs,
                       cudaStream_t st) {
  const int64_t total = int64_t(B) * Hkv * ((S + 15) / 16);
  auto kern = logits_mma_kernel<BMSE, NT>;
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kLogitThreads, 0);
  int64_t grid = int64_t(sm_count()) * (per_sm > 0 ? per_sm : 1);
  const int64_t needed = (total + kLogitThreads / 32 - 1) / (kLogitThreads / 32);
  if (grid > needed) grid = needed;
  kern<<<int(grid), kLogitThreads, 0, st>>>(payload, norms, S, Hq, Hkv, total, frags, hs, ctx->lut, out);
  return cudaGetLastError();
}

}  // namespace

size_t qprep_bytes(const tq_ctx* ctx, int64_t groups, int heads_per_group) {
  if (!fast_path(ctx)) return 256;
  const int nt = (heads_per_group + HPT - 1) / HPT;
  const size_t frag = size_t(groups) * nt * kFragWords * 4;
  const size_t scales = size_t(groups) * heads_per_group * sizeof(HeadScale);
  return ((frag + 255) / 256) * 256 + ((scales + 255) / 256) * 256;
}

cudaError_t launch_logits(const tq_ctx* ctx, const float* q, int B, int Hq, int Hkv, int64_t S,
                          const uint8_t* payload, const uint16_t* norms, float scale, float* out, void* ws,
                          cudaStream_t st) {
  const int G = Hq / Hkv;
  if (!fast_path(ctx) || G > 8) {
    const size_t smem = size_t(2 * ctx->d + ctx->m) * 4;
    dim3 grid(unsigned(B * Hq), unsigned(std::min<int64_t>((S + 255) / 256, 64)));
    logits_simt_kernel<<<grid, 256, smem, st>>>(q, Hq, Hkv, S, ctx->dRt, ctx->dPt, ctx->d, ctx->m, ctx->bmse,
                                                ctx->cb, payload, norms, scale, out);
    return cudaGetLastError();
  }
  const int nt = (G + HPT - 1) / HPT;
  const int64_t groups = int64_t(B) * Hkv;
  uint32_t* frags = static_cast<uint32_t*>(ws);
  const size_t frag_bytes = ((size_t(groups) * nt * kFragWords * 4 + 255) / 256) * 256;
  HeadScale* hs = reinterpret_cast<HeadScale*>(static_cast<uint8_t*>(ws) + frag_bytes);
  qprep_kernel<<<unsigned(groups * nt * HPT), 128, 0, st>>>(q, Hq, Hkv, nt, ctx->dRt, ctx->dPt,
                                                             ctx->lut.inv_scale, scale,
                                                             float(kQjlConst / ctx->m), frags, hs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (S == 0) return cudaSuccess;
  switch (ctx->bmse * 10 + nt) {
    case 11: return launch_mma<1, 1>(ctx, B, Hq, Hkv, S, payload, norms, out, frags, hs, st);
    case 12: return launch_mma<1, 2>(ctx, B, Hq, Hkv, S, payload, norms, out, frags, hs, st);
    case 21: return launch_mma<2, 1>(ctx, B, Hq, Hkv, S, payload, norms, out, frags, hs, st);
    case 22: return launch_mma<2, 2>(ctx, B, Hq, Hkv, S, payload, norms, out, frags, hs, st);
    case 31: return launch_mma<3, 1>(ctx, B, Hq, Hkv, S, payload, norms, out, frags, hs, st);
    default: return launch_mma<3, 2>(ctx, B, Hq, Hkv, S, payload, norms, out, frags, hs, st);
  }
}

}  // namespace tq
