// Decode attention logits against the packed cache: the TurboQuant
// inner-product estimator (airosetta.com "Google TurboQuant", stage 2)
//   s = n16 sum_j c[idx_j] (R q)_j + sqrt(pi/2)/m rho16 sum_i sigma_i (S q)_i
// for every (query head, key) of a GQA decode step.  The work is HBM bound
// (mooersco.com section 2.2): 4 query heads share each key of a KV head.
//
// Fast path (d = 128, m = 128 or 0, b' = 1..3, this file's logits_mma_kernel;
// with m = 0, the MSE-only variant, the sign term and its MMAs are dropped;
// logits_split_kernel applies the same scheme to the two 64-channel groups of
// a channel split):
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
#include <type_traits>

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
  float code;      // multiplies the code dot product (int32, after the correction below)
  float sign;      // multiplies the sign dot product
  int32_t ccode;   // one-bit codes: integer correction of the code dot product (see qprep_kernel)
  int32_t csign;   // integer correction of the sign dot product
};

// Coordinate j (of d = 128) is "register 3" of its unit when ((j % 32) / 4) % 4 == 3
// (the register whose operand bytes come from the mode bit of a byte permute).
__device__ __forceinline__ bool reg3_coordinate(int j) { return ((j >> 2) & 3) == 3; }

// ---------------------------------------------------------------------------
// Query preparation: x = R q, y = P x (= S q), int16 fixed point per head,
// split into two signed int8 limbs, written in MMA B-fragment order.
// One block per (batch, KV head group, up to cpb chunks of up to 8
// query heads): R^T and P^T are copied to shared memory (128 KB) once, then
// the block computes the NT head slots of each of its chunks in turn (slots
// past the group's heads are zero).
//
// The logits kernel turns a one-bit field (sign bit, or a one-bit code) into
// operand bytes a = -bit (registers 0..2 of a unit) or a = 1 - bit (register
// 3), so the B operand holds -y (and -x for one-bit codes); then
//   sum_i sigma_i y_i = 2 sum_i bit_i y_i - Y = 2 acc + (2 Y3 - Y),
// acc = sum_i a_i (-y_i) = sum_i bit_i y_i - Y3, with Y = sum_i y_i and Y3 the
// sum over register-3 coordinates; csign = 2 Y3 - Y (exact integers).
// One-bit codes (levels -c1, +c1) use the same form with x.
// ---------------------------------------------------------------------------
constexpr int kMaxSlots = 8;
constexpr int kQChunks = 8;   // at most this many head chunks per query-preparation block

__global__ void __launch_bounds__(256) qprep_kernel(const float* __restrict__ q, int Hq, int Hkv, int nchunk, int cpb,
                                                    int nt,
                                                    const float* __restrict__ Rt, const float* __restrict__ Pt,
                                                    float code_inv_scale, float scale, float qjl_over_m,
                                                    int one_bit_codes, uint32_t* __restrict__ frags,
                                                    HeadScale* __restrict__ hscale) {
  extern __shared__ __align__(16) float smq[];
  float* matR = smq;                                 // [D][D] R^T
  float* matP = matR + D * D;                        // [D][D] P^T
  float* sq = matP + D * D;                          // [slots][D] queries
  float* sx = sq + kMaxSlots * D;                    // [slots][D] x
  __shared__ float red[2][kMaxSlots][4];
  __shared__ int ired[4][kMaxSlots][4];              // [Y, Y3, X, X3][slot][warp of the quad]
  __shared__ int8_t limbs[kMaxSlots][2][2][D];       // [slot][x/y][hi/lo][coordinate]
  const int G = Hq / Hkv;
  const int slots = nt * HPT;
  const int nblk = (nchunk + cpb - 1) / cpb;
  const int grp = blockIdx.x / nblk, cb = blockIdx.x - grp * nblk;
  const int b = grp / Hkv, hkv = grp % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // thread (quad hq, coordinate j): the slots 4 hq .. 4 hq + 3 at coordinate j
  const int j = tid & (D - 1), hq = tid >> 7, wq = warp & 3;
  // the logits grid may start streaming the cache now; it waits for this grid before reading fragments
  asm volatile("griddepcontrol.launch_dependents;");
  // both matrices in flight at once (asynchronous 16-byte copies)
  for (int i = tid; i < D * D / 4; i += 256) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(uint32_t(__cvta_generic_to_shared(matR + 4 * i))),
                 "l"(Rt + 4 * i)
                 : "memory");
    if (Pt)   // no JL matrix in the MSE-only variant
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(uint32_t(__cvta_generic_to_shared(matP + 4 * i))),
                   "l"(Pt + 4 * i)
                   : "memory");
  }
  // 128 x 128 matrix (transposed, in shared memory) times the quad's four
  // vectors v[4 hq + k] (in shared memory, read four coordinates at a time)
  auto matvec4 = [&](const float* mat, const float* v, float (&acc)[4]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = 0.f;
#pragma unroll 2
    for (int i = 0; i < D; i += 4) {
      const float r0 = mat[i * D + j], r1 = mat[(i + 1) * D + j], r2 = mat[(i + 2) * D + j],
                  r3 = mat[(i + 3) * D + j];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 vv = *reinterpret_cast<const float4*>(v + (4 * hq + k) * D + i);
        acc[k] = fmaf(r3, vv.w, fmaf(r2, vv.z, fmaf(r1, vv.y, fmaf(r0, vv.x, acc[k]))));
      }
    }
  };
  const bool quad_on = 4 * hq < slots;              // nt = 1: only the first quad has slots
  const int c_end = (cb + 1) * cpb < nchunk ? (cb + 1) * cpb : nchunk;
  for (int chunk = cb * cpb; chunk < c_end; ++chunk) {
    const int vg = grp * nchunk + chunk;
    const int h0 = chunk * 2 * HPT;                  // first head of the chunk within the group
    if (chunk > cb * cpb) __syncthreads();            // the previous chunk's buffers are read
    for (int idx = tid; idx < slots * D; idx += 256) {
      const int h = idx / D, c = idx - h * D;
      sq[idx] = h0 + h < G ? q[(size_t(b) * Hq + hkv * G + h0 + h) * D + c] : 0.f;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    float acc[4], accy[4];
    if (quad_on) {
      matvec4(matR, sq, acc);
#pragma unroll
      for (int k = 0; k < 4; ++k) sx[(4 * hq + k) * D + j] = acc[k];
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) accy[k] = 0.f;
    if (quad_on && Pt) matvec4(matP, sx, accy);
    // per-slot max |x|, max |y| over the quad's four warps
    if (quad_on) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float ax = fabsf(acc[k]), ay = fabsf(accy[k]);
        for (int o = 16; o; o >>= 1) {
          ax = fmaxf(ax, __shfl_xor_sync(0xffffffffu, ax, o));
          ay = fmaxf(ay, __shfl_xor_sync(0xffffffffu, ay, o));
        }
        if (lane == 0) {
          red[0][4 * hq + k][wq] = ax;
          red[1][4 * hq + k][wq] = ay;
        }
      }
    }
    __syncthreads();
    float kxs[4], kys[4];
    if (quad_on) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int h = 4 * hq + k;
        const float mx = fmaxf(fmaxf(red[0][h][0], red[0][h][1]), fmaxf(red[0][h][2], red[0][h][3]));
        const float my = fmaxf(fmaxf(red[1][h][0], red[1][h][1]), fmaxf(red[1][h][2], red[1][h][3]));
        const float kx = mx > 0.f ? 32000.f / mx : 0.f;
        const float ky = my > 0.f ? 32000.f / my : 0.f;
        kxs[k] = kx;
        kys[k] = ky;
        const int xi = __float2int_rn(acc[k] * kx);
        const int yi = __float2int_rn(accy[k] * ky);
        // the B operand holds -y (and -x for one-bit codes): see the comment above
        const int xb = one_bit_codes ? -xi : xi, yb = -yi;
        const int xh = (xb + 128) >> 8, yh = (yb + 128) >> 8;
        limbs[h][0][0][j] = int8_t(xh);
        limbs[h][0][1][j] = int8_t(xb - 256 * xh);
        limbs[h][1][0][j] = int8_t(yh);
        limbs[h][1][1][j] = int8_t(yb - 256 * yh);
        int ty = yi, ty3 = reg3_coordinate(j) ? yi : 0, tx = xi, tx3 = reg3_coordinate(j) ? xi : 0;
        for (int o = 16; o; o >>= 1) {
          ty += __shfl_xor_sync(0xffffffffu, ty, o);
          ty3 += __shfl_xor_sync(0xffffffffu, ty3, o);
          tx += __shfl_xor_sync(0xffffffffu, tx, o);
          tx3 += __shfl_xor_sync(0xffffffffu, tx3, o);
        }
        if (lane == 0) {
          ired[0][h][wq] = ty;
          ired[1][h][wq] = ty3;
          ired[2][h][wq] = tx;
          ired[3][h][wq] = tx3;
        }
      }
    }
    __syncthreads();
    if (quad_on && j == 0) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int h = 4 * hq + k;
        if (h0 + h < G) {
          const int Y = ired[0][h][0] + ired[0][h][1] + ired[0][h][2] + ired[0][h][3];
          const int Y3 = ired[1][h][0] + ired[1][h][1] + ired[1][h][2] + ired[1][h][3];
          const int X = ired[2][h][0] + ired[2][h][1] + ired[2][h][2] + ired[2][h][3];
          const int X3 = ired[3][h][0] + ired[3][h][1] + ired[3][h][2] + ired[3][h][3];
          HeadScale hsc;
          hsc.code = kxs[k] > 0.f ? scale * code_inv_scale / kxs[k] : 0.f;
          hsc.sign = kys[k] > 0.f ? scale * qjl_over_m / kys[k] : 0.f;
          hsc.ccode = 2 * X3 - X;
          hsc.csign = 2 * Y3 - Y;
          hscale[size_t(b) * Hq + hkv * G + h0 + h] = hsc;
        }
      }
    }
    // Fragment word (xy, s, reg, lane) of N-tile t holds B[k = 16 reg + 4 tig + e][n = lane / 4],
    // e = 0..3; column n is (head slot 4 t + n / 2, limb n % 2); K position k of step s is
    // coordinate tig * D/4 + 4 (2s + reg) + e.
    for (int w = tid; w < nt * kFragWords; w += 256) {
      const int t = w / kFragWords, rem = w - t * kFragWords;
      const int ln = rem & 31, reg = (rem >> 5) & 1, s = (rem >> 6) % KS, xy = (rem >> 6) / KS;
      const int n = ln >> 2, tig = ln & 3;
      const int slot = t * HPT + (n >> 1), limb = n & 1;
      uint32_t word = 0;
      for (int e = 0; e < 4; ++e) {
        const int c = tig * (D / 4) + 4 * (2 * s + reg) + e;
        word |= uint32_t(uint8_t(limbs[slot][xy][limb][c])) << (8 * e);
      }
      frags[size_t(vg) * nt * kFragWords + w] = word;
    }
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

// First k-step: D = A B with a zero accumulator input.
__device__ __forceinline__ void mma_s8_first(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  const int z = 0;
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};\n"
      : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(z));
}

// Chunk of one key for one quarter: BMSE * 2 halfwords of codes (two units)
// and 2 halfwords of signs, as 32-bit words.
template <int BMSE, bool JL = true>
struct Chunk {
  static constexpr int kWords = BMSE + (JL ? 1 : 0);
  uint32_t w[kWords];
};

template <int BMSE, bool JL>
__device__ __forceinline__ void load_chunk(Chunk<BMSE, JL>& c, const uint8_t* row, int tig, bool ok) {
  constexpr int kW = Chunk<BMSE, JL>::kWords;
  const uint32_t* p = reinterpret_cast<const uint32_t*>(row + tig * 4 * kW);
  if constexpr (!JL) {
    // MSE-only rows: the quarter's code words only (4 BMSE bytes)
    if constexpr (kW == 2) {
      const uint2 v = ok ? __ldg(reinterpret_cast<const uint2*>(p)) : make_uint2(0, 0);
      c.w[0] = v.x;
      c.w[1] = v.y;
    } else {
#pragma unroll
      for (int i = 0; i < kW; ++i) c.w[i] = ok ? __ldg(p + i) : 0u;
    }
  } else if constexpr (BMSE == 3) {
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

// Byte-permute selectors (4 nibbles, mode bit clear) of the 8 code registers
// of a quarter: nibble e of selector r is the code of coordinate (r, e).
// Only the low 16 bits of a selector are read by the permute, so a word can
// be masked once for both of its halfwords, and the upper halfword of a word
// needs only a shift.
// Byte-permute selectors (4 nibbles, mode bit clear) of the 8 code registers
// of a quarter: nibble e of selector r is the code of coordinate (r, e).
// Only the low 16 bits of a selector are read by the permute, so a word can
// be masked once for both of its halfwords, and the upper halfword of a word
// needs only a shift.  (Shifts as multiply-highs on the FMA pipe measured
// slower: their latency lengthens the dependency chains.)
template <int BMSE, bool JL>
__device__ __forceinline__ void code_selectors(const Chunk<BMSE, JL>& c, uint32_t (&sel)[8]) {
  if constexpr (BMSE == 3) {
    // words: w0 = H0(u0) | H1(u0), w1 = H2(u0) | H0(u1), w2 = H1(u1) | H2(u1) (low | high halfword)
    const uint32_t m0 = c.w[0] & 0x77777777u, m1 = c.w[1] & 0x77777777u, m2 = c.w[2] & 0x77777777u;
    const uint32_t b0 = c.w[0] & 0x88888888u, b1 = c.w[1] & 0x88888888u, b2 = c.w[2] & 0x88888888u;
    sel[0] = m0;
    sel[1] = m0 >> 16;
    sel[2] = m1;
    sel[4] = m1 >> 16;
    sel[5] = m2;
    sel[6] = m2 >> 16;
    // register 3 of a unit: bit i of its code is bit 3 of the nibble of H_i
    // (the shifted terms have disjoint bits in the low halfword)
    sel[3] = (b0 >> 3) | (b0 >> 18) | (b1 >> 1);     // H0(u0) >> 3, H1(u0) >> 2, H2(u0) >> 1
    sel[7] = (b1 >> 19) | (b2 >> 2) | (b2 >> 17);    // H0(u1) >> 3, H1(u1) >> 2, H2(u1) >> 1
  } else if constexpr (BMSE == 2) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      // word u = H0(u) | H1(u): H0 holds registers 4u (bits 0-1 of a nibble) and 4u + 1 (bits 2-3),
      // H1 registers 4u + 2 and 4u + 3
      const uint32_t a = c.w[u] & 0x33333333u;
      const uint32_t b = (c.w[u] >> 2) & 0x33333333u;
      sel[4 * u + 0] = a;
      sel[4 * u + 1] = b;
      sel[4 * u + 2] = a >> 16;
      sel[4 * u + 3] = b >> 16;
    }
  }
}

// Operand bytes of a one-bit field (a sign bit, or a one-bit code) for the 8
// registers of a quarter: unit u's halfword has bit i of nibble e for
// register 4u + i, coordinate e.  The raw halfword is the permute selector:
// the byte tables of registers 0..2 hold -bit(j, i) in {0x00, 0xFF}, which
// the selector's mode bit (nibble bit 3) leaves unchanged, and the table of
// register 3 is all 0x01, which the mode bit turns into 0x00; so the bytes are
// -bit (registers 0..2) and 1 - bit (register 3), without any mask.
__device__ __forceinline__ void bit_operands(uint32_t w, uint32_t (&a)[8]) {
  const uint32_t h1 = w >> 16;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const uint32_t h = u ? h1 : w;
    a[4 * u + 0] = prmt(0xFF00FF00u, 0xFF00FF00u, h);
    a[4 * u + 1] = prmt(0xFFFF0000u, 0xFFFF0000u, h);
    a[4 * u + 2] = prmt(0x00000000u, 0xFFFFFFFFu, h);
    a[4 * u + 3] = prmt(0x01010101u, 0x01010101u, h);
  }
}

// One 16-key MMA row tile of a 32-key tile: decode, multiply, combine, store.
template <int BMSE, int NT, bool JL>
__device__ __forceinline__ void row_tile(const Chunk<BMSE, JL>& ca, const Chunk<BMSE, JL>& cb, uint32_t na, uint32_t nb,
                                         bool okA, bool okB, const uint32_t (&bx)[NT][KS][2],
                                         const uint32_t (&by)[NT][KS][2], const HeadScale (&hs)[NT],
                                         float* const (&orow)[NT], int g, const CodeLut& lut) {
  int acc_hi[NT][4], acc_lo[NT][4], acc_sg[NT][4];
  if constexpr (BMSE >= 2) {
    uint32_t sa[8], sb[8];
    code_selectors<BMSE, JL>(ca, sa);
    code_selectors<BMSE, JL>(cb, sb);
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
        if (s == 0) {
          mma_s8_first(acc_hi[nt], ah0, ah1, ah2, ah3, bx[nt][s][0], bx[nt][s][1]);
          mma_s8_first(acc_lo[nt], al0, al1, al2, al3, bx[nt][s][0], bx[nt][s][1]);
        } else {
          mma_s8(acc_hi[nt], ah0, ah1, ah2, ah3, bx[nt][s][0], bx[nt][s][1]);
          mma_s8(acc_lo[nt], al0, al1, al2, al3, bx[nt][s][0], bx[nt][s][1]);
        }
      }
    }
  } else {
    // one-bit codes (levels -c1, +c1): the one-bit operand form, one MMA per k-step
    uint32_t ga[8], gb[8];
    bit_operands(ca.w[0], ga);
    bit_operands(cb.w[0], gb);
#pragma unroll
    for (int s = 0; s < KS; ++s)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (s == 0)
          mma_s8_first(acc_hi[nt], ga[0], gb[0], ga[1], gb[1], bx[nt][0][0], bx[nt][0][1]);
        else
          mma_s8(acc_hi[nt], ga[2 * s], gb[2 * s], ga[2 * s + 1], gb[2 * s + 1], bx[nt][s][0], bx[nt][s][1]);
      }
  }
  if constexpr (JL) {
    uint32_t ga[8], gb[8];
    bit_operands(ca.w[BMSE], ga);
    bit_operands(cb.w[BMSE], gb);
#pragma unroll
    for (int s = 0; s < KS; ++s)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (s == 0)
          mma_s8_first(acc_sg[nt], ga[0], gb[0], ga[1], gb[1], by[nt][0][0], by[nt][0][1]);
        else
          mma_s8(acc_sg[nt], ga[2 * s], gb[2 * s], ga[2 * s + 1], gb[2 * s + 1], by[nt][s][0], by[nt][s][1]);
      }
  }
  // epilogue: C[row][2 tig + limb] -> head tig of each N-tile (scales are 0 for padded heads)
  const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&na));   // (||k||, ||r||) of key g
  const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&nb));   // of key g + 8
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float codeA, codeB;
    if constexpr (BMSE >= 2) {
      // |cross terms| <= 2 * 128 * 128 * 128 and |low terms| < 2^21: the integer sums fit in 32 bits
      codeA = fmaf(float(acc_hi[nt][0]), 65536.f, float((acc_hi[nt][1] + acc_lo[nt][0]) * 256 + acc_lo[nt][1]));
      codeB = fmaf(float(acc_hi[nt][2]), 65536.f, float((acc_hi[nt][3] + acc_lo[nt][2]) * 256 + acc_lo[nt][3]));
    } else {
      codeA = float(2 * (acc_hi[nt][0] * 256 + acc_hi[nt][1]) + hs[nt].ccode);
      codeB = float(2 * (acc_hi[nt][2] * 256 + acc_hi[nt][3]) + hs[nt].ccode);
    }
    const float signA = JL ? float(2 * (acc_sg[nt][0] * 256 + acc_sg[nt][1]) + hs[nt].csign) : 0.f;
    const float signB = JL ? float(2 * (acc_sg[nt][2] * 256 + acc_sg[nt][3]) + hs[nt].csign) : 0.f;
    if (orow[nt]) {
      if (okA) orow[nt][g] = fmaf(fa.x * hs[nt].code, codeA, fa.y * hs[nt].sign * signA);
      if (okB) orow[nt][g + 8] = fmaf(fb.x * hs[nt].code, codeB, fb.y * hs[nt].sign * signB);
    }
  }
}

// Each warp streams a contiguous range of 32-key tiles (two MMA row tiles
// sharing the query fragments of their group), the next tile's rows loaded
// with 128-bit loads before this tile's math.  A tile's group is a
// (batch, KV head, chunk of up to 8 query heads) triple: with more than 8
// query heads per KV head, every chunk reads the rows again (from L2, as the
// chunks of one KV head are adjacent in the tile order).

// Tile cursor: (row group, head chunk, first key) advanced without divisions.
struct TileCursor {
  int64_t rg;
  int chunk;
  int64_t s0;
  __device__ __forceinline__ void init(int64_t t, int64_t tpp, int nchunk) {
    const int64_t vg = t / tpp;
    s0 = (t - vg * tpp) * 32;
    rg = vg / nchunk;
    chunk = int(vg - rg * nchunk);
  }
  __device__ __forceinline__ void next(int64_t S, int nchunk) {
    s0 += 32;
    if (s0 >= S) {
      s0 = 0;
      if (++chunk == nchunk) {
        chunk = 0;
        ++rg;
      }
    }
  }
};

template <int BMSE, int NT, bool JL>
__global__ void __launch_bounds__(kLogitThreads) logits_mma_kernel(
    const uint8_t* __restrict__ payload, const uint16_t* __restrict__ norms, int64_t S, int Hq, int Hkv, int nchunk,
    int64_t total_tiles, const uint32_t* __restrict__ frags, const HeadScale* __restrict__ hscale, CodeLut lut,
    float* __restrict__ out) {
  constexpr int kRowBytes = D * BMSE / 8 + (JL ? D / 8 : 0);
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int64_t nwarps = int64_t(gridDim.x) * (kLogitThreads / 32);
  const int64_t gw = int64_t(blockIdx.x) * (kLogitThreads / 32) + (threadIdx.x >> 5);
  const int64_t t_begin = gw * total_tiles / nwarps, t_end = (gw + 1) * total_tiles / nwarps;
  const int G = Hq / Hkv;
  const int64_t tpp = (S + 31) / 32;
  const uint32_t* norms32 = reinterpret_cast<const uint32_t*>(norms);

  auto load_tile = [&](const TileCursor& c, Chunk<BMSE, JL> (&ch)[4], uint32_t (&nn)[4]) {
    const int64_t row0 = c.rg * S + c.s0 + g;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool ok = c.s0 + g + 8 * k < S;
      load_chunk<BMSE, JL>(ch[k], payload + (row0 + 8 * k) * kRowBytes, tig, ok);
      nn[k] = ok ? __ldg(norms32 + row0 + 8 * k) : 0u;
    }
  };
  TileCursor cc;
  cc.init(t_begin, tpp, nchunk);
  Chunk<BMSE, JL> cur[4];
  uint32_t curn[4];
  if (t_begin < t_end) load_tile(cc, cur, curn);

  // the query fragments are written by the preceding query-preparation grid
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (t_begin >= t_end) return;

  uint32_t bx[NT][KS][2], by[NT][KS][2];
  HeadScale hs[NT];
  float* orow[NT];
  auto load_group = [&](const TileCursor& c) {
    const int b = int(c.rg / Hkv), hkv = int(c.rg - int64_t(b) * Hkv);
    const int64_t gi = c.rg * nchunk + c.chunk;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint32_t* fr = frags + (size_t(gi) * NT + nt) * kFragWords;
#pragma unroll
      for (int s = 0; s < KS; ++s)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          bx[nt][s][r] = __ldg(fr + ((0 * KS + s) * 2 + r) * 32 + lane);
          by[nt][s][r] = __ldg(fr + ((1 * KS + s) * 2 + r) * 32 + lane);
        }
      const int hg = c.chunk * 2 * HPT + nt * HPT + tig;
      const int hh = hg < G ? hg : 0;
      hs[nt] = hscale[size_t(b) * Hq + hkv * G + hh];
      orow[nt] = hg < G ? out + (size_t(b) * Hq + hkv * G + hh) * S : nullptr;
    }
  };
  load_group(cc);

  for (int64_t t = t_begin; t < t_end; ++t) {
    // next tile coordinates and its loads, issued before this tile's math
    TileCursor nc = cc;
    nc.next(S, nchunk);
    Chunk<BMSE, JL> nxt[4];
    uint32_t nxtn[4] = {0u, 0u, 0u, 0u};
    if (t + 1 < t_end) load_tile(nc, nxt, nxtn);

    float* orow_t[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) orow_t[nt] = orow[nt] ? orow[nt] + cc.s0 : nullptr;
    row_tile<BMSE, NT, JL>(cur[0], cur[1], curn[0], curn[1], cc.s0 + g < S, cc.s0 + g + 8 < S, bx, by, hs, orow_t, g,
                           lut);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) orow_t[nt] = orow[nt] ? orow[nt] + cc.s0 + 16 : nullptr;
    row_tile<BMSE, NT, JL>(cur[2], cur[3], curn[2], curn[3], cc.s0 + g + 16 < S, cc.s0 + g + 24 < S, bx, by, hs,
                           orow_t, g, lut);

    if (t + 1 < t_end) {
      if (nc.rg != cc.rg || nc.chunk != cc.chunk) load_group(nc);
      cc = nc;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        cur[k] = nxt[k];
        curn[k] = nxtn[k];
      }
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
                                                          float* __restrict__ out, ChannelGather gth,
                                                          int accumulate) {
  extern __shared__ float sm[];
  float* sq = sm;
  float* sx = sq + d;
  float* sy = sx + d;
  const int bh = blockIdx.x;
  const int b = bh / Hq, h = bh % Hq, G = Hq / Hkv, hkv = h / G;
  // split: the query's channels in the group order of its KV head
  for (int i = threadIdx.x; i < d; i += blockDim.x)
    sq[i] = gth.perm ? q[size_t(bh) * gth.dtot + gth.perm[hkv * gth.dtot + gth.off + i]] : q[size_t(bh) * d + i];
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
  const float qc = m > 0 ? float(kQjlConst) / float(m) : 0.f;   // m = 0: no sign term
  const int64_t base_row = (int64_t(b) * Hkv + hkv) * S;
  for (int64_t s = blockIdx.y * blockDim.x + threadIdx.x; s < S; s += int64_t(gridDim.y) * blockDim.x) {
    const uint16_t* hw = reinterpret_cast<const uint16_t*>(payload + (base_row + s) * gm.row_bytes);
    float a = 0.f, c = 0.f;
    for (int j = 0; j < d; ++j) a = fmaf(cb.c[unpack_code(hw, gm, j)], sx[j], a);
    for (int i = 0; i < m; ++i) c += unpack_sign(hw, gm, i) ? sy[i] : -sy[i];
    const float n16 = half_bits_to_float(norms[2 * (base_row + s)]);
    const float r16 = half_bits_to_float(norms[2 * (base_row + s) + 1]);
    const float v = scale * (n16 * a + qc * r16 * c);
    out[size_t(bh) * S + s] = accumulate ? out[size_t(bh) * S + s] + v : v;
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

bool fast_path(const tq_ctx* ctx) {
  return ctx->d == D && (ctx->m == D || ctx->m == 0) && ctx->bmse >= 1 && ctx->bmse <= 3;
}

template <int BMSE, int NT, bool JL>
cudaError_t launch_mma(const tq_ctx* ctx, int B, int Hq, int Hkv, int64_t S, int nchunk, const uint8_t* payload,
                       const uint16_t* norms, float* out, const uint32_t* frags, const HeadScale* hs,
                       cudaStream_t st) {
  const int64_t total = int64_t(B) * Hkv * nchunk * ((S + 31) / 32);
  auto kern = logits_mma_kernel<BMSE, NT, JL>;
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kLogitThreads, 0);
  int64_t grid = int64_t(sm_count()) * (per_sm > 0 ? per_sm : 1);
  const int64_t needed = (total + kLogitThreads / 32 - 1) / (kLogitThreads / 32);
  if (grid > needed) grid = needed;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(kLogitThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap with the query preparation
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, payload, norms, S, Hq, Hkv, nchunk, total, frags, hs, ctx->lut, out);
}

// ---------------------------------------------------------------------------
// Split cache (two groups of d = m = 64 channels per key, each with its own
// context; see k_split.cu): the same int8 MMA scheme, group by group.  A
// thread's quarter of a key is chunk tig of each group row (16 coordinates:
// two k-steps per group).  The codes and signs of the two groups accumulate
// separately because each group has its own norms and query scales; the
// epilogue adds the four terms.
// ---------------------------------------------------------------------------
constexpr int GD = 64;          // group dimension of the split fast path
constexpr int GKS = GD / 32;    // k-steps per group

struct SplitScale {
  float code[2];     // per group (0 high, 1 low): multiplies the code dot product
  float sign[2];     // multiplies the sign dot product
  int32_t ccode[2];  // one-bit codes: integer correction of the code dot product (as in qprep_kernel)
  int32_t csign[2];  // integer correction of the sign dot product
};

// Query preparation of the split: per (batch, KV head) group, the query's
// channels gathered in the head's split order, x_g = R_g q_g and
// y_g = P_g x_g (= S_g q_g) per group g, int16 fixed point per (head, group),
// two int8 limbs, MMA B-fragment order: word
// ((((nt 2 + g) 2 + xy) 2 + s) 2 + reg) 32 + lane holds K positions
// k = 4 tig + e (reg 0) or 16 + 4 tig + e (reg 1) of step s, i.e. group
// coordinates 16 tig + 4 (2 s + reg) + e, for column n = lane / 4 = (head
// slot 4 nt + n / 2, limb n % 2).
__global__ void __launch_bounds__(128) qprep_split_kernel(const float* __restrict__ q, int Hq, int Hkv,
                                                          int nt_per_group, const int32_t* __restrict__ perm,
                                                          const float* __restrict__ Rt_hi,
                                                          const float* __restrict__ Pt_hi,
                                                          const float* __restrict__ Rt_lo,
                                                          const float* __restrict__ Pt_lo, float inv_hi, float inv_lo,
                                                          float scale, float qjl_hi, float qjl_lo, int one_bit_hi,
                                                          int one_bit_lo, uint32_t* __restrict__ frags,
                                                          SplitScale* __restrict__ hscale) {
  __shared__ float sq[kMaxSlots][2 * GD];   // gathered queries [high | low]
  __shared__ float sx[kMaxSlots][2 * GD];
  __shared__ float red[2][kMaxSlots][4];
  __shared__ int ired[4][kMaxSlots][4];     // [Y, Y3, X, X3][slot][warp]
  __shared__ int8_t limbs[kMaxSlots][2][2][2 * GD];   // [slot][x/y][hi/lo limb][coordinate of high | low]
  const int G = Hq / Hkv;
  const int slots = nt_per_group * HPT;
  const int grp = blockIdx.x, b = grp / Hkv, hkv = grp % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gi = tid >> 6, j = tid & 63;   // group and group coordinate of this thread
  asm volatile("griddepcontrol.launch_dependents;");
  const int ch = perm[hkv * 2 * GD + tid];
  for (int h = 0; h < slots; ++h) sq[h][tid] = h < G ? q[(size_t(b) * Hq + hkv * G + h) * (2 * GD) + ch] : 0.f;
  __syncthreads();
  const float* Rt = gi ? Rt_lo : Rt_hi;
  const float* Pt = gi ? Pt_lo : Pt_hi;
  float acc[kMaxSlots];
#pragma unroll
  for (int h = 0; h < kMaxSlots; ++h) acc[h] = 0.f;
  for (int p = 0; p < GD; ++p) {
    const float r = __ldg(Rt + p * GD + j);   // R_g[j][p]
#pragma unroll
    for (int h = 0; h < kMaxSlots; ++h)
      if (h < slots) acc[h] = fmaf(r, sq[h][gi * GD + p], acc[h]);
  }
#pragma unroll
  for (int h = 0; h < kMaxSlots; ++h)
    if (h < slots) sx[h][tid] = acc[h];
  __syncthreads();
  float accy[kMaxSlots];
#pragma unroll
  for (int h = 0; h < kMaxSlots; ++h) accy[h] = 0.f;
  for (int p = 0; p < GD; ++p) {
    const float pv = __ldg(Pt + p * GD + j);  // P_g[j][p]
#pragma unroll
    for (int h = 0; h < kMaxSlots; ++h)
      if (h < slots) accy[h] = fmaf(pv, sx[h][gi * GD + p], accy[h]);
  }
#pragma unroll
  for (int h = 0; h < kMaxSlots; ++h) {
    if (h >= slots) break;
    float ax = fabsf(acc[h]), ay = fabsf(accy[h]);
    for (int o = 16; o; o >>= 1) {
      ax = fmaxf(ax, __shfl_xor_sync(0xffffffffu, ax, o));
      ay = fmaxf(ay, __shfl_xor_sync(0xffffffffu, ay, o));
    }
    if (lane == 0) {
      red[0][h][warp] = ax;
      red[1][h][warp] = ay;
    }
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < kMaxSlots; ++h) {
    if (h >= slots) break;
    const float mx = fmaxf(red[0][h][2 * gi], red[0][h][2 * gi + 1]);
    const float my = fmaxf(red[1][h][2 * gi], red[1][h][2 * gi + 1]);
    const float kx = mx > 0.f ? 32000.f / mx : 0.f;
    const float ky = my > 0.f ? 32000.f / my : 0.f;
    const int xi = __float2int_rn(acc[h] * kx);
    const int yi = __float2int_rn(accy[h] * ky);
    // the B operand holds -y (and -x for a group of one-bit codes): the
    // one-bit operand form of qprep_kernel
    const int xb = (gi ? one_bit_lo : one_bit_hi) ? -xi : xi, yb = -yi;
    const int xh = (xb + 128) >> 8, yh = (yb + 128) >> 8;
    limbs[h][0][0][tid] = int8_t(xh);
    limbs[h][0][1][tid] = int8_t(xb - 256 * xh);
    limbs[h][1][0][tid] = int8_t(yh);
    limbs[h][1][1][tid] = int8_t(yb - 256 * yh);
    int ty = yi, ty3 = reg3_coordinate(j) ? yi : 0, tx = xi, tx3 = reg3_coordinate(j) ? xi : 0;
    for (int o = 16; o; o >>= 1) {
      ty += __shfl_xor_sync(0xffffffffu, ty, o);
      ty3 += __shfl_xor_sync(0xffffffffu, ty3, o);
      tx += __shfl_xor_sync(0xffffffffu, tx, o);
      tx3 += __shfl_xor_sync(0xffffffffu, tx3, o);
    }
    if (lane == 0) {
      ired[0][h][warp] = ty;
      ired[1][h][warp] = ty3;
      ired[2][h][warp] = tx;
      ired[3][h][warp] = tx3;
    }
    if (j == 0 && h < G) {
      SplitScale* hs = hscale + size_t(b) * Hq + hkv * G + h;
      hs->code[gi] = mx > 0.f ? scale * (gi ? inv_lo : inv_hi) / kx : 0.f;
      hs->sign[gi] = my > 0.f ? scale * (gi ? qjl_lo : qjl_hi) / ky : 0.f;
    }
  }
  __syncthreads();
  // group gi's integer corrections from its two warps' sums
  if (j == 0) {
#pragma unroll
    for (int h = 0; h < kMaxSlots; ++h) {
      if (h >= slots || h >= G) break;
      SplitScale* hs = hscale + size_t(b) * Hq + hkv * G + h;
      const int Y = ired[0][h][2 * gi] + ired[0][h][2 * gi + 1], Y3 = ired[1][h][2 * gi] + ired[1][h][2 * gi + 1];
      const int X = ired[2][h][2 * gi] + ired[2][h][2 * gi + 1], X3 = ired[3][h][2 * gi] + ired[3][h][2 * gi + 1];
      hs->ccode[gi] = 2 * X3 - X;
      hs->csign[gi] = 2 * Y3 - Y;
    }
  }
  for (int w = tid; w < nt_per_group * kFragWords; w += 128) {
    const int ln = w & 31, reg = (w >> 5) & 1, st = (w >> 6) & 1, xy = (w >> 7) & 1, g2 = (w >> 8) & 1;
    const int nt = w >> 9;
    const int n = ln >> 2, tig = ln & 3;
    const int slot = nt * HPT + (n >> 1), limb = n & 1;
    uint32_t word = 0;
    for (int e = 0; e < 4; ++e) {
      const int jj = g2 * GD + tig * (GD / 4) + 4 * (2 * st + reg) + e;
      word |= uint32_t(uint8_t(limbs[slot][xy][limb][jj])) << (8 * e);
    }
    frags[size_t(grp) * nt_per_group * kFragWords + w] = word;
  }
}

// One group's chunk tig of a key (d = m = 64): BM code halfwords, then the
// sign halfword, packed two per word (halfword i in word i / 2).
template <int BM>
struct GChunk {
  uint32_t w[(BM + 2) / 2];
  __device__ __forceinline__ uint32_t h(int i) const { return (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu); }
};

template <int BM>
__device__ __forceinline__ void load_gchunk(GChunk<BM>& c, const uint8_t* row, int tig, bool ok) {
  const uint8_t* p = row + tig * 2 * (BM + 1);
  if constexpr (BM == 1) {
    c.w[0] = ok ? __ldg(reinterpret_cast<const uint32_t*>(p)) : 0u;
  } else if constexpr (BM == 3) {
    const uint2 v = ok ? __ldg(reinterpret_cast<const uint2*>(p)) : make_uint2(0u, 0u);
    c.w[0] = v.x;
    c.w[1] = v.y;
  } else {
    // 6 bytes at a 2-byte boundary
    const unsigned short* p16 = reinterpret_cast<const unsigned short*>(p);
    c.w[0] = ok ? uint32_t(__ldg(p16)) | (uint32_t(__ldg(p16 + 1)) << 16) : 0u;
    c.w[1] = ok ? uint32_t(__ldg(p16 + 2)) : 0u;
  }
}

// Byte-permute selectors of the 4 registers of one unit (as code_selectors).
template <int BM>
__device__ __forceinline__ void gcode_selectors(const GChunk<BM>& c, uint32_t (&sel)[4]) {
  if constexpr (BM == 3) {
    const uint32_t h0 = c.h(0), h1 = c.h(1), h2 = c.h(2);
    sel[0] = h0 & 0x7777u;
    sel[1] = h1 & 0x7777u;
    sel[2] = h2 & 0x7777u;
    sel[3] = ((h0 >> 3) & 0x1111u) | ((h1 >> 2) & 0x2222u) | ((h2 >> 1) & 0x4444u);
  } else if constexpr (BM == 2) {
    sel[0] = c.h(0) & 0x3333u;
    sel[1] = (c.h(0) >> 2) & 0x3333u;
    sel[2] = c.h(1) & 0x3333u;
    sel[3] = (c.h(1) >> 2) & 0x3333u;
  }
}

// The one-bit operand form (see bit_operands) for the 4 registers of one unit.
__device__ __forceinline__ void bit_operands4(uint32_t h, uint32_t (&a)[4]) {
  a[0] = prmt(0xFF00FF00u, 0xFF00FF00u, h);
  a[1] = prmt(0xFFFF0000u, 0xFFFF0000u, h);
  a[2] = prmt(0x00000000u, 0xFFFFFFFFu, h);
  a[3] = prmt(0x01010101u, 0x01010101u, h);
}

// Products of one group for a 16-key row tile: code planes (hi, lo; one-bit
// codes: one plane in the one-bit form, in ah) and signs.
template <int BM, int NT>
__device__ __forceinline__ void group_mma(const GChunk<BM>& ca, const GChunk<BM>& cb, const CodeLut& lut,
                                          const uint32_t (&bx)[NT][GKS][2], const uint32_t (&by)[NT][GKS][2],
                                          int (&ah)[NT][4], int (&al)[NT][4], int (&sg)[NT][4]) {
  if constexpr (BM >= 2) {
    uint32_t sa[4], sb[4];
    gcode_selectors<BM>(ca, sa);
    gcode_selectors<BM>(cb, sb);
#pragma unroll
    for (int s = 0; s < GKS; ++s) {
      const uint32_t h0 = prmt(lut.hi[0], lut.hi[1], sa[2 * s]), h1 = prmt(lut.hi[0], lut.hi[1], sb[2 * s]);
      const uint32_t h2 = prmt(lut.hi[0], lut.hi[1], sa[2 * s + 1]), h3 = prmt(lut.hi[0], lut.hi[1], sb[2 * s + 1]);
      const uint32_t l0 = prmt(lut.lo[0], lut.lo[1], sa[2 * s]), l1 = prmt(lut.lo[0], lut.lo[1], sb[2 * s]);
      const uint32_t l2 = prmt(lut.lo[0], lut.lo[1], sa[2 * s + 1]), l3 = prmt(lut.lo[0], lut.lo[1], sb[2 * s + 1]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (s == 0) {
          mma_s8_first(ah[nt], h0, h1, h2, h3, bx[nt][s][0], bx[nt][s][1]);
          mma_s8_first(al[nt], l0, l1, l2, l3, bx[nt][s][0], bx[nt][s][1]);
        } else {
          mma_s8(ah[nt], h0, h1, h2, h3, bx[nt][s][0], bx[nt][s][1]);
          mma_s8(al[nt], l0, l1, l2, l3, bx[nt][s][0], bx[nt][s][1]);
        }
      }
    }
  } else {
    uint32_t ca4[4], cb4[4];
    bit_operands4(ca.h(0), ca4);
    bit_operands4(cb.h(0), cb4);
#pragma unroll
    for (int s = 0; s < GKS; ++s)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (s == 0)
          mma_s8_first(ah[nt], ca4[0], cb4[0], ca4[1], cb4[1], bx[nt][0][0], bx[nt][0][1]);
        else
          mma_s8(ah[nt], ca4[2 * s], cb4[2 * s], ca4[2 * s + 1], cb4[2 * s + 1], bx[nt][s][0], bx[nt][s][1]);
      }
  }
  uint32_t ga[4], gb[4];
  bit_operands4(ca.h(BM), ga);
  bit_operands4(cb.h(BM), gb);
#pragma unroll
  for (int s = 0; s < GKS; ++s)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (s == 0)
        mma_s8_first(sg[nt], ga[0], gb[0], ga[1], gb[1], by[nt][0][0], by[nt][0][1]);
      else
        mma_s8(sg[nt], ga[2 * s], gb[2 * s], ga[2 * s + 1], gb[2 * s + 1], by[nt][s][0], by[nt][s][1]);
    }
}

// Code dot product of key row r (0: key g, 2: key g + 8) of a group.
template <int BM>
__device__ __forceinline__ float group_code(const int (&a)[4], const int (&b)[4], int r, int ccode) {
  if constexpr (BM >= 2)   // |cross terms| <= 2 * 64 * 128 * 128 and |low terms| < 2^20: the sums fit in 32 bits
    return fmaf(float(a[r]), 65536.f, float((a[r + 1] + b[r]) * 256 + b[r + 1]));
  else
    return float(2 * (a[r] * 256 + a[r + 1]) + ccode);
}
__device__ __forceinline__ float group_sign(const int (&a)[4], int r, int csign) {
  return float(2 * (a[r] * 256 + a[r + 1]) + csign);
}

template <int BHI, int BLO, int NT>
__device__ __forceinline__ void split_row_tile(const GChunk<BHI>& ha, const GChunk<BHI>& hb, const GChunk<BLO>& la,
                                               const GChunk<BLO>& lb, uint32_t nha, uint32_t nhb, uint32_t nla,
                                               uint32_t nlb, bool okA, bool okB, const uint32_t (&bx)[2][NT][GKS][2],
                                               const uint32_t (&by)[2][NT][GKS][2], const SplitScale (&sc)[NT],
                                               float* const (&orow)[NT], int g, const CodeLut& lut_hi,
                                               const CodeLut& lut_lo) {
  int hh[NT][4], hl[NT][4], hs[NT][4], lh[NT][4], ll[NT][4], ls[NT][4];
  group_mma<BHI, NT>(ha, hb, lut_hi, bx[0], by[0], hh, hl, hs);
  group_mma<BLO, NT>(la, lb, lut_lo, bx[1], by[1], lh, ll, ls);
  const float2 fha = __half22float2(*reinterpret_cast<const __half2*>(&nha));   // (||k_hi||, ||r_hi||) of key g
  const float2 fhb = __half22float2(*reinterpret_cast<const __half2*>(&nhb));   // of key g + 8
  const float2 fla = __half22float2(*reinterpret_cast<const __half2*>(&nla));
  const float2 flb = __half22float2(*reinterpret_cast<const __half2*>(&nlb));
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    if (!orow[nt]) continue;
    const SplitScale& c = sc[nt];
    const float vA = fmaf(fha.x * c.code[0], group_code<BHI>(hh[nt], hl[nt], 0, c.ccode[0]),
                          fmaf(fha.y * c.sign[0], group_sign(hs[nt], 0, c.csign[0]),
                               fmaf(fla.x * c.code[1], group_code<BLO>(lh[nt], ll[nt], 0, c.ccode[1]),
                                    fla.y * c.sign[1] * group_sign(ls[nt], 0, c.csign[1]))));
    const float vB = fmaf(fhb.x * c.code[0], group_code<BHI>(hh[nt], hl[nt], 2, c.ccode[0]),
                          fmaf(fhb.y * c.sign[0], group_sign(hs[nt], 2, c.csign[0]),
                               fmaf(flb.x * c.code[1], group_code<BLO>(lh[nt], ll[nt], 2, c.ccode[1]),
                                    flb.y * c.sign[1] * group_sign(ls[nt], 2, c.csign[1]))));
    if (okA) orow[nt][g] = vA;
    if (okB) orow[nt][g + 8] = vB;
  }
}

template <int BHI, int BLO, int NT>
__global__ void __launch_bounds__(kLogitThreads, NT == 1 ? 2 : 1) logits_split_kernel(
    const uint8_t* __restrict__ payload_hi, const uint16_t* __restrict__ norms_hi,
    const uint8_t* __restrict__ payload_lo, const uint16_t* __restrict__ norms_lo, int64_t S, int Hq, int Hkv,
    int64_t total_tiles, const uint32_t* __restrict__ frags, const SplitScale* __restrict__ hscale, CodeLut lut_hi,
    CodeLut lut_lo, float* __restrict__ out) {
  constexpr int kRowHi = 8 * (BHI + 1), kRowLo = 8 * (BLO + 1);
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int64_t nwarps = int64_t(gridDim.x) * (kLogitThreads / 32);
  const int64_t gw = int64_t(blockIdx.x) * (kLogitThreads / 32) + (threadIdx.x >> 5);
  const int64_t t_begin = gw * total_tiles / nwarps, t_end = (gw + 1) * total_tiles / nwarps;
  const int G = Hq / Hkv;
  const int64_t tpp = (S + 31) / 32;
  int64_t grp = t_begin / tpp;
  int64_t s0 = (t_begin - grp * tpp) * 32;

  auto load_tile = [&](int64_t gi, int64_t so, GChunk<BHI> (&ch)[4], GChunk<BLO> (&cl)[4], uint32_t (&nh)[4],
                       uint32_t (&nl)[4]) {
    const int64_t row0 = gi * S + so + g;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool ok = so + g + 8 * k < S;
      load_gchunk<BHI>(ch[k], payload_hi + (row0 + 8 * k) * kRowHi, tig, ok);
      load_gchunk<BLO>(cl[k], payload_lo + (row0 + 8 * k) * kRowLo, tig, ok);
      nh[k] = ok ? __ldg(reinterpret_cast<const uint32_t*>(norms_hi) + row0 + 8 * k) : 0u;
      nl[k] = ok ? __ldg(reinterpret_cast<const uint32_t*>(norms_lo) + row0 + 8 * k) : 0u;
    }
  };
  GChunk<BHI> ch[4];
  GChunk<BLO> cl[4];
  uint32_t nh[4], nl[4];
  if (t_begin < t_end) load_tile(grp, s0, ch, cl, nh, nl);

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (t_begin >= t_end) return;

  uint32_t bx[2][NT][GKS][2], by[2][NT][GKS][2];
  SplitScale sc[NT];
  float* orow[NT];
  auto load_group = [&](int64_t gi) {
    const int b = int(gi / Hkv), hkv = int(gi - int64_t(b) * Hkv);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint32_t* fr = frags + (size_t(gi) * NT + nt) * kFragWords;
#pragma unroll
      for (int g2 = 0; g2 < 2; ++g2)
#pragma unroll
        for (int s = 0; s < GKS; ++s)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            bx[g2][nt][s][r] = __ldg(fr + ((((g2 * 2 + 0) * 2 + s) * 2 + r) * 32) + lane);
            by[g2][nt][s][r] = __ldg(fr + ((((g2 * 2 + 1) * 2 + s) * 2 + r) * 32) + lane);
          }
      const int hg = nt * HPT + tig;
      const int hh = hg < G ? hg : 0;
      sc[nt] = hscale[size_t(b) * Hq + hkv * G + hh];
      orow[nt] = hg < G ? out + (size_t(b) * Hq + hkv * G + hh) * S : nullptr;
    }
  };
  load_group(grp);

  for (int64_t t = t_begin; t < t_end; ++t) {
    int64_t ngrp = grp, ns0 = s0 + 32;
    if (ns0 >= S) {
      ns0 = 0;
      ++ngrp;
    }
    GChunk<BHI> nch[4];
    GChunk<BLO> ncl[4];
    uint32_t nnh[4] = {0u, 0u, 0u, 0u}, nnl[4] = {0u, 0u, 0u, 0u};
    if (t + 1 < t_end) load_tile(ngrp, ns0, nch, ncl, nnh, nnl);

    float* orow_t[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) orow_t[nt] = orow[nt] ? orow[nt] + s0 : nullptr;
    split_row_tile<BHI, BLO, NT>(ch[0], ch[1], cl[0], cl[1], nh[0], nh[1], nl[0], nl[1], s0 + g < S,
                                 s0 + g + 8 < S, bx, by, sc, orow_t, g, lut_hi, lut_lo);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) orow_t[nt] = orow[nt] ? orow[nt] + s0 + 16 : nullptr;
    split_row_tile<BHI, BLO, NT>(ch[2], ch[3], cl[2], cl[3], nh[2], nh[3], nl[2], nl[3], s0 + g + 16 < S,
                                 s0 + g + 24 < S, bx, by, sc, orow_t, g, lut_hi, lut_lo);

    if (t + 1 < t_end) {
      if (ngrp != grp) load_group(ngrp);
      grp = ngrp;
      s0 = ns0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        ch[k] = nch[k];
        cl[k] = ncl[k];
        nh[k] = nnh[k];
        nl[k] = nnl[k];
      }
    }
  }
}

}  // namespace

cudaError_t launch_logits_simt(const tq_ctx* ctx, const float* q, int B, int Hq, int Hkv, int64_t S,
                               const uint8_t* payload, const uint16_t* norms, float scale, float* out,
                               ChannelGather gather, int accumulate, cudaStream_t st) {
  if (S == 0 || B == 0 || Hq == 0) return cudaSuccess;
  const size_t smem = size_t(2 * ctx->d + ctx->m) * 4;
  dim3 grid(unsigned(B * Hq), unsigned(std::min<int64_t>((S + 255) / 256, 64)));
  logits_simt_kernel<<<grid, 256, smem, st>>>(q, Hq, Hkv, S, ctx->dRt, ctx->dPt, ctx->d, ctx->m, ctx->bmse,
                                              ctx->cb, payload, norms, scale, out, gather, accumulate);
  return cudaGetLastError();
}

// Query heads per chunk of a (batch, KV head) group and the MMA N-tiles of a chunk.
int chunks_of(int G) { return (G + 2 * HPT - 1) / (2 * HPT); }
int tiles_of(int G) { return G >= 2 * HPT ? 2 : (G + HPT - 1) / HPT; }

size_t qprep_bytes(const tq_ctx* ctx, int64_t groups, int heads_per_group) {
  if (!fast_path(ctx)) return 256;
  const size_t frag = size_t(groups) * chunks_of(heads_per_group) * tiles_of(heads_per_group) * kFragWords * 4;
  const size_t scales = size_t(groups) * heads_per_group * sizeof(HeadScale);
  return ((frag + 255) / 256) * 256 + ((scales + 255) / 256) * 256;
}

cudaError_t launch_logits(const tq_ctx* ctx, const float* q, int B, int Hq, int Hkv, int64_t S,
                          const uint8_t* payload, const uint16_t* norms, float scale, float* out, void* ws,
                          cudaStream_t st) {
  const int G = Hq / Hkv;
  if (!fast_path(ctx))
    return launch_logits_simt(ctx, q, B, Hq, Hkv, S, payload, norms, scale, out,
                              ChannelGather{nullptr, 1, 1, 0, 0}, 0, st);
  const int nchunk = chunks_of(G), nt = tiles_of(G);
  const int64_t groups = int64_t(B) * Hkv;
  uint32_t* frags = static_cast<uint32_t*>(ws);
  const size_t frag_bytes = ((size_t(groups) * nchunk * nt * kFragWords * 4 + 255) / 256) * 256;
  HeadScale* hs = reinterpret_cast<HeadScale*>(static_cast<uint8_t*>(ws) + frag_bytes);
  const size_t qp_smem = size_t(2 * D * D + 2 * kMaxSlots * D) * 4;
  cudaFuncSetAttribute(qprep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(qp_smem));
  // one-bit codes (levels -c1, +c1) use the one-bit operand form: the code scale is c1
  const float code_scale = ctx->bmse == 1 ? float(ctx->c[1]) : ctx->lut.inv_scale;
  // blocks per group: as many as two waves of blocks allow (a small batch is
  // latency bound: one chunk per block), down to one per group for large
  // batches (each block then copies R and P once for up to kQChunks chunks);
  // the chunks are split evenly over a group's blocks
  int64_t nbg = 2 * int64_t(sm_count()) / groups;
  if (nbg < (nchunk + kQChunks - 1) / kQChunks) nbg = (nchunk + kQChunks - 1) / kQChunks;
  if (nbg > nchunk) nbg = nchunk;
  const int cpb = int((nchunk + nbg - 1) / nbg);
  qprep_kernel<<<unsigned(groups * ((nchunk + cpb - 1) / cpb)), 256, qp_smem, st>>>(
      q, Hq, Hkv, nchunk, cpb, nt, ctx->dRt, ctx->dPt, code_scale, scale,
      float(ctx->m > 0 ? kQjlConst / ctx->m : 0.0), ctx->bmse == 1 ? 1 : 0, frags, hs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (S == 0) return cudaSuccess;
  auto go = [&](auto jl) -> cudaError_t {
    constexpr bool J = decltype(jl)::value;
    switch (ctx->bmse * 10 + nt) {
      case 11: return launch_mma<1, 1, J>(ctx, B, Hq, Hkv, S, nchunk, payload, norms, out, frags, hs, st);
      case 12: return launch_mma<1, 2, J>(ctx, B, Hq, Hkv, S, nchunk, payload, norms, out, frags, hs, st);
      case 21: return launch_mma<2, 1, J>(ctx, B, Hq, Hkv, S, nchunk, payload, norms, out, frags, hs, st);
      case 22: return launch_mma<2, 2, J>(ctx, B, Hq, Hkv, S, nchunk, payload, norms, out, frags, hs, st);
      case 31: return launch_mma<3, 1, J>(ctx, B, Hq, Hkv, S, nchunk, payload, norms, out, frags, hs, st);
      default: return launch_mma<3, 2, J>(ctx, B, Hq, Hkv, S, nchunk, payload, norms, out, frags, hs, st);
    }
  };
  return ctx->m > 0 ? go(std::true_type{}) : go(std::false_type{});
}

namespace {

bool split_fast_path(const tq_split* sp, int G) {
  return sp->d == 2 * GD && sp->hi->d == GD && sp->lo->d == GD && sp->hi->m == GD && sp->lo->m == GD &&
         sp->hi->bmse >= 1 && sp->hi->bmse <= 3 && sp->lo->bmse >= 1 && sp->lo->bmse <= 3 && G <= 8;
}

template <int BHI, int BLO, int NT>
cudaError_t launch_split_mma(const tq_split* sp, int B, int Hq, int64_t S, const uint8_t* ph, const uint16_t* nh,
                             const uint8_t* pl, const uint16_t* nl, float* out, const uint32_t* frags,
                             const SplitScale* hs, cudaStream_t st) {
  const int Hkv = sp->Hkv;
  const int64_t total = int64_t(B) * Hkv * ((S + 31) / 32);
  auto kern = logits_split_kernel<BHI, BLO, NT>;
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kLogitThreads, 0);
  int64_t grid = int64_t(sm_count()) * (per_sm > 0 ? per_sm : 1);
  const int64_t needed = (total + kLogitThreads / 32 - 1) / (kLogitThreads / 32);
  if (grid > needed) grid = needed;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(kLogitThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, ph, nh, pl, nl, S, Hq, Hkv, total, frags, hs, sp->hi->lut, sp->lo->lut, out);
}

template <int NT>
cudaError_t dispatch_split(const tq_split* sp, int B, int Hq, int64_t S, const uint8_t* ph, const uint16_t* nh,
                           const uint8_t* pl, const uint16_t* nl, float* out, const uint32_t* frags,
                           const SplitScale* hs, cudaStream_t st) {
  switch (sp->hi->bmse * 4 + sp->lo->bmse) {
    case 5: return launch_split_mma<1, 1, NT>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st);
    case 6: return launch_split_mma<1, 2, NT>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st);
    case 7: return launch_split_mma<1, 3, NT>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st);
    case 9: return launch_split_mma<2, 1, NT>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st);
    case 10: return launch_split_mma<2, 2, NT>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st);
    case 11: return launch_split_mma<2, 3, NT>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st);
    case 13: return launch_split_mma<3, 1, NT>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st);
    case 14: return launch_split_mma<3, 2, NT>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st);
    default: return launch_split_mma<3, 3, NT>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st);
  }
}

}  // namespace

size_t split_logits_ws_bytes(const tq_split* sp, int B, int Hq) {
  const int G = Hq / sp->Hkv;
  if (!split_fast_path(sp, G)) return 256;
  const int64_t groups = int64_t(B) * sp->Hkv;
  const int nt = (G + HPT - 1) / HPT;
  const size_t frag = size_t(groups) * nt * kFragWords * 4;
  const size_t scales = size_t(groups) * G * sizeof(SplitScale);
  return ((frag + 255) / 256) * 256 + ((scales + 255) / 256) * 256;
}

cudaError_t launch_split_logits(const tq_split* sp, const float* q, int B, int Hq, int64_t S, const uint8_t* ph,
                                const uint16_t* nh, const uint8_t* pl, const uint16_t* nl, float scale, float* out,
                                void* ws, cudaStream_t st) {
  const int Hkv = sp->Hkv, G = Hq / Hkv;
  if (!split_fast_path(sp, G)) {
    const ChannelGather ghi{sp->dperm, S > 0 ? S : 1, Hkv, sp->d, 0};
    const ChannelGather glo{sp->dperm, S > 0 ? S : 1, Hkv, sp->d, sp->hi->d};
    cudaError_t e = launch_logits_simt(sp->hi, q, B, Hq, Hkv, S, ph, nh, scale, out, ghi, 0, st);
    if (e != cudaSuccess) return e;
    return launch_logits_simt(sp->lo, q, B, Hq, Hkv, S, pl, nl, scale, out, glo, 1, st);
  }
  const int nt = (G + HPT - 1) / HPT;
  const int64_t groups = int64_t(B) * Hkv;
  uint32_t* frags = static_cast<uint32_t*>(ws);
  const size_t frag_bytes = ((size_t(groups) * nt * kFragWords * 4 + 255) / 256) * 256;
  SplitScale* hs = reinterpret_cast<SplitScale*>(static_cast<uint8_t*>(ws) + frag_bytes);
  qprep_split_kernel<<<unsigned(groups), 128, 0, st>>>(
      q, Hq, Hkv, nt, sp->dperm, sp->hi->dRt, sp->hi->dPt, sp->lo->dRt, sp->lo->dPt,
      sp->hi->bmse == 1 ? float(sp->hi->c[1]) : sp->hi->lut.inv_scale,
      sp->lo->bmse == 1 ? float(sp->lo->c[1]) : sp->lo->lut.inv_scale, scale, float(kQjlConst / sp->hi->m),
      float(kQjlConst / sp->lo->m), sp->hi->bmse == 1 ? 1 : 0, sp->lo->bmse == 1 ? 1 : 0, frags, hs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (S == 0) return cudaSuccess;
  return nt == 1 ? dispatch_split<1>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st)
                 : dispatch_split<2>(sp, B, Hq, S, ph, nh, pl, nl, out, frags, hs, st);
}

}  // namespace tq
