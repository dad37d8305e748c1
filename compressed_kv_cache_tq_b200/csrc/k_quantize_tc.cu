// Tensor-core quantize kernels for keys of d = 128 (sm_100a):
//   quantize_tc_kernel<b', JL, F32>  one context, m = 128 (JL) or m = 0 (the
//                                MSE-only variant: no JL product, no signs);
//                                bf16 keys, or fp32 keys (F32: split into bf16
//                                hi + lo on the way in, described below);
//   quantize_split_tc_kernel     the per-KV-head channel split into two
//                                64-channel groups (described further down).
//
// What it computes per key k (airosetta.com "Google TurboQuant", stage 1 and
// stage 2; mooersco.com section 1.1, the key multiplied by the rotation):
//   y = R k                      (tcgen05 MMA: K R_hi^T + K R_lo^T, fp32 in TMEM)
//   n = ||k||                    (from the key tile in shared memory, fp32)
//   idx_j = #{i : t_i < y_j / n} (Lloyd-Max cell search in registers)
//   r_rot = y / n - c[idx]       (the residual on the unit sphere, R r / n)
//   z = P r_rot                  (tcgen05 MMA, fp16 hi/lo split of r_rot and
//                                 the fp16 JL samples P, two passes, fp32 in TMEM)
//   sign_i = [z_i >= 0]          (= [(S r)_i >= 0] since S r = n P r_rot)
//   ||r|| = n ||r_rot||; both norms rounded to fp16.
//
// Precision: R = R_hi + R_lo in bf16 represents R to about 2^-17, so y / n is
// within about 4e-7 of R k / ||k|| (codes differ from exact arithmetic only
// for coordinates within that distance of a boundary); n is taken from
// ||y|| = ||R k|| (relative error about 4e-7); the JL product uses an fp16 hi +
// lo split of r_rot (scaled by 2^7) against P, which is stored exactly in fp16.
//
// Structure (one CTA per SM, persistent over 128-key tiles, two tiles in flight):
//   warp 0        : TMA producer (the constant B operands once, then key tiles
//                   into a three-deep ring)
//   warp 1        : TMEM allocation and the single-thread MMA issue, in the
//                   order MMA1(0), MMA1(1), MMA2(0), MMA1(2), MMA2(1), ...
//   warps 2 .. 17 : epilogue, two teams of eight warps; the team of TMEM slot s
//                   handles the local tiles of parity s, one thread per key row
//                   (= TMEM lane) and half of its coordinates (two quarters).
//                   While one team waits for the tensor cores (the JL product
//                   of its tile, then the rotation of its next one), the other
//                   team's cell search keeps the FMA pipes busy.
// Shared memory: B operands R_hi, R_lo, P (96 KB), three key tiles (3 x 32 KB,
// TMA 128-byte swizzle) and the two halves' per-row partial sums.
// TMEM: 512 columns, two slots of 256: y accumulates in columns 0..127 of a
// slot; the epilogue reads it and writes the residual's fp16 hi / lo pairs
// back over it (A operand of the JL product, read by the MMA from TMEM); z
// accumulates in columns 128..255.
// Without the sketch (m = 0) P is not loaded, there is no JL product, and a
// TMEM slot's y columns are released to the next rotation as soon as the
// epilogue has read them.
// Every wait on an mbarrier is bounded; a wait that gives up sets the
// context's status word, and all roles then leave their loops (there is no
// unbounded barrier between roles).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "tc_sm100.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr int kThreadsTc = 576;   // 2 control warps + 16 epilogue warps
constexpr int kTeamThreads = 256;  // epilogue threads per TMEM slot

constexpr uint32_t kOffRhi = 0, kOffRlo = 32768, kOffP = 65536;
constexpr uint32_t kConstBytes = 98304;  // R_hi, R_lo (bf16), P (fp16)
constexpr int kKeyStages = 3;            // key-tile ring depth (covers HBM latency under load)
constexpr uint32_t kOffKey = 98304;      // kKeyStages 32 KB key tiles
constexpr uint32_t kOffPn2 = kOffKey + 32768u * kKeyStages;   // [slot][parity][half][row] partial ||y||^2
constexpr uint32_t kOffPrr = kOffPn2 + 2u * 2u * 2u * 128u * 4u;  // [slot][half][row] partial ||r_rot||^2
constexpr uint32_t kOffBar = kOffPrr + 2u * 2u * 128u * 4u;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;   // + slack for 1024-byte alignment
static_assert(kSmemBytes <= 232448, "shared memory per block");

// barriers; the per-slot ones come in pairs (slot 0, slot 1)
enum Bar {
  kBarConst = 0,
  kBarKFull = 1,                        // one per key stage
  kBarKEmpty = kBarKFull + kKeyStages,
  kBarD1Full = kBarKEmpty + kKeyStages, // one per TMEM slot from here on
  kBarN2 = kBarD1Full + 2,              // both halves' partial sums of ||y||^2 written
  kBarRFull = kBarN2 + 2,               // residual in TMEM
  kBarRR = kBarRFull + 2,               // both halves' partial sums of ||r_rot||^2 written
  kBarD2Full = kBarRR + 2,
  kBarD2Free = kBarD2Full + 2,          // z read
  kNumBars = kBarD2Free + 2
};
static_assert(8 * kNumBars + 8 <= 256, "barrier area");

// fp32 keys: TMA brings 128-row x 32-column fp32 quarter tiles (16 KB, 128-byte
// swizzle) into a staging ring; two converter warps split each key into
// bf16 hi = RN(k) and lo = RN(k - hi) and write them as the A operand of one
// K half (hi 16 KB, lo 16 KB, 128-byte swizzle) into a two-entry ring; the
// rotation is then K_hi R_hi + K_hi R_lo + K_lo R_hi (K_lo R_lo is below
// 2^-18 of the product).
constexpr int kThreadsF32 = 640;    // 2 control + 2 converter + 16 epilogue warps
constexpr int kStageF32 = 3;        // fp32 quarter tiles in flight
constexpr int kRingF32 = 2;         // bf16 K halves
constexpr uint32_t kOffStageF = kConstBytes;
constexpr uint32_t kOffRingF = kOffStageF + 16384u * kStageF32;

template <bool F32>
struct QLayout {
  static constexpr int kThreads = F32 ? kThreadsF32 : kThreadsTc;
  static constexpr int kEpi0 = F32 ? 4 : 2;   // first epilogue warp
  static constexpr uint32_t kOffPn2 = F32 ? kOffRingF + 32768u * kRingF32 : kOffKey + 32768u * kKeyStages;
  static constexpr uint32_t kOffPrr = kOffPn2 + 2u * 2u * 2u * 128u * 4u;
  static constexpr uint32_t kOffBar = kOffPrr + 2u * 2u * 128u * 4u;
  static constexpr uint32_t kSmem = kOffBar + 256 + 1024;
  // barriers: constants, key pipeline (bf16: key stages; fp32: staging, then
  // the bf16 ring), then one pair per TMEM slot
  static constexpr int kStages = F32 ? kStageF32 : kKeyStages;
  static constexpr int kKFull = 1, kKEmpty = kKFull + kStages;
  static constexpr int kRingFull = kKEmpty + kStages, kRingEmpty = kRingFull + (F32 ? kRingF32 : 0);
  static constexpr int kD1Full = kRingEmpty + (F32 ? kRingF32 : 0);
  static constexpr int kN2 = kD1Full + 2, kRFull = kN2 + 2, kRR = kRFull + 2, kD2Full = kRR + 2, kD2Free = kD2Full + 2;
  static constexpr int kNumBars = kD2Free + 2;
  static_assert(kSmem <= 232448, "shared memory per block");
  static_assert(8 * kNumBars + 8 <= 256, "barrier area");
};

using namespace tc;

// Cycles a wait of this file's kernels spins before it gives up: set by
// thread 0 of each block before the first wait (the context's test budget,
// or about 2 s).  The drains before a block exits always use the full budget,
// so that no copy or MMA is in flight when shared and tensor memory are freed.
__shared__ long long g_wait_budget;

// A budget below the default (the test hook) waits by non-blocking tests, so
// that a suspended try_wait cannot outlast it.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, uint32_t* status) {
  if (g_wait_budget < tc::kWaitCycles)
    return tc::mbar_wait_polling(bar, parity, abort_flag, status, kStatusQuantizeTc, g_wait_budget);
  return tc::mbar_wait(bar, parity, abort_flag, status, kStatusQuantizeTc, g_wait_budget);
}
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                               uint32_t* status) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort_flag, status));
}
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           uint32_t* status) {
  tc::mbar_drain(bar, parity, abort_flag, status, kStatusQuantizeTc);
}

// Positive half of the symmetric codebook, scaled by 128 (the residual scale),
// pre-arranged for the arithmetic cell search below.
struct HalfBook {
  float Tneg[3];   // -2^100 x boundaries above 0 (t_{L/2} .. t_{L-2})
  float C0;        // smallest positive level
  float dC[3];     // level steps c_{L/2+i+1} - c_{L/2+i}
  // two-level search (4 positive levels): first the middle boundary, then the
  // outer (p2 = 1) or inner (p2 = 0) one; level = B + p_lo A with
  // A = dC0 + p2 (dC2 - dC0), B = C0 + p2 (C2 - C0)
  float dT31;      // -2^100 (t_{L-2} - t_{L/2}) : outer minus inner scaled boundary
  float dA;        // dC2 - dC0
  float C20;       // C2 - C0
};

constexpr float kBig = 0x1p100f;

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// Cell indices and scaled residuals of two rotated coordinates u = y s128
// (scaled by 128), with packed two-wide fused multiply-adds.  The codebook is
// symmetric with t_{L/2-1} = 0, so idx = #{i : t_i < u} = L/2 + m for u > 0
// and L/2 - 1 - m otherwise, where m = #{boundaries above 0 that are below
// |u|}.  Each indicator [|u| > T] is sat(2^100 |u| - 2^100 T): exactly 0 or 1,
// because the difference of two floats of this range is either 0 or far
// above 2^-100 (an exact tie at a boundary resolves within rounding of the
// boundary).  Returns the float bit patterns of 2^23 + (L - 1 - idx): the
// complemented index costs one operation less (L - 1 - idx = L/2 - [u > 0]
// - sign(u) m), and complementing every b-bit code of a packed word is
// complementing the word.
template <int BMSE>
__device__ __forceinline__ uint2 cell2(float2 y, float s128, const HalfBook& hb, float2& r) {
  const float2 u = __fmul2_rn(y, f2(s128));
  const float2 sp = make_float2(__saturatef(u.x * kBig), __saturatef(u.y * kBig));   // [u > 0]
  const float2 nsgn = __ffma2_rn(f2(-2.f), sp, f2(1.f));                              // -sign(u), 0 -> +1
  float2 m, lv;
  if constexpr (BMSE == 3) {
    const float2 p2 = make_float2(__saturatef(fmaf(fabsf(u.x), kBig, hb.Tneg[1])),
                                  __saturatef(fmaf(fabsf(u.y), kBig, hb.Tneg[1])));
    const float2 tsel = __ffma2_rn(p2, f2(hb.dT31), f2(hb.Tneg[0]));   // -2^100 t_outer or t_inner
    const float2 plo = make_float2(__saturatef(fmaf(fabsf(u.x), kBig, tsel.x)),
                                   __saturatef(fmaf(fabsf(u.y), kBig, tsel.y)));
    m = __ffma2_rn(p2, f2(2.f), plo);
    const float2 A = __ffma2_rn(p2, f2(hb.dA), f2(hb.dC[0]));
    const float2 B = __ffma2_rn(p2, f2(hb.C20), f2(hb.C0));
    lv = __ffma2_rn(plo, A, B);
  } else if constexpr (BMSE == 2) {
    m = make_float2(__saturatef(fmaf(fabsf(u.x), kBig, hb.Tneg[0])),
                    __saturatef(fmaf(fabsf(u.y), kBig, hb.Tneg[0])));
    lv = __ffma2_rn(m, f2(hb.dC[0]), f2(hb.C0));
  } else {
    m = make_float2(0.f, 0.f);
    lv = f2(hb.C0);
  }
  r = __ffma2_rn(nsgn, lv, u);                                                        // u - sign(u) level
  constexpr float kHalfL = float(1 << (BMSE - 1)) + 8388608.f;                        // 2^23 + L/2
  const float2 t = __ffma2_rn(sp, f2(-1.f), f2(kHalfL));
  const float2 idx = __ffma2_rn(nsgn, m, t);
  return make_uint2(__float_as_uint(idx.x), __float_as_uint(idx.y));
}

template <int BMSE, bool JL, bool F32>
__global__ void __launch_bounds__(QLayout<F32>::kThreads, 1) quantize_tc_kernel(const __grid_constant__ CUtensorMap key_map,
                                                                   int64_t n, const uint8_t* __restrict__ bimg,
                                                                   HalfBook book,
                                                                   uint8_t* __restrict__ payload,
                                                                   uint16_t* __restrict__ norms,
                                                                   uint32_t* __restrict__ status,
                                                                   long long wait_budget) {
  using QL = QLayout<F32>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;   // the swizzle pattern is anchored to 1024-byte boundaries
  uint8_t* sbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + QL::kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + QL::kOffBar + 8 * QL::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + QL::kOffBar + 8 * QL::kNumBars + 4);
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  float* pn2 = reinterpret_cast<float*>(sbase + QL::kOffPn2);
  float* prr = reinterpret_cast<float*>(sbase + QL::kOffPrr);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t num_tiles = (n + kTile - 1) / kTile;
  const int64_t my_tiles = num_tiles > blockIdx.x ? (num_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarConst), 1);
    for (int s = 0; s < QL::kStages; ++s) {
      mbar_init(bar(QL::kKFull + s), 1);
      mbar_init(bar(QL::kKEmpty + s), F32 ? 64 : 1);   // fp32: released by the two converter warps
    }
    if constexpr (F32) {
      for (int s = 0; s < kRingF32; ++s) {
        mbar_init(bar(QL::kRingFull + s), 64);         // written by the two converter warps
        mbar_init(bar(QL::kRingEmpty + s), 1);         // MMA commit
      }
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(QL::kD1Full + s), 1);
      mbar_init(bar(QL::kN2 + s), kTeamThreads);
      mbar_init(bar(QL::kRFull + s), kTeamThreads);
      mbar_init(bar(QL::kRR + s), kTeamThreads);
      mbar_init(bar(QL::kD2Full + s), 1);
      mbar_init(bar(QL::kD2Free + s), kTeamThreads);
    }
    *abort_flag = 0;
    g_wait_budget = wait_budget > 0 ? wait_budget : tc::kWaitCycles;
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
  if (warp < 2) {
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        // R_hi, R_lo and (with the sign sketch) P
        constexpr uint32_t kConst = JL ? kConstBytes : kOffP;
        mbar_expect_tx(bar(kBarConst), kConst);
        for (int c = 0; c < int(kConst / 16384u); ++c)
          bulk_load(base + 16384u * c, bimg + 16384 * c, 16384u, bar(kBarConst));
        // bf16 keys: one 32 KB tile per stage; fp32 keys: four 16 KB quarter tiles per tile
        constexpr int kPer = F32 ? 4 : 1;
        constexpr int kStg = QL::kStages;
        const int64_t loads = my_tiles * kPer;
        int64_t i = 0;
        for (; i < loads; ++i) {
          const int kb = int(i % kStg);
          if (i >= kStg && !mbar_wait(bar(QL::kKEmpty + kb), uint32_t((i / kStg - 1) & 1), abort_flag, status))
            break;
          const int64_t tile = blockIdx.x + (i / kPer) * gridDim.x;
          if constexpr (F32) {
            mbar_expect_tx(bar(QL::kKFull + kb), 16384u);
            tma_load_2d(base + kOffStageF + 16384u * kb, &key_map, 32 * int(i & 3), int(tile * kTile),
                        bar(QL::kKFull + kb));
          } else {
            const uint32_t dst = base + kOffKey + 32768u * kb;
            mbar_expect_tx(bar(QL::kKFull + kb), 32768u);
            tma_load_2d(dst, &key_map, 0, int(tile * kTile), bar(QL::kKFull + kb));
            tma_load_2d(dst + 16384u, &key_map, 64, int(tile * kTile), bar(QL::kKFull + kb));
          }
        }
        // leave no copy in flight: wait for the last loads issued to each buffer
        for (int64_t j = (i >= kStg ? i - kStg : 0); j < i; ++j)
          mbar_drain(bar(QL::kKFull + int(j % kStg)), uint32_t((j / kStg) & 1), abort_flag, status);
        mbar_drain(bar(kBarConst), 0u, abort_flag, status);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issue
      if (lane == 0) {
        auto issue_mma1 = [&](int64_t i) -> bool {
          const int sl = int(i & 1);
          if constexpr (F32) {
            // the slot's columns are free as in the bf16 case; then per K half
            // of the bf16 ring: K_hi R_hi + K_hi R_lo + K_lo R_hi
            if (i >= 2 &&
                !mbar_wait(bar((JL ? QL::kD2Full : QL::kRFull) + sl), uint32_t(((i >> 1) - 1) & 1), abort_flag,
                           status))
              return false;
            const uint32_t d1 = tmem + 256u * sl;
            uint32_t acc = 0;
            for (int kh = 0; kh < 2; ++kh) {
              const int64_t e = 2 * i + kh;
              const int rs = int(e & 1);
              if (!mbar_wait(bar(QL::kRingFull + rs), uint32_t((e >> 1) & 1), abort_flag, status)) return false;
              tc_fence_after();
              const uint32_t abase = base + kOffRingF + 32768u * rs;
              for (int pass = 0; pass < 3; ++pass)
                for (int ks = 0; ks < 4; ++ks) {
                  const uint32_t a = abase + (pass == 2 ? 16384u : 0u) + 32u * ks;
                  const uint32_t b = base + (pass == 1 ? kOffRlo : kOffRhi) + 16384u * kh + 32u * ks;
                  mma_f16(d1, smem_desc(a), smem_desc(b), kIdescBf16, acc);
                  acc = 1;
                }
              mma_commit(bar(QL::kRingEmpty + rs));
            }
            mma_commit(bar(QL::kD1Full + sl));
            return true;
          }
          const int kb = int(i % kKeyStages);
          if (!mbar_wait(bar(QL::kKFull + kb), uint32_t((i / kKeyStages) & 1), abort_flag, status)) return false;
          // the slot's y / residual columns are free once the JL MMA of tile i - 2 completed
          // (without the sign sketch: once the epilogue of tile i - 2 has read y)
          if (i >= 2 &&
              !mbar_wait(bar((JL ? QL::kD2Full : QL::kRFull) + sl), uint32_t(((i >> 1) - 1) & 1), abort_flag, status))
            return false;
          tc_fence_after();
          const uint32_t d1 = tmem + 256u * sl;
          const uint32_t kbase = base + kOffKey + 32768u * kb;
          uint32_t acc = 0;
          for (int pass = 0; pass < 2; ++pass)
            for (int kh = 0; kh < 2; ++kh)
              for (int ks = 0; ks < 4; ++ks) {
                const uint32_t off = 16384u * kh + 32u * ks;
                mma_f16(d1, smem_desc(kbase + off), smem_desc(base + (pass ? kOffRlo : kOffRhi) + off), kIdescBf16,
                        acc);
                acc = 1;
              }
          mma_commit(bar(QL::kD1Full + sl));
          mma_commit(bar(QL::kKEmpty + kb));
          return true;
        };
        auto issue_mma2 = [&](int64_t i) -> bool {
          const int sl = int(i & 1);
          if (!mbar_wait(bar(QL::kRFull + sl), uint32_t((i >> 1) & 1), abort_flag, status)) return false;
          // the slot's z columns are free once the epilogue of tile i - 2 read them
          if (i >= 2 && !mbar_wait(bar(QL::kD2Free + sl), uint32_t(((i >> 1) - 1) & 1), abort_flag, status))
            return false;
          tc_fence_after();
          const uint32_t d1 = tmem + 256u * sl, d2 = d1 + 128u;
          uint32_t acc = 0;
          for (int pass = 0; pass < 2; ++pass) {          // z = r_hi P^T + r_lo P^T
            const uint32_t a_lo = pass == 1 ? 16u : 0u;
            for (int k = 0; k < 8; ++k) {
              // residual coordinates 16k .. 16k+15: chunk k/2, half k%2 (8 columns of packed pairs)
              const uint32_t a_tmem = d1 + 32u * uint32_t(k >> 1) + 8u * uint32_t(k & 1) + a_lo;
              const uint32_t off = 16384u * uint32_t(k >> 2) + 32u * uint32_t(k & 3);
              mma_f16_ts(d2, a_tmem, smem_desc(base + kOffP + off), kIdescF16, acc);
              acc = 1;
            }
          }
          mma_commit(bar(QL::kD2Full + sl));
          return true;
        };
        int64_t n1 = 0, n2 = 0;   // rotation / JL MMA groups issued
        bool ok = mbar_wait(bar(kBarConst), 0u, abort_flag, status);
        if (ok && my_tiles > 0) {
          ok = issue_mma1(0);
          n1 += ok;
        }
        for (int64_t i = 0; ok && i < my_tiles; ++i) {
          if (i + 1 < my_tiles) {
            if (!issue_mma1(i + 1)) break;
            ++n1;
          }
          if constexpr (JL) {
            if (!issue_mma2(i)) break;
            ++n2;
          }
        }
        // before TMEM is released: the commit of the last group of each kind
        // tracks every MMA issued before it
        if (n1 > 0) mbar_drain(bar(QL::kD1Full + int((n1 - 1) & 1)), uint32_t(((n1 - 1) >> 1) & 1), abort_flag, status);
        if (n2 > 0) mbar_drain(bar(QL::kD2Full + int((n2 - 1) & 1)), uint32_t(((n2 - 1) >> 1) & 1), abort_flag, status);
      }
    }
  } else if (F32 && warp < 4) {
    // ------------------------------------------------------------ fp32 -> bf16 hi / lo converter
    // quarter tile j (tile j / 4, columns 32 (j % 4) ..): row r, 8-float group
    // g of the staging tile -> 16-byte chunk 4 (j % 2) + g of row r of K half
    // (j % 4) / 2 of the ring entry (both 128-byte swizzled)
    const int c = threadIdx.x - 64;
    const int64_t loads = 4 * my_tiles;
    for (int64_t j = 0; j < loads; ++j) {
      const int sb = int(j % kStageF32);
      const int q = int(j & 3);
      const int64_t e = j >> 1;             // ring entry use: (tile, K half)
      const int rs = int(e & 1);
      if ((q & 1) == 0 && e >= 2 &&
          !mbar_wait_warp(bar(QL::kRingEmpty + rs), uint32_t(((e >> 1) - 1) & 1), abort_flag, status))
        break;
      if (!mbar_wait_warp(bar(QL::kKFull + sb), uint32_t((j / kStageF32) & 1), abort_flag, status)) break;
      const uint8_t* src = sbase + kOffStageF + 16384u * sb;
      uint8_t* dst = sbase + kOffRingF + 32768u * rs;
      // thread c converts rows c / 4 + 16 u (u = 0..7) of 8-float group c % 4, four
      // rows' loads issued before their conversions and stores (the swizzle of
      // those rows is the same: r % 8 = (c / 4) % 8)
      const int r0 = c >> 2, g = c & 3, sw = r0 & 7;
#pragma unroll
      for (int b4 = 0; b4 < 2; ++b4) {
        float4 va[4], vb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = r0 + 16 * (4 * b4 + u);
          va[u] = *reinterpret_cast<const float4*>(src + r * 128 + (((2 * g) ^ sw) << 4));
          vb[u] = *reinterpret_cast<const float4*>(src + r * 128 + (((2 * g + 1) ^ sw) << 4));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = r0 + 16 * (4 * b4 + u);
          const float2 x[4] = {make_float2(va[u].x, va[u].y), make_float2(va[u].z, va[u].w), make_float2(vb[u].x, vb[u].y),
                               make_float2(vb[u].z, vb[u].w)};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const __nv_bfloat162 h = __float22bfloat162_rn(x[t]);
            const float2 hf = __bfloat1622float2(h);
            const __nv_bfloat162 l = __float22bfloat162_rn(__ffma2_rn(hf, f2(-1.f), x[t]));
            hi[t] = *reinterpret_cast<const uint32_t*>(&h);
            lo[t] = *reinterpret_cast<const uint32_t*>(&l);
          }
          const uint32_t off = uint32_t(r * 128 + (((4 * (q & 1) + g) ^ sw) << 4));
          *reinterpret_cast<uint4*>(dst + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(dst + 16384u + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      // the tensor core reads the ring through the async proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(bar(QL::kKEmpty + sb));
      if (q & 1) mbar_arrive(bar(QL::kRingFull + rs));
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w (e = w - first epilogue warp): team (TMEM slot) (e >> 2) & 1,
    // half e >> 3 (quarters 2 half and 2 half + 1 of every row), TMEM lanes
    // 32 (w & 3) .. +31.
    const int eg = (warp - QL::kEpi0) >> 2;
    const int slot = eg & 1, half = eg >> 1;
    const int row = (warp & 3) * 32 + lane;          // TMEM lane = key row within the tile
    const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
    const uint32_t d1 = tmem + 256u * slot + lane_addr, d2 = d1 + 128u;
    constexpr int kW = BMSE + (JL ? 1 : 0);          // words per quarter chunk
    constexpr int kRowBytes = 16 * kW;               // kD BMSE / 8 (+ kD / 8 sign bytes)
    const int q0 = 2 * half;
    float* rrbuf = prr + slot * 256;
    int64_t k = 0;
    for (int64_t i = slot; i < my_tiles; i += 2, ++k) {
      const uint32_t par = uint32_t(k & 1);
      if (!mbar_wait_warp(bar(QL::kD1Full + slot), par, abort_flag, status)) break;
      tc_fence_after();
      // ||k||^2 = ||R k||^2 from the rotated row, half a row per half-team; the
      // partial sums alternate between two buffers, so that a half that runs
      // ahead never overwrites sums the other half has not read yet
      float* n2buf = pn2 + (slot * 2 + int(par)) * 256;
      {
        // both quarters loaded before one wait (one TMEM round trip)
        float y0[32], y1[32];
        tmem_ld32(d1 + 32u * q0, y0);
        tmem_ld32(d1 + 32u * (q0 + 1), y1);
        tmem_wait32(y0);
        tmem_wait32(y1);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          acc = __ffma2_rn(make_float2(y0[j], y0[j + 1]), make_float2(y0[j], y0[j + 1]), acc);
          acc = __ffma2_rn(make_float2(y1[j], y1[j + 1]), make_float2(y1[j], y1[j + 1]), acc);
        }
        n2buf[half * 128 + row] = acc.x + acc.y;
      }
      mbar_arrive(bar(QL::kN2 + slot));
      if (!mbar_wait_warp(bar(QL::kN2 + slot), par, abort_flag, status)) break;
      const float n2 = n2buf[row] + n2buf[128 + row];
      const float nk = sqrtf(n2);
      const bool zero = !(n2 > 0.f);
      const float s128 = zero ? 0.f : 128.f / nk;
      HalfBook hb = book;
      if (zero) {
        hb.C0 = 0.f;
#pragma unroll
        for (int c = 0; c < 3; ++c) hb.dC[c] = 0.f;
        hb.dA = 0.f;
        hb.C20 = 0.f;
      }
      float2 rr2 = make_float2(0.f, 0.f);
      uint32_t cw[2][BMSE];
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int q = q0 + qq;
        float y[32];
        tmem_ld32(d1 + 32u * q, y);
        tmem_wait32(y);
        uint32_t hw[2 * BMSE], hw3[2] = {0u, 0u};
#pragma unroll
        for (int h = 0; h < 2 * BMSE; ++h) hw[h] = 0;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t rh[8], rl[8];
#pragma unroll
          for (int jp = 0; jp < 16; jp += 2) {
            const int j0 = 16 * hh + jp;
            float2 rp;
            const uint2 bb = cell2<BMSE>(make_float2(y[j0], y[j0 + 1]), s128, hb, rp);
            rr2 = __ffma2_rn(rp, rp, rr2);
            const __half2 hi = __float22half2_rn(rp);
            const float2 hf = __half22float2(hi);
            const __half2 lo = __float22half2_rn(__ffma2_rn(hf, f2(-1.f), rp));
            rh[jp >> 1] = *reinterpret_cast<const uint32_t*>(&hi);
            rl[jp >> 1] = *reinterpret_cast<const uint32_t*>(&lo);
#pragma unroll
            for (int t2 = 0; t2 < 2; ++t2) {
              // bits = float pattern of 2^23 + code: the code in bits 0..2, the
              // constant part only reaches bits >= 24 of each shifted term
              const int jc = j0 + t2;
              const uint32_t bits = t2 ? bb.y : bb.x;
              const int rreg = jc >> 2, e = jc & 3, uu = rreg >> 2, ii = rreg & 3;
              if constexpr (BMSE == 3) {
                if (ii < 3)
                  hw[uu * 3 + ii] += bits << (4 * e);
                else
                  hw3[uu] += bits << (4 * e);     // spread into bit 3 of H0..H2 below
              } else if constexpr (BMSE == 2) {
                hw[uu * 2 + (ii >> 1)] += bits << (4 * e + 2 * (ii & 1));
              } else {
                hw[uu] += bits << (4 * e + ii);
              }
            }
          }
          // the residual overwrites the columns of y just read (A operand of the JL product):
          // coordinates 32q + 16hh .. +15 -> hi pairs at column 32q + 8hh, lo pairs 16 further
          if constexpr (JL) {
            tmem_st8(d1 + 32u * q + 8u * hh, rh);
            tmem_st8(d1 + 32u * q + 16u + 8u * hh, rl);
          }
        }
        if constexpr (BMSE == 3) {
#pragma unroll
          for (int uu = 0; uu < 2; ++uu)
#pragma unroll
            for (int b = 0; b < 3; ++b) hw[uu * 3 + b] |= ((hw3[uu] >> b) & 0x1111u) << 3;
        }
#pragma unroll
        for (int w = 0; w < BMSE; ++w) cw[qq][w] = zero ? 0u : ~__byte_perm(hw[2 * w], hw[2 * w + 1], 0x5410);
      }
      if constexpr (JL) asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(bar(QL::kRFull + slot));   // residual in TMEM (without the sketch: y read)
      rrbuf[half * 128 + row] = rr2.x + rr2.y;
      mbar_arrive(bar(QL::kRR + slot));
      uint32_t sw[2] = {0u, 0u};
      if constexpr (JL) {
      if (!mbar_wait_warp(bar(QL::kD2Full + slot), par, abort_flag, status)) break;
      tc_fence_after();
      // bit = [z >= 0] = not the sign bit (z = -0 cannot arise for a nonzero
      // residual; zero keys get all ones).  Bit p of quarter q's word holds
      // coordinate 32q + 16 (p >> 4) + 4 (p & 3) + ((p >> 2) & 3); the bits are
      // shifted in from the top, p = 31 first.
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        uint32_t neg = 0;
#pragma unroll
        for (int hz = 1; hz >= 0; --hz) {   // coordinates 32q + 16hz .. +15 fill bits 16hz .. 16hz + 15
          float z[16];
          tmem_ld16(d2 + 32u * (q0 + qq) + 16u * hz, z);
          tmem_wait16(z);
#pragma unroll
          for (int p = 15; p >= 0; --p) {
            const int jj = 4 * (p & 3) + ((p >> 2) & 3);
            neg = __funnelshift_l(__float_as_uint(z[jj]), neg, 1);
          }
        }
        sw[qq] = zero ? 0xFFFFFFFFu : ~neg;
      }
      tc_fence_before();
      mbar_arrive(bar(QL::kD2Free + slot));
      }
      const int64_t key = (blockIdx.x + i * gridDim.x) * kTile + row;
      if (key < n) {
        // this half's two quarter chunks
        uint32_t wv[2 * kW];
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
#pragma unroll
          for (int w = 0; w < BMSE; ++w) wv[qq * kW + w] = cw[qq][w];
          if constexpr (JL) wv[qq * kW + BMSE] = sw[qq];
        }
        uint8_t* dst = payload + key * kRowBytes + q0 * 4 * kW;
        if constexpr (kW % 2 == 0) {   // 16-byte aligned half rows
#pragma unroll
          for (int v = 0; v < kW / 2; ++v)
            reinterpret_cast<uint4*>(dst)[v] = make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
        } else {                       // 8-byte aligned
#pragma unroll
          for (int v = 0; v < kW; ++v) reinterpret_cast<uint2*>(dst)[v] = make_uint2(wv[2 * v], wv[2 * v + 1]);
        }
      }
      if (half == 0) {
        // ||r|| = n ||r_rot|| from both halves' sums (r_rot scaled by 128); the
        // other half writes these sums again only after its next N2 wait, which
        // needs this thread's next arrival
        if (!mbar_wait_warp(bar(QL::kRR + slot), par, abort_flag, status)) break;
        const float rho = nk * sqrtf(rrbuf[row] + rrbuf[128 + row]) * (1.0f / 128.f);
        const uint32_t nn = uint32_t(__half_as_ushort(__float2half_rn(nk))) |
                            (uint32_t(__half_as_ushort(__float2half_rn(rho))) << 16);
        if (key < n) {
          reinterpret_cast<uint32_t*>(norms)[key] = nn;
          flag_norm_range(nn, status);
        }
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

// ---------------------------------------------------------------------------
// Split quantize: keys of d = 128 channels split per KV head into a high and a
// low group of 64 channels, each group a d = m = 64 quantizer of its own.  The
// pipeline is the one above with two operands changed: the rotation operand
// is the head's M_h (M_h k = (R_hi k_hi, R_lo k_lo): both groups' rotations
// of the gathered key in one product, the gather folded into the columns of
// M_h), and the JL operand is diag(P_hi, P_lo).  Rotated coordinates 0..63
// belong to the high group and 64..127 to the low group.  Each epilogue
// thread takes one quarter of each group (so both halves run the same code,
// which keeps the instruction footprint of one epilogue), and the halves
// combine their partial group norms and residual norms through shared memory
// as the single-context kernel does.  Each CTA serves one KV head, so it loads
// the head's operand once.
// ---------------------------------------------------------------------------

struct SplitGeom {
  int64_t S;     // keys per (batch, KV head) pair
  int64_t tps;   // 128-key tiles per pair
  int Hkv, head, cph, sub;   // KV heads, this CTA's head, CTAs per head, index among them
};

// Shared memory of the split kernel: the single-context layout up to the key
// ring, then per-group partial sums exchanged between the epilogue halves.
constexpr uint32_t kOffSPn2 = kOffPn2;                                    // [slot][parity][half][group][row] ||y_g||^2
constexpr uint32_t kOffSPrr = kOffSPn2 + 2u * 2u * 2u * 2u * 128u * 4u;   // [slot][half][group][row] ||r_g||^2
constexpr uint32_t kOffSBar = kOffSPrr + 2u * 2u * 2u * 128u * 4u;
constexpr uint32_t kSmemSplit = kOffSBar + 256 + 1024;
static_assert(kSmemSplit <= 232448, "shared memory per block");

// One 32-coordinate quarter q of a group (b' = BM): cells, residual to TMEM
// (fp16 hi / lo pairs over the columns of y), and the code halfwords of the
// group's chunks 2 (q & 1) and 2 (q & 1) + 1.  Returns the quarter's part of
// ||r_rot||^2 (scaled by 128^2).
template <int BM>
__device__ __forceinline__ float split_quarter(uint32_t d1, int q, float s128, bool zero, const HalfBook& hb,
                                               uint32_t (&chw)[2][BM]) {
  float y[32];
  tmem_ld32(d1 + 32u * q, y);
  tmem_wait32(y);
  float2 rr2 = make_float2(0.f, 0.f);
  uint32_t hw[2 * BM], hw3[2] = {0u, 0u};
#pragma unroll
  for (int h = 0; h < 2 * BM; ++h) hw[h] = 0;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    uint32_t rh[8], rl[8];
#pragma unroll
    for (int jp = 0; jp < 16; jp += 2) {
      const int j0 = 16 * hh + jp;
      float2 rp;
      const uint2 bb = cell2<BM>(make_float2(y[j0], y[j0 + 1]), s128, hb, rp);
      rr2 = __ffma2_rn(rp, rp, rr2);
      const __half2 hi = __float22half2_rn(rp);
      const float2 hf = __half22float2(hi);
      const __half2 lo = __float22half2_rn(__ffma2_rn(hf, f2(-1.f), rp));
      rh[jp >> 1] = *reinterpret_cast<const uint32_t*>(&hi);
      rl[jp >> 1] = *reinterpret_cast<const uint32_t*>(&lo);
#pragma unroll
      for (int t2 = 0; t2 < 2; ++t2) {
        // quarter coordinate jc: chunk unit uu, register ii, nibble e
        const int jc = j0 + t2;
        const uint32_t bits = t2 ? bb.y : bb.x;
        const int rreg = jc >> 2, e = jc & 3, uu = rreg >> 2, ii = rreg & 3;
        if constexpr (BM == 3) {
          if (ii < 3)
            hw[uu * 3 + ii] += bits << (4 * e);
          else
            hw3[uu] += bits << (4 * e);
        } else if constexpr (BM == 2) {
          hw[uu * 2 + (ii >> 1)] += bits << (4 * e + 2 * (ii & 1));
        } else {
          hw[uu] += bits << (4 * e + ii);
        }
      }
    }
    tmem_st8(d1 + 32u * q + 8u * hh, rh);
    tmem_st8(d1 + 32u * q + 16u + 8u * hh, rl);
  }
  if constexpr (BM == 3) {
#pragma unroll
    for (int uu = 0; uu < 2; ++uu)
#pragma unroll
      for (int b = 0; b < 3; ++b) hw[uu * 3 + b] |= ((hw3[uu] >> b) & 0x1111u) << 3;
  }
  // the low halfword of each sum holds the complemented codes
#pragma unroll
  for (int uu = 0; uu < 2; ++uu)
#pragma unroll
    for (int w = 0; w < BM; ++w) chw[uu][w] = zero ? 0u : (~hw[uu * BM + w]) & 0xFFFFu;
  return rr2.x + rr2.y;
}

// Sign word of z quarter q: bit p = sign coordinate 32 (q & 1) + 16 (p >> 4)
// + 4 (p & 3) + ((p >> 2) & 3) of the group, i.e. the sign halfwords of the
// group's chunks 2 (q & 1) (low half) and 2 (q & 1) + 1 (high half).
__device__ __forceinline__ uint32_t split_signs(uint32_t d2, int q, bool zero) {
  uint32_t neg = 0;
#pragma unroll
  for (int hz = 1; hz >= 0; --hz) {
    float z[16];
    tmem_ld16(d2 + 32u * q + 16u * hz, z);
    tmem_wait16(z);
#pragma unroll
    for (int p = 15; p >= 0; --p) {
      const int jj = 4 * (p & 3) + ((p >> 2) & 3);
      neg = __funnelshift_l(__float_as_uint(z[jj]), neg, 1);
    }
  }
  return zero ? 0xFFFFFFFFu : ~neg;
}

// This half's part of a group row: chunks 2 half and 2 half + 1, each BM code
// halfwords then the sign halfword; BM + 1 words at byte 4 half (BM + 1).
template <int BM>
__device__ __forceinline__ void split_store(uint8_t* row, int half, const uint32_t (&chw)[2][BM], uint32_t sw) {
  uint32_t hv[2 * (BM + 1)];
#pragma unroll
  for (int uu = 0; uu < 2; ++uu) {
#pragma unroll
    for (int w = 0; w < BM; ++w) hv[uu * (BM + 1) + w] = chw[uu][w];
    hv[uu * (BM + 1) + BM] = (sw >> (16 * uu)) & 0xFFFFu;
  }
  uint32_t wv[BM + 1];
#pragma unroll
  for (int x = 0; x < BM + 1; ++x) wv[x] = hv[2 * x] | (hv[2 * x + 1] << 16);
  uint8_t* dst = row + 4 * half * (BM + 1);
  if constexpr (BM == 3) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  } else if constexpr (BM == 1) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(wv[0], wv[1]);
  } else {
#pragma unroll
    for (int x = 0; x < BM + 1; ++x) reinterpret_cast<uint32_t*>(dst)[x] = wv[x];
  }
}

// Epilogue of the split kernel: every thread takes quarter `half` of the high
// group (TMEM columns 32 half ..) and quarter `half` of the low group (64 +
// 32 half ..), so both halves run the same code; the group norms and residual
// norms combine the two halves' partial sums through shared memory, as in the
// single-context kernel.
template <int BHI, int BLO>
__device__ __forceinline__ void split_epilogue(uint32_t bar0, uint32_t d1, uint32_t d2, int slot, int half, int row,
                                               int64_t my_tiles, const SplitGeom& sg, const HalfBook& book_hi,
                                               const HalfBook& book_lo, uint8_t* __restrict__ payload_hi,
                                               uint16_t* __restrict__ norms_hi, uint8_t* __restrict__ payload_lo,
                                               uint16_t* __restrict__ norms_lo, float* pn2, float* prr,
                                               volatile int* abort_flag, uint32_t* status) {
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  float* rrbuf = prr + slot * 512;
  const int qh = half, ql = 2 + half;   // this thread's quarter of each group
  int64_t k = 0;
  for (int64_t i = slot; i < my_tiles; i += 2, ++k) {
    const uint32_t par = uint32_t(k & 1);
    if (!mbar_wait_warp(bar(kBarD1Full + slot), par, abort_flag, status)) break;
    tc_fence_after();
    // partial ||y_g||^2 of both groups; double-buffered by tile parity, so a
    // half that runs ahead never overwrites sums the other half still reads
    float* n2buf = pn2 + (slot * 2 + int(par)) * 512;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      float y[32];
      tmem_ld32(d1 + 32u * (g ? ql : qh), y);
      tmem_wait32(y);
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 32; j += 2)
        acc = __ffma2_rn(make_float2(y[j], y[j + 1]), make_float2(y[j], y[j + 1]), acc);
      n2buf[(half * 2 + g) * 128 + row] = acc.x + acc.y;
    }
    mbar_arrive(bar(kBarN2 + slot));
    if (!mbar_wait_warp(bar(kBarN2 + slot), par, abort_flag, status)) break;
    float nk[2], s128[2];
    bool zero[2];
    HalfBook hb[2] = {book_hi, book_lo};
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const float n2 = n2buf[g * 128 + row] + n2buf[(2 + g) * 128 + row];
      nk[g] = sqrtf(n2);
      zero[g] = !(n2 > 0.f);
      s128[g] = zero[g] ? 0.f : 128.f / nk[g];
      if (zero[g]) {
        hb[g].C0 = 0.f;
#pragma unroll
        for (int c = 0; c < 3; ++c) hb[g].dC[c] = 0.f;
        hb[g].dA = 0.f;
        hb[g].C20 = 0.f;
      }
    }
    uint32_t chi[2][BHI], clo[2][BLO];
    const float rr_hi = split_quarter<BHI>(d1, qh, s128[0], zero[0], hb[0], chi);
    const float rr_lo = split_quarter<BLO>(d1, ql, s128[1], zero[1], hb[1], clo);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    tc_fence_before();
    mbar_arrive(bar(kBarRFull + slot));
    rrbuf[(half * 2 + 0) * 128 + row] = rr_hi;
    rrbuf[(half * 2 + 1) * 128 + row] = rr_lo;
    mbar_arrive(bar(kBarRR + slot));
    if (!mbar_wait_warp(bar(kBarD2Full + slot), par, abort_flag, status)) break;
    tc_fence_after();
    const uint32_t sw_hi = split_signs(d2, qh, zero[0]);
    const uint32_t sw_lo = split_signs(d2, ql, zero[1]);
    tc_fence_before();
    mbar_arrive(bar(kBarD2Free + slot));
    const int64_t t = sg.sub + i * sg.cph;
    const int64_t b = t / sg.tps, st = t - b * sg.tps;
    const int64_t s = st * kTile + row;
    const bool valid = s < sg.S;
    const int64_t key = (b * sg.Hkv + sg.head) * sg.S + s;
    if (valid) {
      split_store<BHI>(payload_hi + key * (8 * (BHI + 1)), half, chi, sw_hi);
      split_store<BLO>(payload_lo + key * (8 * (BLO + 1)), half, clo, sw_lo);
    }
    // both halves' residual sums of this tile: half 0 writes the high group's
    // norms, half 1 the low group's.  A half rewrites these sums only after its
    // next N2 wait, which needs the other half's next arrival.
    if (!mbar_wait_warp(bar(kBarRR + slot), par, abort_flag, status)) break;
    const int g = half;
    const float rho = nk[g] * sqrtf(rrbuf[g * 128 + row] + rrbuf[(2 + g) * 128 + row]) * (1.0f / 128.f);
    if (valid) {
      uint16_t* nr = g ? norms_lo : norms_hi;
      const uint32_t nn = uint32_t(__half_as_ushort(__float2half_rn(nk[g]))) |
                          (uint32_t(__half_as_ushort(__float2half_rn(rho))) << 16);
      reinterpret_cast<uint32_t*>(nr)[key] = nn;
      flag_norm_range(nn, status);
    }
  }
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");   // none in flight on an early exit
}

template <int BHI, int BLO>
__global__ void __launch_bounds__(kThreadsTc, 1) quantize_split_tc_kernel(
    const __grid_constant__ CUtensorMap key_map, int B, int Hkv, int64_t S, int cph,
    const uint8_t* __restrict__ dimg, HalfBook book_hi, HalfBook book_lo, uint8_t* __restrict__ payload_hi,
    uint16_t* __restrict__ norms_hi, uint8_t* __restrict__ payload_lo, uint16_t* __restrict__ norms_lo,
    uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + kOffSBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kOffSBar + 8 * kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kOffSBar + 8 * kNumBars + 4);
  float* pn2 = reinterpret_cast<float*>(sbase + kOffSPn2);
  float* prr = reinterpret_cast<float*>(sbase + kOffSPrr);
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  SplitGeom sg;
  sg.S = S;
  sg.tps = (S + kTile - 1) / kTile;
  sg.Hkv = Hkv;
  sg.head = int(blockIdx.x) / cph;
  sg.cph = cph;
  sg.sub = int(blockIdx.x) - sg.head * cph;
  const int64_t head_tiles = int64_t(B) * sg.tps;
  const int64_t my_tiles = head_tiles > sg.sub ? (head_tiles - sg.sub + cph - 1) / cph : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarConst), 1);
    for (int st = 0; st < kKeyStages; ++st) {
      mbar_init(bar(kBarKFull + st), 1);
      mbar_init(bar(kBarKEmpty + st), 1);
    }
    for (int sl = 0; sl < 2; ++sl) {
      mbar_init(bar(kBarD1Full + sl), 1);
      mbar_init(bar(kBarN2 + sl), kTeamThreads);
      mbar_init(bar(kBarRFull + sl), kTeamThreads);
      mbar_init(bar(kBarRR + sl), kTeamThreads);
      mbar_init(bar(kBarD2Full + sl), 1);
      mbar_init(bar(kBarD2Free + sl), kTeamThreads);
    }
    *abort_flag = 0;
    g_wait_budget = tc::kWaitCycles;
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
    if (lane == 0) {
      mbar_expect_tx(bar(kBarConst), kConstBytes);
      const uint8_t* himg = dimg + size_t(sg.head) * 65536;   // M_h hi, lo
      const uint8_t* pimg = dimg + size_t(Hkv) * 65536;       // diag(P_hi, P_lo)
      for (int c = 0; c < 4; ++c) bulk_load(base + kOffRhi + 16384u * c, himg + 16384 * c, 16384u, bar(kBarConst));
      for (int c = 0; c < 2; ++c) bulk_load(base + kOffP + 16384u * c, pimg + 16384 * c, 16384u, bar(kBarConst));
      int64_t i = 0;
      for (; i < my_tiles; ++i) {
        const int kb = int(i % kKeyStages);
        if (i >= kKeyStages &&
            !mbar_wait(bar(kBarKEmpty + kb), uint32_t((i / kKeyStages - 1) & 1), abort_flag, status))
          break;
        const int64_t t = sg.sub + i * cph;
        const int64_t b = t / sg.tps, st = t - b * sg.tps;
        const int pair = int(b * Hkv + sg.head);
        const uint32_t dst = base + kOffKey + 32768u * kb;
        mbar_expect_tx(bar(kBarKFull + kb), 32768u);
        tma_load_3d(dst, &key_map, 0, int(st * kTile), pair, bar(kBarKFull + kb));
        tma_load_3d(dst + 16384u, &key_map, 64, int(st * kTile), pair, bar(kBarKFull + kb));
      }
      for (int64_t j = (i >= kKeyStages ? i - kKeyStages : 0); j < i; ++j)
        mbar_drain(bar(kBarKFull + int(j % kKeyStages)), uint32_t((j / kKeyStages) & 1), abort_flag, status);
      mbar_drain(bar(kBarConst), 0u, abort_flag, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      auto issue_mma1 = [&](int64_t i) -> bool {
        const int sl = int(i & 1);
        const int kb = int(i % kKeyStages);
        if (!mbar_wait(bar(kBarKFull + kb), uint32_t((i / kKeyStages) & 1), abort_flag, status)) return false;
        if (i >= 2 && !mbar_wait(bar(kBarD2Full + sl), uint32_t(((i >> 1) - 1) & 1), abort_flag, status))
          return false;
        tc_fence_after();
        const uint32_t d1 = tmem + 256u * sl;
        const uint32_t kbase = base + kOffKey + 32768u * kb;
        uint32_t acc = 0;
        for (int pass = 0; pass < 2; ++pass)
          for (int kh = 0; kh < 2; ++kh)
            for (int ks = 0; ks < 4; ++ks) {
              const uint32_t off = 16384u * kh + 32u * ks;
              mma_f16(d1, smem_desc(kbase + off), smem_desc(base + (pass ? kOffRlo : kOffRhi) + off), kIdescBf16,
                      acc);
              acc = 1;
            }
        mma_commit(bar(kBarD1Full + sl));
        mma_commit(bar(kBarKEmpty + kb));
        return true;
      };
      auto issue_mma2 = [&](int64_t i) -> bool {
        const int sl = int(i & 1);
        if (!mbar_wait(bar(kBarRFull + sl), uint32_t((i >> 1) & 1), abort_flag, status)) return false;
        if (i >= 2 && !mbar_wait(bar(kBarD2Free + sl), uint32_t(((i >> 1) - 1) & 1), abort_flag, status))
          return false;
        tc_fence_after();
        const uint32_t d1 = tmem + 256u * sl, d2 = d1 + 128u;
        uint32_t acc = 0;
        for (int pass = 0; pass < 2; ++pass) {
          const uint32_t a_lo = pass == 1 ? 16u : 0u;
          for (int k = 0; k < 8; ++k) {
            const uint32_t a_tmem = d1 + 32u * uint32_t(k >> 1) + 8u * uint32_t(k & 1) + a_lo;
            const uint32_t off = 16384u * uint32_t(k >> 2) + 32u * uint32_t(k & 3);
            mma_f16_ts(d2, a_tmem, smem_desc(base + kOffP + off), kIdescF16, acc);
            acc = 1;
          }
        }
        mma_commit(bar(kBarD2Full + sl));
        return true;
      };
      int64_t n1 = 0, n2 = 0;
      bool ok = mbar_wait(bar(kBarConst), 0u, abort_flag, status);
      if (ok && my_tiles > 0) {
        ok = issue_mma1(0);
        n1 += ok;
      }
      for (int64_t i = 0; ok && i < my_tiles; ++i) {
        if (i + 1 < my_tiles) {
          if (!issue_mma1(i + 1)) break;
          ++n1;
        }
        if (!issue_mma2(i)) break;
        ++n2;
      }
      if (n1 > 0) mbar_drain(bar(kBarD1Full + int((n1 - 1) & 1)), uint32_t(((n1 - 1) >> 1) & 1), abort_flag, status);
      if (n2 > 0) mbar_drain(bar(kBarD2Full + int((n2 - 1) & 1)), uint32_t(((n2 - 1) >> 1) & 1), abort_flag, status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w: TMEM slot ((w - 2) >> 2) & 1, half (w - 2) >> 3
    const int eg = (warp - 2) >> 2;
    const int slot = eg & 1, half = eg >> 1;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
    const uint32_t d1 = tmem + 256u * slot + lane_addr, d2 = d1 + 128u;
    split_epilogue<BHI, BLO>(bar0, d1, d2, slot, half, row, my_tiles, sg, book_hi, book_lo, payload_hi, norms_hi,
                             payload_lo, norms_lo, pn2, prr, abort_flag, status);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// ---------------------------------------------------------------------------
// Wide quantizer: 192 < d <= 256 with m = d (the vector-search workload's
// d = 200), fp32 keys.  The layout has dp = mp = 256 slots (four quarters of
// 64); the products run over Np = d rounded up to 16 output coordinates and
// input coordinates (13 k-steps at d = 200).  R_hi, R_lo (bf16) and P (fp16)
// padded with zeros do not fit in shared memory at this size (3 x 104 KB), so
// they stream from L2 as 64-column atoms (Np rows of 128 bytes) through a
// three-entry ring, in the order the MMA issuer uses them: per key tile
// R_hi / R_lo of atoms 0..3 for the rotation, then P of atoms 0..3 for the
// JL product.  One tile at a time in tensor memory: y (then the residual's
// fp16 hi / lo pairs) in columns [0, Np), z in [256, 256 + Np).
//   warp 0     : TMA producer (fp32 quarter tiles, operand atoms)
//   warp 1     : TMEM allocation, single-thread MMA issue
//   warps 2, 3 : fp32 -> bf16 hi / lo converters (as in the fp32 path above)
//   warps 4..19: epilogue, thread (key row, quarter): 64 layout slots of a row
// Slots past d get code 0, sign bit 0 and no residual (the layout's padding).
// ---------------------------------------------------------------------------
constexpr int kWThreads = 640;
constexpr int kWStage = 3;                      // fp32 quarter tiles (128 x 32, 16 KB)
constexpr int kWRing = 2;                       // bf16 key atoms (hi 16 KB + lo 16 KB)
constexpr int kWBRing = 3;                      // operand atoms (up to 256 rows x 128 B)
constexpr uint32_t kWOffStage = 0;
constexpr uint32_t kWOffRing = kWOffStage + 16384u * kWStage;
constexpr uint32_t kWOffB = kWOffRing + 32768u * kWRing;
constexpr uint32_t kWBAtomMax = 256u * 128u;
constexpr uint32_t kWOffN2 = kWOffB + kWBAtomMax * kWBRing;   // [parity][quarter][row] partial ||y||^2
constexpr uint32_t kWOffRR = kWOffN2 + 2u * 4u * 128u * 4u;   // [parity][quarter][row] partial ||r_rot||^2
constexpr uint32_t kWOffBar = kWOffRR + 2u * 4u * 128u * 4u;
constexpr uint32_t kWSmem = kWOffBar + 256 + 1024;
static_assert(kWSmem <= 232448, "shared memory per block");

enum WBar {
  kWSFull = 0,                          // staging quarter tiles
  kWSEmpty = kWSFull + kWStage,
  kWRFull = kWSEmpty + kWStage,         // bf16 key atoms
  kWREmpty = kWRFull + kWRing,
  kWBFull = kWREmpty + kWRing,          // operand atoms
  kWBEmpty = kWBFull + kWBRing,
  kWD1Full = kWBEmpty + kWBRing,        // y in TMEM
  kWN2 = kWD1Full + 1,                  // all quarters' partial ||y||^2 written
  kWResid = kWN2 + 1,                   // residual in TMEM
  kWD2Full = kWResid + 1,               // z in TMEM
  kWD2Free = kWD2Full + 1,              // z read
  kWRR = kWD2Free + 1,                  // all quarters' partial ||r_rot||^2 written
  kWNumBars = kWRR + 1
};
static_assert(8 * kWNumBars + 8 <= 256, "barrier area");

// Bits of the stored words that belong to slots below d, per quarter: code
// words (2 b' per quarter) and sign words (2 per quarter).
struct WideMasks {
  uint32_t code[4][6];
  uint32_t sign[4][2];
};

template <int BMSE>
__global__ void __launch_bounds__(kWThreads, 1) quantize_wide_kernel(const __grid_constant__ CUtensorMap key_map,
                                                                     int64_t n, int d, int np,
                                                                     const uint8_t* __restrict__ bimg,
                                                                     HalfBook book,
                                                                     const __grid_constant__ WideMasks masks,
                                                                     uint8_t* __restrict__ payload,
                                                                     uint16_t* __restrict__ norms,
                                                                     uint32_t* __restrict__ status,
                                                                     long long wait_budget) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + kWOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kWOffBar + 8 * kWNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kWOffBar + 8 * kWNumBars + 4);
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  float* pn2 = reinterpret_cast<float*>(sbase + kWOffN2);
  float* prr = reinterpret_cast<float*>(sbase + kWOffRR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t num_tiles = (n + kTile - 1) / kTile;
  const int64_t my_tiles = num_tiles > blockIdx.x ? (num_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const int ka = (np + 63) / 64;          // operand atoms per matrix
  const int qt = (np + 31) / 32;          // fp32 quarter tiles per key tile
  const uint32_t atom_bytes = uint32_t(np) * 128u;
  const size_t mat_bytes = size_t(np) * 256 * 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWStage; ++s) {
      mbar_init(bar(kWSFull + s), 1);
      mbar_init(bar(kWSEmpty + s), 64);
    }
    for (int s = 0; s < kWRing; ++s) {
      mbar_init(bar(kWRFull + s), 64);
      mbar_init(bar(kWREmpty + s), 1);
    }
    for (int s = 0; s < kWBRing; ++s) {
      mbar_init(bar(kWBFull + s), 1);
      mbar_init(bar(kWBEmpty + s), 1);
    }
    mbar_init(bar(kWD1Full), 1);
    mbar_init(bar(kWN2), 512);
    mbar_init(bar(kWResid), 512);
    mbar_init(bar(kWD2Full), 1);
    mbar_init(bar(kWD2Free), 512);
    mbar_init(bar(kWRR), 512);
    *abort_flag = 0;
    g_wait_budget = wait_budget > 0 ? wait_budget : tc::kWaitCycles;
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
    if (lane == 0) {
      int64_t sq = 0, bq = 0;   // staging loads, operand atom loads issued
      bool ok = true;
      auto load_b = [&](int mat, int a) -> bool {
        const int sb = int(bq % kWBRing);
        if (bq >= kWBRing &&
            !mbar_wait(bar(kWBEmpty + sb), uint32_t((bq / kWBRing - 1) & 1), abort_flag, status))
          return false;
        mbar_expect_tx(bar(kWBFull + sb), atom_bytes);
        bulk_load(base + kWOffB + kWBAtomMax * sb, bimg + mat * mat_bytes + size_t(a) * atom_bytes, atom_bytes,
                  bar(kWBFull + sb));
        ++bq;
        return true;
      };
      for (int64_t i = 0; ok && i < my_tiles; ++i) {
        const int64_t tile = blockIdx.x + i * gridDim.x;
        for (int a = 0; ok && a < ka; ++a) {
          for (int h = 0; ok && h < 2; ++h) {
            const int q = 2 * a + h;
            if (q >= qt) break;
            const int s = int(sq % kWStage);
            if (sq >= kWStage &&
                !mbar_wait(bar(kWSEmpty + s), uint32_t((sq / kWStage - 1) & 1), abort_flag, status)) {
              ok = false;
              break;
            }
            mbar_expect_tx(bar(kWSFull + s), 16384u);
            tma_load_2d(base + kWOffStage + 16384u * s, &key_map, 32 * q, int(tile * kTile), bar(kWSFull + s));
            ++sq;
          }
          if (ok) ok = load_b(0, a) && load_b(1, a);   // R_hi, R_lo of atom a
        }
        for (int a = 0; ok && a < ka; ++a) ok = load_b(2, a);   // P
      }
      // leave no copy in flight: wait for the last loads issued to each buffer
      for (int64_t j = (sq >= kWStage ? sq - kWStage : 0); j < sq; ++j)
        mbar_drain(bar(kWSFull + int(j % kWStage)), uint32_t((j / kWStage) & 1), abort_flag, status);
      for (int64_t j = (bq >= kWBRing ? bq - kWBRing : 0); j < bq; ++j)
        mbar_drain(bar(kWBFull + int(j % kWBRing)), uint32_t((j / kWBRing) & 1), abort_flag, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc1 = idesc_f16(1, 128, uint32_t(np)), idesc2 = idesc_f16(0, 128, uint32_t(np));
      const uint32_t ty = tmem, tz = tmem + 256u;
      int64_t bq = 0, n1 = 0, n2 = 0;
      bool ok = true;
      auto wait_b = [&]() -> uint32_t {
        const int sb = int(bq % kWBRing);
        if (!mbar_wait(bar(kWBFull + sb), uint32_t((bq / kWBRing) & 1), abort_flag, status)) return 0u;
        return base + kWOffB + kWBAtomMax * sb;
      };
      auto free_b = [&]() {
        mma_commit(bar(kWBEmpty + int(bq % kWBRing)));
        ++bq;
      };
      for (int64_t i = 0; ok && i < my_tiles; ++i) {
        // y's columns hold the previous tile's residual until its JL product completed
        if (i >= 1 && !mbar_wait(bar(kWD2Full), uint32_t((i - 1) & 1), abort_flag, status)) break;
        tc_fence_after();
        uint32_t acc = 0;
        for (int a = 0; ok && a < ka; ++a) {
          const int64_t e = i * ka + a;
          const int rs = int(e % kWRing);
          if (!mbar_wait(bar(kWRFull + rs), uint32_t((e / kWRing) & 1), abort_flag, status)) {
            ok = false;
            break;
          }
          const uint32_t abase = base + kWOffRing + 32768u * rs;
          for (int mat = 0; mat < 2; ++mat) {
            const uint32_t bb = wait_b();
            if (!bb) {
              ok = false;
              break;
            }
            tc_fence_after();
            for (int ks = 0; ks < 4 && 64 * a + 16 * ks < np; ++ks) {
              // R_hi: K_hi R_hi + K_lo R_hi; R_lo: K_hi R_lo
              mma_f16(ty, smem_desc(abase + 32u * ks), smem_desc(bb + 32u * ks), idesc1, acc);
              acc = 1;
              if (mat == 0) mma_f16(ty, smem_desc(abase + 16384u + 32u * ks), smem_desc(bb + 32u * ks), idesc1, 1u);
            }
            free_b();
          }
          if (!ok) break;
          mma_commit(bar(kWREmpty + rs));
        }
        if (!ok) break;
        mma_commit(bar(kWD1Full));
        ++n1;
        // JL product once the epilogue has written the residual and read the previous z
        if (!mbar_wait(bar(kWResid), uint32_t(i & 1), abort_flag, status)) break;
        if (i >= 1 && !mbar_wait(bar(kWD2Free), uint32_t((i - 1) & 1), abort_flag, status)) break;
        tc_fence_after();
        acc = 0;
        for (int a = 0; ok && a < ka; ++a) {
          const uint32_t bb = wait_b();
          if (!bb) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int ks = 0; ks < 4 && 64 * a + 16 * ks < np; ++ks) {
            const uint32_t k16 = uint32_t(4 * a + ks);   // residual coordinates 16 k16 .. +15
            mma_f16_ts(tz, ty + 16u * k16, smem_desc(bb + 32u * ks), idesc2, acc);
            acc = 1;
            mma_f16_ts(tz, ty + 16u * k16 + 8u, smem_desc(bb + 32u * ks), idesc2, 1u);
          }
          free_b();
        }
        if (!ok) break;
        mma_commit(bar(kWD2Full));
        ++n2;
      }
      // before TMEM is released: the last commit of each kind tracks every MMA issued before it
      if (n1 > 0) mbar_drain(bar(kWD1Full), uint32_t((n1 - 1) & 1), abort_flag, status);
      if (n2 > 0) mbar_drain(bar(kWD2Full), uint32_t((n2 - 1) & 1), abort_flag, status);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ fp32 -> bf16 hi / lo converter
    const int c = threadIdx.x - 64;
    for (int64_t i = 0; i < my_tiles; ++i) {
      bool ok = true;
      for (int q = 0; q < qt; ++q) {
        const int64_t j = i * qt + q;              // staging use
        const int sb = int(j % kWStage);
        const int64_t e = i * ka + (q >> 1);       // key atom use
        const int rs = int(e % kWRing);
        if ((q & 1) == 0 && e >= kWRing &&
            !mbar_wait_warp(bar(kWREmpty + rs), uint32_t((e / kWRing - 1) & 1), abort_flag, status)) {
          ok = false;
          break;
        }
        if (!mbar_wait_warp(bar(kWSFull + sb), uint32_t((j / kWStage) & 1), abort_flag, status)) {
          ok = false;
          break;
        }
        const uint8_t* src = sbase + kWOffStage + 16384u * sb;
        uint8_t* dst = sbase + kWOffRing + 32768u * rs;
        // thread c converts rows c / 4 + 16 u (u = 0..7) of 8-float group c % 4, four
        // rows' loads issued before their conversions and stores (the swizzle of
        // those rows is the same: r % 8 = (c / 4) % 8)
        const int r0 = c >> 2, g = c & 3, sw = r0 & 7;
#pragma unroll
        for (int b4 = 0; b4 < 2; ++b4) {
          float4 va[4], vb[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int r = r0 + 16 * (4 * b4 + u);
            va[u] = *reinterpret_cast<const float4*>(src + r * 128 + (((2 * g) ^ sw) << 4));
            vb[u] = *reinterpret_cast<const float4*>(src + r * 128 + (((2 * g + 1) ^ sw) << 4));
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int r = r0 + 16 * (4 * b4 + u);
            const float2 x[4] = {make_float2(va[u].x, va[u].y), make_float2(va[u].z, va[u].w), make_float2(vb[u].x, vb[u].y),
                                 make_float2(vb[u].z, vb[u].w)};
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const __nv_bfloat162 h = __float22bfloat162_rn(x[t]);
              const float2 hf = __bfloat1622float2(h);
              const __nv_bfloat162 l = __float22bfloat162_rn(__ffma2_rn(hf, f2(-1.f), x[t]));
              hi[t] = *reinterpret_cast<const uint32_t*>(&h);
              lo[t] = *reinterpret_cast<const uint32_t*>(&l);
            }
            const uint32_t off = uint32_t(r * 128 + (((4 * (q & 1) + g) ^ sw) << 4));
            *reinterpret_cast<uint4*>(dst + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(dst + 16384u + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(bar(kWSEmpty + sb));
        if ((q & 1) || q == qt - 1) mbar_arrive(bar(kWRFull + rs));
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int qd = (warp - 4) >> 2;                   // layout quarter: slots 64 qd .. 64 qd + 63
    const int row = (warp & 3) * 32 + lane;           // TMEM lane = key row within the tile
    const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
    const uint32_t ty = tmem + lane_addr + 64u * qd, tz = tmem + lane_addr + 256u + 64u * qd;
    const int valid = d - 64 * qd < 64 ? (d - 64 * qd > 0 ? d - 64 * qd : 0) : 64;   // slots below d
    constexpr int kW = BMSE + 1;                      // words per half quarter (32 slots)
    const int row_bytes = 8 * (4 * BMSE + 4);
    for (int64_t i = 0; i < my_tiles; ++i) {
      const uint32_t par = uint32_t(i & 1);
      if (!mbar_wait_warp(bar(kWD1Full), par, abort_flag, status)) break;
      tc_fence_after();
      float y[2][32];
      tmem_ld32(ty, y[0]);
      tmem_ld32(ty + 32u, y[1]);
      tmem_wait32(y[0]);
      tmem_wait32(y[1]);
      float* n2buf = pn2 + int(par) * 512;
      {
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 v = make_float2(32 * h + j < valid ? y[h][j] : 0.f, 32 * h + j + 1 < valid ? y[h][j + 1] : 0.f);
            acc = __ffma2_rn(v, v, acc);
          }
        n2buf[qd * 128 + row] = acc.x + acc.y;
      }
      mbar_arrive(bar(kWN2));
      if (!mbar_wait_warp(bar(kWN2), par, abort_flag, status)) break;
      const float n2 = n2buf[row] + n2buf[128 + row] + n2buf[256 + row] + n2buf[384 + row];
      const float nk = sqrtf(n2);
      const bool zero = !(n2 > 0.f);
      const float s128 = zero ? 0.f : 128.f / nk;
      HalfBook hb = book;
      if (zero) {
        hb.C0 = 0.f;
#pragma unroll
        for (int c = 0; c < 3; ++c) hb.dC[c] = 0.f;
        hb.dA = 0.f;
        hb.C20 = 0.f;
      }
      float2 rr2 = make_float2(0.f, 0.f);
      uint32_t cw[2][BMSE];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // slots 32 h .. 32 h + 31 of the quarter: units 2 h and 2 h + 1
        uint32_t hw[2 * BMSE], hw3[2] = {0u, 0u};
#pragma unroll
        for (int t = 0; t < 2 * BMSE; ++t) hw[t] = 0;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t rh[8], rl[8];
#pragma unroll
          for (int jp = 0; jp < 16; jp += 2) {
            const int j0 = 16 * hh + jp;
            float2 rp;
            const uint2 bb = cell2<BMSE>(make_float2(y[h][j0], y[h][j0 + 1]), s128, hb, rp);
            // slots past d: no residual (their code and sign bits are masked below)
            if (32 * h + j0 >= valid) rp.x = 0.f;
            if (32 * h + j0 + 1 >= valid) rp.y = 0.f;
            rr2 = __ffma2_rn(rp, rp, rr2);
            const __half2 hi = __float22half2_rn(rp);
            const float2 hf = __half22float2(hi);
            const __half2 lo = __float22half2_rn(__ffma2_rn(hf, f2(-1.f), rp));
            rh[jp >> 1] = *reinterpret_cast<const uint32_t*>(&hi);
            rl[jp >> 1] = *reinterpret_cast<const uint32_t*>(&lo);
#pragma unroll
            for (int t2 = 0; t2 < 2; ++t2) {
              const int jc = j0 + t2;
              const uint32_t bits = t2 ? bb.y : bb.x;
              const int rreg = jc >> 2, e = jc & 3, uu = rreg >> 2, ii = rreg & 3;
              if constexpr (BMSE == 3) {
                if (ii < 3)
                  hw[uu * 3 + ii] += bits << (4 * e);
                else
                  hw3[uu] += bits << (4 * e);
              } else if constexpr (BMSE == 2) {
                hw[uu * 2 + (ii >> 1)] += bits << (4 * e + 2 * (ii & 1));
              } else {
                hw[uu] += bits << (4 * e + ii);
              }
            }
          }
          // residual coordinates 64 qd + 32 h + 16 hh .. +15 (group k16 = 4 qd + 2 h + hh):
          // hi pairs at column 16 k16, lo pairs at 16 k16 + 8
          tmem_st8(ty + 32u * h + 16u * hh, rh);
          tmem_st8(ty + 32u * h + 16u * hh + 8u, rl);
        }
        if constexpr (BMSE == 3) {
#pragma unroll
          for (int uu = 0; uu < 2; ++uu)
#pragma unroll
            for (int b = 0; b < 3; ++b) hw[uu * 3 + b] |= ((hw3[uu] >> b) & 0x1111u) << 3;
        }
#pragma unroll
        for (int w = 0; w < BMSE; ++w) cw[h][w] = zero ? 0u : ~__byte_perm(hw[2 * w], hw[2 * w + 1], 0x5410);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(bar(kWResid));
      float* rrbuf = prr + int(par) * 512;
      rrbuf[qd * 128 + row] = rr2.x + rr2.y;
      mbar_arrive(bar(kWRR));
      if (!mbar_wait_warp(bar(kWD2Full), par, abort_flag, status)) break;
      tc_fence_after();
      // bit = [z >= 0]; bit p of half h's word holds slot 32 h + 16 (p >> 4) + 4 (p & 3) + ((p >> 2) & 3)
      uint32_t sw[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t neg = 0;
#pragma unroll
        for (int hz = 1; hz >= 0; --hz) {
          float z[16];
          tmem_ld16(tz + 32u * h + 16u * hz, z);
          tmem_wait16(z);
#pragma unroll
          for (int p = 15; p >= 0; --p) {
            const int jj = 4 * (p & 3) + ((p >> 2) & 3);
            neg = __funnelshift_l(__float_as_uint(z[jj]), neg, 1);
          }
        }
        sw[h] = zero ? 0xFFFFFFFFu : ~neg;
      }
      tc_fence_before();
      mbar_arrive(bar(kWD2Free));
      const int64_t key = (blockIdx.x + i * gridDim.x) * kTile + row;
      if (key < n) {
        // quarter chunk: the 4 b' code halfwords of units 0..3, then the 4 sign halfwords
        uint32_t wv[2 * kW];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int w = 0; w < BMSE; ++w) wv[h * BMSE + w] = cw[h][w] & masks.code[qd][h * BMSE + w];
        wv[2 * BMSE] = sw[0] & masks.sign[qd][0];
        wv[2 * BMSE + 1] = sw[1] & masks.sign[qd][1];
        uint8_t* dst = payload + key * row_bytes + qd * 8 * kW;
        if constexpr (kW % 2 == 0) {
#pragma unroll
          for (int v = 0; v < kW / 2; ++v)
            reinterpret_cast<uint4*>(dst)[v] = make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
        } else {
#pragma unroll
          for (int v = 0; v < kW; ++v) reinterpret_cast<uint2*>(dst)[v] = make_uint2(wv[2 * v], wv[2 * v + 1]);
        }
      }
      if (qd == 0) {
        if (!mbar_wait_warp(bar(kWRR), par, abort_flag, status)) break;
        const float rr = rrbuf[row] + rrbuf[128 + row] + rrbuf[256 + row] + rrbuf[384 + row];
        const float rho = nk * sqrtf(rr) * (1.0f / 128.f);
        const uint32_t nn = uint32_t(__half_as_ushort(__float2half_rn(nk))) |
                            (uint32_t(__half_as_ushort(__float2half_rn(rho))) << 16);
        if (key < n) {
          reinterpret_cast<uint32_t*>(norms)[key] = nn;
          flag_norm_range(nn, status);
        }
      }
    }
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

HalfBook make_halfbook(const tq_ctx* ctx) {
  HalfBook hb{};
  const int L = ctx->levels;
  for (int i = 0; i < L / 2 - 1; ++i) hb.Tneg[i] = -float(128.0 * ctx->t[L / 2 + i]) * 0x1p100f;
  hb.C0 = float(128.0 * ctx->c[L / 2]);
  for (int i = 0; i + 1 < L / 2; ++i) hb.dC[i] = float(128.0 * ctx->c[L / 2 + i + 1]) - float(128.0 * ctx->c[L / 2 + i]);
  if (L == 8) {
    hb.dT31 = hb.Tneg[2] - hb.Tneg[0];
    hb.dA = hb.dC[2] - hb.dC[0];
    hb.C20 = float(128.0 * ctx->c[L / 2 + 2]) - hb.C0;
  }
  return hb;
}

}  // namespace

bool quantize_tc_supported(const tq_ctx* ctx, int dtype, int64_t ld, const void* keys) {
  return ctx->d == kD && (ctx->m == kD || ctx->m == 0) && (dtype == TQ_BF16 || dtype == TQ_F32) &&
         ctx->bmse >= 1 && ctx->bmse <= 3 && ctx->dBimg != nullptr && ld % 8 == 0 &&
         (reinterpret_cast<uintptr_t>(keys) & 15) == 0 && device_is_sm100() && get_encode() != nullptr;
}

cudaError_t launch_quantize_tc(const tq_ctx* ctx, const void* keys, int dtype, int64_t n, int64_t ld,
                               uint8_t* payload, uint16_t* norms, cudaStream_t st) {
  const bool f32 = dtype == TQ_F32;
  CUtensorMap map;
  const cuuint64_t dims[2] = {cuuint64_t(kD), cuuint64_t(n)};
  const cuuint64_t strides[1] = {cuuint64_t(ld) * (f32 ? 4 : 2)};
  // bf16: 64-column halves (128 bytes per row); fp32: 32-column quarters (128 bytes per row)
  const cuuint32_t box[2] = {f32 ? 32u : 64u, 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = get_encode()(&map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                  const_cast<void*>(keys), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (n + kTile - 1) / kTile;
  const int grid = int(tiles < sms ? tiles : sms);
  const HalfBook hb = make_halfbook(ctx);
  auto run = [&](auto kern, auto f) {
    using QL = QLayout<decltype(f)::value>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(QL::kSmem));
    kern<<<grid, QL::kThreads, QL::kSmem, st>>>(map, n, ctx->dBimg, hb, payload, norms, ctx->dstatus,
                                                ctx->wait_budget);
  };
  const bool jl = ctx->m > 0;
  auto go = [&](auto f) {
    constexpr bool F = decltype(f)::value;
    switch (ctx->bmse * 2 + (jl ? 1 : 0)) {
      case 2: run(quantize_tc_kernel<1, false, F>, f); break;
      case 3: run(quantize_tc_kernel<1, true, F>, f); break;
      case 4: run(quantize_tc_kernel<2, false, F>, f); break;
      case 5: run(quantize_tc_kernel<2, true, F>, f); break;
      case 6: run(quantize_tc_kernel<3, false, F>, f); break;
      default: run(quantize_tc_kernel<3, true, F>, f); break;
    }
  };
  if (f32)
    go(std::true_type{});
  else
    go(std::false_type{});
  return cudaGetLastError();
}

bool quantize_wide_supported(const tq_ctx* ctx, int dtype, int64_t ld, const void* keys) {
  return ctx->dBimgWide != nullptr && ctx->d > 192 && ctx->d <= 256 && ctx->m == ctx->d && dtype == TQ_F32 &&
         ctx->bmse >= 1 && ctx->bmse <= 3 && ld % 4 == 0 && (reinterpret_cast<uintptr_t>(keys) & 15) == 0 &&
         device_is_sm100() && get_encode() != nullptr;
}

namespace {

// Bits of the stored code and sign words that belong to slots below d (the
// packing of quantize_wide_kernel: half h of a quarter holds units 2h, 2h+1).
WideMasks wide_masks(int d, int bmse) {
  WideMasks wm{};
  for (int qd = 0; qd < 4; ++qd)
    for (int jq = 0; jq < 64; ++jq) {
      if (64 * qd + jq >= d) continue;
      const int e = jq & 3, i = (jq >> 2) & 3, u = jq >> 4, h = u >> 1, uu = u & 1;
      auto set_code = [&](int hw, int bit) { wm.code[qd][h * bmse + (hw >> 1)] |= 1u << (bit + 16 * (hw & 1)); };
      if (bmse == 3) {
        if (i < 3) {
          for (int b = 0; b < 3; ++b) set_code(uu * 3 + i, 4 * e + b);
        } else {
          for (int b = 0; b < 3; ++b) set_code(uu * 3 + b, 4 * e + 3);
        }
      } else if (bmse == 2) {
        for (int b = 0; b < 2; ++b) set_code(uu * 2 + (i >> 1), 4 * e + 2 * (i & 1) + b);
      } else {
        set_code(uu, 4 * e + i);
      }
      wm.sign[qd][h] |= 1u << (16 * uu + 4 * e + i);
    }
  return wm;
}

}  // namespace

cudaError_t launch_quantize_wide(const tq_ctx* ctx, const void* keys, int64_t n, int64_t ld, uint8_t* payload,
                                 uint16_t* norms, cudaStream_t st) {
  CUtensorMap map;
  const cuuint64_t dims[2] = {cuuint64_t(ctx->d), cuuint64_t(n)};
  const cuuint64_t strides[1] = {cuuint64_t(ld) * 4};
  const cuuint32_t box[2] = {32u, 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = get_encode()(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(keys), dims, strides,
                                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (n + kTile - 1) / kTile;
  const int grid = int(tiles < sms ? tiles : sms);
  const HalfBook hb = make_halfbook(ctx);
  const WideMasks wm = wide_masks(ctx->d, ctx->bmse);
  const int np = (ctx->d + 15) / 16 * 16;
  auto run = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kWSmem));
    kern<<<grid, kWThreads, kWSmem, st>>>(map, n, ctx->d, np, ctx->dBimgWide, hb, wm, payload, norms, ctx->dstatus,
                                         ctx->wait_budget);
  };
  switch (ctx->bmse) {
    case 1: run(quantize_wide_kernel<1>); break;
    case 2: run(quantize_wide_kernel<2>); break;
    default: run(quantize_wide_kernel<3>); break;
  }
  return cudaGetLastError();
}

bool split_tc_supported(const tq_split* sp, int dtype, const void* keys) {
  return sp->dimg != nullptr && dtype == TQ_BF16 && (reinterpret_cast<uintptr_t>(keys) & 15) == 0 &&
         device_is_sm100() && get_encode() != nullptr;
}

namespace {

template <int BHI, int BLO>
cudaError_t launch_split_kernel(dim3 grid, cudaStream_t st, const CUtensorMap& map, int B, int Hkv, int64_t S,
                                int cph, const uint8_t* dimg, const HalfBook& bh, const HalfBook& bl,
                                uint8_t* ph, uint16_t* nh, uint8_t* pl, uint16_t* nl, uint32_t* status) {
  auto k = quantize_split_tc_kernel<BHI, BLO>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemSplit));
  k<<<grid, kThreadsTc, kSmemSplit, st>>>(map, B, Hkv, S, cph, dimg, bh, bl, ph, nh, pl, nl, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_split_quantize_tc(const tq_split* sp, const void* keys, int B, int64_t S, uint8_t* payload_hi,
                                     uint16_t* norms_hi, uint8_t* payload_lo, uint16_t* norms_lo, cudaStream_t st) {
  CUtensorMap map;
  const int Hkv = sp->Hkv;
  const cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(S), cuuint64_t(int64_t(B) * Hkv)};
  const cuuint64_t strides[2] = {cuuint64_t(kD) * 2, cuuint64_t(S) * kD * 2};
  const cuuint32_t box[3] = {64u, 128u, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = get_encode()(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(keys), dims, strides,
                                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t head_tiles = int64_t(B) * ((S + kTile - 1) / kTile);
  int64_t cph = sms / Hkv > 1 ? sms / Hkv : 1;
  if (cph > head_tiles) cph = head_tiles;
  const dim3 grid(unsigned(Hkv * cph));
  const HalfBook bh = make_halfbook(sp->hi), bl = make_halfbook(sp->lo);
  uint32_t* status = sp->hi->dstatus;
  const uint8_t* img = sp->dimg;
  const int c = int(cph);
  switch (sp->hi->bmse * 4 + sp->lo->bmse) {
    case 5: return launch_split_kernel<1, 1>(grid, st, map, B, Hkv, S, c, img, bh, bl, payload_hi, norms_hi, payload_lo, norms_lo, status);
    case 6: return launch_split_kernel<1, 2>(grid, st, map, B, Hkv, S, c, img, bh, bl, payload_hi, norms_hi, payload_lo, norms_lo, status);
    case 7: return launch_split_kernel<1, 3>(grid, st, map, B, Hkv, S, c, img, bh, bl, payload_hi, norms_hi, payload_lo, norms_lo, status);
    case 9: return launch_split_kernel<2, 1>(grid, st, map, B, Hkv, S, c, img, bh, bl, payload_hi, norms_hi, payload_lo, norms_lo, status);
    case 10: return launch_split_kernel<2, 2>(grid, st, map, B, Hkv, S, c, img, bh, bl, payload_hi, norms_hi, payload_lo, norms_lo, status);
    case 11: return launch_split_kernel<2, 3>(grid, st, map, B, Hkv, S, c, img, bh, bl, payload_hi, norms_hi, payload_lo, norms_lo, status);
    case 13: return launch_split_kernel<3, 1>(grid, st, map, B, Hkv, S, c, img, bh, bl, payload_hi, norms_hi, payload_lo, norms_lo, status);
    case 14: return launch_split_kernel<3, 2>(grid, st, map, B, Hkv, S, c, img, bh, bl, payload_hi, norms_hi, payload_lo, norms_lo, status);
    default: return launch_split_kernel<3, 3>(grid, st, map, B, Hkv, S, c, img, bh, bl, payload_hi, norms_hi, payload_lo, norms_lo, status);
  }
}

}  // namespace tq
