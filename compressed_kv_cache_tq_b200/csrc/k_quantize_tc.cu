// Tensor-core quantize kernel for d = m = 128 and bf16 keys (sm_100a).
//
// What it computes per key k (airosetta.com "Google TurboQuant", stage 1 and
// stage 2; mooersco.com section 1.1 "rotated = key @ rotation"):
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
// ||y|| = ||R k|| (relative error about 4e-7); the JL product uses an fp16
// hi + lo split of r_rot (scaled by 2^7) against P, which is stored exactly in fp16.
//
// Structure (one CTA per SM, persistent over 128-key tiles, two tiles in flight):
//   warp 0       : TMA producer (the constant B operands once, then key tiles
//                  into a two-deep ring)
//   warp 1       : TMEM allocation and the single-thread MMA issue, in the
//                  order MMA1(0), MMA1(1), MMA2(0), MMA1(2), MMA2(1), ...
//   warps 2 .. 5 : epilogue of even local tiles (TMEM slot 0)
//   warps 6 .. 9 : epilogue of odd local tiles (TMEM slot 1)
//                  one thread per key row (= TMEM lane)
// Shared memory: B operands R_hi, R_lo, P (96 KB), two key tiles (2 x 32 KB,
// TMA 128-byte swizzle) and the packed rows of the two slots.
// TMEM: 512 columns, two slots of 256: y accumulates in columns 0..127 of a
// slot; the epilogue reads it and writes the residual's fp16 hi / lo pairs
// back over it (A operand of the JL product, read by the MMA from TMEM); z
// accumulates in columns 128..255.
// Every wait on an mbarrier is bounded; a wait that gives up sets the
// context's status word, and all roles then leave their loops.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr int kThreadsTc = 576;   // 2 control warps + 16 epilogue warps

constexpr uint32_t kOffRhi = 0, kOffRlo = 32768, kOffP = 65536;
constexpr uint32_t kConstBytes = 98304;  // R_hi, R_lo (bf16), P (fp16)
constexpr uint32_t kOffKey = 98304;      // two 32 KB key tiles
constexpr uint32_t kOffStage = 163840;   // packed rows of the two slots
constexpr int kStageWords = 20;         // 64-byte row padded to 80 bytes (conflict-free 16-byte accesses)
constexpr uint32_t kStageBytes = 128u * kStageWords * 4u;
constexpr uint32_t kOffPart = kOffStage + 2 * kStageBytes;   // row partial sums [slot][n^2 | rr][half][row]
constexpr uint32_t kOffBar = kOffPart + 2 * 512 * 4;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;   // + slack for 1024-byte alignment

// barriers; the per-slot ones come in pairs (slot 0, slot 1)
enum Bar {
  kBarConst = 0,
  kBarKFull = 1,
  kBarKEmpty = 3,
  kBarD1Full = 5,
  kBarRFull = 7,
  kBarD2Full = 9,
  kBarD2Free = 11,
  kNumBars = 13
};

constexpr long long kWaitCycles = 4000000000LL;   // about 2 s at the boost clock

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// One test of the phase with a suspend-time hint: the thread may sleep until
// the phase completes (or about 0.5 ms pass) instead of spinning.
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(500000u)
      : "memory");
  return ok != 0;
}
// Bounded wait: false when the budget ran out or another role gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort_flag = 1;
      atomicOr(status, kStatusQuantizeTc);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major operand in the 128-byte swizzle layout: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  uint64_t d = uint64_t((addr & 0x3FFFFu) >> 4);
  d |= uint64_t(1) << 16;            // leading byte offset (unused for this layout)
  d |= uint64_t(1024 >> 4) << 32;    // stride byte offset
  d |= uint64_t(1) << 46;            // descriptor version
  d |= uint64_t(2) << 61;            // 128-byte swizzle
  return d;
}

// kind::f16 instruction descriptor: fp32 accumulate, K-major A and B, M = N = 128.
__host__ __device__ constexpr uint32_t idesc_f16(uint32_t ab_format) {
  return (1u << 4) | (ab_format << 7) | (ab_format << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
}
constexpr uint32_t kIdescBf16 = idesc_f16(1);
constexpr uint32_t kIdescF16 = idesc_f16(0);

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 consecutive TMEM columns of this thread's lane, without waiting (the
// registers are valid after tmem_wait_ld()).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// A operand from tensor memory, B from shared memory.
__device__ __forceinline__ void mma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc,
                                           uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Positive half of the symmetric codebook, scaled by 128 (the residual scale),
// pre-arranged for the arithmetic cell search below.
struct HalfBook {
  float Tneg[3];   // -2^100 x boundaries above 0 (t_{L/2} .. t_{L-2})
  float C0;        // smallest positive level
  float dC[3];     // level steps c_{L/2+i+1} - c_{L/2+i}
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
// boundary).  Returns the float bit patterns of 2^23 + idx.
template <int BMSE>
__device__ __forceinline__ uint2 cell2(float2 y, float s128, const HalfBook& hb, float2& r) {
  const float2 u = __fmul2_rn(y, f2(s128));
  const float2 sp = make_float2(__saturatef(u.x * kBig), __saturatef(u.y * kBig));   // [u > 0]
  const float2 sgn = __ffma2_rn(f2(2.f), sp, f2(-1.f));                               // sign(u), 0 -> -1
  const float2 nsgn = __ffma2_rn(f2(-2.f), sp, f2(1.f));
  float2 m = make_float2(0.f, 0.f), lv = f2(hb.C0);
#pragma unroll
  for (int i = 0; i < (1 << (BMSE - 1)) - 1; ++i) {
    const float2 step = make_float2(__saturatef(fmaf(fabsf(u.x), kBig, hb.Tneg[i])),
                                    __saturatef(fmaf(fabsf(u.y), kBig, hb.Tneg[i])));
    m = i == 0 ? step : __fadd2_rn(m, step);
    lv = __ffma2_rn(step, f2(hb.dC[i]), lv);
  }
  r = __ffma2_rn(nsgn, lv, u);                                                        // u - sign(u) level
  constexpr float half_l = float(1 << (BMSE - 1)) - 0.5f;
  const float2 base = __ffma2_rn(sgn, f2(0.5f), f2(half_l));                          // L/2 or L/2 - 1
  const float2 idx = __fadd2_rn(__ffma2_rn(sgn, m, base), f2(8388608.f));
  return make_uint2(__float_as_uint(idx.x), __float_as_uint(idx.y));
}

template <int BMSE>
__global__ void __launch_bounds__(kThreadsTc, 1) quantize_tc_kernel(const __grid_constant__ CUtensorMap key_map,
                                                                   int64_t n, const uint8_t* __restrict__ bimg,
                                                                   HalfBook book,
                                                                   uint8_t* __restrict__ payload,
                                                                   uint16_t* __restrict__ norms,
                                                                   uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;   // the swizzle pattern is anchored to 1024-byte boundaries
  uint8_t* sbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kOffBar + 8 * kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kOffBar + 8 * kNumBars + 4);
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t num_tiles = (n + kTile - 1) / kTile;
  const int64_t my_tiles = num_tiles > blockIdx.x ? (num_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarConst), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarD1Full + s), 1);
      mbar_init(bar(kBarRFull + s), 256);
      mbar_init(bar(kBarD2Full + s), 1);
      mbar_init(bar(kBarD2Free + s), 256);
    }
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
    if (lane == 0) {
      mbar_expect_tx(bar(kBarConst), kConstBytes);
      for (int c = 0; c < int(kConstBytes / 16384u); ++c)
        bulk_load(base + 16384u * c, bimg + 16384 * c, 16384u, bar(kBarConst));
      int64_t i = 0;
      for (; i < my_tiles; ++i) {
        const int kb = int(i & 1);
        if (i >= 2 && !mbar_wait(bar(kBarKEmpty + kb), uint32_t(((i >> 1) - 1) & 1), abort_flag, status)) break;
        const int64_t tile = blockIdx.x + i * gridDim.x;
        const uint32_t dst = base + kOffKey + 32768u * kb;
        mbar_expect_tx(bar(kBarKFull + kb), 32768u);
        tma_load_2d(dst, &key_map, 0, int(tile * kTile), bar(kBarKFull + kb));
        tma_load_2d(dst + 16384u, &key_map, 64, int(tile * kTile), bar(kBarKFull + kb));
      }
      // leave no copy in flight: wait for the last loads issued to each buffer
      for (int64_t j = (i >= 2 ? i - 2 : 0); j < i; ++j)
        mbar_wait(bar(kBarKFull + int(j & 1)), uint32_t((j >> 1) & 1), abort_flag, status);
      mbar_wait(bar(kBarConst), 0u, abort_flag, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      auto issue_mma1 = [&](int64_t i) -> bool {
        const int sl = int(i & 1);
        if (!mbar_wait(bar(kBarKFull + sl), uint32_t((i >> 1) & 1), abort_flag, status)) return false;
        // the slot's y / residual columns are free once the JL MMA of tile i - 2 completed
        if (i >= 2 && !mbar_wait(bar(kBarD2Full + sl), uint32_t(((i >> 1) - 1) & 1), abort_flag, status))
          return false;
        tc_fence_after();
        const uint32_t d1 = tmem + 256u * sl;
        const uint32_t kbase = base + kOffKey + 32768u * sl;
        uint32_t acc = 0;
        for (int pass = 0; pass < 2; ++pass)
          for (int kb = 0; kb < 2; ++kb)
            for (int ks = 0; ks < 4; ++ks) {
              const uint32_t off = 16384u * kb + 32u * ks;
              mma_f16(d1, smem_desc(kbase + off), smem_desc(base + (pass ? kOffRlo : kOffRhi) + off), kIdescBf16,
                      acc);
              acc = 1;
            }
        mma_commit(bar(kBarD1Full + sl));
        mma_commit(bar(kBarKEmpty + sl));
        return true;
      };
      auto issue_mma2 = [&](int64_t i) -> bool {
        const int sl = int(i & 1);
        if (!mbar_wait(bar(kBarRFull + sl), uint32_t((i >> 1) & 1), abort_flag, status)) return false;
        // the slot's z columns are free once the epilogue of tile i - 2 read them
        if (i >= 2 && !mbar_wait(bar(kBarD2Free + sl), uint32_t(((i >> 1) - 1) & 1), abort_flag, status))
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
        mma_commit(bar(kBarD2Full + sl));
        return true;
      };
      bool ok = mbar_wait(bar(kBarConst), 0u, abort_flag, status);
      if (ok && my_tiles > 0) ok = issue_mma1(0);
      int64_t i = 0;
      for (; ok && i < my_tiles; ++i) {
        if (i + 1 < my_tiles && !issue_mma1(i + 1)) break;
        if (!issue_mma2(i)) break;
      }
      // wait for the last MMAs before TMEM is released
      for (int64_t j = (i >= 2 ? i - 2 : 0); j < i; ++j)
        mbar_wait(bar(kBarD2Full + int(j & 1)), uint32_t((j >> 1) & 1), abort_flag, status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // 16 warps in 4 groups: group eg serves TMEM slot eg & 1 (local tiles of
    // that parity) and quarters 2 (eg >> 1), 2 (eg >> 1) + 1 of every row; the
    // two groups of a slot combine their row partial sums through shared
    // memory around a named barrier (id 1 + slot, 256 threads).
    const int eg = (warp - 2) >> 2;
    const int slot = eg & 1, half = eg >> 1;
    const int row = (warp & 3) * 32 + lane;          // TMEM lane = key row within the tile
    const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
    const uint32_t d1 = tmem + 256u * slot + lane_addr, d2 = d1 + 128u;
    constexpr int kRowBytes = kD * BMSE / 8 + kD / 8;  // = 16 (BMSE + 1)
    float* part = reinterpret_cast<float*>(sbase + kOffPart) + slot * 512;   // [n^2 | rr][half][row]
    uint32_t* srow = reinterpret_cast<uint32_t*>(sbase + kOffStage + slot * kStageBytes) + row * kStageWords;
    const int q0 = 2 * half;
    int64_t k = 0;
    for (int64_t i = slot; i < my_tiles; i += 2, ++k) {
      const uint32_t par = uint32_t(k & 1);
      if (!mbar_wait(bar(kBarD1Full + slot), par, abort_flag, status)) break;
      tc_fence_after();
      // ||k||^2 = ||R k||^2 from the rotated row, half a row per group
      float n2p = 0.f;
      {
        float y0[32], y1[32];
        tmem_ld32_nowait(d1 + 32u * q0, y0);
        tmem_ld32_nowait(d1 + 32u * (q0 + 1), y1);
        tmem_wait_ld();
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 32; j += 2) acc = __ffma2_rn(make_float2(y0[j], y0[j + 1]), make_float2(y0[j], y0[j + 1]), acc);
#pragma unroll
        for (int j = 0; j < 32; j += 2) acc = __ffma2_rn(make_float2(y1[j], y1[j + 1]), make_float2(y1[j], y1[j + 1]), acc);
        n2p = acc.x + acc.y;
      }
      part[half * 128 + row] = n2p;
      named_barrier(1 + slot, 256);
      const float n2 = part[row] + part[128 + row];
      const float nk = sqrtf(n2);
      const bool zero = !(n2 > 0.f);
      const float s128 = zero ? 0.f : 128.f / nk;
      HalfBook hb = book;
      if (zero) {
        hb.C0 = 0.f;
#pragma unroll
        for (int c = 0; c < 3; ++c) hb.dC[c] = 0.f;
      }
      float2 rr2 = make_float2(0.f, 0.f);
#pragma unroll 1
      for (int qq = 0; qq < 2; ++qq) {
        const int q = q0 + qq;
        float y[32];
        tmem_ld32(d1 + 32u * q, y);
        uint32_t hw[2 * BMSE];
#pragma unroll
        for (int h = 0; h < 2 * BMSE; ++h) hw[h] = 0;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t rh[8], rl[8];
#pragma unroll
          for (int jp = 0; jp < 16; jp += 2) {
            const int jj = 16 * hh + jp;
            float2 rp;
            const uint2 bb = cell2<BMSE>(make_float2(y[jj], y[jj + 1]), s128, hb, rp);
            const uint32_t b0 = bb.x, b1 = bb.y;
            rr2 = __ffma2_rn(rp, rp, rr2);
            const __half2 hi = __float22half2_rn(rp);
            const float2 hf = __half22float2(hi);
            const __half2 lo = __float22half2_rn(__ffma2_rn(hf, f2(-1.f), rp));
            rh[jp >> 1] = *reinterpret_cast<const uint32_t*>(&hi);
            rl[jp >> 1] = *reinterpret_cast<const uint32_t*>(&lo);
#pragma unroll
            for (int t2 = 0; t2 < 2; ++t2) {
              // bits = float pattern of 2^23 + idx: idx in bits 0..2, the constant
              // part only reaches bits >= 24 of each shifted term
              const int j = jj + t2;
              const uint32_t bits = t2 ? b1 : b0;
              const int rreg = j >> 2, e = j & 3, uu = rreg >> 2, ii = rreg & 3;
              if constexpr (BMSE == 3) {
                if (ii < 3) {
                  hw[uu * 3 + ii] += bits << (4 * e);
                } else {
#pragma unroll
                  for (int b = 0; b < 3; ++b) hw[uu * 3 + b] |= ((bits >> b) & 1u) << (4 * e + 3);
                }
              } else if constexpr (BMSE == 2) {
                hw[uu * 2 + (ii >> 1)] += bits << (4 * e + 2 * (ii & 1));
              } else {
                hw[uu] += bits << (4 * e + ii);
              }
            }
          }
          // the residual overwrites the columns of y just read (A operand of the JL product):
          // coordinates 32q + 16hh .. +15 -> hi pairs at column 32q + 8hh, lo pairs 16 further
          tmem_st8(d1 + 32u * q + 8u * hh, rh);
          tmem_st8(d1 + 32u * q + 16u + 8u * hh, rl);
        }
#pragma unroll
        for (int w = 0; w < BMSE; ++w)
          srow[q * (BMSE + 1) + w] = zero ? 0u : __byte_perm(hw[2 * w], hw[2 * w + 1], 0x5410);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(bar(kBarRFull + slot));
      part[256 + half * 128 + row] = rr2.x + rr2.y;
      if (!mbar_wait(bar(kBarD2Full + slot), par, abort_flag, status)) break;
      tc_fence_after();
      float z0[32], z1[32];
      tmem_ld32_nowait(d2 + 32u * q0, z0);
      tmem_ld32_nowait(d2 + 32u * (q0 + 1), z1);
      tmem_wait_ld();
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const float* z = qq ? z1 : z0;
        uint32_t sw = 0;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int rreg = jj >> 2, e = jj & 3, uu = rreg >> 2, ii = rreg & 3;
          sw |= (z[jj] >= 0.f ? 1u : 0u) << (16 * uu + 4 * e + ii);
        }
        srow[(q0 + qq) * (BMSE + 1) + BMSE] = zero ? 0xFFFFFFFFu : sw;
      }
      tc_fence_before();
      mbar_arrive(bar(kBarD2Free + slot));
      named_barrier(1 + slot, 256);
      const int64_t key = (blockIdx.x + i * gridDim.x) * kTile + row;
      if (key < n) {
        // each group writes its two quarter chunks; group 0 of the slot writes the norms
        uint8_t* dst = payload + key * kRowBytes + q0 * 4 * (BMSE + 1);
        const uint32_t* src = srow + q0 * (BMSE + 1);
        if constexpr (BMSE == 3) {
          reinterpret_cast<uint4*>(dst)[0] = reinterpret_cast<const uint4*>(src)[0];
          reinterpret_cast<uint4*>(dst)[1] = reinterpret_cast<const uint4*>(src)[1];
        } else if constexpr (BMSE == 1) {
          reinterpret_cast<uint4*>(dst)[0] = reinterpret_cast<const uint4*>(src)[0];
        } else {
#pragma unroll
          for (int w = 0; w < 6; ++w) reinterpret_cast<uint32_t*>(dst)[w] = src[w];
        }
        if (half == 0) {
          const float rho = nk * sqrtf(part[256 + row] + part[384 + row]) * (1.0f / 128.f);
          const uint32_t nn = uint32_t(__half_as_ushort(__float2half_rn(nk))) |
                              (uint32_t(__half_as_ushort(__float2half_rn(rho))) << 16);
          reinterpret_cast<uint32_t*>(norms)[key] = nn;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool device_is_sm100() {
  int dev = 0, major = 0, minor = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  return major == 10 && minor == 0;
}

}  // namespace

bool quantize_tc_supported(const tq_ctx* ctx, int dtype, int64_t ld, const void* keys) {
  return ctx->d == kD && ctx->m == kD && dtype == TQ_BF16 && ctx->bmse >= 1 && ctx->bmse <= 3 &&
         ctx->dBimg != nullptr && ld % 8 == 0 && (reinterpret_cast<uintptr_t>(keys) & 15) == 0 &&
         device_is_sm100() && get_encode() != nullptr;
}

cudaError_t launch_quantize_tc(const tq_ctx* ctx, const void* keys, int dtype, int64_t n, int64_t ld,
                               uint8_t* payload, uint16_t* norms, cudaStream_t st) {
  (void)dtype;
  CUtensorMap map;
  const cuuint64_t dims[2] = {cuuint64_t(kD), cuuint64_t(n)};
  const cuuint64_t strides[1] = {cuuint64_t(ld) * 2};
  const cuuint32_t box[2] = {64u, 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = get_encode()(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(keys), dims, strides,
                                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (n + kTile - 1) / kTile;
  const int grid = int(tiles < sms ? tiles : sms);
  HalfBook hb{};
  const int L = ctx->levels;
  for (int i = 0; i < L / 2 - 1; ++i) hb.Tneg[i] = -float(128.0 * ctx->t[L / 2 + i]) * 0x1p100f;
  hb.C0 = float(128.0 * ctx->c[L / 2]);
  for (int i = 0; i + 1 < L / 2; ++i) hb.dC[i] = float(128.0 * ctx->c[L / 2 + i + 1]) - float(128.0 * ctx->c[L / 2 + i]);
  switch (ctx->bmse) {
    case 1: {
      auto k = quantize_tc_kernel<1>;
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
      k<<<grid, kThreadsTc, kSmemBytes, st>>>(map, n, ctx->dBimg, hb, payload, norms, ctx->dstatus);
      break;
    }
    case 2: {
      auto k = quantize_tc_kernel<2>;
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
      k<<<grid, kThreadsTc, kSmemBytes, st>>>(map, n, ctx->dBimg, hb, payload, norms, ctx->dstatus);
      break;
    }
    default: {
      auto k = quantize_tc_kernel<3>;
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
      k<<<grid, kThreadsTc, kSmemBytes, st>>>(map, n, ctx->dBimg, hb, payload, norms, ctx->dstatus);
      break;
    }
  }
  return cudaGetLastError();
}

}  // namespace tq
