// Tensor-core quantize kernel for d = m = 128 and bf16 keys (sm_100a).
//
// What it computes per key k (airosetta.com "Google TurboQuant", stage 1 and
// stage 2; mooersco.com section 1.1 "rotated = key @ rotation"):
//   y = R k                      (tcgen05 MMA: K R_hi^T + K R_lo^T, fp32 in TMEM)
//   n = ||k||                    (from the key tile in shared memory, fp32)
//   idx_j = #{i : t_i < y_j / n} (Lloyd-Max cell search in registers)
//   r_rot = y / n - c[idx]       (the residual on the unit sphere, R r / n)
//   z = P r_rot                  (tcgen05 MMA, fp16 hi/lo split of both
//                                 operands, three passes, fp32 in TMEM)
//   sign_i = [z_i >= 0]          (= [(S r)_i >= 0] since S r = n P r_rot)
//   ||r|| = n ||r_rot||; both norms rounded to fp16.
//
// Precision: R = R_hi + R_lo in bf16 represents R to about 2^-17, so y / n is
// within about 4e-7 of R k / ||k|| (codes differ from exact arithmetic only
// for coordinates within that distance of a boundary); the JL product uses an
// fp16 hi + lo split of r_rot (scaled by 2^7) and of P, dropping only lo * lo.
//
// Structure (one CTA per SM, persistent over 128-key tiles):
//   warp 4       : TMA producer (the constant B operands once, then key tiles)
//   warp 5       : TMEM allocation and the single-thread MMA issue
//   warps 0 .. 3 : epilogue, one thread per key row (= TMEM lane)
// Shared memory: B operands R_hi, R_lo, P_hi, P_lo (128 KB), one key tile
// (32 KB, TMA 128-byte swizzle) and the residual tiles r_hi, r_lo (64 KB).
// TMEM: 256 columns, D1 = y (columns 0..127), D2 = z (columns 128..255).
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
constexpr int kThreadsTc = 192;

constexpr uint32_t kOffRhi = 0, kOffRlo = 32768, kOffPhi = 65536, kOffPlo = 98304;
constexpr uint32_t kOffKey = 131072;
constexpr uint32_t kOffAhi = 163840, kOffAlo = 196608;
constexpr uint32_t kOffBar = 229376;
constexpr uint32_t kSmemBytes = kOffBar + 128 + 1024;   // + slack for 1024-byte alignment

enum Bar { kBarConst = 0, kBarKFull, kBarKEmpty, kBarD1Full, kBarD1Empty, kBarRFull, kBarD2Full, kBarD2Empty, kNumBars };

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
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false when the budget ran out or another role gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
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

template <int BMSE>
__global__ void __launch_bounds__(kThreadsTc, 1) quantize_tc_kernel(const __grid_constant__ CUtensorMap key_map,
                                                                   int64_t n, const uint8_t* __restrict__ bimg,
                                                                   CodebookParams cb,
                                                                   uint8_t* __restrict__ payload,
                                                                   uint16_t* __restrict__ norms,
                                                                   uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base (the swizzle pattern is anchored to the address)
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kOffBar + 8 * kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kOffBar + 8 * kNumBars + 4);
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t num_tiles = (n + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarConst), 1);
    mbar_init(bar(kBarKFull), 1);
    mbar_init(bar(kBarKEmpty), 128);
    mbar_init(bar(kBarD1Full), 1);
    mbar_init(bar(kBarD1Empty), 128);
    mbar_init(bar(kBarRFull), 128);
    mbar_init(bar(kBarD2Full), 1);
    mbar_init(bar(kBarD2Empty), 128);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(256));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_d1 = tmem, tmem_d2 = tmem + 128;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(bar(kBarConst), 131072u);
      for (int c = 0; c < 8; ++c) bulk_load(base + 16384u * c, bimg + 16384 * c, 16384u, bar(kBarConst));
      int64_t i = 0;
      for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
        if (i > 0 && !mbar_wait(bar(kBarKEmpty), uint32_t((i - 1) & 1), abort_flag, status)) break;
        mbar_expect_tx(bar(kBarKFull), 32768u);
        tma_load_2d(base + kOffKey, &key_map, 0, int(tile * kTile), bar(kBarKFull));
        tma_load_2d(base + kOffKey + 16384u, &key_map, 64, int(tile * kTile), bar(kBarKFull));
      }
      // do not leave with a copy in flight
      if (i > 0) mbar_wait(bar(kBarKFull), uint32_t((i - 1) & 1), abort_flag, status);
      mbar_wait(bar(kBarConst), 0u, abort_flag, status);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      bool ok = mbar_wait(bar(kBarConst), 0u, abort_flag, status);
      int64_t i = 0;
      for (int64_t tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++i) {
        if (!mbar_wait(bar(kBarKFull), uint32_t(i & 1), abort_flag, status)) break;
        if (i > 0 && !mbar_wait(bar(kBarD1Empty), uint32_t((i - 1) & 1), abort_flag, status)) break;
        tc_fence_after();
        uint32_t acc = 0;
        for (int pass = 0; pass < 2; ++pass)
          for (int kb = 0; kb < 2; ++kb)
            for (int ks = 0; ks < 4; ++ks) {
              const uint32_t off = 16384u * kb + 32u * ks;
              mma_f16(tmem_d1, smem_desc(base + kOffKey + off), smem_desc(base + (pass ? kOffRlo : kOffRhi) + off),
                      kIdescBf16, acc);
              acc = 1;
            }
        mma_commit(bar(kBarD1Full));
        if (!mbar_wait(bar(kBarRFull), uint32_t(i & 1), abort_flag, status)) break;
        if (i > 0 && !mbar_wait(bar(kBarD2Empty), uint32_t((i - 1) & 1), abort_flag, status)) break;
        tc_fence_after();
        acc = 0;
        for (int pass = 0; pass < 3; ++pass) {
          const uint32_t a_off = pass == 2 ? kOffAlo : kOffAhi;
          const uint32_t b_off = pass == 1 ? kOffPlo : kOffPhi;
          for (int kb = 0; kb < 2; ++kb)
            for (int ks = 0; ks < 4; ++ks) {
              const uint32_t off = 16384u * kb + 32u * ks;
              mma_f16(tmem_d2, smem_desc(base + a_off + off), smem_desc(base + b_off + off), kIdescF16, acc);
              acc = 1;
            }
        }
        mma_commit(bar(kBarD2Full));
      }
      // wait for the last MMAs before TMEM is released
      if (i > 0) mbar_wait(bar(kBarD2Full), uint32_t((i - 1) & 1), abort_flag, status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int row = threadIdx.x;          // 0..127 = TMEM lane
    const uint32_t lane_addr = uint32_t(warp * 32) << 16;
    constexpr int kCodeWords = BMSE;      // per quarter: 2 units x BMSE halfwords = BMSE words
    constexpr int kRowBytes = kD * BMSE / 8 + kD / 8;
    int64_t i = 0;
    for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
      const uint32_t par = uint32_t(i & 1);
      if (!mbar_wait(bar(kBarKFull), par, abort_flag, status)) break;
      // ||k||^2 from this row of the swizzled key tile
      float n2 = 0.f;
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(sbase + kOffKey + 16384 * kb + row * 128 +
                                                          ((c ^ (row & 7)) * 16));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float lo = __uint_as_float(w[h] << 16), hi = __uint_as_float(w[h] & 0xFFFF0000u);
            n2 = fmaf(lo, lo, n2);
            n2 = fmaf(hi, hi, n2);
          }
        }
      const float nk = sqrtf(n2);
      const float inv_n = nk > 0.f ? 1.0f / nk : 0.f;
      if (!mbar_wait(bar(kBarD1Full), par, abort_flag, status)) break;
      mbar_arrive(bar(kBarKEmpty));
      tc_fence_after();
      uint32_t codew[4][kCodeWords];
      float rr = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float y[32];
        tmem_ld32(tmem_d1 + lane_addr + 32u * q, y);
        uint32_t hw[2 * BMSE];
#pragma unroll
        for (int h = 0; h < 2 * BMSE; ++h) hw[h] = 0;
        uint32_t rh[16], rl[16];    // 32 fp16 values of r_hi / r_lo, packed in pairs
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const float u = y[jj] * inv_n;
          int code = 0;
          float level = cb.c[0];
#pragma unroll
          for (int b = 0; b < (1 << BMSE) - 1; ++b) {
            const bool above = u > cb.t[b];
            code += above ? 1 : 0;
            level = above ? cb.c[b + 1] : level;
          }
          const float r = nk > 0.f ? u - level : 0.f;
          if (nk == 0.f) code = 0;
          rr = fmaf(r, r, rr);
          const int rreg = jj >> 2, e = jj & 3, uu = rreg >> 2, ii = rreg & 3;
          if constexpr (BMSE == 3) {
            if (ii < 3) {
              hw[uu * 3 + ii] |= uint32_t(code) << (4 * e);
            } else {
#pragma unroll
              for (int b = 0; b < 3; ++b) hw[uu * 3 + b] |= uint32_t((code >> b) & 1) << (4 * e + 3);
            }
          } else if constexpr (BMSE == 2) {
            hw[uu * 2 + (ii >> 1)] |= uint32_t(code) << (4 * e + 2 * (ii & 1));
          } else {
            hw[uu] |= uint32_t(code) << (4 * e + ii);
          }
          const float rs = r * 128.f;
          const __half hi = __float2half_rn(rs);
          const __half lo = __float2half_rn(rs - __half2float(hi));
          const uint32_t hb = __half_as_ushort(hi), lb = __half_as_ushort(lo);
          if (jj & 1) {
            rh[jj >> 1] |= hb << 16;
            rl[jj >> 1] |= lb << 16;
          } else {
            rh[jj >> 1] = hb;
            rl[jj >> 1] = lb;
          }
        }
#pragma unroll
        for (int w = 0; w < kCodeWords; ++w) codew[q][w] = hw[2 * w] | (hw[2 * w + 1] << 16);
        // residual columns 32q .. 32q+31 -> K block q/2, 16-byte chunks 4(q%2) .. 4(q%2)+3
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int chunk = 4 * (q & 1) + cc;
          const uint32_t off = 16384u * uint32_t(q >> 1) + uint32_t(row) * 128u + uint32_t((chunk ^ (row & 7)) * 16);
          *reinterpret_cast<uint4*>(sbase + kOffAhi + off) =
              make_uint4(rh[4 * cc], rh[4 * cc + 1], rh[4 * cc + 2], rh[4 * cc + 3]);
          *reinterpret_cast<uint4*>(sbase + kOffAlo + off) =
              make_uint4(rl[4 * cc], rl[4 * cc + 1], rl[4 * cc + 2], rl[4 * cc + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(kBarD1Empty));
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(bar(kBarRFull));
      const float rho = nk * sqrtf(rr);
      if (!mbar_wait(bar(kBarD2Full), par, abort_flag, status)) break;
      tc_fence_after();
      uint32_t signw[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float z[32];
        tmem_ld32(tmem_d2 + lane_addr + 32u * q, z);
        uint32_t s0 = 0, s1 = 0;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int rreg = jj >> 2, e = jj & 3, uu = rreg >> 2, ii = rreg & 3;
          const uint32_t bit = z[jj] >= 0.f ? 1u : 0u;
          if (uu == 0)
            s0 |= bit << (4 * e + ii);
          else
            s1 |= bit << (4 * e + ii);
        }
        signw[q] = s0 | (s1 << 16);
      }
      tc_fence_before();
      mbar_arrive(bar(kBarD2Empty));
      const int64_t key = tile * kTile + row;
      if (key < n) {
        uint8_t* dst = payload + key * kRowBytes;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t* d32 = reinterpret_cast<uint32_t*>(dst + q * 4 * (BMSE + 1));
          if constexpr (BMSE == 3) {
            *reinterpret_cast<uint4*>(d32) = make_uint4(codew[q][0], codew[q][1], codew[q][2], signw[q]);
          } else if constexpr (BMSE == 1) {
            *reinterpret_cast<uint2*>(d32) = make_uint2(codew[q][0], signw[q]);
          } else {
            d32[0] = codew[q][0];
            d32[1] = codew[q][1];
            d32[2] = signw[q];
          }
        }
        const uint32_t nn = uint32_t(__half_as_ushort(__float2half_rn(nk))) |
                            (uint32_t(__half_as_ushort(__float2half_rn(rho))) << 16);
        reinterpret_cast<uint32_t*>(norms)[key] = nn;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256));
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
  switch (ctx->bmse) {
    case 1: {
      auto k = quantize_tc_kernel<1>;
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
      k<<<grid, kThreadsTc, kSmemBytes, st>>>(map, n, ctx->dBimg, ctx->cb, payload, norms, ctx->dstatus);
      break;
    }
    case 2: {
      auto k = quantize_tc_kernel<2>;
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
      k<<<grid, kThreadsTc, kSmemBytes, st>>>(map, n, ctx->dBimg, ctx->cb, payload, norms, ctx->dstatus);
      break;
    }
    default: {
      auto k = quantize_tc_kernel<3>;
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
      k<<<grid, kThreadsTc, kSmemBytes, st>>>(map, n, ctx->dBimg, ctx->cb, payload, norms, ctx->dstatus);
      break;
    }
  }
  return cudaGetLastError();
}

}  // namespace tq
