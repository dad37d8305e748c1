// Channel split of a key cache into a high-variance and a low-variance group
// (fractional bit rates such as 2.5 bits per channel: the rom4ai.github.io
// note "TurboQuant: Online Vector Quantization with Near-Optimal Distortion
// Rate" states the cache size as 3.5 bits per channel; mooersco.com section
// 2.1 lists a 2.5-bit setting; zhengruan.com reports its small quality loss;
// mooersco.com's FAQ says channel variances differ by orders of magnitude
// before rotation).
//
// Plan: per KV head, the variance of every channel over all B x S keys of the
// head; the hi->d channels of largest variance (ties to the lower channel)
// form the high group, in ascending channel order, followed by the others in
// ascending order.  Two kernels: fp64 partial sums over fixed row chunks,
// then a per-head reduction in chunk order and a rank count, so the plan does
// not depend on scheduling.  Sums are taken about the head's first key (a
// shift that leaves the variance unchanged and keeps the one-pass formula
// free of cancellation for channels with a large mean).
//
// Images: the tensor-core operands of the fast split quantizer (d = 128 split
// 64 + 64): per head the 128 x 128 matrix M_h with M_h[j][perm[p]] = R_hi[j][p]
// (j, p < 64) and M_h[64 + j][perm[64 + p]] = R_lo[j][p], so that M_h k is the
// two groups' rotations of the gathered key at once, split into bf16 hi + lo
// and stored in the 128-byte-swizzled K-major layout; then the block-diagonal
// JL samples diag(P_hi, P_lo) in fp16 (shared by all heads).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kPlanChunks = 256;   // row chunks per head for the partial sums

template <typename T>
__device__ __forceinline__ double load_channel(const T* p);
template <>
__device__ __forceinline__ double load_channel<float>(const float* p) { return double(*p); }
template <>
__device__ __forceinline__ double load_channel<__nv_bfloat16>(const __nv_bfloat16* p) {
  return double(__bfloat162float(*p));
}

// grid (Hkv, kPlanChunks), d threads: thread c sums channel c of the rows of
// its chunk: ws[h][chunk][0][c] = sum (x - x0), ws[h][chunk][1][c] = sum (x - x0)^2,
// x0 the channel's value in the head's first key.
template <typename T>
__global__ void split_stats_kernel(const T* __restrict__ keys, int B, int Hkv, int64_t S, int d,
                                   double* __restrict__ ws) {
  const int h = blockIdx.x, chunk = blockIdx.y, c = threadIdx.x;
  if (c >= d) return;
  const int64_t rows = int64_t(B) * S;
  const int64_t r0 = rows * chunk / kPlanChunks, r1 = rows * (chunk + 1) / kPlanChunks;
  double s1 = 0.0, s2 = 0.0;
  if (rows > 0) {
    const double x0 = load_channel(keys + (int64_t(h) * S) * d + c);   // row (b = 0, h, s = 0)
    int64_t b = r0 / S, s = r0 - b * S;
#pragma unroll 4
    for (int64_t t = r0; t < r1; ++t) {
      const double x = load_channel(keys + ((b * Hkv + h) * S + s) * d + c) - x0;
      s1 += x;
      s2 = fma(x, x, s2);
      if (++s == S) {
        s = 0;
        ++b;
      }
    }
  }
  double* o = ws + (size_t(h) * kPlanChunks + chunk) * 2 * d;
  o[c] = s1;
  o[d + c] = s2;
}

// One block per head, d threads: the variances (times the row count), the
// rank of every channel and its position in the plan.
__global__ void split_select_kernel(const double* __restrict__ ws, int Hkv, int64_t rows, int d, int d_hi,
                                    int32_t* __restrict__ perm) {
  extern __shared__ double svar[];
  __shared__ int shi[512];
  const int h = blockIdx.x, c = threadIdx.x;
  if (c < d) {
    double s1 = 0.0, s2 = 0.0;
    for (int k = 0; k < kPlanChunks; ++k) {
      const double* o = ws + (size_t(h) * kPlanChunks + k) * 2 * d;
      s1 += o[c];
      s2 += o[d + c];
    }
    svar[c] = rows > 0 ? s2 - s1 * s1 / double(rows) : 0.0;
  }
  __syncthreads();
  if (c < d) {
    const double v = svar[c];
    int rank = 0;
    for (int k = 0; k < d; ++k) rank += (svar[k] > v || (svar[k] == v && k < c)) ? 1 : 0;
    shi[c] = rank < d_hi ? 1 : 0;
  }
  __syncthreads();
  if (c < d) {
    const int hi = shi[c];
    int pos = hi ? 0 : d_hi;
    for (int k = 0; k < c; ++k) pos += (shi[k] == hi) ? 1 : 0;
    perm[h * d + pos] = c;
  }
}

// byte offset of element (row r, column c) in a 128-row, K = 128 swizzled operand image
__device__ __forceinline__ uint32_t swz_offset(int r, int c) {
  const int kb = c >> 6, chunk = (c & 63) >> 3, e = c & 7;
  return uint32_t(kb) * 16384u + uint32_t(r) * 128u + uint32_t((chunk ^ (r & 7)) * 16 + e * 2);
}

// grid Hkv: M_h (bf16 hi at +0, lo at +32 KB) of head h at dimg + 64 KB h.
__global__ void split_images_kernel(const int32_t* __restrict__ perm, const double* __restrict__ Rhi,
                                    const double* __restrict__ Rlo, uint8_t* __restrict__ dimg) {
  __shared__ int inv[128];
  const int h = blockIdx.x;
  for (int p = threadIdx.x; p < 128; p += blockDim.x) inv[perm[h * 128 + p]] = p;
  __syncthreads();
  uint8_t* img = dimg + size_t(h) * 65536;
  for (int idx = threadIdx.x; idx < 128 * 128; idx += blockDim.x) {
    const int r = idx >> 7, c = idx & 127;
    const int p = inv[c];
    double v = 0.0;
    if (r < 64 && p < 64) v = Rhi[r * 64 + p];
    if (r >= 64 && p >= 64) v = Rlo[(r - 64) * 64 + (p - 64)];
    const __nv_bfloat16 hi = __double2bfloat16(v);
    const __nv_bfloat16 lo = __double2bfloat16(v - double(__bfloat162float(hi)));
    const uint32_t off = swz_offset(r, c);
    *reinterpret_cast<__nv_bfloat16*>(img + off) = hi;
    *reinterpret_cast<__nv_bfloat16*>(img + 32768 + off) = lo;
  }
}

// The block-diagonal JL samples diag(P_hi, P_lo) (fp16, exact) after the head images.
__global__ void split_pimage_kernel(const double* __restrict__ Phi, const double* __restrict__ Plo,
                                    uint8_t* __restrict__ pimg) {
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < 128 * 128; idx += gridDim.x * blockDim.x) {
    const int r = idx >> 7, c = idx & 127;
    double v = 0.0;
    if (r < 64 && c < 64) v = Phi[r * 64 + c];
    if (r >= 64 && c >= 64) v = Plo[(r - 64) * 64 + (c - 64)];
    *reinterpret_cast<__half*>(pimg + swz_offset(r, c)) = __double2half(v);
  }
}

}  // namespace

size_t split_plan_ws_bytes(const tq_split* sp) { return size_t(sp->Hkv) * kPlanChunks * 2 * sp->d * 8; }

cudaError_t launch_split_plan(tq_split* sp, const void* keys, int dtype, int B, int64_t S, void* ws,
                              cudaStream_t st) {
  const int d = sp->d;
  double* sums = static_cast<double*>(ws);
  dim3 grid(unsigned(sp->Hkv), unsigned(kPlanChunks));
  if (dtype == TQ_F32)
    split_stats_kernel<float><<<grid, d, 0, st>>>(static_cast<const float*>(keys), B, sp->Hkv, S, d, sums);
  else
    split_stats_kernel<__nv_bfloat16><<<grid, d, 0, st>>>(static_cast<const __nv_bfloat16*>(keys), B, sp->Hkv, S,
                                                           d, sums);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  split_select_kernel<<<sp->Hkv, d, size_t(d) * 8, st>>>(sums, sp->Hkv, int64_t(B) * S, d, sp->hi->d, sp->dperm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_split_images(sp, st);
}

cudaError_t launch_split_images(tq_split* sp, cudaStream_t st) {
  if (!sp->dimg) return cudaSuccess;
  split_images_kernel<<<sp->Hkv, 256, 0, st>>>(sp->dperm, sp->hi->dR64, sp->lo->dR64, sp->dimg);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  split_pimage_kernel<<<16, 256, 0, st>>>(sp->hi->dP64, sp->lo->dP64, sp->dimg + size_t(sp->Hkv) * 65536);
  return cudaGetLastError();
}

}  // namespace tq
