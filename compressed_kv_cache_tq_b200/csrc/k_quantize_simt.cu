// CUDA-core quantize and dequantize kernels for every supported shape
// (d, m multiples of 8 from 64 to 256, fp32 or bf16 keys).  The tensor-core
// quantize kernel (k_quantize_tc.cu) covers d = m = 128 with bf16 keys; this
// file covers the rest and the dequantisation.
//
// quantize: per key k (airosetta.com "Google TurboQuant", stage 1 and 2)
//   n = ||k||, u = R k / n, idx_j = #{i: t_i < u_j}, r_rot = u - c[idx],
//   sign_i = [(P r_rot)_i >= 0]  (= sign of (S r)_i since S r = n P r_rot),
//   rho = n ||r_rot||, both norms rounded to fp16.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kThreads = 128;
constexpr int kKeys = 16;      // keys per block iteration

template <typename T>
__device__ inline float load_key(const T* p);
template <>
__device__ inline float load_key<float>(const float* p) { return *p; }
template <>
__device__ inline float load_key<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T>
__global__ void __launch_bounds__(kThreads) quantize_simt_kernel(const T* __restrict__ keys, int64_t n, int64_t ld,
                                                                 const float* __restrict__ Rt,
                                                                 const float* __restrict__ Pt, int d, int m,
                                                                 int bmse, CodebookParams cb,
                                                                 uint8_t* __restrict__ payload,
                                                                 uint16_t* __restrict__ norms,
                                                                 ChannelGather gth, uint32_t* __restrict__ status) {
  extern __shared__ float smem[];
  float* sk = smem;                          // [kKeys][d] keys, later r_rot
  float* sn = sk + kKeys * d;                // [kKeys] norms
  float* srr = sn + kKeys;                   // [kKeys] ||r_rot||^2
  const RowGeom g = make_geom(d, m, bmse);
  uint8_t* scode = reinterpret_cast<uint8_t*>(srr + kKeys);   // [kKeys][dp] layout slots
  uint8_t* sbit = scode + kKeys * g.dp;                        // [kKeys][mp]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the slots past d and m are never written below: zero them once
  for (int idx = tid; idx < kKeys * g.dp; idx += kThreads) scode[idx] = 0;
  for (int idx = tid; idx < kKeys * g.mp; idx += kThreads) sbit[idx] = 0;

  for (int64_t base = int64_t(blockIdx.x) * kKeys; base < n; base += int64_t(gridDim.x) * kKeys) {
    const int nk = (n - base) < kKeys ? int(n - base) : kKeys;
    for (int idx = tid; idx < kKeys * d; idx += kThreads) {
      const int k = idx / d, j = idx - k * d;
      float v = 0.f;
      if (k < nk) {
        const int64_t row = base + k;
        // split: coordinate j of the group is a channel of the row's KV head
        const int col = gth.perm ? gth.perm[int((row / gth.S) % gth.Hkv) * gth.dtot + gth.off + j] : j;
        v = load_key(keys + row * ld + col);
      }
      sk[idx] = v;
    }
    if (tid < kKeys) srr[tid] = 0.f;
    __syncthreads();
    for (int k = warp; k < kKeys; k += kThreads / 32) {
      float s = 0.f;
      for (int j = lane; j < d; j += 32) s = fmaf(sk[k * d + j], sk[k * d + j], s);
      for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) sn[k] = sqrtf(s);
    }
    __syncthreads();
    // rotation y = R k; thread handles coordinates j = tid, tid + 128
    float y[2][kKeys];
    for (int jj = 0; jj < 2; ++jj)
      for (int k = 0; k < kKeys; ++k) y[jj][k] = 0.f;
    for (int i = 0; i < d; ++i) {
      for (int jj = 0; jj < 2; ++jj) {
        const int j = tid + jj * kThreads;
        if (j < d) {
          const float r = Rt[i * d + j];
          for (int k = 0; k < kKeys; ++k) y[jj][k] = fmaf(r, sk[k * d + i], y[jj][k]);
        }
      }
    }
    __syncthreads();   // every thread is done reading the keys
    for (int jj = 0; jj < 2; ++jj) {
      const int j = tid + jj * kThreads;
      if (j >= d) continue;
      for (int k = 0; k < kKeys; ++k) {
        const float nk_ = sn[k];
        int code = 0;
        float rr = 0.f;
        if (nk_ > 0.f) {
          const float u = y[jj][k] * (1.0f / nk_);
          for (int i = 0; i < cb.levels - 1; ++i) code += (u > cb.t[i]) ? 1 : 0;
          rr = u - cb.c[code];
        }
        scode[k * g.dp + j] = uint8_t(code);
        sk[k * d + j] = rr;
      }
    }
    __syncthreads();
    // ||r_rot||^2 per key
    for (int k = warp; k < kKeys; k += kThreads / 32) {
      float s = 0.f;
      for (int j = lane; j < d; j += 32) s = fmaf(sk[k * d + j], sk[k * d + j], s);
      for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) srr[k] = s;
    }
    // JL projection z = P r_rot; thread handles rows i = tid, tid + 128
    float z[2][kKeys];
    for (int ii = 0; ii < 2; ++ii)
      for (int k = 0; k < kKeys; ++k) z[ii][k] = 0.f;
    for (int j = 0; j < d; ++j) {
      for (int ii = 0; ii < 2; ++ii) {
        const int i = tid + ii * kThreads;
        if (i < m) {
          const float p = Pt[j * m + i];
          for (int k = 0; k < kKeys; ++k) z[ii][k] = fmaf(p, sk[k * d + j], z[ii][k]);
        }
      }
    }
    for (int ii = 0; ii < 2; ++ii) {
      const int i = tid + ii * kThreads;
      if (i < m)
        for (int k = 0; k < kKeys; ++k) sbit[k * g.mp + i] = z[ii][k] >= 0.f ? 1 : 0;
    }
    __syncthreads();
    const int hw_per_row = g.row_bytes / 2;
    for (int idx = tid; idx < nk * hw_per_row; idx += kThreads) {
      const int k = idx / hw_per_row, h = idx - k * hw_per_row;
      const uint16_t v = pack_halfword(scode + k * g.dp, sbit + k * g.mp, g, h);
      reinterpret_cast<uint16_t*>(payload + (base + k) * g.row_bytes)[h] = v;
    }
    if (tid < nk) {
      const float nk_ = sn[tid];
      const float rho = nk_ * sqrtf(srr[tid]);
      const uint32_t nn = uint32_t(__half_as_ushort(__float2half_rn(nk_))) |
                          (uint32_t(__half_as_ushort(__float2half_rn(rho))) << 16);
      norms[2 * (base + tid)] = uint16_t(nn);
      norms[2 * (base + tid) + 1] = uint16_t(nn >> 16);
      flag_norm_range(nn, status);
    }
    __syncthreads();
  }
}

// x_hat = R^T (n16 c[idx] + [full] sqrt(pi/2)/m rho16 P^T sigma)
//   (= n16 R^T c[idx] + sqrt(pi/2)/m rho16 S^T sigma with S = P R)
__global__ void __launch_bounds__(kThreads) dequantize_kernel(const uint8_t* __restrict__ payload,
                                                              const uint16_t* __restrict__ norms, int64_t n,
                                                              int full, const float* __restrict__ R,
                                                              const float* __restrict__ P, int d, int m,
                                                              int bmse, CodebookParams cb,
                                                              float* __restrict__ out) {
  extern __shared__ float smem[];
  float* sv = smem;                 // [kKeys][d] rotated-domain vector v
  float* ssig = sv + kKeys * d;     // [kKeys][m] sigma
  const RowGeom g = make_geom(d, m, bmse);
  const int tid = threadIdx.x;
  const float qc = m > 0 ? float(kQjlConst) / float(m) : 0.f;   // m = 0: no sign term
  for (int64_t base = int64_t(blockIdx.x) * kKeys; base < n; base += int64_t(gridDim.x) * kKeys) {
    const int nk = (n - base) < kKeys ? int(n - base) : kKeys;
    for (int idx = tid; idx < kKeys * m; idx += kThreads) {
      const int k = idx / m, i = idx - k * m;
      float s = 0.f;
      if (k < nk) {
        const uint16_t* hw = reinterpret_cast<const uint16_t*>(payload + (base + k) * g.row_bytes);
        s = unpack_sign(hw, g, i) ? 1.f : -1.f;
      }
      ssig[idx] = s;
    }
    __syncthreads();
    for (int j = tid; j < d; j += kThreads) {
      float acc[kKeys];
      for (int k = 0; k < kKeys; ++k) acc[k] = 0.f;
      if (full) {
        for (int i = 0; i < m; ++i) {
          const float p = P[i * d + j];
          for (int k = 0; k < kKeys; ++k) acc[k] = fmaf(p, ssig[k * m + i], acc[k]);
        }
      }
      for (int k = 0; k < kKeys; ++k) {
        float v = 0.f;
        if (k < nk) {
          const uint16_t* hw = reinterpret_cast<const uint16_t*>(payload + (base + k) * g.row_bytes);
          const float n16 = half_bits_to_float(norms[2 * (base + k)]);
          const float r16 = half_bits_to_float(norms[2 * (base + k) + 1]);
          v = n16 * cb.c[unpack_code(hw, g, j)] + qc * r16 * acc[k];
        }
        sv[k * d + j] = v;
      }
    }
    __syncthreads();
    for (int i = tid; i < d; i += kThreads) {
      float acc[kKeys];
      for (int k = 0; k < kKeys; ++k) acc[k] = 0.f;
      for (int j = 0; j < d; ++j) {
        const float r = R[j * d + i];
        for (int k = 0; k < kKeys; ++k) acc[k] = fmaf(r, sv[k * d + j], acc[k]);
      }
      for (int k = 0; k < nk; ++k) out[(base + k) * d + i] = acc[k];
    }
    __syncthreads();
  }
}

int grid_for(int64_t n) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = (n + kKeys - 1) / kKeys;
  return int(blocks < int64_t(sms) * 8 ? blocks : int64_t(sms) * 8);
}

}  // namespace

cudaError_t launch_quantize_simt(const tq_ctx* ctx, const void* keys, int dtype, int64_t n, int64_t ld,
                                 uint8_t* payload, uint16_t* norms, cudaStream_t st, ChannelGather gather,
                                 uint32_t* status) {
  const int d = ctx->d, m = ctx->m;
  if (!status) status = ctx->dstatus;
  const RowGeom g = make_geom(d, m, ctx->bmse);
  const size_t smem = size_t(kKeys) * d * 4 + 2 * kKeys * 4 + size_t(kKeys) * (g.dp + g.mp);
  const int grid = grid_for(n);
  if (dtype == TQ_F32) {
    auto kern = quantize_simt_kernel<float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    kern<<<grid, kThreads, smem, st>>>(static_cast<const float*>(keys), n, ld, ctx->dRt, ctx->dPt, d, m,
                                        ctx->bmse, ctx->cb, payload, norms, gather, status);
  } else {
    auto kern = quantize_simt_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    kern<<<grid, kThreads, smem, st>>>(static_cast<const __nv_bfloat16*>(keys), n, ld, ctx->dRt, ctx->dPt, d,
                                        m, ctx->bmse, ctx->cb, payload, norms, gather, status);
  }
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const tq_ctx* ctx, const uint8_t* payload, const uint16_t* norms, int64_t n,
                              int full, float* out, cudaStream_t st) {
  const size_t smem = size_t(kKeys) * (ctx->d + ctx->m) * 4;
  cudaFuncSetAttribute(dequantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  dequantize_kernel<<<grid_for(n), kThreads, smem, st>>>(payload, norms, n, full, ctx->dR, ctx->dP, ctx->d,
                                                          ctx->m, ctx->bmse, ctx->cb, out);
  return cudaGetLastError();
}

}  // namespace tq
