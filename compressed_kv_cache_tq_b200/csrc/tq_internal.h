// Internal declarations shared by the libtq translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/tq.h"

namespace tq {

constexpr int kMaxLevels = 8;          // 2^(bits-1) for bits <= 4
constexpr double kQjlConst = 1.2533141373155002512;  // sqrt(pi / 2)

// Small tables passed to kernels by value.
struct CodebookParams {
  float c[kMaxLevels];       // Lloyd-Max levels (unit-sphere scale)
  float t[kMaxLevels - 1];   // decision boundaries
  int levels;
};

// int16 fixed-point codebook split into two signed byte planes for the
// byte-permute lookup in the logits kernel: c ~ (256 hi + lo) * inv_scale.
struct CodeLut {
  uint32_t hi[2];            // bytes v = 0..7 of the hi plane (v < 4 in [0])
  uint32_t lo[2];
  float inv_scale;
};

}  // namespace tq

struct tq_ctx {
  int d, m, bits, bmse, levels, row_bytes;
  uint64_t seed;
  uint32_t stream_base;
  int device;
  // fp64 masters (host)
  std::vector<double> R, P, c, t;
  // device tables
  float* dR = nullptr;      // R, fp32, d x d row-major
  float* dRt = nullptr;     // R^T
  float* dP = nullptr;      // P, fp32, m x d
  float* dPt = nullptr;     // P^T
  double* dR64 = nullptr;   // fp64 masters on the device (top-k re-scoring)
  double* dP64 = nullptr;
  double* dc64 = nullptr;
  uint8_t* dBimg = nullptr; // tensor-core B operands (d = m = 128): R_hi, R_lo (bf16), P (fp16), smem image
  uint32_t* dstatus = nullptr;
  tq::CodebookParams cb;
  tq::CodeLut lut;
};

namespace tq {

// Device status bits (set by bounded waits that gave up).
constexpr uint32_t kStatusQuantizeTc = 1u << 0;
constexpr uint32_t kStatusSearchTc = 1u << 1;

void set_cuda_error(cudaError_t e);

// Kernel launchers (defined in the .cu files).  All return cudaGetLastError().
cudaError_t launch_quantize_simt(const tq_ctx* ctx, const void* keys, int dtype, int64_t n, int64_t ld,
                                 uint8_t* payload, uint16_t* norms, cudaStream_t st);
bool quantize_tc_supported(const tq_ctx* ctx, int dtype, int64_t ld, const void* keys);
cudaError_t launch_quantize_tc(const tq_ctx* ctx, const void* keys, int dtype, int64_t n, int64_t ld,
                               uint8_t* payload, uint16_t* norms, cudaStream_t st);
cudaError_t launch_dequantize(const tq_ctx* ctx, const uint8_t* payload, const uint16_t* norms, int64_t n,
                              int full, float* out, cudaStream_t st);

size_t qprep_bytes(const tq_ctx* ctx, int64_t groups, int heads_per_group);
cudaError_t launch_logits(const tq_ctx* ctx, const float* q, int B, int Hq, int Hkv, int64_t S,
                          const uint8_t* payload, const uint16_t* norms, float scale, float* out,
                          void* ws, cudaStream_t st);
size_t topk_ws_bytes(const tq_ctx* ctx, int64_t nq, int64_t n, int k);
bool search_tc_supported(const tq_ctx* ctx, int64_t nq, int64_t n, int k);
size_t search_ws_bytes(const tq_ctx* ctx, int64_t nq, int64_t n);
cudaError_t launch_search_tc(const tq_ctx* ctx, const float* q, int64_t nq, const uint8_t* payload,
                             const uint16_t* norms, int64_t n, int k, int64_t* ids, float* scores, void* ws,
                             cudaStream_t st);
cudaError_t launch_topk(const tq_ctx* ctx, const float* q, int64_t nq, const uint8_t* payload,
                        const uint16_t* norms, int64_t n, int k, int64_t* ids, float* scores, void* ws,
                        cudaStream_t st);

}  // namespace tq
