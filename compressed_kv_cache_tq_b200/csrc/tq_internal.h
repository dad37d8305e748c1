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

// Channel gather of the split (per KV head channel order): group coordinate
// j of key row `row` is channel perm[((row / S) % Hkv) * dtot + off + j] of a
// row of dtot channels.  perm == nullptr: no gather (coordinate j = column j).
struct ChannelGather {
  const int32_t* perm;
  int64_t S;
  int Hkv, dtot, off;
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
  uint8_t* dBimgWide = nullptr;  // wide tensor-core quantizer (192 < d <= 256, m = d): R_hi, R_lo, P as
                                 // 4 streamed 64-column atoms each (Np = d rounded up to 16 rows)
  uint32_t* dstatus = nullptr;
  long long wait_budget = 0;   // tensor-core quantizer: cycles a wait spins before giving up (0: default)
  tq::CodebookParams cb;
  tq::CodeLut lut;
};

// A per-KV-head channel split of d = hi->d + lo->d channels into two groups,
// each quantised with its own context (see tq.h, "Channel split").
struct tq_split {
  const tq_ctx* hi = nullptr;
  const tq_ctx* lo = nullptr;
  int d = 0, Hkv = 0, device = 0;
  int32_t* dperm = nullptr;   // [Hkv][d] channel of group coordinate p (p < hi->d: high group)
  uint8_t* dimg = nullptr;    // tensor-core operands of the fast path: per head M_h hi / lo (64 KB), then
                              // the block-diagonal JL samples (32 KB); nullptr without a fast path
};

namespace tq {

// Device status bits (set by bounded waits that gave up).
constexpr uint32_t kStatusQuantizeTc = TQ_STATUS_QUANTIZE_WAIT;
constexpr uint32_t kStatusSearchTc = TQ_STATUS_SEARCH_WAIT;
constexpr uint32_t kStatusRange = TQ_STATUS_RANGE;   // a stored norm is not finite in fp16

#ifdef __CUDACC__
// Set the range bit when either fp16 norm of a packed pair (||k|| low,
// ||r|| high) is inf or NaN.
__device__ __forceinline__ void flag_norm_range(uint32_t pair, uint32_t* status) {
  if (((pair & 0x7C00u) == 0x7C00u) || ((pair & 0x7C000000u) == 0x7C000000u)) atomicOr(status, kStatusRange);
}
#endif

void set_cuda_error(cudaError_t e);

// Kernel launchers (defined in the .cu files).  All return cudaGetLastError().
cudaError_t launch_quantize_simt(const tq_ctx* ctx, const void* keys, int dtype, int64_t n, int64_t ld,
                                 uint8_t* payload, uint16_t* norms, cudaStream_t st,
                                 ChannelGather gather = ChannelGather{nullptr, 1, 1, 0, 0},
                                 uint32_t* status = nullptr);   // range bit target (nullptr: ctx's)
bool quantize_tc_supported(const tq_ctx* ctx, int dtype, int64_t ld, const void* keys);
cudaError_t launch_quantize_tc(const tq_ctx* ctx, const void* keys, int dtype, int64_t n, int64_t ld,
                               uint8_t* payload, uint16_t* norms, cudaStream_t st);
bool quantize_wide_supported(const tq_ctx* ctx, int dtype, int64_t ld, const void* keys);
cudaError_t launch_quantize_wide(const tq_ctx* ctx, const void* keys, int64_t n, int64_t ld, uint8_t* payload,
                                 uint16_t* norms, cudaStream_t st);
cudaError_t launch_dequantize(const tq_ctx* ctx, const uint8_t* payload, const uint16_t* norms, int64_t n,
                              int full, float* out, cudaStream_t st);

size_t qprep_bytes(const tq_ctx* ctx, int64_t groups, int heads_per_group);
cudaError_t launch_logits(const tq_ctx* ctx, const float* q, int B, int Hq, int Hkv, int64_t S,
                          const uint8_t* payload, const uint16_t* norms, float scale, float* out,
                          void* ws, cudaStream_t st);
// CUDA-core logits of one group of a split: q rows of gather.dtot channels,
// gathered per KV head; accumulate != 0 adds to out instead of overwriting.
cudaError_t launch_logits_simt(const tq_ctx* ctx, const float* q, int B, int Hq, int Hkv, int64_t S,
                               const uint8_t* payload, const uint16_t* norms, float scale, float* out,
                               ChannelGather gather, int accumulate, cudaStream_t st);

// Merge of per-shard top-k lists (k_topk_merge.cu)
constexpr int kMaxMergeParts = 64;
constexpr int kMaxMergeCandidates = 4096;   // parts * k
struct MergeOffsets {
  int64_t first_row[kMaxMergeParts];
};
cudaError_t launch_topk_merge(const float* scores, const int64_t* ids, const MergeOffsets& off, int64_t nq, int parts,
                              int k, int64_t* out_ids, float* out_scores, cudaStream_t st);

// Value path (k_attend.cu)
bool attend_supported(const tq_ctx* ctx, int Hq, int Hkv);
size_t attend_ws_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int64_t S);
cudaError_t launch_attend(const tq_ctx* ctx, const float* logits, int B, int Hq, int Hkv, int64_t S,
                          const uint8_t* payload, const uint16_t* norms, float* out, void* ws, cudaStream_t st);

// Channel split (k_split.cu, k_quantize_tc.cu, k_logits.cu)
size_t split_plan_ws_bytes(const tq_split* sp);
cudaError_t launch_split_plan(tq_split* sp, const void* keys, int dtype, int B, int64_t S, void* ws,
                              cudaStream_t st);
cudaError_t launch_split_images(tq_split* sp, cudaStream_t st);
bool split_tc_supported(const tq_split* sp, int dtype, const void* keys);
cudaError_t launch_split_quantize_tc(const tq_split* sp, const void* keys, int B, int64_t S, uint8_t* payload_hi,
                                     uint16_t* norms_hi, uint8_t* payload_lo, uint16_t* norms_lo, cudaStream_t st);
size_t split_logits_ws_bytes(const tq_split* sp, int B, int Hq);
cudaError_t launch_split_logits(const tq_split* sp, const float* q, int B, int Hq, int64_t S, const uint8_t* ph,
                                const uint16_t* nh, const uint8_t* pl, const uint16_t* nl, float scale, float* out,
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
