// C-ABI entry points of libtq: argument validation and dispatch to the
// kernels.  Semantics and error behaviour are documented in include/tq.h.
#include <cuda_runtime.h>

#include "tq_internal.h"

namespace {

tq_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return TQ_OK;
  tq::set_cuda_error(e);
  return e == cudaErrorMemoryAllocation ? TQ_ERR_NOMEM : TQ_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" {

tq_status tq_quantize(const tq_ctx* ctx, const void* keys, tq_dtype dtype, int64_t n, int64_t ld, uint8_t* payload,
                      uint16_t* norms, void* stream) {
  if (!ctx || n < 0) return TQ_ERR_ARG;
  if (n == 0) return TQ_OK;
  if (!keys || !payload || !norms) return TQ_ERR_ARG;
  if (dtype != TQ_F32 && dtype != TQ_BF16) return TQ_ERR_ARG;
  if (ld < ctx->d || ld % 8 || !aligned(keys, 16) || !aligned(payload, 16) || !aligned(norms, 4))
    return TQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (tq::quantize_tc_supported(ctx, dtype, ld, keys))
    e = tq::launch_quantize_tc(ctx, keys, dtype, n, ld, payload, norms, st);
  else if (tq::quantize_wide_supported(ctx, dtype, ld, keys))
    e = tq::launch_quantize_wide(ctx, keys, n, ld, payload, norms, st);
  else
    e = tq::launch_quantize_simt(ctx, keys, dtype, n, ld, payload, norms, st);
  return cuda_status(e);
}

tq_status tq_dequantize(const tq_ctx* ctx, const uint8_t* payload, const uint16_t* norms, int64_t n, int full,
                        float* out, void* stream) {
  if (!ctx || n < 0) return TQ_ERR_ARG;
  if (n == 0) return TQ_OK;
  if (!payload || !norms || !out || !aligned(payload, 2) || !aligned(norms, 2) || !aligned(out, 4))
    return TQ_ERR_ARG;
  return cuda_status(
      tq::launch_dequantize(ctx, payload, norms, n, full, out, static_cast<cudaStream_t>(stream)));
}

size_t tq_logits_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv) {
  if (!ctx || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return 0;
  return tq::qprep_bytes(ctx, int64_t(B) * Hkv, Hq / Hkv);
}

tq_status tq_logits(const tq_ctx* ctx, const float* q, int B, int Hq, int Hkv, int64_t S, const uint8_t* payload,
                    const uint16_t* norms, float scale, float* out, void* workspace, size_t workspace_bytes,
                    void* stream) {
  if (!ctx || B < 0 || Hq < 0 || Hkv < 0 || S < 0) return TQ_ERR_ARG;
  if (B == 0 || Hq == 0) return TQ_OK;
  if (Hkv == 0 || Hq % Hkv) return TQ_ERR_ARG;
  if (!q || !out || (S > 0 && (!payload || !norms))) return TQ_ERR_ARG;
  if (!aligned(payload, 16) || !aligned(norms, 4) || !aligned(q, 4) || !aligned(out, 4)) return TQ_ERR_ARG;
  if (!workspace || !aligned(workspace, 256)) return TQ_ERR_ARG;
  if (workspace_bytes < tq_logits_workspace_bytes(ctx, B, Hq, Hkv)) return TQ_ERR_WORKSPACE;
  return cuda_status(tq::launch_logits(ctx, q, B, Hq, Hkv, S, payload, norms, scale, out, workspace,
                                       static_cast<cudaStream_t>(stream)));
}

size_t tq_attend_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int64_t S) {
  if (!ctx || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || S < 0) return 0;
  return tq::attend_ws_bytes(ctx, B, Hq, Hkv, S);
}

tq_status tq_attend(const tq_ctx* ctx, const float* logits, int B, int Hq, int Hkv, int64_t S,
                    const uint8_t* payload, const uint16_t* norms, float* out, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (!ctx || B < 0 || Hq < 0 || Hkv < 0 || S < 0) return TQ_ERR_ARG;
  if (B == 0 || Hq == 0) return TQ_OK;
  if (Hkv == 0 || Hq % Hkv) return TQ_ERR_ARG;
  if (!out || (S > 0 && (!logits || !payload || !norms))) return TQ_ERR_ARG;
  if (!aligned(payload, 16) || !aligned(norms, 4) || !aligned(logits, 4) || !aligned(out, 4)) return TQ_ERR_ARG;
  if (!tq::attend_supported(ctx, Hq, Hkv)) return TQ_ERR_UNSUPPORTED;
  if (!workspace || !aligned(workspace, 256)) return TQ_ERR_ARG;
  if (workspace_bytes < tq_attend_workspace_bytes(ctx, B, Hq, Hkv, S)) return TQ_ERR_WORKSPACE;
  return cuda_status(tq::launch_attend(ctx, logits, B, Hq, Hkv, S, payload, norms, out, workspace,
                                       static_cast<cudaStream_t>(stream)));
}

size_t tq_topk_workspace_bytes(const tq_ctx* ctx, int64_t nq, int64_t n, int k) {
  if (!ctx || nq <= 0 || n <= 0 || k <= 0) return 0;
  return tq::topk_ws_bytes(ctx, nq, n, k);
}

tq_status tq_topk(const tq_ctx* ctx, const float* q, int64_t nq, const uint8_t* payload, const uint16_t* norms,
                  int64_t n, int k, int64_t* ids, float* scores, void* workspace, size_t workspace_bytes,
                  void* stream) {
  if (!ctx || nq < 0 || n < 0) return TQ_ERR_ARG;
  if (nq == 0) return TQ_OK;
  if (k < 1 || k > 256 || k > n) return TQ_ERR_ARG;
  if (!q || !payload || !norms || !ids || !scores || !workspace) return TQ_ERR_ARG;
  if (!aligned(payload, 16) || !aligned(norms, 4) || !aligned(workspace, 256)) return TQ_ERR_ARG;
  if (!aligned(q, 4) || !aligned(ids, 8) || !aligned(scores, 4)) return TQ_ERR_ARG;
  if (workspace_bytes < tq_topk_workspace_bytes(ctx, nq, n, k)) return TQ_ERR_WORKSPACE;
  return cuda_status(tq::launch_topk(ctx, q, nq, payload, norms, n, k, ids, scores, workspace,
                                     static_cast<cudaStream_t>(stream)));
}

tq_status tq_topk_merge(const float* scores, const int64_t* ids, const int64_t* first_rows, int parts, int64_t nq,
                        int k, int64_t* out_ids, float* out_scores, void* stream) {
  if (parts < 1 || parts > tq::kMaxMergeParts || nq < 0 || k < 1) return TQ_ERR_ARG;
  if (int64_t(parts) * k > tq::kMaxMergeCandidates) return TQ_ERR_UNSUPPORTED;
  if (nq == 0) return TQ_OK;
  if (!scores || !ids || !first_rows || !out_ids || !out_scores) return TQ_ERR_ARG;
  if (!aligned(scores, 4) || !aligned(ids, 8) || !aligned(out_ids, 8) || !aligned(out_scores, 4)) return TQ_ERR_ARG;
  tq::MergeOffsets off{};
  for (int p = 0; p < parts; ++p) {
    if (first_rows[p] < 0) return TQ_ERR_ARG;
    off.first_row[p] = first_rows[p];
  }
  return cuda_status(tq::launch_topk_merge(scores, ids, off, nq, parts, k, out_ids, out_scores,
                                           static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
