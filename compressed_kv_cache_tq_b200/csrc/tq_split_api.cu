// C-ABI entry points of the channel split: validation and dispatch.
// Semantics and error behaviour are documented in include/tq.h.
#include <cuda_runtime.h>

#include <vector>

#include "tq_internal.h"

namespace {

tq_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return TQ_OK;
  tq::set_cuda_error(e);
  return e == cudaErrorMemoryAllocation ? TQ_ERR_NOMEM : TQ_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool has_fast_path(const tq_ctx* hi, const tq_ctx* lo) {
  return hi->d == 64 && lo->d == 64 && hi->m == 64 && lo->m == 64 && hi->bmse >= 1 && hi->bmse <= 3 &&
         lo->bmse >= 1 && lo->bmse <= 3;
}

tq::ChannelGather gather_of(const tq_split* sp, int64_t S, bool high) {
  return tq::ChannelGather{sp->dperm, S > 0 ? S : 1, sp->Hkv, sp->d, high ? 0 : sp->hi->d};
}

}  // namespace

extern "C" {

tq_status tq_split_create(const tq_ctx* hi, const tq_ctx* lo, int Hkv, tq_split** out) {
  if (!out) return TQ_ERR_ARG;
  *out = nullptr;
  if (!hi || !lo || Hkv < 1 || hi->device != lo->device) return TQ_ERR_ARG;
  if (hi->d + lo->d > 512) return TQ_ERR_UNSUPPORTED;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev != hi->device) return TQ_ERR_ARG;
  tq_split* sp = new tq_split();
  sp->hi = hi;
  sp->lo = lo;
  sp->d = hi->d + lo->d;
  sp->Hkv = Hkv;
  sp->device = dev;
  std::vector<int32_t> ident(size_t(Hkv) * sp->d);
  for (int h = 0; h < Hkv; ++h)
    for (int c = 0; c < sp->d; ++c) ident[size_t(h) * sp->d + c] = c;
  e = cudaMalloc(&sp->dperm, ident.size() * sizeof(int32_t));
  if (e == cudaSuccess) e = cudaMemcpy(sp->dperm, ident.data(), ident.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess && has_fast_path(hi, lo)) {
    e = cudaMalloc(&sp->dimg, size_t(Hkv) * 65536 + 32768);
    if (e == cudaSuccess) e = tq::launch_split_images(sp, nullptr);
    if (e == cudaSuccess) e = cudaStreamSynchronize(nullptr);
  }
  if (e != cudaSuccess) {
    tq_split_free(sp);
    return cuda_status(e);
  }
  *out = sp;
  return TQ_OK;
}

void tq_split_free(tq_split* sp) {
  if (!sp) return;
  cudaFree(sp->dperm);
  cudaFree(sp->dimg);
  delete sp;
}

size_t tq_split_plan_workspace_bytes(const tq_split* sp) { return sp ? tq::split_plan_ws_bytes(sp) : 0; }

tq_status tq_split_plan(tq_split* sp, const void* keys, tq_dtype dtype, int B, int64_t S, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!sp || B < 0 || S < 0) return TQ_ERR_ARG;
  if (dtype != TQ_F32 && dtype != TQ_BF16) return TQ_ERR_ARG;
  if ((int64_t(B) * S > 0 && !keys) || !workspace || !aligned(workspace, 8)) return TQ_ERR_ARG;
  if (!aligned(keys, dtype == TQ_F32 ? 4 : 2)) return TQ_ERR_ARG;
  if (workspace_bytes < tq::split_plan_ws_bytes(sp)) return TQ_ERR_WORKSPACE;
  return cuda_status(tq::launch_split_plan(sp, keys, dtype, B, S, workspace, static_cast<cudaStream_t>(stream)));
}

tq_status tq_split_set_plan(tq_split* sp, const int32_t* perm) {
  if (!sp || !perm) return TQ_ERR_ARG;
  for (int h = 0; h < sp->Hkv; ++h) {
    std::vector<char> seen(sp->d, 0);
    for (int p = 0; p < sp->d; ++p) {
      const int32_t c = perm[size_t(h) * sp->d + p];
      if (c < 0 || c >= sp->d || seen[c]) return TQ_ERR_ARG;
      seen[c] = 1;
    }
  }
  cudaError_t e = cudaMemcpy(sp->dperm, perm, size_t(sp->Hkv) * sp->d * sizeof(int32_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = tq::launch_split_images(sp, nullptr);
  if (e == cudaSuccess) e = cudaStreamSynchronize(nullptr);
  return cuda_status(e);
}

tq_status tq_split_get_plan(const tq_split* sp, int32_t* perm) {
  if (!sp || !perm) return TQ_ERR_ARG;
  return cuda_status(
      cudaMemcpy(perm, sp->dperm, size_t(sp->Hkv) * sp->d * sizeof(int32_t), cudaMemcpyDeviceToHost));
}

tq_status tq_split_quantize(const tq_split* sp, const void* keys, tq_dtype dtype, int B, int64_t S,
                            uint8_t* payload_hi, uint16_t* norms_hi, uint8_t* payload_lo, uint16_t* norms_lo,
                            void* stream) {
  if (!sp || B < 0 || S < 0) return TQ_ERR_ARG;
  if (dtype != TQ_F32 && dtype != TQ_BF16) return TQ_ERR_ARG;
  const int64_t n = int64_t(B) * sp->Hkv * S;
  if (n == 0) return TQ_OK;
  if (!keys || !payload_hi || !norms_hi || !payload_lo || !norms_lo) return TQ_ERR_ARG;
  if (!aligned(keys, 16) || !aligned(payload_hi, 16) || !aligned(payload_lo, 16) || !aligned(norms_hi, 4) ||
      !aligned(norms_lo, 4))
    return TQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tq::split_tc_supported(sp, dtype, keys))
    return cuda_status(
        tq::launch_split_quantize_tc(sp, keys, B, S, payload_hi, norms_hi, payload_lo, norms_lo, st));
  cudaError_t e = tq::launch_quantize_simt(sp->hi, keys, dtype, n, sp->d, payload_hi, norms_hi, st,
                                           gather_of(sp, S, true));
  if (e == cudaSuccess)
    e = tq::launch_quantize_simt(sp->lo, keys, dtype, n, sp->d, payload_lo, norms_lo, st, gather_of(sp, S, false),
                                 sp->hi->dstatus);
  return cuda_status(e);
}

size_t tq_split_logits_workspace_bytes(const tq_split* sp, int B, int Hq) {
  if (!sp || B <= 0 || Hq <= 0 || Hq % sp->Hkv) return 0;
  return tq::split_logits_ws_bytes(sp, B, Hq);
}

tq_status tq_split_logits(const tq_split* sp, const float* q, int B, int Hq, int64_t S, const uint8_t* payload_hi,
                          const uint16_t* norms_hi, const uint8_t* payload_lo, const uint16_t* norms_lo,
                          float scale, float* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!sp || B < 0 || Hq < 0 || S < 0) return TQ_ERR_ARG;
  if (B == 0 || Hq == 0) return TQ_OK;
  if (Hq % sp->Hkv) return TQ_ERR_ARG;
  if (!q || !out || (S > 0 && (!payload_hi || !norms_hi || !payload_lo || !norms_lo))) return TQ_ERR_ARG;
  if (!aligned(payload_hi, 16) || !aligned(payload_lo, 16) || !aligned(norms_hi, 4) || !aligned(norms_lo, 4) ||
      !aligned(q, 4) || !aligned(out, 4))
    return TQ_ERR_ARG;
  if (!workspace || !aligned(workspace, 256)) return TQ_ERR_ARG;
  if (workspace_bytes < tq_split_logits_workspace_bytes(sp, B, Hq)) return TQ_ERR_WORKSPACE;
  return cuda_status(tq::launch_split_logits(sp, q, B, Hq, S, payload_hi, norms_hi, payload_lo, norms_lo, scale, out,
                                             workspace, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
