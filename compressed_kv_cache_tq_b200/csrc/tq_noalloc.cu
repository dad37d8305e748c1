// tq_logits_noalloc: the decode-logits call for callers that cannot allocate
// device memory at the point of use.  Its scratch memory (the prepared query
// fragments and per-head scales that tq_logits keeps in the caller's
// workspace) lives in one file-scope device array of this library instead.
#include <cuda_runtime.h>

#include <mutex>

#include "tq_internal.h"

namespace {

// Every GPU that loads libtq holds this array until the process exits.
static __device__ __align__(256) uint8_t g_logits_scratch[TQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the array on device `dev` (the current device).  In host
// code the array's name is only a host-side stand-in, so the address is looked
// up once per device, with that device current, and cached.  A cached address
// belongs to the device's context at the time of the look-up: after a
// cudaDeviceReset of that device it is stale, and the process must not call
// this entry point on that device again.
cudaError_t scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_logits_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

tq_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return TQ_OK;
  tq::set_cuda_error(e);
  return e == cudaErrorMemoryAllocation ? TQ_ERR_NOMEM : TQ_ERR_CUDA;
}

}  // namespace

extern "C" tq_status tq_logits_noalloc(const tq_ctx* ctx, const float* q, int B, int Hq, int Hkv, int64_t S,
                                       const uint8_t* payload, const uint16_t* norms, float scale, float* out,
                                       void* stream) {
  if (!ctx || B < 0 || Hq < 0 || Hkv < 0 || S < 0) return TQ_ERR_ARG;
  if (B == 0 || Hq == 0) return TQ_OK;
  if (Hkv == 0 || Hq % Hkv) return TQ_ERR_ARG;
  if (!q || !out || (S > 0 && (!payload || !norms))) return TQ_ERR_ARG;
  if (!aligned(payload, 16) || !aligned(norms, 4) || !aligned(q, 4) || !aligned(out, 4)) return TQ_ERR_ARG;
  if (tq_logits_workspace_bytes(ctx, B, Hq, Hkv) > TQ_NOALLOC_SCRATCH_BYTES) return TQ_ERR_WORKSPACE;
  // the kernels run on the current device and read ctx's tables: they must be the same device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev != ctx->device) return TQ_ERR_ARG;
  void* scratch = nullptr;
  e = scratch_address(dev, &scratch);
  if (e == cudaSuccess)
    e = tq::launch_logits(ctx, q, B, Hq, Hkv, S, payload, norms, scale, out, scratch,
                          static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}
