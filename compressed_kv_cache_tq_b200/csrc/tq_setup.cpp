// Host-side construction of the data-oblivious TurboQuant parameters
// (airosetta.com "Google TurboQuant", stage 1: rotation from the QR of a
// Gaussian matrix, Lloyd-Max codebook for the Beta coordinate law, codebook
// precomputed; stage 2: Gaussian JL matrix).  Everything here runs once per
// context in fp64 and is uploaded to the device.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "tq_internal.h"

namespace {

// ---------------------------------------------------------------------------
// Philox4x32-10 counter-based generator (Salmon et al., SC'11).
// ---------------------------------------------------------------------------
struct Philox4 {
  uint32_t v[4];
};

Philox4 philox4x32_10(Philox4 x, uint32_t k0, uint32_t k1) {
  for (int round = 0; round < 10; ++round) {
    const uint64_t prod0 = uint64_t(0xD2511F53u) * x.v[0];
    const uint64_t prod1 = uint64_t(0xCD9E8D57u) * x.v[2];
    Philox4 y;
    y.v[0] = uint32_t(prod1 >> 32) ^ x.v[1] ^ k0;
    y.v[1] = uint32_t(prod1);
    y.v[2] = uint32_t(prod0 >> 32) ^ x.v[3] ^ k1;
    y.v[3] = uint32_t(prod0);
    x = y;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return x;
}

// Normals 2b and 2b+1 of (seed, stream) come from Philox block b: two 53-bit
// uniforms (the first shifted into (0, 1]) and the Box-Muller transform.
void fill_gaussian(uint64_t seed, uint32_t stream, size_t count, double* out) {
  const uint32_t k0 = uint32_t(seed), k1 = uint32_t(seed >> 32);
  const double two53 = 9007199254740992.0;
  for (size_t b = 0; 2 * b < count; ++b) {
    Philox4 c{{uint32_t(b), uint32_t(uint64_t(b) >> 32), stream, 0u}};
    Philox4 w = philox4x32_10(c, k0, k1);
    const uint64_t ia = (uint64_t(w.v[0] >> 5) << 26) | uint64_t(w.v[1] >> 6);
    const uint64_t ib = (uint64_t(w.v[2] >> 5) << 26) | uint64_t(w.v[3] >> 6);
    const double u1 = (double(ia) + 1.0) / two53;
    const double u2 = double(ib) / two53;
    const double radius = std::sqrt(-2.0 * std::log(u1));
    const double angle = 6.283185307179586476925286766559 * u2;
    out[2 * b] = radius * std::cos(angle);
    if (2 * b + 1 < count) out[2 * b + 1] = radius * std::sin(angle);
  }
}

// ---------------------------------------------------------------------------
// Householder QR: G = Q T, Q orthogonal, columns of Q flipped so that the
// diagonal of T is positive.  Returns Q (row-major d x d).
// ---------------------------------------------------------------------------
std::vector<double> orthogonal_factor(std::vector<double> A, int d) {
  std::vector<double> Q(size_t(d) * d, 0.0);
  for (int i = 0; i < d; ++i) Q[size_t(i) * d + i] = 1.0;
  std::vector<double> v(d), w(d);
  for (int k = 0; k < d; ++k) {
    double norm2 = 0.0;
    for (int i = k; i < d; ++i) norm2 += A[size_t(i) * d + k] * A[size_t(i) * d + k];
    const double xnorm = std::sqrt(norm2);
    if (xnorm == 0.0) continue;
    const double x0 = A[size_t(k) * d + k];
    const double alpha = (x0 >= 0.0) ? -xnorm : xnorm;   // reflect x onto alpha e1
    for (int i = k; i < d; ++i) v[i] = A[size_t(i) * d + k];
    v[k] -= alpha;
    double vv = 0.0;
    for (int i = k; i < d; ++i) vv += v[i] * v[i];
    if (vv == 0.0) continue;
    const double beta = 2.0 / vv;
    // A[k:, k:] -= beta v (v^T A[k:, k:])
    for (int j = k; j < d; ++j) {
      double s = 0.0;
      for (int i = k; i < d; ++i) s += v[i] * A[size_t(i) * d + j];
      s *= beta;
      for (int i = k; i < d; ++i) A[size_t(i) * d + j] -= s * v[i];
    }
    // Q[:, k:] -= beta (Q[:, k:] v) v^T   (Q accumulates H_0 H_1 ... H_k)
    for (int i = 0; i < d; ++i) {
      double s = 0.0;
      for (int j = k; j < d; ++j) s += Q[size_t(i) * d + j] * v[j];
      s *= beta;
      for (int j = k; j < d; ++j) Q[size_t(i) * d + j] -= s * v[j];
    }
  }
  for (int k = 0; k < d; ++k) {
    if (A[size_t(k) * d + k] < 0.0)
      for (int i = 0; i < d; ++i) Q[size_t(i) * d + k] = -Q[size_t(i) * d + k];
  }
  return Q;
}

// ---------------------------------------------------------------------------
// Lloyd-Max codebook for w(x) = (1 - x^2)^((d-3)/2) on [-1, 1] (the law of
// one coordinate of a uniformly random unit vector in R^d).  Cell integrals
// by composite Gauss-Legendre quadrature; the normalising constant cancels in
// the centroid.
// ---------------------------------------------------------------------------
struct GaussLegendre {
  std::vector<double> x, w;
  explicit GaussLegendre(int n) : x(n), w(n) {
    for (int i = 0; i < n; ++i) {
      double z = std::cos(3.141592653589793238462643 * (i + 0.75) / (n + 0.5));
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = 0.0;
        for (int j = 1; j <= n; ++j) {
          const double p2 = p1;
          p1 = p0;
          p0 = ((2.0 * j - 1.0) * z * p1 - (j - 1.0) * p2) / j;
        }
        const double dp = n * (z * p0 - p1) / (z * z - 1.0);
        const double dz = p0 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) {
          x[i] = z;
          w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
          break;
        }
        x[i] = z;
        w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
      }
    }
  }
};

struct CellIntegrals {
  double mass, moment;
};

CellIntegrals cell_integrals(double lo, double hi, double alpha, double width, const GaussLegendre& gl) {
  CellIntegrals r{0.0, 0.0};
  if (hi <= lo) return r;
  const int panels = std::max(1, int(std::ceil((hi - lo) / width)));
  const double h = (hi - lo) / panels;
  for (int p = 0; p < panels; ++p) {
    const double a = lo + p * h, mid = a + 0.5 * h;
    for (size_t i = 0; i < gl.x.size(); ++i) {
      const double x = mid + 0.5 * h * gl.x[i];
      const double wx = std::pow(std::max(0.0, 1.0 - x * x), alpha) * gl.w[i] * 0.5 * h;
      r.mass += wx;
      r.moment += wx * x;
    }
  }
  return r;
}

void lloyd_max(int d, int bmse, std::vector<double>& c, std::vector<double>& t) {
  const int L = 1 << bmse;
  const double alpha = 0.5 * (d - 3);
  const double width = std::min(0.25, 0.5 / std::sqrt(double(d)));
  GaussLegendre gl(24);
  c.assign(L, 0.0);
  t.assign(L - 1, 0.0);
  // start: uniform levels over +-3 standard deviations of the coordinate law
  const double sd = 1.0 / std::sqrt(double(d));
  for (int i = 0; i < L; ++i) c[i] = std::max(-0.999, std::min(0.999, sd * (-3.0 + 6.0 * (i + 0.5) / L)));
  double best = 1e300;
  int stall = 0;
  for (int it = 0; it < 200000; ++it) {
    for (int i = 0; i + 1 < L; ++i) t[i] = 0.5 * (c[i] + c[i + 1]);
    double delta = 0.0;
    for (int i = 0; i < L; ++i) {
      const double lo = (i == 0) ? -1.0 : t[i - 1];
      const double hi = (i == L - 1) ? 1.0 : t[i];
      const CellIntegrals ci = cell_integrals(lo, hi, alpha, width, gl);
      const double nc = ci.mass > 0 ? ci.moment / ci.mass : 0.5 * (lo + hi);
      delta = std::max(delta, std::fabs(nc - c[i]));
      c[i] = nc;
    }
    if (delta < 1e-16) break;
    if (delta < best) {
      best = delta;
      stall = 0;
    } else if (++stall > 50 && delta < 1e-13) {
      break;
    }
  }
  std::vector<double> s(L);
  for (int i = 0; i < L; ++i) s[i] = 0.5 * (c[i] - c[L - 1 - i]);
  c = s;
  for (int i = 0; i + 1 < L; ++i) t[i] = 0.5 * (c[i] + c[i + 1]);
}

// Shared-memory image of one K-major operand tile for tcgen05 with the
// 128-byte swizzle: rows of 64 16-bit elements per K block, 16-byte chunk
// index XORed with (row mod 8).  rows x K elements, K a multiple of 64.
template <typename T>
void write_swizzled(const std::vector<T>& src, int rows, int K, uint8_t* dst) {
  const int kblocks = K / 64;
  for (int kb = 0; kb < kblocks; ++kb)
    for (int r = 0; r < rows; ++r)
      for (int chunk = 0; chunk < 8; ++chunk) {
        uint8_t* out = dst + size_t(kb) * rows * 128 + size_t(r) * 128 + size_t((chunk ^ (r & 7)) * 16);
        std::memcpy(out, &src[size_t(r) * K + kb * 64 + chunk * 8], 16);
      }
}

template <typename T>
cudaError_t upload(const std::vector<T>& h, T** d) {
  *d = nullptr;
  if (h.empty()) return cudaSuccess;   // the JL tables of the MSE-only variant
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(d), h.size() * sizeof(T));
  if (e != cudaSuccess) return e;
  return cudaMemcpy(*d, h.data(), h.size() * sizeof(T), cudaMemcpyHostToDevice);
}

}  // namespace

namespace tq {
static thread_local char g_cuda_msg[256] = "";
void set_cuda_error(cudaError_t e) {
  std::snprintf(g_cuda_msg, sizeof(g_cuda_msg), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
}
}  // namespace tq

extern "C" {

const char* tq_last_cuda_error(void) { return tq::g_cuda_msg; }

const char* tq_strerror(tq_status s) {
  switch (s) {
    case TQ_OK: return "ok";
    case TQ_ERR_ARG: return "invalid argument";
    case TQ_ERR_UNSUPPORTED: return "unsupported shape or type";
    case TQ_ERR_CUDA: return "CUDA error";
    case TQ_ERR_NOMEM: return "out of memory";
    case TQ_ERR_WORKSPACE: return "workspace too small";
    case TQ_ERR_DEVICE: return "a kernel reported a device-side error";
    case TQ_ERR_RANGE: return "a norm exceeded the fp16 range";
  }
  return "unknown status";
}

void tq_free(tq_ctx* ctx) {
  if (!ctx) return;
  cudaFree(ctx->dR);
  cudaFree(ctx->dRt);
  cudaFree(ctx->dP);
  cudaFree(ctx->dPt);
  cudaFree(ctx->dR64);
  cudaFree(ctx->dP64);
  cudaFree(ctx->dc64);
  cudaFree(ctx->dBimg);
  cudaFree(ctx->dBimgWide);
  cudaFree(ctx->dstatus);
  delete ctx;
}

// m = 0: the MSE-only variant (no sign sketch)
static bool dims_ok(int d, int bits, int m) {
  return !(d < 64 || d > 256 || d % 8 || (m != 0 && (m < 64 || m > 256 || m % 8)) || bits < 2 || bits > 4);
}

static void build_tables(int d, int bits, int m, uint64_t seed, uint32_t stream_base, std::vector<double>& R,
                         std::vector<double>& P, std::vector<double>& c, std::vector<double>& t) {
  std::vector<double> G(size_t(d) * d);
  fill_gaussian(seed, stream_base, G.size(), G.data());
  R = orthogonal_factor(G, d);
  P.resize(size_t(m) * d);
  fill_gaussian(seed, stream_base + 1, P.size(), P.data());
  // the JL Gaussian is stored as fp16 samples (nearest value, one rounding)
  for (double& v : P) v = double(__half2float(__double2half(v)));
  lloyd_max(d, bits - 1, c, t);
}

tq_status tq_host_tables(int d, int bits, int m, uint64_t seed, uint32_t stream_base, double* R, double* P,
                         double* c, double* t) {
  if (!dims_ok(d, bits, m)) return TQ_ERR_UNSUPPORTED;
  std::vector<double> vR, vP, vc, vt;
  build_tables(d, bits, m, seed, stream_base, vR, vP, vc, vt);
  if (R) std::memcpy(R, vR.data(), vR.size() * sizeof(double));
  if (P) std::memcpy(P, vP.data(), vP.size() * sizeof(double));
  if (c) std::memcpy(c, vc.data(), vc.size() * sizeof(double));
  if (t) std::memcpy(t, vt.data(), vt.size() * sizeof(double));
  return TQ_OK;
}

tq_status tq_init_ex(int d, int bits, int m, uint64_t seed, uint32_t stream_base, tq_ctx** out) {
  if (!out) return TQ_ERR_ARG;
  *out = nullptr;
  if (!dims_ok(d, bits, m)) return TQ_ERR_UNSUPPORTED;
  tq_ctx* ctx = new (std::nothrow) tq_ctx();
  if (!ctx) return TQ_ERR_NOMEM;
  ctx->d = d;
  ctx->m = m;
  ctx->bits = bits;
  ctx->bmse = bits - 1;
  ctx->levels = 1 << (bits - 1);
  // layout slots: d and m rounded up to multiples of 64 (zero padding slots)
  ctx->row_bytes = (d + 63) / 64 * 64 * (bits - 1) / 8 + (m + 63) / 64 * 8;
  ctx->seed = seed;
  ctx->stream_base = stream_base;
  cudaGetDevice(&ctx->device);

  build_tables(d, bits, m, seed, stream_base, ctx->R, ctx->P, ctx->c, ctx->t);

  // kernel-side small tables
  ctx->cb.levels = ctx->levels;
  for (int i = 0; i < tq::kMaxLevels; ++i) ctx->cb.c[i] = i < ctx->levels ? float(ctx->c[i]) : 0.f;
  for (int i = 0; i < tq::kMaxLevels - 1; ++i) ctx->cb.t[i] = i < ctx->levels - 1 ? float(ctx->t[i]) : 2.f;
  double cmax = 0.0;
  for (double v : ctx->c) cmax = std::max(cmax, std::fabs(v));
  const double kc = 32000.0 / cmax;
  ctx->lut = tq::CodeLut{};
  for (int v = 0; v < ctx->levels; ++v) {
    const long ci = std::lrint(ctx->c[v] * kc);
    const long hi = long(std::floor((ci + 128) / 256.0));
    const long lo = ci - 256 * hi;
    ctx->lut.hi[v / 4] |= uint32_t(uint8_t(int8_t(hi))) << (8 * (v % 4));
    ctx->lut.lo[v / 4] |= uint32_t(uint8_t(int8_t(lo))) << (8 * (v % 4));
  }
  ctx->lut.inv_scale = float(1.0 / kc);

  std::vector<float> Rf(size_t(d) * d), Rt(size_t(d) * d), Pf(size_t(m) * d), Pt(size_t(m) * d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) {
      Rf[size_t(i) * d + j] = float(ctx->R[size_t(i) * d + j]);
      Rt[size_t(j) * d + i] = float(ctx->R[size_t(i) * d + j]);
    }
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < d; ++j) {
      Pf[size_t(i) * d + j] = float(ctx->P[size_t(i) * d + j]);
      Pt[size_t(j) * m + i] = float(ctx->P[size_t(i) * d + j]);
    }
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = upload(Rf, &ctx->dR);
  if (e == cudaSuccess) e = upload(Rt, &ctx->dRt);
  if (e == cudaSuccess) e = upload(Pf, &ctx->dP);
  if (e == cudaSuccess) e = upload(Pt, &ctx->dPt);
  if (e == cudaSuccess) e = upload(ctx->R, &ctx->dR64);
  if (e == cudaSuccess) e = upload(ctx->P, &ctx->dP64);
  if (e == cudaSuccess) e = upload(ctx->c, &ctx->dc64);
  if (e == cudaSuccess && d == 128 && (m == 128 || m == 0)) {
    // R split into bf16 hi + lo (keys are bf16, so K R^T needs two MMAs); the
    // stored JL samples P are exact in fp16 (the residual is split into fp16
    // hi + lo in the kernel).  B operand rows are output coordinates, K the
    // input ones.
    std::vector<__nv_bfloat16> rh(size_t(d) * d), rl(size_t(d) * d);
    std::vector<__half> ph(size_t(m) * d);
    for (size_t i = 0; i < rh.size(); ++i) {
      const double v = ctx->R[i];
      rh[i] = __float2bfloat16_rn(float(v));
      rl[i] = __float2bfloat16_rn(float(v - double(__bfloat162float(rh[i]))));
    }
    for (size_t i = 0; i < ph.size(); ++i) ph[i] = __double2half(ctx->P[i]);
    std::vector<uint8_t> img(size_t(3) * 128 * 128 * 2);
    write_swizzled(rh, 128, 128, img.data());
    write_swizzled(rl, 128, 128, img.data() + 32768);
    if (m == 128) write_swizzled(ph, 128, 128, img.data() + 65536);   // m = 0: no JL operand
    e = upload(img, &ctx->dBimg);
  }
  if (e == cudaSuccess && d > 192 && d <= 256 && m == d) {
    // Wide quantizer (192 < d <= 256, m = d: a layout of 256 slots): the same operands padded with
    // zeros to Np = d rounded up to 16 rows and 256 input columns, stored as
    // four 64-column atoms per matrix (R_hi, R_lo, P), each atom contiguous
    // (Np rows of 128 bytes, 128-byte swizzle) so that it streams into shared
    // memory with one bulk copy.
    const int np = (d + 15) / 16 * 16, kp = 256;
    std::vector<__nv_bfloat16> rh(size_t(np) * kp, __float2bfloat16_rn(0.f)), rl(rh);
    std::vector<__half> ph(size_t(np) * kp, __float2half_rn(0.f));
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < d; ++j) {
        const double v = ctx->R[size_t(i) * d + j];
        const __nv_bfloat16 hi = __float2bfloat16_rn(float(v));
        rh[size_t(i) * kp + j] = hi;
        rl[size_t(i) * kp + j] = __float2bfloat16_rn(float(v - double(__bfloat162float(hi))));
        ph[size_t(i) * kp + j] = __double2half(ctx->P[size_t(i) * d + j]);
      }
    const size_t mat = size_t(np) * kp * 2;
    std::vector<uint8_t> img(3 * mat);
    write_swizzled(rh, np, kp, img.data());
    write_swizzled(rl, np, kp, img.data() + mat);
    write_swizzled(ph, np, kp, img.data() + 2 * mat);
    e = upload(img, &ctx->dBimgWide);
  }
  if (e == cudaSuccess) e = cudaMalloc(&ctx->dstatus, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(ctx->dstatus, 0, sizeof(uint32_t));
  if (e != cudaSuccess) {
    tq::set_cuda_error(e);
    tq_free(ctx);
    return e == cudaErrorMemoryAllocation ? TQ_ERR_NOMEM : TQ_ERR_CUDA;
  }
  *out = ctx;
  return TQ_OK;
}

tq_status tq_init(int d, int bits, uint64_t seed, tq_ctx** out) {
  return tq_init_ex(d, bits, d, seed, 0u, out);
}

tq_status tq_info(const tq_ctx* ctx, int* d, int* bits, int* m, int* row_bytes) {
  if (!ctx) return TQ_ERR_ARG;
  if (d) *d = ctx->d;
  if (bits) *bits = ctx->bits;
  if (m) *m = ctx->m;
  if (row_bytes) *row_bytes = ctx->row_bytes;
  return TQ_OK;
}

tq_status tq_export_tables(const tq_ctx* ctx, double* R, double* P, double* c, double* t) {
  if (!ctx) return TQ_ERR_ARG;
  if (R) std::memcpy(R, ctx->R.data(), ctx->R.size() * sizeof(double));
  if (P) std::memcpy(P, ctx->P.data(), ctx->P.size() * sizeof(double));
  if (c) std::memcpy(c, ctx->c.data(), ctx->c.size() * sizeof(double));
  if (t) std::memcpy(t, ctx->t.data(), ctx->t.size() * sizeof(double));
  return TQ_OK;
}

tq_status tq_set_wait_budget(tq_ctx* ctx, int64_t cycles) {
  if (!ctx || cycles < 0) return TQ_ERR_ARG;
  ctx->wait_budget = cycles;
  return TQ_OK;
}

tq_status tq_check_device_status(const tq_ctx* ctx, void* stream, uint32_t* word) {
  if (!ctx) return TQ_ERR_ARG;
  uint32_t h = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&h, ctx->dstatus, sizeof(uint32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && h) e = cudaMemsetAsync(ctx->dstatus, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) {
    tq::set_cuda_error(e);
    return TQ_ERR_CUDA;
  }
  if (word) *word = h;
  if (h & (tq::kStatusQuantizeTc | tq::kStatusSearchTc)) return TQ_ERR_DEVICE;
  return h ? TQ_ERR_RANGE : TQ_OK;
}

}  // extern "C"
