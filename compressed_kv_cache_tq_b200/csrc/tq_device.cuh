// Device helpers shared by the libtq kernels: packed-layout addressing
// (the layout is specified in include/tq.h) and fp16 helpers.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace tq {

// Geometry of the packed row for (d, m, b').  The layout has dp and mp slots:
// d and m rounded up to multiples of 64; the slots past d (codes) and past m
// (sign bits) are zero.
struct RowGeom {
  int d, m, bmse;
  int dp, mp;          // layout slots
  int uq, uqm;         // code units and sign units per quarter (dp/64, mp/64)
  int per_q;           // halfwords per quarter chunk
  int row_bytes;
};

__host__ __device__ inline RowGeom make_geom(int d, int m, int bmse) {
  RowGeom g;
  g.d = d;
  g.m = m;
  g.bmse = bmse;
  g.dp = (d + 63) / 64 * 64;
  g.mp = (m + 63) / 64 * 64;
  g.uq = g.dp / 64;
  g.uqm = g.mp / 64;
  g.per_q = bmse * g.uq + g.uqm;
  g.row_bytes = 8 * g.per_q;   // 4 quarters x 2 bytes x per_q
  return g;
}

// Code of rotated coordinate j in a packed row (halfword view).
__device__ inline int unpack_code(const uint16_t* hw, const RowGeom& g, int j) {
  const int qd = g.dp / 4;
  const int q = j / qd, rem = j - q * qd;
  const int r = rem >> 2, e = rem & 3, u = r >> 2, i = r & 3;
  const uint16_t* base = hw + q * g.per_q + u * g.bmse;
  switch (g.bmse) {
    case 1:
      return (base[0] >> (4 * e + i)) & 1;
    case 2:
      return (base[i >> 1] >> (4 * e + 2 * (i & 1))) & 3;
    default:
      if (i < 3) return (base[i] >> (4 * e)) & 7;
      return ((base[0] >> (4 * e + 3)) & 1) | (((base[1] >> (4 * e + 3)) & 1) << 1) |
             (((base[2] >> (4 * e + 3)) & 1) << 2);
  }
}

// Sign bit (1 = +1) of JL coordinate i in a packed row.
__device__ inline int unpack_sign(const uint16_t* hw, const RowGeom& g, int i) {
  const int qm = g.mp / 4;
  const int q = i / qm, rem = i - q * qm;
  const int r = rem >> 2, e = rem & 3, u = r >> 2, ii = r & 3;
  const uint16_t h = hw[q * g.per_q + g.bmse * g.uq + u];
  return (h >> (4 * e + ii)) & 1;
}

// Build packed halfword `h` of a row from per-slot codes and sign bits held in
// shared memory (codes[0 .. dp), bits[0 .. mp) as bytes, zero past d and m).
__device__ inline uint16_t pack_halfword(const uint8_t* codes, const uint8_t* bits, const RowGeom& g, int h) {
  const int q = h / g.per_q, loc = h - q * g.per_q;
  uint32_t out = 0;
  if (loc < g.bmse * g.uq) {
    const int u = loc / g.bmse, ih = loc - u * g.bmse;
    const uint8_t* cq = codes + q * (g.dp / 4);
    for (int e = 0; e < 4; ++e) {
      if (g.bmse == 1) {
        for (int i = 0; i < 4; ++i) out |= uint32_t(cq[4 * (4 * u + i) + e] & 1) << (4 * e + i);
      } else if (g.bmse == 2) {
        out |= uint32_t(cq[4 * (4 * u + 2 * ih) + e] & 3) << (4 * e);
        out |= uint32_t(cq[4 * (4 * u + 2 * ih + 1) + e] & 3) << (4 * e + 2);
      } else {
        out |= uint32_t(cq[4 * (4 * u + ih) + e] & 7) << (4 * e);
        out |= uint32_t((cq[4 * (4 * u + 3) + e] >> ih) & 1) << (4 * e + 3);
      }
    }
  } else {
    const int u = loc - g.bmse * g.uq;
    const uint8_t* bq = bits + q * (g.mp / 4);
    for (int e = 0; e < 4; ++e)
      for (int i = 0; i < 4; ++i) out |= uint32_t(bq[4 * (4 * u + i) + e] & 1) << (4 * e + i);
  }
  return uint16_t(out);
}

__device__ inline float half_bits_to_float(uint16_t b) { return __half2float(__ushort_as_half(b)); }

}  // namespace tq
