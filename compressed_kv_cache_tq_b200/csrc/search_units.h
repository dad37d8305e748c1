// Work schedule of the tensor-core search (k_search_tc.cu): which (query
// tile, row tile) units each CTA scores, and the group size the launcher
// picks.  Host and device code; the host test compiles it alone.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define TQ_SU_HD __host__ __device__
#else
#define TQ_SU_HD
#endif

namespace tq {

// Work: unit (query tile, row tile).  The grid is cut into groups of G
// consecutive CTAs and the query tiles into groups of G consecutive tiles.
// Group g of the NG = ctas / G takes the contiguous units [U g / NG,
// U (g + 1) / NG) of the U = ceil(qtiles / G) x row_tiles pairs (query-tile
// group qg, row tile t), qg-major, and its member r works on query tile
// G qg + r of each: a CTA keeps one query tile (or two) for long stretches,
// and the G members of a group read the same row tiles in the same order, so
// that all but the first find each tile in L2 (the row matrix crosses HBM
// about ceil(qtiles / G) times instead of qtiles times).  A member whose
// query tile is past the last one skips those units.  (A part-major
// round-robin order that makes all CTAs stream the same rows at the same
// time, restarting each query's running k-th best at every part, measured
// slower: 17.0 against 13.7 ms at 10^6 x 10^4.)
struct Units {
  int64_t qtiles, row_tiles, u, u1;
  int64_t qt, t;
  int64_t G, r;
  TQ_SU_HD Units(int64_t qtiles_, int64_t row_tiles_, int64_t cta, int64_t ctas, int64_t G_)
      : qtiles(qtiles_), row_tiles(row_tiles_), G(G_) {
    const int64_t ng = ctas / G, g = cta / G;
    r = cta - g * G;
    const int64_t total = ((qtiles + G - 1) / G) * row_tiles;
    u = total * g / ng - 1;
    u1 = total * (g + 1) / ng;
    qt = t = 0;
  }
  // advance to the next (query tile, row tile); false when done
  TQ_SU_HD bool next() {
    while (++u < u1) {
      const int64_t qg = u / row_tiles;
      qt = qg * G + r;
      if (qt >= qtiles) {   // no such tile: skip the rest of this query-tile group
        u = (qg + 1) * row_tiles - 1;
        continue;
      }
      t = u - qg * row_tiles;
      return true;
    }
    return false;
  }
};

// CTAs per group of the schedule above (host side): groups of eight when
// there are enough query tiles that an idle member (query tile past the end)
// costs little; the grid is then the largest multiple of the group size that
// fits the SMs (144 of 148).  Measured at 10^6 rows x 10^4 queries (79 query
// tiles): 12.1 / 13.5 ms (b = 2 / 4) for single CTAs, 11.9 / 13.4 for groups
// of four, 11.5 / 12.6 for groups of eight.
inline int64_t search_group(int64_t qtiles, int sms) {
  int64_t g = qtiles >= 32 ? 8 : qtiles >= 16 ? 4 : qtiles >= 8 ? 2 : 1;
  while (g > 1 && sms < g) g >>= 1;
  return g;
}

}  // namespace tq
