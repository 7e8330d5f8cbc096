// How the persistent tensor-core GEMM deals a launch's tiles to its CTAs.
//
// A launch's tiles are ordered by cost (k-blocks per tile), largest first. Plain round robin
// (CTA c takes tiles c, c + ctas, ...) leaves the CTAs that drew one of the few largest tiles
// with a whole large tile more work than the rest. The phased dealing below gives those CTAs
// correspondingly fewer of the next tiles:
//   phase A: r0 full rounds of round robin (the largest class, as far as it fills rounds);
//   phase B: the b (< ctas) remaining tiles of that class, one each to CTAs 0 .. b-1;
//   phase C: q rounds over CTAs b .. ctas-1 only (about one large tile's worth of the next
//            tiles each);
//   phase D: round robin over all CTAs for the rest.
// b = 0 is plain round robin. Every tile goes to exactly one CTA, and each CTA's tiles come
// in increasing order (the kernel walks its matrices forward).
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define WQ_DEAL_HD __host__ __device__ __forceinline__
#else
#define WQ_DEAL_HD inline
#endif

namespace wq {

struct TileDeal {
  int r0;  // phase A rounds
  int b;   // phase B tiles (0: plain round robin)
  int q;   // phase C rounds
};

// Index of CTA `cta`'s j-th tile (j = 0, 1, ...) among `total` tiles dealt to `ctas` CTAs,
// or -1 once the CTA has no more.
WQ_DEAL_HD int dealt_tile(int cta, int j, int ctas, int total, TileDeal d) {
  int64_t t;
  if (d.b <= 0 || j < d.r0) {
    t = (int64_t)cta + (int64_t)ctas * j;
  } else {
    const int64_t ta = (int64_t)ctas * d.r0;           // first tile of phase B
    const int64_t tc = ta + d.b + (int64_t)(ctas - d.b) * d.q;  // first tile of phase D
    const int jj = j - d.r0;
    if (cta < d.b) {
      t = jj == 0 ? ta + cta : tc + cta + (int64_t)ctas * (jj - 1);
    } else {
      t = jj < d.q ? ta + d.b + (cta - d.b) + (int64_t)(ctas - d.b) * jj
                   : tc + cta + (int64_t)ctas * (jj - d.q);
    }
  }
  return t < total ? (int)t : -1;
}

// The dealing for tiles whose costs are non-increasing: n1 tiles of the largest cost c1,
// then tiles whose largest cost is c2 (0 when there are none).
WQ_DEAL_HD TileDeal plan_deal(int ctas, int n1, int c1, int c2) {
  TileDeal d{0, 0, 0};
  if (ctas <= 1 || c2 <= 0 || n1 <= 0) return d;
  d.r0 = n1 / ctas;
  d.b = n1 % ctas;
  d.q = d.b > 0 ? (c1 + c2 / 2) / c2 : 0;
  if (d.q == 0) d.b = 0;
  return d;
}

}  // namespace wq
