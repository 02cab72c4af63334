// Work lists of the CTA-pair GEMM (k_tc_pair): which (tile, k-tile) pieces
// each pair computes, in which order, under the data-parallel or the
// stream-K schedule. Plain C++ usable on the host as well, so that the
// schedule's invariants can be checked without a GPU.
//
// Data-parallel: pair q takes tiles q, q + npairs, ... whole.
// Stream-K: the first ntiles / npairs - 1 waves stay data-parallel; the
// remaining tiles' (tile, k-tile) space (between one and two waves) is cut
// into npairs equal contiguous ranges, one per pair. A range that ends inside
// a tile computes its first k-tiles (HEAD, stored as an fp32 partial), the
// next pair's range starts inside that tile and computes the rest (TAIL,
// which adds the partial). Each range holds at least one tile's worth of
// k-tiles, so a tile is cut at most once and the HEAD and TAIL of one range
// lie in different tiles. A pair takes its HEAD first and its TAIL only
// after at least as many k-tiles as the HEAD it reads (plus kSkMargin) or,
// failing that, after all its full tiles.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define QLORA_HD __host__ __device__ __forceinline__
#else
#define QLORA_HD inline
#endif

namespace qlora {
namespace psched {

enum { SEG_FULL = 0, SEG_HEAD = 1, SEG_TAIL = 2 };
constexpr int kSkMargin = 4;   // k-tiles of slack between a HEAD's end and the TAIL that reads it

// One piece of work of a CTA pair: k-tiles [k0, k1) of a tile.
struct Seg {
  int tile, k0, k1, kind;
};

// The work list of one CTA pair.
struct PairWork {
  int nseg, items, kt, pair, npairs;
  bool sk;
  int dp;                   // stream-K: data-parallel tiles pair, pair + npairs, ... done first
  int head_tile, head_k1;   // HEAD: k-tiles [0, head_k1) of head_tile (head_tile < 0: none)
  int tail_tile, tail_k0;   // TAIL: k-tiles [tail_k0, kt) of tail_tile (tail_tile < 0: none)
  int full0, nfull, nf_before;   // full tiles full0 .. full0 + nfull - 1; nf_before of them precede the TAIL
};

QLORA_HD PairWork make_work(int pair, int npairs, int ntiles, int kt, bool sk) {
  PairWork w{};
  w.kt = kt;
  w.pair = pair;
  w.npairs = npairs;
  w.sk = sk;
  w.head_tile = -1;
  w.tail_tile = -1;
  if (!sk) {
    w.nseg = (ntiles - pair + npairs - 1) / npairs;
    w.items = w.nseg * kt;
    return w;
  }
  // all but the last full wave stay data-parallel; the rest (at least one
  // wave) is split, so every range holds at least kt k-tiles: a tile is cut
  // at most once, and the HEAD and TAIL of one range lie in different tiles
  w.dp = ntiles / npairs - 1;
  const int base = w.dp * npairs;
  const int64_t total = static_cast<int64_t>(ntiles - base) * kt;
  const int64_t s0 = static_cast<int64_t>(base) * kt + static_cast<int64_t>(pair) * total / npairs;
  const int64_t e0 = static_cast<int64_t>(base) * kt + static_cast<int64_t>(pair + 1) * total / npairs;
  const int a = static_cast<int>(s0 / kt), ka = static_cast<int>(s0 % kt);
  const int b = static_cast<int>(e0 / kt), kb = static_cast<int>(e0 % kt);
  w.items = static_cast<int>(e0 - s0) + w.dp * kt;
  w.full0 = a;
  if (ka > 0) {
    w.tail_tile = a;
    w.tail_k0 = ka;
    w.full0 = a + 1;
  }
  if (kb > 0) {
    w.head_tile = b;
    w.head_k1 = kb;
  }
  w.nfull = b - w.full0;
  int done = kb, nb = 0;
  if (ka > 0)
    while (nb < w.nfull && done + (kt - ka) < ka + kSkMargin) {
      done += kt;
      ++nb;
    }
  w.nf_before = nb;
  w.nseg = w.dp + w.nfull + (ka > 0 ? 1 : 0) + (kb > 0 ? 1 : 0);
  return w;
}

QLORA_HD Seg seg_at(const PairWork& w, int i) {
  if (!w.sk || i < w.dp) return Seg{w.pair + i * w.npairs, 0, w.kt, SEG_FULL};
  i -= w.dp;
  if (w.head_tile >= 0) {
    if (i == 0) return Seg{w.head_tile, 0, w.head_k1, SEG_HEAD};
    --i;
  }
  if (w.tail_tile >= 0) {
    if (i == w.nf_before) return Seg{w.tail_tile, w.tail_k0, w.kt, SEG_TAIL};
    if (i > w.nf_before) --i;
  }
  return Seg{w.full0 + i, 0, w.kt, SEG_FULL};
}


}  // namespace psched
}  // namespace qlora
