// Host-side check of the CTA-pair GEMM work lists (bit_nf4_quantized_06_b200/csrc/pair_sched.h):
// for many (tile count, pair count, k-tiles per tile) combinations, under both schedules,
//   * every (tile, k-tile) is computed by exactly one pair, and each pair's items add up;
//   * full tiles are whole; a cut tile has exactly one HEAD (k-tiles [0, c)) and one TAIL
//     (k-tiles [c, kt)), the TAIL in the next pair;
//   * a HEAD is its pair's first segment after the data-parallel waves;
//   * a TAIL comes after at least as many of its pair's k-tiles as the HEAD it reads plus the
//     margin, or after all of that pair's full tiles.
// Prints "ok <cases>" and exits 0, or prints the first failure and exits 1.
#include <cstdio>
#include <vector>

#include "pair_sched.h"

using namespace qlora::psched;

static int fail(const char* what, int ntiles, int npairs, int kt, bool sk, int q) {
  std::printf("FAIL %s: ntiles=%d npairs=%d kt=%d sk=%d pair=%d\n", what, ntiles, npairs, kt, sk ? 1 : 0, q);
  return 1;
}

static int check(int ntiles, int npairs, int kt, bool sk) {
  std::vector<int> owner(static_cast<size_t>(ntiles) * kt, -1);
  std::vector<int> head_pair(ntiles, -1), head_k1(ntiles, -1), tail_pair(ntiles, -1), tail_k0(ntiles, -1);
  for (int q = 0; q < npairs; ++q) {
    if (!sk && q >= ntiles) break;   // the data-parallel launch has min(tiles, pairs) pairs
    const PairWork w = make_work(q, npairs, ntiles, kt, sk);
    if (w.nseg < 1) return fail("empty work list", ntiles, npairs, kt, sk, q);
    long items = 0;
    for (int i = 0; i < w.nseg; ++i) {
      const Seg g = seg_at(w, i);
      if (g.tile < 0 || g.tile >= ntiles || g.k0 < 0 || g.k0 >= g.k1 || g.k1 > kt)
        return fail("segment out of range", ntiles, npairs, kt, sk, q);
      for (int t = g.k0; t < g.k1; ++t) {
        int& o = owner[static_cast<size_t>(g.tile) * kt + t];
        if (o != -1) return fail("k-tile computed twice", ntiles, npairs, kt, sk, q);
        o = q;
      }
      items += g.k1 - g.k0;
      if (g.kind == SEG_FULL && (g.k0 != 0 || g.k1 != kt)) return fail("partial FULL", ntiles, npairs, kt, sk, q);
      if (g.kind == SEG_HEAD) {
        if (!sk || g.k0 != 0 || g.k1 >= kt || i != w.dp) return fail("bad HEAD", ntiles, npairs, kt, sk, q);
        head_pair[g.tile] = q;
        head_k1[g.tile] = g.k1;
      }
      if (g.kind == SEG_TAIL) {
        if (!sk || g.k0 == 0 || g.k1 != kt) return fail("bad TAIL", ntiles, npairs, kt, sk, q);
        tail_pair[g.tile] = q;
        tail_k0[g.tile] = g.k0;
        // k-tiles this pair has computed (after its data-parallel waves) once the TAIL is done
        long done = 0;
        for (int j = w.dp; j <= i; ++j) done += seg_at(w, j).k1 - seg_at(w, j).k0;
        bool fulls_after = false;
        for (int j = i + 1; j < w.nseg; ++j) fulls_after |= seg_at(w, j).kind == SEG_FULL;
        if (done < g.k0 + kSkMargin && fulls_after) return fail("TAIL too early", ntiles, npairs, kt, sk, q);
      }
    }
    if (items != w.items) return fail("item count", ntiles, npairs, kt, sk, q);
  }
  for (size_t i = 0; i < owner.size(); ++i)
    if (owner[i] == -1) return fail("k-tile never computed", ntiles, npairs, kt, sk, -1);
  for (int t = 0; t < ntiles; ++t) {
    if ((head_pair[t] >= 0) != (tail_pair[t] >= 0)) return fail("HEAD without TAIL", ntiles, npairs, kt, sk, t);
    if (head_pair[t] >= 0 && (tail_pair[t] != head_pair[t] + 1 || head_k1[t] != tail_k0[t]))
      return fail("HEAD/TAIL mismatch", ntiles, npairs, kt, sk, t);
  }
  return 0;
}

int main() {
  const int pairs[] = {1, 2, 3, 7, 37, 72, 74};
  const int kts[] = {1, 2, 3, 5, 17, 65, 173, 345};
  std::vector<int> tiles;
  for (int t = 1; t <= 150; ++t) tiles.push_back(t);
  for (int t : {199, 256, 344, 368, 688}) tiles.push_back(t);
  long cases = 0;
  for (int nt : tiles)
    for (int np : pairs)
      for (int kt : kts) {
        if (check(nt, np, kt, false)) return 1;
        ++cases;
        if (nt >= np) {
          if (check(nt, np, kt, true)) return 1;
          ++cases;
        }
      }
  std::printf("ok %ld\n", cases);
  return 0;
}
