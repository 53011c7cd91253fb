// Host-side check of the fused kernel's work schedule (get_item in fl_gemm.cuh, the same
// function the kernel's producer, MMA and epilogue warps call), on the CPU.
// For each case it enumerates every cluster's items and checks that:
//   * every (tile, K block) unit is computed exactly once;
//   * a cluster has at most one PARTIAL item and at most one FINISH item; its PARTIAL
//     item, if any, is its first stream-K item, and its FINISH item its last;
//   * every tile cut by the stream-K ranges has exactly one FINISH item, held by the
//     cluster that computes the tile's first K block, and its writer list w0..w1 is
//     exactly the set of clusters with a PARTIAL item of that tile;
//   * a FINISH item's writers all have higher cluster indices.
// Prints "schedule ok: N cases" and exits 0, or the first violation and exits 1.
#include <cstdio>
#include <algorithm>
#include <cstdlib>
#include <vector>

#include "../../gemm_bias_activation_tcgen05_b200/csrc/fl_gemm.cuh"

using fl::Item;
using fl::KParams;

static int fail(const char* what, int a, int b, int c) {
  std::printf("schedule violation: %s (%d, %d, %d)\n", what, a, b, c);
  return 1;
}

// tiles_a x tiles_b tiles, nkb K blocks, sk stream-K tiles over skc clusters, ncl clusters
static int check(int tiles_a, int tiles_b, int nkb, int sk, int skc, int ncl) {
  KParams p{};
  p.tiles_a = tiles_a;
  p.tiles_b = tiles_b;
  p.num_kb = nkb;
  p.sk_tiles = sk;
  p.sk_clusters = skc;
  fl::set_dp_split(p, ncl);
  const int T = tiles_a * tiles_b;
  std::vector<int> cover((size_t)T * nkb, 0), finisher(T, -1), nfinish(T, 0);
  std::vector<std::vector<int>> writers(T), listed(T);
  for (int cl = 0; cl < ncl; ++cl) {
    int partials = 0, finishes = 0, sk_items = 0, last_kind = -1;
    for (int i = 0;; ++i) {
      Item it;
      if (!fl::get_item(p, cl, ncl, 0, nkb, i, it)) break;
      if (i > 100000) return fail("runaway item list", cl, i, 0);
      if (it.tile < 0 || it.tile >= T || it.kb0 < 0 || it.kb1 > nkb || it.kb0 >= it.kb1)
        return fail("item out of range", cl, it.tile, it.kb0);
      for (int kb = it.kb0; kb < it.kb1; ++kb) cover[(size_t)it.tile * nkb + kb]++;
      const bool is_sk = it.tile >= T - sk;
      if (is_sk) ++sk_items;
      if (it.kind == fl::IT_PARTIAL) {
        if (++partials > 1) return fail("two partial items", cl, it.tile, 0);
        if (sk_items != 1) return fail("partial item is not the first stream-K item", cl, it.tile, sk_items);
        if (it.kb0 == 0) return fail("partial item holds the tile's first K block", cl, it.tile, 0);
        writers[it.tile].push_back(cl);
      } else if (it.kind == fl::IT_FINISH) {
        if (++finishes > 1) return fail("two finish items", cl, it.tile, 0);
        if (it.kb0 != 0 || it.kb1 == nkb) return fail("finish item is not a head segment", cl, it.tile, it.kb1);
        if (it.w0 != cl + 1 || it.w1 < it.w0) return fail("finish writer range", cl, it.w0, it.w1);
        finisher[it.tile] = cl;
        nfinish[it.tile]++;
        for (int w = it.w0; w <= it.w1; ++w) listed[it.tile].push_back(w);
      } else if (it.kb0 != 0 || it.kb1 != nkb) {
        return fail("full item does not cover the tile", cl, it.tile, it.kb0);
      }
      if (last_kind == fl::IT_FINISH) return fail("finish item is not the last item", cl, it.tile, 0);
      last_kind = it.kind;
    }
  }
  for (size_t u = 0; u < cover.size(); ++u)
    if (cover[u] != 1) return fail("unit not computed exactly once", (int)(u / nkb), (int)(u % nkb), cover[u]);
  for (int t = 0; t < T; ++t) {
    if (writers[t].empty()) {
      if (nfinish[t] != 0) return fail("finish item on an uncut tile", t, 0, 0);
      continue;
    }
    if (nfinish[t] != 1) return fail("cut tile without exactly one finisher", t, nfinish[t], 0);
    if (listed[t] != writers[t]) return fail("finisher's writer list differs from the partial items", t, 0, 0);
  }
  return 0;
}

// The kernel's tile raster (division-free) against the plain formula: group g of 8 A-side
// tiles, B-side swept inside it, and every tile exactly once.
static int check_coords(int tiles_a, int tiles_b) {
  KParams p{};
  p.tiles_a = tiles_a;
  p.tiles_b = tiles_b;
  fl::set_dp_split(p, 1);
  const int T = tiles_a * tiles_b;
  std::vector<char> seen((size_t)T, 0);
  for (int t = 0; t < T; ++t) {
    int ta, tb;
    fl::tile_coords(t, p, ta, tb);
    const int gs = 8 * tiles_b, g = t / gs, first = 8 * g, ga = std::min(8, tiles_a - first), r = t - g * gs;
    if (ta != first + r % ga || tb != r / ga) return fail("tile coordinates", tiles_a, tiles_b, t);
    if (seen[(size_t)ta * tiles_b + tb]++) return fail("tile visited twice", tiles_a, tiles_b, t);
  }
  return 0;
}

int main() {
  int cases = 0;
  for (int a = 1; a <= 40; ++a)
    for (int b = 1; b <= 40; ++b)
      if (check_coords(a, b)) return 1;
  const int big[][2] = {{2048, 3}, {7, 4099}, {600, 600}, {4096, 16}, {33, 1025}, {9, 1}};
  for (const auto& s : big)
    if (check_coords(s[0], s[1])) return 1;
  // the synthetic workloads on 74 CTA pairs (tiles_a, tiles_b, K blocks, stream-K tiles,
  // stream-K pairs, pairs launched), as fl_plan splits them
  const int known[][6] = {{16, 16, 32, 108, 74, 74},  // 4096^3: 34 left over plus one round
                          {2, 16, 32, 32, 64, 64},    // M = 512 tail: each tile in two K halves
                          {8, 16, 32, 128, 74, 74},   // M = 2048 tail
                          {32, 3, 24, 96, 74, 74},    // GeGLU down projection
                          {32, 24, 6, 102, 74, 74},   // GeGLU gate/up (stream-K forced)
                          {16, 16, 32, 34, 74, 74},   // ranges shorter than a tile
                          {4, 12, 6, 48, 74, 74}};    // ranges shorter than a tile
  for (const auto& k : known) {
    if (check(k[0], k[1], k[2], k[3], k[4], k[5])) return 1;
    ++cases;
  }
  // random shapes, with and without stream-K
  std::srand(12345);
  for (int n = 0; n < 3000; ++n) {
    const int ta = 1 + std::rand() % 20, tb = 1 + std::rand() % 20, nkb = 1 + std::rand() % 40;
    const int ncl = 1 + std::rand() % 80;
    const int T = ta * tb;
    const int sk = (std::rand() % 3 == 0) ? 0 : std::min(T, 1 + std::rand() % (2 * ncl));
    // the full rounds before the stream-K tiles are whole rounds of the ncl clusters
    const int dp = T - sk;
    if (sk > 0 && dp % ncl != 0) continue;
    const int skc = sk > 0 ? std::min(ncl, sk * nkb) : 0;
    if (check(ta, tb, nkb, sk, skc, ncl)) return 1;
    ++cases;
    // every tile split in two K halves over 2T clusters
    if (2 * T <= 160 && nkb >= 2) {
      if (check(ta, tb, nkb, T, 2 * T, 2 * T)) return 1;
      ++cases;
    }
  }
  std::printf("schedule ok: %d cases, tile raster on 1606 grids\n", cases);
  return 0;
}
