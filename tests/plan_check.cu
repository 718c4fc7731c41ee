// Host-side check of the tensor-core GEMM's work schedule (lmhead.cuh: Plan, unit_of,
// for_each_tile), compiled by nvcc as a plain host program and run on the CPU.
//
// For each case (masked row count, V, work holders, CTA group) it verifies that
//   - the tiles of all holders cover every (m-tile, vocabulary tile) exactly once;
//   - each holder writes its partials to slots no other holder writes, inside
//     part_entries(); the number of writers of an m-tile equals the unit count the
//     epilogue's merge waits for;
//   - without remainder holders, the streams of a group differ by at most one tile; with
//     them, no holder runs more tiles than the busiest stream would without them;
//   - in every full group of a problem with several groups, the holders of one stream run
//     the same number of tiles (what the pair body's pacing compares);
//   - a problem of one m-tile uses the fewest streams that keep the busiest stream's tile
//     count (the other holders stay idle);
//   - part_entries() fits the partial region the workspace reserves: groups x holders x
//     rows per m-tile, or (holders + gmax^2) x rows per m-tile when the problem fits one
//     group (remainder holders), for any masked count up to the capacity.
// Prints "ok <cases>" and exits 0, or prints the first failing case and exits 1.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <random>
#include <set>
#include <utility>
#include <vector>

#include "lmhead.cuh"

using namespace dllm::lm;

namespace {

bool fail(const char* what, int count, int V, int ctas, int cg) {
  std::printf("FAIL %s: count=%d V=%d holders=%d cg=%d\n", what, count, V, ctas, cg);
  return false;
}

bool check_case(int count, int V, int ctas, int cg) {
  const int bm = 128 * cg, gmax = cg == 2 ? DLLM_GROUP_M2 : DLLM_GROUP_M1;
  const Plan pl = Plan::make(count, V, ctas, gmax, bm);
  std::vector<std::vector<int>> tiles(pl.numM);
  std::vector<int> per_holder(ctas, 0);
  std::vector<int> writers(pl.numM, 0);
  std::set<long long> slots_used;
  const long long entries = pl.part_entries();
  const long long reserve = std::max(static_cast<long long>(pl.ngroups) * ctas * bm,
                                     pl.ngroups == 1 ? (static_cast<long long>(ctas) + gmax * gmax) * bm
                                                     : 0LL);
  if (entries > reserve) return fail("partials exceed the workspace reserve", count, V, ctas, cg);
  for (int h = 0; h < ctas; ++h) {
    bool bad_tile = false;
    auto rec = [&](int m, int n) -> bool {
      if (m < 0 || m >= pl.numM || n < 0 || n >= pl.numN) {
        bad_tile = true;
        return false;
      }
      tiles[m].push_back(n);
      ++per_holder[h];
      return true;
    };
    if (!for_each_tile(pl, h, rec) || bad_tile) return fail("tile shape", count, V, ctas, cg);
    for (int g = 0; g < pl.ngroups; ++g) {
      Unit u;
      if (!unit_of(pl, g, h, u)) continue;
      std::vector<int> ms;
      if (u.leftover) {
        for (long long i = u.i0; i < u.i1; ++i) {
          const int m_local = static_cast<int>(i / pl.rr);
          if (ms.empty() || ms.back() != m_local) ms.push_back(m_local);
        }
      } else {
        ms.push_back(u.m_local);
      }
      for (int m_local : ms) {
        ++writers[g * pl.gmax + m_local];
        for (int r = 0; r < bm; r += 37) {
          const long long e = pl.part_index(g, u.G, u.p, m_local * bm + r);
          if (e < 0 || e >= entries) return fail("partial slot out of range", count, V, ctas, cg);
          if (!slots_used.insert(e).second) return fail("partial slot shared", count, V, ctas, cg);
        }
      }
    }
  }
  for (int m = 0; m < pl.numM; ++m) {
    auto& t = tiles[m];
    std::sort(t.begin(), t.end());
    if (static_cast<int>(t.size()) != pl.numN) return fail("coverage", count, V, ctas, cg);
    for (int i = 0; i < pl.numN; ++i)
      if (t[i] != i) return fail("coverage gap or overlap", count, V, ctas, cg);
    // the merge waits for P stream units plus the remainder holders of this m-tile
    const int g = m / pl.gmax, G = pl.group_size(g);
    int j_lo = 0, j_hi = -1;
    if (pl.rem) pl.leftovers_of(m - g * pl.gmax, G, j_lo, j_hi);
    const int units = Plan::streams(G, ctas, pl.numN) + (j_hi >= j_lo ? j_hi - j_lo + 1 : 0);
    if (writers[m] != units) return fail("writer count", count, V, ctas, cg);
  }
  // one m-tile: the fewest streams that keep the busiest stream's tile count of an even
  // split over min(holders, tiles) streams
  if (pl.numM == 1 && pl.ngroups == 1) {
    const int P = Plan::streams(1, ctas, pl.numN);
    const int P0 = std::max(1, std::min(ctas, pl.numN));
    const int busiest = (pl.numN + P0 - 1) / P0;
    if ((pl.numN + P - 1) / P != busiest) return fail("fewest streams: busiest count", count, V, ctas, cg);
    if (P > 1 && (pl.numN + P - 2) / (P - 1) == busiest)
      return fail("fewest streams: not the fewest", count, V, ctas, cg);
  }
  // pacing compares the tiles started by the holders of one stream: in every full group all
  // holders of a stream run the same number of tiles, and the same in every full group
  if (!pl.rem && pl.ngroups > 1) {
    std::vector<int> per_stream_tiles;
    for (int g = 0; g < pl.ngroups; ++g) {
      if (pl.group_size(g) != pl.gmax) continue;
      for (int h = 0; h < ctas; ++h) {
        Unit u;
        if (!unit_of(pl, g, h, u) || u.leftover) continue;
        if (u.G != pl.gmax || u.p != h / pl.gmax) return fail("stream of a full group", count, V, ctas, cg);
        const int t = u.n1 - u.n0;
        if (static_cast<int>(per_stream_tiles.size()) <= u.p) per_stream_tiles.resize(u.p + 1, -1);
        if (per_stream_tiles[u.p] < 0) per_stream_tiles[u.p] = t;
        if (per_stream_tiles[u.p] != t) return fail("pacing: unequal tiles in a stream", count, V, ctas, cg);
      }
    }
  }
  if (!pl.rem) {
    for (int g = 0; g < pl.ngroups; ++g) {
      int lo = 1 << 30, hi = 0;
      for (int h = 0; h < ctas; ++h) {
        Unit u;
        if (!unit_of(pl, g, h, u) || u.leftover) continue;
        lo = std::min(lo, u.n1 - u.n0);
        hi = std::max(hi, u.n1 - u.n0);
      }
      if (hi - lo > 1) return fail("stream balance", count, V, ctas, cg);
    }
  } else {
    const int G = pl.numM, P = Plan::streams(G, ctas, pl.numN);
    const int even = (pl.numN + P - 1) / P;
    for (int h = 0; h < ctas; ++h)
      if (per_holder[h] >= even) return fail("remainder holders do not help", count, V, ctas, cg);
  }
  return true;
}

}  // namespace

int main(int argc, char** argv) {
  const int n_random = argc > 1 ? std::atoi(argv[1]) : 2000;
  int cases = 0;
  // the named workloads (masked rows, V) on B200's 148 SMs / 74 pairs
  const int named[][2] = {{128, 4096}, {1024, 126464}, {64, 126464}, {29491, 126464},
                          {13107, 126464}, {65536, 126464}, {117965, 126464}, {32768, 151936},
                          {256, 151936}};
  for (auto& w : named)
    for (int cg = 1; cg <= 2; ++cg) {
      if (!check_case(w[0], w[1], cg == 1 ? 148 : 74, cg)) return 1;
      ++cases;
    }
  std::mt19937 rng(12345);
  const int holder_choices[] = {1, 2, 3, 7, 37, 74, 80, 132, 148, 160};
  for (int i = 0; i < n_random; ++i) {
    const int cg = 1 + static_cast<int>(rng() % 2);
    int ctas = holder_choices[rng() % 10];
    if (cg == 2) ctas = std::max(1, ctas / 2);
    const int V = 1 + static_cast<int>(rng() % (i % 10 == 0 ? 160000 : 20000));
    const int count = static_cast<int>(rng() % (i % 7 == 0 ? 60000 : 3000));
    if (!check_case(count, V, ctas, cg)) return 1;
    ++cases;
  }
  std::printf("ok %d\n", cases);
  return 0;
}
