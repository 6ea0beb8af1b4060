// Host-side check of the grouped GEMMs' tile decoding (decode_tile and
// problem_id of ns_tiles.cuh, the code both GEMM kernels run) against the
// planner's tile lists, for the bench workloads' shapes and random mixes of
// shapes, worker counts and precision flags.  For every op (Gram, quintic
// square, apply) and both problem sets (M workers, one), each tile index must
// decode to a tile inside its problem's output, every output tile must come
// out exactly once (only tm <= tn for the symmetric Gram), and the problem
// id must name the right matrix.  No GPU is needed.  Built and run by
// tests/test_cpu_tile_decode.py; exit status 0 on success.
#include <cstdio>
#include <random>
#include <set>
#include <string>
#include <tuple>
#include <vector>

#include "ns_tiles.cuh"
#include "plan.h"
#include "signmuon.h"

using namespace sm;

static int check(const std::vector<int64_t>& shapes, int M, unsigned flags) {
  Plan p;
  std::string err;
  const int n_mats = (int)shapes.size() / 2;
  if (make_plan(shapes.data(), n_mats, M, 5, SIGNMUON_SCALE_SPECTRAL, 2, flags, &p, &err)) return 1;
  for (int op = 0; op < 3; ++op) {
    for (int slot = 0; slot < 2; ++slot) {
      const TileTable& tt = p.tiles[op][slot];
      const int nw = slot ? 1 : M;
      GemmArgs a{};
      a.tiles = tt.groups.data();
      a.n_tile_groups = (int)tt.groups.size();
      a.total_tiles = tt.total;
      a.groups = p.groups.data();
      a.group_mats = p.group_mats.data();
      a.n_mats = p.n_mats;
      a.param_tables = 0;
      std::set<std::tuple<int, int, int, int>> seen;
      int64_t expect = 0;
      for (const TileGroup& t : tt.groups) {
        const int per = t.sym ? t.tiles_m * (t.tiles_m + 1) / 2 : t.tiles_m * t.tiles_n;
        expect += (int64_t)per * t.batch;
        if (t.sym && (t.BM != t.BN || t.Mdim != t.Ndim)) return 10;
      }
      if (expect != tt.total) return 11;
      for (int tile = 0; tile < tt.total; ++tile) {
        const TileCoord c = decode_tile(a, tile);
        const TileGroup& t = tt.groups[c.tg];
        const GroupInfo& g = p.groups[c.group];
        if (t.group != c.group) return 2;
        if (c.b < 0 || c.b >= nw * g.count) return 3;
        if (c.m0 < 0 || c.m0 >= c.Mdim || c.n0 < 0 || c.n0 >= c.Ndim) return 4;
        if (c.m0 % t.BM != 0 || c.n0 % t.BN != 0) return 5;
        if (t.sym && c.m0 > c.n0) return 6;
        if (!seen.insert(std::make_tuple(c.group, c.b, c.m0, c.n0)).second) return 7;  // twice
        int mat = -1;
        const int pid = problem_id(a, g, c.b, &mat);
        if (mat < 0 || mat >= n_mats || p.mats[mat].group != c.group) return 8;
        if (p.mats[mat].q != c.b % g.count || pid != (c.b / g.count) * n_mats + mat) return 9;
      }
      // distinct, in range, and as many as the lists hold: every tile exactly once
      if ((int64_t)seen.size() != expect) return 12;
    }
  }
  return 0;
}

int main() {
  const unsigned flag_sets[4] = {0u, SIGNMUON_NS_FP32, SIGNMUON_NS_QUINTIC, SIGNMUON_NS_FP32 | SIGNMUON_NS_QUINTIC};
  int plans = 0;
  // nanoGPT-124M weight shapes, M = 8
  std::vector<int64_t> nano;
  const int64_t layer[8] = {2304, 768, 768, 768, 3072, 768, 768, 3072};
  for (int i = 0; i < 48; ++i) {
    nano.push_back(layer[2 * (i % 4)]);
    nano.push_back(layer[2 * (i % 4) + 1]);
  }
  for (unsigned f : flag_sets) {
    const int rc = check(nano, 8, f);
    if (rc) {
      std::printf("nanoGPT flags %u: check %d failed\n", f, rc);
      return rc;
    }
    ++plans;
  }
  // random mixes: 1-6 shapes with sides 1-700 (some repeated), M 1-9
  std::mt19937 rng(20260512u);
  for (int trial = 0; trial < 400; ++trial) {
    std::vector<int64_t> s;
    const int n = 1 + (int)(rng() % 6);
    for (int i = 0; i < n; ++i) {
      if (i > 0 && rng() % 4 == 0) {
        const int j = (int)(rng() % i);
        s.push_back(s[2 * j]);
        s.push_back(s[2 * j + 1]);
      } else {
        s.push_back(1 + (int64_t)(rng() % 700));
        s.push_back(1 + (int64_t)(rng() % 700));
      }
    }
    const int M = 1 + (int)(rng() % 9);
    const unsigned f = flag_sets[rng() % 4];
    const int rc = check(s, M, f);
    if (rc) {
      std::printf("trial %d (M=%d flags=%u): check %d failed\n", trial, M, f, rc);
      return rc;
    }
    ++plans;
  }
  std::printf("tile decode ok: %d plans\n", plans);
  return 0;
}
