// plan.cpp -- host planning for a Sign-Muon handle (see plan.h).
#include "plan.h"

#include <algorithm>
#include <climits>
#include <map>
#include <queue>
#include <utility>

#include "../../include/signmuon.h"

namespace sm {

namespace {

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Output tile width for the 2-SM tensor-core kernel (256 rows per CTA pair):
// N=256 moves the fewest operand bytes per flop, N=128 wastes less on ragged
// edges.
int pick_bn(int n) {
  const int cand[2] = {256, 128};
  const double speed[2] = {1.0, 0.85};
  int best = 128;
  double best_eff = -1.0;
  for (int i = 0; i < 2; ++i) {
    if (cand[i] > SM_TC_BN_MAX) continue;
    const int64_t tiles = (n + cand[i] - 1) / cand[i];
    const double eff = (double)n / (double)(tiles * cand[i]) * speed[i];
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = cand[i];
    }
  }
  return best;
}

// force_sym: square 256 x 256 tiles for GRAM and SQUARE (the Gram-space
// iteration needs their outputs exactly symmetric, which the upper-triangle
// tiles and their mirror give)
void build_tiles(Plan& p, int op, int nw, TileTable* tt, bool force_sym = false) {
  std::vector<TileGroup> v;
  for (int gidx = 0; gidx < (int)p.groups.size(); ++gidx) {
    const GroupInfo& g = p.groups[gidx];
    TileGroup t{};
    t.group = gidx;
    if (op == OP_GRAM) {
      t.Mdim = t.Ndim = g.g;
      t.Kdim = g.wide ? g.cols : g.rows;
    } else if (op == OP_SQUARE) {
      t.Mdim = t.Ndim = t.Kdim = g.g;
    } else {
      t.Mdim = g.rows;
      t.Ndim = g.cols;
      t.Kdim = g.g;
    }
    t.BM = p.fp32 ? 128 : 256;
    t.BN = p.fp32 ? 128 : ((force_sym && op != OP_APPLY) ? 256 : pick_bn(t.Ndim));
    t.tiles_m = (t.Mdim + t.BM - 1) / t.BM;
    t.tiles_n = (t.Ndim + t.BN - 1) / t.BN;
    // the Gram X X^T, and the square's products of commuting symmetric m x m
    // matrices, are symmetric: with square tiles only the upper ones run
    t.sym = ((op == OP_GRAM || op == OP_SQUARE) && !p.fp32 && t.BM == t.BN) ? 1 : 0;
    t.batch = nw * g.count;
    v.push_back(t);
  }
  // longest tiles first: a better static round-robin balance
  std::stable_sort(v.begin(), v.end(), [](const TileGroup& x, const TileGroup& y) { return x.Kdim > y.Kdim; });
  int start = 0;
  for (auto& t : v) {
    t.tile_start = start;
    const int per = t.sym ? t.tiles_m * (t.tiles_m + 1) / 2 : t.tiles_m * t.tiles_n;
    start += per * t.batch;
  }
  tt->groups = v;
  tt->total = start;
}

// flops of every tile of a launch as it runs (2 BM BN K per tile)
double tile_flops(const TileTable& tt) {
  double f = 0.0;
  for (const TileGroup& t : tt.groups) {
    const int per = t.sym ? t.tiles_m * (t.tiles_m + 1) / 2 : t.tiles_m * t.tiles_n;
    f += 2.0 * t.BM * t.BN * t.Kdim * (double)per * t.batch;
  }
  return f;
}

}  // namespace

std::vector<int> tile_schedule(const TileTable& tt, int ncl, double* rr, double* greedy) {
  std::vector<int> out;
  if (rr) *rr = 0.0;
  if (greedy) *greedy = 0.0;
  if (tt.total <= 0 || ncl <= 0) return out;
  std::vector<double> cost((size_t)tt.total);
  for (const TileGroup& t : tt.groups) {
    const int per = t.sym ? t.tiles_m * (t.tiles_m + 1) / 2 : t.tiles_m * t.tiles_n;
    const double c = (double)((t.Kdim + 63) / 64) + 3.0;
    for (int i = 0; i < per * t.batch; ++i) cost[(size_t)t.tile_start + i] = c;
  }
  std::vector<double> load_rr((size_t)ncl, 0.0), load_g((size_t)ncl, 0.0);
  std::vector<std::vector<int>> lists((size_t)ncl);
  // (load, cluster): the least-loaded cluster first, ties to the lower index
  std::priority_queue<std::pair<double, int>, std::vector<std::pair<double, int>>, std::greater<>> q;
  for (int c = 0; c < ncl; ++c) q.push({0.0, c});
  for (int t = 0; t < tt.total; ++t) {
    load_rr[(size_t)(t % ncl)] += cost[(size_t)t];
    const auto [l, c] = q.top();
    q.pop();
    lists[(size_t)c].push_back(t);
    load_g[(size_t)c] = l + cost[(size_t)t];
    q.push({load_g[(size_t)c], c});
  }
  const double m_rr = *std::max_element(load_rr.begin(), load_rr.end());
  const double m_g = *std::max_element(load_g.begin(), load_g.end());
  if (rr) *rr = m_rr;
  if (greedy) *greedy = m_g;
  if (!(m_g < 0.97 * m_rr)) return out;
  out.reserve((size_t)(ncl + 1 + tt.total));
  int start = 0;
  for (int c = 0; c < ncl; ++c) {
    out.push_back(start);
    start += (int)lists[(size_t)c].size();
  }
  out.push_back(start);
  for (int c = 0; c < ncl; ++c) out.insert(out.end(), lists[(size_t)c].begin(), lists[(size_t)c].end());
  return out;
}

int make_plan(const int64_t* shapes, int n_mats, int M, int K, int scale, int P, unsigned flags,
              Plan* plan, std::string* err) {
  if (shapes == nullptr || n_mats < 1) { *err = "need at least one matrix shape"; return SIGNMUON_E_INVALID; }
  if (M < 1 || M > kMaxWorkers) { *err = "M must be in [1, 256]"; return SIGNMUON_E_INVALID; }
  if ((flags & SIGNMUON_ACC_INT8) && M > 127) { *err = "int8 vote sums overflow for M > 127"; return SIGNMUON_E_OVERFLOW; }
  if (K < 0) { *err = "K must be >= 0"; return SIGNMUON_E_INVALID; }
  if (scale != SIGNMUON_SCALE_FRO && scale != SIGNMUON_SCALE_SPECTRAL) { *err = "unknown scale"; return SIGNMUON_E_INVALID; }
  if (scale == SIGNMUON_SCALE_SPECTRAL && P < 1) { *err = "spectral scaling needs P >= 1"; return SIGNMUON_E_INVALID; }
  if ((flags & SIGNMUON_POLAR_AFTER_ONLY) && !(flags & SIGNMUON_POST_POLAR)) {
    *err = "SIGNMUON_POLAR_AFTER_ONLY requires SIGNMUON_POST_POLAR";
    return SIGNMUON_E_INVALID;
  }
  if ((flags & SIGNMUON_MUON_MEAN) &&
      (flags & (SIGNMUON_POST_POLAR | SIGNMUON_POLAR_AFTER_ONLY | SIGNMUON_TERNARY | SIGNMUON_NORMALIZED_SIGN))) {
    *err = "SIGNMUON_MUON_MEAN sends no signs: it cannot be combined with the post-vote step or the sign wire flags";
    return SIGNMUON_E_INVALID;
  }
  if ((flags & SIGNMUON_NORMALIZED_SIGN) && (flags & SIGNMUON_POST_POLAR)) {
    *err = "SIGNMUON_NORMALIZED_SIGN replaces the post-vote polar step: drop SIGNMUON_POST_POLAR";
    return SIGNMUON_E_INVALID;
  }
  Plan& p = *plan;
  p = Plan();
  p.M = M;
  p.n_mats = n_mats;
  p.fp32 = (flags & SIGNMUON_NS_FP32) != 0;
  p.quintic = (flags & SIGNMUON_NS_QUINTIC) != 0;
  std::map<std::pair<int64_t, int64_t>, int> gid;
  int64_t off = 0;
  for (int i = 0; i < n_mats; ++i) {
    const int64_t r = shapes[2 * i], c = shapes[2 * i + 1];
    if (r < 1 || c < 1) { *err = "matrix " + std::to_string(i) + " has a non-positive dimension"; return SIGNMUON_E_INVALID; }
    if (r * c > (int64_t)INT_MAX) { *err = "matrix " + std::to_string(i) + " has more than 2^31-1 entries"; return SIGNMUON_E_INVALID; }
    auto key = std::make_pair(r, c);
    auto it = gid.find(key);
    int g;
    if (it == gid.end()) {
      g = (int)p.groups.size();
      gid[key] = g;
      GroupInfo gi{};
      gi.rows = (int)r;
      gi.cols = (int)c;
      gi.ld = (int)round_up(c, 8);
      gi.wide = r <= c ? 1 : 0;
      gi.g = (int)std::min(r, c);
      gi.gld = (int)round_up(gi.g, 8);
      gi.count = 0;
      p.groups.push_back(gi);
    } else {
      g = it->second;
    }
    MatInfo mi{};
    mi.off = off;
    mi.rows = (int)r;
    mi.cols = (int)c;
    mi.group = g;
    mi.q = p.groups[g].count++;
    p.mats.push_back(mi);
    p.mat_off.push_back(off);
    off += r * c;
  }
  p.d = off;
  p.dpad = round_up(p.d, 64);
  p.nb = (p.d + 7) / 8;
  p.nb_pad = round_up(p.nb, 16);
  // group -> matrices, group bases (every base a multiple of 8 elements)
  int first = 0;
  for (auto& g : p.groups) {
    g.first = first;
    first += g.count;
  }
  p.group_mats.assign(n_mats, 0);
  for (int i = 0; i < n_mats; ++i) {
    const MatInfo& mi = p.mats[i];
    p.group_mats[p.groups[mi.group].first + mi.q] = i;
  }
  int64_t xb = 0, ab = 0;
  for (auto& g : p.groups) {
    g.x_base = xb;
    g.a_base = ab;
    xb += (int64_t)M * g.count * g.rows * g.ld;
    ab += (int64_t)M * g.count * g.g * g.gld;
  }
  p.x_elems = xb;
  p.a_elems = ab;
  // elementwise chunks: pieces of <= kChunk elements, never crossing a matrix
  p.mat_chunk0.resize(n_mats);
  p.mat_nchunks.resize(n_mats);
  for (int i = 0; i < n_mats; ++i) {
    const int64_t n = (int64_t)p.mats[i].rows * p.mats[i].cols;
    p.mat_chunk0[i] = (int)p.chunks.size();
    for (int64_t s = 0; s < n; s += kChunk) {
      Chunk c{};
      c.mat = i;
      c.start = s;
      c.len = (int)std::min<int64_t>(kChunk, n - s);
      p.chunks.push_back(c);
      // flat offset of the chunk, and its offset in a one-problem-set X
      // when the matrix's rows are unpadded there
      const GroupInfo& g = p.groups[p.mats[i].group];
      p.stage_off.push_back(p.mats[i].off + s);
      p.stage_off.push_back(g.x_base + (int64_t)p.mats[i].q * g.rows * g.ld + s);
    }
    p.mat_nchunks[i] = (int)p.chunks.size() - p.mat_chunk0[i];
  }
  for (int op = 0; op < 3; ++op) {
    build_tiles(p, op, M, &p.tiles[op][0]);
    build_tiles(p, op, 1, &p.tiles[op][1]);
  }
  // X space: K x (Gram + apply).  Gram space: one Gram, 3K - 3 m x m products
  // (T_k = a A_k + b A_k^2, A_{k+1} = a T_k + b A_k T_k, Q_{k+1} = a Q_k + b A_k Q_k)
  // and one apply.  Tile flops, counted as the tiles run; with SIGNMUON_NS_GRAM
  // the Gram-space form is taken when it saves more than 15 % (its extra
  // launches and its elementwise start cost a little) and every Gram side is
  // at least 256:
  // small Grams gain little time, and rounding their squared spectrum to
  // bf16 flips twice as many of the smallest entries' signs.
  bool big = true;
  for (const GroupInfo& g : p.groups) big = big && g.g >= 256;
  if ((flags & SIGNMUON_NS_GRAM) && !p.fp32 && !p.quintic && K >= 2 && big) {
    // both forms counted with the Gram on square tiles, as Gram space runs it
    TileTable gram[2], square[2];
    for (int s = 0; s < 2; ++s) {
      build_tiles(p, OP_GRAM, s == 0 ? M : 1, &gram[s], true);
      build_tiles(p, OP_SQUARE, s == 0 ? M : 1, &square[s], true);
    }
    const double xs = K * (tile_flops(gram[0]) + tile_flops(p.tiles[OP_APPLY][0]));
    const double gs = tile_flops(gram[0]) + (3.0 * K - 3.0) * tile_flops(square[0]) + tile_flops(p.tiles[OP_APPLY][0]);
    p.gram_ns = gs < 0.85 * xs;
    if (p.gram_ns) {
      for (int s = 0; s < 2; ++s) {
        p.tiles[OP_GRAM][s] = gram[s];
        p.tiles[OP_SQUARE][s] = square[s];
      }
    }
  }
  // power iteration tables (worker-major problems so worker 0 is a prefix)
  int64_t u = 0, part = 0;
  for (int w = 0; w < M; ++w) {
    for (int i = 0; i < n_mats; ++i) {
      const MatInfo& mi = p.mats[i];
      const GroupInfo& g = p.groups[mi.group];
      const int pid = w * n_mats + i;
      const int nt = (int)((g.g + kPiTile - 1) / kPiTile);
      p.uoff.push_back(u);
      p.poff.push_back(part);
      p.prob_g.push_back(g.g);
      p.prob_gld.push_back(g.gld);
      p.prob_aoff.push_back(g.a_base + (int64_t)(w * g.count + mi.q) * g.g * g.gld);
      const int soff = (int)p.pi_slices.size();
      p.soff.push_back(soff);
      for (int bi = 0; bi < nt; ++bi) {
        p.pi_slices.push_back(PiSlice{u, part, pid, g.g, bi, soff});
        for (int bj = bi; bj < nt; ++bj)
          p.pi_tiles.push_back(PiTile{p.prob_aoff.back(), u, part, pid, g.g, g.gld, bi, bj, 0});
      }
      u += g.g;
      part += (int64_t)nt * nt * kPiTile;
    }
    if (w == 0) {
      p.n_pi_tiles_one = (int)p.pi_tiles.size();
      p.n_pi_slices_one = (int)p.pi_slices.size();
      p.u_elems_one = u;
    }
  }
  p.part_elems = part;
  p.u_elems = u;
  const int64_t esz = p.fp32 ? 4 : 2;
  int64_t bytes = 0;
  if (!(flags & SIGNMUON_VOTE_ONLY)) {
    bytes += 2 * (int64_t)M * p.dpad * 4;                 // momentum, U
    bytes += 2 * p.x_elems * esz;                         // X ping/pong
    bytes += p.a_elems * esz * (p.quintic ? 2 : 1);       // A (and B)
    if (p.gram_ns) bytes += p.a_elems * esz * 4;          // B, A2, Q0, Q1 of the Gram-space iteration
    bytes += (int64_t)M * p.nb_pad;                       // packed bits
    if (flags & SIGNMUON_TERNARY) bytes += (int64_t)M * p.dpad;  // int8 ternary signs
    bytes += p.dpad * 4;                                  // D
    bytes += (int64_t)p.chunks.size() * M * 4;            // norm partials
    bytes += (int64_t)M * n_mats * (4 + 8 + 8);           // scales, coefficients
    bytes += 2 * p.u_elems * 4;                           // power-iteration vectors
    bytes += p.part_elems * 4;                            // power-iteration partial sums
    bytes += (int64_t)p.pi_slices.size() * 8;             // per-slice figures
    bytes += (int64_t)M * n_mats * 8;                     // per-problem counters, 1/||y||
    if (flags & SIGNMUON_PI_WARM) bytes += p.u_elems_one * 4;  // warm state of one problem set
    bytes += (int64_t)p.groups.size() * kMapsPerGroup * 128;  // tensor maps
  }
  p.device_bytes = bytes;
  (void)K;
  return SIGNMUON_OK;
}

}  // namespace sm
