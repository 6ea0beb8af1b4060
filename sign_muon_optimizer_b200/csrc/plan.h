// plan.h -- host-side planning of one Sign-Muon handle: shape groups, chunk
// lists, grouped GEMM tile lists, power-iteration tiles and buffer
// sizes.  Pure host code (no CUDA calls), so that it can be checked without a
// GPU through signmuon_plan().
#pragma once
#include <cstdint>
#include <string>
#include <vector>

#include "common.cuh"

namespace sm {

struct TileTable {
  std::vector<TileGroup> groups;
  int total = 0;
};

struct Plan {
  int M = 0, n_mats = 0;
  bool fp32 = false, quintic = false;
  // bf16 cubic Newton-Schulz in Gram space (m x m products, one final X
  // product) rather than on X: with SIGNMUON_NS_GRAM, when it needs fewer
  // tile flops
  bool gram_ns = false;
  int64_t d = 0;        // parameters
  int64_t dpad = 0;     // stride of the library's flat per-worker vectors
  int64_t nb = 0;       // ceil(d/8) packed bytes per worker
  int64_t nb_pad = 0;   // stride of the library's packed buffers (16-byte multiple)
  std::vector<MatInfo> mats;
  std::vector<GroupInfo> groups;
  std::vector<int> group_mats;
  std::vector<int64_t> mat_off;
  std::vector<Chunk> chunks;
  std::vector<int> mat_chunk0, mat_nchunks;
  std::vector<int64_t> stage_off;  // per chunk: flat offset, offset in a one-problem-set X
  int64_t x_elems = 0;  // elements of one grouped X buffer (all workers)
  int64_t a_elems = 0;  // elements of the grouped A (and B) buffer
  // tile lists: [op][0 = all M workers, 1 = one worker]
  TileTable tiles[3][2];
  // power iteration: problems p = worker*n_mats + mat (worker-major)
  std::vector<PiTile> pi_tiles;    // the 128 x 128 tiles on and above each Gram's diagonal
  std::vector<PiSlice> pi_slices;  // 128-row slices of every problem
  int n_pi_tiles_one = 0;          // tiles of worker 0's problems (prefix)
  int n_pi_slices_one = 0;         // slices of worker 0's problems (prefix)
  std::vector<int> soff;           // first slice of each problem
  std::vector<int64_t> uoff;
  std::vector<int64_t> poff;       // partial-sum offsets (nt^2 * 128 entries per problem)
  int64_t part_elems = 0;
  std::vector<int> prob_g, prob_gld;
  std::vector<int64_t> prob_aoff;
  int64_t u_elems = 0;
  int64_t u_elems_one = 0;  // power-iteration vector entries of worker 0 (one problem set)
  int64_t device_bytes = 0;  // everything the handle allocates
};

// Validates and plans; returns a SIGNMUON_* status and fills *err on failure.
int make_plan(const int64_t* shapes, int n_mats, int M, int K, int scale, int P, unsigned flags,
              Plan* plan, std::string* err);

// Tile schedule of one tensor-core GEMM launch over ncl clusters.  The
// kernel's default is round robin (cluster c takes tiles c, c + ncl, ...).
// With tiles of very different depth (the launch's list runs deepest first)
// a greedy list schedule -- each tile, in list order, to the cluster with
// the least work so far, a tile costing ceil(K / 64) + 3 k-blocks -- ends
// sooner.  Returns the table [start of cluster 0 .. ncl (ncl + 1 entries),
// then the clusters' tiles one after another], or an empty vector when the
// greedy schedule's longest cluster is not at least 3 % shorter than round
// robin's.  *rr and *greedy (if non-null) get the two makespans in k-blocks.
std::vector<int> tile_schedule(const TileTable& tt, int ncl, double* rr, double* greedy);

}  // namespace sm
