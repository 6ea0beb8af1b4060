// ns_tiles.cuh -- tile decoding and operand roles of the grouped
// Newton-Schulz GEMMs (shared by the tcgen05 and the fp32 SIMT kernels).
//
// One NS iteration on a matrix X (rows x cols, natural row-major layout) is
// ([paper] "SignMuon: 通信高效的分布式Muon优化" §3 two-coefficient form, §4 cubic):
//   wide (rows <= cols):  A = X X^T          X' = a X + b A X
//   tall (rows >  cols):  A = X^T X          X' = a X + b X A
// and for the quintic form a third GEMM B = b A + c A A, X' = a X + B X
// (or X B).  Operand roles in C[i][j] = sum_k Aop(i,k) Bop(k,j):
//   GRAM   wide: Aop = X   (K-major), Bop(k,j) = X[j][k] (K-major),  K = cols
//          tall: Aop = X^T (MN-major), Bop = X           (MN-major), K = rows
//   SQUARE      Aop = A (K-major), Bop(k,j) = A[j][k] (A symmetric), K = g
//   APPLY  wide: Aop = P (K-major), Bop = X (MN-major), M = rows, N = cols, K = g
//          tall: Aop = X (K-major), Bop(k,j) = P[j][k] (K-major), M = rows, N = cols
// where P is A (cubic) or B (quintic).  "K-major" means consecutive k are
// adjacent in memory; "MN-major" means consecutive i (or j) are.
//
// The functions below are host-callable too, so that a CPU program can check
// the decoding against the planner's tile lists.
#pragma once
#include "common.cuh"

namespace sm {

struct TileCoord {
  int tg;        // index into the launch's TileGroup list
  int group;
  int b;         // problem within the group (worker*count + q)
  int m0, n0;    // tile origin in the output
  int Mdim, Ndim, Kdim, BN;
  int sym;       // only tiles on or above the diagonal run (symmetric output)
};

__host__ __device__ __forceinline__ const TileGroup* tile_table(const GemmArgs& a) {
  return a.param_tables ? a.ptiles : a.tiles;
}
__host__ __device__ __forceinline__ const GroupInfo& group_info(const GemmArgs& a, int g) {
  return a.param_tables ? a.pgroups[g] : a.groups[g];
}

__host__ __device__ __forceinline__ TileCoord decode_tile(const GemmArgs& a, int tile) {
  const TileGroup* tiles = tile_table(a);
  int t = 0;
  while (t + 1 < a.n_tile_groups && tiles[t + 1].tile_start <= tile) ++t;
  const TileGroup tg = tiles[t];
  const int local = tile - tg.tile_start;
  const int per = tg.sym ? tg.tiles_m * (tg.tiles_m + 1) / 2 : tg.tiles_m * tg.tiles_n;
  TileCoord c;
  c.tg = t;
  c.group = tg.group;
  c.b = local / per;
  int rem = local - c.b * per;
  int tm, tn;
  if (tg.sym) {  // row tm holds the tiles tn = tm .. tiles_m-1
    tm = 0;
    while (rem >= tg.tiles_m - tm) {
      rem -= tg.tiles_m - tm;
      ++tm;
    }
    tn = tm + rem;
  } else {
    tm = rem / tg.tiles_n;
    tn = rem - tm * tg.tiles_n;
  }
  c.m0 = tm * tg.BM;
  c.n0 = tn * tg.BN;
  c.Mdim = tg.Mdim;
  c.Ndim = tg.Ndim;
  c.Kdim = tg.Kdim;
  c.BN = tg.BN;
  c.sym = tg.sym;
  return c;
}

// problem id p = worker*n_mats + matrix, used for the per-problem coefficients
__host__ __device__ __forceinline__ int problem_id(const GemmArgs& a, const GroupInfo& gi, int b, int* mat_out) {
  const int w = b / gi.count;
  const int q = b - w * gi.count;
  const int mat = a.param_tables ? a.pgroup_mats[gi.first + q] : a.group_mats[gi.first + q];
  *mat_out = mat;
  return w * a.n_mats + mat;
}

// operand majorness (1 = MN-major) for an op/orientation
__host__ __device__ __forceinline__ int a_is_mn(int op, int wide) { return (op == OP_GRAM && !wide) ? 1 : 0; }
__host__ __device__ __forceinline__ int b_is_mn(int op, int wide) {
  return ((op == OP_GRAM && !wide) || (op == OP_APPLY && wide)) ? 1 : 0;
}

}  // namespace sm
