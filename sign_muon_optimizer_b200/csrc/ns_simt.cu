// ns_simt.cu -- fp32 grouped Newton-Schulz GEMM on the CUDA cores (FFMA).
//
// The fp32 path of PolarNS ([paper] "SignMuon: 通信高效的分布式Muon优化" §4):
// the same three GEMM roles and epilogues as the tcgen05 kernel, computed in
// full fp32 so that the polar factor meets a 1e-4 tolerance.  A 128x128
// output tile per 256-thread block, 8x8 outputs per thread, k-slabs of 16
// staged in shared memory (double-buffered through registers).
#include "ns_tiles.cuh"

namespace sm {
namespace {

constexpr int TM = 128, TN = 128, TK = 16, NT = 256;

struct Operand {
  const float* p;
  int ld;
  int mn;     // 1: element (i,k) at p[k*ld + i]; 0: at p[i*ld + k]
  int ext;    // extent of the i (row of Aop / column of Bop) dimension
};

// Load a TK x 128 slab of an operand into registers (8 values per thread),
// zero outside [0, ext) x [0, K).
__device__ __forceinline__ void load_slab(const Operand& o, int i0, int k0, int K, float (&r)[8]) {
  const int t = threadIdx.x;
  if (o.mn) {
    const int k = t >> 4;             // 0..15
    const int i = (t & 15) * 8;       // 0..120
    const int gk = k0 + k;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gi = i0 + i + 4 * h;
      if (gk < K && gi + 3 < o.ext) {
        const float4 v = *reinterpret_cast<const float4*>(o.p + (int64_t)gk * o.ld + gi);
        r[4 * h] = v.x; r[4 * h + 1] = v.y; r[4 * h + 2] = v.z; r[4 * h + 3] = v.w;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          r[4 * h + u] = (gk < K && gi + u < o.ext) ? o.p[(int64_t)gk * o.ld + gi + u] : 0.f;
      }
    }
  } else {
    const int i = t >> 1;             // 0..127
    const int k = (t & 1) * 8;        // 0 or 8
    const int gi = i0 + i;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gk = k0 + k + 4 * h;
      if (gi < o.ext && gk + 3 < K) {
        const float4 v = *reinterpret_cast<const float4*>(o.p + (int64_t)gi * o.ld + gk);
        r[4 * h] = v.x; r[4 * h + 1] = v.y; r[4 * h + 2] = v.z; r[4 * h + 3] = v.w;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          r[4 * h + u] = (gi < o.ext && gk + u < K) ? o.p[(int64_t)gi * o.ld + gk + u] : 0.f;
      }
    }
  }
}

// Store the registers of load_slab into s[k][i] (k-major rows of 128).
__device__ __forceinline__ void store_slab(const Operand& o, float (*s)[TM + 4], const float (&r)[8]) {
  const int t = threadIdx.x;
  if (o.mn) {
    const int k = t >> 4, i = (t & 15) * 8;
#pragma unroll
    for (int u = 0; u < 8; ++u) s[k][i + u] = r[u];
  } else {
    const int i = t >> 1, k = (t & 1) * 8;
#pragma unroll
    for (int u = 0; u < 8; ++u) s[k + u][i] = r[u];
  }
}

__global__ void __launch_bounds__(NT)
k_gemm_simt(const __grid_constant__ GemmArgs a) {
  griddep_wait();
  griddep_launch();
  __shared__ __align__(16) float As[2][TK][TM + 4];
  __shared__ __align__(16) float Bs[2][TK][TN + 4];

  const TileCoord tc = decode_tile(a, blockIdx.x);
  const GroupInfo gi = group_info(a, tc.group);
  int mat = 0;
  const int p = problem_id(a, gi, tc.b, &mat);
  const int op = a.op;
  const int64_t xoff = gi.x_base + (int64_t)tc.b * gi.rows * gi.ld;
  const int64_t aoff = gi.a_base + (int64_t)tc.b * gi.g * gi.gld;
  const float* X = reinterpret_cast<const float*>(a.X_src) + xoff;
  const float* Am = reinterpret_cast<const float*>(a.A) + aoff;
  const float* Pm = (a.p_from_b ? reinterpret_cast<const float*>(a.B) : reinterpret_cast<const float*>(a.A)) + aoff;

  Operand oa, ob;
  if (op == OP_GRAM) {
    oa = Operand{X, gi.ld, gi.wide ? 0 : 1, tc.Mdim};
    ob = Operand{X, gi.ld, gi.wide ? 0 : 1, tc.Ndim};
  } else if (op == OP_SQUARE) {
    oa = Operand{Am, gi.gld, 0, tc.Mdim};
    ob = Operand{Am, gi.gld, 0, tc.Ndim};
  } else if (gi.wide) {
    oa = Operand{Pm, gi.gld, 0, tc.Mdim};
    ob = Operand{X, gi.ld, 1, tc.Ndim};
  } else {
    oa = Operand{X, gi.ld, 0, tc.Mdim};
    ob = Operand{Pm, gi.gld, 0, tc.Ndim};
  }

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int K = tc.Kdim;
  const int nk = (K + TK - 1) / TK;
  float ra[8], rb[8];
  load_slab(oa, tc.m0, 0, K, ra);
  load_slab(ob, tc.n0, 0, K, rb);
  store_slab(oa, As[0], ra);
  store_slab(ob, Bs[0], rb);
  __syncthreads();
  for (int kb = 0; kb < nk; ++kb) {
    const int cur = kb & 1;
    if (kb + 1 < nk) {
      load_slab(oa, tc.m0, (kb + 1) * TK, K, ra);
      load_slab(ob, tc.n0, (kb + 1) * TK, K, rb);
    }
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][k][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][k][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (kb + 1 < nk) {
      store_slab(oa, As[cur ^ 1], ra);
      store_slab(ob, Bs[cur ^ 1], rb);
    }
    __syncthreads();
  }

  // ---- epilogue ----
  float c0 = a.c0, c1 = a.c1;
  if (a.coef != nullptr) {
    const float2 cf = a.coef[p];
    c0 = cf.x;
    c1 = cf.y;
  }
  const int w = tc.b / gi.count;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = tc.m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (row >= tc.Mdim) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int col = tc.n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (col >= tc.Ndim) continue;
      const float v = acc[i][j];
      if (op == OP_GRAM) {
        reinterpret_cast<float*>(a.A)[aoff + (int64_t)row * gi.gld + col] = v;
      } else if (op == OP_SQUARE) {
        const float prev = Am[(int64_t)row * gi.gld + col];
        reinterpret_cast<float*>(a.B)[aoff + (int64_t)row * gi.gld + col] = fmaf(c0, prev, c1 * v);
      } else {
        const float xv = X[(int64_t)row * gi.ld + col];
        const float o = fmaf(c0, xv, c1 * v);
        if (a.final_out)
          a.out[(int64_t)w * a.out_stride + a.mat_off[mat] + (int64_t)row * gi.cols + col] = o;
        else
          reinterpret_cast<float*>(a.X_dst)[xoff + (int64_t)row * gi.ld + col] = o;
      }
    }
  }
}

}  // namespace

void launch_gemm_simt(cudaStream_t s, const GemmArgs& a, int /*x_f32*/) {
  if (a.total_tiles <= 0) return;
  count_launch();
  launch_pdl(k_gemm_simt, dim3(a.total_tiles), dim3(NT), 0, s, a);
}

}  // namespace sm
