// kernels_elem.cu -- the HBM-bound kernels of the Sign-Muon step:
//   momentum pass (weight decay + momentum + X staging + Frobenius partials),
//   scale finalisation, power iteration on the Gram matrix, one-bit pack,
//   majority vote (API form, fused with the update, or emitting D), update.
//
// Sources, by page title:
//   [paper] "SignMuon: 通信高效的分布式Muon优化" (a rendering of arXiv 2605.16311)
//   [blog]  "SignMuon: Matrix Directions, Majority Votes, and the Actual Bytes Sent"
#include "common.cuh"

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>
#include <tuple>

namespace sm {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Fixed-order block reduction (deterministic): warp sums, then warp 0.
template <typename T>
__device__ T block_sum(T v, T* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  v = (sizeof(T) == 8) ? (T)warp_sum_d((double)v) : (T)warp_sum((float)v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  T t = 0;
  if (wid == 0) {
    t = (lane < (int)(blockDim.x >> 5)) ? red[lane] : (T)0;
    t = (sizeof(T) == 8) ? (T)warp_sum_d((double)t) : (T)warp_sum((float)t);
  }
  return t;  // valid in thread 0
}

// 16-byte global -> shared copy that bypasses the registers (and L1)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void store_x(void* X, int64_t idx, float v, bool bf16) {
  if (bf16) reinterpret_cast<__nv_bfloat16*>(X)[idx] = __float2bfloat16_rn(v);
  else reinterpret_cast<float*>(X)[idx] = v;
}
__device__ __forceinline__ void store_x4(void* X, int64_t idx, float4 v, bool bf16) {
  if (bf16) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(X) + idx) = u;
  } else {
    st4(reinterpret_cast<float*>(X) + idx, v);
  }
}

// ---------------------------------------------------------------------------
// Momentum pass ([paper] Algorithm 1 / Algorithm 2: G~ = G + lambda W, then
// Mom <- beta Mom + (1-beta) G~).  One block owns one chunk of one matrix
// and loops over the workers, so W is read once per element.  It writes the
// new momentum, the Newton-Schulz input X (bf16 or fp32, grouped layout) and
// the chunk's sum of squares per worker (for the Frobenius scale and the
// non-finite check).  MOMENTUM=false stages a caller's vector unchanged.
// ---------------------------------------------------------------------------
template <bool MOMENTUM>
__global__ void __launch_bounds__(kThreads)
k_momentum(WorkerPtrs G, const float* __restrict__ W, float* __restrict__ Mom, int64_t d, int M,
           float beta, float lambda, void* __restrict__ X, int x_bf16,
           const Chunk* __restrict__ chunks, const MatInfo* __restrict__ mats,
           const GroupInfo* __restrict__ groups, float* __restrict__ partials) {
  griddep_wait();
  griddep_launch();
  // per-(worker, warp) partial sums of squares: one block barrier at the
  // end instead of two per worker, so that the warps run through the
  // workers independently
  __shared__ float red[kMaxWorkers * (kThreads / 32)];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const Chunk ch = chunks[blockIdx.x];
  const MatInfo mi = mats[ch.mat];
  const GroupInfo gi = groups[mi.group];
  const int64_t base = mi.off + ch.start;
  const bool vec = ((base & 3) == 0) && ((ch.len & 3) == 0) && ((mi.cols & 3) == 0);
  const float omb = 1.f - beta;
  const bool bf = x_bf16 != 0;
  constexpr int kV = kChunk / (kThreads * 4);  // float4 groups per thread
  float4 wv[kV];
  if (MOMENTUM && vec) {
#pragma unroll
    for (int j = 0; j < kV; ++j) {
      const int e = (threadIdx.x + j * kThreads) * 4;
      wv[j] = (e < ch.len) ? ld4(W + base + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  for (int m = 0; m < M; ++m) {
    const float* g = G.p[m];
    float* mom = MOMENTUM ? Mom + (int64_t)m * d : nullptr;
    const int64_t xb = gi.x_base + (int64_t)(m * gi.count + mi.q) * gi.rows * gi.ld;
    float ss = 0.f;
    if (vec) {
#pragma unroll
      for (int j = 0; j < kV; ++j) {
        const int e = (threadIdx.x + j * kThreads) * 4;
        if (e < ch.len) {
          const int64_t fe = base + e;
          float4 v = ld4(g + fe);
          if (MOMENTUM) {
            const float4 mo = ld4(mom + fe);
            v.x = fmaf(beta, mo.x, omb * fmaf(lambda, wv[j].x, v.x));
            v.y = fmaf(beta, mo.y, omb * fmaf(lambda, wv[j].y, v.y));
            v.z = fmaf(beta, mo.z, omb * fmaf(lambda, wv[j].z, v.z));
            v.w = fmaf(beta, mo.w, omb * fmaf(lambda, wv[j].w, v.w));
            st4(mom + fe, v);
          }
          ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
          const int le = (int)(ch.start + e);
          const int r = le / mi.cols, c = le - r * mi.cols;
          store_x4(X, xb + (int64_t)r * gi.ld + c, v, bf);
        }
      }
    } else {
      for (int e = threadIdx.x; e < ch.len; e += kThreads) {
        const int64_t fe = base + e;
        float v = g[fe];
        if (MOMENTUM) {
          v = fmaf(beta, mom[fe], omb * fmaf(lambda, W[fe], v));
          mom[fe] = v;
        }
        ss += v * v;
        const int le = (int)(ch.start + e);
        const int r = le / mi.cols, c = le - r * mi.cols;
        store_x(X, xb + (int64_t)r * gi.ld + c, v, bf);
      }
    }
    ss = warp_sum(ss);
    if (lane == 0) red[m * (kThreads / 32) + wid] = ss;
  }
  __syncthreads();
  for (int m = threadIdx.x; m < M; m += kThreads) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) t += red[m * (kThreads / 32) + w];
    partials[(int64_t)blockIdx.x * M + m] = t;
  }
}

__device__ __forceinline__ void set_coefs(int p, float cc, int quintic, float a, float b, float c,
                                          float2* coef_apply, float2* coef_square, float2* coef_gram) {
  // Iteration 0 runs on the unscaled X~ and Gram A~ = X~ X~^T.  With X0 = cc X~:
  //   cubic:   X1 = a cc X~ + b cc^3 A~ X~
  //   quintic: B = b cc^2 A~ + c cc^4 A~^2;  X1 = cc (a X~ + B X~)
  // and in Gram space (cubic, A0 = cc^2 A~): Q1 = a cc I + b cc^3 A~ (the
  // apply coefficients), T0 = a cc^2 A~ + b cc^4 A~^2 (coef_square), and
  // A1 = a T0 + b cc^2 A~ T0 (coef_gram)
  if (!quintic) {
    coef_apply[p] = make_float2(a * cc, b * cc * cc * cc);
    if (coef_gram != nullptr) {
      coef_square[p] = make_float2(a * cc * cc, b * cc * cc * cc * cc);
      coef_gram[p] = make_float2(a, b * cc * cc);
    }
  } else {
    coef_square[p] = make_float2(b * cc * cc, c * cc * cc * cc * cc);
    coef_apply[p] = make_float2(a * cc, cc);
  }
}

// Sum the chunk partials of each (worker, matrix) in a fixed order.
__global__ void __launch_bounds__(kThreads)
k_fro_finalize(int n_mats, int M, const float* __restrict__ partials, const int* __restrict__ mat_chunk0,
               const int* __restrict__ mat_nchunks, int use_for_scale, float eps, int quintic,
               float a, float b, float c, float* __restrict__ scale, float2* coef_apply,
               float2* coef_square, float2* coef_gram, int* status) {
  griddep_wait();
  griddep_launch();
  __shared__ double red[32];
  const int p = blockIdx.x;
  const int w = p / n_mats, i = p - w * n_mats;
  const int c0 = mat_chunk0[i], nc = mat_nchunks[i];
  double s = 0.0;
  for (int j = threadIdx.x; j < nc; j += kThreads) s += (double)partials[(int64_t)(c0 + j) * M + w];
  const double t = block_sum<double>(s, red);
  if (threadIdx.x == 0) {
    if (!isfinite(t)) atomicOr(status, 1);
    if (use_for_scale) {
      const float sc = (float)sqrt(t);
      scale[p] = sc;
      set_coefs(p, 1.f / (sc + eps), quintic, a, b, c, coef_apply, coef_square, coef_gram);
    }
  }
}

// ---------------------------------------------------------------------------
// Power iteration on the Gram matrix A~ = X~ X~^T of the wide orientation
// ([paper] Algorithm 1 inputs scale=spectral and P; §4 spectral
// normalisation by power iteration): u0 = ones/sqrt(g); u <- A~u/||A~u|| P
// times; sigma^2 = u^T A~ u (= ||X~^T u||^2).  The Gram is the first
// Newton-Schulz GEMM's output, so no extra pass over X is needed.
// With warm set, a problem whose stored iterate (the one the previous call
// ended with) is non-zero and finite starts from it instead of ones/sqrt(g).
//
// A~ is symmetric, so a pass reads only the tiles (I, J), I <= J, of a
// 128 x 128 tiling: an off-diagonal tile gives A_IJ v_J to y_I (its row sums)
// and A_IJ^T v_I to y_J (its column sums), a diagonal tile A_II v_I.  A block
// takes one tile; each contribution has its own slot in a partial-sum buffer
// (slot K of slice I comes from the tile that pairs slices I and K), and
// k_pi_reduce adds the slots of a slice in slot order, so the result does
// not depend on the schedule.  A diagonal tile reads its upper triangle only
// (its rows give the entries on and above the diagonal, its columns the ones
// above), so a pass reads about g (g + 1) / 2 of the g^2 entries.  The
// normalisation of an iterate is folded into the passes: the reduction's
// last block per problem forms 1/||y||, and the next pass scales y by it
// while staging it; after the last pass it forms sigma^2 = u^T y and the
// scale instead.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads)
k_pi_init(const int64_t* __restrict__ uoff, const int* __restrict__ prob_g, float* __restrict__ u, int warm) {
  griddep_wait();
  griddep_launch();
  __shared__ double red[32];
  __shared__ int keep;
  const int p = blockIdx.x;
  const int g = prob_g[p];
  float* up = u + uoff[p];
  if (warm) {
    double s = 0.0;
    for (int k = threadIdx.x; k < g; k += kThreads) s += (double)up[k] * (double)up[k];
    const double t = block_sum<double>(s, red);
    if (threadIdx.x == 0) keep = (t > 0.0 && isfinite(t)) ? 1 : 0;
    __syncthreads();
    if (keep) return;  // the whole block leaves together
  }
  const float v = rsqrtf((float)g);
  for (int k = threadIdx.x; k < g; k += kThreads) up[k] = v;
}

// A lane's share of a 128 x 128 tile: NL 16-byte vectors of columns cl ..
// cl + V - 1, one per tile row rw, rw + RPS, ...
template <bool BF16>
struct PiLane {
  static constexpr int T = kPiTile;
  static constexpr int V = BF16 ? 8 : 4;            // entries per 16-byte vector
  static constexpr int LPR = T / V;                 // lanes per tile row: 16 or 32
  static constexpr int RPS = 32 / LPR;              // tile rows per warp step: 2 or 1
  static constexpr int RPW = T / (kThreads / 32);   // tile rows per warp
  static constexpr int NL = RPW / RPS;              // vectors per lane: 8 or 16
  static constexpr int ROWB = T * (BF16 ? 2 : 4);   // bytes of a tile row
  static constexpr int TILEB = T * ROWB;            // 32 KB or 64 KB
};

// Two fp32 FMAs in one instruction (PTX fma.rn.f32x2, sm_100): the same
// correctly rounded a * b + c per lane as fmaf.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(r)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)),
        "l"(*reinterpret_cast<const uint64_t*>(&c)));
  return *reinterpret_cast<const float2*>(&r);
}

// Sums of one tile out of shared memory: this lane's partial of each of its
// rows (over its V columns) into rowp[r], its column partials into cacc
// (pairs).  With MASK, entries past row or column g (whose vectors were not
// loaded) and, on a diagonal tile, below the diagonal count as zero, and the
// diagonal itself only in the row sums.
template <bool BF16, bool MASK>
__device__ __forceinline__ void pi_tile_sums(const uint8_t* tile, int rw, int cl, int rows_left, int nvalid,
                                             bool diag, const float2* vjr, const float* vi, float* rowp,
                                             float2* cacc) {
  using L = PiLane<BF16>;
#pragma unroll
  for (int j = 0; j < L::NL; ++j) {
    const int r = rw + j * L::RPS;
    const uint4 raw = *reinterpret_cast<const uint4*>(tile + r * L::ROWB + cl * (BF16 ? 2 : 4));
    float2 a[L::V / 2];
    if (BF16) {
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&raw);
#pragma unroll
      for (int t = 0; t < L::V / 2; ++t)  // bf16 -> fp32 is a 16-bit shift
        a[t] = make_float2(__uint_as_float(w[t] << 16), __uint_as_float(w[t] & 0xFFFF0000u));
    } else {
      const float2* fv = reinterpret_cast<const float2*>(&raw);
#pragma unroll
      for (int t = 0; t < L::V / 2; ++t) a[t] = fv[t];
    }
    int lo = 0;
    if (MASK) {
      lo = diag ? r - cl : 0;  // entries e < lo lie below the diagonal
      const bool live = r < rows_left;
#pragma unroll
      for (int t = 0; t < L::V / 2; ++t) {
        a[t].x = (live && 2 * t < nvalid && 2 * t >= lo) ? a[t].x : 0.f;
        a[t].y = (live && 2 * t + 1 < nvalid && 2 * t + 1 >= lo) ? a[t].y : 0.f;
      }
    }
    float2 sr = make_float2(0.f, 0.f);
#pragma unroll
    for (int t = 0; t < L::V / 2; ++t) sr = fma2(a[t], vjr[t], sr);
    rowp[r] = sr.x + sr.y;
    const float2 vr = make_float2(vi[r], vi[r]);
#pragma unroll
    for (int t = 0; t < L::V / 2; ++t) {
      float2 ac = a[t];
      if (MASK && diag) {
        if (2 * t == lo) ac.x = 0.f;
        if (2 * t + 1 == lo) ac.y = 0.f;
      }
      cacc[t] = fma2(ac, vr, cacc[t]);
    }
  }
}

// One block per tile (I, J), I <= J: the tile comes into shared memory by
// cp.async (vectors past row or column g, and on a diagonal tile the ones
// wholly below the diagonal, are not read) while v_I and v_J are staged.
// Its row sums go to slot J of slice I, its column sums (J > I) to slot I of
// slice J; a diagonal tile adds its column sums to its row sums.
template <bool BF16>
__global__ void __launch_bounds__(kThreads)
k_pi_tiles(const PiTile* __restrict__ tiles, const void* __restrict__ A, const float* __restrict__ src,
           const float* __restrict__ inv, float* __restrict__ u, float* __restrict__ part, int fold) {
  griddep_wait();
  griddep_launch();
  using L = PiLane<BF16>;
  constexpr int T = kPiTile;
  constexpr int esz = BF16 ? 2 : 4;
  static_assert(kThreads == 2 * T, "one staging thread per entry of v_I and v_J");
  __shared__ float vi[T], vj[T];
  __shared__ float cols_s[kThreads / 32][T];     // warp w's column sums
  __shared__ float rowp[L::LPR * (T + 1)];       // [c][r]: row r over column group c (stride T + 1)
  extern __shared__ __align__(16) uint8_t pi_tile_smem[];   // the tile
  const PiTile tl = tiles[blockIdx.x];
  const int g = tl.g, I = tl.bi, J = tl.bj;
  const bool diag = I == J;
  const int nt = (g + T - 1) / T;
  const int r0 = I * T, c0 = J * T, rows_left = g - r0;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int cl = (lane % L::LPR) * L::V;        // this lane's first column in the tile
  const int rw = wid * L::RPW + lane / L::LPR;  // its first tile row
  const int nvalid = g - (c0 + cl);             // entries of its vector inside the matrix
  {
    // A is g x gld with gld a multiple of 8, so a 16-byte vector that starts
    // inside a row stays inside it
    const char* src_a = reinterpret_cast<const char*>(A) + (tl.aoff + (int64_t)r0 * tl.gld + c0 + cl) * esz;
    const int64_t row_bytes = (int64_t)tl.gld * esz;
    const uint32_t dst = (uint32_t)__cvta_generic_to_shared(pi_tile_smem) + (uint32_t)(cl * esz);
#pragma unroll
    for (int j = 0; j < L::NL; ++j) {
      const int r = rw + j * L::RPS;
      if (r < rows_left && nvalid > 0 && (!diag || cl + L::V - 1 >= r))
        cp_async16(dst + (uint32_t)(r * L::ROWB), src_a + (int64_t)r * row_bytes);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  {
    // src == nullptr: a cold start, v = u0 = ones / sqrt(g) (no stored vector)
    const float sc = fold ? inv[tl.p] : 1.f;
    const float v0 = rsqrtf((float)g);
    const int k = threadIdx.x & (T - 1);
    if (threadIdx.x < T) {
      const float v = (r0 + k < g) ? (src ? src[tl.uoff + r0 + k] * sc : v0) : 0.f;
      vi[k] = v;
      if (fold && diag && r0 + k < g) u[tl.uoff + r0 + k] = v;  // the normalised iterate, once per slice
    } else {
      vj[k] = (c0 + k < g) ? (src ? src[tl.uoff + c0 + k] * sc : v0) : 0.f;
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  float2 vjr[L::V / 2], cacc[L::V / 2];
#pragma unroll
  for (int t = 0; t < L::V / 2; ++t) {
    vjr[t] = make_float2(vj[cl + 2 * t], vj[cl + 2 * t + 1]);
    cacc[t] = make_float2(0.f, 0.f);
  }
  float* rowp_c = rowp + (lane % L::LPR) * (T + 1);
  if (diag || rows_left < T || c0 + T > g)   // block-uniform
    pi_tile_sums<BF16, true>(pi_tile_smem, rw, cl, rows_left, nvalid, diag, vjr, vi, rowp_c, cacc);
  else
    pi_tile_sums<BF16, false>(pi_tile_smem, rw, cl, rows_left, nvalid, false, vjr, vi, rowp_c, cacc);
  if (L::RPS == 2) {
#pragma unroll
    for (int t = 0; t < L::V / 2; ++t) {
      cacc[t].x += __shfl_xor_sync(0xffffffffu, cacc[t].x, 16);
      cacc[t].y += __shfl_xor_sync(0xffffffffu, cacc[t].y, 16);
    }
  }
  if (lane < L::LPR) {
#pragma unroll
    for (int t = 0; t < L::V / 2; ++t) {
      cols_s[wid][cl + 2 * t] = cacc[t].x;
      cols_s[wid][cl + 2 * t + 1] = cacc[t].y;
    }
  }
  __syncthreads();
  float* pp = part + tl.poff;
  const int64_t gp = (int64_t)nt * T;
  const int k = threadIdx.x & (T - 1);
  float cs = 0.f;
  if (diag || threadIdx.x >= T) {
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) cs += cols_s[w][k];
  }
  if (threadIdx.x < T) {
    float rs = 0.f;
#pragma unroll
    for (int c = 0; c < L::LPR; ++c) rs += rowp[c * (T + 1) + k];
    // slice I, slot J: the row sums (a diagonal tile adds its column sums,
    // the mirror of its strict upper triangle)
    pp[(int64_t)J * gp + r0 + k] = diag ? rs + cs : rs;
  } else if (!diag) {
    pp[(int64_t)I * gp + c0 + k] = cs;  // slice J, slot I
  }
}

// One block per 128-row slice: y = its nt slots added in slot order,
// ||y_slice||^2 (or, on the last pass, u_slice . y_slice) in fp64; the
// problem's last slice to finish adds the slices' figures in slice order:
// 1 / ||y|| for the next pass, or sigma^2 = u^T y and the scale.
__global__ void __launch_bounds__(kPiTile)
k_pi_reduce(const PiSlice* __restrict__ slices, const float* __restrict__ part, float* __restrict__ y,
            PiReduce rd) {
  griddep_wait();
  griddep_launch();
  constexpr int T = kPiTile;
  __shared__ double red[32];
  __shared__ int is_last;
  const PiSlice sl = slices[blockIdx.x];
  const int g = sl.g;
  const int nt = (g + T - 1) / T;
  const int64_t gp = (int64_t)nt * T;
  const int r = sl.bi * T + threadIdx.x;
  const float* pp = part + sl.poff + r;
  float v = 0.f;
#pragma unroll 8
  for (int k = 0; k < nt; ++k) v += pp[(int64_t)k * gp];
  double acc = 0.0;
  if (r < g) {
    y[sl.uoff + r] = v;
    acc = rd.last ? (double)rd.u[sl.uoff + r] * (double)v : (double)v * (double)v;
  }
  const double t = block_sum<double>(acc, red);
  if (threadIdx.x == 0) {
    rd.sq[sl.soff + sl.bi] = t;
    __threadfence();
    is_last = (atomicAdd(&rd.counters[sl.p], 1) == nt - 1);
  }
  __syncthreads();
  if (!is_last || threadIdx.x != 0) return;
  __threadfence();
  double tt = 0.0;
  for (int i = 0; i < nt; ++i) tt += __ldcg(rd.sq + sl.soff + i);
  rd.counters[sl.p] = 0;
  if (!rd.last) {
    rd.inv[sl.p] = (tt > 0.0) ? (float)(1.0 / sqrt(tt)) : 0.f;  // a zero iterate stays zero
    return;
  }
  const float scv = (float)sqrt(fmax(tt, 0.0));
  if (!isfinite(tt)) atomicOr(rd.status, 1);
  rd.scale[sl.p] = scv;
  set_coefs(sl.p, 1.f / (scv + rd.eps), rd.quintic, rd.a, rd.b, rd.c, rd.coef_apply, rd.coef_square,
            rd.coef_gram);
}

// K = 0: U = X0 = in / (s + eps) straight from the fp32 input.
__global__ void __launch_bounds__(kThreads)
k_scale_flat(WorkerPtrs in, float* __restrict__ out, int64_t out_stride,
             const Chunk* __restrict__ chunks, const MatInfo* __restrict__ mats, int n_mats,
             const float* __restrict__ scale, float eps) {
  griddep_wait();
  griddep_launch();
  const Chunk ch = chunks[blockIdx.x];
  const int w = blockIdx.y;
  const MatInfo mi = mats[ch.mat];
  const float cc = 1.f / (scale[w * n_mats + ch.mat] + eps);
  const float* src = in.p[w];
  float* dst = out + (int64_t)w * out_stride;
  const int64_t base = mi.off + ch.start;
  for (int e = threadIdx.x; e < ch.len; e += kThreads) dst[base + e] = src[base + e] * cc;
}

// ---------------------------------------------------------------------------
// One-bit pack ([paper] §3 entrywise sign; [blog] d/8-byte payload).
// bit = (u >= 0): 0 and -0 send +1, NaN sends 0.  A warp takes 1024
// consecutive entries as 8 rounds of 32 lanes x float4; four __ballot_sync
// calls per round give the sign of entry 4*lane+j in bit lane of mask j, and
// a bit interleave turns the four masks into the round's four LSB-first words.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t spread8(uint32_t x) {  // bit i -> bit 4i
  x = (x | (x << 12)) & 0x000F000Fu;
  x = (x | (x << 6)) & 0x03030303u;
  x = (x | (x << 3)) & 0x11111111u;
  return x;
}

__global__ void __launch_bounds__(kThreads)
k_pack(const float* __restrict__ U, int64_t u_stride, int64_t d, uint8_t* __restrict__ out,
       int64_t out_stride) {
  griddep_wait();
  griddep_launch();
  const int w = blockIdx.y;
  U += (int64_t)w * u_stride;
  out += (int64_t)w * out_stride;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
  const int64_t nchunks = (d + 1023) >> 10;
  const int64_t nb = (d + 7) >> 3;
  const int k = lane & 3;
  for (int64_t c = warp0; c < nchunks; c += nwarps) {
    uint32_t mine = 0;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int64_t e = c * 1024 + it * 128 + lane * 4;
      bool b0, b1, b2, b3;
      if (e + 3 < d) {
        const float4 v = ld4(U + e);
        b0 = v.x >= 0.f; b1 = v.y >= 0.f; b2 = v.z >= 0.f; b3 = v.w >= 0.f;
      } else {
        b0 = (e < d) && (U[e] >= 0.f);
        b1 = (e + 1 < d) && (U[e + 1] >= 0.f);
        b2 = (e + 2 < d) && (U[e + 2] >= 0.f);
        b3 = (e + 3 < d) && (U[e + 3] >= 0.f);
      }
      const uint32_t m0 = __ballot_sync(0xffffffffu, b0);
      const uint32_t m1 = __ballot_sync(0xffffffffu, b1);
      const uint32_t m2 = __ballot_sync(0xffffffffu, b2);
      const uint32_t m3 = __ballot_sync(0xffffffffu, b3);
      const int sh = 8 * k;
      const uint32_t word = spread8((m0 >> sh) & 0xFFu) | (spread8((m1 >> sh) & 0xFFu) << 1) |
                            (spread8((m2 >> sh) & 0xFFu) << 2) | (spread8((m3 >> sh) & 0xFFu) << 3);
      if ((lane >> 2) == it) mine = word;
    }
    const int64_t byte0 = (c * 32 + lane) * 4;
    if (byte0 + 4 <= nb) {
      *reinterpret_cast<uint32_t*>(out + byte0) = mine;
    } else {
      for (int t = 0; t < 4; ++t)
        if (byte0 + t < nb) out[byte0 + t] = (uint8_t)(mine >> (8 * t));
    }
  }
}

// ---------------------------------------------------------------------------
// Majority vote ([paper] Algorithm 2: integer SUM of the signs then sign();
// [blog]: ties give 0, sums lie in [-M, M]).
__device__ __forceinline__ int sgn(int s) { return (s > 0) - (s < 0); }
// majority of a vote sum: sign(s) with a tie sent to 0, or to +1 when
// tie_plus is set ([paper] Algorithm 2's default, a named variant)
__device__ __forceinline__ int vmaj(int s, int tie_plus) { return tie_plus ? (s >= 0 ? 1 : -1) : sgn(s); }

// MODE 0: API vote (sums + majority); 1: fused update of W; 2: write D = majority.
// A warp takes 512 consecutive entries (4 blocks of 128) per step.  The 8
// lanes of group j = lane / 8 share block j: each loads that block's 16 bytes
// of every worker's stream (so one load instruction reads 64 contiguous
// bytes per worker) and counts 4 of its 32 nibbles: lane g = lane % 8 takes
// entries 32k + 4g .. 32k + 4g + 3 (k = 0..3), so that each store
// instruction writes whole 128-byte lines.  Byte-lane counters: nibble *
// 0x00204081 & 0x01010101 spreads 4 bits into 4 byte lanes, flushed every 248
// workers so that no lane overflows; 8 workers' loads are in flight at once.
template <int MODE, bool ACC8>
__global__ void __launch_bounds__(kThreads)
k_vote(WorkerPtrs signs, int M, int64_t d,
       void* __restrict__ sums, int8_t* __restrict__ maj, float* __restrict__ W, float eta,
       float* __restrict__ D, const int* __restrict__ status, int tie_plus) {
  griddep_wait();
  griddep_launch();
  if (MODE == 1 && status != nullptr && (status[0] | status[1]) != 0) return;  // keep W on error
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
  const int64_t nblk = d >> 7;                  // full 128-entry blocks
  const int grp = lane >> 3, g = lane & 7, shift = 4 * g;
  auto stream = [&](int m) { return reinterpret_cast<const uint8_t*>(signs.p[m]); };
  for (int64_t st = gw; st * 4 < nblk; st += nw) {
    const int64_t b = st * 4 + grp;               // this lane group's block
    const bool on = b < nblk;
    int cnt[4][4];
#pragma unroll
    for (int k = 0; k < 4; ++k) cnt[k][0] = cnt[k][1] = cnt[k][2] = cnt[k][3] = 0;
    uint32_t acc[4] = {0u, 0u, 0u, 0u};
    for (int m = 0; m < M; m += 8) {
      uint4 wv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        wv[i] = (on && m + i < M) ? __ldg(reinterpret_cast<const uint4*>(stream(m + i) + b * 16))
                                  : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[0] += (((wv[i].x >> shift) & 0xFu) * 0x00204081u) & 0x01010101u;
        acc[1] += (((wv[i].y >> shift) & 0xFu) * 0x00204081u) & 0x01010101u;
        acc[2] += (((wv[i].z >> shift) & 0xFu) * 0x00204081u) & 0x01010101u;
        acc[3] += (((wv[i].w >> shift) & 0xFu) * 0x00204081u) & 0x01010101u;
      }
      if (((m + 8) % 248) == 0 || m + 8 >= M) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          cnt[k][0] += acc[k] & 0xFF;
          cnt[k][1] += (acc[k] >> 8) & 0xFF;
          cnt[k][2] += (acc[k] >> 16) & 0xFF;
          cnt[k][3] += acc[k] >> 24;
          acc[k] = 0;
        }
      }
    }
    if (!on) continue;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int s0 = 2 * cnt[k][0] - M, s1 = 2 * cnt[k][1] - M, s2 = 2 * cnt[k][2] - M, s3 = 2 * cnt[k][3] - M;
      const int64_t e = b * 128 + 32 * k + 4 * g;
      if (MODE == 0) {
        if (sums != nullptr) {
          if (ACC8) {
            char4 v = make_char4((signed char)s0, (signed char)s1, (signed char)s2, (signed char)s3);
            *reinterpret_cast<char4*>(reinterpret_cast<int8_t*>(sums) + e) = v;
          } else {
            *reinterpret_cast<int4*>(reinterpret_cast<int32_t*>(sums) + e) = make_int4(s0, s1, s2, s3);
          }
        }
        if (maj != nullptr)
          *reinterpret_cast<char4*>(maj + e) =
              make_char4((signed char)vmaj(s0, tie_plus), (signed char)vmaj(s1, tie_plus), (signed char)vmaj(s2, tie_plus), (signed char)vmaj(s3, tie_plus));
      } else if (MODE == 1) {
        float4 w = ld4(W + e);
        w.x = fmaf(-eta, (float)vmaj(s0, tie_plus), w.x);
        w.y = fmaf(-eta, (float)vmaj(s1, tie_plus), w.y);
        w.z = fmaf(-eta, (float)vmaj(s2, tie_plus), w.z);
        w.w = fmaf(-eta, (float)vmaj(s3, tie_plus), w.w);
        st4(W + e, w);
      } else {
        st4(D + e, make_float4((float)vmaj(s0, tie_plus), (float)vmaj(s1, tie_plus), (float)vmaj(s2, tie_plus), (float)vmaj(s3, tie_plus)));
      }
    }
  }
  // ragged tail (< 128 entries): bit loads, one entry per thread
  if (blockIdx.x == gridDim.x - 1) {
    for (int64_t e = nblk * 128 + threadIdx.x; e < d; e += kThreads) {
      int c = 0;
      for (int m = 0; m < M; ++m) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(signs.p[m]);
        c += (src[e >> 3] >> (e & 7)) & 1;
      }
      const int sm_ = 2 * c - M;
      if (MODE == 0) {
        if (sums != nullptr) {
          if (ACC8) reinterpret_cast<int8_t*>(sums)[e] = (int8_t)sm_;
          else reinterpret_cast<int32_t*>(sums)[e] = sm_;
        }
        if (maj != nullptr) maj[e] = (int8_t)vmaj(sm_, tie_plus);
      } else if (MODE == 1) {
        W[e] = fmaf(-eta, (float)vmaj(sm_, tie_plus), W[e]);
      } else {
        D[e] = (float)vmaj(sm_, tie_plus);
      }
    }
  }
}

// Byte-lane helpers of the vote's output: x holds four counts c (one per byte,
// c <= M <= 255).
// 2c - M per byte, modulo 256 (an exact int8 when M <= 127): 2c <= 254 has no
// carry out of its byte, and the subtraction borrows nothing across bytes.
__device__ __forceinline__ uint32_t swar_twice_minus(uint32_t x, int M) {
  const uint32_t a = x << 1, b = (uint32_t)M * 0x01010101u, H = 0x80808080u;
  return ((a | H) - (b & ~H)) ^ ((a ^ ~b) & H);
}
// sign(2c - M) per byte as int8 (+1 = 0x01, -1 = 0xFF, a tie 0x00, or 0x01
// with tie_plus): c > M/2 <=> c + 127 - floor(M/2) has bit 7 set, and c < M/2
// <=> c + 128 - ceil(M/2) has not (neither sum leaves its byte for M <= 255).
__device__ __forceinline__ uint32_t swar_majority(uint32_t x, int M, int tie_plus) {
  const uint32_t H = 0x80808080u;
  const uint32_t gt = (x + (uint32_t)(127 - M / 2) * 0x01010101u) & H;
  const uint32_t lt = ~(x + (uint32_t)(128 - (M + 1) / 2) * 0x01010101u) & H;
  if (tie_plus) return ((lt >> 7) * 0xFEu) + 0x01010101u;
  return (gt >> 7) | ((lt >> 7) * 0xFFu);
}

// PTX prmt in its default mode with b = 0: byte n of the result is byte
// (SEL >> 4n) & 7 of {a, b} (a = bytes 0-3), and bit 3 of that selector
// nibble replicates the selected byte's top bit over the result byte.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t prmt_sx(uint32_t a) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(a), "n"(SEL));
  return r;
}

// Streaming vote for M <= 255 (byte-lane counters): each warp takes tiles of 4096 consecutive entries (512 bytes of
// every worker's stream).  The bytes come into shared memory by cp.async, 16
// per lane (each load instruction reads 512 contiguous bytes of one stream),
// kVoteBatch workers at a time, double-buffered so that the next batch is in
// flight while this one is counted.  Lane t then counts entries 128 j + 4 t
// .. + 3 for j = 0..31 (nibble t % 8 of word 4 j + t / 8, a shared-memory
// broadcast among 8 lanes) into byte-lane counters, and writes each group of
// 4 results with one vector store (the warp's stores are contiguous).
constexpr int kVoteBatch = 8;
constexpr int kVoteWarps = 4;                  // warps per block
constexpr int kVoteTileB = 512;                // bytes of one stream per tile


// MODE 3 (staging of the post-vote polar step's input): the work items are
// the plan's chunks instead of flat tiles.  Chunk c covers entries base ..
// base + len - 1 of the flat vector (base = its matrix's offset + its start,
// a multiple of 128; len <= 4096); its majorities go to the bf16 X of the
// one-problem-set Newton-Schulz input, which for a matrix with a multiple of
// 8 columns is the chunk's contiguous range starting at its X offset, and
// partials[c] receives the chunk's count of non-zero majorities (its sum of
// squares).  off[c] = (base, X offset), precomputed so that a chunk's bytes
// can be requested after a single table load.
struct VoteStage {
  __nv_bfloat16* X;
  const Chunk* chunks;
  const longlong2* off;
  float* partials;
};

template <int MODE, bool ACC8>
__global__ void __launch_bounds__(kVoteWarps * 32, 6)
k_vote_stream(WorkerPtrs signs, int M, int64_t ntiles,
              void* __restrict__ sums, int8_t* __restrict__ maj, float* __restrict__ W, float eta,
              float* __restrict__ D, const int* __restrict__ status, int tie_plus, VoteStage st) {
  griddep_wait();
  griddep_launch();
  constexpr bool STAGE = MODE >= 3;  // chunks of the post-vote input (MODE 4 also writes D)
  if (MODE == 1 && status != nullptr && (status[0] | status[1]) != 0) return;  // keep W on error
  extern __shared__ __align__(16) uint8_t vsm[];   // [warp][2][kVoteBatch][512]
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t gw = (int64_t)blockIdx.x * kVoteWarps + wid;
  const int64_t nw = (int64_t)gridDim.x * kVoteWarps;
  const uint32_t buf0 = (uint32_t)__cvta_generic_to_shared(vsm) + (uint32_t)wid * (2 * kVoteBatch * kVoteTileB);
  const int nbatch = (M + kVoteBatch - 1) / kVoteBatch;
  auto stream = [&](int m) { return reinterpret_cast<const uint8_t*>(signs.p[m]); };
  // (tile, batch) work items of this warp, in order
  int64_t tile = gw;
  int batch = 0;
  // flat start and length of work item t (a whole tile, or one chunk)
  auto item_base = [&](int64_t t) -> int64_t {
    if (STAGE) return st.off[t].x;
    return t * 4096;
  };
  auto item_len = [&](int64_t t) -> int { return STAGE ? st.chunks[t].len : 4096; };
  auto issue = [&](int64_t t, int bt, int buf) {
    const uint32_t dst = buf0 + (uint32_t)buf * (kVoteBatch * kVoteTileB) + (uint32_t)lane * 16;
    const int64_t boff = item_base(t) >> 3;
    // a lane's 16 bytes hold entries 128 lane .. 128 lane + 127 of the item;
    // pieces wholly past a short chunk's end are not read
    const bool live = !STAGE || lane * 128 < item_len(t);
#pragma unroll
    for (int i = 0; i < kVoteBatch; ++i) {
      const int m = bt * kVoteBatch + i;
      if (m < M && live) cp_async16(dst + (uint32_t)i * kVoteTileB, stream(m) + boff + lane * 16);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  if (tile >= ntiles) return;
  issue(tile, 0, 0);
  int cur = 0;
  // Counting: lane t counts the 128 entries it loaded itself (entries 128 t ..
  // 128 t + 127 of the item, four 32-bit words of every stream).  Bit g + 4 q
  // of word w goes to nibble q of the vertical counter nib[w][g] (one
  // shift-and-add per 8 entries and worker); after each batch of <= 8 workers
  // the nibbles move into byte counters: byte b of cb[w][g][0] counts entry
  // 32 w + 8 b + g, of cb[w][g][1] entry 32 w + 8 b + 4 + g.
  uint32_t cb[4][4][2];
#pragma unroll
  for (int w = 0; w < 4; ++w)
#pragma unroll
    for (int g = 0; g < 4; ++g) cb[w][g][0] = cb[w][g][1] = 0;
  while (true) {
    // the next work item goes out before this one is counted
    int64_t ntile = tile;
    int nbt = batch + 1;
    if (nbt == nbatch) { nbt = 0; ntile += nw; }
    if (ntile < ntiles) {
      issue(ntile, nbt, cur ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncwarp();
    const uint32_t src = buf0 + (uint32_t)cur * (kVoteBatch * kVoteTileB);
    const int nm = min(kVoteBatch, M - batch * kVoteBatch);
    {
      uint32_t nib[4][4];
#pragma unroll
      for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int g = 0; g < 4; ++g) nib[w][g] = 0;
      for (int i = 0; i < nm; ++i) {
        uint32_t v[4];
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                     : "r"(src + (uint32_t)i * kVoteTileB + (uint32_t)lane * 16));
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
          for (int g = 0; g < 4; ++g) nib[w][g] += (v[w] >> g) & 0x11111111u;
      }
#pragma unroll
      for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          cb[w][g][0] += nib[w][g] & 0x0F0F0F0Fu;
          cb[w][g][1] += (nib[w][g] >> 4) & 0x0F0F0F0Fu;
        }
    }
    __syncwarp();
    uint32_t acc[32];   // byte lane i of acc[j]: the count of entry 128 j + 4 lane + i
    if (batch == nbatch - 1) {
      // Byte counts in entry order for this lane's 128 entries: word 8 w + 2 b
      // + h holds entries 32 w + 8 b + 4 h .. + 3 (a 4 x 4 byte transpose of
      // cb[w][0..3][h]), written to row `lane` of the (consumed) batch buffer
      // with an XOR swizzle; column reads then give lane t the words of
      // entries 128 j + 4 t .. + 3, so that each warp store below writes
      // consecutive entries.  Both passes are free of bank conflicts.
      const uint32_t tr = src;   // 32 x 32 words = 4 KB of the buffer just counted
#pragma unroll
      for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t t0 = __byte_perm(cb[w][0][h], cb[w][1][h], 0x5140);
          const uint32_t t1 = __byte_perm(cb[w][0][h], cb[w][1][h], 0x7362);
          const uint32_t t2 = __byte_perm(cb[w][2][h], cb[w][3][h], 0x5140);
          const uint32_t t3 = __byte_perm(cb[w][2][h], cb[w][3][h], 0x7362);
          const uint32_t o[4] = {__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632),
                                 __byte_perm(t1, t3, 0x5410), __byte_perm(t1, t3, 0x7632)};
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int k = 8 * w + 2 * b + h;
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(tr + (uint32_t)(lane * 32 + (k ^ lane)) * 4), "r"(o[b])
                         : "memory");
          }
          cb[w][0][h] = cb[w][1][h] = cb[w][2][h] = cb[w][3][h] = 0;
        }
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 32; ++j)
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(acc[j]) : "r"(tr + (uint32_t)(j * 32 + (lane ^ j)) * 4) : "memory");
      __syncwarp();
    }
    if (batch == nbatch - 1 && STAGE) {
      // chunk done: its majorities into X (4 bf16 per lane and step, so each
      // warp store writes 256 contiguous bytes) and (MODE 4) D, its non-zero
      // count
      const longlong2 o = st.off[tile];
      const int len = st.chunks[tile].len;
      __nv_bfloat16* xo = st.X + o.y;
      const int64_t fb = o.x;
      const uint32_t H = 0x80808080u;
      const uint32_t kgt = (uint32_t)(127 - M / 2) * 0x01010101u;
      const uint32_t klt = (uint32_t)(128 - (M + 1) / 2) * 0x01010101u;
      int nz = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int e = j * 128 + lane * 4;
        if (e < len) {
          // per byte lane (count c): bit 7 of neg when c < M/2 (majority -1),
          // of nzm when the majority is not 0 (c > M/2 too; every entry with
          // tie_plus); as bf16 pairs +1 = 0x3F80, -1 = 0xBF80, 0 = 0
          const uint32_t x = acc[j];
          const uint32_t neg = ~(x + klt) & H;
          const uint32_t nzm = tie_plus ? H : (((x + kgt) & H) | neg);
          nz += __popc(nzm);
          uint2 u;
          u.x = (prmt_sx<0x9988>(nzm) & 0x3F803F80u) | (prmt_sx<0x9988>(neg) & 0x80008000u);
          u.y = (prmt_sx<0xBBAA>(nzm) & 0x3F803F80u) | (prmt_sx<0xBBAA>(neg) & 0x80008000u);
          *reinterpret_cast<uint2*>(xo + e) = u;
          if (MODE == 4) {
            const int c0 = x & 0xFF, c1 = (x >> 8) & 0xFF, c2 = (x >> 16) & 0xFF, c3 = x >> 24;
            st4(D + fb + e, make_float4((float)vmaj(2 * c0 - M, tie_plus), (float)vmaj(2 * c1 - M, tie_plus),
                                        (float)vmaj(2 * c2 - M, tie_plus), (float)vmaj(2 * c3 - M, tie_plus)));
          }
        }
      }
      nz = __reduce_add_sync(0xffffffffu, nz);
      if (lane == 0) st.partials[tile] = (float)nz;
    } else if (!STAGE && batch == nbatch - 1) {
      // tile done: write its 4096 results
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int c0 = acc[j] & 0xFF, c1 = (acc[j] >> 8) & 0xFF, c2 = (acc[j] >> 16) & 0xFF, c3 = acc[j] >> 24;
        const int s0 = 2 * c0 - M, s1 = 2 * c1 - M, s2 = 2 * c2 - M, s3 = 2 * c3 - M;
        const int64_t e = tile * 4096 + j * 128 + lane * 4;
        if (MODE == 0) {
          // the four results in byte lanes at once (acc[j] holds 4 counts c <= M)
          if (sums != nullptr) {
            if (ACC8) {
              // 2c - M mod 256 per byte: exact, since M <= 127 on this path
              *reinterpret_cast<uint32_t*>(reinterpret_cast<int8_t*>(sums) + e) = swar_twice_minus(acc[j], M);
            } else if (M <= 127) {
              // the same exact int8 sums, sign-extended to int32
              const uint32_t s8 = swar_twice_minus(acc[j], M);
              *reinterpret_cast<int4*>(reinterpret_cast<int32_t*>(sums) + e) =
                  make_int4((int)(s8 << 24) >> 24, (int)(s8 << 16) >> 24, (int)(s8 << 8) >> 24, (int)s8 >> 24);
            } else {
              *reinterpret_cast<int4*>(reinterpret_cast<int32_t*>(sums) + e) = make_int4(s0, s1, s2, s3);
            }
          }
          if (maj != nullptr) *reinterpret_cast<uint32_t*>(maj + e) = swar_majority(acc[j], M, tie_plus);
        } else if (MODE == 1) {
          float4 wv = ld4(W + e);
          wv.x = fmaf(-eta, (float)vmaj(s0, tie_plus), wv.x);
          wv.y = fmaf(-eta, (float)vmaj(s1, tie_plus), wv.y);
          wv.z = fmaf(-eta, (float)vmaj(s2, tie_plus), wv.z);
          wv.w = fmaf(-eta, (float)vmaj(s3, tie_plus), wv.w);
          st4(W + e, wv);
        } else {
          st4(D + e, make_float4((float)vmaj(s0, tie_plus), (float)vmaj(s1, tie_plus), (float)vmaj(s2, tie_plus), (float)vmaj(s3, tie_plus)));
        }
      }
    }
    tile = ntile;
    batch = nbt;
    cur ^= 1;
    if (tile >= ntiles) break;
  }
}

// Vote staging for M <= 15 (the post-vote input without D, as k_vote_stream
// MODE 3 computes it): bit-sliced counters.  Lane t of a warp takes entries
// 128 t .. 128 t + 127 of its chunk, four 32-bit words of every worker's
// stream, loaded as in k_vote_stream (8 workers per batch, double-buffered).
// Each word keeps four bit planes of the count c of set bits, one ripple add
// per worker (7 logic operations for 32 entries); the majority sgn(2c - M)
// is +1 where c >= TP and -1 where c < TN (bit masks P and N, from a borrow
// chain against each constant), 0 on a tie; and a 16-entry table in shared
// memory turns each pair of entries' four mask bits into their two bf16
// values (+1 = 0x3F80, -1 = 0xBF80, 0), which go out through shared memory so
// that every store writes whole 128-byte rows of the chunk's X.
constexpr int kVoteSlicedMaxM = 15;

// c >= T for the count in bit planes c[0..3] (c <= 15): no borrow out of c - T
__device__ __forceinline__ uint32_t planes_ge(const uint32_t (&c)[4], int T) {
  if (T <= 0) return 0xFFFFFFFFu;
  if (T > 15) return 0u;
  uint32_t b = 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) b = ((T >> j) & 1) ? (~c[j] | b) : (~c[j] & b);
  return ~b;
}

__global__ void __launch_bounds__(kVoteWarps * 32, 6)
k_vote_stage_sliced(WorkerPtrs signs, int M, int64_t nchunks, int tie_plus, VoteStage st) {
  griddep_wait();
  griddep_launch();
  __shared__ uint32_t lut[16];
  extern __shared__ __align__(16) uint8_t vsm[];   // [warp][2][kVoteBatch][512]
  if (threadIdx.x < 16) {
    // index bits 0, 1: entries 2k, 2k + 1 are +1; bits 2, 3: they are -1
    const uint32_t i = threadIdx.x;
    const uint32_t lo = (i & 1u) ? 0x3F80u : ((i & 4u) ? 0xBF80u : 0u);
    const uint32_t hi = (i & 2u) ? 0x3F80u : ((i & 8u) ? 0xBF80u : 0u);
    lut[i] = lo | (hi << 16);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t gw = (int64_t)blockIdx.x * kVoteWarps + wid;
  const int64_t nw = (int64_t)gridDim.x * kVoteWarps;
  const uint32_t buf0 = (uint32_t)__cvta_generic_to_shared(vsm) + (uint32_t)wid * (2 * kVoteBatch * kVoteTileB);
  const int nbatch = (M + kVoteBatch - 1) / kVoteBatch;
  const int TP = tie_plus ? (M + 1) / 2 : M / 2 + 1;   // c >= TP: the majority is +1
  const int TN = (M + 1) / 2;                           // c < TN: it is -1
  auto issue = [&](int64_t t, int bt, int buf) {
    const uint32_t dst = buf0 + (uint32_t)buf * (kVoteBatch * kVoteTileB) + (uint32_t)lane * 16;
    const int64_t boff = st.off[t].x >> 3;
    // a lane's 16 bytes hold entries 128 lane .. 128 lane + 127 of the chunk;
    // pieces wholly past a short chunk's end are not read
    const bool live = lane * 128 < st.chunks[t].len;
#pragma unroll
    for (int i = 0; i < kVoteBatch; ++i) {
      const int m = bt * kVoteBatch + i;
      if (m < M && live)
        cp_async16(dst + (uint32_t)i * kVoteTileB, reinterpret_cast<const uint8_t*>(signs.p[m]) + boff + lane * 16);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  int64_t tile = gw;
  int batch = 0;
  if (tile >= nchunks) return;
  issue(tile, 0, 0);
  int cur = 0;
  uint32_t c[4][4];   // [word][plane]
#pragma unroll
  for (int w = 0; w < 4; ++w)
#pragma unroll
    for (int j = 0; j < 4; ++j) c[w][j] = 0u;
  while (true) {
    int64_t ntile = tile;
    int nbt = batch + 1;
    if (nbt == nbatch) { nbt = 0; ntile += nw; }
    if (ntile < nchunks) {
      issue(ntile, nbt, cur ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncwarp();
    const uint32_t src = buf0 + (uint32_t)cur * (kVoteBatch * kVoteTileB);
    const int nm = min(kVoteBatch, M - batch * kVoteBatch);
    for (int i = 0; i < nm; ++i) {
      uint32_t v[4];
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                   : "r"(src + (uint32_t)i * kVoteTileB + (uint32_t)lane * 16));
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        // count += bit, in bit planes (counts stay below 16)
        const uint32_t t0 = c[w][0] & v[w];
        c[w][0] ^= v[w];
        const uint32_t t1 = c[w][1] & t0;
        c[w][1] ^= t0;
        const uint32_t t2 = c[w][2] & t1;
        c[w][2] ^= t1;
        c[w][3] ^= t2;
      }
    }
    __syncwarp();
    if (batch == nbatch - 1) {
      const longlong2 o = st.off[tile];
      const int len = st.chunks[tile].len;
      __nv_bfloat16* xo = st.X + o.y;
      uint32_t P[4], N[4];
      int nz = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int e0 = lane * 128 + w * 32;
        const uint32_t valid = e0 >= len ? 0u : (e0 + 32 <= len ? 0xFFFFFFFFu : ((1u << (len - e0)) - 1u));
        P[w] = planes_ge(c[w], TP) & valid;
        N[w] = ~planes_ge(c[w], TN) & valid;
        nz += __popc(P[w] | N[w]);
#pragma unroll
        for (int j = 0; j < 4; ++j) c[w][j] = 0u;
      }
      nz = __reduce_add_sync(0xffffffffu, nz);
      if (lane == 0) st.partials[tile] = (float)nz;
      // The bf16 values through the batch buffer just counted (32 rows of
      // 128 bytes, 16-byte units XOR-swizzled by row), in two halves of 64
      // entries per lane: lane t writes row t, then each store instruction
      // sends four whole rows (128 contiguous bytes each) to the chunk's X.
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {   // 8 entries = 16 bytes each
          const uint32_t p8 = (P[2 * hlf + u / 4] >> (8 * (u & 3))) & 0xFFu;
          const uint32_t n8 = (N[2 * hlf + u / 4] >> (8 * (u & 3))) & 0xFFu;
          uint32_t q[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) q[k] = lut[((p8 >> (2 * k)) & 3u) | (((n8 >> (2 * k)) & 3u) << 2)];
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(src + (uint32_t)(lane * 128 + ((u ^ (lane & 7)) * 16))),
                       "r"(q[0]), "r"(q[1]), "r"(q[2]), "r"(q[3])
                       : "memory");
        }
        __syncwarp();
#pragma unroll
        for (int jr = 0; jr < 8; ++jr) {
          const int row = 4 * jr + lane / 8, u = lane & 7;
          const int e = row * 128 + 64 * hlf + 8 * u;   // the unit's first entry in the chunk
          uint4 q;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(q.x), "=r"(q.y), "=r"(q.z), "=r"(q.w)
                       : "r"(src + (uint32_t)(row * 128 + ((u ^ (row & 7)) * 16)))
                       : "memory");
          if (e < len) *reinterpret_cast<uint4*>(xo + e) = q;   // len is a multiple of 8
        }
        __syncwarp();
      }
    }
    tile = ntile;
    batch = nbt;
    cur ^= 1;
    if (tile >= nchunks) break;
  }
}

// Majority of the packed signs staged straight into the Newton-Schulz input of
// the post-vote polar step ([paper] §4, orthogonalising the aggregated
// direction): per 4096-entry chunk of one matrix, the majority sgn(2c - M) of
// every entry goes to X (bf16 or fp32, grouped layout) and, when D is
// non-null, to D (fp32 flat); partials[chunk] gets the chunk's sum of
// squares (its non-zero count) for the Frobenius scale and the finite check.
__global__ void __launch_bounds__(kThreads)
k_vote_stage(WorkerPtrs signs, int M, void* __restrict__ X, int x_bf16,
             const Chunk* __restrict__ chunks, const MatInfo* __restrict__ mats,
             const GroupInfo* __restrict__ groups, float* __restrict__ partials, float* __restrict__ D, int tie_plus) {
  griddep_wait();
  griddep_launch();
  __shared__ float red[32];
  const Chunk ch = chunks[blockIdx.x];
  const MatInfo mi = mats[ch.mat];
  const GroupInfo gi = groups[mi.group];
  const int64_t base = mi.off + ch.start;
  // vector path: whole bytes of the bit streams, 8-entry runs inside a row
  const bool vec = ((base & 7) == 0) && ((ch.len & 7) == 0) && ((mi.cols & 7) == 0);
  const bool bf = x_bf16 != 0;
  const int64_t xb = gi.x_base + (int64_t)mi.q * gi.rows * gi.ld;
  float ss = 0.f;
  if (vec) {
    // 8 consecutive entries per thread and step: one byte of every worker's
    // stream, counted in two SWAR accumulators (byte lane i of lo / hi counts
    // entry i / i + 4)
    constexpr int kV = kChunk / (kThreads * 8);
    int64_t fe[kV];
    bool on[kV];
#pragma unroll
    for (int j = 0; j < kV; ++j) {
      const int e = (threadIdx.x + j * kThreads) * 8;
      on[j] = e < ch.len;
      fe[j] = base + e;
    }
    int cnt[kV][8];
#pragma unroll
    for (int j = 0; j < kV; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) cnt[j][i] = 0;
    // 8 workers' bytes are loaded before any is counted (one memory round
    // trip per 8 workers, not one per worker); counters flushed every 248
    uint32_t lo[kV], hi[kV];
#pragma unroll
    for (int j = 0; j < kV; ++j) lo[j] = hi[j] = 0;
    for (int m = 0; m < M; m += 8) {
      uint32_t by[8][kV];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint8_t* bm = (m + i < M) ? reinterpret_cast<const uint8_t*>(signs.p[m + i]) : nullptr;
#pragma unroll
        for (int j = 0; j < kV; ++j) by[i][j] = (m + i < M && on[j]) ? (uint32_t)bm[fe[j] >> 3] : 0u;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < kV; ++j) {
          lo[j] += ((by[i][j] & 0xFu) * 0x00204081u) & 0x01010101u;
          hi[j] += ((by[i][j] >> 4) * 0x00204081u) & 0x01010101u;
        }
      if (((m + 8) % 248) == 0 || m + 8 >= M) {
#pragma unroll
        for (int j = 0; j < kV; ++j) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            cnt[j][i] += (lo[j] >> (8 * i)) & 0xFF;
            cnt[j][i + 4] += (hi[j] >> (8 * i)) & 0xFF;
          }
          lo[j] = hi[j] = 0;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kV; ++j) {
      if (!on[j]) continue;
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] = (float)vmaj(2 * cnt[j][i] - M, tie_plus);
        ss += v[i] * v[i];
      }
      const float4 v0 = make_float4(v[0], v[1], v[2], v[3]), v1 = make_float4(v[4], v[5], v[6], v[7]);
      if (D != nullptr) {
        st4(D + fe[j], v0);
        st4(D + fe[j] + 4, v1);
      }
      const int le = (int)(fe[j] - mi.off);
      const int r = le / mi.cols, c = le - r * mi.cols;
      store_x4(X, xb + (int64_t)r * gi.ld + c, v0, bf);
      store_x4(X, xb + (int64_t)r * gi.ld + c + 4, v1, bf);
    }
  } else {
    for (int e = threadIdx.x; e < ch.len; e += kThreads) {
      const int64_t fe = base + e;
      int c = 0;
      for (int m = 0; m < M; ++m) c += (reinterpret_cast<const uint8_t*>(signs.p[m])[fe >> 3] >> (fe & 7)) & 1;
      const float v = (float)vmaj(2 * c - M, tie_plus);
      ss += v * v;
      if (D != nullptr) D[fe] = v;
      const int le = (int)(ch.start + e);
      const int r = le / mi.cols, cc = le - r * mi.cols;
      store_x(X, xb + (int64_t)r * gi.ld + cc, v, bf);
    }
  }
  const float t = block_sum<float>(ss, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = t;
}

// Muon baseline ([paper] §4 Muon update, Table 1): the mean of the M
// workers' momenta (summed in worker order in fp32, times 1/M) staged into
// the Newton-Schulz input of one problem set, with its sum-of-squares
// partials; the fp32 mean also goes to D when non-null (K == 0).
__global__ void __launch_bounds__(kThreads)
k_mean_stage(const float* __restrict__ Mom, int64_t mom_stride, int M, void* __restrict__ X, int x_bf16,
             const Chunk* __restrict__ chunks, const MatInfo* __restrict__ mats,
             const GroupInfo* __restrict__ groups, float* __restrict__ partials, float* __restrict__ D) {
  griddep_wait();
  griddep_launch();
  __shared__ float red[32];
  const Chunk ch = chunks[blockIdx.x];
  const MatInfo mi = mats[ch.mat];
  const GroupInfo gi = groups[mi.group];
  const int64_t base = mi.off + ch.start;
  const bool vec = ((base & 3) == 0) && ((ch.len & 3) == 0) && ((mi.cols & 3) == 0);
  const bool bf = x_bf16 != 0;
  const int64_t xb = gi.x_base + (int64_t)mi.q * gi.rows * gi.ld;
  const float inv = 1.f / (float)M;
  float ss = 0.f;
  if (vec) {
    for (int e = threadIdx.x * 4; e < ch.len; e += kThreads * 4) {
      const int64_t fe = base + e;
      float4 acc = ld4(Mom + fe);
      for (int m = 1; m < M; ++m) {
        const float4 v = ld4(Mom + (int64_t)m * mom_stride + fe);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
      ss += acc.x * acc.x + acc.y * acc.y + acc.z * acc.z + acc.w * acc.w;
      if (D != nullptr) st4(D + fe, acc);
      const int le = (int)(ch.start + e);
      const int r = le / mi.cols, c = le - r * mi.cols;
      store_x4(X, xb + (int64_t)r * gi.ld + c, acc, bf);
    }
  } else {
    for (int e = threadIdx.x; e < ch.len; e += kThreads) {
      const int64_t fe = base + e;
      float acc = Mom[fe];
      for (int m = 1; m < M; ++m) acc += Mom[(int64_t)m * mom_stride + fe];
      acc *= inv;
      ss += acc * acc;
      if (D != nullptr) D[fe] = acc;
      const int le = (int)(ch.start + e);
      const int r = le / mi.cols, c = le - r * mi.cols;
      store_x(X, xb + (int64_t)r * gi.ld + c, acc, bf);
    }
  }
  const float t = block_sum<float>(ss, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = t;
}

// W <- fl32(W - eta D), one rounding ([paper] Algorithm 1/2 update).
__global__ void __launch_bounds__(kThreads)
k_update(float* __restrict__ W, const float* __restrict__ D, int64_t d, float eta,
         const int* __restrict__ status) {
  griddep_wait();
  griddep_launch();
  if (status != nullptr && (status[0] | status[1]) != 0) return;  // keep W on error
  const int64_t n4 = d >> 2;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n4; i += stride) {
    float4 w = ld4(W + 4 * i);
    const float4 dd = ld4(D + 4 * i);
    w.x = fmaf(-eta, dd.x, w.x);
    w.y = fmaf(-eta, dd.y, w.y);
    w.z = fmaf(-eta, dd.z, w.z);
    w.w = fmaf(-eta, dd.w, w.w);
    st4(W + 4 * i, w);
  }
  if (blockIdx.x == 0)
    for (int64_t e = 4 * n4 + threadIdx.x; e < d; e += kThreads) W[e] = fmaf(-eta, D[e], W[e]);
}

int g_num_sms = 0;

}  // namespace

int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

int resident_per_sm(const void* kernel, int threads, size_t smem) {
  // looked up once per (kernel, block shape); launches come from one host
  // thread per handle, but handles may live on several threads
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, size_t>, int> cache;
  const auto key = std::make_tuple(kernel, threads, smem);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = 1;
  }
  cache[key] = n;
  return n;
}

int stream_grid(const void* kernel, int threads, size_t smem, int64_t work_items, int per_sm) {
  const int fit = resident_per_sm(kernel, threads, smem);
  const int64_t cap = (int64_t)num_sms() * (per_sm < fit ? per_sm : fit);
  if (work_items < 1) return 1;
  return (int)(work_items < cap ? work_items : cap);
}

// ---- launch wrappers --------------------------------------------------------

void launch_momentum(cudaStream_t s, const WorkerPtrs& G, const float* W, float* Mom, int64_t d,
                     int M, float beta, float lambda, void* X, int x_bf16, const Chunk* chunks,
                     int n_chunks, const MatInfo* mats, const GroupInfo* groups, float* partials) {
  if (n_chunks <= 0) return;
  count_launch();
  launch_pdl(k_momentum<true>, dim3(n_chunks), dim3(kThreads), 0, s, G, W, Mom, d, M, beta, lambda, X, x_bf16, chunks,
                                                 mats, groups, partials);
}

void launch_stage(cudaStream_t s, const WorkerPtrs& in, int M, void* X, int x_bf16,
                  const Chunk* chunks, int n_chunks, const MatInfo* mats, const GroupInfo* groups,
                  float* partials) {
  if (n_chunks <= 0) return;
  count_launch();
  launch_pdl(k_momentum<false>, dim3(n_chunks), dim3(kThreads), 0, s, in, nullptr, nullptr, 0, M, 0.f, 0.f, X, x_bf16,
                                                  chunks, mats, groups, partials);
}

void launch_fro_finalize(cudaStream_t s, int n_probs, int n_mats, int M, const float* partials,
                         const int* mat_chunk0, const int* mat_nchunks, int use_for_scale,
                         float eps, int quintic, float a, float b, float c, float* scale,
                         float2* coef_apply, float2* coef_square, float2* coef_gram, int* status) {
  count_launch();
  launch_pdl(k_fro_finalize, dim3(n_probs), dim3(kThreads), 0, s, n_mats, M, partials, mat_chunk0, mat_nchunks,
             use_for_scale, eps, quintic, a, b, c, scale, coef_apply, coef_square, coef_gram, status);
}

// Gram space: Q1 = alpha I + beta A~ per problem, (alpha, beta) = coef[p]
// (the cubic iteration 0's apply coefficients, a cc and b cc^3), over the
// whole g x gld rows of each problem's m x m buffer.  8 bf16 per thread.
__global__ void __launch_bounds__(kThreads)
k_gram_q1(const __nv_bfloat16* __restrict__ A, __nv_bfloat16* __restrict__ Q, const int64_t* __restrict__ prob_aoff,
          const int* __restrict__ prob_g, const int* __restrict__ prob_gld, const float2* __restrict__ coef) {
  griddep_wait();
  griddep_launch();
  const int p = blockIdx.y;
  const int g = prob_g[p], gld = prob_gld[p];
  const int64_t base = prob_aoff[p];
  const float2 cf = coef[p];
  const int64_t n8 = (int64_t)g * gld / 8;   // gld is a multiple of 8
  for (int64_t v = (int64_t)blockIdx.x * kThreads + threadIdx.x; v < n8; v += (int64_t)gridDim.x * kThreads) {
    const int64_t e = 8 * v;
    const int r = (int)(e / gld), c0 = (int)(e - (int64_t)r * gld);
    const uint4 raw = *reinterpret_cast<const uint4*>(A + base + e);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint4 out;
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 f = __bfloat1622float2(h[t]);
      float x = cf.y * f.x, y = cf.y * f.y;
      if (c0 + 2 * t == r) x += cf.x;
      if (c0 + 2 * t + 1 == r) y += cf.x;
      const __nv_bfloat162 q = __floats2bfloat162_rn(x, y);
      o[t] = *reinterpret_cast<const uint32_t*>(&q);
    }
    *reinterpret_cast<uint4*>(Q + base + e) = out;
  }
}

void launch_gram_q1(cudaStream_t s, int n_probs, const void* A, void* Q, const int64_t* prob_aoff,
                    const int* prob_g, const int* prob_gld, const float2* coef, int max_g, int max_gld) {
  if (n_probs <= 0) return;
  count_launch();
  const int64_t n8 = (int64_t)max_g * max_gld / 8;
  const int bx = (int)std::min<int64_t>((n8 + kThreads - 1) / kThreads, 64);
  launch_pdl(k_gram_q1, dim3(bx, n_probs), dim3(kThreads), 0, s, reinterpret_cast<const __nv_bfloat16*>(A),
             reinterpret_cast<__nv_bfloat16*>(Q), prob_aoff, prob_g, prob_gld, coef);
}

void launch_pi_init(cudaStream_t s, int n_probs, const int64_t* uoff, const int* prob_g, float* u, int warm) {
  count_launch();
  launch_pdl(k_pi_init, dim3(n_probs), dim3(kThreads), 0, s, uoff, prob_g, u, warm);
}

void launch_pi_tiles(cudaStream_t s, const PiTile* tiles, int n_tiles, const void* A, int a_bf16,
                     const float* src, const float* inv, float* u, float* part, int fold) {
  if (n_tiles <= 0) return;
  count_launch();
  if (a_bf16) {
    const size_t smem = (size_t)PiLane<true>::TILEB;
    launch_pdl(k_pi_tiles<true>, dim3(n_tiles), dim3(kThreads), smem, s, tiles, A, src, inv, u, part, fold);
  } else {
    // 64 KB of dynamic shared memory needs the opt-in (per device)
    const size_t smem = (size_t)PiLane<false>::TILEB;
    cudaFuncSetAttribute(k_pi_tiles<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_pdl(k_pi_tiles<false>, dim3(n_tiles), dim3(kThreads), smem, s, tiles, A, src, inv, u, part, fold);
  }
}

void launch_pi_reduce(cudaStream_t s, const PiSlice* slices, int n_slices, const float* part, float* y,
                      const PiReduce& r) {
  if (n_slices <= 0) return;
  count_launch();
  launch_pdl(k_pi_reduce, dim3(n_slices), dim3(kPiTile), 0, s, slices, part, y, r);
}

void launch_scale_flat(cudaStream_t s, const WorkerPtrs& in, int M, float* out, int64_t out_stride,
                       const Chunk* chunks, int n_chunks, const MatInfo* mats, int n_mats,
                       const float* scale, float eps) {
  if (n_chunks <= 0) return;
  count_launch();
  dim3 grid(n_chunks, M);
  launch_pdl(k_scale_flat, dim3(grid), dim3(kThreads), 0, s, in, out, out_stride, chunks, mats, n_mats, scale, eps);
}

void launch_pack(cudaStream_t s, const float* U, int64_t u_stride, int64_t d, uint8_t* out,
                 int64_t out_stride, int M) {
  if (d <= 0) return;
  count_launch();
  const int64_t warps = (d + 1023) / 1024;
  const int blocks = stream_grid((const void*)k_pack, kThreads, 0, (warps + 7) / 8, 16);
  dim3 grid(blocks, M);
  launch_pdl(k_pack, dim3(grid), dim3(kThreads), 0, s, U, u_stride, d, out, out_stride);
}

// Full 4096-entry tiles by the streaming kernel (M <= 255), the rest (and
// every entry for larger M) by the register kernel on offset pointers.
// Worker m's packed signs start at signs.p[m] (16-byte aligned), which may
// be this GPU's memory or a peer's mapped over NVLink.
template <int MODE, bool ACC8>
void vote_dispatch(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, void* sums, int8_t* maj, float* W,
                   float eta, float* D, const int* status, int tie_plus) {
  int64_t done = 0;
  if (M <= 255 && d >= 4096) {
    const int64_t ntiles = d / 4096;
    const size_t smem = (size_t)kVoteWarps * 2 * kVoteBatch * kVoteTileB;
    const int blocks = stream_grid((const void*)k_vote_stream<MODE, ACC8>, kVoteWarps * 32, smem,
                                   (ntiles + kVoteWarps - 1) / kVoteWarps, 8);
    count_launch();
    launch_pdl(k_vote_stream<MODE, ACC8>, dim3(blocks), dim3(kVoteWarps * 32), smem, s, signs, M, ntiles, sums, maj,
               W, eta, D, status, tie_plus, VoteStage{});
    done = ntiles * 4096;
  }
  const int64_t rest = d - done;
  if (rest <= 0) return;
  const int64_t boff = done / 8;  // byte offset in every stream (a multiple of 512)
  WorkerPtrs sp = signs;
  for (int m = 0; m < M; ++m) sp.p[m] = reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(signs.p[m]) + boff);
  void* sums2 = sums == nullptr ? nullptr : reinterpret_cast<uint8_t*>(sums) + done * (ACC8 ? 1 : 4);
  count_launch();
  const int blocks = stream_grid((const void*)k_vote<MODE, ACC8>, kThreads, 0, (rest / 512 + 8) / 8 + 1, 8);
  launch_pdl(k_vote<MODE, ACC8>, dim3(blocks), dim3(kThreads), 0, s, sp, M, rest, sums2,
             maj == nullptr ? nullptr : maj + done, W == nullptr ? nullptr : W + done, eta,
             D == nullptr ? nullptr : D + done, status, tie_plus);
}

void launch_vote(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, void* sums, int acc8,
                 int8_t* majority, int tie_plus) {
  if (d <= 0) return;
  if (acc8) vote_dispatch<0, true>(s, signs, M, d, sums, majority, nullptr, 0.f, nullptr, nullptr, tie_plus);
  else vote_dispatch<0, false>(s, signs, M, d, sums, majority, nullptr, 0.f, nullptr, nullptr, tie_plus);
}

void launch_vote_update(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, float* W, float eta,
                        const int* status, int tie_plus) {
  if (d <= 0) return;
  vote_dispatch<1, false>(s, signs, M, d, nullptr, nullptr, W, eta, nullptr, status, tie_plus);
}

void launch_vote_major(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, float* D, int tie_plus) {
  if (d <= 0) return;
  vote_dispatch<2, false>(s, signs, M, d, nullptr, nullptr, nullptr, 0.f, D, nullptr, tie_plus);
}

void launch_vote_stage(cudaStream_t s, const WorkerPtrs& signs, int M, void* X, int x_bf16,
                       const Chunk* chunks, int n_chunks, const MatInfo* mats, const GroupInfo* groups,
                       float* partials, float* D, int tie_plus, const int64_t* stage_off) {
  if (n_chunks <= 0) return;
  count_launch();
  if (stage_off != nullptr && x_bf16 && M <= 255) {
    // one warp per chunk, the next chunk's bytes in flight while one is counted
    const size_t smem = (size_t)kVoteWarps * 2 * kVoteBatch * kVoteTileB;
    const VoteStage st{reinterpret_cast<__nv_bfloat16*>(X), chunks, reinterpret_cast<const longlong2*>(stage_off),
                       partials};
    const int64_t warps = ((int64_t)n_chunks + kVoteWarps - 1) / kVoteWarps;
    if (D == nullptr && M <= kVoteSlicedMaxM) {
      const int blocks = stream_grid((const void*)k_vote_stage_sliced, kVoteWarps * 32, smem, warps, 8);
      launch_pdl(k_vote_stage_sliced, dim3(blocks), dim3(kVoteWarps * 32), smem, s, signs, M, (int64_t)n_chunks,
                 tie_plus, st);
    } else if (D == nullptr) {
      const int blocks = stream_grid((const void*)k_vote_stream<3, false>, kVoteWarps * 32, smem, warps, 8);
      launch_pdl(k_vote_stream<3, false>, dim3(blocks), dim3(kVoteWarps * 32), smem, s, signs, M, (int64_t)n_chunks,
                 nullptr, nullptr, nullptr, 0.f, nullptr, nullptr, tie_plus, st);
    } else {
      const int blocks = stream_grid((const void*)k_vote_stream<4, false>, kVoteWarps * 32, smem, warps, 8);
      launch_pdl(k_vote_stream<4, false>, dim3(blocks), dim3(kVoteWarps * 32), smem, s, signs, M, (int64_t)n_chunks,
                 nullptr, nullptr, nullptr, 0.f, D, nullptr, tie_plus, st);
    }
    return;
  }
  launch_pdl(k_vote_stage, dim3(n_chunks), dim3(kThreads), 0, s, signs, M, X, x_bf16, chunks, mats, groups, partials,
             D, tie_plus);
}

void launch_mean_stage(cudaStream_t s, const float* Mom, int64_t mom_stride, int M, void* X, int x_bf16,
                       const Chunk* chunks, int n_chunks, const MatInfo* mats, const GroupInfo* groups,
                       float* partials, float* D) {
  if (n_chunks <= 0) return;
  count_launch();
  launch_pdl(k_mean_stage, dim3(n_chunks), dim3(kThreads), 0, s, Mom, mom_stride, M, X, x_bf16, chunks, mats, groups, partials, D);
}

void launch_update(cudaStream_t s, float* W, const float* D, int64_t d, float eta,
                   const int* status) {
  if (d <= 0) return;
  count_launch();
  const int blocks = stream_grid((const void*)k_update, kThreads, 0, (d / 4 + kThreads - 1) / kThreads + 1, 8);
  launch_pdl(k_update, dim3(blocks), dim3(kThreads), 0, s, W, D, d, eta, status);
}

}  // namespace sm
