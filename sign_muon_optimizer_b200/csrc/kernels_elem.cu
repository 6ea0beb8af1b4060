// kernels_elem.cu -- the HBM-bound kernels of the Sign-Muon step:
//   momentum pass (weight decay + momentum + X staging + Frobenius partials),
//   scale finalisation, power iteration on the Gram matrix, one-bit pack,
//   majority vote (API form, fused with the update, or emitting D), update.
//
// Sources, by page title:
//   [paper] "SignMuon: 通信高效的分布式Muon优化" (a rendering of arXiv 2605.16311)
//   [blog]  "SignMuon: Matrix Directions, Majority Votes, and the Actual Bytes Sent"
#include "common.cuh"

#include <cmath>

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
                                          float2* coef_apply, float2* coef_square) {
  // Iteration 0 runs on the unscaled X~ and Gram A~ = X~ X~^T.  With X0 = cc X~:
  //   cubic:   X1 = a cc X~ + b cc^3 A~ X~
  //   quintic: B = b cc^2 A~ + c cc^4 A~^2;  X1 = cc (a X~ + B X~)
  if (!quintic) {
    coef_apply[p] = make_float2(a * cc, b * cc * cc * cc);
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
               float2* coef_square, int* status) {
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
      set_coefs(p, 1.f / (sc + eps), quintic, a, b, c, coef_apply, coef_square);
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

template <bool BF16>
__global__ void __launch_bounds__(kThreads)
k_pi_matvec(const ProbRows* __restrict__ rows, const void* __restrict__ A,
            const int64_t* __restrict__ prob_a_off, const int* __restrict__ prob_g,
            const int* __restrict__ prob_gld, const int64_t* __restrict__ uoff,
            const float* __restrict__ u, float* __restrict__ y) {
  griddep_wait();
  griddep_launch();
  // y[r] = sum_k A[r][k] u[k] for the block's kPiRows rows of one problem.
  // u is staged in shared memory; each warp streams kRowsPerWarp rows at
  // once (one 16-byte load per row and lane in flight per step) so that the
  // HBM stream of A has enough loads in flight.
  extern __shared__ float us[];
  const ProbRows pr = rows[blockIdx.x];
  const int p = pr.p;
  const int g = prob_g[p], gld = prob_gld[p];
  const float* up = u + uoff[p];
  for (int k = threadIdx.x; k < g; k += kThreads) us[k] = up[k];
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  constexpr int R = kPiRows / (kThreads / 32);
  const int r0 = pr.row0 + wid * R;
  float acc[R];
#pragma unroll
  for (int j = 0; j < R; ++j) acc[j] = 0.f;
  if (BF16) {
    const __nv_bfloat16* a0 = reinterpret_cast<const __nv_bfloat16*>(A) + prob_a_off[p] + (int64_t)r0 * gld;
    const int g8 = g & ~7;
    for (int k = lane * 8; k < g8; k += 256) {
      uint4 raw[R];
#pragma unroll
      for (int j = 0; j < R; ++j)
        raw[j] = (r0 + j < g) ? __ldcs(reinterpret_cast<const uint4*>(a0 + (int64_t)j * gld + k)) : make_uint4(0, 0, 0, 0);
      const float4 u0 = *reinterpret_cast<const float4*>(us + k);
      const float4 u1 = *reinterpret_cast<const float4*>(us + k + 4);
      const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[j]);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 f = __bfloat1622float2(h[t]);
          acc[j] = fmaf(f.x, uv[2 * t], acc[j]);
          acc[j] = fmaf(f.y, uv[2 * t + 1], acc[j]);
        }
      }
    }
    for (int k = g8 + lane; k < g; k += 32) {
#pragma unroll
      for (int j = 0; j < R; ++j)
        if (r0 + j < g) acc[j] = fmaf(__bfloat162float(a0[(int64_t)j * gld + k]), us[k], acc[j]);
    }
  } else {
    const float* a0 = reinterpret_cast<const float*>(A) + prob_a_off[p] + (int64_t)r0 * gld;
    const int g4 = g & ~3;
    for (int k = lane * 4; k < g4; k += 128) {
      float4 f[R];
#pragma unroll
      for (int j = 0; j < R; ++j)
        f[j] = (r0 + j < g) ? __ldcs(reinterpret_cast<const float4*>(a0 + (int64_t)j * gld + k)) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 uv = *reinterpret_cast<const float4*>(us + k);
#pragma unroll
      for (int j = 0; j < R; ++j) {
        acc[j] = fmaf(f[j].x, uv.x, acc[j]);
        acc[j] = fmaf(f[j].y, uv.y, acc[j]);
        acc[j] = fmaf(f[j].z, uv.z, acc[j]);
        acc[j] = fmaf(f[j].w, uv.w, acc[j]);
      }
    }
    for (int k = g4 + lane; k < g; k += 32) {
#pragma unroll
      for (int j = 0; j < R; ++j)
        if (r0 + j < g) acc[j] = fmaf(a0[(int64_t)j * gld + k], us[k], acc[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < R; ++j) {
    const float v = warp_sum(acc[j]);
    if (lane == 0 && r0 + j < g) y[uoff[p] + r0 + j] = v;
  }
}

__global__ void __launch_bounds__(kThreads)
k_pi_normalize(const int64_t* __restrict__ uoff, const int* __restrict__ prob_g,
               const float* __restrict__ y, float* __restrict__ u) {
  griddep_wait();
  griddep_launch();
  __shared__ double red[32];
  __shared__ float inv;
  const int p = blockIdx.x;
  const int g = prob_g[p];
  const float* yp = y + uoff[p];
  double s = 0.0;
  for (int k = threadIdx.x; k < g; k += kThreads) s += (double)yp[k] * (double)yp[k];
  const double t = block_sum<double>(s, red);
  if (threadIdx.x == 0) inv = (t > 0.0) ? (float)(1.0 / sqrt(t)) : 0.f;  // a zero iterate stays zero
  __syncthreads();
  for (int k = threadIdx.x; k < g; k += kThreads) u[uoff[p] + k] = yp[k] * inv;
}

__global__ void __launch_bounds__(kThreads)
k_pi_finalize(const int64_t* __restrict__ uoff, const int* __restrict__ prob_g,
              const float* __restrict__ u, const float* __restrict__ y, float eps, int quintic,
              float a, float b, float c, float* __restrict__ scale, float2* coef_apply,
              float2* coef_square, int* status) {
  griddep_wait();
  griddep_launch();
  __shared__ double red[32];
  const int p = blockIdx.x;
  const int g = prob_g[p];
  double s = 0.0;
  for (int k = threadIdx.x; k < g; k += kThreads) s += (double)u[uoff[p] + k] * (double)y[uoff[p] + k];
  const double t = block_sum<double>(s, red);
  if (threadIdx.x == 0) {
    const float sc = (float)sqrt(fmax(t, 0.0));
    if (!isfinite(t)) atomicOr(status, 1);
    scale[p] = sc;
    set_coefs(p, 1.f / (sc + eps), quintic, a, b, c, coef_apply, coef_square);
  }
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// MODE 3 (staging of the post-vote polar step's input): the work items are
// the plan's chunks instead of flat tiles.  Chunk c covers entries base ..
// base + len - 1 of the flat vector (base = its matrix's offset + its start,
// a multiple of 128; len <= 4096); its majorities go to the bf16 X of the
// one-problem-set Newton-Schulz input, which for a matrix with a multiple of
// 8 columns is the chunk's contiguous range starting at xb + start, and
// partials[c] receives the chunk's count of non-zero majorities (its sum of
// squares).
struct VoteStage {
  __nv_bfloat16* X;
  const Chunk* chunks;
  const MatInfo* mats;
  const GroupInfo* groups;
  float* partials;
};

template <int MODE, bool ACC8>
__global__ void __launch_bounds__(kVoteWarps * 32)
k_vote_stream(WorkerPtrs signs, int M, int64_t ntiles,
              void* __restrict__ sums, int8_t* __restrict__ maj, float* __restrict__ W, float eta,
              float* __restrict__ D, const int* __restrict__ status, int tie_plus, VoteStage st) {
  griddep_wait();
  griddep_launch();
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
    if (MODE == 3) {
      const Chunk c = st.chunks[t];
      return st.mats[c.mat].off + c.start;
    }
    return t * 4096;
  };
  auto item_len = [&](int64_t t) -> int { return MODE == 3 ? st.chunks[t].len : 4096; };
  auto issue = [&](int64_t t, int bt, int buf) {
    const uint32_t dst = buf0 + (uint32_t)buf * (kVoteBatch * kVoteTileB) + (uint32_t)lane * 16;
    const int64_t boff = item_base(t) >> 3;
    // a lane's 16 bytes hold entries 128 lane .. 128 lane + 127 of the item;
    // pieces wholly past a short chunk's end are not read
    const bool live = MODE != 3 || lane * 128 < item_len(t);
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
    if (batch == nbatch - 1 && MODE == 3) {
      // chunk done: its majorities into X (4 bf16 per lane and step, so each
      // warp store writes 256 contiguous bytes) and D, its non-zero count
      const Chunk ch = st.chunks[tile];
      const MatInfo mi = st.mats[ch.mat];
      const GroupInfo gi = st.groups[mi.group];
      __nv_bfloat16* xo = st.X + gi.x_base + (int64_t)mi.q * gi.rows * gi.ld + ch.start;
      const int64_t fb = mi.off + ch.start;
      int nz = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int e = j * 128 + lane * 4;
        if (e < ch.len) {
          // the four majorities as int8 byte lanes (0x01, 0xFF or 0), then as
          // bf16 pairs: +1 = 0x3F80, -1 = 0xBF80, 0 = 0 (sign at bit 15 of a half)
          const uint32_t mj = swar_majority(acc[j], M, tie_plus);
          const uint32_t nzb = (mj | (mj << 7)) & 0x80808080u;    // bit 7 of a non-zero byte
          const uint32_t sgn = mj & 0x80808080u;                  // bit 7 of a -1 byte
          nz += __popc(nzb);
          uint2 u;
          u.x = ((__byte_perm(nzb, 0, 0x1404) >> 15) * 0xFFFFu & 0x3F803F80u) | __byte_perm(sgn, 0, 0x1404);
          u.y = ((__byte_perm(nzb, 0, 0x3424) >> 15) * 0xFFFFu & 0x3F803F80u) | __byte_perm(sgn, 0, 0x3424);
          *reinterpret_cast<uint2*>(xo + e) = u;
          if (D != nullptr) {
            const int c0 = acc[j] & 0xFF, c1 = (acc[j] >> 8) & 0xFF, c2 = (acc[j] >> 16) & 0xFF, c3 = acc[j] >> 24;
            st4(D + fb + e, make_float4((float)vmaj(2 * c0 - M, tie_plus), (float)vmaj(2 * c1 - M, tie_plus),
                                        (float)vmaj(2 * c2 - M, tie_plus), (float)vmaj(2 * c3 - M, tie_plus)));
          }
        }
      }
      nz = __reduce_add_sync(0xffffffffu, nz);
      if (lane == 0) st.partials[tile] = (float)nz;
    } else if (batch == nbatch - 1) {
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

int stream_grid(int64_t work_items, int per_sm) {
  const int64_t cap = (int64_t)num_sms() * per_sm;
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
                         float2* coef_apply, float2* coef_square, int* status) {
  count_launch();
  launch_pdl(k_fro_finalize, dim3(n_probs), dim3(kThreads), 0, s, n_mats, M, partials, mat_chunk0, mat_nchunks,
                                              use_for_scale, eps, quintic, a, b, c, scale,
                                              coef_apply, coef_square, status);
}

void launch_pi_init(cudaStream_t s, int n_probs, const int64_t* uoff, const int* prob_g, float* u, int warm) {
  count_launch();
  launch_pdl(k_pi_init, dim3(n_probs), dim3(kThreads), 0, s, uoff, prob_g, u, warm);
}

void launch_pi_matvec(cudaStream_t s, const ProbRows* rows, int n_rows, const void* A, int a_bf16,
                      const int64_t* prob_a_off, const int* prob_g, const int* prob_gld,
                      const int64_t* uoff, const float* u, float* y, int max_g) {
  count_launch();
  const size_t smem = (size_t)max_g * sizeof(float);
  if (a_bf16) {
    if (smem > 48 * 1024) cudaFuncSetAttribute(k_pi_matvec<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_pdl(k_pi_matvec<true>, dim3(n_rows), dim3(kThreads), smem, s, rows, A, prob_a_off, prob_g, prob_gld, uoff, u, y);
  } else {
    if (smem > 48 * 1024) cudaFuncSetAttribute(k_pi_matvec<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_pdl(k_pi_matvec<false>, dim3(n_rows), dim3(kThreads), smem, s, rows, A, prob_a_off, prob_g, prob_gld, uoff, u, y);
  }
}

void launch_pi_normalize(cudaStream_t s, int n_probs, const int64_t* uoff, const int* prob_g,
                         const float* y, float* u) {
  count_launch();
  launch_pdl(k_pi_normalize, dim3(n_probs), dim3(kThreads), 0, s, uoff, prob_g, y, u);
}

void launch_pi_finalize(cudaStream_t s, int n_probs, const int64_t* uoff, const int* prob_g,
                        const float* u, const float* y, float eps, int quintic, float a, float b,
                        float c, float* scale, float2* coef_apply, float2* coef_square, int* status) {
  count_launch();
  launch_pdl(k_pi_finalize, dim3(n_probs), dim3(kThreads), 0, s, uoff, prob_g, u, y, eps, quintic, a, b, c, scale,
                                             coef_apply, coef_square, status);
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
  const int blocks = stream_grid((warps + 7) / 8, 16);
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
    const int64_t want = (ntiles + kVoteWarps - 1) / kVoteWarps;
    const int64_t cap = (int64_t)num_sms() * 6;
    const int blocks = (int)(want < cap ? want : cap);
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
  const int blocks = stream_grid((rest / 512 + 8) / 8 + 1, 8);
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
                       float* partials, float* D, int tie_plus, int streamable) {
  if (n_chunks <= 0) return;
  count_launch();
  if (streamable && x_bf16 && M <= 255) {
    // one warp per chunk, the next chunk's bytes in flight while one is counted
    const size_t smem = (size_t)kVoteWarps * 2 * kVoteBatch * kVoteTileB;
    const int64_t want = ((int64_t)n_chunks + kVoteWarps - 1) / kVoteWarps;
    const int64_t cap = (int64_t)num_sms() * 6;
    const int blocks = (int)(want < cap ? want : cap);
    const VoteStage st{reinterpret_cast<__nv_bfloat16*>(X), chunks, mats, groups, partials};
    launch_pdl(k_vote_stream<3, false>, dim3(blocks), dim3(kVoteWarps * 32), smem, s, signs, M, (int64_t)n_chunks,
               nullptr, nullptr, nullptr, 0.f, D, nullptr, tie_plus, st);
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
  const int blocks = stream_grid((d / 4 + kThreads - 1) / kThreads + 1, 8);
  launch_pdl(k_update, dim3(blocks), dim3(kThreads), 0, s, W, D, d, eta, status);
}

}  // namespace sm
