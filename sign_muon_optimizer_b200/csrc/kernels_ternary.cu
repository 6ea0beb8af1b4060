// kernels_ternary.cu -- the int8 ternary sign wire: sign(U) in {-1, 0, +1},
// one byte per entry and worker, and the majority vote over M such buffers
// (API form with int32 or int8 sums, fused with the update, or emitting D);
// and the majority of integer vote sums that arrive already added up (the
// SUM all-reduce of the workers' signs).
//
// Sources, by page title:
//   [paper] "SignMuon: 通信高效的分布式Muon优化" (a rendering of arXiv 2605.16311):
//           §3 defines sign(0) = 0; Algorithm 2 sums the workers' signs with one
//           int8 SUM all-reduce whose payload is d bytes per worker.
//   [blog]  "SignMuon: Matrix Directions, Majority Votes, and the Actual Bytes
//           Sent": the worked vote on ternary signs, ties giving 0.
#include "common.cuh"

namespace sm {

namespace {

constexpr int kTThreads = 256;

// sign with sign(0) = sign(-0) = 0; NaN compares false both ways and gives 0
__device__ __forceinline__ int tsign(float v) { return (v > 0.f) - (v < 0.f); }

// majority of a vote sum: sign(s), a tie giving 0 (or +1 with tie_plus)
__device__ __forceinline__ int tmaj(int s, int tie_plus) {
  return tie_plus ? (s >= 0 ? 1 : -1) : ((s > 0) - (s < 0));
}

// signed value of byte lane b of w
__device__ __forceinline__ int sbyte(uint32_t w, int b) { return (int)(w << (24 - 8 * b)) >> 24; }

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
         ((uint32_t)(d & 0xFF) << 24);
}

// ---------------------------------------------------------------------------
// Ternary sign of M flat fp32 vectors: worker w = blockIdx.y reads
// U + w*u_stride and writes out + w*out_stride.  A thread takes 16
// consecutive entries per step (four float4 loads, one 16-byte store); the
// d % 16 tail goes entry by entry in the last block of each worker.
// Host-checked layout: U and out 16-byte aligned, u_stride a multiple of 4
// floats, out_stride a multiple of 16 bytes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kTThreads)
k_sign8(const float* __restrict__ U, int64_t u_stride, int64_t d, int8_t* __restrict__ out, int64_t out_stride) {
  griddep_wait();
  griddep_launch();
  const int w = blockIdx.y;
  U += (int64_t)w * u_stride;
  out += (int64_t)w * out_stride;
  const int64_t n16 = d >> 4;
  const int64_t stride = (int64_t)gridDim.x * kTThreads;
  for (int64_t i = (int64_t)blockIdx.x * kTThreads + threadIdx.x; i < n16; i += stride) {
    const float4* src = reinterpret_cast<const float4*>(U + 16 * i);
    uint32_t word[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = __ldcs(src + q);
      word[q] = pack4(tsign(v.x), tsign(v.y), tsign(v.z), tsign(v.w));
    }
    *reinterpret_cast<uint4*>(out + 16 * i) = make_uint4(word[0], word[1], word[2], word[3]);
  }
  if (blockIdx.x == gridDim.x - 1)
    for (int64_t e = 16 * n16 + threadIdx.x; e < d; e += kTThreads) out[e] = (int8_t)tsign(U[e]);
}

// ---------------------------------------------------------------------------
// Majority vote over M int8 ternary buffers.
// MODE 0: API vote (sums int32 or int8, majority int8; either may be null);
// MODE 1: fused update W <- fl32(W - eta*maj) (skipped when the step's status
//         is set, so that W stays unchanged on an error);
// MODE 2: D = majority as floats.
// A thread takes 16 consecutive entries per step: one 16-byte load per
// worker, 8 workers' loads in flight at once, added into four words of
// signed byte lanes with __vadd4 (lane-wise, no carry between lanes).  The
// entries are -1, 0 or +1, so a lane holds the exact sum of up to 127
// workers; the lanes go into int counters every 120 workers and at the end.
// Entries outside {-1, 0, +1} give unspecified sums (never an out-of-range
// access).  Host-checked layout: every buffer 16-byte aligned.
// ---------------------------------------------------------------------------
template <int MODE, bool ACC8>
__global__ void __launch_bounds__(kTThreads)
k_vote_tern(WorkerPtrs signs, int M, int64_t d, void* __restrict__ sums, int8_t* __restrict__ maj,
            float* __restrict__ W, float eta, float* __restrict__ D, const int* __restrict__ status,
            int tie_plus) {
  griddep_wait();
  griddep_launch();
  if (MODE == 1 && status != nullptr && (status[0] | status[1]) != 0) return;
  const int64_t n16 = d >> 4;
  const int64_t stride = (int64_t)gridDim.x * kTThreads;
  for (int64_t i = (int64_t)blockIdx.x * kTThreads + threadIdx.x; i < n16; i += stride) {
    int cnt[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) cnt[k] = 0;
    uint32_t acc[4] = {0u, 0u, 0u, 0u};
    for (int m = 0; m < M; m += 8) {
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        v[j] = (m + j < M)
                   ? __ldcs(reinterpret_cast<const uint4*>(reinterpret_cast<const int8_t*>(signs.p[m + j]) + 16 * i))
                   : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        acc[0] = __vadd4(acc[0], v[j].x);
        acc[1] = __vadd4(acc[1], v[j].y);
        acc[2] = __vadd4(acc[2], v[j].z);
        acc[3] = __vadd4(acc[3], v[j].w);
      }
      if (((m + 8) % 120) == 0 || m + 8 >= M) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int b = 0; b < 4; ++b) cnt[4 * q + b] += sbyte(acc[q], b);
          acc[q] = 0u;
        }
      }
    }
    const int64_t e0 = 16 * i;
    if (MODE == 0) {
      if (sums != nullptr) {
        if (ACC8) {
          *reinterpret_cast<uint4*>(reinterpret_cast<int8_t*>(sums) + e0) =
              make_uint4(pack4(cnt[0], cnt[1], cnt[2], cnt[3]), pack4(cnt[4], cnt[5], cnt[6], cnt[7]),
                         pack4(cnt[8], cnt[9], cnt[10], cnt[11]), pack4(cnt[12], cnt[13], cnt[14], cnt[15]));
        } else {
          int4* s4 = reinterpret_cast<int4*>(reinterpret_cast<int32_t*>(sums) + e0);
#pragma unroll
          for (int q = 0; q < 4; ++q) s4[q] = make_int4(cnt[4 * q], cnt[4 * q + 1], cnt[4 * q + 2], cnt[4 * q + 3]);
        }
      }
      if (maj != nullptr) {
        uint32_t mw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          mw[q] = pack4(tmaj(cnt[4 * q], tie_plus), tmaj(cnt[4 * q + 1], tie_plus), tmaj(cnt[4 * q + 2], tie_plus),
                        tmaj(cnt[4 * q + 3], tie_plus));
        *reinterpret_cast<uint4*>(maj + e0) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
      }
    } else if (MODE == 1) {
      float4* w4 = reinterpret_cast<float4*>(W + e0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float4 w = w4[q];
        w.x = fmaf(-eta, (float)tmaj(cnt[4 * q], tie_plus), w.x);
        w.y = fmaf(-eta, (float)tmaj(cnt[4 * q + 1], tie_plus), w.y);
        w.z = fmaf(-eta, (float)tmaj(cnt[4 * q + 2], tie_plus), w.z);
        w.w = fmaf(-eta, (float)tmaj(cnt[4 * q + 3], tie_plus), w.w);
        w4[q] = w;
      }
    } else {
      float4* d4 = reinterpret_cast<float4*>(D + e0);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        d4[q] = make_float4((float)tmaj(cnt[4 * q], tie_plus), (float)tmaj(cnt[4 * q + 1], tie_plus),
                            (float)tmaj(cnt[4 * q + 2], tie_plus), (float)tmaj(cnt[4 * q + 3], tie_plus));
    }
  }
  // ragged tail (< 16 entries), entry by entry in the last block
  if (blockIdx.x == gridDim.x - 1) {
    for (int64_t e = 16 * n16 + threadIdx.x; e < d; e += kTThreads) {
      int c = 0;
      for (int m = 0; m < M; ++m) c += reinterpret_cast<const int8_t*>(signs.p[m])[e];
      if (MODE == 0) {
        if (sums != nullptr) {
          if (ACC8) reinterpret_cast<int8_t*>(sums)[e] = (int8_t)c;
          else reinterpret_cast<int32_t*>(sums)[e] = c;
        }
        if (maj != nullptr) maj[e] = (int8_t)tmaj(c, tie_plus);
      } else if (MODE == 1) {
        W[e] = fmaf(-eta, (float)tmaj(c, tie_plus), W[e]);
      } else {
        D[e] = (float)tmaj(c, tie_plus);
      }
    }
  }
}

template <int MODE, bool ACC8>
void vote_tern(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, void* sums, int8_t* maj, float* W,
               float eta, float* D, const int* status, int tie_plus) {
  count_launch();
  const int blocks = stream_grid((const void*)k_vote_tern<MODE, ACC8>, kTThreads, 0,
                                 ((d >> 4) + kTThreads - 1) / kTThreads, 8);
  launch_pdl(k_vote_tern<MODE, ACC8>, dim3(blocks), dim3(kTThreads), 0, s, signs, M, d, sums, maj, W, eta, D, status, tie_plus);
}

// D = majority of integer vote sums (int32, or int8 when ACC8): four entries
// per thread and step (one 16- or 4-byte load, one float4 store), the d % 4
// tail entry by entry in the last block.  Host-checked: sums 16-byte aligned.
template <bool ACC8>
__global__ void __launch_bounds__(kTThreads)
k_sums_major(const void* __restrict__ sums, int64_t d, float* __restrict__ D, int tie_plus) {
  griddep_wait();
  griddep_launch();
  const int64_t n4 = d >> 2;
  const int64_t stride = (int64_t)gridDim.x * kTThreads;
  for (int64_t i = (int64_t)blockIdx.x * kTThreads + threadIdx.x; i < n4; i += stride) {
    int s0, s1, s2, s3;
    if (ACC8) {
      const char4 v = reinterpret_cast<const char4*>(sums)[i];
      s0 = v.x; s1 = v.y; s2 = v.z; s3 = v.w;
    } else {
      const int4 v = reinterpret_cast<const int4*>(sums)[i];
      s0 = v.x; s1 = v.y; s2 = v.z; s3 = v.w;
    }
    reinterpret_cast<float4*>(D)[i] = make_float4((float)tmaj(s0, tie_plus), (float)tmaj(s1, tie_plus),
                                                  (float)tmaj(s2, tie_plus), (float)tmaj(s3, tie_plus));
  }
  if (blockIdx.x == gridDim.x - 1)
    for (int64_t e = 4 * n4 + threadIdx.x; e < d; e += kTThreads) {
      const int sv = ACC8 ? (int)reinterpret_cast<const int8_t*>(sums)[e] : reinterpret_cast<const int32_t*>(sums)[e];
      D[e] = (float)tmaj(sv, tie_plus);
    }
}

}  // namespace

// ---- launch wrappers --------------------------------------------------------

void launch_sign8(cudaStream_t s, const float* U, int64_t u_stride, int64_t d, int8_t* out, int64_t out_stride,
                  int M) {
  if (d <= 0 || M <= 0) return;
  count_launch();
  const int blocks = stream_grid((const void*)k_sign8, kTThreads, 0, ((d >> 4) + kTThreads - 1) / kTThreads, 8);
  dim3 grid(blocks, M);
  launch_pdl(k_sign8, dim3(grid), dim3(kTThreads), 0, s, U, u_stride, d, out, out_stride);
}

void launch_vote_ternary(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, void* sums, int acc8,
                         int8_t* majority, int tie_plus) {
  if (d <= 0) return;
  if (acc8) vote_tern<0, true>(s, signs, M, d, sums, majority, nullptr, 0.f, nullptr, nullptr, tie_plus);
  else vote_tern<0, false>(s, signs, M, d, sums, majority, nullptr, 0.f, nullptr, nullptr, tie_plus);
}

void launch_vote_ternary_update(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, float* W, float eta,
                                const int* status, int tie_plus) {
  if (d <= 0) return;
  vote_tern<1, false>(s, signs, M, d, nullptr, nullptr, W, eta, nullptr, status, tie_plus);
}

void launch_vote_ternary_major(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, float* D, int tie_plus) {
  if (d <= 0) return;
  vote_tern<2, false>(s, signs, M, d, nullptr, nullptr, nullptr, 0.f, D, nullptr, tie_plus);
}

void launch_sums_major(cudaStream_t s, const void* sums, int acc8, int64_t d, float* D, int tie_plus) {
  if (d <= 0) return;
  count_launch();
  const int blocks = acc8 ? stream_grid((const void*)k_sums_major<true>, kTThreads, 0, ((d >> 2) + kTThreads - 1) / kTThreads, 8)
                         : stream_grid((const void*)k_sums_major<false>, kTThreads, 0, ((d >> 2) + kTThreads - 1) / kTThreads, 8);
  if (acc8) launch_pdl(k_sums_major<true>, dim3(blocks), dim3(kTThreads), 0, s, sums, d, D, tie_plus);
  else launch_pdl(k_sums_major<false>, dim3(blocks), dim3(kTThreads), 0, s, sums, d, D, tie_plus);
}

}  // namespace sm
