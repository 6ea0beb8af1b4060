// noalloc.cu -- signmuon_spectral_norm_noalloc: the power-iteration estimate
// of a matrix's largest singular value for callers that cannot allocate
// device memory.
//
// Why it exists: some callers cannot call cudaMalloc at all -- for example
// code running while a CUDA graph is being captured (allocation calls are
// not allowed into a capture), code inside a framework that owns every byte
// of device memory through its own allocator, or a real-time path that must
// never enter the driver's allocator.  signmuon_init allocates the step's
// workspace, so such a caller cannot use it; this entry point takes only the
// caller's input and output pointers and keeps its working vectors in one
// statically sized device array that exists as long as the library is
// loaded.
//
// It computes the same estimate as the step's spectral scale (power
// iteration on the orientation with the smaller side m: u0 = ones/sqrt(m),
// u <- X(X^T u)/||X(X^T u)||, sigma = ||X^T u||), but directly on the fp32
// matrix with two matrix-vector products per iteration instead of on a Gram
// matrix, so it needs only O(rows + cols) scratch.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "../../include/signmuon.h"
#include "common.cuh"

namespace sm {
namespace {

// Scratch shared by every call in the process: w (n floats), y (m), u (m).
// Every call writes u before reading it and w, y before reading them, so no
// state carries over from the previous call.  1 Mi floats = 4 MiB of device
// memory per GPU that loads the library.
constexpr int64_t kNaScratchFloats = int64_t(1) << 20;
static __device__ __align__(256) float g_na_scratch[kNaScratchFloats];

constexpr int kT = 256;

// out[r] = sum_c X[r*cols + c] * v[c] for r < rows (a warp per row)
__global__ void __launch_bounds__(kT) k_na_rowdot(const float* __restrict__ X, int64_t rows, int64_t cols,
                                                 const float* __restrict__ v, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t r = ((int64_t)blockIdx.x * kT + threadIdx.x) >> 5;
  if (r >= rows) return;
  const float* x = X + r * cols;
  float acc = 0.f;
  for (int64_t c = lane; c < cols; c += 32) acc = fmaf(x[c], v[c], acc);
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) out[r] = acc;
}

// out[c] = sum_r X[r*cols + c] * v[r] for c < cols (a thread per column)
__global__ void __launch_bounds__(kT) k_na_coldot(const float* __restrict__ X, int64_t rows, int64_t cols,
                                                 const float* __restrict__ v, float* __restrict__ out) {
  const int64_t c = (int64_t)blockIdx.x * kT + threadIdx.x;
  if (c >= cols) return;
  float acc = 0.f;
  for (int64_t r = 0; r < rows; ++r) acc = fmaf(X[r * cols + c], v[r], acc);
  out[c] = acc;
}

// one block: u = y/||y|| (a zero vector stays zero), or u0 = ones/sqrt(m)
__global__ void __launch_bounds__(kT) k_na_normalize(const float* __restrict__ y, float* __restrict__ u,
                                                    int64_t m, int init) {
  __shared__ double red[kT / 32];
  __shared__ float scale;
  if (init) {
    const float v = rsqrtf((float)m);
    for (int64_t i = threadIdx.x; i < m; i += kT) u[i] = v;
    return;
  }
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < m; i += kT) s += (double)y[i] * (double)y[i];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kT / 32; ++w) t += red[w];
    scale = t > 0.0 ? (float)(1.0 / sqrt(t)) : 0.f;
  }
  __syncthreads();
  for (int64_t i = threadIdx.x; i < m; i += kT) u[i] = y[i] * scale;
}

// one block: sigma = ||w||
__global__ void __launch_bounds__(kT) k_na_norm(const float* __restrict__ w, int64_t n, float* __restrict__ sigma) {
  __shared__ double red[kT / 32];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += kT) s += (double)w[i] * (double)w[i];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int k = 0; k < kT / 32; ++k) t += red[k];
    *sigma = (float)sqrt(t);
  }
}

// Device address of g_na_scratch for each device, looked up once per device.
std::mutex g_na_mutex;
float* g_na_ptr[64] = {nullptr};

int na_scratch(int dev, float** out) {
  if (dev < 0 || dev >= 64) return SIGNMUON_E_INVALID;
  std::lock_guard<std::mutex> lock(g_na_mutex);
  if (g_na_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_na_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SIGNMUON_E_CUDA;
    }
    g_na_ptr[dev] = reinterpret_cast<float*>(p);
  }
  *out = g_na_ptr[dev];
  return SIGNMUON_OK;
}

}  // namespace
}  // namespace sm

extern "C" int signmuon_spectral_norm_noalloc(const float* X, int64_t rows, int64_t cols, int P, float* sigma,
                                              void* stream) {
  using namespace sm;
  if (X == nullptr || sigma == nullptr || rows < 1 || cols < 1 || P < 1) {
    set_global_error("spectral_norm_noalloc: null pointer, non-positive dimension or P < 1");
    return SIGNMUON_E_INVALID;
  }
  const int64_t m = rows < cols ? rows : cols;
  const int64_t n = rows < cols ? cols : rows;
  if (n + 2 * m > kNaScratchFloats) {
    set_global_error("spectral_norm_noalloc: max(rows, cols) + 2*min(rows, cols) exceeds the static scratch of "
                     "1048576 floats");
    return SIGNMUON_E_INVALID;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    set_global_error("spectral_norm_noalloc: no current CUDA device");
    return SIGNMUON_E_CUDA;
  }
  float* scratch = nullptr;
  const int rc = na_scratch(dev, &scratch);
  if (rc) {
    set_global_error("spectral_norm_noalloc: cudaGetSymbolAddress of the static scratch failed");
    return rc;
  }
  float* w = scratch;       // n: X_wide^T u
  float* y = w + n;         // m: X_wide w
  float* u = y + m;         // m: the iterate
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool wide = rows <= cols;
  auto xt_u = [&](const float* v, float* out) {  // out = X_wide^T v (length n)
    if (wide) k_na_coldot<<<(int)((cols + kT - 1) / kT), kT, 0, s>>>(X, rows, cols, v, out);
    else k_na_rowdot<<<(int)((rows * 32 + kT - 1) / kT), kT, 0, s>>>(X, rows, cols, v, out);
    count_launch();
  };
  auto x_w = [&](const float* v, float* out) {   // out = X_wide v (length m)
    if (wide) k_na_rowdot<<<(int)((rows * 32 + kT - 1) / kT), kT, 0, s>>>(X, rows, cols, v, out);
    else k_na_coldot<<<(int)((cols + kT - 1) / kT), kT, 0, s>>>(X, rows, cols, v, out);
    count_launch();
  };
  k_na_normalize<<<1, kT, 0, s>>>(nullptr, u, m, 1);  // u0 = ones/sqrt(m) (nothing carried over)
  count_launch();
  for (int it = 0; it < P; ++it) {
    xt_u(u, w);
    x_w(w, y);
    k_na_normalize<<<1, kT, 0, s>>>(y, u, m, 0);
    count_launch();
  }
  xt_u(u, w);
  k_na_norm<<<1, kT, 0, s>>>(w, n, sigma);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) {
    set_global_error("spectral_norm_noalloc: kernel launch failed");
    return SIGNMUON_E_CUDA;
  }
  return SIGNMUON_OK;
}
