// signmuon_api.cu -- the C ABI of libsignmuon.so (declared in
// include/signmuon.h): handle life cycle, device buffers, TMA tensor maps and
// the kernel sequence of one Sign-Muon step.
//
// Step sequence on the handle's stream ([paper] "SignMuon: 通信高效的分布式Muon优化"
// Algorithm 2; the vote of [blog] "SignMuon: Matrix Directions, Majority
// Votes, and the Actual Bytes Sent"):
//   momentum pass -> Frobenius partials -> NS GEMMs (GRAM [-> power iteration]
//   [-> SQUARE] -> APPLY) x K -> one-bit pack (or int8 ternary sign) -> vote
//   fused with the update, or vote -> stage -> NS x K -> update for the
//   post-vote polar step (K = 0 there for the normalised sign step).
#include <cuda.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <new>
#include <string>
#include <utility>
#include <vector>

#include "../../include/signmuon.h"
#include "common.cuh"
#include "plan.h"

namespace sm {
static std::atomic<int64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace sm

using sm::Plan;

struct signmuon_ctx {
  Plan plan;
  int M = 0, K = 0, scale = 0, P = 1;
  float beta = 0.f, lambda = 0.f, eps = 0.f;
  float ns_a = 1.5f, ns_b = -0.5f, ns_c = 0.f;
  unsigned flags = 0;
  cudaStream_t stream = nullptr;
  int device = 0, n_sm = 148;
  bool vote_only = false;
  bool u_valid = true;          // U holds the last step's (or polar call's) polar factors
  bool bits_valid = true;       // bits hold the last step's packed signs
  bool t_valid = false;         // sign8 holds the last step's ternary signs
  bool dir_valid = false;       // get_direction can give the last step's D
  bool dir_in_D = false;        // ... and it is in D (else: the majority of the handle's own signs)
  // device plan tables
  sm::MatInfo* d_mats = nullptr;
  sm::GroupInfo* d_groups = nullptr;
  int* d_group_mats = nullptr;
  int64_t* d_mat_off = nullptr;
  sm::Chunk* d_chunks = nullptr;
  int* d_mat_chunk0 = nullptr;
  int* d_mat_nchunks = nullptr;
  int64_t* d_stage_off = nullptr;
  sm::TileGroup* d_tiles[3][2] = {{nullptr}};
  int* d_sched[3][2] = {{nullptr}};   // tensor-core tile schedules (null: round robin)
  sm::PiTile* d_pi_tiles = nullptr;
  sm::PiSlice* d_pi_slices = nullptr;
  int64_t* d_uoff = nullptr;
  int* d_prob_g = nullptr;
  int* d_prob_gld = nullptr;
  int64_t* d_prob_aoff = nullptr;
  void* d_maps = nullptr;
  // device state / workspace
  float* Mom = nullptr;
  void* X[2] = {nullptr, nullptr};
  void* A = nullptr;
  void* B = nullptr;
  void* A2 = nullptr;           // Gram space: the second A buffer and the Q pair
  void* Q[2] = {nullptr, nullptr};
  float* U = nullptr;
  uint8_t* bits = nullptr;
  int8_t* sign8 = nullptr;      // TERNARY: int8 signs, M x dpad bytes
  float* D = nullptr;
  float* partials = nullptr;
  float* scale_v = nullptr;
  float2* coef_apply = nullptr;
  float2* coef_square = nullptr;
  float2* coef_gram = nullptr;  // Gram space: A1 = a T0 + b cc^2 A~ T0
  float* pi_u = nullptr;        // power-iteration iterates of the M-worker problems (warm state)
  float* pi_u1 = nullptr;       // PI_WARM: iterates of the one-problem-set PolarNS (warm state)
  float* pi_y = nullptr;
  float* pi_part = nullptr;     // per-tile partial sums of A v
  float* pi_inv = nullptr;      // per-problem 1/||y|| between passes
  double* pi_sq = nullptr;      // per-slice ||y||^2 or u.y
  int* pi_cnt = nullptr;        // per-problem slice counters (zero between launches)
  int* status = nullptr;        // [0] non-finite flag, [1] kernel error code
  int* h_status = nullptr;      // pinned mirror
  bool pending = false;         // an async step's status not yet read
  // the ternary signs of the step's last Newton-Schulz GEMM (bf16 path): set
  // by local_part around its run_ns, read by gemm() for the final apply
  int8_t* final_sign8 = nullptr;
  int64_t final_sign8_stride = 0;
  // step_host staging: W, and two gradient buffers so that a call's
  // gradients can come in (on the copy stream) while the step before runs
  float* hw_W = nullptr;
  float* hw_G[2] = {nullptr, nullptr};
  int hw_next = 0;                      // the gradient buffer of the next call
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t g_ready[2] = {nullptr, nullptr};   // buffer b holds its call's gradients
  cudaEvent_t g_free[2] = {nullptr, nullptr};    // the step that read buffer b is done
  cudaEvent_t w_ready = nullptr;                 // W of the current call is on the device
  cudaEvent_t w_free = nullptr;                  // the previous call's W has gone back
  std::vector<void*> allocs;
  int64_t bytes = 0;
  std::string err;
  // optional per-kernel timing: event pairs recorded around each launch
  bool prof = false;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_used = 0;
  std::vector<int> ev_kind;           // kind of each recorded pair
  double prof_ms[SIGNMUON_PROF_KINDS] = {0};
  int64_t prof_n[SIGNMUON_PROF_KINDS] = {0};
};

namespace {

std::string g_noh_err;  // errors raised before a handle exists

}  // namespace

void sm::set_global_error(const char* msg) { g_noh_err = msg; }

namespace {

int fail(signmuon_t h, int code, const std::string& msg) {
  if (h) h->err = msg;
  else g_noh_err = msg;
  return code;
}

#define CK(h, call)                                                                   \
  do {                                                                                \
    cudaError_t e_ = (call);                                                          \
    if (e_ != cudaSuccess) {                                                          \
      cudaGetLastError();                                                             \
      return fail((h), e_ == cudaErrorMemoryAllocation ? SIGNMUON_E_NOMEM : SIGNMUON_E_CUDA, \
                  std::string(#call) + ": " + cudaGetErrorString(e_));                \
    }                                                                                 \
  } while (0)

template <typename T>
int dalloc(signmuon_t h, T** p, int64_t count) {
  *p = nullptr;
  if (count <= 0) count = 1;
  void* q = nullptr;
  cudaError_t e = cudaMalloc(&q, (size_t)count * sizeof(T));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(h, SIGNMUON_E_NOMEM, std::string("cudaMalloc: ") + cudaGetErrorString(e));
  }
  h->allocs.push_back(q);
  h->bytes += count * (int64_t)sizeof(T);
  *p = reinterpret_cast<T*>(q);
  return SIGNMUON_OK;
}

template <typename T>
int upload(signmuon_t h, T** dst, const std::vector<T>& src) {
  int rc = dalloc(h, dst, (int64_t)src.size());
  if (rc) return rc;
  if (!src.empty()) CK(h, cudaMemcpy(*dst, src.data(), src.size() * sizeof(T), cudaMemcpyHostToDevice));
  return SIGNMUON_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// 3-D bf16 tensor map over `batch` matrices of rows x cols (row stride ld),
// boxes of 64 columns x box_rows rows with the 128-byte swizzle;
// out-of-range parts of a box read as zeros and are not written.
int encode_map(signmuon_t h, CUtensorMap* m, void* base, int cols, int rows, int ld, int batch, int box_rows) {
  EncodeTiledFn fn = get_encode();
  if (!fn) return fail(h, SIGNMUON_E_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)rows * ld * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(h, SIGNMUON_E_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return SIGNMUON_OK;
}

// 4-D view of the same matrices: (64-column atom, row, atom index, matrix),
// strides (row, 128 B, matrix); a box of `atoms` atoms x box_rows rows lands
// in shared memory atom after atom.  Requires cols % 64 == 0, so that no
// atom reaches past the end of a row and stores clip at the last column.
int encode_map_atoms(signmuon_t h, CUtensorMap* m, void* base, int cols, int rows, int ld, int batch, int box_rows,
                     int atoms) {
  EncodeTiledFn fn = get_encode();
  if (!fn) return fail(h, SIGNMUON_E_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[4] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64), (cuuint64_t)batch};
  cuuint64_t strides[3] = {(cuuint64_t)ld * 2, 128, (cuuint64_t)rows * ld * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, (cuuint32_t)atoms, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(h, SIGNMUON_E_CUDA, "cuTensorMapEncodeTiled (4-D) failed: " + std::to_string((int)r));
  return SIGNMUON_OK;
}

sm::WorkerPtrs worker_ptrs(const float* const* p, int M) {
  sm::WorkerPtrs w{};
  for (int m = 0; m < M; ++m) w.p[m] = p[m];
  return w;
}

sm::WorkerPtrs strided_ptrs(const float* base, int64_t stride, int M) {
  sm::WorkerPtrs w{};
  for (int m = 0; m < M; ++m) w.p[m] = base + (int64_t)m * stride;
  return w;
}

// worker m's sign buffer at base + m * stride bytes
sm::WorkerPtrs byte_ptrs(const uint8_t* base, int64_t stride, int M) {
  sm::WorkerPtrs w{};
  for (int m = 0; m < M; ++m) w.p[m] = reinterpret_cast<const float*>(base + (int64_t)m * stride);
  return w;
}

// NVTX range names of the profiling kinds (signmuon_profile's numbering)
const char* const kKindNames[SIGNMUON_PROF_KINDS] = {
    "signmuon momentum",      "signmuon norm finalize",  "signmuon NS gram",       "signmuon NS square",
    "signmuon NS apply",      "signmuon power iteration", "signmuon sign",         "signmuon vote",
    "signmuon mean stage",    "signmuon post NS gram",    "signmuon post NS square", "signmuon post NS apply",
    "signmuon update",        "signmuon K=0 scale"};

// A host NVTX range for the lifetime of a scope (a no-op unless a tool such
// as ncu --nvtx is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

// One kernel launch of `kind`: an NVTX range always, and the CUDA event pair
// only while timing (signmuon_profile).
struct ProfScope {
  signmuon_t h;
  int kind;
  cudaEvent_t e1 = nullptr;
  NvtxRange range;
  ProfScope(signmuon_t h_, int kind_) : h(h_), kind(kind_), range(kKindNames[kind_]) {
    if (!h->prof) return;
    while (h->ev_pool.size() < h->ev_used + 2) {
      cudaEvent_t e;
      cudaEventCreate(&e);
      h->ev_pool.push_back(e);
    }
    cudaEventRecord(h->ev_pool[h->ev_used], h->stream);
    e1 = h->ev_pool[h->ev_used + 1];
    h->ev_used += 2;
    h->ev_kind.push_back(kind);
  }
  ~ProfScope() {
    if (e1) cudaEventRecord(e1, h->stream);
  }
};

void prof_collect(signmuon_t h) {
  if (h->ev_used == 0) return;
  cudaStreamSynchronize(h->stream);
  for (size_t i = 0; i < h->ev_kind.size(); ++i) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, h->ev_pool[2 * i], h->ev_pool[2 * i + 1]) == cudaSuccess) {
      h->prof_ms[h->ev_kind[i]] += ms;
      h->prof_n[h->ev_kind[i]] += 1;
    }
  }
  cudaGetLastError();
  h->ev_used = 0;
  h->ev_kind.clear();
}

// ---------------------------------------------------------------------------
// PolarNS with K iterations for nw workers whose X~ (unscaled) is staged in
// X[0]; the Frobenius scale (if used) is already final.  Writes U (fp32,
// flat) to out + worker*out_stride.  kzero_in is the fp32 input used when
// K == 0.
// ---------------------------------------------------------------------------
// m x m bf16 buffer by index (sm::MmBuf)
void* mm_ptr(signmuon_t h, int buf) {
  switch (buf) {
    case sm::MM_A: return h->A;
    case sm::MM_B: return h->B;
    case sm::MM_A2: return h->A2;
    case sm::MM_Q0: return h->Q[0];
    default: return h->Q[1];
  }
}

// One grouped GEMM launch.  SQUARE (bf16): out buffer sq_out = c0 R + c1 L R
// + cdiag I with L = buffer sq_l, R = buffer sq_r; APPLY multiplies X by
// buffer p_buf (default: B for quintic, else A).
void gemm(signmuon_t h, int op, int slot, int src, int nw, const float2* coef, float c0, float c1,
          bool final_out, float* out, int64_t out_stride, uint32_t* out_bits = nullptr, int64_t bits_stride = 0,
          float cdiag = 0.f, bool plain = false, int sq_l = sm::MM_A, int sq_r = sm::MM_A, int sq_out = sm::MM_B,
          int p_buf = -1) {
  const Plan& p = h->plan;
  sm::GemmArgs a{};
  a.tiles = h->d_tiles[op][slot];
  a.sched = h->d_sched[op][slot];
  a.n_tile_groups = (int)p.tiles[op][slot].groups.size();
  a.total_tiles = p.tiles[op][slot].total;
  a.groups = h->d_groups;
  a.group_mats = h->d_group_mats;
  a.mat_off = h->d_mat_off;
  a.n_mats = p.n_mats;
  a.op = op;
  a.X_src = h->X[src];
  a.X_dst = h->X[src ^ 1];
  a.A = h->A;
  a.B = h->B;
  a.p_from_b = (op == sm::OP_APPLY && p.quintic) ? 1 : 0;
  a.p_buf = p_buf >= 0 ? p_buf : (a.p_from_b ? sm::MM_B : sm::MM_A);
  a.sq_l = sq_l;
  a.sq_r = sq_r;
  a.sq_out = mm_ptr(h, sq_out);
  a.sym_exact = p.gram_ns ? 1 : 0;
  a.map_src = src;
  a.map_dst = src ^ 1;
  a.coef = coef;
  a.c0 = c0;
  a.c1 = c1;
  a.cdiag = cdiag;
  a.plain = plain ? 1 : 0;
  a.out = out;
  a.out_stride = out_stride;
  a.final_out = final_out ? 1 : 0;
  a.out_bits = out_bits;
  a.bits_stride = bits_stride;
  if (final_out && op == sm::OP_APPLY) {
    a.out_sign8 = h->final_sign8;
    a.sign8_stride = h->final_sign8_stride;
  }
  a.err = h->status + 1;
  (void)nw;
  const auto& tg = p.tiles[op][slot].groups;
  if ((int)tg.size() <= sm::kParamGroups && (int)p.groups.size() <= sm::kParamGroups &&
      p.n_mats <= sm::kParamMats) {
    a.param_tables = 1;
    for (size_t i = 0; i < tg.size(); ++i) a.ptiles[i] = tg[i];
    for (size_t i = 0; i < p.groups.size(); ++i) a.pgroups[i] = p.groups[i];
    for (int i = 0; i < p.n_mats; ++i) a.pgroup_mats[i] = p.group_mats[i];
  }
  ProfScope ps(h, (nw == 1 ? 9 : 2) + op);
  if (p.fp32) sm::launch_gemm_simt(h->stream, a, 1);
  else sm::launch_gemm_tc(h->stream, a, h->d_maps, h->n_sm);
}

// P power iterations on the Gram of nw problem sets.  With SIGNMUON_PI_WARM
// each problem starts from the iterate it ended with last time: the M-worker
// PolarNS (step or signmuon_polar) keeps its iterates in pi_u, the
// one-problem-set PolarNS (post-vote, normalised sign, Muon mean) in pi_u1.
void power_iteration(signmuon_t h, int nw) {
  const Plan& p = h->plan;
  const int nprob = nw * p.n_mats;
  const int ntiles = nw == 1 ? p.n_pi_tiles_one : (int)p.pi_tiles.size();
  const bool warm = (h->flags & SIGNMUON_PI_WARM) != 0;
  float* u = (warm && nw == 1) ? h->pi_u1 : h->pi_u;
  const int bf16 = p.fp32 ? 0 : 1;
  ProfScope ps(h, 5);
  const int nslices = nw == 1 ? p.n_pi_slices_one : (int)p.pi_slices.size();
  const sm::PiReduce mid{0, u, h->pi_sq, h->pi_cnt, h->pi_inv, h->eps, p.quintic ? 1 : 0, h->ns_a, h->ns_b,
                         h->ns_c, h->scale_v, h->coef_apply, h->coef_square, h->coef_gram, h->status};
  sm::PiReduce fin = mid;
  fin.last = 1;
  // y = A u0 (a cold start stages u0 = ones / sqrt(g) in the first pass
  // itself; a warm one keeps the stored iterate when it is usable); then P
  // times y = A (y / ||y||), storing y / ||y|| as u
  if (warm) sm::launch_pi_init(h->stream, nprob, h->d_uoff, h->d_prob_g, u, 1);
  sm::launch_pi_tiles(h->stream, h->d_pi_tiles, ntiles, h->A, bf16, warm ? u : nullptr, nullptr, u, h->pi_part, 0);
  for (int it = 0; it < h->P; ++it) {
    sm::launch_pi_reduce(h->stream, h->d_pi_slices, nslices, h->pi_part, h->pi_y, mid);
    sm::launch_pi_tiles(h->stream, h->d_pi_tiles, ntiles, h->A, bf16, h->pi_y, h->pi_inv, u, h->pi_part, 1);
  }
  sm::launch_pi_reduce(h->stream, h->d_pi_slices, nslices, h->pi_part, h->pi_y, fin);
}

// The streaming vote kernel stages the post-vote input when every matrix
// starts at a multiple of 128 entries (16-byte aligned in every bit stream)
// and has a multiple of 8 columns (its rows are unpadded in X, so a chunk's
// range is contiguous there).
bool stage_streamable(signmuon_t h) {
  for (const sm::MatInfo& mi : h->plan.mats)
    if ((mi.off % 128) != 0 || (mi.cols % 8) != 0) return false;
  return true;
}

// The one-bit signs come out of the last Newton-Schulz GEMM on the bf16
// path (K > 0).  Every 32-column chunk of an output row is then one aligned
// word of the bit stream when every matrix has a multiple of 32 columns;
// otherwise chunks that straddle words OR their bits in, and the buffer is
// zeroed first (signs_ragged).
bool signs_in_gemm(signmuon_t h) {
  const Plan& p = h->plan;
  return !p.fp32 && h->K > 0 && (p.nb_pad % 4) == 0;
}

bool signs_ragged(signmuon_t h) {
  for (const sm::GroupInfo& gi : h->plan.groups)
    if (gi.cols % 32 != 0) return true;
  return false;
}

void run_ns(signmuon_t h, int K, int nw, const sm::WorkerPtrs& kzero_in, float* out, int64_t out_stride,
            uint32_t* out_bits = nullptr, int64_t bits_stride = 0) {
  const Plan& p = h->plan;
  const int slot = nw == 1 ? 1 : 0;
  const bool spectral = h->scale == SIGNMUON_SCALE_SPECTRAL;
  if (K == 0) {
    if (spectral) {
      gemm(h, sm::OP_GRAM, slot, 0, nw, nullptr, 0.f, 1.f, false, nullptr, 0);
      power_iteration(h, nw);
    }
    ProfScope ps(h, 13);
    sm::launch_scale_flat(h->stream, kzero_in, nw, out, out_stride, h->d_chunks, (int)p.chunks.size(), h->d_mats,
                          p.n_mats, h->scale_v, h->eps);
    return;
  }
  if (p.gram_ns && K >= 2) {
    // The same iteration in Gram space (bf16 cubic): with P_k = a I + b A_k,
    // A_{k+1} = P_k A_k P_k and Q_{k+1} = P_k Q_k, all polynomials in
    // A0 = cc^2 A~, so every product commutes and is symmetric:
    //   T_k     = a A_k + b A_k^2          (square: L = R = A_k)
    //   A_{k+1} = a T_k + b A_k T_k        (L = A_k, R = T_k)
    //   Q_{k+1} = a Q_k + b A_k Q_k        (L = A_k, R = Q_k)
    // from Q1 = cc P_0 = a cc I + b cc^3 A~, then X_K = Q_K X~ once.  Iteration
    // 0 works on the unscaled Gram (the power iteration's input), its scale
    // in per-problem coefficients.
    gemm(h, sm::OP_GRAM, slot, 0, nw, nullptr, 0.f, 1.f, false, nullptr, 0);
    if (spectral) power_iteration(h, nw);
    {
      ProfScope ps(h, nw == 1 ? 10 : 3);
      int max_g = 1, max_gld = 8;
      for (const sm::GroupInfo& gi : p.groups) {
        max_g = std::max(max_g, gi.g);
        max_gld = std::max(max_gld, gi.gld);
      }
      sm::launch_gram_q1(h->stream, nw * p.n_mats, h->A, h->Q[0], h->d_prob_aoff, h->d_prob_g, h->d_prob_gld,
                         h->coef_apply, max_g, max_gld);
    }
    const float a = h->ns_a, b = h->ns_b;
    gemm(h, sm::OP_SQUARE, slot, 0, nw, h->coef_square, 0.f, 0.f, false, nullptr, 0, nullptr, 0, 0.f, false,
         sm::MM_A, sm::MM_A, sm::MM_B);                                             // T0
    gemm(h, sm::OP_SQUARE, slot, 0, nw, h->coef_gram, 0.f, 0.f, false, nullptr, 0, nullptr, 0, 0.f, false,
         sm::MM_A, sm::MM_B, sm::MM_A2);                                            // A1
    int acur = sm::MM_A2, aoth = sm::MM_A, qcur = sm::MM_Q0, qoth = sm::MM_Q1;
    for (int k = 1; k < K; ++k) {
      gemm(h, sm::OP_SQUARE, slot, 0, nw, nullptr, a, b, false, nullptr, 0, nullptr, 0, 0.f, false, acur, qcur,
           qoth);                                                                   // Q_{k+1}
      if (k + 1 < K) {
        gemm(h, sm::OP_SQUARE, slot, 0, nw, nullptr, a, b, false, nullptr, 0, nullptr, 0, 0.f, false, acur, acur,
             sm::MM_B);                                                             // T_k
        gemm(h, sm::OP_SQUARE, slot, 0, nw, nullptr, a, b, false, nullptr, 0, nullptr, 0, 0.f, false, acur,
             sm::MM_B, aoth);                                                       // A_{k+1}
        std::swap(acur, aoth);
      }
      std::swap(qcur, qoth);
    }
    gemm(h, sm::OP_APPLY, slot, 0, nw, nullptr, 0.f, 1.f, true, out, out_stride, out_bits, bits_stride, 0.f, true,
         sm::MM_A, sm::MM_A, sm::MM_B, qcur);                                       // X_K = Q_K X~
    return;
  }
  // After the first iteration (bf16 path) the a X term joins the apply's
  // operator: the Gram GEMM writes P = b A + a I (cubic) or the square GEMM
  // B = b A + c A^2 + a I (quintic), and the apply is a plain GEMM X' = P X
  // (X P for the tall orientation) whose epilogue reads no operand.  The
  // first iteration keeps the affine epilogue: its coefficients carry the
  // scale, which the power iteration takes from that iteration's pure Gram.
  int cur = 0;
  for (int k = 0; k < K; ++k) {
    const bool fold = !p.fp32 && k > 0;
    const bool last = (k == K - 1);
    if (fold && !p.quintic)
      gemm(h, sm::OP_GRAM, slot, cur, nw, nullptr, 0.f, h->ns_b, false, nullptr, 0, nullptr, 0, h->ns_a);
    else
      gemm(h, sm::OP_GRAM, slot, cur, nw, nullptr, 0.f, 1.f, false, nullptr, 0);
    if (k == 0 && spectral) power_iteration(h, nw);
    if (p.quintic)
      gemm(h, sm::OP_SQUARE, slot, cur, nw, k == 0 ? h->coef_square : nullptr, h->ns_b, h->ns_c, false, nullptr, 0,
           nullptr, 0, fold ? h->ns_a : 0.f);
    if (fold)
      gemm(h, sm::OP_APPLY, slot, cur, nw, nullptr, 0.f, 1.f, last, out, out_stride, last ? out_bits : nullptr,
           bits_stride, 0.f, true);
    else
      gemm(h, sm::OP_APPLY, slot, cur, nw, k == 0 ? h->coef_apply : nullptr, h->ns_a, p.quintic ? 1.f : h->ns_b,
           last, out, out_stride, last ? out_bits : nullptr, bits_stride);
    cur ^= 1;
  }
}

void fro_finalize(signmuon_t h, int nw) {
  const Plan& p = h->plan;
  ProfScope ps(h, 1);
  sm::launch_fro_finalize(h->stream, nw * p.n_mats, p.n_mats, nw, h->partials, h->d_mat_chunk0, h->d_mat_nchunks,
                          h->scale == SIGNMUON_SCALE_FRO ? 1 : 0, h->eps, p.quintic ? 1 : 0, h->ns_a, h->ns_b,
                          h->ns_c, h->scale_v, h->coef_apply, h->coef_square, h->coef_gram, h->status);
}

// Clear the device status at the start of a call, unless an asynchronous
// call's status is still unread: then its flags stay set, so the update
// kernels of this call leave W alone and signmuon_sync reports the first
// error since the last sync.
cudaError_t begin_status(signmuon_t h) {
  if (h->pending) return cudaSuccess;
  return cudaMemsetAsync(h->status, 0, 2 * sizeof(int), h->stream);
}

int finish(signmuon_t h, bool wait) {
  CK(h, cudaMemcpyAsync(h->h_status, h->status, 2 * sizeof(int), cudaMemcpyDeviceToHost, h->stream));
  CK(h, cudaGetLastError());
  if (!wait) {
    h->pending = true;
    return SIGNMUON_OK;
  }
  CK(h, cudaStreamSynchronize(h->stream));
  h->pending = false;
  if (h->h_status[1] != 0) return fail(h, SIGNMUON_E_TIMEOUT, "a kernel's bounded wait expired");
  if (h->h_status[0] != 0) return fail(h, SIGNMUON_E_NONFINITE, "a momentum norm is NaN or Inf; W was not updated");
  return SIGNMUON_OK;
}

// Makes the handle's device current for the duration of one entry point and
// gives the caller's current device back on return, so that a call on a
// handle of another GPU leaves the caller's device selection as it was.
struct DeviceGuard {
  int saved = -1;
  explicit DeviceGuard(signmuon_t h) {
    if (h == nullptr) return;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
      cudaGetLastError();
      dev = -1;
    }
    if (dev != h->device && cudaSetDevice(h->device) == cudaSuccess) saved = dev;
  }
  ~DeviceGuard() {
    if (saved >= 0) cudaSetDevice(saved);
  }
  DeviceGuard(const DeviceGuard&) = delete;
  DeviceGuard& operator=(const DeviceGuard&) = delete;
};

int check_handle(signmuon_t h, bool need_step) {
  if (h == nullptr) return fail(nullptr, SIGNMUON_E_INVALID, "null handle");
  if (need_step && h->vote_only) return fail(h, SIGNMUON_E_UNSUPPORTED, "handle was created with SIGNMUON_VOTE_ONLY");
  return SIGNMUON_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* signmuon_status_string(int s) {
  switch (s) {
    case SIGNMUON_OK: return "ok";
    case SIGNMUON_E_INVALID: return "invalid argument";
    case SIGNMUON_E_OVERFLOW: return "int8 accumulator overflow (M > 127)";
    case SIGNMUON_E_NONFINITE: return "non-finite momentum norm";
    case SIGNMUON_E_CUDA: return "CUDA error";
    case SIGNMUON_E_NOMEM: return "out of device memory";
    case SIGNMUON_E_TIMEOUT: return "kernel wait timed out";
    case SIGNMUON_E_UNSUPPORTED: return "unsupported for this handle";
    default: return "unknown status";
  }
}

const char* signmuon_last_error(signmuon_t h) { return h ? h->err.c_str() : g_noh_err.c_str(); }

int64_t signmuon_kernel_launches(void) { return sm::g_launches.load(); }

static void fill_info(const Plan& p, int64_t* out, int n) {
  const int64_t v[8] = {p.d, p.nb, p.device_bytes, (int64_t)p.groups.size(), p.M, p.n_mats, p.u_elems, p.u_elems_one};
  for (int i = 0; i < n && i < 8; ++i) out[i] = v[i];
}

int signmuon_plan(const int64_t* shapes, int n_mats, int M, int K, int scale, int P, unsigned flags,
                  int64_t* out, int n) {
  Plan p;
  std::string err;
  const int rc = sm::make_plan(shapes, n_mats, M, K, scale, P, flags, &p, &err);
  if (rc) return fail(nullptr, rc, err);
  if (out) fill_info(p, out, n);
  return SIGNMUON_OK;
}

int signmuon_plan_tables(const int64_t* shapes, int n_mats, int M, int K, int scale, int P, unsigned flags,
                         char* buf, int64_t cap, int64_t* need) {
  Plan p;
  std::string err;
  const int rc = sm::make_plan(shapes, n_mats, M, K, scale, P, flags, &p, &err);
  if (rc) return fail(nullptr, rc, err);
  std::string j;
  j.reserve(1 << 16);
  auto num = [&](int64_t v) { j += std::to_string(v); };
  auto list = [&](const char* name, auto n, auto item) {
    j += '"';
    j += name;
    j += "\":[";
    for (size_t i = 0; i < (size_t)n; ++i) {
      if (i) j += ',';
      item(i);
    }
    j += "],";
  };
  auto tuple = [&](std::initializer_list<int64_t> v) {
    j += '[';
    bool first = true;
    for (int64_t x : v) {
      if (!first) j += ',';
      first = false;
      num(x);
    }
    j += ']';
  };
  j += "{";
  const std::pair<const char*, int64_t> scalars[] = {
      {"d", p.d}, {"dpad", p.dpad}, {"nb", p.nb}, {"nb_pad", p.nb_pad}, {"x_elems", p.x_elems},
      {"a_elems", p.a_elems}, {"u_elems", p.u_elems}, {"u_elems_one", p.u_elems_one},
      {"n_pi_tiles_one", p.n_pi_tiles_one},
      {"n_pi_slices", (int64_t)p.pi_slices.size()}, {"n_pi_slices_one", p.n_pi_slices_one},
      {"part_elems", p.part_elems}, {"M", p.M}, {"n_mats", p.n_mats}, {"fp32", p.fp32 ? 1 : 0},
      {"quintic", p.quintic ? 1 : 0}, {"gram_ns", p.gram_ns ? 1 : 0}, {"device_bytes", p.device_bytes}};
  for (const auto& kv : scalars) {
    j += '"';
    j += kv.first;
    j += "\":";
    num(kv.second);
    j += ',';
  }
  list("groups", p.groups.size(), [&](size_t i) {
    const sm::GroupInfo& g = p.groups[i];
    tuple({g.rows, g.cols, g.ld, g.g, g.gld, g.wide, g.count, g.first, g.x_base, g.a_base});
  });
  list("mats", p.mats.size(), [&](size_t i) {
    const sm::MatInfo& m = p.mats[i];
    tuple({m.off, m.rows, m.cols, m.group, m.q});
  });
  list("group_mats", p.group_mats.size(), [&](size_t i) { num(p.group_mats[i]); });
  list("chunks", p.chunks.size(), [&](size_t i) {
    const sm::Chunk& c = p.chunks[i];
    tuple({c.mat, c.len, c.start});
  });
  list("mat_chunk0", p.mat_chunk0.size(), [&](size_t i) { num(p.mat_chunk0[i]); });
  list("mat_nchunks", p.mat_nchunks.size(), [&](size_t i) { num(p.mat_nchunks[i]); });
  list("tiles", 6, [&](size_t k) {
    const sm::TileTable& t = p.tiles[k / 2][k % 2];
    j += "{\"total\":";
    num(t.total);
    j += ",\"groups\":[";
    for (size_t i = 0; i < t.groups.size(); ++i) {
      const sm::TileGroup& x = t.groups[i];
      if (i) j += ',';
      tuple({x.group, x.Mdim, x.Ndim, x.Kdim, x.BM, x.BN, x.sym, x.tiles_m, x.tiles_n, x.batch, x.tile_start});
    }
    // the tensor-core launch's schedule for a 148-SM B200 (74 clusters),
    // empty for round robin, and both makespans in k-blocks
    const int ncl = std::min(t.total, 74);
    double rr = 0.0, greedy = 0.0;
    const std::vector<int> sched = sm::tile_schedule(t, ncl, &rr, &greedy);
    j += "],\"clusters\":";
    num(ncl);
    j += ",\"makespan_rr\":";
    num((int64_t)rr);
    j += ",\"makespan_greedy\":";
    num((int64_t)greedy);
    j += ",\"sched\":[";
    for (size_t i = 0; i < sched.size(); ++i) {
      if (i) j += ',';
      num(sched[i]);
    }
    j += "]}";
  });
  list("pi_tiles", p.pi_tiles.size(), [&](size_t i) {
    const sm::PiTile& t = p.pi_tiles[i];
    tuple({t.p, t.bi, t.bj, t.aoff, t.uoff, t.poff, t.g, t.gld});
  });
  list("pi_slices", p.pi_slices.size(), [&](size_t i) {
    const sm::PiSlice& t = p.pi_slices[i];
    tuple({t.p, t.bi, t.uoff, t.poff, t.g, t.soff});
  });
  list("uoff", p.uoff.size(), [&](size_t i) { num(p.uoff[i]); });
  list("poff", p.poff.size(), [&](size_t i) { num(p.poff[i]); });
  list("soff", p.soff.size(), [&](size_t i) { num(p.soff[i]); });
  list("prob_g", p.prob_g.size(), [&](size_t i) { num(p.prob_g[i]); });
  list("prob_gld", p.prob_gld.size(), [&](size_t i) { num(p.prob_gld[i]); });
  list("prob_aoff", p.prob_aoff.size(), [&](size_t i) { num(p.prob_aoff[i]); });
  j.back() = '}';
  const int64_t n = (int64_t)j.size() + 1;
  if (need) *need = n;
  if (buf == nullptr) return SIGNMUON_OK;
  if (cap < n) return fail(nullptr, SIGNMUON_E_INVALID, "buffer too small: " + std::to_string(n) + " bytes needed");
  std::memcpy(buf, j.c_str(), (size_t)n);
  return SIGNMUON_OK;
}

void signmuon_destroy(signmuon_t h) {
  if (!h) return;
  DeviceGuard dev_guard(h);
  cudaStreamSynchronize(h->stream);
  if (h->copy_stream) {
    cudaStreamSynchronize(h->copy_stream);
    cudaStreamDestroy(h->copy_stream);
  }
  for (int b = 0; b < 2; ++b) {
    if (h->g_ready[b]) cudaEventDestroy(h->g_ready[b]);
    if (h->g_free[b]) cudaEventDestroy(h->g_free[b]);
  }
  if (h->w_ready) cudaEventDestroy(h->w_ready);
  if (h->w_free) cudaEventDestroy(h->w_free);
  for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
  for (void* q : h->allocs) cudaFree(q);
  if (h->h_status) cudaFreeHost(h->h_status);
  delete h;
}

int signmuon_init(signmuon_t* out, const int64_t* shapes, int n_mats, int M, float beta, float lambda, int K,
                  float eps, int scale, int P, unsigned flags, void* stream) {
  if (out == nullptr) return fail(nullptr, SIGNMUON_E_INVALID, "null out-pointer");
  *out = nullptr;
  if (!(beta >= 0.f && beta < 1.f)) return fail(nullptr, SIGNMUON_E_INVALID, "beta must be in [0, 1)");
  if (!(lambda >= 0.f)) return fail(nullptr, SIGNMUON_E_INVALID, "lambda must be >= 0");
  if (!(eps > 0.f)) return fail(nullptr, SIGNMUON_E_INVALID, "eps must be > 0");
  signmuon_t h = new (std::nothrow) signmuon_ctx();
  if (!h) return fail(nullptr, SIGNMUON_E_NOMEM, "host allocation failed");
  std::string err;
  int rc = sm::make_plan(shapes, n_mats, M, K, scale, P, flags, &h->plan, &err);
  if (rc) {
    delete h;
    return fail(nullptr, rc, err);
  }
  h->M = M; h->K = K; h->scale = scale; h->P = P;
  h->beta = beta; h->lambda = lambda; h->eps = eps; h->flags = flags;
  h->stream = reinterpret_cast<cudaStream_t>(stream);
  h->vote_only = (flags & SIGNMUON_VOTE_ONLY) != 0;
  if (flags & SIGNMUON_NS_QUINTIC) { h->ns_a = 15.f / 8.f; h->ns_b = -10.f / 8.f; h->ns_c = 3.f / 8.f; }
  cudaError_t e = cudaGetDevice(&h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->n_sm, cudaDevAttrMultiProcessorCount, h->device);
  if (e == cudaSuccess) e = cudaMallocHost(&h->h_status, 2 * sizeof(int));
  if (e != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return fail(nullptr, SIGNMUON_E_CUDA, std::string("CUDA unavailable: ") + cudaGetErrorString(e));
  }
  h->h_status[0] = h->h_status[1] = 0;
  auto bail = [&](int code) {
    g_noh_err = h->err;
    signmuon_destroy(h);
    return code;
  };
  if ((rc = dalloc(h, &h->status, 2))) return bail(rc);
  if (cudaMemset(h->status, 0, 2 * sizeof(int)) != cudaSuccess) return bail(fail(h, SIGNMUON_E_CUDA, "memset"));
  if (h->vote_only) {
    *out = h;
    return SIGNMUON_OK;
  }
  const Plan& p = h->plan;
  if ((rc = upload(h, &h->d_mats, p.mats))) return bail(rc);
  if ((rc = upload(h, &h->d_groups, p.groups))) return bail(rc);
  if ((rc = upload(h, &h->d_group_mats, p.group_mats))) return bail(rc);
  if ((rc = upload(h, &h->d_mat_off, p.mat_off))) return bail(rc);
  if ((rc = upload(h, &h->d_chunks, p.chunks))) return bail(rc);
  if ((rc = upload(h, &h->d_mat_chunk0, p.mat_chunk0))) return bail(rc);
  if ((rc = upload(h, &h->d_mat_nchunks, p.mat_nchunks))) return bail(rc);
  if ((rc = upload(h, &h->d_stage_off, p.stage_off))) return bail(rc);
  for (int op = 0; op < 3; ++op)
    for (int s = 0; s < 2; ++s) {
      if ((rc = upload(h, &h->d_tiles[op][s], p.tiles[op][s].groups))) return bail(rc);
      // a launch of the tensor-core kernel runs min(tiles, SMs / 2) clusters
      const int total = p.tiles[op][s].total;
      const int ncl = std::min(total, h->n_sm / 2);
      if (!p.fp32 && ncl > 0) {
        const std::vector<int> sched = sm::tile_schedule(p.tiles[op][s], ncl, nullptr, nullptr);
        if (!sched.empty() && (rc = upload(h, &h->d_sched[op][s], sched))) return bail(rc);
      }
    }
  if ((rc = upload(h, &h->d_pi_tiles, p.pi_tiles))) return bail(rc);
  if ((rc = upload(h, &h->d_pi_slices, p.pi_slices))) return bail(rc);
  if ((rc = upload(h, &h->d_uoff, p.uoff))) return bail(rc);
  if ((rc = upload(h, &h->d_prob_g, p.prob_g))) return bail(rc);
  if ((rc = upload(h, &h->d_prob_gld, p.prob_gld))) return bail(rc);
  if ((rc = upload(h, &h->d_prob_aoff, p.prob_aoff))) return bail(rc);
  const int64_t esz = p.fp32 ? 4 : 2;
  if ((rc = dalloc(h, &h->Mom, (int64_t)M * p.dpad))) return bail(rc);
  if ((rc = dalloc(h, &h->U, (int64_t)M * p.dpad))) return bail(rc);
  for (int i = 0; i < 2; ++i) {
    uint8_t* x = nullptr;
    if ((rc = dalloc(h, &x, p.x_elems * esz))) return bail(rc);
    h->X[i] = x;
  }
  {
    uint8_t* x = nullptr;
    if ((rc = dalloc(h, &x, p.a_elems * esz))) return bail(rc);
    h->A = x;
    if (p.quintic || p.gram_ns) {
      if ((rc = dalloc(h, &x, p.a_elems * esz))) return bail(rc);
      h->B = x;
    } else {
      h->B = h->A;
    }
    if (p.gram_ns) {
      if ((rc = dalloc(h, &x, p.a_elems * esz))) return bail(rc);
      h->A2 = x;
      for (int i = 0; i < 2; ++i) {
        if ((rc = dalloc(h, &x, p.a_elems * esz))) return bail(rc);
        h->Q[i] = x;
      }
    }
  }
  if ((rc = dalloc(h, &h->bits, (int64_t)M * p.nb_pad))) return bail(rc);
  if (flags & SIGNMUON_TERNARY) {
    if ((rc = dalloc(h, &h->sign8, (int64_t)M * p.dpad))) return bail(rc);
    if (cudaMemset(h->sign8, 0, (size_t)M * p.dpad) != cudaSuccess) return bail(fail(h, SIGNMUON_E_CUDA, "memset"));
  }
  if ((rc = dalloc(h, &h->D, p.dpad))) return bail(rc);
  if ((rc = dalloc(h, &h->partials, (int64_t)p.chunks.size() * M))) return bail(rc);
  if ((rc = dalloc(h, &h->scale_v, (int64_t)M * p.n_mats))) return bail(rc);
  if ((rc = dalloc(h, &h->coef_apply, (int64_t)M * p.n_mats))) return bail(rc);
  if ((rc = dalloc(h, &h->coef_square, (int64_t)M * p.n_mats))) return bail(rc);
  if (p.gram_ns && (rc = dalloc(h, &h->coef_gram, (int64_t)M * p.n_mats))) return bail(rc);
  if ((rc = dalloc(h, &h->pi_u, p.u_elems))) return bail(rc);
  if ((rc = dalloc(h, &h->pi_y, p.u_elems))) return bail(rc);
  if ((rc = dalloc(h, &h->pi_part, p.part_elems))) return bail(rc);
  if ((rc = dalloc(h, &h->pi_cnt, (int64_t)M * p.n_mats))) return bail(rc);
  if ((rc = dalloc(h, &h->pi_inv, (int64_t)M * p.n_mats))) return bail(rc);
  if ((rc = dalloc(h, &h->pi_sq, (int64_t)p.pi_slices.size()))) return bail(rc);
  if (cudaMemset(h->pi_cnt, 0, (size_t)M * p.n_mats * sizeof(int)) != cudaSuccess)
    return bail(fail(h, SIGNMUON_E_CUDA, "memset"));
  if (flags & SIGNMUON_PI_WARM) {
    // zero state: the first power iteration of every problem starts cold
    if ((rc = dalloc(h, &h->pi_u1, p.u_elems_one))) return bail(rc);
    if (cudaMemset(h->pi_u, 0, (size_t)p.u_elems * 4) != cudaSuccess ||
        cudaMemset(h->pi_u1, 0, (size_t)p.u_elems_one * 4) != cudaSuccess)
      return bail(fail(h, SIGNMUON_E_CUDA, "memset"));
  }
  if (cudaMemset(h->Mom, 0, (size_t)M * p.dpad * 4) != cudaSuccess ||
      cudaMemset(h->bits, 0, (size_t)M * p.nb_pad) != cudaSuccess ||
      cudaMemset(h->scale_v, 0, (size_t)M * p.n_mats * 4) != cudaSuccess)
    return bail(fail(h, SIGNMUON_E_CUDA, "memset"));
  if (!p.fp32) {
    // per group: slots 0..3 = X ping, X pong, A, B with 64-row boxes;
    // slots 4..7 = the same tensors with 128-row boxes; when X's column
    // count is a multiple of 64, X ping/pong as 4-D atom views with 2-atom x
    // 64-row boxes at 8/9; slots 10..13 = the first four with 32-row boxes;
    // Gram space: A2, Q0, Q1 with 64-, 128- and 32-row boxes at 14..22
    std::vector<CUtensorMap> maps(p.groups.size() * sm::kMapsPerGroup);
    std::memset(maps.data(), 0, maps.size() * sizeof(CUtensorMap));
    for (size_t g = 0; g < p.groups.size(); ++g) {
      const sm::GroupInfo& gi = p.groups[g];
      const int batch = M * gi.count;
      for (int box = 0; box < 3; ++box) {
        const int br = box == 0 ? 64 : (box == 1 ? 128 : 32);
        CUtensorMap* mm = &maps[g * sm::kMapsPerGroup + (box == 2 ? 10 : 4 * box)];
        for (int i = 0; i < 2; ++i) {
          void* xb = reinterpret_cast<__nv_bfloat16*>(h->X[i]) + gi.x_base;
          if ((rc = encode_map(h, &mm[i], xb, gi.cols, gi.rows, gi.ld, batch, br))) return bail(rc);
        }
        void* ab = reinterpret_cast<__nv_bfloat16*>(h->A) + gi.a_base;
        void* bb = reinterpret_cast<__nv_bfloat16*>(h->B) + gi.a_base;
        if ((rc = encode_map(h, &mm[2], ab, gi.g, gi.g, gi.gld, batch, br))) return bail(rc);
        if ((rc = encode_map(h, &mm[3], bb, gi.g, gi.g, gi.gld, batch, br))) return bail(rc);
        if (p.gram_ns) {
          void* const gbuf[3] = {h->A2, h->Q[0], h->Q[1]};
          for (int j = 0; j < 3; ++j) {
            void* base = reinterpret_cast<__nv_bfloat16*>(gbuf[j]) + gi.a_base;
            CUtensorMap* gm = &maps[g * sm::kMapsPerGroup + sm::mm_slot(sm::MM_A2 + j, box)];
            if ((rc = encode_map(h, gm, base, gi.g, gi.g, gi.gld, batch, br))) return bail(rc);
          }
        }
      }
      if (gi.cols % 64 == 0) {
        for (int i = 0; i < 2; ++i) {
          void* xb = reinterpret_cast<__nv_bfloat16*>(h->X[i]) + gi.x_base;
          if ((rc = encode_map_atoms(h, &maps[g * sm::kMapsPerGroup + 8 + i], xb, gi.cols, gi.rows, gi.ld, batch, 64,
                                     2)))
            return bail(rc);
        }
      }
    }
    uint8_t* m = nullptr;
    if ((rc = dalloc(h, &m, (int64_t)(maps.size() * sizeof(CUtensorMap) + 128)))) return bail(rc);
    h->d_maps = reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(m) + 127) & ~(uintptr_t)127);
    if (cudaMemcpy(h->d_maps, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice) != cudaSuccess)
      return bail(fail(h, SIGNMUON_E_CUDA, "tensor map upload"));
  }
  if (cudaDeviceSynchronize() != cudaSuccess) return bail(fail(h, SIGNMUON_E_CUDA, "init sync"));
  *out = h;
  return SIGNMUON_OK;
}

int signmuon_set_ns_coeffs(signmuon_t h, const float* c, int n) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, false);
  if (rc) return rc;
  if (c == nullptr) return fail(h, SIGNMUON_E_INVALID, "null coefficients");
  if (h->plan.quintic) {
    if (n != 3) return fail(h, SIGNMUON_E_INVALID, "quintic NS takes 3 coefficients");
    h->ns_a = c[0]; h->ns_b = c[1]; h->ns_c = c[2];
  } else {
    if (n != 2) return fail(h, SIGNMUON_E_INVALID, "NS takes 2 coefficients (a, b)");
    h->ns_a = c[0]; h->ns_b = c[1];
  }
  return SIGNMUON_OK;
}

// The step in two parts, so that the signs can cross a collective in
// between (one worker per GPU, [paper] Algorithm 2's exchange).
// local_part: momentum -> scale -> PolarNS -> signs of the handle's M workers,
// worker m's at dst + m*stride (packed bits, or int8 ternary signs).
static void local_part(signmuon_t h, const float* W, const sm::WorkerPtrs& gp, uint8_t* dst, int64_t stride) {
  const Plan& p = h->plan;
  cudaStream_t s = h->stream;
  {
    ProfScope ps(h, 0);
    sm::launch_momentum(s, gp, W, h->Mom, p.dpad, h->M, h->beta, h->lambda, h->X[0], p.fp32 ? 0 : 1, h->d_chunks,
                        (int)p.chunks.size(), h->d_mats, h->d_groups, h->partials);
  }
  fro_finalize(h, h->M);
  const bool ternary = (h->flags & SIGNMUON_TERNARY) != 0;
  int8_t* dst8 = reinterpret_cast<int8_t*>(dst);
  if (h->flags & SIGNMUON_POLAR_AFTER_ONLY) {
    // after-only placement: the signs of the momentum itself
    h->u_valid = false;
    ProfScope ps(h, 6);
    if (ternary) sm::launch_sign8(s, h->Mom, p.dpad, p.d, dst8, stride, h->M);
    else sm::launch_pack(s, h->Mom, p.dpad, p.d, dst, stride, h->M);
    return;
  }
  // The one-bit signs come out of the last Newton-Schulz GEMM itself (K > 0,
  // bf16 path, see signs_in_gemm); U is written only when kept for get_polar.
  // The int8 ternary signs come out of the last GEMM on the bf16 path (any
  // shapes: a chunk's 32 signs are stored bytewise where unaligned).
  const bool fused = !ternary && signs_in_gemm(h);
  const bool fused8 = ternary && !p.fp32 && h->K > 0;
  h->u_valid = !(fused || fused8) || (h->flags & SIGNMUON_KEEP_POLAR) != 0;
  if (fused) {
    // (an error here is the runtime's last error, which the step's status read reports)
    if (signs_ragged(h)) cudaMemsetAsync(dst, 0, (size_t)h->M * (size_t)stride, s);
    run_ns(h, h->K, h->M, strided_ptrs(h->Mom, p.dpad, h->M), h->u_valid ? h->U : nullptr, p.dpad,
           reinterpret_cast<uint32_t*>(dst), stride / 4);
  } else if (fused8) {
    h->final_sign8 = dst8;
    h->final_sign8_stride = stride;
    run_ns(h, h->K, h->M, strided_ptrs(h->Mom, p.dpad, h->M), h->u_valid ? h->U : nullptr, p.dpad);
    h->final_sign8 = nullptr;
    h->final_sign8_stride = 0;
  } else {
    run_ns(h, h->K, h->M, strided_ptrs(h->Mom, p.dpad, h->M), h->U, p.dpad);
    ProfScope ps(h, 6);
    if (ternary) sm::launch_sign8(s, h->U, p.dpad, p.d, dst8, stride, h->M);
    else sm::launch_pack(s, h->U, p.dpad, p.d, dst, stride, h->M);
  }
}

// vote_part: the majority of Mv sign buffers (worker j's at src.p[j], this
// GPU's memory or a peer's), then the post-vote step (PolarNS with the
// handle's K, or with none for the normalised sign step) and the update, or
// the vote fused with the update.
static void vote_part(signmuon_t h, float* W, const sm::WorkerPtrs& src, int Mv, float eta) {
  const Plan& p = h->plan;
  cudaStream_t s = h->stream;
  const int tie = (h->flags & SIGNMUON_TIE_PLUS) ? 1 : 0;
  const bool ternary = (h->flags & SIGNMUON_TERNARY) != 0;
  if (h->flags & (SIGNMUON_POST_POLAR | SIGNMUON_NORMALIZED_SIGN)) {
    const int k_post = (h->flags & SIGNMUON_NORMALIZED_SIGN) ? 0 : h->K;
    {
      ProfScope ps(h, 7);
      if (ternary) {
        // majority -> D, then D staged as the step's input (a one-worker
        // mean, which is D itself) with its sum-of-squares partials
        sm::launch_vote_ternary_major(s, src, Mv, p.d, h->D, tie);
        sm::launch_mean_stage(s, h->D, 0, 1, h->X[0], p.fp32 ? 0 : 1, h->d_chunks, (int)p.chunks.size(), h->d_mats,
                              h->d_groups, h->partials, nullptr);
      } else {
        // the majority goes straight into the step's input (and into D only
        // when K == 0, where the result is the scaled input itself)
        sm::launch_vote_stage(s, src, Mv, h->X[0], p.fp32 ? 0 : 1, h->d_chunks, (int)p.chunks.size(),
                              h->d_mats, h->d_groups, h->partials, k_post == 0 ? h->D : nullptr, tie,
                              stage_streamable(h) ? h->d_stage_off : nullptr);
      }
    }
    fro_finalize(h, 1);
    run_ns(h, k_post, 1, strided_ptrs(h->D, 0, 1), h->D, 0);
    ProfScope ps(h, 12);
    sm::launch_update(s, W, h->D, p.d, eta, h->status);
  } else {
    ProfScope ps(h, 7);
    if (ternary) sm::launch_vote_ternary_update(s, src, Mv, p.d, W, eta, h->status, tie);
    else sm::launch_vote_update(s, src, Mv, p.d, W, eta, h->status, tie);
  }
}

int signmuon_step(signmuon_t h, float* W, const float* const* G, float eta) {
  NvtxRange range("signmuon_step");
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  const Plan& p = h->plan;
  if (W == nullptr || G == nullptr) return fail(h, SIGNMUON_E_INVALID, "null W or G");
  if (!aligned16(W)) return fail(h, SIGNMUON_E_INVALID, "W must be 16-byte aligned");
  for (int m = 0; m < h->M; ++m)
    if (G[m] == nullptr || !aligned16(G[m])) return fail(h, SIGNMUON_E_INVALID, "G[m] null or not 16-byte aligned");
  cudaStream_t s = h->stream;
  CK(h, begin_status(h));
  const sm::WorkerPtrs gp = worker_ptrs(G, h->M);
  if (h->flags & SIGNMUON_MUON_MEAN) {
    // Muon baseline: the workers' mean momentum through one PolarNS
    h->u_valid = false;
    h->bits_valid = false;
    h->dir_valid = true;
    h->dir_in_D = true;
    {
      ProfScope ps(h, 0);
      sm::launch_momentum(s, gp, W, h->Mom, p.dpad, h->M, h->beta, h->lambda, h->X[0], p.fp32 ? 0 : 1, h->d_chunks,
                          (int)p.chunks.size(), h->d_mats, h->d_groups, h->partials);
    }
    fro_finalize(h, h->M);
    {
      ProfScope ps(h, 8);
      sm::launch_mean_stage(s, h->Mom, p.dpad, h->M, h->X[0], p.fp32 ? 0 : 1, h->d_chunks, (int)p.chunks.size(),
                            h->d_mats, h->d_groups, h->partials, h->K == 0 ? h->D : nullptr);
    }
    fro_finalize(h, 1);
    run_ns(h, h->K, 1, strided_ptrs(h->D, 0, 1), h->D, 0);
    ProfScope ps(h, 12);
    sm::launch_update(s, W, h->D, p.d, eta, h->status);
    return finish(h, (h->flags & SIGNMUON_ASYNC) == 0);
  }
  // one bit per entry, or (TERNARY) one int8 sign in {-1, 0, +1}
  const bool ternary = (h->flags & SIGNMUON_TERNARY) != 0;
  h->bits_valid = !ternary;
  h->t_valid = ternary;
  h->dir_valid = true;
  h->dir_in_D = (h->flags & (SIGNMUON_POST_POLAR | SIGNMUON_NORMALIZED_SIGN)) != 0;
  uint8_t* own = ternary ? reinterpret_cast<uint8_t*>(h->sign8) : h->bits;
  const int64_t own_stride = ternary ? p.dpad : p.nb_pad;
  local_part(h, W, gp, own, own_stride);
  vote_part(h, W, byte_ptrs(own, own_stride, h->M), h->M, eta);
  return finish(h, (h->flags & SIGNMUON_ASYNC) == 0);
}

int signmuon_local_signs(signmuon_t h, const float* W, const float* const* G, uint8_t* signs, int64_t stride) {
  NvtxRange range("signmuon_local_signs");
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  const Plan& p = h->plan;
  if (h->flags & SIGNMUON_MUON_MEAN) return fail(h, SIGNMUON_E_UNSUPPORTED, "a SIGNMUON_MUON_MEAN handle sends no signs");
  if (W == nullptr || G == nullptr || signs == nullptr) return fail(h, SIGNMUON_E_INVALID, "null W, G or signs");
  if (!aligned16(W) || !aligned16(signs)) return fail(h, SIGNMUON_E_INVALID, "W and signs must be 16-byte aligned");
  for (int m = 0; m < h->M; ++m)
    if (G[m] == nullptr || !aligned16(G[m])) return fail(h, SIGNMUON_E_INVALID, "G[m] null or not 16-byte aligned");
  const int64_t need = (h->flags & SIGNMUON_TERNARY) ? p.d : p.nb;
  if (stride < need || stride % 16 != 0)
    return fail(h, SIGNMUON_E_INVALID, "stride must be a multiple of 16 bytes and hold one worker's signs");
  CK(h, begin_status(h));
  // the handle's own sign buffers do not hold these signs
  h->bits_valid = false;
  h->t_valid = false;
  h->dir_valid = false;
  local_part(h, W, worker_ptrs(G, h->M), signs, stride);
  return finish(h, (h->flags & SIGNMUON_ASYNC) == 0);
}

int signmuon_vote_step(signmuon_t h, float* W, const uint8_t* signs, int64_t stride, int M, float eta) {
  NvtxRange range("signmuon_vote_step");
  const bool post = h != nullptr && (h->flags & (SIGNMUON_POST_POLAR | SIGNMUON_NORMALIZED_SIGN)) != 0;
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, post);
  if (rc) return rc;
  const Plan& p = h->plan;
  if (h->flags & SIGNMUON_MUON_MEAN) return fail(h, SIGNMUON_E_UNSUPPORTED, "a SIGNMUON_MUON_MEAN handle takes no vote");
  if (M < 1 || M > sm::kMaxWorkers) return fail(h, SIGNMUON_E_INVALID, "M must be in [1, 256]");
  if (W == nullptr || signs == nullptr) return fail(h, SIGNMUON_E_INVALID, "null W or signs");
  if (!aligned16(W) || !aligned16(signs)) return fail(h, SIGNMUON_E_INVALID, "W and signs must be 16-byte aligned");
  const int64_t need = (h->flags & SIGNMUON_TERNARY) ? p.d : p.nb;
  if (stride < need || stride % 16 != 0)
    return fail(h, SIGNMUON_E_INVALID, "stride must be a multiple of 16 bytes and hold one worker's signs");
  CK(h, begin_status(h));
  h->dir_valid = post;  // D is kept only by the post-vote steps
  h->dir_in_D = post;
  vote_part(h, W, byte_ptrs(signs, stride, M), M, eta);
  return finish(h, (h->flags & SIGNMUON_ASYNC) == 0);
}

int signmuon_vote_step_ptrs(signmuon_t h, float* W, const uint8_t* const* signs, int M, float eta) {
  NvtxRange range("signmuon_vote_step_ptrs");
  const bool post = h != nullptr && (h->flags & (SIGNMUON_POST_POLAR | SIGNMUON_NORMALIZED_SIGN)) != 0;
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, post);
  if (rc) return rc;
  if (h->flags & SIGNMUON_MUON_MEAN) return fail(h, SIGNMUON_E_UNSUPPORTED, "a SIGNMUON_MUON_MEAN handle takes no vote");
  if (M < 1 || M > sm::kMaxWorkers) return fail(h, SIGNMUON_E_INVALID, "M must be in [1, 256]");
  if (W == nullptr || signs == nullptr) return fail(h, SIGNMUON_E_INVALID, "null W or signs");
  if (!aligned16(W)) return fail(h, SIGNMUON_E_INVALID, "W must be 16-byte aligned");
  for (int m = 0; m < M; ++m)
    if (signs[m] == nullptr || !aligned16(signs[m]))
      return fail(h, SIGNMUON_E_INVALID, "signs[m] null or not 16-byte aligned");
  CK(h, begin_status(h));
  h->dir_valid = post;
  h->dir_in_D = post;
  sm::WorkerPtrs sp{};
  for (int m = 0; m < M; ++m) sp.p[m] = reinterpret_cast<const float*>(signs[m]);
  vote_part(h, W, sp, M, eta);
  return finish(h, (h->flags & SIGNMUON_ASYNC) == 0);
}

int signmuon_sums_step(signmuon_t h, float* W, const void* sums, float eta) {
  NvtxRange range("signmuon_sums_step");
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  const Plan& p = h->plan;
  if (h->flags & SIGNMUON_MUON_MEAN) return fail(h, SIGNMUON_E_UNSUPPORTED, "a SIGNMUON_MUON_MEAN handle takes no vote");
  if (W == nullptr || sums == nullptr) return fail(h, SIGNMUON_E_INVALID, "null W or sums");
  if (!aligned16(W) || !aligned16(sums)) return fail(h, SIGNMUON_E_INVALID, "W and sums must be 16-byte aligned");
  cudaStream_t s = h->stream;
  CK(h, begin_status(h));
  const int tie = (h->flags & SIGNMUON_TIE_PLUS) ? 1 : 0;
  {
    // the majority into D; for the post-vote steps D is then staged as
    // their input (a one-worker mean, which is D itself)
    ProfScope ps(h, 7);
    sm::launch_sums_major(s, sums, (h->flags & SIGNMUON_ACC_INT8) ? 1 : 0, p.d, h->D, tie);
  }
  if (h->flags & (SIGNMUON_POST_POLAR | SIGNMUON_NORMALIZED_SIGN)) {
    const int k_post = (h->flags & SIGNMUON_NORMALIZED_SIGN) ? 0 : h->K;
    {
      ProfScope ps(h, 7);
      sm::launch_mean_stage(s, h->D, 0, 1, h->X[0], p.fp32 ? 0 : 1, h->d_chunks, (int)p.chunks.size(), h->d_mats,
                            h->d_groups, h->partials, nullptr);
    }
    fro_finalize(h, 1);
    run_ns(h, k_post, 1, strided_ptrs(h->D, 0, 1), h->D, 0);
  }
  {
    ProfScope ps(h, 12);
    sm::launch_update(s, W, h->D, p.d, eta, h->status);
  }
  h->dir_valid = true;
  h->dir_in_D = true;
  return finish(h, (h->flags & SIGNMUON_ASYNC) == 0);
}

int signmuon_step_host(signmuon_t h, float* W_host, const float* const* G_host, float eta) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  const Plan& p = h->plan;
  if (W_host == nullptr || G_host == nullptr) return fail(h, SIGNMUON_E_INVALID, "null W or G");
  for (int m = 0; m < h->M; ++m)
    if (G_host[m] == nullptr) return fail(h, SIGNMUON_E_INVALID, "null G[m]");
  // first use: each piece is made once, so a call after a failed one
  // finishes the set-up
  if (!h->hw_W && (rc = dalloc(h, &h->hw_W, p.dpad))) return rc;
  for (int b = 0; b < 2; ++b)
    if (!h->hw_G[b] && (rc = dalloc(h, &h->hw_G[b], (int64_t)h->M * p.dpad))) return rc;
  if (!h->copy_stream) CK(h, cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking));
  auto make_event = [&](cudaEvent_t* e, bool record) -> int {
    if (*e) return SIGNMUON_OK;
    CK(h, cudaEventCreateWithFlags(e, cudaEventDisableTiming));
    if (record) CK(h, cudaEventRecord(*e, h->stream));
    return SIGNMUON_OK;
  };
  for (int b = 0; b < 2; ++b)
    if ((rc = make_event(&h->g_ready[b], false)) || (rc = make_event(&h->g_free[b], true))) return rc;
  if ((rc = make_event(&h->w_ready, false)) || (rc = make_event(&h->w_free, true))) return rc;
  const int b = h->hw_next;
  h->hw_next ^= 1;
  cudaStream_t s = h->stream, cs = h->copy_stream;
  // Every host-to-device copy goes on the copy stream: first the gradients
  // into buffer b, once the step that read it last (two calls ago) is done;
  // then W, once the previous call's W has gone back to the host.  With
  // SIGNMUON_ASYNC the gradients come in while the step of the call before
  // still runs, so the host-to-device link stays busy.
  CK(h, cudaStreamWaitEvent(cs, h->g_free[b], 0));
  std::vector<const float*> gd(h->M);
  for (int m = 0; m < h->M; ++m) {
    gd[m] = h->hw_G[b] + (int64_t)m * p.dpad;
    CK(h, cudaMemcpyAsync(const_cast<float*>(gd[m]), G_host[m], (size_t)p.d * 4, cudaMemcpyHostToDevice, cs));
  }
  CK(h, cudaEventRecord(h->g_ready[b], cs));
  CK(h, cudaStreamWaitEvent(cs, h->w_free, 0));
  CK(h, cudaMemcpyAsync(h->hw_W, W_host, (size_t)p.d * 4, cudaMemcpyHostToDevice, cs));
  CK(h, cudaEventRecord(h->w_ready, cs));
  CK(h, cudaStreamWaitEvent(s, h->g_ready[b], 0));
  CK(h, cudaStreamWaitEvent(s, h->w_ready, 0));
  const unsigned saved = h->flags;
  h->flags |= SIGNMUON_ASYNC;
  rc = signmuon_step(h, h->hw_W, gd.data(), eta);
  h->flags = saved;
  if (rc) return rc;
  CK(h, cudaEventRecord(h->g_free[b], s));
  CK(h, cudaMemcpyAsync(W_host, h->hw_W, (size_t)p.d * 4, cudaMemcpyDeviceToHost, s));
  CK(h, cudaEventRecord(h->w_free, s));
  return (h->flags & SIGNMUON_ASYNC) ? SIGNMUON_OK : signmuon_sync(h);
}

// ---- CUDA IPC: map a buffer of one process into another (peer GPUs) ------
namespace {
typedef CUresult (*AddrRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
AddrRangeFn get_addr_range() {
  static AddrRangeFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddrRangeFn>(f);
  }
  return fn;
}
}  // namespace

int signmuon_ipc_get_handle(const void* dev_ptr, void* handle, int64_t* offset) {
  if (dev_ptr == nullptr || handle == nullptr || offset == nullptr)
    return fail(nullptr, SIGNMUON_E_INVALID, "ipc_get_handle: null pointer");
  AddrRangeFn range = get_addr_range();
  if (!range) return fail(nullptr, SIGNMUON_E_CUDA, "cuMemGetAddressRange is not available from the driver");
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return fail(nullptr, SIGNMUON_E_INVALID, "ipc_get_handle: not a device allocation");
  cudaIpcMemHandle_t hd;
  const cudaError_t e = cudaIpcGetMemHandle(&hd, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(nullptr, SIGNMUON_E_CUDA, std::string("cudaIpcGetMemHandle: ") + cudaGetErrorString(e));
  }
  static_assert(sizeof(cudaIpcMemHandle_t) == SIGNMUON_IPC_HANDLE_BYTES, "IPC handle size");
  std::memcpy(handle, &hd, sizeof(hd));
  *offset = (int64_t)(reinterpret_cast<uintptr_t>(dev_ptr) - (uintptr_t)base);
  return SIGNMUON_OK;
}

int signmuon_ipc_open(const void* handle, void** base) {
  if (handle == nullptr || base == nullptr) return fail(nullptr, SIGNMUON_E_INVALID, "ipc_open: null pointer");
  cudaIpcMemHandle_t hd;
  std::memcpy(&hd, handle, sizeof(hd));
  *base = nullptr;
  const cudaError_t e = cudaIpcOpenMemHandle(base, hd, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(nullptr, SIGNMUON_E_CUDA, std::string("cudaIpcOpenMemHandle: ") + cudaGetErrorString(e));
  }
  return SIGNMUON_OK;
}

int signmuon_ipc_close(void* base) {
  if (base == nullptr) return fail(nullptr, SIGNMUON_E_INVALID, "ipc_close: null pointer");
  const cudaError_t e = cudaIpcCloseMemHandle(base);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(nullptr, SIGNMUON_E_CUDA, std::string("cudaIpcCloseMemHandle: ") + cudaGetErrorString(e));
  }
  return SIGNMUON_OK;
}

int signmuon_sync(signmuon_t h) {
  if (h == nullptr) return fail(nullptr, SIGNMUON_E_INVALID, "null handle");
  DeviceGuard dev_guard(h);
  CK(h, cudaStreamSynchronize(h->stream));
  if (!h->pending) return SIGNMUON_OK;
  h->pending = false;
  if (h->h_status[1] != 0) return fail(h, SIGNMUON_E_TIMEOUT, "a kernel's bounded wait expired");
  if (h->h_status[0] != 0) return fail(h, SIGNMUON_E_NONFINITE, "a momentum norm is NaN or Inf; W was not updated");
  return SIGNMUON_OK;
}

int signmuon_vote(signmuon_t h, const uint8_t* const* signs, int64_t d, void* sums, int8_t* majority) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, false);
  if (rc) return rc;
  if (d < 0 || signs == nullptr) return fail(h, SIGNMUON_E_INVALID, "bad vote arguments");
  for (int m = 0; m < h->M; ++m)
    if (signs[m] == nullptr || !aligned16(signs[m])) return fail(h, SIGNMUON_E_INVALID, "signs[m] null or misaligned");
  if ((sums && !aligned16(sums)) || (majority && !aligned16(majority)))
    return fail(h, SIGNMUON_E_INVALID, "sums/majority must be 16-byte aligned");
  sm::WorkerPtrs sp{};
  for (int m = 0; m < h->M; ++m) sp.p[m] = reinterpret_cast<const float*>(signs[m]);
  sm::launch_vote(h->stream, sp, h->M, d, sums, (h->flags & SIGNMUON_ACC_INT8) ? 1 : 0, majority,
                  (h->flags & SIGNMUON_TIE_PLUS) ? 1 : 0);
  CK(h, cudaGetLastError());
  return SIGNMUON_OK;
}

int signmuon_pack(signmuon_t h, const float* U, int64_t d, uint8_t* out) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, false);
  if (rc) return rc;
  if (d < 0 || (d > 0 && (U == nullptr || out == nullptr))) return fail(h, SIGNMUON_E_INVALID, "bad pack arguments");
  if (!aligned16(U) || !aligned16(out)) return fail(h, SIGNMUON_E_INVALID, "U/out must be 16-byte aligned");
  sm::launch_pack(h->stream, U, 0, d, out, 0, 1);
  CK(h, cudaGetLastError());
  return SIGNMUON_OK;
}

int signmuon_sign_ternary(signmuon_t h, const float* U, int64_t d, int8_t* out) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, false);
  if (rc) return rc;
  if (d < 0 || (d > 0 && (U == nullptr || out == nullptr))) return fail(h, SIGNMUON_E_INVALID, "bad sign arguments");
  if (!aligned16(U) || !aligned16(out)) return fail(h, SIGNMUON_E_INVALID, "U/out must be 16-byte aligned");
  sm::launch_sign8(h->stream, U, 0, d, out, 0, 1);
  CK(h, cudaGetLastError());
  return SIGNMUON_OK;
}

int signmuon_vote_ternary(signmuon_t h, const int8_t* const* signs, int64_t d, void* sums, int8_t* majority) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, false);
  if (rc) return rc;
  if (d < 0 || signs == nullptr) return fail(h, SIGNMUON_E_INVALID, "bad vote arguments");
  for (int m = 0; m < h->M; ++m)
    if (signs[m] == nullptr || !aligned16(signs[m])) return fail(h, SIGNMUON_E_INVALID, "signs[m] null or misaligned");
  if ((sums && !aligned16(sums)) || (majority && !aligned16(majority)))
    return fail(h, SIGNMUON_E_INVALID, "sums/majority must be 16-byte aligned");
  sm::WorkerPtrs sp{};
  for (int m = 0; m < h->M; ++m) sp.p[m] = reinterpret_cast<const float*>(signs[m]);
  sm::launch_vote_ternary(h->stream, sp, h->M, d, sums, (h->flags & SIGNMUON_ACC_INT8) ? 1 : 0, majority,
                          (h->flags & SIGNMUON_TIE_PLUS) ? 1 : 0);
  CK(h, cudaGetLastError());
  return SIGNMUON_OK;
}

int signmuon_apply_update(signmuon_t h, float* W, const float* D, int64_t d, float eta) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, false);
  if (rc) return rc;
  if (d < 0 || (d > 0 && (W == nullptr || D == nullptr))) return fail(h, SIGNMUON_E_INVALID, "bad update arguments");
  if (!aligned16(W) || !aligned16(D)) return fail(h, SIGNMUON_E_INVALID, "W/D must be 16-byte aligned");
  sm::launch_update(h->stream, W, D, d, eta, nullptr);
  CK(h, cudaGetLastError());
  return SIGNMUON_OK;
}

int signmuon_polar(signmuon_t h, const float* const* X, float* const* U) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  const Plan& p = h->plan;
  if (X == nullptr || U == nullptr) return fail(h, SIGNMUON_E_INVALID, "null X or U");
  for (int m = 0; m < h->M; ++m)
    if (!X[m] || !U[m] || !aligned16(X[m]) || !aligned16(U[m]))
      return fail(h, SIGNMUON_E_INVALID, "X[m]/U[m] null or misaligned");
  cudaStream_t s = h->stream;
  CK(h, begin_status(h));
  const sm::WorkerPtrs xp = worker_ptrs(X, h->M);
  sm::launch_stage(s, xp, h->M, h->X[0], p.fp32 ? 0 : 1, h->d_chunks, (int)p.chunks.size(), h->d_mats, h->d_groups,
                   h->partials);
  fro_finalize(h, h->M);
  run_ns(h, h->K, h->M, xp, h->U, p.dpad);
  h->u_valid = true;
  for (int m = 0; m < h->M; ++m)
    CK(h, cudaMemcpyAsync(U[m], h->U + (int64_t)m * p.dpad, (size_t)p.d * 4, cudaMemcpyDeviceToDevice, s));
  return finish(h, (h->flags & SIGNMUON_ASYNC) == 0);
}

int signmuon_get_momentum(signmuon_t h, int m, float* dst) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  if (m < 0 || m >= h->M || !dst) return fail(h, SIGNMUON_E_INVALID, "bad worker index or null dst");
  CK(h, cudaMemcpyAsync(dst, h->Mom + (int64_t)m * h->plan.dpad, (size_t)h->plan.d * 4, cudaMemcpyDeviceToDevice,
                        h->stream));
  return SIGNMUON_OK;
}

int signmuon_set_momentum(signmuon_t h, int m, const float* src) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  if (m < 0 || m >= h->M || !src) return fail(h, SIGNMUON_E_INVALID, "bad worker index or null src");
  CK(h, cudaMemcpyAsync(h->Mom + (int64_t)m * h->plan.dpad, src, (size_t)h->plan.d * 4, cudaMemcpyDeviceToDevice,
                        h->stream));
  return SIGNMUON_OK;
}

// the warm power-iteration state: which = 0 (M-worker problems), 1 (one problem set)
static int pi_state_buffer(signmuon_t h, int which, float** buf, int64_t* n) {
  if (!(h->flags & SIGNMUON_PI_WARM)) return fail(h, SIGNMUON_E_UNSUPPORTED, "the handle has no SIGNMUON_PI_WARM state");
  if (which == 0) {
    *buf = h->pi_u;
    *n = h->plan.u_elems;
  } else if (which == 1) {
    *buf = h->pi_u1;
    *n = h->plan.u_elems_one;
  } else {
    return fail(h, SIGNMUON_E_INVALID, "which must be 0 (workers) or 1 (one problem set)");
  }
  return SIGNMUON_OK;
}

int signmuon_get_pi_state(signmuon_t h, int which, float* dst) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  float* buf = nullptr;
  int64_t n = 0;
  if ((rc = pi_state_buffer(h, which, &buf, &n))) return rc;
  if (!dst) return fail(h, SIGNMUON_E_INVALID, "null dst");
  CK(h, cudaMemcpyAsync(dst, buf, (size_t)n * 4, cudaMemcpyDeviceToDevice, h->stream));
  return SIGNMUON_OK;
}

int signmuon_set_pi_state(signmuon_t h, int which, const float* src) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  float* buf = nullptr;
  int64_t n = 0;
  if ((rc = pi_state_buffer(h, which, &buf, &n))) return rc;
  if (!src) return fail(h, SIGNMUON_E_INVALID, "null src");
  CK(h, cudaMemcpyAsync(buf, src, (size_t)n * 4, cudaMemcpyDeviceToDevice, h->stream));
  return SIGNMUON_OK;
}

int signmuon_get_polar(signmuon_t h, int m, float* dst) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  if (m < 0 || m >= h->M || !dst) return fail(h, SIGNMUON_E_INVALID, "bad worker index or null dst");
  if (!h->u_valid)
    return fail(h, SIGNMUON_E_UNSUPPORTED,
                "the last step packed its signs inside the Newton-Schulz GEMM and kept no U; create the handle "
                "with SIGNMUON_KEEP_POLAR");
  CK(h, cudaMemcpyAsync(dst, h->U + (int64_t)m * h->plan.dpad, (size_t)h->plan.d * 4, cudaMemcpyDeviceToDevice,
                        h->stream));
  return SIGNMUON_OK;
}

int signmuon_get_signs(signmuon_t h, int m, uint8_t* dst) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  if (m < 0 || m >= h->M || !dst) return fail(h, SIGNMUON_E_INVALID, "bad worker index or null dst");
  if (!h->bits_valid)
    return fail(h, SIGNMUON_E_UNSUPPORTED,
                (h->flags & SIGNMUON_TERNARY)     ? "a SIGNMUON_TERNARY step sends int8 signs: use signmuon_get_ternary_signs"
                : (h->flags & SIGNMUON_MUON_MEAN) ? "a SIGNMUON_MUON_MEAN step packs no signs"
                                                  : "no step has left its signs in the handle (signmuon_local_signs "
                                                    "writes them to the caller's buffer)");
  CK(h, cudaMemcpyAsync(dst, h->bits + (int64_t)m * h->plan.nb_pad, (size_t)h->plan.nb, cudaMemcpyDeviceToDevice,
                        h->stream));
  return SIGNMUON_OK;
}

int signmuon_get_ternary_signs(signmuon_t h, int m, int8_t* dst) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  if (m < 0 || m >= h->M || !dst) return fail(h, SIGNMUON_E_INVALID, "bad worker index or null dst");
  if (!h->t_valid)
    return fail(h, SIGNMUON_E_UNSUPPORTED, "no SIGNMUON_TERNARY step has left its signs in the handle");
  CK(h, cudaMemcpyAsync(dst, h->sign8 + (int64_t)m * h->plan.dpad, (size_t)h->plan.d, cudaMemcpyDeviceToDevice,
                        h->stream));
  return SIGNMUON_OK;
}

int signmuon_get_direction(signmuon_t h, float* dst) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  if (!dst || !aligned16(dst)) return fail(h, SIGNMUON_E_INVALID, "null or misaligned dst");
  const Plan& p = h->plan;
  if (!h->dir_valid)
    return fail(h, SIGNMUON_E_UNSUPPORTED,
                "no D to give: no step yet, or the last vote (signmuon_vote_step) was fused with the update");
  if (h->dir_in_D) {
    CK(h, cudaMemcpyAsync(dst, h->D, (size_t)p.d * 4, cudaMemcpyDeviceToDevice, h->stream));
  } else if (h->flags & SIGNMUON_TERNARY) {
    // the step fuses the vote into the update; recompute the majority from
    // the last step's ternary signs
    sm::launch_vote_ternary_major(h->stream, byte_ptrs(reinterpret_cast<const uint8_t*>(h->sign8), p.dpad, h->M),
                                  h->M, p.d, dst, (h->flags & SIGNMUON_TIE_PLUS) ? 1 : 0);
    CK(h, cudaGetLastError());
  } else {
    // the step fuses the vote into the update; recompute the majority from
    // the last step's packed signs
    sm::launch_vote_major(h->stream, byte_ptrs(h->bits, p.nb_pad, h->M), h->M, p.d, dst,
                          (h->flags & SIGNMUON_TIE_PLUS) ? 1 : 0);
    CK(h, cudaGetLastError());
  }
  return SIGNMUON_OK;
}

int signmuon_get_scales(signmuon_t h, float* dst_host) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  if (!dst_host) return fail(h, SIGNMUON_E_INVALID, "null dst");
  CK(h, cudaMemcpyAsync(dst_host, h->scale_v, (size_t)h->M * h->plan.n_mats * 4, cudaMemcpyDeviceToHost, h->stream));
  CK(h, cudaStreamSynchronize(h->stream));
  return SIGNMUON_OK;
}

int signmuon_profile(signmuon_t h, int enable) {
  if (h == nullptr) return fail(nullptr, SIGNMUON_E_INVALID, "null handle");
  DeviceGuard dev_guard(h);
  prof_collect(h);
  h->prof = enable != 0;
  return SIGNMUON_OK;
}

int signmuon_profile_read(signmuon_t h, double* ms, int64_t* launches, int n) {
  if (h == nullptr) return fail(nullptr, SIGNMUON_E_INVALID, "null handle");
  DeviceGuard dev_guard(h);
  prof_collect(h);
  for (int k = 0; k < n && k < SIGNMUON_PROF_KINDS; ++k) {
    if (ms) ms[k] = h->prof_ms[k];
    if (launches) launches[k] = h->prof_n[k];
    h->prof_ms[k] = 0.0;
    h->prof_n[k] = 0;
  }
  return SIGNMUON_OK;
}

int signmuon_get_gram(signmuon_t h, int m, int mat, float* dst_host) {
  DeviceGuard dev_guard(h);
  int rc = check_handle(h, true);
  if (rc) return rc;
  const Plan& p = h->plan;
  if (m < 0 || m >= h->M || mat < 0 || mat >= p.n_mats || !dst_host)
    return fail(h, SIGNMUON_E_INVALID, "bad worker/matrix index or null dst");
  const sm::MatInfo& mi = p.mats[mat];
  const sm::GroupInfo& g = p.groups[mi.group];
  const int64_t off = g.a_base + (int64_t)(m * g.count + mi.q) * g.g * g.gld;
  const size_t esz = p.fp32 ? 4 : 2;
  std::vector<uint8_t> buf((size_t)g.g * g.gld * esz);
  CK(h, cudaStreamSynchronize(h->stream));
  CK(h, cudaMemcpy(buf.data(), reinterpret_cast<uint8_t*>(h->A) + off * esz, buf.size(), cudaMemcpyDeviceToHost));
  for (int r = 0; r < g.g; ++r)
    for (int c = 0; c < g.g; ++c) {
      const size_t i = (size_t)r * g.gld + c;
      if (p.fp32) {
        dst_host[(size_t)r * g.g + c] = reinterpret_cast<const float*>(buf.data())[i];
      } else {
        const uint32_t bits = (uint32_t)reinterpret_cast<const uint16_t*>(buf.data())[i] << 16;
        float f;
        std::memcpy(&f, &bits, 4);
        dst_host[(size_t)r * g.g + c] = f;
      }
    }
  return SIGNMUON_OK;
}

int signmuon_info(signmuon_t h, int64_t* out, int n) {
  if (h == nullptr) return fail(nullptr, SIGNMUON_E_INVALID, "null handle");
  if (!out) return fail(h, SIGNMUON_E_INVALID, "null out");
  fill_info(h->plan, out, n);
  if (n > 2) out[2] = h->bytes;
  return SIGNMUON_OK;
}

}  // extern "C"
