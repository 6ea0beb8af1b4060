// common.cuh -- device-side plan records and launch wrappers shared by the
// kernels of libsignmuon.so.
//
// Data layout in HBM (one handle):
//   flat vectors      W, G_m, Mom_m, U_m, D: d floats, matrices in plan order,
//                     each row-major (the caller's layout)
//   grouped X / A / B matrices of equal shape share a "group"; problem b of a
//                     group (b = worker*count + index-in-group) sits at
//                     base + b*rows*ld (X) or base + b*g*gld (A, B); rows are
//                     padded to ld = round_up(cols, 8) elements so that every
//                     row starts on a 16-byte boundary (TMA stride rule)
//   packed bits       one ceil(d/8)-byte stream per worker, padded to 16 bytes
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace sm {

// widest tensor-core output tile the planner may choose (build-time knob)
#ifndef SM_TC_BN_MAX
#define SM_TC_BN_MAX 256
#endif

constexpr int kMaxWorkers = 256;

struct MatInfo {      // one parameter matrix
  int64_t off;        // start in the flat vector
  int rows, cols;
  int group, q;       // shape group and index within it
};

struct GroupInfo {    // all matrices of one shape
  int rows, cols, ld; // natural shape, padded row stride of X
  int g, gld;         // g = min(rows, cols): Gram side; padded row stride of A/B
  int wide;           // rows <= cols: Gram X X^T; else X^T X
  int count;          // matrices of this shape
  int first;          // index into the group->matrix list
  int64_t x_base;     // element offset of the group in an X buffer
  int64_t a_base;     // element offset of the group in the A/B buffers
};

struct Chunk {        // a piece of one matrix for the flat elementwise kernels
  int mat;
  int len;            // <= kChunk elements
  int64_t start;      // element offset within the matrix
};
constexpr int kChunk = 4096;

// Power iteration on a symmetric Gram: a 128 x 128 tiling of each problem's
// g x g matrix; a pass visits the tiles (bi, bj) with bi <= bj only.
constexpr int kPiTile = 128;
struct PiTile {       // one upper-triangle tile of one problem: all that its block needs
  int64_t aoff;       // the problem's Gram (elements of A)
  int64_t uoff;       // its vectors (g entries)
  int64_t poff;       // its partial sums (nt * nt * 128 entries, nt = ceil(g / 128))
  int p;              // problem id (worker*n_mats + mat)
  int g, gld;         // Gram side and row stride
  int bi, bj;         // row and column slice, bi <= bj
  int pad;
};
struct PiSlice {      // one 128-row slice of one problem's iterate
  int64_t uoff;
  int64_t poff;
  int p, g;
  int bi;
  int soff;           // index of the problem's first slice
};
struct PiReduce {     // what k_pi_reduce writes besides y
  int last;           // the last pass: sigma^2 = u^T y, then the scale
  const float* u;     // (last) the normalised iterate y came from
  double* sq;         // per slice: ||y_slice||^2, or (last) u_slice . y_slice
  int* counters;      // per problem, zero between launches
  float* inv;         // (not last) per problem: 1 / ||y||, or 0 for a zero y
  float eps;
  int quintic;
  float a, b, c;
  float* scale;
  float2* coef_apply;
  float2* coef_square;
  float2* coef_gram;  // Gram-space start (null when the handle iterates on X)
  int* status;
};

struct WorkerPtrs {   // per-worker device pointers passed by value
  const float* p[kMaxWorkers];
};

// One shape group's tiles inside one grouped GEMM launch.
struct TileGroup {
  int group;
  int Mdim, Ndim, Kdim;
  int BM, BN;         // output tile (tensor cores: 256 x {128, 256}; fp32 SIMT: 128 x 128)
  int sym;            // symmetric output: only tiles with tm <= tn (tiles_m == tiles_n)
  int tiles_m, tiles_n;
  int batch;          // problems of this group in the launch
  int tile_start;     // first global tile index of this group
};

enum GemmOp { OP_GRAM = 0, OP_SQUARE = 1, OP_APPLY = 2 };

// Tile and group tables small enough to travel inside the kernel
// parameters (read through the constant cache; a per-tile decode from global
// memory is a chain of dependent loads).
constexpr int kParamGroups = 24;
// TMA tensor maps per shape group (bf16 path): X ping/pong, A, B with 64-row
// and 128-row boxes (slots 0..3, 4..7), X ping/pong as 4-D atom views with
// two-atom operand boxes (8, 9), and X ping/pong, A, B with 32-row boxes (an
// epilogue warp's atom; 10..13); then the m x m buffers of the Gram-space
// iteration, A2, Q0 and Q1, each with 64-, 128- and 32-row boxes (14..22).
constexpr int kMapsPerGroup = 23;
// m x m bf16 buffers addressed by index: 0 = A, 1 = B, 2 = A2, 3 = Q0, 4 = Q1
enum MmBuf { MM_A = 0, MM_B = 1, MM_A2 = 2, MM_Q0 = 3, MM_Q1 = 4 };
// tensor-map slot of m x m buffer `buf` with 64- (box 0), 128- (box 1) or
// 32-row (box 2) boxes
__host__ __device__ __forceinline__ int mm_slot(int buf, int box) {
  if (buf <= MM_B) return box == 0 ? 2 + buf : (box == 1 ? 6 + buf : 12 + buf);
  return 14 + 3 * (buf - MM_A2) + box;
}
constexpr int kParamMats = 64;

// Arguments of one grouped Newton-Schulz GEMM launch (both precisions).
struct GemmArgs {
  const TileGroup* tiles;
  int n_tile_groups;
  int total_tiles;
  // tensor-core launch: null for round robin (cluster c takes tiles c,
  // c + clusters, ...), else [start of each cluster's list (clusters + 1
  // entries), then the lists] from tile_schedule
  const int* sched;
  const GroupInfo* groups;
  const int* group_mats;     // matrices of each group, in order
  const int64_t* mat_off;    // flat offset of each matrix
  int n_mats;
  int op;
  void* X_src;               // X buffer read (APPLY/GRAM operand and APPLY epilogue)
  void* X_dst;               // X buffer written by a non-final APPLY
  void* A;                   // Gram buffer
  void* B;                   // quintic polynomial buffer
  int p_from_b;              // APPLY multiplies by B (quintic) instead of A (fp32 path)
  // bf16 path: APPLY's operator is m x m buffer p_buf; SQUARE computes
  // L R^T (= L R, both symmetric) with L = buffer sq_l and R = buffer sq_r,
  // its affine operand is R, and it writes sq_out (an m x m buffer)
  int p_buf;
  int sq_l, sq_r;
  void* sq_out;
  int sym_exact;             // symmetric outputs stored exactly symmetric (diagonal tiles too)
  int map_src, map_dst;      // tensor-map slots of X_src / X_dst (TMA path)
  // epilogue coefficients: per-problem float2 when coef is non-null, else (c0, c1).
  //   GRAM:   out = c1 acc + cdiag [row == col]
  //   SQUARE: out = c0 R + c1 acc + cdiag [row == col]  (R = A on the fp32 path)
  //   APPLY:  out = c0 X + c1 acc, or (plain) out = acc
  const float2* coef;
  float c0, c1;
  float cdiag;
  int plain;                 // APPLY without the affine operand (its operator already holds a I)
  // final APPLY: fp32 flat output out + worker*out_stride + mat_off + r*cols + c
  // (skipped when out is null), and, when out_bits is non-null, the one-bit
  // signs (U >= 0) as LSB-first 32-bit words at out_bits + worker*bits_stride
  // + flat/32 (every matrix has a multiple of 32 columns)
  float* out;
  int64_t out_stride;
  int final_out;
  uint32_t* out_bits;
  int64_t bits_stride;       // in 32-bit words
  // (bf16 path) when non-null, the ternary signs sign(U) in {-1, 0, +1} as
  // int8 at out_sign8 + worker*sign8_stride + flat index
  int8_t* out_sign8;
  int64_t sign8_stride;
  int* err;
  int param_tables;                        // 1: the p* copies below are valid
  TileGroup ptiles[kParamGroups];
  GroupInfo pgroups[kParamGroups];
  int pgroup_mats[kParamMats];
};

// ---- programmatic dependent launch -----------------------------------------
// Every kernel of the step is launched with programmatic stream
// serialization, so that it can be scheduled while the kernel before it on
// the stream is finishing; it starts with griddep_wait() (no global memory is
// read or written before the previous kernel has completed and its writes are
// visible), then lets the next kernel be scheduled.  Outside such a launch
// both instructions do nothing.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// ---- launch wrappers (host) ----------------------------------------------
void count_launch();
void set_global_error(const char* msg);  // text for signmuon_last_error(NULL)
int num_sms();                                   // SMs of the current device
// Blocks that the current device keeps resident per SM for a kernel launched
// with `threads` threads and `smem` bytes of dynamic shared memory (at least 1).
int resident_per_sm(const void* kernel, int threads, size_t smem);
// Grid of a grid-stride kernel: min(work_items, SMs * min(per_sm, resident
// blocks per SM)), at least 1 -- one full wave, never a partial second one.
int stream_grid(const void* kernel, int threads, size_t smem, int64_t work_items, int per_sm);

void launch_momentum(cudaStream_t s, const WorkerPtrs& G, const float* W, float* Mom, int64_t d,
                     int M, float beta, float lambda, void* X, int x_bf16, const Chunk* chunks,
                     int n_chunks, const MatInfo* mats, const GroupInfo* groups, float* partials);
void launch_stage(cudaStream_t s, const WorkerPtrs& in, int M, void* X, int x_bf16,
                  const Chunk* chunks, int n_chunks, const MatInfo* mats, const GroupInfo* groups,
                  float* partials);
void launch_fro_finalize(cudaStream_t s, int n_probs, int n_mats, int M, const float* partials,
                         const int* mat_chunk0, const int* mat_nchunks, int use_for_scale,
                         float eps, int quintic, float a, float b, float c, float* scale,
                         float2* coef_apply, float2* coef_square, float2* coef_gram, int* status);
// Gram space: Q1 = coef[p].x I + coef[p].y A per problem (bf16 m x m buffers)
void launch_gram_q1(cudaStream_t s, int n_probs, const void* A, void* Q, const int64_t* prob_aoff,
                    const int* prob_g, const int* prob_gld, const float2* coef, int max_g, int max_gld);
// warm != 0: keep each problem's stored iterate when it is non-zero and finite
void launch_pi_init(cudaStream_t s, int n_probs, const int64_t* uoff, const int* prob_g, float* u, int warm);
// one pass over the upper-triangle tiles, one block per tile: partial sums
// of A v, v = src (fold = 0; src == nullptr: v = ones / sqrt(g)) or
// v = src * inv[p] (fold = 1, which also stores v into u)
void launch_pi_tiles(cudaStream_t s, const PiTile* tiles, int n_tiles, const void* A, int a_bf16,
                     const float* src, const float* inv, float* u, float* part, int fold);
// y = the sum of each slice's partials in a fixed order; per problem 1 / ||y||
// or, with r.last, sigma^2 = u^T y and the problem's scale and coefficients
void launch_pi_reduce(cudaStream_t s, const PiSlice* slices, int n_slices, const float* part, float* y,
                      const PiReduce& r);
void launch_scale_flat(cudaStream_t s, const WorkerPtrs& in, int M, float* out, int64_t out_stride,
                       const Chunk* chunks, int n_chunks, const MatInfo* mats, int n_mats,
                       const float* scale, float eps);
void launch_pack(cudaStream_t s, const float* U, int64_t u_stride, int64_t d, uint8_t* out,
                 int64_t out_stride, int M);
void launch_vote(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, void* sums, int acc8,
                 int8_t* majority, int tie_plus);
// The vote kernels take worker m's packed signs at signs.p[m]: this GPU's
// memory or a peer's mapped over NVLink (16-byte aligned, ceil(d/8) bytes
// padded to a multiple of 16).
void launch_vote_update(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, float* W, float eta,
                        const int* status, int tie_plus);
void launch_vote_major(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, float* D, int tie_plus);
// stage_off (two int64 per chunk: flat offset, offset in a one-problem-set
// X) selects the streaming kernel; pass it only when every matrix starts at a
// multiple of 128 entries and has a multiple of 8 columns (its layout rule),
// else NULL
void launch_vote_stage(cudaStream_t s, const WorkerPtrs& signs, int M, void* X, int x_bf16,
                       const Chunk* chunks, int n_chunks, const MatInfo* mats, const GroupInfo* groups,
                       float* partials, float* D, int tie_plus, const int64_t* stage_off);
void launch_mean_stage(cudaStream_t s, const float* Mom, int64_t mom_stride, int M, void* X, int x_bf16,
                       const Chunk* chunks, int n_chunks, const MatInfo* mats, const GroupInfo* groups,
                       float* partials, float* D);
void launch_update(cudaStream_t s, float* W, const float* D, int64_t d, float eta,
                   const int* status);
// int8 ternary sign wire (kernels_ternary.cu)
void launch_sign8(cudaStream_t s, const float* U, int64_t u_stride, int64_t d, int8_t* out, int64_t out_stride,
                  int M);
void launch_vote_ternary(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, void* sums, int acc8,
                         int8_t* majority, int tie_plus);
void launch_vote_ternary_update(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, float* W, float eta,
                                const int* status, int tie_plus);
void launch_vote_ternary_major(cudaStream_t s, const WorkerPtrs& signs, int M, int64_t d, float* D, int tie_plus);
// D = majority of int32 (or int8, acc8) vote sums
void launch_sums_major(cudaStream_t s, const void* sums, int acc8, int64_t d, float* D, int tie_plus);

void launch_gemm_simt(cudaStream_t s, const GemmArgs& a, int x_f32);
int gemm_tc_smem_bytes();
void launch_gemm_tc(cudaStream_t s, const GemmArgs& a, const void* maps, int n_sm);

}  // namespace sm
