// ns_tc.cu -- bf16 grouped Newton-Schulz GEMM on the 5th-generation tensor
// cores: 2-SM tcgen05.mma (cta_group::2), fp32 accumulators in TMEM, operands
// staged by TMA (no multicast loads).
//
// PolarNS of [paper] "SignMuon: 通信高效的分布式Muon优化" §3/§4 batched over
// every (worker, matrix) problem of the step: one persistent launch per GEMM
// role (GRAM, SQUARE, APPLY, see ns_tiles.cuh) walks a tile list that spans
// all shape groups.  A cluster of two CTAs (one per SM) computes one 256 x BN
// output tile: each CTA stages its 128 rows of the A operand and its BN/2
// rows of the B operand, so an SM moves 32 KB per 64-deep k-block for
// 2*128*BN*64 flops (a one-SM 128 x BN tile needs 48 KB).  Per CTA, 384
// threads:
//   warps 0..2  TMA producers taking turns over the k-blocks: bf16 boxes of
//               64 columns (128-byte swizzle) into a 7-stage ring (6 for
//               APPLY and SQUARE, whose epilogue takes the last), one box per
//               lane; both CTAs' loads complete on the leader CTA's "full"
//               barrier
//   warp 3      allocates 512 TMEM columns (cta_group::2); in the leader CTA
//               one lane issues tcgen05.mma.cta_group::2 (M=256, N=BN, K=16)
//               and tcgen05.commit multicast to both CTAs' barriers
//   warps 4..11 epilogue, each on its own 32-row x BN/2 slice of the tile:
//               per 32-column chunk tcgen05.ld 32x32b.x32 -> (APPLY, SQUARE)
//               a*operand + b*acc, the operand's 32 x 64 atom brought into a
//               4 KB shared-memory slice by TMA -> bf16 results stored
//               straight to global memory (64 bytes per lane and row, no
//               shared memory).  The last APPLY of a step writes sign bits
//               (and U / D in fp32 only when asked for) instead.
// The Gram matrix is symmetric: only tiles on or above the diagonal are
// computed, and the epilogue also writes each off-diagonal tile transposed.
// Every mbarrier wait is bounded (2 s): on expiry the CTA records
// SIGNMUON_E_TIMEOUT in the error word, drains what it issued and frees TMEM.
#include "ns_tiles.cuh"

#include <cuda.h>

namespace sm {
namespace {

constexpr int BK = 64;
constexpr int BOX_BYTES = 64 * 64 * 2;                  // one 64x64 bf16 TMA box
constexpr int A_BYTES = 128 * BK * 2;                   // 16 KB: this CTA's 128 rows of A
constexpr int B_BYTES = 128 * BK * 2;                   // 16 KB: this CTA's BN/2 <= 128 rows of B
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
// Shared memory: a 7-stage operand ring (224 KB) and the barriers.  The ring
// depth is what hides the operand latency: a freed stage is refilled ~2,500
// cycles later under load, against 500-700 cycles of MMA work per stage.  The
// ring's TMA writes and the tensor cores' operand reads already take about
// all of the SM's shared-memory bandwidth at full MMA rate, so the epilogue
// stores its results straight to global memory; only the affine operand of
// APPLY and SQUARE passes through shared memory (TMA in, one read), in the
// last stage's 32 KB, which those launches take out of the ring.
constexpr int RING = 7, RING_MAX = RING;
constexpr int EPI_SLICE = 32 * 64 * 2;                  // 4 KB: one 32 x 64 operand atom per epilogue warp
constexpr int DATA_BYTES = RING * STAGE_BYTES;
constexpr int TMEM_COLS = 512;
// Warp roles.  A warp completes only about one TMA load instruction every
// 500-700 cycles however many it has in flight, while the lanes of one
// instruction and separate warps overlap (measured on B200 with boxes of
// 8-32 KB).  So all boxes of one k-block go out in a single instruction, one
// box per lane, and three producer warps take turns over the k-blocks; each
// epilogue warp loads and stores its own slice of the staging tile.  (Twelve
// warps keep 168 registers per thread for the epilogue; from 13 warps on the
// compiler caps them at 128.)
constexpr int NPROD = 3;                    // producer warps 0..2
constexpr int MMA_WARP = NPROD;             // TMEM allocation + MMA issue
constexpr int EPI_WARP0 = NPROD + 1;        // 8 epilogue warps
constexpr int NTHREADS = (NPROD + 1 + 8) * 32;
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // 2 s
constexpr int SMEM_BYTES = DATA_BYTES + 1024 /*align*/ + 256 /*barriers*/;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t n_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// address of the same shared-memory location in the cluster's CTA 0 (leader)
__device__ __forceinline__ uint32_t leader_addr(uint32_t a) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(a));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
// Relaxed forms: no release fence in front of the arrival (a release at
// cluster scope held the arriving warp for ~2,000 cycles).  Used where the
// arrival orders nothing but tcgen05 reads already completed by
// tcgen05.wait::ld, or precedes the transfer it announces.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx_relaxed(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.relaxed.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false when the CTA is aborting or 2 s passed (then the error
// word gets the timeout code and the abort flag is raised).
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u) {
      if (*abort_flag) return false;
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kTimeoutNs) {
        *abort_flag = 1;
        atomicExch(err, 6);
        return false;
      }
    }
  }
}
// first attempt inline; the bounded loop only when the phase is not done yet
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err) {
  return mbar_try_wait(bar, parity) || mbar_wait_slow(bar, parity, abort_flag, err);
}
// 2-SM TMA load: the transaction bytes complete on `bar_cl`, a barrier of the
// leader CTA given by its shared::cluster address.
__device__ __forceinline__ void tma_load_pair(uint32_t dst, const void* map, uint32_t bar_cl, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar_cl)
      : "memory");
}
// 2-SM TMA load of a 4-D box (the two-atom views of slots 8/9)
__device__ __forceinline__ void tma_load_pair4(uint32_t dst, const void* map, uint32_t bar_cl, int x, int y, int z,
                                               int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar_cl)
      : "memory");
}
// plain one-CTA TMA load completing on this CTA's barrier
__device__ __forceinline__ void tma_load_local(uint32_t dst, const void* map, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// commit: arrive (once) on the barrier at this offset in both CTAs of the pair
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
      ::"r"(bar), "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
// tcgen05.ld without the wait; tmem_wait_ld() then reg_fence() before use
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// keeps the compiler from moving uses of r above the preceding wait
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}
// Shared-memory matrix descriptors, 128-byte swizzle, sm_100 version bit.
//   K-major tile:  rows of 64 bf16 (128 B), 8-row groups 1024 B apart (SBO)
//   MN-major tile: 64-element MN blocks 8 KB apart (LBO, one TMA box each),
//                  8-row K groups 1024 B apart (SBO)
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(BOX_BYTES >> 4) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// Instruction descriptor: f32 accumulate, bf16 A and B, majorness, N, M=256.
__device__ __forceinline__ uint32_t instr_desc(int a_mn, int b_mn, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

// ---- the epilogue's direct global accesses --------------------------------
__device__ __forceinline__ void stg_v8(void* p, const uint32_t* w) {
  asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}
// the first n (1..32) of 32 bf16 (pairs in w) to one row at p (16-byte aligned)
__device__ __forceinline__ void store_row_chunk(__nv_bfloat16* p, int n, const uint32_t (&w)[16]) {
  if (n >= 32 && (reinterpret_cast<uintptr_t>(p) & 31u) == 0) {
    stg_v8(p, &w[0]);
    stg_v8(p + 16, &w[8]);
    return;
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    if (8 * g + 8 <= n) {
      *reinterpret_cast<uint4*>(p + 8 * g) = make_uint4(w[4 * g], w[4 * g + 1], w[4 * g + 2], w[4 * g + 3]);
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (8 * g + u < n) {
          const uint32_t pair = w[4 * g + u / 2];
          const unsigned short h = (u & 1) ? (unsigned short)(pair >> 16) : (unsigned short)(pair & 0xFFFFu);
          reinterpret_cast<unsigned short*>(p)[8 * g + u] = h;
        }
      }
    }
  }
}
// the first n (1..32) of 32 floats to p (any 4-byte alignment)
// The ternary signs (v > 0) - (v < 0) of a chunk's n <= 32 entries as int8
// (0 for a zero or NaN, as the ternary sign kernel gives them).
__device__ __forceinline__ int8_t tsign8(float f) { return (int8_t)((f > 0.f) - (f < 0.f)); }
__device__ __forceinline__ void store_row_sign8(int8_t* p, int n, const float (&v)[32]) {
  if (n >= 32 && (reinterpret_cast<uintptr_t>(p) & 15u) == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int e = 16 * h + 4 * k;
        w[k] = (uint32_t)(uint8_t)tsign8(v[e]) | (uint32_t)(uint8_t)tsign8(v[e + 1]) << 8 |
               (uint32_t)(uint8_t)tsign8(v[e + 2]) << 16 | (uint32_t)(uint8_t)tsign8(v[e + 3]) << 24;
      }
      *reinterpret_cast<uint4*>(p + 16 * h) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    return;
  }
#pragma unroll
  for (int u = 0; u < 32; ++u)
    if (u < n) p[u] = tsign8(v[u]);
}

__device__ __forceinline__ void store_row_f32(float* p, int n, const float (&v)[32]) {
  const uintptr_t al = reinterpret_cast<uintptr_t>(p);
  if (n >= 32 && (al & 31u) == 0) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t w8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) w8[u] = __float_as_uint(v[8 * g + u]);
      stg_v8(p + 8 * g, w8);
    }
    return;
  }
  if ((al & 15u) == 0) {
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if (4 * g + 4 <= n) {
        *reinterpret_cast<float4*>(p + 4 * g) = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (4 * g + u < n) p[4 * g + u] = v[4 * g + u];
      }
    }
    return;
  }
#pragma unroll
  for (int u = 0; u < 32; ++u)
    if (u < n) p[u] = v[u];
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Tensor-map slots per group: 0/1 = X ping/pong, 2 = A, 3 = B, with 64-row
// boxes; the same four with 128-row boxes at slot + 4.  When X's column
// count is a multiple of 64, slots 8/9 hold X ping/pong as 4-D views
// (64-column atom, row, atom index, matrix) with a box of two atoms x 64
// rows: an MN-major operand half of a k-block in one request.  Slots 10..13
// hold the first four with 32-row boxes (an epilogue warp's operand atom).
// The m x m buffers (A, B and the Gram-space A2, Q0, Q1) are addressed by
// mm_slot(buffer, box).
// The i-th tile of cluster cid (of ncl), or -1 past its last: round robin
// over the launch's tile list, or the cluster's own list of a schedule.
__device__ __forceinline__ int tile_at(const GemmArgs& a, int cid, int ncl, int i) {
  if (a.sched == nullptr) {
    const int t = cid + i * ncl;
    return t < a.total_tiles ? t : -1;
  }
  const int s = __ldg(a.sched + cid) + i;
  return s < __ldg(a.sched + cid + 1) ? __ldg(a.sched + ncl + 1 + s) : -1;
}

__device__ __forceinline__ const CUtensorMap* map_at(const CUtensorMap* maps, int group, int slot) {
  return maps + group * kMapsPerGroup + slot;
}
__device__ __forceinline__ const CUtensorMap* map128(const CUtensorMap* m) { return m + 4; }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
k_gemm_tc(const __grid_constant__ GemmArgs a, const CUtensorMap* __restrict__ maps) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int op = a.op;
  const bool affine = op == OP_SQUARE || (op == OP_APPLY && !a.plain);  // epilogue reads an operand
  const int nst = affine ? RING - 1 : RING;                    // operand ring depth
  const uint32_t epi0 = base + (RING - 1) * STAGE_BYTES;       // operand slices (affine)
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + DATA_BYTES);
  // bars: full[RING_MAX], empty[RING_MAX], tmem_full[2], tmem_empty[2],
  // epi_full[8] (one per epilogue warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * RING_MAX + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_addr(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (RING_MAX + s); };
  auto tfull_bar = [&](int s) { return bar0 + 8u * (2 * RING_MAX + s); };
  auto tempty_bar = [&](int s) { return bar0 + 8u * (2 * RING_MAX + 2 + s); };
  auto efull_bar = [&](int b) { return bar0 + 8u * (2 * RING_MAX + 4 + b); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();          // 0 = leader (issues the MMAs)
  const int cid = (int)cluster_id_x(), ncl = (int)n_clusters_x();
  if (threadIdx.x == 0) {
    for (int s = 0; s < RING_MAX; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(tfull_bar(s), 1);
      mbar_init(tempty_bar(s), 16);  // 8 epilogue warps in each CTA of the pair
    }
    for (int b = 0; b < 8; ++b) mbar_init(efull_bar(b), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  // the prologue above touches no global memory: it overlaps the end of the
  // previous kernel on the stream
  griddep_wait();
  griddep_launch();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < NPROD) {
    // ---------------- TMA producers (both CTAs) ----------------
    // k-block j of this CTA's tile sequence goes to ring stage j mod nst and
    // is loaded by producer warp j mod NPROD (NPROD <= nst, so a warp never
    // waits on a stage barrier more than one phase ahead).  Lane 0 waits
    // until the stage is free and posts the expected bytes; then lanes
    // 0..n-1 issue the stage's n boxes (A first, then B) in one instruction.
    int stage = 0, turn = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, last_par = 0;   // lane 0: stages this warp loaded, their parity
    bool ok = true;
    for (int ti = 0, tile = tile_at(a, cid, ncl, 0); tile >= 0 && ok; tile = tile_at(a, cid, ncl, ++ti)) {
      const TileCoord tc = decode_tile(a, tile);
      const GroupInfo gi = group_info(a, tc.group);
      const int nk = (tc.Kdim + BK - 1) / BK;
      const int amn = a_is_mn(op, gi.wide), bmn = b_is_mn(op, gi.wide);
      // each operand's map with 64-row boxes, and with 128-row boxes
      const CUtensorMap *mA, *mB, *mA128, *mB128;
      if (op == OP_GRAM) {
        mA = mB = map_at(maps, tc.group, a.map_src);
        mA128 = mB128 = map128(mA);
      } else if (op == OP_SQUARE) {
        mA = map_at(maps, tc.group, mm_slot(a.sq_l, 0));
        mA128 = map_at(maps, tc.group, mm_slot(a.sq_l, 1));
        mB = map_at(maps, tc.group, mm_slot(a.sq_r, 0));
        mB128 = map_at(maps, tc.group, mm_slot(a.sq_r, 1));
      } else {
        const CUtensorMap* mP = map_at(maps, tc.group, mm_slot(a.p_buf, 0));
        const CUtensorMap* mP128 = map_at(maps, tc.group, mm_slot(a.p_buf, 1));
        const CUtensorMap* mX = map_at(maps, tc.group, a.map_src);
        mA = gi.wide ? mP : mX;
        mB = gi.wide ? mX : mP;
        mA128 = gi.wide ? mP128 : map128(mX);
        mB128 = gi.wide ? map128(mX) : mP128;
      }
      const int a0 = tc.m0 + 128 * (int)rank;          // this CTA's A rows
      const int hb = tc.BN / 2;                        // this CTA's B rows
      const int b0 = tc.n0 + hb * (int)rank;
      const uint32_t bytes = 2u * (uint32_t)(128 + hb) * BK * 2;   // both CTAs
      // This lane's box, if any: K-major tiles come in one box of 128 (or
      // hb) rows; MN-major tiles (always X) in one 4-D box of two 64x64
      // atoms when X's column count is a multiple of 64, else as one 64x64
      // box per 64 MN indices.
      const bool x4 = (gi.cols % 64) == 0;
      const CUtensorMap* mX4 = map_at(maps, tc.group, 8 + a.map_src);
      const int nA = amn ? (x4 ? 1 : 2) : 1;
      const int nB = bmn ? ((x4 && hb == 128) ? 1 : hb / 64) : 1;
      const bool box_a = lane < nA, box_b = !box_a && lane < nA + nB;
      const CUtensorMap* lmap = nullptr;
      uint32_t loff = 0;
      int lx = 0, ly = 0;            // MN-major: (mn index, -); K-major: (-, row)
      bool lmn = false, l4 = false;
      if (box_a) {
        lmn = amn;
        l4 = amn && x4;
        lmap = l4 ? mX4 : (amn ? mA : mA128);
        loff = (uint32_t)lane * BOX_BYTES;
        lx = a0 + 64 * lane;
        ly = a0;
      } else if (box_b) {
        const int i = lane - nA;
        lmn = bmn;
        l4 = bmn && x4 && hb == 128;
        lmap = l4 ? mX4 : (bmn ? mB : (hb == 128 ? mB128 : mB));
        loff = A_BYTES + (uint32_t)i * BOX_BYTES;
        lx = b0 + 64 * i;
        ly = b0;
      }
      for (int kb = 0; kb < nk; ++kb) {
        if (turn == warp) {
          int w_ok = 1;
          if (lane == 0) w_ok = mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.err) ? 1 : 0;
          w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
          if (!w_ok) { ok = false; break; }
          if (lane == 0 && rank == 0) mbar_expect_tx_relaxed(full_bar(stage), bytes);
          __syncwarp();
          const int k0 = kb * BK;
          if (l4)
            tma_load_pair4(base + stage * STAGE_BYTES + loff, lmap, leader_addr(full_bar(stage)), 0, k0, lx >> 6, tc.b);
          else if (box_a || box_b)
            tma_load_pair(base + stage * STAGE_BYTES + loff, lmap, leader_addr(full_bar(stage)), lmn ? lx : k0,
                          lmn ? k0 : ly, tc.b);
          __syncwarp();
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
        }
        if (++turn == NPROD) turn = 0;
        if (++stage == nst) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok && rank == 0 && lane == 0) {
      // drain: the last loads this warp issued into each stage must land
      for (int s = 0; s < nst; ++s) {
        if (!(issued & (1u << s))) continue;
        const uint32_t par = (last_par >> s) & 1u;
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(full_bar(s), par) && globaltimer() - t0 < kTimeoutNs) {}
      }
    } else if (!ok && lane == 0 && issued != 0) {
      // The peer CTA's loads complete on the leader's barriers, which this
      // CTA cannot wait on: give the loads it issued time to land (a load
      // takes microseconds; 50 us is a bound on a live memory system).
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 50000ull) {}
    }
  } else if (warp == MMA_WARP) {
    // ---------------- MMA issuer (leader CTA) ----------------
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      int committed = 0;
      int last_acc = 0;
      uint32_t last_acc_par = 0;
      bool ok = true;
      bool pending_mma = false;     // MMAs issued since the last accumulator commit
      // the next tile is decoded while the current one's first MMAs run, so
      // that a tile boundary costs the MMA queue no decode time
      const int tile0 = tile_at(a, cid, ncl, 0);
      TileCoord tn = decode_tile(a, tile0 >= 0 ? tile0 : 0);
      for (int ti = 0, tile = tile0; tile >= 0 && ok; tile = tile_at(a, cid, ncl, ++ti)) {
        const TileCoord tc = tn;
        const GroupInfo gi = group_info(a, tc.group);
        const int nk = (tc.Kdim + BK - 1) / BK;
        const int amn = a_is_mn(op, gi.wide), bmn = b_is_mn(op, gi.wide);
        const uint32_t idesc = instr_desc(amn, bmn, tc.BN);
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, a.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = amn ? desc_mnmajor(sa + kk * 2048) : desc_kmajor(sa + kk * 32);
            const uint64_t bd = bmn ? desc_mnmajor(sb + kk * 2048) : desc_kmajor(sb + kk * 32);
            tc_mma(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          pending_mma = true;
          tc_commit_pair(empty_bar(stage));
          if (++stage == nst) { stage = 0; phase ^= 1u; }
          if (kb == 0) {
            const int t2 = tile_at(a, cid, ncl, ti + 1);
            if (t2 >= 0) tn = decode_tile(a, t2);
          }
        }
        if (!ok) break;
        tc_commit_pair(tfull_bar(acc));
        pending_mma = false;
        committed++;
        last_acc = acc;
        last_acc_par = acc_phase;
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok && pending_mma) {
        // a tile aborted after some of its MMAs went out: commit them too, so
        // that the wait below covers every MMA before TMEM is freed
        tc_commit_pair(tfull_bar(acc));
        committed++;
        last_acc = acc;
        last_acc_par = acc_phase;
      }
      if (!ok && committed > 0) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(tfull_bar(last_acc), last_acc_par) && globaltimer() - t0 < kTimeoutNs) {}
      }
    }
  } else {
    // ---------------- epilogue (warps 4..11, both CTAs) ----------------
    // Warp e = warp - 4 owns rows 32 q .. 32 q + 31 of the CTA's 128 (its TMEM
    // lane quarter q = warp % 4; lane i holds row 32 q + i) and the column
    // half e / 4 of the tile, i.e. BN/64 chunks of 32 columns.  It uses no
    // shared memory, which the operand ring and the tensor cores keep busy:
    // the affine operand of all its chunks (X for APPLY, R for SQUARE) is
    // loaded into registers before the accumulator is ready; then, chunk by
    // chunk, tcgen05.ld 32x32b.x32, the fp32 combination c0 * operand +
    // c1 * acc, and 64 contiguous bytes of bf16 per lane stored straight to
    // global memory (two 32-byte stores when aligned).  The last APPLY of a
    // step writes the sign bits (and U / D in fp32 only when asked for).
    const int e = warp - EPI_WARP0;
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int half = e >> 2;               // column half of the tile
    const bool final_out = (op == OP_APPLY) && a.final_out;
    const uint32_t tempty_leader0 = leader_addr(tempty_bar(0));
    const uint32_t tempty_leader1 = leader_addr(tempty_bar(1));
    __nv_bfloat16* dst_base =
        reinterpret_cast<__nv_bfloat16*>(op == OP_GRAM ? a.A : (op == OP_SQUARE ? a.sq_out : a.X_dst));
    // This warp's operand slice: one 32-row x 64-column atom (128-byte rows,
    // 128-byte swizzle) of the affine operand at a time, by TMA.
    const uint32_t slice = epi0 + (uint32_t)e * EPI_SLICE;
    const uint32_t my_efull = efull_bar(e);
    const int opnd_slot = (op == OP_SQUARE) ? mm_slot(a.sq_r, 2) : 10 + a.map_src;
    auto load_operand = [&](const TileCoord& t2, int i) {
      const int j = half * (t2.BN / 128) + i;   // atom index within the tile
      if (lane == 0) {
        mbar_expect_tx_relaxed(my_efull, (uint32_t)EPI_SLICE);
        tma_load_local(slice, map_at(maps, t2.group, opnd_slot), my_efull, t2.n0 + 64 * j,
                       t2.m0 + 128 * (int)rank + 32 * q, t2.b);
      }
    };
    uint32_t e_par = 0;          // phase of my operand barrier
    bool load_pending = false;   // an operand load is in flight
    const int tile0 = tile_at(a, cid, ncl, 0);
    if (affine && tile0 >= 0) {
      load_operand(decode_tile(a, tile0), 0);
      load_pending = true;
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int it = 0, tile = tile0; tile >= 0; tile = tile_at(a, cid, ncl, ++it)) {
      const TileCoord tc = decode_tile(a, tile);
      const int tile_next = tile_at(a, cid, ncl, it + 1);
      const bool more = tile_next >= 0;
      const GroupInfo gi = group_info(a, tc.group);
      int mat = 0;
      const int p = problem_id(a, gi, tc.b, &mat);
      float c0 = a.c0, c1 = a.c1;
      if (a.coef != nullptr) {
        const float2 cf = a.coef[p];
        c0 = cf.x;
        c1 = cf.y;
      }
      const int row = tc.m0 + 128 * (int)rank + q * 32 + lane;
      const bool row_ok = row < tc.Mdim;
      const int atoms = tc.BN / 128;                  // 64-column atoms of this warp (1 or 2)
      const int ch0 = half * (tc.BN / 64);            // first 32-column chunk of this warp
      // X (APPLY) rows have stride ld; the Gram A and the quintic B stride gld
      const bool on_x = op == OP_APPLY;
      const int64_t ldm = on_x ? gi.ld : gi.gld;
      const int64_t mrow = (on_x ? gi.x_base + (int64_t)tc.b * gi.rows * gi.ld
                                 : gi.a_base + (int64_t)tc.b * gi.g * gi.gld) + (int64_t)row * ldm;
      const int w = tc.b / gi.count;
      int okw = 1;
      if (lane == 0) okw = mbar_wait(tfull_bar(acc), acc_phase, abort_flag, a.err) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      tc_fence_after();
      // Symmetric output (the Gram, and the m x m products of symmetric
      // operands that commute): an off-diagonal tile is also written
      // transposed.  With sym_exact a diagonal tile writes its entries on and
      // above the diagonal and their mirror, so that the stored matrix is
      // exactly symmetric: a later SQUARE multiplies by R^T, which must equal R.
      const bool sym_out = (op != OP_APPLY) && tc.sym;
      const bool diag_tile = sym_out && a.sym_exact && (tc.n0 == tc.m0);
      const uint32_t tm_row = tmem_base + (uint32_t)(acc * 256) + ((uint32_t)(q * 32) << 16);
      bool alive = true;
#pragma unroll 1
      for (int i = 0; i < atoms; ++i) {
        if (affine) {
          // the atom's operand has landed
          int okw2 = 1;
          if (lane == 0) okw2 = mbar_wait(my_efull, e_par, abort_flag, a.err) ? 1 : 0;
          okw2 = __shfl_sync(0xffffffffu, okw2, 0);
          if (!okw2) { alive = false; break; }
          e_par ^= 1u;
          load_pending = false;
        }
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          const int ch = ch0 + 2 * i + hc;
          const int col0 = tc.n0 + ch * 32;
          uint32_t r[32];
          tmem_ld32_async(tm_row + (uint32_t)(ch * 32), r);
          tmem_wait_ld();
          reg_fence(r);
          if (i + 1 == atoms && hc == 1) {
            // the accumulator slice is free once its last TMEM load is done
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(acc == 0 ? tempty_leader0 : tempty_leader1);
          }
          float v[32];
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] = __uint_as_float(r[u]);
          if (affine) {
            // this lane's row of the chunk: 4 swizzled 16-byte units of the atom
            const uint32_t rowa = slice + (uint32_t)(lane * 128);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 xo;
              asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(xo.x), "=r"(xo.y), "=r"(xo.z), "=r"(xo.w)
                           : "r"(rowa + (uint32_t)(((hc * 4 + u) ^ (lane & 7)) * 16)));
              const uint32_t xw[4] = {xo.x, xo.y, xo.z, xo.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[k]));
                v[8 * u + 2 * k] = fmaf(c0, x.x, c1 * v[8 * u + 2 * k]);
                v[8 * u + 2 * k + 1] = fmaf(c0, x.y, c1 * v[8 * u + 2 * k + 1]);
              }
            }
          }
          if (op == OP_GRAM) {
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] *= c1;
          }
          if (a.cdiag != 0.f && row >= col0 && row < col0 + 32) {
            // the a I term of the apply's operator: the chunk holds this row's
            // diagonal entry (any tile the diagonal crosses, 256 x 128 ones too)
#pragma unroll
            for (int u = 0; u < 32; ++u)
              if (col0 + u == row) v[u] += a.cdiag;
          }
          const bool live = row_ok && col0 < tc.Ndim;
          const int ncol = live ? min(32, tc.Ndim - col0) : 0;
          if (final_out) {
            if (live && a.out_bits != nullptr) {
              // the chunk's ncol signs (U >= 0), LSB-first from its flat
              // index: one word of the bit stream when that is a multiple of
              // 32 and the chunk is whole, else OR-ed into the two words it
              // straddles (the buffer was zeroed for such shapes)
              const int64_t flat = a.mat_off[mat] + (int64_t)row * gi.cols + col0;
              uint32_t word = 0;
#pragma unroll
              for (int u = 0; u < 32; ++u) word |= (u < ncol && v[u] >= 0.f ? 1u : 0u) << u;
              uint32_t* wp = a.out_bits + (int64_t)w * a.bits_stride + (flat >> 5);
              const int sh = (int)(flat & 31);
              if (sh == 0 && ncol == 32) {
                *wp = word;
              } else {
                atomicOr(wp, word << sh);
                if (sh != 0 && ncol + sh > 32) atomicOr(wp + 1, word >> (32 - sh));
              }
            }
            if (live && a.out_sign8 != nullptr) {
              store_row_sign8(a.out_sign8 + (int64_t)w * a.sign8_stride + a.mat_off[mat] + (int64_t)row * gi.cols + col0,
                              ncol, v);
            }
            if (live && a.out != nullptr) {
              float* dst = a.out + (int64_t)w * a.out_stride + a.mat_off[mat] + (int64_t)row * gi.cols + col0;
              store_row_f32(dst, ncol, v);
            }
            continue;
          }
          uint32_t ow[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) ow[k] = pack_bf16x2(v[2 * k], v[2 * k + 1]);
          if (live) {
            if (!diag_tile || col0 > row) {
              store_row_chunk(dst_base + mrow + col0, ncol, ow);
            } else if (col0 + 31 >= row) {
              // the chunk crosses the diagonal: only the entries on or above it
#pragma unroll
              for (int u = 0; u < 32; ++u)
                if (u < ncol && col0 + u >= row) dst_base[mrow + col0 + u] = __float2bfloat16_rn(v[u]);
            }
            // (a chunk wholly below the diagonal comes from the mirror of the lanes above)
          }
          if (sym_out && live && (tc.n0 != tc.m0 || (diag_tile && col0 + 31 > row))) {
            // lanes hold consecutive rows: each store below is 64 contiguous bytes
            __nv_bfloat16* At = dst_base + gi.a_base + (int64_t)tc.b * gi.g * gi.gld;
#pragma unroll
            for (int u = 0; u < 32; ++u)
              if (u < ncol && (!diag_tile || col0 + u > row))
                At[(int64_t)(col0 + u) * gi.gld + row] = __float2bfloat16_rn(v[u]);
          }
        }
        if (affine) {
          // the slice takes the next atom once every lane has read this one
          __syncwarp();
          if (i + 1 < atoms) {
            load_operand(tc, i + 1);
            load_pending = true;
          } else if (more) {
            load_operand(decode_tile(a, tile_next), 0);
            load_pending = true;
          }
        }
      }
      if (!alive) break;
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (load_pending && lane == 0) {
      // a wait gave up with an operand load in flight: let it land
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(my_efull, e_par) && globaltimer() - t0 < kTimeoutNs) {}
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs are done with the pair's TMEM and barriers
  if (warp == MMA_WARP) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS));
  }
}

}  // namespace

int gemm_tc_smem_bytes() { return SMEM_BYTES; }

void launch_gemm_tc(cudaStream_t s, const GemmArgs& a, const void* maps, int n_sm) {
  if (a.total_tiles <= 0) return;
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    attr_set = true;
  }
  count_launch();
  const int pairs = n_sm / 2;
  const int clusters = a.total_tiles < pairs ? a.total_tiles : pairs;
  launch_pdl(k_gemm_tc, dim3(2 * clusters), dim3(NTHREADS), SMEM_BYTES, s, a, reinterpret_cast<const CUtensorMap*>(maps));
}

}  // namespace sm
