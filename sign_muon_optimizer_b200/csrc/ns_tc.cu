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
//               64 columns (128-byte swizzle) into a 6-deep ring, one box per
//               lane; both CTAs' loads complete on the leader CTA's "full"
//               barrier
//   warp 3      allocates 512 TMEM columns (cta_group::2); in the leader CTA
//               one lane issues tcgen05.mma.cta_group::2 (M=256, N=BN, K=16)
//               and tcgen05.commit multicast to both CTAs' barriers
//   warps 4..11 epilogue, each on its own 32-row x BN/2 slice of the tile,
//               one 32 x 64 atom at a time: the atom of the affine operand (X
//               for APPLY, A for SQUARE) comes into shared memory by TMA;
//               tcgen05.ld 32x32b.x32 -> a*operand + b*acc -> bf16 results
//               written over the operand -> TMA store of the atom.  The last
//               APPLY of a step writes sign bits (and U / D in fp32 only when
//               asked for) instead.
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
constexpr int EPI_BYTES = 8 * 32 * 64 * 2;              // 32 KB: one 32x64 atom per epilogue warp
// Shared memory: a 6-deep operand ring and the epilogue's staging atoms
// (224 KB).  The ring depth is what hides the operand latency: a freed stage
// is refilled ~2,500 cycles later under load, against ~650 cycles of MMA work
// per stage.
constexpr int RING = 6, RING_MAX = RING;
constexpr int DATA_BYTES = RING * STAGE_BYTES + EPI_BYTES;
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
// shared-memory 16-byte load / store by shared-window address
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
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
// 2-SM TMA load of a 4-D box (the two-atom views of slots 12/13)
__device__ __forceinline__ void tma_load_pair4(uint32_t dst, const void* map, uint32_t bar_cl, int x, int y, int z,
                                               int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar_cl)
      : "memory");
}
__device__ __forceinline__ void tma_store3(const void* map, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(src)
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

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void unpack_bf16x8(uint4 u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
// Tensor-map slots per group: 0/1 = X ping/pong, 2 = A, 3 = B, with 64-row
// boxes; the same four with 128-row boxes at slot + 4 and with 32-row boxes
// (an epilogue warp's atom) at slot + 8.  When X's column count is a
// multiple of 64, slots 12/13 hold X ping/pong as 4-D views (64-column atom,
// row, atom index, matrix) with a box of two atoms x 64 rows: an MN-major
// operand half of a k-block in one request.
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
  const int nst = RING;                                        // operand ring depth
  const uint32_t epi0 = base + nst * STAGE_BYTES;              // staging tile
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
    for (int tile = cid; tile < a.total_tiles && ok; tile += ncl) {
      const TileCoord tc = decode_tile(a, tile);
      const GroupInfo gi = group_info(a, tc.group);
      const int nk = (tc.Kdim + BK - 1) / BK;
      const int amn = a_is_mn(op, gi.wide), bmn = b_is_mn(op, gi.wide);
      const CUtensorMap* mA;
      const CUtensorMap* mB;
      if (op == OP_GRAM) {
        mA = mB = map_at(maps, tc.group, a.map_src);
      } else if (op == OP_SQUARE) {
        mA = mB = map_at(maps, tc.group, 2);
      } else {
        const CUtensorMap* mP = map_at(maps, tc.group, a.p_from_b ? 3 : 2);
        const CUtensorMap* mX = map_at(maps, tc.group, a.map_src);
        mA = gi.wide ? mP : mX;
        mB = gi.wide ? mX : mP;
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
      const CUtensorMap* mX4 = map_at(maps, tc.group, 12 + a.map_src);
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
        lmap = l4 ? mX4 : (amn ? mA : map128(mA));
        loff = (uint32_t)lane * BOX_BYTES;
        lx = a0 + 64 * lane;
        ly = a0;
      } else if (box_b) {
        const int i = lane - nA;
        lmn = bmn;
        l4 = bmn && x4 && hb == 128;
        lmap = l4 ? mX4 : (bmn ? mB : (hb == 128 ? map128(mB) : mB));
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
      // the next tile is decoded while the current one's first MMAs run, so
      // that a tile boundary costs the MMA queue no decode time
      TileCoord tn = decode_tile(a, cid < a.total_tiles ? cid : 0);
      for (int tile = cid; tile < a.total_tiles && ok; tile += ncl) {
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
          tc_commit_pair(empty_bar(stage));
          if (++stage == nst) { stage = 0; phase ^= 1u; }
          if (kb == 0 && tile + ncl < a.total_tiles) tn = decode_tile(a, tile + ncl);
        }
        if (!ok) break;
        tc_commit_pair(tfull_bar(acc));
        committed++;
        last_acc = acc;
        last_acc_par = acc_phase;
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok && committed > 0) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(tfull_bar(last_acc), last_acc_par) && globaltimer() - t0 < kTimeoutNs) {}
      }
    }
  } else {
    // ---------------- epilogue (warps 6..13, both CTAs) ----------------
    // Warp e = warp - 6 owns rows 32*q .. 32*q+31 of the CTA's 128 (its TMEM
    // lane quarter q = warp % 4) and the column half e / 4 of the tile, i.e.
    // one 32-row slice of one or two 64-column atoms of the staging tile
    // (swizzled box layout [atom][128 rows][128 B]).  Each warp runs on its
    // own: it TMA-loads its slice of the affine operand (X for APPLY, A for
    // SQUARE), drains its accumulator slice, writes bf16 results over the
    // operand and TMA-stores the slice, with no barrier between warps.
    const int e = warp - EPI_WARP0;
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int half = e >> 2;               // column half of the tile
    const int rloc = q * 32 + lane;        // row within this CTA's 128 rows
    const bool affine = op != OP_GRAM;
    const bool final_out = (op == OP_APPLY) && a.final_out;
    const uint32_t tempty_leader0 = leader_addr(tempty_bar(0));
    const uint32_t tempty_leader1 = leader_addr(tempty_bar(1));
    const uint32_t my_efull = efull_bar(e);
    // This warp's staging slice is one atom, 32 rows x 64 columns (4 KB,
    // 128-byte rows, swizzled); the warp's 64- or 128-column part of a tile
    // passes through it one atom at a time.
    const uint32_t slice = epi0 + (uint32_t)e * 4096u;
    const int opnd_slot = (op == OP_SQUARE) ? 2 : a.map_src;
    const int dst_slot = (op == OP_GRAM) ? 2 : (op == OP_SQUARE ? 3 : a.map_dst);
    // atom i (of this warp's part) of a tile's affine operand, 64 x 32 box
    auto load_operand = [&](const TileCoord& t2, int i) {
      const int j = half * (t2.BN / 128) + i;
      if (lane == 0) {
        mbar_expect_tx_relaxed(my_efull, 4096u);
        tma_load_local(slice, map_at(maps, t2.group, 8 + opnd_slot), my_efull, t2.n0 + 64 * j,
                       t2.m0 + 128 * (int)rank + 32 * q, t2.b);
      }
    };
    uint32_t e_par = 0;          // phase of my operand barrier
    bool load_pending = false;   // an operand load is in flight
    if (affine && cid < a.total_tiles) {
      load_operand(decode_tile(a, cid), 0);
      load_pending = true;
    }
    // lane 0 waits for my operand barrier; false if the wait gave up
    auto wait_operand = [&]() {
      int okw = 1;
      if (lane == 0) okw = mbar_wait(my_efull, e_par, abort_flag, a.err) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (okw) {
        e_par ^= 1u;
        load_pending = false;
      }
      return okw != 0;
    };
    int acc = 0;
    uint32_t acc_phase = 0;
    bool alive = true;
    for (int tile = cid; tile < a.total_tiles && alive; tile += ncl) {
      const TileCoord tc = decode_tile(a, tile);
      const bool more = tile + ncl < a.total_tiles;
      const TileCoord tnext = decode_tile(a, more ? tile + ncl : tile);
      const GroupInfo gi = group_info(a, tc.group);
      int mat = 0;
      const int p = problem_id(a, gi, tc.b, &mat);
      float c0 = a.c0, c1 = a.c1;
      if (a.coef != nullptr) {
        const float2 cf = a.coef[p];
        c0 = cf.x;
        c1 = cf.y;
      }
      const int rbase = tc.m0 + 128 * (int)rank;
      const int row = rbase + rloc;
      const bool row_ok = row < tc.Mdim;
      const int64_t aoff = gi.a_base + (int64_t)tc.b * gi.g * gi.gld;
      const int w = tc.b / gi.count;
      const int atoms = tc.BN / 128;                 // atoms of this warp
      const int ch0 = half * (tc.BN / 64);           // first 32-column chunk
      int okw = 1;
      if (lane == 0) okw = mbar_wait(tfull_bar(acc), acc_phase, abort_flag, a.err) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      tc_fence_after();
      // symmetric Gram: an off-diagonal tile is also written transposed
      const bool mirror = (op == OP_GRAM) && (tc.n0 != tc.m0);
      const uint32_t tm_row = tmem_base + (uint32_t)(acc * 256) + ((uint32_t)(q * 32) << 16);
      // results of one 32-column chunk from its accumulator registers
      auto form = [&](int ch, uint32_t (&rr)[32]) {
        float v[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = __uint_as_float(rr[u]);
        const int col0 = tc.n0 + ch * 32;
        const bool live = row_ok && col0 < tc.Ndim;
        const int ncol = live ? min(32, tc.Ndim - col0) : 0;
        const uint32_t rowa = slice + (uint32_t)(lane * 128);
        if (affine) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 xo = lds128(rowa + (uint32_t)((((ch & 1) * 4 + u) ^ (lane & 7)) * 16));
            float xv[8];
            unpack_bf16x8(xo, xv);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[8 * u + i] = fmaf(c0, xv[i], c1 * v[8 * u + i]);
          }
        }
        if (final_out) {
          // fp32 results go back into rr for write_out_f32; the signs (when
          // asked for) are one LSB-first word of the bit stream per chunk
#pragma unroll
          for (int u = 0; u < 32; ++u) rr[u] = __float_as_uint(v[u]);
          if (live && a.out_bits != nullptr) {
            const int64_t flat = a.mat_off[mat] + (int64_t)row * gi.cols + col0;
            uint32_t word = 0;
#pragma unroll
            for (int u = 0; u < 32; ++u) word |= (v[u] >= 0.f ? 1u : 0u) << u;
            a.out_bits[(int64_t)w * a.bits_stride + (flat >> 5)] = word;
          }
          (void)ncol;
          return;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int unit = ((ch & 1) * 4 + u) ^ (lane & 7);
          uint4 o;
          o.x = pack_bf16x2(v[8 * u + 0], v[8 * u + 1]);
          o.y = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
          o.z = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]);
          o.w = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
          sts128(rowa + (uint32_t)(unit * 16), o);
        }
        if (mirror && live) {
          // lanes hold consecutive rows: each store below is 64 contiguous bytes
          __nv_bfloat16* A = reinterpret_cast<__nv_bfloat16*>(a.A) + aoff;
#pragma unroll
          for (int u = 0; u < 32; ++u)
            if (u < ncol) A[(int64_t)(col0 + u) * gi.gld + row] = __float2bfloat16_rn(v[u]);
        }
      };
      // fp32 output of one chunk (final APPLY): the warp's 32 rows x 32
      // columns pass through the slice (one 128-byte swizzled row per lane),
      // then each store instruction writes four whole 128-byte row segments
      auto write_out_f32 = [&](int ch, uint32_t (&rr)[32]) {
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 8; ++u)
          sts128(slice + (uint32_t)(lane * 128 + ((u ^ (lane & 7)) * 16)),
                 make_uint4(rr[4 * u], rr[4 * u + 1], rr[4 * u + 2], rr[4 * u + 3]));
        __syncwarp();
        const int uu = lane & 7;
        const int colg = tc.n0 + ch * 32 + uu * 4;
#pragma unroll 2
        for (int it = 0; it < 8; ++it) {
          const int rl = it * 4 + (lane >> 3);
          const int rowg = rbase + q * 32 + rl;
          if (rowg >= tc.Mdim || colg >= tc.Ndim) continue;
          const uint4 val = lds128(slice + (uint32_t)(rl * 128 + ((uu ^ (rl & 7)) * 16)));
          float* dst = a.out + (int64_t)w * a.out_stride + a.mat_off[mat] + (int64_t)rowg * gi.cols + colg;
          if (colg + 3 < tc.Ndim && ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0)) {
            *reinterpret_cast<uint4*>(dst) = val;
          } else {
            const uint32_t e4[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
            for (int t = 0; t < 4; ++t)
              if (colg + t < tc.Ndim) dst[t] = __uint_as_float(e4[t]);
          }
        }
      };
#pragma unroll 1
      for (int i = 0; i < atoms; ++i) {
        const int ch = ch0 + 2 * i;
        // the atom's operand has landed (affine); the slice is free of my
        // previous store (Gram)
        if (affine) {
          if (!wait_operand()) { alive = false; break; }
        } else {
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          __syncwarp();
        }
        // two 32-column chunks per TMEM round trip; the accumulator slice is
        // released after its last TMEM load
        uint32_t r[2][32];
        tmem_ld32_async(tm_row + (uint32_t)(ch * 32), r[0]);
        tmem_ld32_async(tm_row + (uint32_t)((ch + 1) * 32), r[1]);
        tmem_wait_ld();
        reg_fence(r[0]);
        reg_fence(r[1]);
        if (i + 1 == atoms) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_relaxed(acc == 0 ? tempty_leader0 : tempty_leader1);
        }
        form(ch, r[0]);
        form(ch + 1, r[1]);
        if (final_out && a.out != nullptr) {
          write_out_f32(ch, r[0]);
          write_out_f32(ch + 1, r[1]);
        }
        // make the staged results visible to the TMA (async proxy), store
        // the atom (one 64 x 32 box in a bulk group of its own)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (!final_out && lane == 0) {
          const int x = tc.n0 + 64 * (half * atoms + i), y = rbase + 32 * q;
          if (y < tc.Mdim && x < tc.Ndim) {
            tma_store3(map_at(maps, tc.group, 8 + dst_slot), slice, x, y, tc.b);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
        }
        if (affine) {
          // the slice takes the next operand atom once my store has read it
          if (!final_out) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          __syncwarp();
          if (i + 1 < atoms) {
            load_operand(tc, i + 1);
            load_pending = true;
          } else if (more) {
            load_operand(tnext, 0);
            load_pending = true;
          }
        }
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
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
  k_gemm_tc<<<2 * clusters, NTHREADS, SMEM_BYTES, s>>>(a, reinterpret_cast<const CUtensorMap*>(maps));
}

}  // namespace sm
