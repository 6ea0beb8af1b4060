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
// 2*128*BN*64 flops (a one-SM 128 x BN tile needs 48 KB).  Per CTA, 192
// threads:
//   warp 0      TMA producer: bf16 boxes of 64 columns (128-byte swizzle)
//               into a 5-deep (Gram) or 3-deep ring; both CTAs' loads
//               complete on the leader CTA's "full" barrier
//   warp 1      allocates 512 TMEM columns (cta_group::2); in the leader CTA
//               one lane issues tcgen05.mma.cta_group::2 (M=256, N=BN, K=16)
//               and tcgen05.commit multicast to both CTAs' barriers
//   warps 2..9  epilogue: the affine operand (X for APPLY, A for SQUARE) of
//               the tile comes into shared memory by TMA while the MMAs run;
//               tcgen05.ld 32x32b.x32 -> a*operand + b*acc -> bf16 results
//               written over the operand in shared memory -> TMA store
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
constexpr int EPI_BYTES = 128 * 256 * 2;                // 64 KB: one staging tile
// Shared memory is split per GEMM role: the Gram runs a 5-deep operand ring
// and one staging tile; SQUARE/APPLY a 3-deep ring and two staging tiles so
// that the next tile's affine operand loads while this tile is processed.
constexpr int RING_GRAM = 5, RING_AFFINE = 3, RING_MAX = 5;
constexpr int DATA_BYTES = RING_GRAM * STAGE_BYTES + EPI_BYTES;   // 224 KB either way
static_assert(RING_AFFINE * STAGE_BYTES + 2 * EPI_BYTES == DATA_BYTES, "smem split");
constexpr int TMEM_COLS = 512;
constexpr int NTHREADS = 320;   // producer, MMA, 8 epilogue warps
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
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// arrive on a barrier given by its shared::cluster address (own or peer CTA)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false when the CTA is aborting or 2 s passed (then the error
// word gets the timeout code and the abort flag is raised).
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err) {
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
// 2-SM TMA load: the transaction bytes complete on `bar_cl`, a barrier of the
// leader CTA given by its shared::cluster address.
__device__ __forceinline__ void tma_load_pair(uint32_t dst, const void* map, uint32_t bar_cl, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar_cl)
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
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// Named barrier of the 8 epilogue warps, also OR-reducing a flag over them.
__device__ __forceinline__ int epi_bar_or(int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\t"
      "selp.b32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred)
      : "memory");
  return r;
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
// boxes; the same four with 128-row boxes at slot + 4.
__device__ __forceinline__ const CUtensorMap* map_at(const CUtensorMap* maps, int group, int slot) {
  return maps + group * 8 + slot;
}
__device__ __forceinline__ const CUtensorMap* map128(const CUtensorMap* m) { return m + 4; }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
k_gemm_tc(const __grid_constant__ GemmArgs a, const CUtensorMap* __restrict__ maps) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int op = a.op;
  const int nst = (op == OP_GRAM) ? RING_GRAM : RING_AFFINE;   // operand ring depth
  const uint32_t epi0 = base + nst * STAGE_BYTES;              // staging tile(s)
  uint8_t* const epi_ptr0 = gbase + nst * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + DATA_BYTES);
  // bars: full[RING_MAX], empty[RING_MAX], tmem_full[2], tmem_empty[2], epi_full[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * RING_MAX + 6);
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
    mbar_init(efull_bar(0), 1);
    mbar_init(efull_bar(1), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
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
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.err)) { ok = false; break; }
          if (rank == 0) mbar_expect_tx(full_bar(stage), bytes);
          const uint32_t fb = leader_addr(full_bar(stage));
          const uint32_t sa = base + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          const int k0 = kb * BK;
          // K-major tiles come in one box of 128 (or hb) rows; MN-major tiles
          // as one 64x64 box per 64 MN indices
          if (amn) {
            tma_load_pair(sa, mA, fb, a0, k0, tc.b);
            tma_load_pair(sa + BOX_BYTES, mA, fb, a0 + 64, k0, tc.b);
          } else {
            tma_load_pair(sa, map128(mA), fb, k0, a0, tc.b);
          }
          if (bmn) {
            for (int j = 0; j < hb / 64; ++j) tma_load_pair(sb + j * BOX_BYTES, mB, fb, b0 + 64 * j, k0, tc.b);
          } else {
            tma_load_pair(sb, hb == 128 ? map128(mB) : mB, fb, k0, b0, tc.b);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == nst) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && rank == 0) {
        // drain: every issued stage's last loads must land before teardown
        for (int s = 0; s < nst; ++s) {
          if (!(issued & (1u << s))) continue;
          const uint32_t par = (last_par >> s) & 1u;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(full_bar(s), par) && globaltimer() - t0 < kTimeoutNs) {}
        }
      }
    }
  } else if (warp == 1) {
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
      for (int tile = cid; tile < a.total_tiles && ok; tile += ncl) {
        const TileCoord tc = decode_tile(a, tile);
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
    // ---------------- epilogue (warps 2..9, both CTAs) ----------------
    // Two warps per TMEM lane quarter, each taking half of the tile's columns.
    // The CTA's 128 x BN output tile is staged in shared memory in the
    // swizzled box layout that TMA reads and writes: SQUARE/APPLY load their
    // affine operand there (one tile ahead, alternating two staging tiles),
    // each thread overwrites its operand chunk with the result, and one
    // thread stores the tile with TMA.
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;      // column half of the tile
    const int rloc = q * 32 + lane;        // row within this CTA's 128 rows
    const bool leader_thr = (warp == 2 && lane == 0);
    const bool affine = op != OP_GRAM;
    const bool final_out = (op == OP_APPLY) && a.final_out;
    const uint32_t tempty_leader0 = leader_addr(tempty_bar(0));
    const uint32_t tempty_leader1 = leader_addr(tempty_bar(1));
    // operand load of `tile` into staging tile `b` (leader thread)
    auto load_operand = [&](int tile, int b) {
      const TileCoord t2 = decode_tile(a, tile);
      const CUtensorMap* mO = (op == OP_SQUARE) ? map_at(maps, t2.group, 2) : map_at(maps, t2.group, a.map_src);
      const int rb = t2.m0 + 128 * (int)rank;
      mbar_expect_tx(efull_bar(b), (uint32_t)(t2.BN / 64) * 2u * BOX_BYTES);
      for (int j = 0; j < t2.BN / 64; ++j)
        tma_load_local(epi0 + (uint32_t)b * EPI_BYTES + (uint32_t)j * 2u * BOX_BYTES, map128(mO), efull_bar(b),
                       t2.n0 + 64 * j, rb, t2.b);
    };
    if (affine && leader_thr && cid < a.total_tiles) load_operand(cid, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t e_phase = 0;       // bit b: phase of staging tile b's operand barrier
    int li = 0;                 // tiles handled by this CTA
    for (int tile = cid; tile < a.total_tiles; tile += ncl, ++li) {
      const TileCoord tc = decode_tile(a, tile);
      const GroupInfo gi = group_info(a, tc.group);
      int mat = 0;
      const int p = problem_id(a, gi, tc.b, &mat);
      float c0 = a.c0, c1 = a.c1;
      if (a.coef != nullptr) {
        const float2 cf = a.coef[p];
        c0 = cf.x;
        c1 = cf.y;
      }
      const int buf = affine ? (li & 1) : 0;
      uint8_t* const epi_ptr = epi_ptr0 + buf * EPI_BYTES;
      const uint32_t epi = epi0 + (uint32_t)buf * EPI_BYTES;
      const int rbase = tc.m0 + 128 * (int)rank;
      const int row = rbase + rloc;
      const bool row_ok = row < tc.Mdim;
      const int64_t aoff = gi.a_base + (int64_t)tc.b * gi.g * gi.gld;
      const int w = tc.b / gi.count;
      const int nch = tc.BN / 32;
      // Gram: the single staging tile is free once the previous tile's TMA
      // store has read it (affine roles wait for this one tile later)
      if (!affine && leader_thr) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      // every epilogue warp is here; stop together if a wait gave up
      if (epi_bar_or(*abort_flag != 0)) break;
      int okw = 1;
      if (lane == 0) {
        okw = mbar_wait(tfull_bar(acc), acc_phase, abort_flag, a.err) ? 1 : 0;
        if (okw && affine) okw = mbar_wait(efull_bar(buf), (e_phase >> buf) & 1u, abort_flag, a.err) ? 1 : 0;
      }
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (affine) e_phase ^= 1u << buf;
      // collective: if any warp's wait gave up, all skip to the next barrier,
      // which then stops them together
      if (epi_bar_or(!okw)) continue;
      tc_fence_after();
      // symmetric Gram: an off-diagonal tile is also written transposed
      const bool mirror = (op == OP_GRAM) && (tc.n0 != tc.m0);
      const int h = rloc >> 6, rr = rloc & 63;
      const int ch0 = half * (nch / 2), ch1 = ch0 + nch / 2;
#pragma unroll 1
      for (int ch = ch0; ch < ch1; ++ch) {
        float v[32];
        tmem_ld32(tmem_base + (uint32_t)(acc * 256 + ch * 32) + ((uint32_t)(q * 32) << 16), v);
        const int col0 = tc.n0 + ch * 32;
        const bool live = row_ok && col0 < tc.Ndim;
        const int ncol = live ? min(32, tc.Ndim - col0) : 0;
        // this thread's 64-byte slice of the staging tile: box (j, h), row rr
        uint8_t* rowp = const_cast<uint8_t*>(epi_ptr) + ((ch >> 1) * 2 + h) * BOX_BYTES + rr * 128;
        if (affine) {
          float xv[32];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int unit = ((ch & 1) * 4 + u) ^ (rr & 7);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(rowp + unit * 16), xv + 8 * u);
          }
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] = fmaf(c0, xv[u], c1 * v[u]);
        }
        if (final_out) {
          if (!live) continue;
          float* dst = a.out + (int64_t)w * a.out_stride + a.mat_off[mat] + (int64_t)row * gi.cols + col0;
          if (ncol == 32 && ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0)) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              reinterpret_cast<float4*>(dst)[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
          } else {
            for (int u = 0; u < ncol; ++u) dst[u] = v[u];
          }
          continue;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int unit = ((ch & 1) * 4 + u) ^ (rr & 7);
          uint4 o;
          o.x = pack_bf16x2(v[8 * u + 0], v[8 * u + 1]);
          o.y = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
          o.z = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]);
          o.w = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
          *reinterpret_cast<uint4*>(rowp + unit * 16) = o;
        }
        if (mirror && live) {
          // lanes hold consecutive rows: each store below is 64 contiguous bytes
          __nv_bfloat16* A = reinterpret_cast<__nv_bfloat16*>(a.A) + aoff;
#pragma unroll 8
          for (int u = 0; u < ncol; ++u) A[(int64_t)(col0 + u) * gi.gld + row] = __float2bfloat16_rn(v[u]);
        }
      }
      // make the staged results visible to the TMA (async proxy), release the
      // accumulator, then one thread stores the tile
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc == 0 ? tempty_leader0 : tempty_leader1);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      if (!final_out) {
        epi_bar_or(0);
        if (leader_thr) {
          const int slot = (op == OP_GRAM) ? 2 : (op == OP_SQUARE ? 3 : a.map_dst);
          const CUtensorMap* mD = map_at(maps, tc.group, slot);
          // one 64-column x 128-row box per store, each in its own bulk
          // group (several vertically adjacent boxes in one group were seen
          // to lose all but the first on this hardware)
          int groups = 0;
          if (rbase < tc.Mdim) {
            for (int j = 0; j < tc.BN / 64; ++j) {
              const int x = tc.n0 + 64 * j;
              if (x >= tc.Ndim) break;
              asm volatile(
                  "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];"
                  ::"l"(reinterpret_cast<uint64_t>(map128(mD))), "r"(x), "r"(rbase), "r"(tc.b),
                  "r"(epi + (uint32_t)j * 2u * BOX_BYTES)
                  : "memory");
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
              ++groups;
            }
          }
          if (affine) {
            // the other staging tile is free once the previous tile's stores
            // (all groups but this tile's) have read it; then prefetch the
            // next tile's operand into it
            switch (groups) {
              case 0: asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); break;
              case 1: asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); break;
              case 2: asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory"); break;
              case 3: asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory"); break;
              default: asm volatile("cp.async.bulk.wait_group.read 4;" ::: "memory"); break;
            }
            if (tile + ncl < a.total_tiles) load_operand(tile + ncl, buf ^ 1);
          }
        }
      } else if (affine && leader_thr) {
        // final APPLY (no stores): prefetch the next tile's operand
        if (tile + ncl < a.total_tiles) load_operand(tile + ncl, buf ^ 1);
      }
    }
    if (leader_thr) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs are done with the pair's TMEM and barriers
  if (warp == 1) {
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
