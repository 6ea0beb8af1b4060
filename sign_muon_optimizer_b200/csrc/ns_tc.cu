// ns_tc.cu -- bf16 grouped Newton-Schulz GEMM on the 5th-generation tensor
// cores (tcgen05.mma, fp32 accumulators in TMEM, operands staged by TMA).
//
// PolarNS of [paper] "SignMuon: 通信高效的分布式Muon优化" §3/§4 batched over
// every (worker, matrix) problem of the step: one persistent launch per GEMM
// role (GRAM, SQUARE, APPLY, see ns_tiles.cuh) walks a tile list that spans
// all shape groups.  Per CTA (one per SM, 192 threads):
//   warp 0      TMA producer: 64x64 bf16 boxes (128-byte swizzle) into a
//               4-stage ring of (A 128x64, B BNx64) tiles; no multicast
//   warp 1      allocates 512 TMEM columns; one lane issues
//               tcgen05.mma.cta_group::1.kind::f16 (M=128, N=BN, K=16) and
//               tcgen05.commit to release smem stages / publish accumulators
//   warps 2..5  epilogue: tcgen05.ld 32x32b.x32 -> registers -> coefficients
//               (a X + b acc, ...) -> bf16 X/A/B tiles or the fp32 result
// Two TMEM accumulators (2 x 256 columns) let the epilogue of tile i overlap
// the mainloop of tile i+1.  Every mbarrier wait is bounded: on expiry the
// CTA records SIGNMUON_E_TIMEOUT in the error word, drains what it issued and
// frees its TMEM.
#include "ns_tiles.cuh"

#include <cuda.h>

namespace sm {
namespace {

constexpr int BM = 128, BK = 64, STAGES = 4;
constexpr int BOX_BYTES = 64 * 64 * 2;                  // one 64x64 bf16 TMA box
constexpr int A_BYTES = BM * BK * 2;                    // 16 KB
constexpr int B_BYTES = 256 * BK * 2;                   // 32 KB (BN <= 256)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int NTHREADS = 192;
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // 2 s
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
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
// Instruction descriptor: f32 accumulate, bf16 A and B, majorness, N, M=128.
__device__ __forceinline__ uint32_t instr_desc(int a_mn, int b_mn, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
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

// Tensor-map slots per group: 0/1 = X ping/pong, 2 = A, 3 = B.
__device__ __forceinline__ const CUtensorMap* map_at(const CUtensorMap* maps, int group, int slot) {
  return maps + group * 4 + slot;
}

__global__ void __launch_bounds__(NTHREADS, 1)
k_gemm_tc(const GemmArgs a, const CUtensorMap* __restrict__ maps) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + STAGES * STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], tmem_full[2], tmem_empty[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_addr(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto tempty_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 2 + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(tfull_bar(s), 1);
      mbar_init(tempty_bar(s), 4);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int op = a.op;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;          // bit s: stage s has been issued at least once
      uint32_t last_par = 0;        // bit s: parity of stage s's last issue
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.total_tiles && ok; tile += gridDim.x) {
        const TileCoord tc = decode_tile(a, tile);
        const GroupInfo gi = a.groups[tc.group];
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
        const uint32_t bytes = (uint32_t)(BM + tc.BN) * BK * 2;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.err)) { ok = false; break; }
          mbar_expect_tx(full_bar(stage), bytes);
          const uint32_t sa = base + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          const int k0 = kb * BK;
          // A tile: 128 (M) x 64 (K) as two boxes
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (amn) tma_load_3d(sa + j * BOX_BYTES, mA, full_bar(stage), tc.m0 + 64 * j, k0, tc.b);
            else     tma_load_3d(sa + j * BOX_BYTES, mA, full_bar(stage), k0, tc.m0 + 64 * j, tc.b);
          }
          for (int j = 0; j < tc.BN / 64; ++j) {
            if (bmn) tma_load_3d(sb + j * BOX_BYTES, mB, full_bar(stage), tc.n0 + 64 * j, k0, tc.b);
            else     tma_load_3d(sb + j * BOX_BYTES, mB, full_bar(stage), k0, tc.n0 + 64 * j, tc.b);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // drain: every issued stage's last load must land before teardown
        for (int s = 0; s < STAGES; ++s) {
          if (!(issued & (1u << s))) continue;
          const uint32_t par = (last_par >> s) & 1u;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(full_bar(s), par) && globaltimer() - t0 < kTimeoutNs) {}
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      int committed = 0;            // accumulators handed to the epilogue
      int last_acc = 0;
      uint32_t last_acc_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.total_tiles && ok; tile += gridDim.x) {
        const TileCoord tc = decode_tile(a, tile);
        const GroupInfo gi = a.groups[tc.group];
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
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        committed++;
        last_acc = acc;
        last_acc_par = acc_phase;
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok && committed > 0) {
        // drain: the last committed MMAs must finish before TMEM is freed
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(tfull_bar(last_acc), last_acc_par) && globaltimer() - t0 < kTimeoutNs) {}
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int rloc = q * 32 + lane;        // row within the 128-row tile
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x) {
      const TileCoord tc = decode_tile(a, tile);
      const GroupInfo gi = a.groups[tc.group];
      int mat = 0;
      const int p = problem_id(a, gi, tc.b, &mat);
      float c0 = a.c0, c1 = a.c1;
      if (a.coef != nullptr) {
        const float2 cf = a.coef[p];
        c0 = cf.x;
        c1 = cf.y;
      }
      // one lane waits, the warp follows (tcgen05.ld below is warp-collective)
      int okw = (lane == 0) ? (mbar_wait(tfull_bar(acc), acc_phase, abort_flag, a.err) ? 1 : 0) : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      tc_fence_after();
      const int row = tc.m0 + rloc;
      const bool row_ok = row < tc.Mdim;
      const int64_t xoff = gi.x_base + (int64_t)tc.b * gi.rows * gi.ld;
      const int64_t aoff = gi.a_base + (int64_t)tc.b * gi.g * gi.gld;
      const int w = tc.b / gi.count;
      for (int ch = 0; ch < tc.BN / 32; ++ch) {
        float v[32];
        tmem_ld32(tmem_base + (uint32_t)(acc * 256 + ch * 32) + ((uint32_t)(q * 32) << 16), v);
        const int col0 = tc.n0 + ch * 32;
        if (!row_ok || col0 >= tc.Ndim) continue;
        const int ncol = min(32, tc.Ndim - col0);
        if (op == OP_GRAM) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.A) + aoff + (int64_t)row * gi.gld + col0;
          if (ncol == 32) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 o;
              o.x = pack_bf16x2(v[8 * u + 0], v[8 * u + 1]);
              o.y = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
              o.z = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]);
              o.w = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
              reinterpret_cast<uint4*>(dst)[u] = o;
            }
          } else {
            for (int u = 0; u < ncol; ++u) dst[u] = __float2bfloat16_rn(v[u]);
          }
        } else {
          // second operand of the affine epilogue: A (SQUARE) or X (APPLY)
          const __nv_bfloat16* src;
          if (op == OP_SQUARE) src = reinterpret_cast<const __nv_bfloat16*>(a.A) + aoff + (int64_t)row * gi.gld + col0;
          else src = reinterpret_cast<const __nv_bfloat16*>(a.X_src) + xoff + (int64_t)row * gi.ld + col0;
          float xv[32];
          if (ncol == 32) {
#pragma unroll
            for (int u = 0; u < 4; ++u) unpack_bf16x8(reinterpret_cast<const uint4*>(src)[u], xv + 8 * u);
          } else {
            for (int u = 0; u < 32; ++u) xv[u] = (u < ncol) ? __bfloat162float(src[u]) : 0.f;
          }
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] = fmaf(c0, xv[u], c1 * v[u]);
          if (op == OP_APPLY && a.final_out) {
            float* dst = a.out + (int64_t)w * a.out_stride + a.mat_off[mat] + (int64_t)row * gi.cols + col0;
            if (ncol == 32 && ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0)) {
#pragma unroll
              for (int u = 0; u < 8; ++u)
                reinterpret_cast<float4*>(dst)[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
            } else {
              for (int u = 0; u < ncol; ++u) dst[u] = v[u];
            }
          } else {
            __nv_bfloat16* dst;
            if (op == OP_SQUARE) dst = reinterpret_cast<__nv_bfloat16*>(a.B) + aoff + (int64_t)row * gi.gld + col0;
            else dst = reinterpret_cast<__nv_bfloat16*>(a.X_dst) + xoff + (int64_t)row * gi.ld + col0;
            if (ncol == 32) {
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                uint4 o;
                o.x = pack_bf16x2(v[8 * u + 0], v[8 * u + 1]);
                o.y = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
                o.z = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]);
                o.w = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
                reinterpret_cast<uint4*>(dst)[u] = o;
              }
            } else {
              for (int u = 0; u < ncol; ++u) dst[u] = __float2bfloat16_rn(v[u]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS));
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
  const int grid = a.total_tiles < n_sm ? a.total_tiles : n_sm;
  k_gemm_tc<<<grid, NTHREADS, SMEM_BYTES, s>>>(a, reinterpret_cast<const CUtensorMap*>(maps));
}

}  // namespace sm
