// Ternary x low-bit product on a pair of SMs (tcgen05 cta_group::2), for token counts >= 256.
//
//   Y[m, n] = s_x[m] * alpha * sum_k q[m, k] * t[k, n]
//
// The layer's product (BitNet v2 walkthrough article, section "H-BitLinear模塊"), exact in int32.
//
// A cluster of two CTAs (one per SM) computes 256 x 256 output tiles: CTA r holds rows
// 128r .. 128r+127 of the A tile and rows 128r .. 128r+127 (output columns) of the B tile in
// shared memory, and rows 128r .. 128r+127 of the accumulator in its tensor memory. The leader
// (rank 0) issues one tcgen05.mma.cta_group::2.kind::i8 per 32-wide k step, which reads both
// CTAs' shared memory; per SM this moves half the B bytes of the single-SM 128 x 256 tile.
//
//   warp 0     TMA producer in each CTA: its A half and B half of every k-block into a 6-stage
//              ring. The copies signal the LEADER's "full" barrier (64 KB per stage in total).
//   warp 1     TMEM: 512 columns in each CTA (two 256-column accumulators). The leader's lane 0
//              waits for full stages and issues the MMAs; each stage is released by a commit
//              that arrives on the "empty" barrier of both CTAs; after the last k-block a commit
//              arrives on the accumulator's "full" barrier of both CTAs.
//   warps 2-5  epilogue in each CTA: tcgen05.ld, scale, store; then one lane per warp arrives on
//              the leader's "accumulator empty" barrier.
// Output tiles are visited in groups of 8 tile rows so that the A and B rows that concurrently
// running clusters read overlap in L2. Every wait is bounded (1 s).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm_tc.cuh"

namespace hbl {

constexpr int kT2BM = 256, kT2BN = 256, kT2BK = 128;  // pair tile
constexpr int kT2Stages = 6;
constexpr int kT2StageA = 128 * kT2BK;                  // bytes per CTA
constexpr int kT2StageB = 128 * kT2BK;                  // bytes per CTA (half of the N tile)
constexpr int kT2Smem = kT2Stages * (kT2StageA + kT2StageB) + 1024;
constexpr int kT2Threads = 192;
constexpr int kT2GroupM = 8;

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA 2-D load into this CTA's shared memory, completion counted on a barrier that may be in
// the peer CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster_addr,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(bar_cluster_addr), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void mma_i8_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on the barrier at this offset in both CTAs of the pair when the MMAs issued so
// far have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
               ::"r"(smem_u32(bar)), "h"(mask) : "memory");
}

struct Tc2Args {
  const float* s_x;
  float alpha;
  int M, N, K;
  void* Y;
  int out_bf16;
  int32_t* acc_debug;
  int tiles_m, tiles_n;  // in 256 x 256 pair tiles
};

__device__ __forceinline__ void tc2_tile_coords(int t, int tiles_m, int tiles_n, int& tm, int& tn) {
  const int group = kT2GroupM * tiles_n;
  const int g = t / group;
  const int first_m = g * kT2GroupM;
  const int gm = min(kT2GroupM, tiles_m - first_m);
  const int r = t - g * group;
  tm = first_m + r % gm;
  tn = r / gm;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kT2Threads, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                const Tc2Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw2[];
  __shared__ __align__(8) uint64_t full_bar[kT2Stages], empty_bar[kT2Stages];
  __shared__ __align__(8) uint64_t accf_bar[2], acce_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_slot;
  __shared__ volatile int abort_flag;

  uint8_t* smem = align_shared<1024>(smem_raw2);
  uint8_t* smA = smem;
  uint8_t* smB = smem + kT2Stages * kT2StageA;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int KB = a.K / kT2BK;
  const int ntiles = a.tiles_m * a.tiles_n;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kT2Stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf_bar[b], 1);
      mbar_init(&acce_bar[b], 8);  // one lane of each epilogue warp of both CTAs
    }
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;"
                 ::"r"(smem_u32(&tmem_base_slot)) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_slot;
  // The setup above may overlap the kernel before this one (programmatic dependent launch); the
  // codes and s_x come from it, so wait for it here. The next kernel may then be scheduled onto
  // the SMs this grid leaves as its clusters finish (it waits for this grid before reading Y).
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full0_leader = mapa_shared(smem_u32(&full_bar[0]), 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = cluster; t < ntiles && ok; t += nclusters) {
        int tm, tn;
        tc2_tile_coords(t, a.tiles_m, a.tiles_n, tm, tn);
        const int rowA = tm * kT2BM + (int)rank * 128;
        const int rowB = tn * kT2BN + (int)rank * 128;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2u * (kT2StageA + kT2StageB));
          const uint32_t fb = full0_leader + (uint32_t)(stage * sizeof(uint64_t));
          tma_load_2d_pair(smA + stage * kT2StageA, &mapA, fb, kb * kT2BK, rowA);
          tma_load_2d_pair(smB + stage * kT2StageB, &mapB, fb, kb * kT2BK, rowB);
          if (++stage == kT2Stages) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kT2BM, kT2BN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true, any = false;
      for (int t = cluster; t < ntiles && ok; t += nclusters, ++local) {
        const int buf = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!mbar_wait(&acce_bar[buf], (use & 1u) ^ 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + (uint32_t)(buf * kT2BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smA + stage * kT2StageA);
          const uint32_t b_addr = smem_u32(smB + stage * kT2StageB);
#pragma unroll
          for (int kk = 0; kk < kT2BK / 32; ++kk) {
            mma_i8_pair(tmem_d, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                        (kb | kk) != 0 ? 1u : 0u);
          }
          any = true;
          mma_commit_pair(&empty_bar[stage]);
          if (++stage == kT2Stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit_pair(&accf_bar[buf]);
      }
      if (!ok && any) {
        // completion of everything issued so far, tracked for the pair's MMAs
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                     ::"r"(smem_u32(&drain_bar)) : "memory");
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5 -> TMEM lane quarter (warp % 4)
    const int q = warp & 3;
    const uint32_t acce_leader = mapa_shared(smem_u32(&acce_bar[0]), 0);
    int local = 0;
    for (int t = cluster; t < ntiles; t += nclusters, ++local) {
      const int buf = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&accf_bar[buf], use & 1u, &abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      int tm, tn;
      tc2_tile_coords(t, a.tiles_m, a.tiles_n, tm, tn);
      const int row = tm * kT2BM + (int)rank * 128 + q * 32 + lane;
      const bool rok = row < a.M;
      const float scale = rok ? a.s_x[row] * a.alpha : 0.f;
#pragma unroll 1
      for (int c = 0; c < kT2BN / 32; ++c) {
        uint32_t r[32];
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kT2BN + c * 32);
        tmem_ld_32x32b_x32(taddr, r);
        const int col0 = tn * kT2BN + c * 32;
        if (rok && col0 < a.N) {
          const bool full = col0 + 32 <= a.N;
          if (a.out_bf16) {
            __nv_bfloat16* yrow = reinterpret_cast<__nv_bfloat16*>(a.Y) + (size_t)row * a.N + col0;
            if (full) {
#pragma unroll
              for (int j = 0; j < 32; j += 8) {
                uint4 o;
                uint32_t* op = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  const __nv_bfloat162 p2 = __floats2bfloat162_rn((float)(int)r[j + 2 * h] * scale,
                                                                 (float)(int)r[j + 2 * h + 1] * scale);
                  op[h] = *reinterpret_cast<const uint32_t*>(&p2);
                }
                *reinterpret_cast<uint4*>(yrow + j) = o;
              }
            } else {
              for (int j = 0; j < 32 && col0 + j < a.N; ++j) yrow[j] = __float2bfloat16_rn((float)(int)r[j] * scale);
            }
          } else {
            float* yrow = reinterpret_cast<float*>(a.Y) + (size_t)row * a.N + col0;
            if (full) {
#pragma unroll
              for (int j = 0; j < 32; j += 4) {
                *reinterpret_cast<float4*>(yrow + j) =
                    make_float4((float)(int)r[j] * scale, (float)(int)r[j + 1] * scale,
                                (float)(int)r[j + 2] * scale, (float)(int)r[j + 3] * scale);
              }
            } else {
              for (int j = 0; j < 32 && col0 + j < a.N; ++j) yrow[j] = (float)(int)r[j] * scale;
            }
          }
          if (a.acc_debug) {
            int32_t* drow = a.acc_debug + (size_t)row * a.N + col0;
            for (int j = 0; j < 32 && col0 + j < a.N; ++j) drow[j] = (int32_t)r[j];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce_leader + (uint32_t)(buf * sizeof(uint64_t)));
    }
  }

  // both CTAs are done with TMEM and with each other's barriers and shared memory
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem_base) : "memory");
  }
}

// ---------------------------------------------------------------- split-K over two SM pairs
//
// For token counts whose 256 x 256 tiles would leave half the SM pairs idle (M = 512 at N = 4096
// gives 32 tiles for 74 pairs), a cluster of four CTAs (two SM pairs) computes one tile: pair p
// accumulates the k-blocks [KB p / 2, KB (p + 1) / 2) in its own tensor memory, exactly as above.
// Then pair 1 writes its int32 partial sums into the shared memory of the matching CTA of pair 0
// (distributed shared memory; the rings are idle by then), and pair 0 adds them to its own in the
// epilogue. Integer sums: the result is bit-identical to the one-pair kernel's.
constexpr int kT2sRed = 128 * kT2BN * 4;  // bytes of one CTA's partial sums (128 rows x 256 int32)
static_assert(kT2sRed <= kT2Stages * (kT2StageA + kT2StageB), "partial sums fit in the ring");

__global__ void __launch_bounds__(kT2Threads, 1)
gemm_tc2s_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                 const Tc2Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw2s[];
  __shared__ __align__(8) uint64_t full_bar[kT2Stages], empty_bar[kT2Stages];
  __shared__ __align__(8) uint64_t accf_bar, drain_bar;
  __shared__ uint32_t tmem_base_slot;
  __shared__ volatile int abort_flag;

  uint8_t* smem = align_shared<1024>(smem_raw2s);
  uint8_t* smA = smem;
  uint8_t* smB = smem + kT2Stages * kT2StageA;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();      // 0..3
  const uint32_t pair = rank >> 1, r = rank & 1;
  const uint32_t lead = rank & ~1u;             // the pair's leader
  const bool leader = r == 0;
  const int t = blockIdx.x >> 2;                // one tile per cluster
  const int tm = t / a.tiles_n, tn = t - tm * a.tiles_n;
  const int KB = a.K / kT2BK;
  const int kb0 = (int)(pair * KB / 2), kb1 = (int)((pair + 1) * KB / 2);
  const uint16_t pair_mask = (uint16_t)(0x3u << (2 * pair));

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int st = 0; st < kT2Stages; ++st) {
      mbar_init(&full_bar[st], 1);
      mbar_init(&empty_bar[st], 1);
    }
    mbar_init(&accf_bar, 1);
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 256;"
                 ::"r"(smem_u32(&tmem_base_slot)) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in all four CTAs
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_slot;
  pdl_wait();  // the codes and s_x come from the kernel before this one
  pdl_launch_dependents();

  bool ok = true;
  if (warp == 0) {
    // ---------------- TMA producer (every CTA): its halves of the pair's k-blocks
    if (lane == 0) {
      const uint32_t full0_leader = mapa_shared(smem_u32(&full_bar[0]), lead);
      const int rowA = tm * kT2BM + (int)r * 128;
      const int rowB = tn * kT2BN + (int)r * 128;
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag)) break;
        if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2u * (kT2StageA + kT2StageB));
        const uint32_t fb = full0_leader + (uint32_t)(stage * sizeof(uint64_t));
        tma_load_2d_pair(smA + stage * kT2StageA, &mapA, fb, kb * kT2BK, rowA);
        tma_load_2d_pair(smB + stage * kT2StageB, &mapB, fb, kb * kT2BK, rowB);
        if (++stage == kT2Stages) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (the pair's leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kT2BM, kT2BN);
      int stage = 0;
      uint32_t phase = 0;
      bool any = false;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full_bar[stage], phase, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smA + stage * kT2StageA);
        const uint32_t b_addr = smem_u32(smB + stage * kT2StageB);
#pragma unroll
        for (int kk = 0; kk < kT2BK / 32; ++kk)
          mma_i8_pair(tmem_base, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                      (kb > kb0 || kk) ? 1u : 0u);
        any = true;
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                     ::"r"(smem_u32(&empty_bar[stage])), "h"(pair_mask) : "memory");
        if (++stage == kT2Stages) { stage = 0; phase ^= 1u; }
      }
      if (ok) {
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                     ::"r"(smem_u32(&accf_bar)), "h"(pair_mask) : "memory");
      } else if (any) {
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                     ::"r"(smem_u32(&drain_bar)) : "memory");
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  }

  // ---------------- the pair's sum is complete in its tensor memory (epilogue warps 2..5, TMEM
  // lane quarter warp % 4: rows 32 q .. 32 q + 31 of this CTA's 128)
  const int q = warp & 3;
  int acc_ok = 1;
  if (warp >= 2) {
    if (lane == 0) acc_ok = mbar_wait(&accf_bar, 0, &abort_flag) ? 1 : 0;
    acc_ok = __shfl_sync(0xffffffffu, acc_ok, 0);
    tc_fence_after();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();  // both pairs' main loops are done: every ring is idle
  tc_fence_after();
  const int lrow = q * 32 + lane;  // row within this CTA's 128
  int32_t* red = reinterpret_cast<int32_t*>(smem);  // [128 rows][256] partial sums of pair 1
  if (warp >= 2 && pair == 1) {
    // pair 1: partial sums into the matching CTA of pair 0, row-major int32
    const uint32_t dst0 = mapa_shared(smem_u32(red), rank - 2);
#pragma unroll 1
    for (int c = 0; c < kT2BN / 32; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * 32), v);
      if (!acc_ok) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0u;
      }
      const uint32_t dst = dst0 + (uint32_t)((lrow * kT2BN + c * 32) * 4);
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};"
                     ::"r"(dst + (uint32_t)(j * 4)), "r"(v[j]), "r"(v[j + 1]), "r"(v[j + 2]), "r"(v[j + 3]) : "memory");
    }
  }
  tc_fence_before();
  cluster_sync_all();  // pair 1's partial sums have landed in pair 0
  tc_fence_after();
  if (warp >= 2 && pair == 0) {
    const int row = tm * kT2BM + (int)r * 128 + lrow;
    const bool rok = row < a.M;
    const float scale = rok ? a.s_x[row] * a.alpha : 0.f;
#pragma unroll 1
    for (int c = 0; c < kT2BN / 32; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * 32), v);
      const int col0 = tn * kT2BN + c * 32;
      if (!rok || col0 >= a.N) continue;
      const int32_t* pr = red + lrow * kT2BN + c * 32;
      int32_t s32[32];
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const int4 p4 = *reinterpret_cast<const int4*>(pr + j);
        s32[j] = (acc_ok ? (int32_t)v[j] : 0) + p4.x;
        s32[j + 1] = (acc_ok ? (int32_t)v[j + 1] : 0) + p4.y;
        s32[j + 2] = (acc_ok ? (int32_t)v[j + 2] : 0) + p4.z;
        s32[j + 3] = (acc_ok ? (int32_t)v[j + 3] : 0) + p4.w;
      }
      const bool full = col0 + 32 <= a.N;
      if (a.out_bf16) {
        __nv_bfloat16* yrow = reinterpret_cast<__nv_bfloat16*>(a.Y) + (size_t)row * a.N + col0;
        if (full) {
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 o;
            uint32_t* op = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const __nv_bfloat162 p2 = __floats2bfloat162_rn((float)s32[j + 2 * h] * scale,
                                                             (float)s32[j + 2 * h + 1] * scale);
              op[h] = *reinterpret_cast<const uint32_t*>(&p2);
            }
            *reinterpret_cast<uint4*>(yrow + j) = o;
          }
        } else {
          for (int j = 0; j < 32 && col0 + j < a.N; ++j) yrow[j] = __float2bfloat16_rn((float)s32[j] * scale);
        }
      } else {
        float* yrow = reinterpret_cast<float*>(a.Y) + (size_t)row * a.N + col0;
        if (full) {
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(yrow + j) = make_float4((float)s32[j] * scale, (float)s32[j + 1] * scale,
                                                               (float)s32[j + 2] * scale, (float)s32[j + 3] * scale);
        } else {
          for (int j = 0; j < 32 && col0 + j < a.N; ++j) yrow[j] = (float)s32[j] * scale;
        }
      }
      if (a.acc_debug) {
        int32_t* drow = a.acc_debug + (size_t)row * a.N + col0;
        for (int j = 0; j < 32 && col0 + j < a.N; ++j) drow[j] = s32[j];
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 256;" ::"r"(tmem_base) : "memory");
  }
}

}  // namespace hbl
