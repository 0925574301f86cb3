// Ternary x low-bit product for prefill-sized token counts on the sm_100a tensor cores.
//
//   Y[m, n] = s_x[m] * alpha * sum_k q[m, k] * t[k, n]
//
// The layer's product (BitNet v2 walkthrough article, section "H-BitLinear模塊"). Integer codes
// (activations in [-8, 7] or [-128, 127], weights in {-1, 0, 1}) are multiplied exactly by
// tcgen05.mma kind::i8 with int32 accumulation in tensor memory.
//
// Structure (one CTA per SM, persistent over 128 x 256 output tiles, 6 warps):
//   warp 0     TMA producer: 128x128-byte A tile and 256x128-byte B tile per k-block into a
//              4-stage shared-memory ring (128-byte swizzle), completion on an mbarrier.
//   warp 1     allocates all 512 TMEM columns (two 256-column accumulators), one thread issues
//              4 MMAs of K = 32 per k-block and commits to the stage's "empty" barrier and,
//              after the last k-block, to the accumulator's "full" barrier.
//   warps 2-5  epilogue: tcgen05.ld 32 lanes x 32 columns at a time, scale by s_x[m] * alpha,
//              store fp32 or bf16; then release the accumulator so the MMA warp can reuse it
//              while the next tile's epilogue runs on the other one.
// Every mbarrier wait is bounded (1 s of wall clock); on time-out the kernel raises the device
// error flag, stops issuing work, waits (bounded) for its own copies and MMAs, frees TMEM and
// returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace hbl {

constexpr int kTcBM = 128, kTcBN = 256, kTcBK = 128;
constexpr int kTcStages = 4;
constexpr int kTcStageA = kTcBM * kTcBK;  // bytes
constexpr int kTcStageB = kTcBN * kTcBK;
constexpr int kTcSmem = kTcStages * (kTcStageA + kTcStageB) + 1024;  // + alignment slack
constexpr int kTcThreads = 192;

struct TcArgs {
  const float* s_x;
  float alpha;
  int M, N, K;
  void* Y;
  int out_bf16;
  int32_t* acc_debug;
  int tiles_m, tiles_n;
};

// ---------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fffu);        // start address
  d |= (uint64_t)1u << 16;                       // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;             // stride byte offset: next 8-row group
  d |= (uint64_t)1u << 46;                       // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                       // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::i8, s8 x s8 -> s32, both K-major, M = 128, N = 256.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4)                    // D format: s32
         | (1u << 7)                  // A: signed 8-bit
         | (1u << 10)                 // B: signed 8-bit
         | ((uint32_t)(N >> 3) << 17)  // N / 8
         | ((uint32_t)(M >> 4) << 24); // M / 16
}

__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns per warp; waits for the load in the same statement so
// that no use of the outputs can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// ---------------------------------------------------------------- the kernel

__global__ void __launch_bounds__(kTcThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
               const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kTcStages], empty_bar[kTcStages];
  __shared__ __align__(8) uint64_t accf_bar[2], acce_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_slot;
  __shared__ volatile int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smem + kTcStages * kTcStageA;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = a.K / kTcBK;
  const int ntiles = a.tiles_m * a.tiles_n;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf_bar[b], 1);
      mbar_init(&acce_bar[b], 128);
    }
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;"
                 ::"r"(smem_u32(&tmem_base_slot)) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_slot;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued[kTcStages] = {0, 0, 0, 0};
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int tm = tile % a.tiles_m, tn = tile / a.tiles_m;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], kTcStageA + kTcStageB);
          tma_load_2d(smA + stage * kTcStageA, &mapA, &full_bar[stage], kb * kTcBK, tm * kTcBM);
          tma_load_2d(smB + stage * kTcStageB, &mapB, &full_bar[stage], kb * kTcBK, tn * kTcBN);
          ++issued[stage];
          if (++stage == kTcStages) { stage = 0; phase ^= 1u; }
        }
      }
      // every copy this thread issued has landed before the CTA may exit
      for (int s = 0; s < kTcStages; ++s) {
        if (issued[s] > 0) {
          // the last phase armed on stage s has parity (issued[s] - 1) & 1
          if (!mbar_try_wait(&full_bar[s], (uint32_t)((issued[s] - 1) & 1))) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&full_bar[s], (uint32_t)((issued[s] - 1) & 1)) &&
                   globaltimer_ns() - t0 < kWaitLimitNs) {
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kTcBM, kTcBN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      bool any = false;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);  // how many times this buffer was used before
        if (!mbar_wait(&acce_bar[buf], (use & 1u) ^ 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + (uint32_t)(buf * kTcBN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smA + stage * kTcStageA);
          const uint32_t b_addr = smem_u32(smB + stage * kTcStageB);
#pragma unroll
          for (int kk = 0; kk < kTcBK / 32; ++kk) {
            mma_i8(tmem_d, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                   (kb | kk) != 0 ? 1u : 0u);
          }
          any = true;
          mma_commit(&empty_bar[stage]);
          if (++stage == kTcStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&accf_bar[buf]);
      }
      if (!ok && any) {
        // no MMA may still be running when TMEM is released
        mma_commit(&drain_bar);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5 -> TMEM lane quarter (warp % 4)
    const int q = warp & 3;
    int local = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++local) {
      const int buf = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      // one lane waits; the outcome is broadcast so that the warp stays converged for the
      // .sync.aligned TMEM loads below
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&accf_bar[buf], use & 1u, &abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int tm = tile % a.tiles_m, tn = tile / a.tiles_m;
      const int row = tm * kTcBM + q * 32 + lane;
      const bool rok = row < a.M;
      const float scale = rok ? a.s_x[row] * a.alpha : 0.f;
#pragma unroll 1
      for (int c = 0; c < kTcBN / 32; ++c) {
        uint32_t r[32];
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kTcBN + c * 32);
        tmem_ld_32x32b_x32(taddr, r);
        const int col0 = tn * kTcBN + c * 32;
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
      mbar_arrive(&acce_bar[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem_base) : "memory");
  }
}

}  // namespace hbl
