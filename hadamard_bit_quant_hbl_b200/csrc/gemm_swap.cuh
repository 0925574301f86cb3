// Ternary x low-bit product for small token counts (M <= 256) on the tensor cores.
//
//   Y[m, n] = s_x[m] * alpha * sum_k q[m, k] * t[k, n]
//
// The layer's product (BitNet v2 walkthrough article, section "H-BitLinear模塊"), exact in int32.
// With few tokens the product is bound by the weight bytes, so the weights are read in their
// 2-bit form (4x fewer bytes than int8) and widened to int8 in shared memory, and the roles are
// swapped: 128 output features form the MMA's M side and the (padded) tokens its N side:
//
//   D[n, m] = sum_k t[k, n] q[m, k],   tcgen05.mma kind::i8, M = 128, N = Mt (16..256), K = 32.
//
// A cluster of S CTAs shares one 128-feature tile and splits K: CTA r owns a contiguous run of
// 128-wide k-blocks, processed in batches of B k-blocks. Its partial sums end in its own shared
// memory and are reduced across the cluster through distributed shared memory, so no global
// workspace is needed.
//
//   warp 0      bulk copies of the 2-bit weight tiles of a batch (B x 4 KB, contiguous in the
//               blob's tile-major section) into a 2-stage ring
//   warp 1      TMEM allocation; one thread issues the batch's B x 4 MMAs and commits once per
//               batch to the "empty" barriers of the widened tiles and of the activations
//   warp 2      TMA copies of the batch's activation tiles (Mt rows x 128 bytes per k-block,
//               128-byte swizzle) into an NA-stage ring
//   warps 3-10  widen the 2-bit rows (two threads per weight row, 64 codes c = t+1 each) to int8
//               t in the 128-byte-swizzled K-major layout the MMA reads (2 batch stages), then
//               the epilogue: tcgen05.ld of the partial sums (warps 3-6), reduction across the
//               cluster, dequant, store.
// The rings take 200 KB (batches of 4 up to 32 tokens, 2 up to 128, else 1), one CTA per SM; the
// partial sums ([Mt][128] int32) reuse them in the epilogue. (Two 100 KB CTAs per SM are faster
// for a lone product but slow the forward pass down: they share SMs with the activation kernel
// that runs before them, whose rows are its critical path.)
// Synchronisation is per batch, not per k-block: one wait, one proxy fence and one arrive per
// widening warp and batch (each costs about as much as widening a k-block).
// The kernel may start while the activation kernel before it still runs (programmatic dependent
// launch): setup, the weight copies and the widening need nothing from it; the activation
// producer and the epilogue wait for it first. Every mbarrier wait is bounded (1 s).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"

namespace hbl {

constexpr int kSwNT = 128;        // output features per tile (MMA M)
constexpr int kSwBK = 128;        // k per block
constexpr int kSwRaw = 128 * 32;  // bytes of one 2-bit weight tile (4 KB, contiguous in the blob)
constexpr int kSwWide = 128 * kSwBK;
constexpr int kSwNR = 2;          // 2-bit copy stages (one batch each)
constexpr int kSwNWB = 2;         // widened batch stages
constexpr int kSwMaxNA = 4;       // activation copy stages (one batch each)
constexpr int kSwWidenWarps = 8;
constexpr int kSwThreads = 32 * (3 + kSwWidenWarps);  // 352
constexpr int kSwSmem = 200 * 1024;  // ring budget, one CTA per SM

struct SwapArgs {
  const uint32_t* w2;  // 2-bit weight section, tile-major (4 KB per 128 x 128 tile)
  const float* s_x;
  float alpha;
  int M, N, K;
  int Mt;           // tokens padded to a multiple of 16 (MMA N)
  int B;            // k-blocks per batch
  int NA;           // activation ring stages
  int S;            // CTAs per cluster (k split)
  int tmem_cols;
  void* Y;
  int out_bf16;
  int32_t* acc_debug;
};

__device__ __forceinline__ uint32_t idesc_i8_mn(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// 32 lanes x 16 consecutive 32-bit columns, waited in the same statement.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Bounded wait for the last phase armed on a barrier (used only on the abort path, so that no
// copy is in flight into shared memory when the CTA exits).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < kWaitLimitNs) {
  }
}

__global__ void __launch_bounds__(kSwThreads, 1)
gemm_swap_kernel(const __grid_constant__ CUtensorMap mapA, const SwapArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw3[];
  __shared__ __align__(8) uint64_t raw_full[kSwNR], raw_empty[kSwNR];
  __shared__ __align__(8) uint64_t act_full[kSwMaxNA], act_empty[kSwMaxNA];
  __shared__ __align__(8) uint64_t wide_full[kSwNWB], wide_empty[kSwNWB], acc_full, drain_bar;
  __shared__ uint32_t tmem_base_slot;
  __shared__ volatile int abort_flag;

  uint8_t* smem = align_shared<1024>(smem_raw3);
  const int NA = a.NA, Mt = a.Mt, B = a.B;
  const int act_bytes = Mt * kSwBK;                 // one k-block of activations, multiple of 2048
  const int act_stage = B * act_bytes;              // one copy: B k-blocks, [B][Mt][128] swizzled
  uint8_t* act = smem;                              // NA x act_stage
  uint8_t* wide = act + NA * act_stage;             // kSwNWB x B x 16 KB (128-byte swizzle)
  uint8_t* raw = wide + kSwNWB * B * kSwWide;       // kSwNR x B x 4 KB

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int S = a.S;
  const int tile = blockIdx.x / S;
  const int n0 = tile * kSwNT;
  const int KB = a.K / kSwBK;
  const int kb0 = (int)(((long)KB * rank) / S), kb1 = (int)(((long)KB * (rank + 1)) / S);
  const int nkb = kb1 - kb0;
  const int nbat = (nkb + B - 1) / B;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kSwNR; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], kSwWidenWarps);  // one lane of each widening warp
    }
    for (int s = 0; s < NA; ++s) {
      mbar_init(&act_full[s], 1);
      mbar_init(&act_empty[s], 1);
    }
    for (int s = 0; s < kSwNWB; ++s) {
      mbar_init(&wide_full[s], kSwWidenWarps);
      mbar_init(&wide_empty[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&mapA);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&tmem_base_slot)), "r"(a.tmem_cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_slot;

  if (warp == 0) {
    // ---------------- 2-bit weight tiles, one bulk copy per batch (runs up to kSwNR ahead)
    if (lane == 0) {
      int b = 0;
      for (; b < nbat; ++b) {
        const int s = b % kSwNR;
        if (!mbar_wait(&raw_empty[s], ((uint32_t)(b / kSwNR) & 1u) ^ 1u, &abort_flag)) break;
        const uint32_t bytes = (uint32_t)min(B, nkb - b * B) * kSwRaw;  // a feature tile's k-blocks are consecutive
        mbar_arrive_expect_tx(&raw_full[s], bytes);
        bulk_load_1d(raw + s * (B * kSwRaw), a.w2 + ((size_t)tile * KB + kb0 + b * B) * 1024, bytes, &raw_full[s]);
      }
      if (abort_flag)  // no copy may still be landing when the CTA exits
        for (int d = max(0, b - kSwNR); d < b; ++d) drain_wait(&raw_full[d % kSwNR], (uint32_t)(d / kSwNR) & 1u);
    }
  } else if (warp == 2) {
    // ---------------- activation tiles, one TMA copy per batch (runs up to NA ahead). The codes
    // may come from the kernel before this one: wait for it (programmatic dependent launch).
    pdl_wait();
    if (lane == 0) {
      int b = 0;
      for (; b < nbat; ++b) {
        const int s = b % NA;
        if (!mbar_wait(&act_empty[s], ((uint32_t)(b / NA) & 1u) ^ 1u, &abort_flag)) break;
        mbar_arrive_expect_tx(&act_full[s], (uint32_t)act_stage);  // the box is always complete
        tma_load_3d(act + s * act_stage, &mapA, &act_full[s], 0, 0, kb0 + b * B);
      }
      if (abort_flag)
        for (int d = max(0, b - NA); d < b; ++d) drain_wait(&act_full[d % NA], (uint32_t)(d / NA) & 1u);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: per batch one wait on each ring, B x 4 MMAs, one commit each
    if (lane == 0) {
      const uint32_t idesc = idesc_i8_mn(kSwNT, Mt);
      bool ok = true, any = false;
      for (int b = 0; b < nbat; ++b) {
        const int ws = b % kSwNWB, as = b % NA;
        if (!mbar_wait(&wide_full[ws], (uint32_t)(b / kSwNWB) & 1u, &abort_flag)) { ok = false; break; }
        if (!mbar_wait(&act_full[as], (uint32_t)(b / NA) & 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const int nb = min(B, nkb - b * B);
        for (int u = 0; u < nb; ++u) {
          const uint32_t w_addr = smem_u32(wide + (ws * B + u) * kSwWide);
          const uint32_t a_addr = smem_u32(act + as * act_stage + u * act_bytes);
#pragma unroll
          for (int kk = 0; kk < kSwBK / 32; ++kk)
            mma_i8(tmem_base, smem_desc_sw128(w_addr + kk * 32), smem_desc_sw128(a_addr + kk * 32), idesc,
                   (b | u | kk) != 0 ? 1u : 0u);
        }
        any = true;
        mma_commit(&wide_empty[ws]);
        mma_commit(&act_empty[as]);
      }
      if (ok && any) mma_commit(&acc_full);
      if (!ok && any) {
        mma_commit(&drain_bar);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ---------------- widen (warps 3-10): thread (row r, half h) turns the 64 codes of words
    // 4h..4h+3 of weight row r into four 16-byte chunks of the swizzled int8 row
    const int tw = threadIdx.x - 96;
    const int row = tw >> 1, h = tw & 1;
    bool ok = true;
    for (int b = 0; b < nbat && ok; ++b) {
      const int rs = b % kSwNR, ws = b % kSwNWB;
      // every lane waits (the copy-written tile must be visible to each reader); the outcome is
      // made uniform so that the warp stays converged
      bool r = mbar_wait(&raw_full[rs], (uint32_t)(b / kSwNR) & 1u, &abort_flag);
      if (r) r = mbar_wait(&wide_empty[ws], ((uint32_t)(b / kSwNWB) & 1u) ^ 1u, &abort_flag);
      if (!__all_sync(0xffffffffu, r)) { ok = false; break; }
      const int nb = min(B, nkb - b * B);
      for (int u = 0; u < nb; ++u) {
        const uint4 wv = *reinterpret_cast<const uint4*>(raw + (rs * B + u) * kSwRaw + row * 32 + h * 16);
        const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
        uint8_t* dst = wide + (ws * B + u) * kSwWide + row * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // word 4h+i: 16 codes k = 16(4h+i) + 4s' + b, c' = t + 1 in {0,1,2}
          uint32_t o[4];
#pragma unroll
          for (int sp = 0; sp < 4; ++sp) {
            const uint32_t u8 = (wd[i] >> (2 * sp)) & 0x03030303u;  // c' per byte
            o[sp] = (u8 + 0x7f7f7f7fu) ^ 0x80808080u;               // int8 t = c' - 1, no carries
          }
          const int c = 4 * h + i;
          *reinterpret_cast<uint4*>(dst + ((c ^ (row & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&raw_empty[rs]);  // this warp's reads of the 2-bit copy are done
      fence_proxy_async_smem();                    // generic-proxy writes -> visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&wide_full[ws]);
    }

    // ---------------- epilogue part 1: partial sums -> own shared memory as [Mt][128] int32
    // (warps 3-6, one per TMEM lane quarter)
    bool r = ok && mbar_wait(&acc_full, 0, &abort_flag);
    r = __all_sync(0xffffffffu, r);
    int32_t* part = reinterpret_cast<int32_t*>(smem);  // the rings are idle now
    if (warp <= 6) {
      const int q = warp & 3;  // TMEM lane quarter
      const int f = q * 32 + lane;
      if (r && nkb > 0) {
        tc_fence_after();
        for (int c0 = 0; c0 < Mt; c0 += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) part[(c0 + j) * kSwNT + f] = (int32_t)v[j];
        }
      } else {
        for (int m = 0; m < Mt; ++m) part[m * kSwNT + f] = 0;
      }
    }
  }

  // the next kernel of the stream may launch now (it waits for this one before reading Y)
  pdl_launch_dependents();
  pdl_wait();  // s_x below comes from the kernel before this one

  // ---------------- epilogue part 2: reduce the cluster's partial sums, dequant, store
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp >= 3) {
    const uint32_t part0 = smem_u32(smem);
    const int t = threadIdx.x - 96;
    const int nt = 32 * kSwWidenWarps;
    for (int e = (int)rank * nt + t; e < Mt * kSwNT; e += S * nt) {
      const int m = e / kSwNT, f = e - m * kSwNT;
      const int n = n0 + f;
      if (m >= a.M || n >= a.N) continue;
      uint32_t pv[8];
#pragma unroll
      for (int p = 0; p < 8; ++p)  // all remote loads in flight before the sum
        pv[p] = p < S ? ld_shared_cluster_u32(mapa_shared(part0 + (uint32_t)e * 4u, (uint32_t)p)) : 0u;
      int32_t acc = 0;
#pragma unroll
      for (int p = 0; p < 8; ++p) acc += (int32_t)pv[p];  // fixed order
      const float y = (float)acc * (a.s_x[m] * a.alpha);
      if (a.out_bf16) reinterpret_cast<__nv_bfloat16*>(a.Y)[(size_t)m * a.N + n] = __float2bfloat16_rn(y);
      else reinterpret_cast<float*>(a.Y)[(size_t)m * a.N + n] = y;
      if (a.acc_debug) a.acc_debug[(size_t)m * a.N + n] = acc;
    }
  }
  __syncwarp();
  cluster_sync_all();  // no CTA leaves while a peer may still read its shared memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(a.tmem_cols)
                 : "memory");
  }
}

}  // namespace hbl
