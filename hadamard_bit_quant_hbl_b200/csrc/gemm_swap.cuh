// Ternary x low-bit product for small token counts (M <= 256) on the tensor cores.
//
//   Y[m, n] = s_x[m] * alpha * sum_k q[m, k] * t[k, n]
//
// The layer's product (BitNet v2 walkthrough article, section "H-BitLinear模塊"), exact in int32.
// With few tokens the product is bound by the weight bytes, so the weights are read in their
// 2-bit form (4x fewer bytes than int8) and the roles are swapped: 128 output features form the
// MMA's M side and the (padded) tokens its N side:
//
//   D[n, m] = sum_k t[k, n] q[m, k],   tcgen05.mma kind::i8, M = 128, N = Mt (16..256), K = 32,
//
// with the weights as the A operand in tensor memory: the widening threads turn each 2-bit row
// into int8 in registers and store it with tcgen05.st, so the widened weights (4x the 2-bit bytes)
// never pass through shared memory, whose bandwidth bounded an earlier form of this kernel. A
// widened byte is 64 t rather than t (two instructions per 4 codes: the code plane shifted to bits
// 6..7 plus 0xc0 per byte, masked to bits 6..7, turns c' = t + 1 in {0, 1, 2} into the int8 bytes
// 0xc0, 0x00, 0x40; the carries only reach the masked-off bits), so the MMAs accumulate
// 64 sum t q, divided back exactly in the epilogue (|64 sum t q| <= 2^28 for K <= 32768).
//
// A cluster of S CTAs shares one 128-feature tile and splits K: CTA r owns a contiguous run of
// 128-wide k-blocks, processed in batches of BK k-blocks. Its partial sums end in its own shared
// memory and are reduced across the cluster through distributed shared memory, so no global
// workspace is needed.
//
//   warp 0      bulk copies of the 2-bit weight tiles of a batch (BK x 4 KB, contiguous in the
//               blob's tile-major section) into an NR-stage ring; the first kSwEarly during setup,
//               the rest only once the first activation copy is issued (the weight copies would
//               otherwise queue ahead of it in DRAM and delay the first MMA)
//   warp 1      TMEM allocation (512 columns: nis accumulators, then NS batch slots of widened
//               weights); one thread issues batches 0, nis, 2 nis, ...: BK x 4 MMAs and one
//               commit to each of the slot's and the activation stage's "empty" barriers
//   warp 2      TMA copies of the batch's activation tiles (Mt rows x 128 bytes per k-block,
//               128-byte swizzle) into an NA-stage ring
//   warp 3      s_x * alpha into shared memory for the epilogue; with nis = 2 (up to 128 tokens)
//               one thread also issues batches 1, 3, ... into the second accumulator: a small-N
//               MMA occupies the tensor core for about 45 cycles, less than one thread needs to
//               issue it while the widening warps share its scheduler
//   warps 4-11  widen: warp w serves TMEM lane quarter w % 4 (thread = weight row) and every
//               kSwW-th batch; then the epilogue (tcgen05.ld of the partial sums by warps 4-7,
//               reduction across the cluster, dequant, store)
// Ring positions advance by counters, not divisions. A thread that takes every p-th batch waits
// on rings whose stage count is a multiple of p (or at least p for the slots, which are filled in
// batch order), so that it never waits two phases ahead, where a parity wait would alias.
// The kernel may start while the activation kernel before it still runs (programmatic dependent
// launch): setup, the weight copies and the widening need nothing from it; the activation
// producer and s_x wait for it first. Every mbarrier wait is bounded (1 s).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm_tc.cuh"

namespace hbl {

constexpr int kSwNT = 128;        // output features per tile (MMA M)
constexpr int kSwBK = 128;        // k per block
constexpr int kSwRaw = 128 * 32;  // bytes of one 2-bit weight tile (4 KB, contiguous in the blob)
constexpr int kSwW = 2;           // widening warps per TMEM lane quarter
constexpr int kSwWidenWarps = 4 * kSwW;
constexpr int kSwThreads = 32 * (4 + kSwWidenWarps);
constexpr int kSwSmem = 200 * 1024;  // ring budget, one CTA per SM
constexpr int kSwMaxNR = 8;          // 2-bit copy stages (one batch each)
constexpr int kSwMaxNA = 8;          // activation copy stages (one batch each)
constexpr int kSwMaxNS = 8;          // widened batch slots in tensor memory
constexpr int kSwTmemCols = 512;
constexpr int kSwEarly = 2;           // weight copies issued before the first activation copy

struct SwapArgs {
  const uint32_t* w2;  // 2-bit weight section, tile-major (4 KB per 128 x 128 tile)
  const float* s_x;
  float alpha;
  int M, N, K;
  int Mt;           // tokens padded to a multiple of 16 (MMA N)
  int NR, NA;       // 2-bit and activation ring stages
  int NS;           // widened batch slots in tensor memory
  int acc_cols;     // tensor-memory columns before the first slot (nis accumulators)
  int acc_stride;   // columns between the accumulators (>= Mt)
  int nis;          // MMA-issuing threads (1 or 2), each with its own accumulator
  int S;            // CTAs per cluster (k split)
  void* Y;
  int out_bf16;
  int32_t* acc_debug;
};

__device__ __forceinline__ uint32_t idesc_i8_mn(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D (TMEM) [+]= A (TMEM, M = 128 lanes x 8 columns of 4 int8) x B (shared memory descriptor).
__device__ __forceinline__ void mma_i8_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from this thread's registers (asynchronous: ordered
// before later reads of those columns by tmem_st_wait and a thread-sync fence).
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

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

// Synchronises the warps that use tensor memory (all but the two copy warps) on a named barrier.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Bounded wait for the last phase armed on a barrier (used only on the abort path, so that no
// copy is in flight into shared memory when the CTA exits).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < kWaitLimitNs) {
  }
}

template <int BK>
__global__ void __launch_bounds__(kSwThreads, 1)
gemm_swap_kernel(const __grid_constant__ CUtensorMap mapA, const SwapArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw3[];
  __shared__ __align__(8) uint64_t raw_full[kSwMaxNR], raw_empty[kSwMaxNR];
  __shared__ __align__(8) uint64_t act_full[kSwMaxNA], act_empty[kSwMaxNA];
  __shared__ __align__(8) uint64_t slot_full[kSwMaxNS], slot_empty[kSwMaxNS], acc_full, drain_bar[2], act_go;
  __shared__ uint32_t tmem_base_slot;
  __shared__ volatile int abort_flag;
  __shared__ float sxa[256];  // s_x[m] * alpha, staged for the epilogue

  uint8_t* smem = align_shared<1024>(smem_raw3);
  const int NA = a.NA, NR = a.NR, NS = a.NS, Mt = a.Mt;
  const int act_bytes = Mt * kSwBK;     // one k-block of activations, multiple of 2048
  const int act_stage = BK * act_bytes;  // one copy: BK k-blocks, [BK][Mt][128] swizzled
  constexpr int raw_stage = BK * kSwRaw;
  uint8_t* act = smem;                   // NA x act_stage
  uint8_t* raw = act + NA * act_stage;   // NR x raw_stage

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int S = a.S;
  const int tile = blockIdx.x / S;
  const int n0 = tile * kSwNT;
  const int KB = a.K / kSwBK;
  const int kb0 = (int)(((long)KB * rank) / S), kb1 = (int)(((long)KB * (rank + 1)) / S);
  const int nkb = kb1 - kb0;
  const int nbat = (nkb + BK - 1) / BK;
  // weight copies issued before the activations are (they would queue ahead of them in DRAM)
  const int early = min(kSwEarly, min(NR, nbat));
  const uint32_t* w2 = a.w2 + ((size_t)tile * KB + kb0) * 1024;  // this CTA's k-blocks, 4 KB each

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < NR; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], 4);  // one warp per lane quarter reads a batch
    }
    for (int s = 0; s < NA; ++s) {
      mbar_init(&act_full[s], 1);
      mbar_init(&act_empty[s], 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&slot_full[s], 4);  // one warp per lane quarter writes a slot
      mbar_init(&slot_empty[s], 1);
    }
    mbar_init(&acc_full, (uint32_t)min(a.nis, nbat));  // one commit per issuer that had work
    mbar_init(&drain_bar[0], 1);
    mbar_init(&drain_bar[1], 1);
    mbar_init(&act_go, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&mapA);
    for (int b = 0; b < early; ++b) {  // no ring slot to wait for
      const uint32_t bytes = (uint32_t)min(BK, nkb - b * BK) * kSwRaw;
      mbar_arrive_expect_tx(&raw_full[b], bytes);
      bulk_load_1d(raw + b * raw_stage, w2 + (size_t)b * BK * 1024, bytes, &raw_full[b]);
    }
  }
  __syncthreads();

  bool ok = true;
  uint32_t tmem_base = 0;
  if (warp == 0) {
    // ---------------- 2-bit weight tiles, one bulk copy per batch into an NR-stage ring; the
    // copies after the early ones wait until the first activation copy has been issued
    if (lane == 0) {
      int b = early;
      RingPos p;
      p.advance(early, NR);
      bool go = nbat <= early || mbar_wait(&act_go, 0, &abort_flag);
      for (; go && b < nbat; ++b) {
        if (!mbar_wait(&raw_empty[p.s], p.ph ^ 1u, &abort_flag)) break;
        const uint32_t bytes = (uint32_t)min(BK, nkb - b * BK) * kSwRaw;  // a feature tile's k-blocks are consecutive
        mbar_arrive_expect_tx(&raw_full[p.s], bytes);
        bulk_load_1d(raw + p.s * raw_stage, w2 + (size_t)b * BK * 1024, bytes, &raw_full[p.s]);
        p.advance(1, NR);
      }
      if (abort_flag)  // no copy may still be landing when the CTA exits
        for (int d = max(0, b - NR); d < b; ++d) drain_wait(&raw_full[d % NR], (uint32_t)(d / NR) & 1u);
    }
  } else if (warp == 2) {
    // ---------------- activation tiles, one TMA copy per batch (runs up to NA ahead). The codes
    // may come from the kernel before this one: wait for it (programmatic dependent launch).
    pdl_wait();
    if (lane == 0) {
      int b = 0;
      RingPos p;
      for (; b < nbat; ++b) {
        if (!mbar_wait(&act_empty[p.s], p.ph ^ 1u, &abort_flag)) break;
        mbar_arrive_expect_tx(&act_full[p.s], (uint32_t)act_stage);  // the box is always complete
        tma_load_3d(act + p.s * act_stage, &mapA, &act_full[p.s], 0, 0, kb0 + b * BK);
        if (b == 0) mbar_arrive(&act_go);
        p.advance(1, NA);
      }
      if (abort_flag)
        for (int d = max(0, b - NA); d < b; ++d) drain_wait(&act_full[d % NA], (uint32_t)(d / NA) & 1u);
    }
  } else {
    if (warp == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                   ::"r"(smem_u32(&tmem_base_slot)), "r"(kSwTmemCols) : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    named_bar_sync(1, 32 * (2 + kSwWidenWarps));  // warps 1, 3 and the widening warps
    tc_fence_after();
    tmem_base = tmem_base_slot;

    if (warp == 3 && a.nis == 1) {
      // ---------------- s_x * alpha staged for the epilogue (s_x may come from the kernel before)
      pdl_wait();
      for (int m = lane; m < a.M; m += 32) sxa[m] = a.s_x[m] * a.alpha;
    } else if (warp == 1 || warp == 3) {
      // ---------------- MMA issuers: lane 0 of warp 1 (and of warp 3 when nis = 2) take batches
      // i, i + nis, ... into accumulator i. Per batch one wait on the slot and one on the
      // activations, BK x 4 MMAs, one commit each. A small-N MMA occupies the tensor core for about
      // 45 cycles, less than one thread takes to issue it next to the widening warps, hence two
      // issuers; the loop keeps to a few instructions per MMA: the activation descriptor is built
      // once, and a stage, a k-block and a 32-byte k step only add to its address field (16-byte
      // units; no carry out of the field below 256 KB).
      const int iss = warp == 1 ? 0 : 1;
      if (warp == 3) {
        pdl_wait();
        for (int m = lane; m < a.M; m += 32) sxa[m] = a.s_x[m] * a.alpha;
      }
      if (lane == 0) {
        const int nis = a.nis;
        const uint32_t idesc = idesc_i8_mn(kSwNT, Mt);
        const uint64_t desc0 = smem_desc_sw128(smem_u32(act));
        const uint32_t dlo0 = (uint32_t)desc0, dhi = (uint32_t)(desc0 >> 32);
        const uint32_t stage16 = (uint32_t)act_stage >> 4, kblock16 = (uint32_t)act_bytes >> 4;
        const uint32_t t_slots = tmem_base + (uint32_t)a.acc_cols;
        const uint32_t d_acc = tmem_base + (uint32_t)(iss * a.acc_stride);
        uint32_t acc0 = 0u;  // the first MMA of each issuer overwrites its accumulator
        bool any = false;
        uint32_t du_off[BK];  // address-field offsets of the k-blocks of a batch
#pragma unroll
        for (int u = 0; u < BK; ++u) du_off[u] = (uint32_t)u * kblock16;
        RingPos ps, pa;
        ps.advance(iss, NS);
        pa.advance(iss, NA);
        for (int b = iss; b < nbat; b += nis) {
          if (!mbar_wait(&slot_full[ps.s], ps.ph, &abort_flag)) { ok = false; break; }
          if (!mbar_wait(&act_full[pa.s], pa.ph, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const int nb = min(BK, nkb - b * BK);
          const uint32_t ta = t_slots + (uint32_t)(ps.s * BK * 32);
          const uint32_t dlo = dlo0 + (uint32_t)pa.s * stage16;
#pragma unroll
          for (int u = 0; u < BK; ++u) {
            if (u < nb) {
              const uint32_t du = dlo + du_off[u];
              mma_i8_ts(d_acc, ta + (uint32_t)(u * 32), ((uint64_t)dhi << 32) | du, idesc, u == 0 ? acc0 : 1u);
              mma_i8_ts(d_acc, ta + (uint32_t)(u * 32 + 8), ((uint64_t)dhi << 32) | (du + 2u), idesc, 1u);
              mma_i8_ts(d_acc, ta + (uint32_t)(u * 32 + 16), ((uint64_t)dhi << 32) | (du + 4u), idesc, 1u);
              mma_i8_ts(d_acc, ta + (uint32_t)(u * 32 + 24), ((uint64_t)dhi << 32) | (du + 6u), idesc, 1u);
            }
          }
          acc0 = 1u;
          any = true;
          mma_commit(&slot_empty[ps.s]);
          mma_commit(&act_empty[pa.s]);
          ps.advance(nis, NS);
          pa.advance(nis, NA);
        }
        if (ok && any) mma_commit(&acc_full);
        if (!ok && any) {
          mma_commit(&drain_bar[iss]);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&drain_bar[iss], 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    } else if (warp >= 4) {
      // ---------------- widen: thread = weight row (lane quarter q = warp % 4); the 128 codes of
      // a k-block (8 words, 16 codes each: k = 16c + 4s + b at bits 8b + 2s, c' = t + 1) become
      // 32 columns of 4 int8 bytes 64 t, column 4c + s holding k = 16c + 4s + 0..3. Warp group g
      // takes batches g, g + kSwW, ...
      const int q = warp & 3, g = (warp - 4) >> 2;
      const int row = q * 32 + lane;
      const uint32_t t_lane = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)a.acc_cols;
      RingPos pr, ps;
      pr.advance(g, NR);
      ps.advance(g, NS);
      for (int b = g; b < nbat; b += kSwW) {
        // every lane waits (the copy-written tile must be visible to each reader); the outcome is
        // made uniform so that the warp stays converged
        bool r = mbar_wait(&raw_full[pr.s], pr.ph, &abort_flag);
        if (r) r = mbar_wait(&slot_empty[ps.s], ps.ph ^ 1u, &abort_flag);
        if (!__all_sync(0xffffffffu, r)) { ok = false; break; }
        tc_fence_after();
        const int nb = min(BK, nkb - b * BK);
        const uint8_t* rp0 = raw + pr.s * raw_stage + row * 32;
        const uint32_t tcol = t_lane + (uint32_t)(ps.s * BK * 32);
#pragma unroll
        for (int u = 0; u < BK; ++u) {
          if (u < nb) {
            const uint4 lo = *reinterpret_cast<const uint4*>(rp0 + u * kSwRaw);
            const uint4 hi = *reinterpret_cast<const uint4*>(rp0 + u * kSwRaw + 16);
            const uint32_t wd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            uint32_t o[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
#pragma unroll
              for (int sp = 0; sp < 4; ++sp)  // plane sp of every byte to bits 6..7, then 64 t
                o[4 * c + sp] = (wd[c] * (1u << (6 - 2 * sp)) + 0xc0c0c0c0u) & 0xc0c0c0c0u;
            }
            tmem_st_32x32b_x32(tcol + (uint32_t)(u * 32), o);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_empty[pr.s]);  // this warp's reads of the 2-bit copy are done
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&slot_full[ps.s]);
        pr.advance(kSwW, NR);
        ps.advance(kSwW, NS);
      }
    }
  }

  // ---------------- epilogue part 1: partial sums -> own shared memory as [Mt][128] int32
  // (warps 4-7, one per TMEM lane quarter)
  int32_t* part = reinterpret_cast<int32_t*>(smem);  // the rings are idle once acc_full completes
  if (warp >= 4) {
    bool r = __all_sync(0xffffffffu, ok);
    r = r && mbar_wait(&acc_full, 0, &abort_flag);
    r = __all_sync(0xffffffffu, r);
    if (warp < 8) {
      const int q = warp & 3;
      const int f = q * 32 + lane;
      if (r && nkb > 0) {
        tc_fence_after();
        const int nacc = min(a.nis, nbat);  // accumulators that received MMAs
        for (int c0 = 0; c0 < Mt; c0 += 16) {
          int32_t sum[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) sum[j] = 0;
          for (int x = 0; x < nacc; ++x) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(x * a.acc_stride + c0), v);
#pragma unroll
            for (int j = 0; j < 16; ++j) sum[j] += (int32_t)v[j];
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) part[(c0 + j) * kSwNT + f] = sum[j] >> 6;  // the MMAs summed 64 t q
        }
      } else {
        for (int m = 0; m < Mt; ++m) part[m * kSwNT + f] = 0;
      }
    }
  }

  // the next kernel of the stream may launch now (it waits for this one before reading Y)
  pdl_launch_dependents();

  // ---------------- epilogue part 2: reduce the cluster's partial sums, dequant, store. Each
  // thread takes two elements at a time with all their remote loads in flight.
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp >= 4) {
    const uint32_t part0 = smem_u32(smem);
    const int t = threadIdx.x - 128;
    const int nt = 32 * kSwWidenWarps;
    const int E = Mt * kSwNT, step = S * nt;
    for (int e0 = (int)rank * nt + t; e0 < E; e0 += 2 * step) {
      uint32_t pv[2][8];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int e = e0 + j * step;
#pragma unroll
        for (int p = 0; p < 8; ++p)
          pv[j][p] = (p < S && e < E) ? ld_shared_cluster_u32(mapa_shared(part0 + (uint32_t)e * 4u, (uint32_t)p)) : 0u;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int e = e0 + j * step;
        const int m = e / kSwNT, f = e - m * kSwNT;
        const int n = n0 + f;
        if (e >= E || m >= a.M || n >= a.N) continue;
        int32_t acc = 0;
#pragma unroll
        for (int p = 0; p < 8; ++p) acc += (int32_t)pv[j][p];  // fixed order
        const float y = (float)acc * sxa[m];
        if (a.out_bf16) reinterpret_cast<__nv_bfloat16*>(a.Y)[(size_t)m * a.N + n] = __float2bfloat16_rn(y);
        else reinterpret_cast<float*>(a.Y)[(size_t)m * a.N + n] = y;
        if (a.acc_debug) a.acc_debug[(size_t)m * a.N + n] = acc;
      }
    }
  }
  __syncwarp();
  cluster_sync_all();  // no CTA leaves while a peer may still read its shared memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kSwTmemCols)
                 : "memory");
  }
}

}  // namespace hbl
