// Fused RMSNorm -> fast Walsh-Hadamard transform -> per-token quantisation with the first
// Kronecker factor of the transform on the tensor cores, for groups of 2 or 4 rows (blocks of
// 8192 or 4096 features), eight consumer warps per group.
//
// Method: BitNet v2 walkthrough article (m.jxzklqfsx.com), section "H-BitLinear模塊": an online
// Hadamard transform of the normalised activations before per-token quantisation.
//
// The product with H_128 over the index bits 9..3 is the one of norm_fht_quant_tc.cuh (a group of
// R rows, R K = 16384, one 128 x 128 x 128 bf16 product per group into 128 TMEM columns c = (row,
// k bits >= 10, k bits 2..0)). What differs is who finishes it: the 128 columns of a group are
// split into two halves of 64 -- the first R/2 rows and the last R/2 rows, so no butterfly stage
// crosses them -- each taken by four warps (one per TMEM lane quarter). A thread holds 64 values
// instead of 128, and one CTA per SM runs two such sets of eight warps on alternate groups: four
// consumer warps per scheduler instead of two for the latency-bound consumers (Wo 8192 x 4096 and
// 3B Wdown 4096 x 8192 alone: 25.8 and 26.0 us against 28.2 and 28.0 us). Rows of 16384 features
// stay on the 4-warp kernel: there k bit 13 splits the halves and is a stage of the transform, and
// the exchange of the halves through tensor memory made that form slower (131 against 93 us).
// Per-row statistics are reduced over the four warps of the row's half through shared memory, one
// barrier of the set per group.
//
//   warps 0-7, 8-15  consumer sets 0 and 1: set s takes the CTA's groups s, s + 2, ...
//   warp 16          TMEM allocation (4 accumulators x 128 columns); one thread copies row groups
//                    into 4 buffers (one bulk copy each) and issues the 8 MMAs of each group
// Every mbarrier wait is bounded (1 s); the consumers of a set vote on the outcome of their waits
// so that they leave their loop together.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"
#include "norm_fht_quant.cuh"
#include "norm_fht_quant_tc.cuh"

namespace hbl {

constexpr int kN2Sets = 2;
constexpr int kN2SetWarps = 8;
constexpr int kN2ProdWarp = kN2Sets * kN2SetWarps;  // 16
constexpr int kN2Threads = 32 * (kN2ProdWarp + 1);  // 544
constexpr int kN2Land = 4;                          // row-group buffers
constexpr int kN2Acc = 4;                           // 128-column accumulators (all 512 columns)
constexpr int kN2Smem = 32768 + kN2Land * kNtRowBytes + 1024;  // H, buffers, alignment slack
// 17 warps put 5 on one scheduler, whose quarter of the register file holds 16384 registers
constexpr int kN2MaxRegs = 96;
static_assert(5 * 32 * kN2MaxRegs <= 16384, "registers of the warps on one scheduler");
static_assert(kN2Smem <= 227 * 1024, "shared memory");

// Named barrier of one consumer set (its 256 threads; id 1 + set); the second form also returns,
// in every thread, the OR of `pred` over the set (a uniform decision).
__device__ __forceinline__ void set_bar(uint32_t id) {
  asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory");
}
__device__ __forceinline__ bool set_bar_or(uint32_t id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %2, 0;\n\t"
      "barrier.red.or.pred q, %1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(id), "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// QM: 0 = a8 absmax, 1 = a4 absmean, 2 = a4 absmax. R: rows per group (R K = 16384). LB: log2 of
// the transform block, which is the whole row (K = 2^LB).
template <int QM, int R, int LB>
__global__ void __maxnreg__(kN2MaxRegs) norm_fht_quant_tc2_kernel(const NfqArgs a) {
  static_assert((R == 2 && LB == 13) || (R == 4 && LB == 12), "groups of 2 or 4 whole-row transforms");
  constexpr int HB = 1 << LB;
  constexpr int P = 128;                        // the tensor-core factor H_128 over k bits 9..3
  constexpr int NSTH = 3 + (LB - 10);           // the other stages: k bits 2..0 and 10..LB-1
  constexpr int RH = R / 2;                     // rows per half
  constexpr int CPR = 64 / RH;                  // columns of a row in a half
  constexpr int RUNS = CPR / 8;                 // runs of 8 consecutive features per row and thread
  const int K = a.K;
  extern __shared__ __align__(1024) uint8_t smem_n2[];
  __shared__ __align__(8) uint64_t land_full[kN2Land], land_empty[kN2Land], acc_full[kN2Acc], acc_empty[kN2Acc];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ float red_ss[kN2Sets][2][R][kN2SetWarps], red_st[kN2Sets][2][R][kN2SetWarps];

  uint8_t* smem = align_shared<1024>(smem_n2);
  uint8_t* hA = smem;            // H_128, two K halves of [128 rows][128 B], 128-byte swizzle
  uint8_t* land = smem + 32768;  // kN2Land buffers of 16384 bf16

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ngroups = (a.M + R - 1) / R;
  const int ng = ngroups > (int)blockIdx.x ? (ngroups - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

  // X (and the codes buffer) may belong to the kernel before this one: wait for it
  pdl_wait();
  pdl_launch_dependents();

  // the rows of the CTA's i-th group that exist, as one contiguous copy into buffer b
  auto copy_group = [&](int i, int b) {
    const int g = (int)blockIdx.x + i * (int)gridDim.x;
    const int rows = a.M - g * R < R ? a.M - g * R : R;
    const uint32_t bytes = (uint32_t)rows * (uint32_t)K * 2u;
    mbar_arrive_expect_tx(&land_full[b], bytes);
    bulk_load_1d(land + b * kNtRowBytes, a.X + (size_t)g * R * K, bytes, &land_full[b]);
  };
  const int first = ng < kN2Land ? ng : kN2Land;
  if (warp == kN2ProdWarp && lane == 0) {
    abort_flag = 0;
    for (int s = 0; s < kN2Land; ++s) {
      mbar_init(&land_full[s], 1);
      mbar_init(&land_empty[s], 1);
    }
    for (int s = 0; s < kN2Acc; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], kN2SetWarps);  // one lane of each warp of the set
    }
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int i = 0; i < first; ++i) copy_group(i, i);  // land while H is built
  }

  // ---- H_128 in the A-operand layout (as in norm_fht_quant_tc.cuh)
  auto hval = [](int r, int k) -> uint32_t { return (__popc(r & k) & 1) ? 0xbf80u : 0x3f80u; };
  for (int e = tid; e < 128 * 64; e += kN2Threads) {
    const int r = e >> 6, k0 = (e & 63) * 2;
    const uint32_t v0 = hval(r, k0);
    const uint32_t v1 = hval(r, k0 + 1);
    const int hh = k0 >> 6, kh = k0 & 63;
    *reinterpret_cast<uint32_t*>(hA + hh * 16384 + r * 128 + (((kh >> 3) ^ (r & 7)) << 4) + (kh & 7) * 2) =
        v0 | (v1 << 16);
  }
  fence_proxy_async_shared();
  if (warp == kN2ProdWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;"
                 ::"r"(smem_u32(&tmem_slot)) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == kN2ProdWarp) {
    // ---------------- group copies and MMAs (one thread)
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 128);
      int issued = first;
      bool ok = true;
      int done = 0;  // groups whose MMAs were issued
      RingPos pl, pc;
      for (int i = 0; i < ng; ++i) {
        if (!mbar_wait(&land_full[pl.s], pl.ph, &abort_flag)) { ok = false; break; }
        if (!mbar_wait(&acc_empty[pc.s], pc.ph ^ 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(pc.s * 128);
        const uint32_t lb = smem_u32(land + pl.s * kNtRowBytes);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)  // a' = 16 ks .. 16 ks + 15
          mma_bf16(d, smem_desc_sw128(smem_u32(hA + (ks >> 2) * 16384 + (ks & 3) * 32)),
                   smem_desc_none(lb + (uint32_t)(ks * 256), 128u, 2048u), idesc, ks > 0 ? 1u : 0u);
        done = i + 1;
        mma_commit(&acc_full[pc.s]);
        mma_commit(&land_empty[pl.s]);
        // the previous group's buffer, once its MMAs have read it, takes the group kN2Land after it
        if (i >= 1 && issued < ng) {
          const int pb = pl.s == 0 ? kN2Land - 1 : pl.s - 1;
          const uint32_t pph = (uint32_t)((i - 1) / kN2Land) & 1u;
          if (!mbar_wait(&land_empty[pb], pph, &abort_flag)) { ok = false; break; }
          copy_group(issued, pb);
          ++issued;
        }
        pl.advance(1, kN2Land);
        pc.advance(1, kN2Acc);
      }
      if (!ok) {  // no copy or MMA may still be running when the CTA exits
        const uint64_t t0 = globaltimer_ns();
        for (int c = done; c < issued; ++c)
          while (!mbar_try_wait(&land_full[c % kN2Land], (uint32_t)(c / kN2Land) & 1u) &&
                 globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        if (done > 0) {
          mma_commit(&drain_bar);
          while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else {
    // ---------------- consumers: set s, half h of the columns, TMEM lane quarter q; thread =
    // accumulator lane a = k bits 9..3
    const int set = warp >> 3, w8 = warp & 7, half = w8 >> 2, q = w8 & 3;
    const uint32_t bar_id = 1u + (uint32_t)set;
    const int arow = q * 32 + lane;
    constexpr float kQ = QM == 0 ? 127.f : (QM == 1 ? 2.6457513110645906f : 7.f);
    constexpr bool kAbsmax = QM != 1;
    const bool packed4 = (a.fmt == 0) && (QM != 0);
    for (int i = set; i < ng; i += kN2Sets) {
      const int slot = i % kN2Acc;
      const int par2 = (i / kN2Sets) & 1;  // statistics buffer
      const int g = (int)blockIdx.x + i * (int)gridDim.x;
      const bool got = mbar_wait(&acc_full[slot], (uint32_t)(i / kN2Acc) & 1u, &abort_flag);
      if (set_bar_or(bar_id, !got || abort_flag)) break;  // the same decision in every warp of the set
      tc_fence_after();

      // ---- this thread's 64 columns: column 64 half + c' of the group, c' = 2 j + (0, 1) in v[j]
      const uint32_t tq = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(slot * 128);
      float2 v[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tq + (uint32_t)(half * 64 + c * 32), r);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[c * 16 + j] = make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[slot]);  // the accumulator may take the group after next

      // sums of squares per row of the half (sum over a row's D^2 = 128 sum x^2)
      float ss[RH], st[RH];
      {
        float2 acc[RH][2];
#pragma unroll
        for (int rr = 0; rr < RH; ++rr) acc[rr][0] = acc[rr][1] = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int rr = (2 * j) / CPR;
          acc[rr][j & 1] = __ffma2_rn(v[j], v[j], acc[rr][j & 1]);
        }
#pragma unroll
        for (int rr = 0; rr < RH; ++rr) ss[rr] = (acc[rr][0].x + acc[rr][0].y) + (acc[rr][1].x + acc[rr][1].y);
      }

      fwht_regs2<64, NSTH>(v);  // the remaining stages, all inside the row

      // ---- the row statistic of y (the unnormalised transform) per row of the half
#pragma unroll
      for (int rr = 0; rr < RH; ++rr) st[rr] = 0.f;
      if constexpr (kAbsmax) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int rr = (2 * j) / CPR;
          st[rr] = fmaxf(st[rr], fmaxf(fabsf(v[j].x), fabsf(v[j].y)));
        }
      } else {
        float2 acc[RH];
#pragma unroll
        for (int rr = 0; rr < RH; ++rr) acc[rr] = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const int rr = (2 * j) / CPR;
          acc[rr] = __fadd2_rn(acc[rr], make_float2(fabsf(v[j].x) + fabsf(v[j].y), fabsf(v[j + 1].x) + fabsf(v[j + 1].y)));
        }
#pragma unroll
        for (int rr = 0; rr < RH; ++rr) st[rr] = acc[rr].x + acc[rr].y;
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
        for (int rr = 0; rr < RH; ++rr) {
          ss[rr] += __shfl_xor_sync(0xffffffffu, ss[rr], o);
          const float t = __shfl_xor_sync(0xffffffffu, st[rr], o);
          st[rr] = kAbsmax ? fmaxf(st[rr], t) : st[rr] + t;
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int rr = 0; rr < RH; ++rr) {
          const int row = half * RH + rr;
          red_ss[set][par2][row][w8] = ss[rr];
          red_st[set][par2][row][w8] = st[rr];
        }
      }
      set_bar(bar_id);

      // ---- per-row multiplier and scale: lane rr of each warp computes them for row rr of its
      // half from the same sums in the same order as every other warp of the row
      float mult_l = 0.f, sx_l = 0.f;
      int lanes16_l = 0;
      {
        const int rr = lane < RH ? lane : 0;
        const int row = half * RH + rr;
        const int w0 = half * 4;
        constexpr int NW = 4;
        const float* rs_ = red_ss[set][par2][row];
        const float* rt_ = red_st[set][par2][row];
        float ssr = 0.f, str = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          ssr += rs_[w0 + w];
          str = kAbsmax ? fmaxf(str, rt_[w0 + w]) : str + rt_[w0 + w];
        }
        const float r_rms = sqrtf(ssr / ((float)P * (float)K) + a.eps_norm);
        const float rs = r_rms * sqrtf((float)HB);
        const float sy = kAbsmax ? str : str / (float)K;
        if (a.eps_q == 0.f) {
          mult_l = sy > 0.f ? kQ / sy : 0.f;
          sx_l = sy > 0.f ? sy / (rs * kQ) : 0.f;
        } else {
          const float stat = sy / rs;
          mult_l = kQ / ((stat + a.eps_q) * rs);
          sx_l = stat / kQ;
        }
        // int16-lane clamp allowed when every rounded product fits an int16 (see codes4)
        lanes16_l = mult_l * sqrtf((float)(HB / P) * ssr) < 30000.f ? 1 : 0;
        if (q == 0 && lane < RH && g * R + row < a.M) a.s_x[g * R + row] = sx_l;
      }

#pragma unroll
      for (int rr = 0; rr < RH; ++rr) {
        const int row = g * R + half * RH + rr;
        if (row >= a.M) break;  // the same in every lane
        const float mult = __shfl_sync(0xffffffffu, mult_l, rr);
        const int lanes16 = __shfl_sync(0xffffffffu, lanes16_l, rr);
        const float2 mult2 = make_float2(mult, mult);
        const float2* vr = v + rr * (CPR / 2);
        uint8_t* row_codes = a.codes + (size_t)row * (packed4 ? K / 2 : K);
        if constexpr (kAbsmax) {
          quant_store<0, RUNS>(vr, mult2, row_codes, packed4, arow, K);
        } else if (lanes16) {
          quant_store<1, RUNS>(vr, mult2, row_codes, packed4, arow, K);
        } else {
          quant_store<2, RUNS>(vr, mult2, row_codes, packed4, arow, K);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kN2ProdWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem_base) : "memory");
  }
}

}  // namespace hbl
