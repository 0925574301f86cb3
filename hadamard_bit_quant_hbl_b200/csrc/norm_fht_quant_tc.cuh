// Fused RMSNorm -> fast Walsh-Hadamard transform -> per-token quantisation for 16384-wide rows,
// with the first Kronecker factor of the transform on the tensor cores.
//
// Method: BitNet v2 walkthrough article (m.jxzklqfsx.com), section "H-BitLinear模塊": an online
// Hadamard transform of the normalised activations before per-token quantisation; the page
// defines the transform as a matrix product computed with the fast Hadamard transform.
//
// H_16384 = H_128 (x) H_128 in Sylvester order: with the index k split into the 7 bits
// a = (k bits 13..10, k bits 2..0) and the 7 bits n = k bits 9..3,
//   y[a, n] = sum_{a'} H_128[a][a'] * sum_{n'} H_128[n][n'] * x[a', n'],
// and the two factors commute. On CUDA cores the 14 butterfly stages cost 14 fp32 adds per
// element and bound the kernel by the FP32 pipe and issue, not by HBM; here the factor over a is
// one exact tensor-core product per row,
//   D[a][n] = sum_{a'} H_128[a][a'] * x[a', n]    (tcgen05.mma kind::f16, bf16 x bf16 -> fp32),
// exact up to fp32 rounding since x is bf16 and H is +-1, and the factor over n is 7 butterfly
// stages on CUDA cores. The MMA's B operand is the bf16 row itself, as the TMA copy lands it:
// 8 consecutive features (k bits 2..0) are one 16-byte row of an 8 x 16-byte core matrix whose
// 8 rows are 8 consecutive n (16 bytes apart), so the K-major no-swizzle layout reads the row with
// core matrices 128 bytes apart along N and 2048 bytes apart along K. TMEM lane a of the
// accumulator then holds, in its 128 columns, exactly the values one thread needs for the
// remaining stages: no widening pass and no regrouping through shared memory.
//
//   warps 0-3  consumers, thread = TMEM lane a: tcgen05.ld of the 128 columns, 7 butterfly
//              stages, row statistics, quantisation, codes through a [k mod 8][k / 8] byte matrix
//              and out in natural order (as the CUDA-core kernel)
//   warp 4     TMEM allocation; one thread copies rows in (one 32 KB bulk copy each) and issues
//              the 8 MMAs (K = 16 each) of a row into one of two TMEM accumulators
// Persistent CTAs (two per SM) walk the rows. (A 6-slot ring of quarter-row copies with separate
// copy and MMA threads measured slower: the consumers, 8 warps per SM at 168 registers, are the
// limit, not the copies.) Every mbarrier wait is bounded (1 s); the
// consumers vote on the outcome of their waits so that they leave their loop together.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"
#include "norm_fht_quant.cuh"

namespace hbl {

constexpr int kNtN = 16384;                       // transform size (the whole row)
constexpr int kNtRowBytes = kNtN * 2;             // one bf16 row
constexpr int kNtThreads = 160;                   // 4 consumer warps + 1 copy / MMA warp
constexpr int kNtTmemCols = 256;                  // two 128-column fp32 accumulators
constexpr int kNtCrow = kNtN / 8 + 16;            // byte stride of a (k mod 8) row of the code matrix
constexpr int kNtSmem = 32768 + kNtRowBytes + 8 * kNtCrow + 1024;  // H, row, codes, alignment slack

// Shared-memory matrix descriptor: K-major, no swizzle, 8 x 16-byte core matrices `lbo` bytes
// apart along K and `sbo` bytes apart along M/N.
__device__ __forceinline__ uint64_t smem_desc_none(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fffu);
  d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
  d |= (uint64_t)1u << 46;  // descriptor version (sm_100); layout type 0: no swizzle
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A and B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A: bf16
         | (1u << 10)                   // B: bf16
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Named barrier of the 128 consumer threads; the second form also returns, in every thread, the
// OR of `pred` over them (a uniform decision).
__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool consumer_bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// QM: 0 = a8 absmax, 1 = a4 absmean, 2 = a4 absmax
template <int QM>
__global__ void __launch_bounds__(kNtThreads, 2) norm_fht_quant_tc_kernel(const NfqArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_nt[];
  __shared__ __align__(8) uint64_t land_full, land_empty, acc_full[2], acc_empty[2], drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ float red_ss[4], red_st[4];

  constexpr int K = kNtN;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_nt) + 1023) & ~uintptr_t(1023));
  uint8_t* hA = smem;                 // H_128, two K halves of [128 rows][128 B], 128-byte swizzle
  uint8_t* land = smem + 32768;       // the bf16 row
  uint8_t* cbuf = land + kNtRowBytes; // codes [k mod 8][k / 8]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nrows = a.M > (int)blockIdx.x ? (a.M - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

  // X (and the codes buffer) may belong to the kernel before this one: wait for it
  pdl_wait();
  pdl_launch_dependents();

  // ---- H_128 in the A-operand layout: element (a, a') = (-1)^popcount(a & a') as bf16, a' in
  // two halves of 64; within a half, 16-byte chunk c of row a sits at chunk c ^ (a & 7)
  for (int e = tid; e < 128 * 64; e += kNtThreads) {  // two elements per 32-bit store
    const int r = e >> 6, k0 = (e & 63) * 2;
    const uint32_t v0 = (__popc(r & k0) & 1) ? 0xbf80u : 0x3f80u;
    const uint32_t v1 = (__popc(r & (k0 + 1)) & 1) ? 0xbf80u : 0x3f80u;
    const int half = k0 >> 6, kh = k0 & 63;
    *reinterpret_cast<uint32_t*>(hA + half * 16384 + r * 128 + (((kh >> 3) ^ (r & 7)) << 4) + (kh & 7) * 2) =
        v0 | (v1 << 16);
  }
  fence_proxy_async_shared();  // generic-proxy writes -> visible to the tensor core
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(&land_full, 1);
    mbar_init(&land_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 4);  // one lane of each consumer warp
    }
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 4) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&tmem_slot)), "r"(kNtTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 4) {
    // ---------------- row copies and MMAs (one thread)
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 128);
      int issued = 0;
      bool ok = true, any = false;
      if (nrows > 0) {
        mbar_arrive_expect_tx(&land_full, (uint32_t)kNtRowBytes);
        bulk_load_1d(land, a.X + (size_t)blockIdx.x * K, (uint32_t)kNtRowBytes, &land_full);
        issued = 1;
      }
      for (int i = 0; i < nrows; ++i) {
        const int as = i & 1;
        if (!mbar_wait(&land_full, (uint32_t)i & 1u, &abort_flag)) { ok = false; break; }
        if (!mbar_wait(&acc_empty[as], ((uint32_t)(i >> 1) & 1u) ^ 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(as * 128);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)  // a' = 16 ks .. 16 ks + 15: k bits 13..10 = 2ks, 2ks+1
          mma_bf16(d, smem_desc_sw128(smem_u32(hA + (ks >> 2) * 16384 + (ks & 3) * 32)),
                   smem_desc_none(smem_u32(land + ks * 4096), 2048u, 128u), idesc, ks > 0 ? 1u : 0u);
        any = true;
        mma_commit(&acc_full[as]);
        mma_commit(&land_empty);
        if (issued < nrows) {  // the next row, once the MMAs have read this one
          if (!mbar_wait(&land_empty, (uint32_t)i & 1u, &abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&land_full, (uint32_t)kNtRowBytes);
          bulk_load_1d(land, a.X + ((size_t)blockIdx.x + (size_t)issued * gridDim.x) * K, (uint32_t)kNtRowBytes,
                       &land_full);
          ++issued;
        }
      }
      if (!ok) {  // no copy or MMA may still be running when the CTA exits
        if (issued > 0) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&land_full, (uint32_t)(issued - 1) & 1u) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
        if (any) {
          mma_commit(&drain_bar);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else {
    // ---------------- consumers: thread = accumulator row a (k bits 13..10 = a >> 3, 2..0 = a & 7)
    const int arow = warp * 32 + lane;
    const int lo3 = arow & 7, hi4 = arow >> 3;
    constexpr float kQ = QM == 0 ? 127.f : (QM == 1 ? 2.6457513110645906f : 7.f);
    constexpr int kLo = QM == 0 ? -128 : -8, kHi = QM == 0 ? 127 : 7;
    constexpr bool kAbsmax = QM != 1;
    const bool packed4 = (a.fmt == 0) && (QM != 0);
    for (int i = 0; i < nrows; ++i) {
      const int as = i & 1;
      const int row = (int)blockIdx.x + i * (int)gridDim.x;
      const bool got = mbar_wait(&acc_full[as], (uint32_t)(i >> 1) & 1u, &abort_flag);
      if (consumer_bar_or(!got || abort_flag)) break;  // the same decision in every consumer
      tc_fence_after();

      // ---- the 128 columns of this lane: D[a][n], n = k bits 9..3
      float2 v[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(as * 128 + c * 32), r);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[c * 16 + j] = make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[as]);  // the accumulator may take the row after next

      // sum of squares: sum_a,n D^2 = 128 sum x^2 (H_128 has orthogonal rows of norm^2 128)
      float2 ss2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int j = 0; j < 64; ++j) ss2[j & 3] = __ffma2_rn(v[j], v[j], ss2[j & 3]);
      float ss = ((ss2[0].x + ss2[0].y) + (ss2[1].x + ss2[1].y)) + ((ss2[2].x + ss2[2].y) + (ss2[3].x + ss2[3].y));

      fwht_regs2<128, 7>(v);  // the factor over n

      float st;
      if constexpr (kAbsmax) {
        float sta[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 64; ++j) sta[j & 3] = fmaxf(sta[j & 3], fmaxf(fabsf(v[j].x), fabsf(v[j].y)));
        st = fmaxf(fmaxf(sta[0], sta[1]), fmaxf(sta[2], sta[3]));
      } else {
        float2 sta2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          const float2 t = make_float2(fabsf(v[j].x) + fabsf(v[j].y), fabsf(v[j + 1].x) + fabsf(v[j + 1].y));
          sta2[(j / 2) & 3] = __fadd2_rn(sta2[(j / 2) & 3], t);
        }
        st = ((sta2[0].x + sta2[0].y) + (sta2[1].x + sta2[1].y)) + ((sta2[2].x + sta2[2].y) + (sta2[3].x + sta2[3].y));
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float t = __shfl_xor_sync(0xffffffffu, st, o);
        st = kAbsmax ? fmaxf(st, t) : st + t;
      }
      if (lane == 0) {
        red_ss[warp] = ss;
        red_st[warp] = st;
      }
      consumer_bar();
      ss = (red_ss[0] + red_ss[1]) + (red_ss[2] + red_ss[3]);  // fixed order, the same in every thread
      st = kAbsmax ? fmaxf(fmaxf(red_st[0], red_st[1]), fmaxf(red_st[2], red_st[3]))
                   : (red_st[0] + red_st[1]) + (red_st[2] + red_st[3]);

      // ---- per-row multiplier and scale (y = the unnormalised transform of x)
      const float r_rms = sqrtf(ss / (128.f * (float)K) + a.eps_norm);
      const float rs = r_rms * sqrtf((float)K);
      const float sy = kAbsmax ? st : st / (float)K;
      float mult, sx;
      if (a.eps_q == 0.f) {
        mult = sy > 0.f ? kQ / sy : 0.f;
        sx = sy > 0.f ? sy / (rs * kQ) : 0.f;
      } else {
        const float stat = sy / rs;
        mult = kQ / ((stat + a.eps_q) * rs);
        sx = stat / kQ;
      }
      if (arow == 0) a.s_x[row] = sx;

      // ---- codes of k = hi4 * 1024 + 8 n + lo3 for n = 0..127: row lo3, columns hi4*128 + n of
      // the [k mod 8][k / 8] byte matrix; fp32 product, clamp (absmean), round by the 1.5 * 2^23 add
      const float2 mult2 = make_float2(mult, mult);
      const float2 magic2 = make_float2(12582912.f, 12582912.f);
      uint8_t* dst = cbuf + lo3 * kNtCrow + hi4 * 128;
#pragma unroll
      for (int j = 0; j < 128; j += 16) {
        uint32_t wds[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r0 = j + 4 * q;
          float2 t0 = __fmul2_rn(v[r0 / 2], mult2);
          float2 t1 = __fmul2_rn(v[r0 / 2 + 1], mult2);
          if constexpr (!kAbsmax) {
            t0.x = fminf(fmaxf(t0.x, (float)kLo), (float)kHi);
            t0.y = fminf(fmaxf(t0.y, (float)kLo), (float)kHi);
            t1.x = fminf(fmaxf(t1.x, (float)kLo), (float)kHi);
            t1.y = fminf(fmaxf(t1.y, (float)kLo), (float)kHi);
          }
          const float2 p0 = __fadd2_rn(t0, magic2);
          const float2 p1 = __fadd2_rn(t1, magic2);
          const uint32_t h0 = __byte_perm(__float_as_uint(p0.x), __float_as_uint(p0.y), 0x5410);
          const uint32_t h1 = __byte_perm(__float_as_uint(p1.x), __float_as_uint(p1.y), 0x5410);
          wds[q] = __byte_perm(h0, h1, 0x6420);
        }
        *reinterpret_cast<uint4*>(dst + j) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
      }
      consumer_bar();

      // ---- stream the codes out in natural order, 32 consecutive codes per unit
#pragma unroll
      for (int it = 0; it < (K / 32) / 128; ++it) {
        const int vcol = arow + it * 128;
        const uint8_t* srcc = cbuf + 4 * vcol;
        uint32_t w[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) w[b] = *reinterpret_cast<const uint32_t*>(srcc + b * kNtCrow);
        // byte j of w[b] is the code of k = 32 * vcol + 8 * j + b
        if (!packed4) {
          uint32_t o[8];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t a01l = __byte_perm(w[4 * h], w[4 * h + 1], 0x5140);
            const uint32_t a01h = __byte_perm(w[4 * h], w[4 * h + 1], 0x7362);
            const uint32_t a23l = __byte_perm(w[4 * h + 2], w[4 * h + 3], 0x5140);
            const uint32_t a23h = __byte_perm(w[4 * h + 2], w[4 * h + 3], 0x7362);
            o[0 + h] = __byte_perm(a01l, a23l, 0x5410);
            o[2 + h] = __byte_perm(a01l, a23l, 0x7632);
            o[4 + h] = __byte_perm(a01h, a23h, 0x5410);
            o[6 + h] = __byte_perm(a01h, a23h, 0x7632);
          }
          uint4* dstg = reinterpret_cast<uint4*>(a.codes + (size_t)row * K + 32 * vcol);
          dstg[0] = make_uint4(o[0], o[1], o[2], o[3]);
          dstg[1] = make_uint4(o[4], o[5], o[6], o[7]);
        } else {
          uint32_t m[4];
#pragma unroll
          for (int i2 = 0; i2 < 4; ++i2) m[i2] = (w[2 * i2] & 0x0f0f0f0fu) | ((w[2 * i2 + 1] & 0x0f0f0f0fu) << 4);
          const uint32_t a01l = __byte_perm(m[0], m[1], 0x5140);
          const uint32_t a01h = __byte_perm(m[0], m[1], 0x7362);
          const uint32_t a23l = __byte_perm(m[2], m[3], 0x5140);
          const uint32_t a23h = __byte_perm(m[2], m[3], 0x7362);
          const uint4 o = make_uint4(__byte_perm(a01l, a23l, 0x5410), __byte_perm(a01l, a23l, 0x7632),
                                     __byte_perm(a01h, a23h, 0x5410), __byte_perm(a01h, a23h, 0x7632));
          *reinterpret_cast<uint4*>(a.codes + (size_t)row * (K / 2) + 16 * vcol) = o;
        }
      }
      // the next row's statistics barrier orders these reads before the matrix is rewritten
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kNtTmemCols)
                 : "memory");
  }
}

}  // namespace hbl
