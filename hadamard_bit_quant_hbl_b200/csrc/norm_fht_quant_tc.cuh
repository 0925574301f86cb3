// Fused RMSNorm -> fast Walsh-Hadamard transform -> per-token quantisation with the first
// Kronecker factor of the transform on the tensor cores.
//
// Method: BitNet v2 walkthrough article (m.jxzklqfsx.com), section "H-BitLinear模塊": an online
// Hadamard transform of the normalised activations before per-token quantisation; the page
// defines the transform as a matrix product computed with the fast Hadamard transform.
//
// A group of R rows (R K <= 16384) lands in one 16384-element bf16 buffer; element index
// e = 1024 nh + 8 a + nl splits into a = e bits 9..3 (7 bits) and the column c = (nh, nl). The
// Sylvester matrix H[k][k'] = (-1)^popcount(k & k') factors over any split of the index bits, so
// the transform of each block of HB = 2^LB features is
//   D[a][c] = sum_{a'} A[a][a'] * buf[a', c]    (tcgen05.mma kind::f16, bf16 x bf16 -> fp32),
// with A = I (x) H_P (P = min(HB / 8, 128): the index bits 9..3 that lie inside a block; the
// others are block-index bits and get the identity), followed by butterfly stages on CUDA cores
// over the remaining in-block bits: nl (k bits 2..0) and, for blocks of 2048 .. 16384, k bits
// 10 .. LB - 1. The product is exact up to fp32 rounding since buf is bf16 and A is 0/+-1. For one
// block of 4096 .. 16384 features this is H_128 on the tensor cores; for K = 43 x 256 (blocks of
// 256, one row per group) it is I_4 (x) H_32 and three stages. Columns past the end of a row hold
// zeros (the buffer's tail is cleared once per CTA) and are neither counted nor stored.
// On CUDA cores alone the 14 butterfly stages of a 16384-point transform cost 14 fp32 adds per
// element and bound the kernel by the FP32 pipe and issue, not by HBM.
//
// The MMA's B operand is the bf16 buffer itself, as the bulk copy lands it, read MN-major: the 128
// contiguous bytes of features 64j .. 64j + 63 are one 8 x 16-byte core matrix whose 16-byte rows
// hold 8 consecutive nl and step through a' (e bits 5..3); core matrices lie 128 bytes apart along
// N (e bits 9..6) and 2048 bytes apart along K (e bit 10). TMEM lane a of the accumulator then
// holds, in its 128 columns, exactly the values one thread needs for the remaining stages, and
// after them runs of 8 consecutive outputs: the thread forms its codes and stores them to global
// memory directly, with no regrouping through shared memory.
//
//   warps 0-3  consumers, thread = TMEM lane a: tcgen05.ld of the 128 columns, the remaining
//              butterfly stages, row statistics (one named barrier), quantisation, stores of 8 codes
//   warp 4     TMEM allocation; one thread copies groups in (one bulk copy each) and issues the 8
//              MMAs (K = 16 each) of a group into one of two TMEM accumulators
// Persistent CTAs (two per SM) walk the groups. (With the consumers' arithmetic taken out the
// copies and MMAs alone run at 5.2 TB/s: the consumers are the limit.) Every mbarrier wait is
// bounded (1 s); the consumers vote on the outcome of their waits so that they leave their loop
// together.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"
#include "norm_fht_quant.cuh"

namespace hbl {

constexpr int kNtN = 16384;                       // transform size (the whole row)
constexpr int kNtRowBytes = kNtN * 2;             // one bf16 row
constexpr int kNtThreads = 160;                   // 4 consumer warps + 1 copy / MMA warp
constexpr int kNtTmemCols = 256;                  // two 128-column fp32 accumulators
constexpr int kNtSmem = 32768 + kNtRowBytes + 1024;  // H, rows, alignment slack
// CTAs resident on one SM. The copy and the MMAs of one CTA overlap the butterflies of the other,
// so the launch sizes its grid to this many per SM. The register file is split into four
// 16384-entry quarters, one per warp scheduler, and two 5-warp CTAs put three warps on one quarter:
// that fits at kNtMaxRegs registers a thread, the count the compiler keeps to under the kernel's
// launch bounds. (The runtime's occupancy query answers 1 for this kernel, so the launch does not
// use it.)
constexpr int kNtCtasPerSm = 2;
constexpr int kNtMaxRegs = 168;
static_assert(kNtCtasPerSm * (kNtSmem + 1024) <= 228 * 1024, "shared memory of the resident CTAs");
static_assert(kNtCtasPerSm * kNtTmemCols <= 512, "TMEM columns of the resident CTAs");
static_assert((kNtCtasPerSm * kNtThreads / 32 + 3) / 4 * 32 * kNtMaxRegs <= 16384,
              "registers of the warps the resident CTAs put on one scheduler");

// Shared-memory matrix descriptor, no swizzle: 8 x 16-byte core matrices (128 contiguous bytes)
// `lbo` bytes apart along K and `sbo` bytes apart along M/N. (Whether the 16-byte rows of a core
// matrix run along K or along M/N is the operand's major-ness in the instruction descriptor.)
__device__ __forceinline__ uint64_t smem_desc_none(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fffu);
  d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
  d |= (uint64_t)1u << 46;  // descriptor version (sm_100); layout type 0: no swizzle
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A and B, fp32 D; A K-major, B MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A: bf16
         | (1u << 10)                   // B: bf16
         | (1u << 16)                   // B: MN-major (A stays K-major)
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

__device__ __forceinline__ uint32_t max_s16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t min_s16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Four codes (features k .. k + 3 in va, vb) as the bytes of one word. fma(y, mult, 1.5 * 2^23)
// rounds the exact product to the nearest integer, ties to even, into the low mantissa bits
// (|y mult| < 2^22). CM 0: no clamp (absmax: the products already lie in [-Q, Q]); CM 1: clamp
// to [-8, 7] on the 16-bit lanes that hold the integers, exact while each fits an int16; CM 2:
// clamp the integer-valued sums themselves, exact always.
template <int CM>
__device__ __forceinline__ uint32_t codes4(float2 va, float2 vb, float2 mult2) {
  const float2 magic2 = make_float2(12582912.f, 12582912.f);
  float2 p0 = __ffma2_rn(va, mult2, magic2);
  float2 p1 = __ffma2_rn(vb, mult2, magic2);
  if constexpr (CM == 2) {
    constexpr float lo = 12582912.f - 8.f, hi = 12582912.f + 7.f;
    p0.x = fminf(fmaxf(p0.x, lo), hi);
    p0.y = fminf(fmaxf(p0.y, lo), hi);
    p1.x = fminf(fmaxf(p1.x, lo), hi);
    p1.y = fminf(fmaxf(p1.y, lo), hi);
  }
  uint32_t h0 = __byte_perm(__float_as_uint(p0.x), __float_as_uint(p0.y), 0x5410);  // int16 lanes k, k+1
  uint32_t h1 = __byte_perm(__float_as_uint(p1.x), __float_as_uint(p1.y), 0x5410);
  if constexpr (CM == 1) {
    h0 = min_s16x2(max_s16x2(h0, 0xfff8fff8u), 0x00070007u);
    h1 = min_s16x2(max_s16x2(h1, 0xfff8fff8u), 0x00070007u);
  }
  return __byte_perm(h0, h1, 0x6420);
}

// The codes of one row's runs in one thread: v[4u .. 4u + 3] are the 8 consecutive features
// 8a + 1024u + 0..7 of the row (a = the thread's accumulator lane). Each run is one store, and the
// 32 lanes of a warp (consecutive a) cover 256 (int8) or 128 (packed int4, low nibble = even
// feature) contiguous bytes.
template <int CM, int RUNS>
__device__ __forceinline__ void quant_store(const float2* v, float2 mult2, uint8_t* row_codes, bool packed4,
                                            int a, int K) {
#pragma unroll
  for (int u = 0; u < RUNS; ++u) {
    if (1024 * u >= K) break;            // past the row: the same in every lane
    if (1024 * u + 8 * a >= K) continue;  // the row ends inside this 1024-feature chunk
    const uint32_t w0 = codes4<CM>(v[4 * u], v[4 * u + 1], mult2);
    const uint32_t w1 = codes4<CM>(v[4 * u + 2], v[4 * u + 3], mult2);
    if (!packed4) {
      *reinterpret_cast<uint2*>(row_codes + 8 * a + 1024 * u) = make_uint2(w0, w1);
    } else {
      // byte 0 of z = code k | code k+1 << 4, byte 2 = code k+2 | code k+3 << 4 (bytes 1, 3 unused)
      const uint32_t z0 = (w0 & 0x000f000fu) | ((w0 >> 4) & 0x00f000f0u);
      const uint32_t z1 = (w1 & 0x000f000fu) | ((w1 >> 4) & 0x00f000f0u);
      *reinterpret_cast<uint32_t*>(row_codes + 4 * a + 512 * u) = __byte_perm(z0, z1, 0x6420);
    }
  }
}

// QM: 0 = a8 absmax, 1 = a4 absmean, 2 = a4 absmax. R: rows per group (R K <= 16384; a row
// shorter than 16384 features that is not a power of two is a group of its own, the rest of the
// buffer zero). LB: log2 of the transform block (K = nb 2^LB).
template <int QM, int R, int LB>
__global__ void __launch_bounds__(kNtThreads, kNtCtasPerSm) norm_fht_quant_tc_kernel(const NfqArgs a) {
  static_assert(R == 1 || R == 2 || R == 4 || R == 8, "rows per group");
  static_assert(LB >= 8 && LB <= 14, "transform block");
  constexpr int HB = 1 << LB;
  constexpr int LP = LB - 3 < 7 ? LB - 3 : 7;  // the tensor-core factor I (x) H_P over k bits 9..3
  constexpr int P = 1 << LP;
  constexpr int NST = 3 + (LB > 10 ? LB - 10 : 0);  // butterfly stages left: k bits 2..0, 10..LB-1
  constexpr int NB = 128 / R;   // accumulator columns per row
  constexpr int RUNS = NB / 8;  // runs of 8 consecutive features per row and thread
  const int K = a.K;
  extern __shared__ __align__(1024) uint8_t smem_nt[];
  __shared__ __align__(8) uint64_t land_full, land_empty, acc_full[2], acc_empty[2], drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ float red_ss[2][R][4], red_st[2][R][4];  // by group parity: one barrier per group suffices

  uint8_t* smem = align_shared<1024>(smem_nt);
  uint8_t* hA = smem;                 // H_128, two K halves of [128 rows][128 B], 128-byte swizzle
  uint8_t* land = smem + 32768;       // the group's R bf16 rows, 16384 elements

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ngroups = (a.M + R - 1) / R;
  const int ng = ngroups > (int)blockIdx.x ? (ngroups - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

  // X (and the codes buffer) may belong to the kernel before this one: wait for it
  pdl_wait();
  pdl_launch_dependents();

  // the rows of group g that exist, as one contiguous copy (a ragged last group copies fewer; the
  // columns of the missing rows then hold stale values that nothing stores)
  auto copy_group = [&](int g) {
    const int rows = a.M - g * R < R ? a.M - g * R : R;
    const uint32_t bytes = (uint32_t)rows * (uint32_t)K * 2u;
    mbar_arrive_expect_tx(&land_full, bytes);
    bulk_load_1d(land, a.X + (size_t)g * R * K, bytes, &land_full);
  };
  // barriers first, then the first group's copy, which lands while every thread builds H
  if (warp == 4 && lane == 0) {
    abort_flag = 0;
    mbar_init(&land_full, 1);
    mbar_init(&land_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 4);  // one lane of each consumer warp
    }
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (ng > 0) copy_group((int)blockIdx.x);
  }

  // ---- I (x) H_P in the A-operand layout: element (a, a') = (-1)^popcount(a & a') as bf16 where
  // a and a' lie in the same block of P, else 0; a' in two halves of 64; within a half, 16-byte
  // chunk c of row a sits at chunk c ^ (a & 7)
  auto hval = [](int r, int k) -> uint32_t {
    if ((r >> LP) != (k >> LP)) return 0u;
    return (__popc(r & k & (P - 1)) & 1) ? 0xbf80u : 0x3f80u;  // the block bits carry no sign
  };
  for (int e = tid; e < 128 * 64; e += kNtThreads) {  // two elements per 32-bit store
    const int r = e >> 6, k0 = (e & 63) * 2;
    const uint32_t v0 = hval(r, k0);
    const uint32_t v1 = hval(r, k0 + 1);
    const int half = k0 >> 6, kh = k0 & 63;
    *reinterpret_cast<uint32_t*>(hA + half * 16384 + r * 128 + (((kh >> 3) ^ (r & 7)) << 4) + (kh & 7) * 2) =
        v0 | (v1 << 16);
  }
  // a row shorter than the buffer: the tail stays zero (copies write only the first K features),
  // so the columns past the row hold exact zeros -- a stale NaN there would reach the valid
  // outputs of its column through the zeros of I (x) H_P
  if (R * K < kNtN)
    for (int e = R * K * 2 + tid * 16; e < kNtRowBytes; e += kNtThreads * 16)
      *reinterpret_cast<uint4*>(land + e) = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_shared();  // generic-proxy writes -> visible to the tensor core
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
    // ---------------- group copies and MMAs (one thread)
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 128);
      int issued = ng > 0 ? 1 : 0;  // the first group's copy is in flight
      bool ok = true, any = false;
      for (int i = 0; i < ng; ++i) {
        const int as = i & 1;
        if (!mbar_wait(&land_full, (uint32_t)i & 1u, &abort_flag)) { ok = false; break; }
        if (!mbar_wait(&acc_empty[as], ((uint32_t)(i >> 1) & 1u) ^ 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(as * 128);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)  // a' = 16 ks .. 16 ks + 15, a' bits 6..4 = ks = k bits 9..7
          mma_bf16(d, smem_desc_sw128(smem_u32(hA + (ks >> 2) * 16384 + (ks & 3) * 32)),
                   smem_desc_none(smem_u32(land + ks * 256), 128u, 2048u), idesc, ks > 0 ? 1u : 0u);
        any = true;
        mma_commit(&acc_full[as]);
        mma_commit(&land_empty);
        if (issued < ng) {  // the next group, once the MMAs have read this one
          if (!mbar_wait(&land_empty, (uint32_t)i & 1u, &abort_flag)) { ok = false; break; }
          copy_group((int)blockIdx.x + issued * (int)gridDim.x);
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
    // ---------------- consumers: thread = accumulator lane a = k bits 9..3 of every row
    const int arow = warp * 32 + lane;
    constexpr float kQ = QM == 0 ? 127.f : (QM == 1 ? 2.6457513110645906f : 7.f);
    constexpr bool kAbsmax = QM != 1;
    constexpr int PER = R >= 4 ? 1 : 4 / R;  // independent accumulators per row
    const bool packed4 = (a.fmt == 0) && (QM != 0);
    for (int i = 0; i < ng; ++i) {
      const int as = i & 1;
      const int g = (int)blockIdx.x + i * (int)gridDim.x;
      const bool got = mbar_wait(&acc_full[as], (uint32_t)(i >> 1) & 1u, &abort_flag);
      if (consumer_bar_or(!got || abort_flag)) break;  // the same decision in every consumer
      tc_fence_after();

      // ---- the 128 columns of this lane: column r NB + 8 nh + nl is D[a] of row r at the features
      // 1024 nh + 8 a + nl
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
      if (lane == 0) mbar_arrive(&acc_empty[as]);  // the accumulator may take the group after next

      // sum of squares per row: sum_a,n D^2 = 128 sum x^2 (H_128 has orthogonal rows of norm^2 128)
      float ss[R], st[R];
      {
        float2 acc[R * PER];
#pragma unroll
        for (int q = 0; q < R * PER; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const int q = (2 * j / NB) * PER + (j % PER);
          acc[q] = __ffma2_rn(v[j], v[j], acc[q]);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float t = 0.f;
#pragma unroll
          for (int q = 0; q < PER; ++q) t += acc[r * PER + q].x + acc[r * PER + q].y;
          ss[r] = t;
        }
      }

      fwht_regs2<128, NST>(v);  // the factor over n within each block

      if constexpr (kAbsmax) {
        float acc[R * PER];
#pragma unroll
        for (int q = 0; q < R * PER; ++q) acc[q] = 0.f;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const int q = (2 * j / NB) * PER + (j % PER);
          acc[q] = fmaxf(acc[q], fmaxf(fabsf(v[j].x), fabsf(v[j].y)));
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float t = 0.f;
#pragma unroll
          for (int q = 0; q < PER; ++q) t = fmaxf(t, acc[r * PER + q]);
          st[r] = t;
        }
      } else {
        float2 acc[R * PER];
#pragma unroll
        for (int q = 0; q < R * PER; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 64; j += 2) {  // v[j], v[j + 1]: the same row
          const int q = (2 * j / NB) * PER + ((j / 2) % PER);
          const float2 t = make_float2(fabsf(v[j].x) + fabsf(v[j].y), fabsf(v[j + 1].x) + fabsf(v[j + 1].y));
          acc[q] = __fadd2_rn(acc[q], t);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float t = 0.f;
#pragma unroll
          for (int q = 0; q < PER; ++q) t += acc[r * PER + q].x + acc[r * PER + q].y;
          st[r] = t;
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          ss[r] += __shfl_xor_sync(0xffffffffu, ss[r], o);
          const float t = __shfl_xor_sync(0xffffffffu, st[r], o);
          st[r] = kAbsmax ? fmaxf(st[r], t) : st[r] + t;
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          red_ss[as][r][warp] = ss[r];
          red_st[as][r][warp] = st[r];
        }
      }
      consumer_bar();

      // ---- per-row multiplier and scale (y = the unnormalised transform of x): row r in lane r of
      // every warp, from the same sums in the same order, so every thread gets the same values
      float mult_l, sx_l;
      int lanes16_l;
      {
        const int r = lane < R ? lane : 0;
        const float* rs_ = red_ss[as][r];
        const float* rt_ = red_st[as][r];
        const float ssr = (rs_[0] + rs_[1]) + (rs_[2] + rs_[3]);
        const float str = kAbsmax ? fmaxf(fmaxf(rt_[0], rt_[1]), fmaxf(rt_[2], rt_[3]))
                                  : (rt_[0] + rt_[1]) + (rt_[2] + rt_[3]);
        const float r_rms = sqrtf(ssr / ((float)P * (float)K) + a.eps_norm);  // sum D^2 = P sum x^2
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
        // the absmean clamp may run on 16-bit lanes when every rounded product fits an int16:
        // |y mult| <= mult ||y||_2 and ||y||_2^2 = (HB / P) ssr (the remaining stages scale the sum
        // of squares by HB / P), so mult sqrt(HB / P ssr) < 30000 guarantees it with room for fp32
        // rounding
        lanes16_l = mult_l * sqrtf((float)(HB / P) * ssr) < 30000.f ? 1 : 0;
      }
      if (warp == 0 && lane < R && g * R + lane < a.M) a.s_x[g * R + lane] = sx_l;

#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int row = g * R + r;
        if (row >= a.M) break;  // the same in every thread
        const float mult = __shfl_sync(0xffffffffu, mult_l, r);
        const int lanes16 = __shfl_sync(0xffffffffu, lanes16_l, r);
        const float2 mult2 = make_float2(mult, mult);
        const float2* vr = v + r * (NB / 2);
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
  if (warp == 4) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kNtTmemCols)
                 : "memory");
  }
}

}  // namespace hbl
