// Fused RMSNorm -> fast Walsh-Hadamard transform -> per-token quantisation (one kernel).
//
// Method: BitNet v2 walkthrough article (m.jxzklqfsx.com), section "H-BitLinear模塊": the layer
// applies an online Hadamard transform, computed with the fast Hadamard transform in
// O(n log n), to the normalised activations before quantising them per token to INT8 or INT4.
//
// A CTA owns `rows` token rows (one row for the big transforms). Its threads load the bf16
// row straight from global memory into registers; several CTAs share an SM, so that one CTA's
// loads are in flight while the others compute.
//
// One token row has K = nb blocks of n = 2^L features (nb = 1 for a transform over all of K).
// A block is transformed by P = 2^(L-EB) threads holding E = 2^EB values each:
//   1. "layout 1": a thread holds 8 consecutive features (index bits 0..2) for each of the
//      2^(EB-3) top index bits; read from global memory as 16-byte vectors; the sum of
//      squares for the RMS accumulates here; all EB butterfly stages run in registers.
//   2. one pass through shared memory (128-bit stores, scalar loads, XOR swizzle checked at
//      compile time) regroups the values so that index bits 3..TOP-1 are in registers
//      ("layout 2"); their L-EB butterfly stages run in registers.
//   3. the row statistic (max|y| or sum|y|) and the sum of squares are reduced over the row;
//      codes are decided in fp32 (product with the per-row multiplier, then round to nearest
//      even), written to a byte matrix [k mod 8][k / 8] in shared memory with 128-bit stores,
//      and streamed out in natural order after a register byte transpose.
// Butterflies use packed fp32x2 adds (two butterflies per instruction) except on the register
// bit that pairs the two halves of a float2. They act on the raw x (times gain): the RMS factor
// and the 1/sqrt(n) of the orthonormal transform only rescale the row, so they are folded into
// the per-row multiplier and into s_x. The stage order differs from a textbook loop; in exact
// arithmetic the stages commute, in fp32 the result differs by rounding only.
#pragma once

#include "common.cuh"

namespace hbl {

struct NfqArgs {
  const uint16_t* X;  // bf16 bits [M][K]
  const float* gain;  // [K] or nullptr
  uint8_t* codes;
  float* s_x;
  int M, K, nb;       // nb = K / n
  int fmt;            // hbl_codes_fmt
  float eps_norm, eps_q;
  int slots;          // blocks of a row transformed concurrently (threads per row = slots * P)
  int rows;           // token rows per group
  int groups;         // ceil(M / rows)
  int pf_dist;        // a CTA prefetches the rows of group blockIdx.x + pf_dist into L2 (0 = none)
};

// ---------------------------------------------------------------- compile-time plan

template <int L_, int EB_>
struct FhtPlan {
  static constexpr int L = L_, EB = EB_;
  static constexpr int n = 1 << L;
  static constexpr int P = 1 << (L - EB);    // threads per block transform
  static constexpr int E = 1 << EB;          // values per thread per block
  static constexpr int NV = 1 << (EB - 3);   // 8-feature vectors per thread per block (layout 1)
  static constexpr int TOP = L - (EB - 3);   // lowest index bit of the register "top" bits
  static constexpr int XB = 2 * EB - L;      // index bits 0..XB-1 also held in registers in layout 2
  static constexpr int S2 = L - EB;          // butterfly stages run in layout 2
  static_assert(EB >= 3 && XB >= 0 && XB <= 1, "unsupported transform split");
  static_assert(S2 >= 4, "layout 2 writes codes in 16-byte groups");
  static_assert(P == 16 || P % 32 == 0, "threads per block must be 16 or a multiple of 32");
  static_assert(TOP >= 7, "swizzle needs TOP >= 7");

  // Layout 1: register r = (vv << 3) | e, thread p  ->  index (vv << TOP) | (p << 3) | e
  static __host__ __device__ constexpr int idx1(int p, int r) {
    return ((r >> 3) << TOP) | (p << 3) | (r & 7);
  }
  // Layout 2: register r: low S2 bits -> index bits 3..TOP-1, high XB bits -> index bits 0..XB-1;
  //           thread p: low 3-XB bits -> index bits XB..2, high bits -> index bits TOP..L-1.
  static __host__ __device__ constexpr int idx2(int p, int r) {
    return ((r & ((1 << S2) - 1)) << 3) | (r >> S2) | ((p & ((1 << (3 - XB)) - 1)) << XB) |
           ((p >> (3 - XB)) << TOP);
  }
  // Address bit that lane bit j selects in layout 2 (lane bits past the block's P threads select
  // the neighbouring block or row, i.e. address bit L, when P == 16).
  static constexpr int lane_bit2(int j) { return (1 << j) < P ? ilog2_c(idx2(1 << j, 0)) : L; }
  // Float swizzle: bits 0-1 untouched (128-bit stores keep 4 floats together); bit 2 ^= bit 5,
  // bit 3 ^= first high lane bit of layout 2, bit 4 ^= the second one.
  static constexpr int H1 = lane_bit2(3 - XB), H2 = lane_bit2(4 - XB);
  static __host__ __device__ constexpr uint32_t swz(uint32_t a) {
    return a ^ ((((a >> 5) & 1u) << 2) | (((a >> H1) & 1u) << 3) | (((a >> H2) & 1u) << 4));
  }

  // Exhaustive compile-time check of bank conflicts: layout-1 128-bit stores (the 8 lanes of a
  // phase must hit distinct 16-byte groups) and layout-2 scalar loads (32 lanes on distinct
  // banks; a two-way conflict is unavoidable when index bit 0 is a register bit).
  static constexpr uint32_t addr(int which, int lane, int r) {
    const int p = lane % (P < 32 ? P : 32);
    const uint32_t blk = (P < 32) ? (uint32_t)(lane / P) : 0u;
    return swz((blk << L) | (uint32_t)(which == 1 ? idx1(p, r) : idx2(p, r)));
  }
  static constexpr bool check_store1() {
    for (int r = 0; r < E; r += 4)
      for (int ph = 0; ph < 4; ++ph) {
        uint32_t seen = 0;
        for (int l = 8 * ph; l < 8 * ph + 8; ++l) {
          const uint32_t g = (addr(1, l, r) >> 2) & 7u;
          if ((seen >> g) & 1u) return false;
          seen |= 1u << g;
        }
      }
    return true;
  }
  static constexpr int load2_ways() {
    int worst = 1;
    for (int r = 0; r < E; ++r) {
      int cnt[32] = {0};
      for (int l = 0; l < 32; ++l) {
        const int b = (int)(addr(2, l, r) & 31u);
        if (++cnt[b] > worst) worst = cnt[b];
      }
    }
    return worst;
  }
};

// Swizzled float index swz(tb) ^ swz(rc) for a runtime thread part tb and compile-time register
// parts rc. Only bits 2..4 of the two swizzled parts overlap (the swizzle mixes nothing else), so
// the thread keeps 8 bases, one per value of those bits, and each access is base + constant:
// the constant folds into the load/store offset instead of costing an XOR per access.
template <class Pl>
struct SwzBases {
  uint32_t b[8];
  __device__ __forceinline__ explicit SwzBases(uint32_t tb) {
    const uint32_t t = Pl::swz(tb);
#pragma unroll
    for (uint32_t c = 0; c < 8; ++c) b[c] = (t & ~0x1cu) | ((((t >> 2) & 7u) ^ c) << 2);
  }
  // index of register part rc (a compile-time constant after unrolling)
  __device__ __forceinline__ uint32_t at(uint32_t rc) const {
    const uint32_t r = Pl::swz(rc);
    return b[(r >> 2) & 7u] + (r & ~0x1cu);
  }
};

// ---------------------------------------------------------------- register butterflies

// Butterfly stages on register-index bits 0 .. NSTAGE-1 of v (E values stored as E/2 float2;
// register r lives in v[r >> 1].x/.y). Sylvester order: (a, b) at (j, j+h) becomes (a+b, a-b).
// With SKIP0 the stage on register bit 0 has already been applied by the caller.
template <int E, int NSTAGE, bool SKIP0 = false>
__device__ __forceinline__ void fwht_regs2(float2 (&v)[E / 2]) {
  // register bit 0: the two halves of each float2
  if constexpr (!SKIP0) {
#pragma unroll
    for (int j = 0; j < E / 2; ++j) {
      const float a = v[j].x, b = v[j].y;
      v[j].x = a + b;
      v[j].y = a - b;
    }
  }
  const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int h = 1; h < (1 << (NSTAGE - 1)); h <<= 1) {  // register bits 1.. -> float2 index bits
#pragma unroll
    for (int j = 0; j < E / 2; ++j) {
      if ((j & h) == 0) {
        const float2 a = v[j], b = v[j + h];
        v[j] = __fadd2_rn(a, b);
        v[j + h] = __ffma2_rn(b, neg1, a);  // a - b, exactly rounded
      }
    }
  }
}

// ---------------------------------------------------------------- the kernel

// Largest CTA a plan is launched with, and the register cap that lets several such CTAs share
// an SM (the big transforms hold 128 values per thread).
// (The block-256 plan runs 352-thread CTAs of 32 values per thread: two of them share an SM
// only at <= 72 registers, since each SM quarter holds 16384 registers and gets 6 of the 22 warps.)
constexpr int nfq_max_threads(int L) { return L >= 11 ? 256 : 512; }
constexpr int nfq_max_regs(int EB, int R) {
  return ((1 << EB) * R) >= 128 ? 168 : (((1 << EB) * R) >= 64 ? 128 : (((1 << EB) * R) >= 32 ? 72 : 64));
}

// 16-byte streaming load that bypasses L1 (every input byte is read once).
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// First butterfly stage straight from a word holding two bf16 features a (low half) and b (high
// half): (a + b, a - b) in fp32, with a read as bf16 by the add itself (exact widening).
__device__ __forceinline__ float2 bf16x2_butterfly(uint32_t u) {
  const float b = __uint_as_float(u & 0xffff0000u);
  float2 r;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.bf16 %0, lo, %3;\n\tsub.rn.f32.bf16 %1, lo, %3;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "r"(u), "f"(b));
  return r;
}

// QM: 0 = a8 absmax, 1 = a4 absmean, 2 = a4 absmax
template <int L, int EB, int R, bool HAS_GAIN, int QM>
__global__ void __maxnreg__(nfq_max_regs(EB, R)) norm_fht_quant_kernel(const NfqArgs a) {
  using Pl = FhtPlan<L, EB>;
  static_assert(Pl::check_store1(), "layout-1 stores have bank conflicts");
  static_assert(Pl::load2_ways() <= (Pl::XB ? 2 : 1), "layout-2 loads have avoidable bank conflicts");
  constexpr int n = Pl::n, P = Pl::P, E = Pl::E, NV = Pl::NV, S2 = Pl::S2, XB = Pl::XB;
  extern __shared__ __align__(128) uint8_t smem_nfq[];
  __shared__ float red_ss[32], red_st[32];

  const int K = a.K, nb = a.nb, rows = a.rows;
  float* fbuf = reinterpret_cast<float*>(smem_nfq);  // rows*K fp32 (regrouping)
  uint8_t* cbuf = smem_nfq;                          // codes, reuses the regrouping buffer
  const int crow = K / 8 + 16;  // byte stride of one (k mod 8) row of the code matrix (padded)

  const int tid = threadIdx.x;
  const int tpr = a.slots * P;
  const int rloc = tid / tpr;
  const int tr = tid - rloc * tpr;
  const int slot = tr / P;
  const int pt = tr - slot * P;
  const int lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.x;
  const int row = g * rows + rloc;
  const bool live_row = row < a.M;
  // Rows past M (last group only) and padding blocks past nb compute on live data and store
  // nothing, so that every load is unconditional.
  const int srow = live_row ? row : a.M - 1;

  // X may come from the kernel before this one (launched early by programmatic dependent
  // launch): wait for it. Then the product that consumes these codes may start: it streams its
  // weights, which this kernel does not write, and waits for this kernel's completion before it
  // reads the codes.
  pdl_wait();
  pdl_launch_dependents();

  // a later group's rows into L2 while this group loads and computes
  if (tid == 0 && a.pf_dist > 0 && g + a.pf_dist < a.groups) {
    const int g2 = g + a.pf_dist;
    const uint32_t bytes = (uint32_t)min(rows, a.M - g2 * rows) * (uint32_t)K * 2u;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.X + (size_t)g2 * rows * K), "r"(bytes)
                 : "memory");
  }

  constexpr float kQ = QM == 0 ? 127.f : (QM == 1 ? 2.6457513110645906f : 7.f);
  constexpr int kLo = QM == 0 ? -128 : -8, kHi = QM == 0 ? 127 : 7;
  constexpr bool kAbsmax = QM != 1;

  // ---- 1. layout 1 straight from global memory (16-byte vectors, every load issued before the
  // first use), sum of squares; without a gain the first butterfly stage (index bit 0, the two
  // halves of a bf16 pair) is taken while widening.
  float2 v[R][E / 2];
  float ss = 0.f;
  {
    uint4 w[R][NV];
#pragma unroll
    for (int rho = 0; rho < R; ++rho) {
      const int blk = slot + rho * a.slots;
      const uint16_t* src = a.X + (size_t)srow * K + (size_t)(blk < nb ? blk : 0) * n + (pt << 3);
#pragma unroll
      for (int vv = 0; vv < NV; ++vv) w[rho][vv] = ldg_stream_v4(src + (vv << Pl::TOP));
    }
#pragma unroll
    for (int rho = 0; rho < R; ++rho) {
      const int blk = slot + rho * a.slots;
      float2 ss2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int vv = 0; vv < NV; ++vv) {
        const uint32_t u[4] = {w[rho][vv].x, w[rho][vv].y, w[rho][vv].z, w[rho][vv].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float2 f;
          if constexpr (HAS_GAIN) {
            f = make_float2(__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xffff0000u));
            ss2[i] = __ffma2_rn(f, f, ss2[i]);
            const float2 gg = *reinterpret_cast<const float2*>(a.gain + (size_t)(blk < nb ? blk : 0) * n +
                                                               (vv << Pl::TOP) + (pt << 3) + 2 * i);
            f = __fmul2_rn(f, gg);
          } else {
            f = bf16x2_butterfly(u[i]);
            ss2[i] = __ffma2_rn(f, f, ss2[i]);  // (a+b)^2 + (a-b)^2 = 2 (a^2 + b^2)
          }
          v[rho][vv * 4 + i] = f;
        }
      }
      const float ssr = ((ss2[0].x + ss2[0].y) + (ss2[1].x + ss2[1].y)) + ((ss2[2].x + ss2[2].y) + (ss2[3].x + ss2[3].y));
      if (blk < nb) ss += ssr;
    }
  }
  if constexpr (!HAS_GAIN) ss *= 0.5f;

#pragma unroll
  for (int rho = 0; rho < R; ++rho) fwht_regs2<E, EB, !HAS_GAIN>(v[rho]);

  // ---- 2. regroup through shared memory (index within the CTA buffer: (rloc*nb + blk)*n + i)
  const uint32_t rowbase = (uint32_t)rloc * (uint32_t)K;
#pragma unroll
  for (int rho = 0; rho < R; ++rho) {
    const int blk = slot + rho * a.slots;
    if (blk < nb) {
      const SwzBases<Pl> sb(rowbase + ((uint32_t)blk << L) + ((uint32_t)pt << 3));
#pragma unroll
      for (int r = 0; r < E; r += 4) {
        const float4 q4 = make_float4(v[rho][r / 2].x, v[rho][r / 2].y, v[rho][r / 2 + 1].x, v[rho][r / 2 + 1].y);
        *reinterpret_cast<float4*>(fbuf + sb.at((uint32_t)Pl::idx1(0, r))) = q4;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int rho = 0; rho < R; ++rho) {
    const int blk = slot + rho * a.slots;
    const SwzBases<Pl> sb(rowbase + ((uint32_t)(blk < nb ? blk : 0) << L) + (uint32_t)Pl::idx2(pt, 0));
#pragma unroll
    for (int r = 0; r < E; r += 2) {
      v[rho][r / 2].x = fbuf[sb.at((uint32_t)Pl::idx2(0, r))];
      v[rho][r / 2].y = fbuf[sb.at((uint32_t)Pl::idx2(0, r + 1))];
    }
    fwht_regs2<E, S2>(v[rho]);
  }

  // ---- 3. row statistics: sum |y| as pairwise sums folded into fp32x2 chains, or max |y|
  float st = 0.f;
#pragma unroll
  for (int rho = 0; rho < R; ++rho) {
    const int blk = slot + rho * a.slots;
    float str;
    if constexpr (kAbsmax) {
      float sta[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int r = 0; r < E / 2; ++r) sta[r & 3] = fmaxf(sta[r & 3], fmaxf(fabsf(v[rho][r].x), fabsf(v[rho][r].y)));
      str = fmaxf(fmaxf(sta[0], sta[1]), fmaxf(sta[2], sta[3]));
    } else {
      float2 sta2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int r = 0; r < E / 2; r += 2) {
        const float2 t = make_float2(fabsf(v[rho][r].x) + fabsf(v[rho][r].y),
                                     fabsf(v[rho][r + 1].x) + fabsf(v[rho][r + 1].y));
        sta2[(r / 2) & 3] = __fadd2_rn(sta2[(r / 2) & 3], t);
      }
      str = ((sta2[0].x + sta2[0].y) + (sta2[1].x + sta2[1].y)) + ((sta2[2].x + sta2[2].y) + (sta2[3].x + sta2[3].y));
    }
    if (blk < nb) st = kAbsmax ? fmaxf(st, str) : st + str;
  }
  if (tpr >= 32) {
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
    __syncthreads();  // also: every layout-2 read is done before codes overwrite the buffer
    const int w0 = (rloc * tpr) >> 5, nw = tpr >> 5;
    ss = 0.f;
    st = 0.f;
    for (int w = 0; w < nw; ++w) {  // fixed order: the same result in every thread of the row
      ss += red_ss[w0 + w];
      st = kAbsmax ? fmaxf(st, red_st[w0 + w]) : st + red_st[w0 + w];
    }
  } else {  // 16 threads per row, two rows per warp
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float t = __shfl_xor_sync(0xffffffffu, st, o);
      st = kAbsmax ? fmaxf(st, t) : st + t;
    }
    __syncthreads();  // every layout-2 read is done before codes overwrite the buffer
  }

  // ---- 4. per-row multiplier and scale
  const float r_rms = sqrtf(ss / (float)K + a.eps_norm);
  const float rs = r_rms * sqrtf((float)n);        // y = xr * rs (xr = orthonormal output)
  const float sy = kAbsmax ? st : st / (float)K;  // statistic of y
  float mult, sx;
  if (a.eps_q == 0.f) {
    mult = sy > 0.f ? kQ / sy : 0.f;
    sx = sy > 0.f ? sy / (rs * kQ) : 0.f;
  } else {
    const float stat = sy / rs;                     // statistic of xr
    mult = kQ / ((stat + a.eps_q) * rs);
    sx = stat / kQ;
  }
  if (live_row && tr == 0) a.s_x[row] = sx;

  // ---- 5. codes: fma(y, mult, 1.5 * 2^23) rounds the exact product to the nearest integer
  // (ties to even) in one step, the integer landing in the low mantissa bits (|y mult| < 2^22);
  // absmean then clamps that integer-valued sum to 1.5 * 2^23 + [-8, 7], exactly (absmax
  // products already lie in [-Q, Q]). The low byte is the code. 4 codes per word, 16 bytes per
  // store, into a byte matrix [k mod 8][k / 8].
  const float2 mult2 = make_float2(mult, mult);
  const float2 magic2 = make_float2(12582912.f, 12582912.f);
#pragma unroll
  for (int rho = 0; rho < R; ++rho) {
    const int blk = slot + rho * a.slots;
    if (blk < nb) {
#pragma unroll
      for (int x = 0; x < (1 << XB); ++x) {
        // codes of registers r = (x << S2) | j are those of k = 8 * (c0 + j) + b
        const int b = x | ((pt & ((1 << (3 - XB)) - 1)) << XB);
        const int c0 = (blk << (L - 3)) + ((pt >> (3 - XB)) << (Pl::TOP - 3));
        uint8_t* dst = cbuf + (size_t)rloc * 8 * crow + (size_t)b * crow + c0;
#pragma unroll
        for (int j = 0; j < (1 << S2); j += 16) {
          uint32_t wds[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int r0 = (x << S2) + j + 4 * q;  // 4 consecutive registers = 2 float2
            float2 p0 = __ffma2_rn(v[rho][r0 / 2], mult2, magic2);
            float2 p1 = __ffma2_rn(v[rho][r0 / 2 + 1], mult2, magic2);
            if constexpr (!kAbsmax) {
              constexpr float lo = 12582912.f + kLo, hi = 12582912.f + kHi;
              p0.x = fminf(fmaxf(p0.x, lo), hi);
              p0.y = fminf(fmaxf(p0.y, lo), hi);
              p1.x = fminf(fmaxf(p1.x, lo), hi);
              p1.y = fminf(fmaxf(p1.y, lo), hi);
            }
            const uint32_t h0 = __byte_perm(__float_as_uint(p0.x), __float_as_uint(p0.y), 0x5410);
            const uint32_t h1 = __byte_perm(__float_as_uint(p1.x), __float_as_uint(p1.y), 0x5410);
            wds[q] = __byte_perm(h0, h1, 0x6420);
          }
          *reinterpret_cast<uint4*>(dst + j) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
        }
      }
    }
  }
  __syncthreads();

  // ---- 6. stream codes out in natural order, 32 consecutive codes per unit. A thread owns at
  // most R*E/32 units (units tid, tid + blockDim, ...). With nb == 1 a row has 2^(L-5) units;
  // with nb > 1 the CTA holds one row.
  const int upr = K / 32;
  const int units = rows * upr;
  const bool packed4 = (a.fmt == 0) && (QM != 0);
#pragma unroll
  for (int it = 0; it < (R * E + 31) / 32; ++it) {
    const int unit = tid + it * (int)blockDim.x;
    if (unit >= units) break;
    const int rl = nb == 1 ? (unit >> (L - 5)) : 0;
    const int vcol = unit - rl * upr;
    const int grow = g * rows + rl;
    if (grow >= a.M) break;  // later units belong to later rows
    const uint8_t* srcc = cbuf + (size_t)rl * 8 * crow + 4 * vcol;
    uint32_t w[8];
#pragma unroll
    for (int b = 0; b < 8; ++b) w[b] = *reinterpret_cast<const uint32_t*>(srcc + (size_t)b * crow);
    // byte j of w[b] is the code of k = 32 * vcol + 8 * j + b
    if (!packed4) {
      uint32_t o[8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // k mod 8 = 4h .. 4h+3
        const uint32_t a01l = __byte_perm(w[4 * h], w[4 * h + 1], 0x5140);
        const uint32_t a01h = __byte_perm(w[4 * h], w[4 * h + 1], 0x7362);
        const uint32_t a23l = __byte_perm(w[4 * h + 2], w[4 * h + 3], 0x5140);
        const uint32_t a23h = __byte_perm(w[4 * h + 2], w[4 * h + 3], 0x7362);
        o[0 + h] = __byte_perm(a01l, a23l, 0x5410);  // j = 0
        o[2 + h] = __byte_perm(a01l, a23l, 0x7632);  // j = 1
        o[4 + h] = __byte_perm(a01h, a23h, 0x5410);  // j = 2
        o[6 + h] = __byte_perm(a01h, a23h, 0x7632);  // j = 3
      }
      uint4* dstg = reinterpret_cast<uint4*>(a.codes + (size_t)grow * K + 32 * vcol);
      dstg[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dstg[1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else {
      // nibble pairs first: byte j of m[i] = code(8j + 2i) | code(8j + 2i + 1) << 4
      uint32_t m[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) m[i] = (w[2 * i] & 0x0f0f0f0fu) | ((w[2 * i + 1] & 0x0f0f0f0fu) << 4);
      const uint32_t a01l = __byte_perm(m[0], m[1], 0x5140);
      const uint32_t a01h = __byte_perm(m[0], m[1], 0x7362);
      const uint32_t a23l = __byte_perm(m[2], m[3], 0x5140);
      const uint32_t a23h = __byte_perm(m[2], m[3], 0x7362);
      const uint4 o = make_uint4(__byte_perm(a01l, a23l, 0x5410), __byte_perm(a01l, a23l, 0x7632),
                                 __byte_perm(a01h, a23h, 0x5410), __byte_perm(a01h, a23h, 0x7632));
      *reinterpret_cast<uint4*>(a.codes + (size_t)grow * (K / 2) + 16 * vcol) = o;
    }
  }
}

}  // namespace hbl
