// Fused RMSNorm -> fast Walsh-Hadamard transform -> per-token quantisation (one kernel).
//
// Method: BitNet v2 walkthrough article (m.jxzklqfsx.com), section "H-BitLinear模塊": the layer
// applies an online Hadamard transform, computed with the fast Hadamard transform in
// O(n log n), to the normalised activations before quantising them per token to INT8 or INT4.
//
// Data flow of one token row (K = nb blocks of n = 2^L features; nb = 1 for a full transform):
//   1. 16-byte coalesced bf16 loads straight into registers ("layout 1"): a thread holds
//      E = 2^EB values of a block: 8 consecutive features (index bits 0..2) for each of the
//      2^(EB-3) top index bits. Sum of squares for the RMS accumulates here.
//   2. All EB butterfly stages whose index bits live in registers run in registers.
//   3. One pass through shared memory (XOR-swizzled so that both the write and the read are
//      free of bank conflicts) regroups the values so that the remaining L-EB index bits live
//      in registers ("layout 2"); their butterfly stages run in registers.
//   4. The row statistic (max|y| or sum|y|) and the sum of squares are reduced across the
//      threads of the row; the codes are decided in fp32 and written as bytes to shared memory
//      (second XOR swizzle), then streamed out with 16-byte loads and 8/16-byte stores.
// The butterflies act on the raw x (times gain); the RMS factor and the 1/sqrt(n) of the
// orthonormal transform only rescale the row, so they are folded into the per-row multiplier
// and into s_x. Stage order differs from a textbook loop; in exact arithmetic the stages
// commute, in fp32 the result differs by rounding only.
#pragma once

#include "common.cuh"

namespace hbl {

struct NfqArgs {
  const uint16_t* X;  // bf16 bits [M][K]
  const float* gain;  // [K] or nullptr
  uint8_t* codes;
  float* s_x;
  int M, K, nb;       // nb = K / n
  int quant;          // hbl_quant
  int fmt;            // hbl_codes_fmt
  float eps_norm, eps_q;
  int slots;          // blocks of a row transformed concurrently (threads per row = slots * P)
  int rows;           // token rows per CTA
};

// ---------------------------------------------------------------- compile-time plan

template <int L_, int EB_>
struct FhtPlan {
  static constexpr int L = L_, EB = EB_;
  static constexpr int n = 1 << L;
  static constexpr int P = 1 << (L - EB);    // threads per block transform
  static constexpr int E = 1 << EB;          // values per thread per block
  static constexpr int NV = 1 << (EB - 3);   // 16-byte vectors per thread per block (layout 1)
  static constexpr int TOP = L - (EB - 3);   // lowest index bit of the register "top" bits
  static constexpr int XB = 2 * EB - L;      // index bits 0..XB-1 also held in registers in layout 2
  static constexpr int S2 = L - EB;          // butterfly stages run in layout 2
  static_assert(EB >= 3 && XB >= 0 && XB <= 3, "unsupported transform split");
  static_assert(P == 16 || P % 32 == 0, "threads per block must be 16 or a multiple of 32");
  static_assert(TOP >= 7, "byte swizzle needs TOP >= 7");

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

  // Address bits that vary across the 32 lanes of a warp in each layout. When P == 16 the
  // fifth lane bit selects the neighbouring block (or row), i.e. address bit L.
  static constexpr uint32_t lanes1() {
    uint32_t m = 0;
    for (int b = 0; b < 5; ++b) {
      if ((1 << b) < P) m |= (uint32_t)idx1(1 << b, 0);
      else m |= 1u << L;
    }
    return m;
  }
  static constexpr uint32_t lanes2() {
    uint32_t m = 0;
    for (int b = 0; b < 5; ++b) {
      if ((1 << b) < P) m |= (uint32_t)idx2(1 << b, 0);
      else m |= 1u << L;
    }
    return m;
  }

  // Byte swizzle of the code staging buffer: XOR byte-address bits 3..6 with bits TOP..TOP+3.
  static __host__ __device__ constexpr uint32_t bswz(uint32_t a) {
    return a ^ (((a >> TOP) & 15u) << 3);
  }
};


// Float swizzle of the regrouping buffer for a plan: bank bit k (address bit k, k < 5) is XORed
// with the parity of (a & S[k]), where S[k] only holds address bits >= 5 (so the map is a
// bijection on every 32-word row). Each layout's lane bits >= 5 are assigned to the bank bits
// that this layout's own low lane bits do not already drive; a lane bit shared by both layouts
// drives one free bank bit of each. check_layout() verifies exhaustively, at compile time, that
// every warp access of both layouts is free of bank conflicts.
template <class Pl>
struct FhtSwizzle {
  struct Masks {
    uint32_t S[5];
  };
  static constexpr Masks solve() {
    Masks s{{0, 0, 0, 0, 0}};
    const uint32_t l1 = Pl::lanes1(), l2 = Pl::lanes2();
    uint32_t need1 = ~l1 & 31u, need2 = ~l2 & 31u;
    uint32_t hi1 = l1 & ~31u, hi2 = l2 & ~31u;
    for (int c = 5; c < 32; ++c) {
      const uint32_t bit = 1u << c;
      if ((hi1 & bit) && (hi2 & bit)) {
        int k1 = 0, k2 = 0;
        while (!((need1 >> k1) & 1u)) ++k1;
        while (!((need2 >> k2) & 1u)) ++k2;
        s.S[k1] |= bit;
        if (k2 != k1) s.S[k2] |= bit;
        need1 &= ~(1u << k1);
        need2 &= ~(1u << k2);
        hi1 &= ~bit;
        hi2 &= ~bit;
      }
    }
    for (int c = 5; c < 32; ++c) {
      const uint32_t bit = 1u << c;
      if (hi1 & bit) {
        int k = 0;
        while (!((need1 >> k) & 1u)) ++k;
        s.S[k] |= bit;
        need1 &= ~(1u << k);
      }
      if (hi2 & bit) {
        int k = 0;
        while (!((need2 >> k) & 1u)) ++k;
        s.S[k] |= bit;
        need2 &= ~(1u << k);
      }
    }
    return s;
  }
  static constexpr uint32_t S0 = solve().S[0], S1 = solve().S[1], S2 = solve().S[2], S3 = solve().S[3],
                            S4 = solve().S[4];

  static __host__ __device__ constexpr uint32_t parity(uint32_t v) {
    v ^= v >> 16; v ^= v >> 8; v ^= v >> 4; v ^= v >> 2; v ^= v >> 1;
    return v & 1u;
  }
  static __host__ __device__ constexpr uint32_t swz(uint32_t a) {
    return a ^ ((parity(a & S0) << 0) | (parity(a & S1) << 1) | (parity(a & S2) << 2) | (parity(a & S3) << 3) |
                (parity(a & S4) << 4));
  }

  // For every register index, the 32 lanes of a warp hit 32 distinct banks.
  static constexpr bool check_layout(int which) {
    for (int r = 0; r < Pl::E; ++r) {
      uint32_t seen = 0;
      for (int lane = 0; lane < 32; ++lane) {
        const int p = lane % (Pl::P < 32 ? Pl::P : 32);
        const uint32_t blk = (Pl::P < 32) ? (uint32_t)(lane / Pl::P) : 0u;
        const uint32_t a = (blk << Pl::L) | (uint32_t)(which == 1 ? Pl::idx1(p, r) : Pl::idx2(p, r));
        const uint32_t bank = swz(a) & 31u;
        if ((seen >> bank) & 1u) return false;
        seen |= 1u << bank;
      }
    }
    return true;
  }
  static_assert(check_layout(1) && check_layout(2), "shared-memory swizzle has bank conflicts");
};

// ---------------------------------------------------------------- register butterflies

// Butterfly stages h = 1, 2, 4, ..., < (1 << NSTAGE) over a register array (Sylvester order:
// (a, b) at (j, j+h) becomes (a + b, a - b)).
template <int E, int NSTAGE>
__device__ __forceinline__ void fwht_regs(float (&v)[E]) {
#pragma unroll
  for (int h = 1; h < (1 << NSTAGE); h <<= 1) {
#pragma unroll
    for (int j = 0; j < E; ++j) {
      if ((j & h) == 0) {
        const float a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
    }
  }
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& w, float* f) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}

// ---------------------------------------------------------------- the kernel

// Largest CTA a plan is launched with (bounds the register budget of the big transforms).
constexpr int nfq_max_threads(int L) { return L >= 13 ? 256 : (L >= 11 ? 512 : 1024); }

template <int L, int EB, int R, bool HAS_GAIN>
__global__ void __launch_bounds__(nfq_max_threads(L)) norm_fht_quant_kernel(const NfqArgs a) {
  using Pl = FhtPlan<L, EB>;
  using Sw = FhtSwizzle<Pl>;
  constexpr int n = Pl::n, P = Pl::P, E = Pl::E, NV = Pl::NV;
  extern __shared__ __align__(16) float smem_f[];
  __shared__ float red_ss[32], red_st[32];

  const int tid = threadIdx.x;
  const int tpr = a.slots * P;
  const int rloc = tid / tpr;
  const int tr = tid - rloc * tpr;
  const int slot = tr / P;
  const int pt = tr - slot * P;
  const int row = blockIdx.x * a.rows + rloc;
  const bool live_row = row < a.M;
  const int K = a.K, nb = a.nb;

  float v[R][E];
  float ss = 0.f;

  // 1. load (layout 1) + sum of squares (+ gain), then in-register stages
#pragma unroll
  for (int rho = 0; rho < R; ++rho) {
    const int blk = slot + rho * a.slots;
    const bool live = live_row && blk < nb;
    const uint16_t* src = a.X + (size_t)row * K + (size_t)blk * n + (pt << 3);
#pragma unroll
    for (int vv = 0; vv < NV; ++vv) {
      float f[8];
      if (live) {
        const uint4 w = __ldcs(reinterpret_cast<const uint4*>(src + (vv << Pl::TOP)));
        bf16x8_to_f32(w, f);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        ss = fmaf(f[e], f[e], ss);
        if constexpr (HAS_GAIN) {
          if (live) f[e] *= __ldg(a.gain + (size_t)blk * n + (vv << Pl::TOP) + (pt << 3) + e);
        }
        v[rho][vv * 8 + e] = f[e];
      }
    }
    fwht_regs<E, EB>(v[rho]);
  }

  // 2. regroup through shared memory. The swizzle acts on the float index inside the CTA's
  // buffer, (rloc * nb + blk) * n + i; the block part has no bits below L, so the swizzle of
  // the thread's part and of the (compile-time) register part combine by XOR.
  const uint32_t rowbase = (uint32_t)rloc * (uint32_t)K;
#pragma unroll
  for (int rho = 0; rho < R; ++rho) {
    const int blk = slot + rho * a.slots;
    if (blk < nb) {
      const uint32_t tb = rowbase + ((uint32_t)blk << L) + ((uint32_t)pt << 3);
      const uint32_t tbs = Sw::swz(tb);
#pragma unroll
      for (int r = 0; r < E; ++r) {
        const uint32_t rc = (uint32_t)Pl::idx1(0, r);
        smem_f[tbs ^ Sw::swz(rc)] = v[rho][r];
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int rho = 0; rho < R; ++rho) {
    const int blk = slot + rho * a.slots;
    if (blk < nb) {
      const uint32_t tb = rowbase + ((uint32_t)blk << L) + (uint32_t)Pl::idx2(pt, 0);
      const uint32_t tbs = Sw::swz(tb);
#pragma unroll
      for (int r = 0; r < E; ++r) {
        const uint32_t rc = (uint32_t)Pl::idx2(0, r);
        v[rho][r] = smem_f[tbs ^ Sw::swz(rc)];
      }
      fwht_regs<E, Pl::S2>(v[rho]);
    } else {
#pragma unroll
      for (int r = 0; r < E; ++r) v[rho][r] = 0.f;
    }
  }

  // 3. row statistics
  const bool use_max = (a.quant != 1);
  float st = 0.f;
#pragma unroll
  for (int rho = 0; rho < R; ++rho) {
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const float m = fabsf(v[rho][r]);
      st = use_max ? fmaxf(st, m) : st + m;
    }
  }
  const int lane = tid & 31, warp = tid >> 5;
  if (tpr >= 32) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float t = __shfl_xor_sync(0xffffffffu, st, o);
      st = use_max ? fmaxf(st, t) : st + t;
    }
    if (lane == 0) {
      red_ss[warp] = ss;
      red_st[warp] = st;
    }
    __syncthreads();
    const int w0 = (rloc * tpr) >> 5, nw = tpr >> 5;
    ss = 0.f;
    st = 0.f;
    for (int w = 0; w < nw; ++w) {  // fixed order: identical result in every thread of the row
      ss += red_ss[w0 + w];
      st = use_max ? fmaxf(st, red_st[w0 + w]) : st + red_st[w0 + w];
    }
  } else {  // 16 threads per row, two rows per warp
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float t = __shfl_xor_sync(0xffffffffu, st, o);
      st = use_max ? fmaxf(st, t) : st + t;
    }
    __syncthreads();  // every layout-2 read is done before codes overwrite shared memory
  }

  // 4. per-row multiplier and scale
  float qmax, lo, hi;
  if (a.quant == 0) { qmax = 127.f; lo = -128.f; hi = 127.f; }
  else if (a.quant == 1) { qmax = 2.6457513110645906f; lo = -8.f; hi = 7.f; }
  else { qmax = 7.f; lo = -8.f; hi = 7.f; }
  const float r_rms = sqrtf(ss / (float)K + a.eps_norm);
  const float rs = r_rms * sqrtf((float)n);           // y = xr * rs  (xr = orthonormal output)
  const float sy = use_max ? st : st / (float)K;     // statistic of y
  float mult, sx;
  if (a.eps_q == 0.f) {
    mult = sy > 0.f ? qmax / sy : 0.f;
    sx = sy > 0.f ? sy / (rs * qmax) : 0.f;
  } else {
    const float stat = sy / rs;                        // statistic of xr
    mult = qmax / ((stat + a.eps_q) * rs);
    sx = stat / qmax;
  }
  if (live_row && tr == 0) a.s_x[row] = sx;

  // 5. codes -> shared bytes (swizzled), layout-2 positions
  uint8_t* sbytes = reinterpret_cast<uint8_t*>(smem_f);
#pragma unroll
  for (int rho = 0; rho < R; ++rho) {
    const int blk = slot + rho * a.slots;
    if (blk < nb) {
#pragma unroll
      for (int r = 0; r < E; ++r) {
        float q = __fmul_rn(v[rho][r], mult);
        q = fminf(fmaxf(q, lo), hi);
        const int qi = __float2int_rn(q);
        const uint32_t ba = rowbase + ((uint32_t)blk << L) + (uint32_t)Pl::idx2(pt, r);
        sbytes[Pl::bswz(ba)] = (uint8_t)(qi & 0xff);
      }
    }
  }
  __syncthreads();

  // 6. stream codes out in natural order
  const int chunks = a.rows * K / 16;
  const bool packed4 = (a.fmt == 0) && (a.quant != 0);
  for (int c = tid; c < chunks; c += blockDim.x) {
    const uint32_t off = (uint32_t)c * 16;
    const int rl = (int)(off / (uint32_t)K);
    const int col = (int)(off - (uint32_t)rl * K);
    const int grow = blockIdx.x * a.rows + rl;
    if (grow >= a.M) continue;
    const uint2 lo8 = *reinterpret_cast<const uint2*>(sbytes + Pl::bswz(off));
    const uint2 hi8 = *reinterpret_cast<const uint2*>(sbytes + Pl::bswz(off + 8));
    if (!packed4) {
      uint4 o = make_uint4(lo8.x, lo8.y, hi8.x, hi8.y);
      *reinterpret_cast<uint4*>(a.codes + (size_t)grow * K + col) = o;
    } else {
      // bytes b0..b15 -> nibble pairs: out byte j = (b[2j] & 15) | (b[2j+1] << 4)
      const uint32_t w[4] = {lo8.x, lo8.y, hi8.x, hi8.y};
      uint32_t o[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t x0 = w[2 * h], x1 = w[2 * h + 1];
        const uint32_t e0 = (x0 & 0x0fu) | ((x0 >> 4) & 0xf0u);             // bytes 0,1
        const uint32_t e1 = ((x0 >> 16) & 0x0fu) | ((x0 >> 20) & 0xf0u);   // bytes 2,3
        const uint32_t e2 = (x1 & 0x0fu) | ((x1 >> 4) & 0xf0u);
        const uint32_t e3 = ((x1 >> 16) & 0x0fu) | ((x1 >> 20) & 0xf0u);
        o[h] = e0 | (e1 << 8) | (e2 << 16) | (e3 << 24);
      }
      *reinterpret_cast<uint2*>(a.codes + (size_t)grow * (K / 2) + col / 2) = make_uint2(o[0], o[1]);
    }
  }
}

}  // namespace hbl
