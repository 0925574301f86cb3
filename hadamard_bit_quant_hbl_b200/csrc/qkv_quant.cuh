// QKV states after RoPE, quantised per head to unsigned b-bit integers with an absmax scale (the
// low-bit attention states and 3-bit KV cache of BitNet v2), and the matching dequantisation.
//
// Method: BitNet v2 walkthrough article (m.jxzklqfsx.com), section "實驗結果" (Tables 2-3): the
// QKV states are quantised after RoPE; each head goes directly to unsigned integers through the
// absmax function, with no calibration data. The formulas were not preserved, so this follows the
// plainest reading: per token and head, gamma = max|x| over the head's D features, and
// [-gamma, gamma] maps linearly onto [0, 2^b - 1] (L = 2^b - 1):
//     u = RoundClip(L (x + gamma) / (2 gamma), 0, L),   x~ = (2u - L) gamma / L.
// RoPE is the LLaMA form of the model's LLaMA-like parts ("BitNet v2：原生4位激活"): feature f of a
// head pairs with f + D/2 and both turn by the angle pos * theta^(-2f/D).
//
// Layout: one CTA per kQkvTokens tokens. Its threads first build the cos/sin table of those
// tokens' D/2 angles in shared memory together (angle formed and reduced modulo 2 pi in fp64, then
// rounded to fp32; one barrier), then each warp takes (token, head) pairs in turn: lane l holds
// features l*E .. l*E+E-1 (E = D/32), whose RoPE partners sit in lane l ^ 16. Codes leave as a
// little-endian bit string per head (code j at bits [b j, b j + b)), each group of 8 codes
// (b bytes) assembled across the lanes that hold it.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace hbl {

constexpr int kQkvTokens = 4;  // tokens per CTA

// Code of one value: u = RoundClip(L (x + gamma) / (2 gamma), 0, L) with mult = (L/2) / gamma.
// t = x mult + L/2 lies in [0, L] up to rounding (|x| <= gamma), so its nearest integer needs no
// clamp; adding 1.5 * 2^23 rounds it (ties to even) into the low mantissa bits, which are the
// code. Only where t lands within 2^-12 of a .5 boundary is the value formed again in fp64 as
// (L x + L gamma) / (2 gamma), which is exact for bf16 inputs (so that a value exactly on a
// boundary goes to the even code) and is the expression a float64 evaluation of the reading uses.
template <int BITS>
__device__ __forceinline__ uint32_t unsigned_code(float x, float g, float mult) {
  constexpr float kL = (float)((1 << BITS) - 1);
  constexpr float kMagic = 12582912.f;  // 1.5 * 2^23
  const float t = fmaf(x, mult, 0.5f * kL);
  const float y = t + kMagic;
  uint32_t q = __float_as_uint(y) & 0xffu;
  if (fabsf(t - (y - kMagic)) > 0.5f - 2.44140625e-4f) {  // within 2^-12 of a boundary
    const double L = (double)kL, xd = (double)x, gd = (double)g;
    const double u = gd > 0.0 ? rint((L * xd + L * gd) / (2.0 * gd)) : rint(0.5 * (double)kL);
    q = (uint32_t)fmin(fmax(u, 0.0), (double)kL);
  }
  return q;
}

struct QkvArgs {
  const uint16_t* X;  // bf16; token m, head h at X + m * row_stride + h * D
  size_t row_stride;  // elements between consecutive tokens
  const int32_t* pos; // [M] token positions, or nullptr: no RoPE (the V states)
  float theta;
  uint8_t* codes;     // [M][H][D * bits / 8]
  float* gamma;       // [M][H]
  int M, H;
};

template <int E>
__device__ __forceinline__ void qkv_load(const uint16_t* p, float (&v)[E]) {
  if constexpr (E == 2) {
    const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
    v[0] = __uint_as_float(u << 16);
    v[1] = __uint_as_float(u & 0xffff0000u);
  } else if constexpr (E == 4) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
}

// Stores the GB bytes of a code group (GB = bits) at p.
template <int GB>
__device__ __forceinline__ void qkv_store_group(uint8_t* p, uint64_t g) {
  if constexpr (GB == 8) {
    *reinterpret_cast<uint2*>(p) = make_uint2((uint32_t)g, (uint32_t)(g >> 32));
  } else if constexpr (GB == 4) {
    *reinterpret_cast<uint32_t*>(p) = (uint32_t)g;
  } else if constexpr (GB == 2) {
    *reinterpret_cast<uint16_t*>(p) = (uint16_t)g;
  } else {
#pragma unroll
    for (int i = 0; i < GB; ++i) p[i] = (uint8_t)(g >> (8 * i));
  }
}

template <int E, int BITS, bool ROPE>
__global__ void __launch_bounds__(256) qkv_quant_kernel(QkvArgs a) {
  static_assert(E == 2 || E == 4 || E == 8, "head size 64, 128 or 256");
  constexpr int D = 32 * E, HALF = D / 2;
  constexpr float kL = (float)((1 << BITS) - 1);
  constexpr int LPG = 8 / E;  // lanes holding one group of 8 codes
  constexpr int HEAD_BYTES = D * BITS / 8;
  __shared__ float cs[kQkvTokens][HALF], sin_tab[kQkvTokens][HALF];

  const int m0 = blockIdx.x * kQkvTokens;
  const int nt = a.M - m0 < kQkvTokens ? a.M - m0 : kQkvTokens;
  // X may come from the kernel before this one (programmatic dependent launch)
  pdl_wait();
  pdl_launch_dependents();
  if constexpr (ROPE) {
    const double two_pi = 6.283185307179586476925;
    const double lt = log((double)a.theta);
    for (int e = threadIdx.x; e < nt * HALF; e += blockDim.x) {
      const int t = e / HALF, f = e - t * HALF;
      const double ang = (double)a.pos[m0 + t] * exp(-2.0 * (double)f / (double)D * lt);
      const double r = ang - two_pi * rint(ang / two_pi);
      double s, c;
      sincos(r, &s, &c);
      cs[t][f] = (float)c;
      sin_tab[t][f] = (float)s;
    }
    __syncthreads();
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  // codes of a group of 8 fit 32 bits up to 4 bits per code
  using Bits = typename std::conditional<(8 * BITS <= 32), uint32_t, unsigned long long>::type;
  const bool first = lane < 16;
  for (int t = 0; t < nt; ++t) {
    const int m = m0 + t;
    // this lane's angles for the token, the same for every head; the first half of a head turns
    // by -sin against its partner, the second by +sin: x' = x c + partner s' with s' = -+ sin
    float c[E], sn[E];
    if constexpr (ROPE) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int f = (lane & 15) * E + e;
        c[e] = cs[t][f];
        sn[e] = first ? -sin_tab[t][f] : sin_tab[t][f];
      }
    }
    // up to four heads of this warp in flight: every load issued before the first is used
    for (int h0 = warp; h0 < a.H; h0 += 4 * nwarps) {
      float v[4][E];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int h = h0 + i * nwarps;
        if (h < a.H) qkv_load<E>(a.X + (size_t)m * a.row_stride + (size_t)h * D + lane * E, v[i]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int h = h0 + i * nwarps;
        if (h >= a.H) break;  // the same in every lane
        if constexpr (ROPE) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float partner = __shfl_xor_sync(0xffffffffu, v[i][e], 16);
            v[i][e] = fmaf(partner, sn[e], v[i][e] * c[e]);
          }
        }
        float g = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) g = fmaxf(g, fabsf(v[i][e]));
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
        const float mult = g > 0.f ? 0.5f * kL / g : 0.f;
        Bits bits = 0;
#pragma unroll
        for (int e = 0; e < E; ++e)
          bits |= (Bits)unsigned_code<BITS>(v[i][e], g, mult) << (((lane % LPG) * E + e) * BITS);
#pragma unroll
        for (int o = 1; o < LPG; o <<= 1) bits |= __shfl_xor_sync(0xffffffffu, bits, o);
        const size_t mh = (size_t)m * a.H + h;
        if (lane % LPG == 0)
          qkv_store_group<BITS>(a.codes + mh * HEAD_BYTES + (lane / LPG) * BITS, (uint64_t)bits);
        if (lane == 0) a.gamma[mh] = g;
      }
    }
  }
}

// x~ = (2u - (2^b - 1)) * gamma / (2^b - 1) as bf16 [M][H][D]: one warp per head, lane l
// producing features l*E .. l*E+E-1.
template <int E, int BITS>
__global__ void __launch_bounds__(256) qkv_dequant_kernel(const uint8_t* __restrict__ codes,
                                                          const float* __restrict__ gamma, int M, int H,
                                                          uint16_t* __restrict__ Y) {
  constexpr int D = 32 * E;
  constexpr int HEAD_BYTES = D * BITS / 8;
  constexpr float kL = (float)((1 << BITS) - 1);
  const int lane = threadIdx.x & 31;
  const size_t mh = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (mh >= (size_t)M * H) return;
  const uint8_t* hp = codes + mh * HEAD_BYTES;
  const int b0 = lane * E * BITS;
  const int byte0 = b0 >> 3, shift = b0 & 7;
  const int nbytes = (shift + E * BITS + 7) >> 3;
  uint64_t w = 0;
  for (int i = 0; i < nbytes; ++i) w |= (uint64_t)hp[byte0 + i] << (8 * i);
  w >>= shift;
  const float step = gamma[mh] / kL;
  uint16_t* out = Y + mh * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float u = (float)((w >> (e * BITS)) & ((1u << BITS) - 1u));
    const float x = (2.f * u - kL) * step;
    // round to nearest even bf16
    const uint32_t xb = __float_as_uint(x);
    out[e] = (uint16_t)((xb + 0x7fffu + ((xb >> 16) & 1u)) >> 16);
  }
}

}  // namespace hbl
