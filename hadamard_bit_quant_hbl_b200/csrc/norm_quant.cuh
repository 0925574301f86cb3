// Fused RMSNorm -> per-token quantisation without a transform (plain BitLinear).
//
// Method: BitNet v2 walkthrough article (m.jxzklqfsx.com), section "BitNet v2：原生4位激活": after
// the second training stage every linear layer except the embeddings runs with INT4 (or INT8)
// activations, and only the attention output and FFN down projections carry the Hadamard
// transform. The other linears (QKV, up/gate) quantise RMS-normalised activations directly. In
// this library that is the block-diagonal transform with blocks of one feature (H_1 = [1]).
//
// The kernel streams rows once: each thread loads up to E features of its row as E/8 16-byte
// vectors (vector v of thread t covers features (v * tpr + t) * 8 .. + 7, so a warp reads 512
// contiguous bytes per vector; vectors past K are skipped), accumulates the sum of squares and the row statistic (max |x g|
// or sum |x g|), and after one reduction over the row rounds its values to codes and stores them
// from registers (8 bytes per vector for int8 codes, 4 for packed int4). The RMS factor only
// rescales the row, so it enters the per-row multiplier and s_x, not the values.
#pragma once

#include "common.cuh"

namespace hbl {

struct NqArgs {
  const uint16_t* X;  // bf16 bits [M][K]
  const float* gain;  // [K] or nullptr
  uint8_t* codes;
  float* s_x;
  int M, K;
  int fmt;            // hbl_codes_fmt
  float eps_norm, eps_q;
  int tpr;            // threads per row: a multiple of 32 with tpr * E >= K
  int rows;           // rows per CTA
};

__device__ __forceinline__ uint4 nq_ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// E features per thread; QM = hbl_quant; G = a gain is given.
template <int E, int QM, bool G>
__global__ void __launch_bounds__(1024) norm_quant_kernel(NqArgs a) {
  static_assert(E % 8 == 0, "whole 16-byte vectors");
  constexpr int NV = E / 8;
  constexpr float kQ = QM == 0 ? 127.f : (QM == 1 ? 2.6457513110645906f : 7.f);
  constexpr int kLo = QM == 0 ? -128 : -8, kHi = QM == 0 ? 127 : 7;
  constexpr bool kAbsmax = QM != 1;
  __shared__ float red_ss[32], red_st[32];

  const int tid = threadIdx.x;
  const int tpr = a.tpr;
  const int rloc = tid / tpr;
  const int tr = tid - rloc * tpr;
  const int lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x * a.rows + rloc;
  const bool live_row = row < a.M;
  const int srow = live_row ? row : a.M - 1;  // rows past M load a live row and store nothing
  const int K = a.K;

  // X may come from the kernel before this one (programmatic dependent launch): wait for it; the
  // product that reads these codes may then launch and stream its weights meanwhile.
  pdl_wait();
  pdl_launch_dependents();

  const int nvec = K >> 3;  // 16-byte vectors per row
  uint4 w[NV];
  const uint16_t* src = a.X + (size_t)srow * K;
#pragma unroll
  for (int vv = 0; vv < NV; ++vv) {
    const int v = vv * tpr + tr;
    w[vv] = v < nvec ? nq_ldg_stream(src + (size_t)v * 8) : make_uint4(0u, 0u, 0u, 0u);
  }

  float f[E];
  float ss0 = 0.f, ss1 = 0.f, st0 = 0.f, st1 = 0.f;
#pragma unroll
  for (int vv = 0; vv < NV; ++vv) {
    const uint32_t u[4] = {w[vv].x, w[vv].y, w[vv].z, w[vv].w};
    float gg[8];
    if constexpr (G) {  // scalar loads: the ABI asks only 4-byte alignment of the gain
      const int v = vv * tpr + tr;
      const float* gp = a.gain + (size_t)(v < nvec ? v : 0) * 8;
#pragma unroll
      for (int j = 0; j < 8; ++j) gg[j] = __ldg(gp + j);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float x0 = __uint_as_float(u[i] << 16), x1 = __uint_as_float(u[i] & 0xffff0000u);
      ss0 = fmaf(x0, x0, ss0);
      ss1 = fmaf(x1, x1, ss1);
      if constexpr (G) {
        x0 *= gg[2 * i];
        x1 *= gg[2 * i + 1];
      }
      if constexpr (kAbsmax) {
        st0 = fmaxf(st0, fabsf(x0));
        st1 = fmaxf(st1, fabsf(x1));
      } else {
        st0 += fabsf(x0);
        st1 += fabsf(x1);
      }
      f[vv * 8 + 2 * i] = x0;
      f[vv * 8 + 2 * i + 1] = x1;
    }
  }
  float ss = ss0 + ss1;
  float st = kAbsmax ? fmaxf(st0, st1) : st0 + st1;

  // ---- row reduction: warp shuffles, then (rows wider than a warp) one pass through shared
  // memory in a fixed order, so that every thread of the row derives the same scalars
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float t = __shfl_xor_sync(0xffffffffu, st, o);
    st = kAbsmax ? fmaxf(st, t) : st + t;
  }
  if (tpr > 32) {
    if (lane == 0) {
      red_ss[warp] = ss;
      red_st[warp] = st;
    }
    __syncthreads();
    const int w0 = (rloc * tpr) >> 5, nw = tpr >> 5;
    ss = 0.f;
    st = 0.f;
    for (int ww = 0; ww < nw; ++ww) {
      ss += red_ss[w0 + ww];
      st = kAbsmax ? fmaxf(st, red_st[w0 + ww]) : st + red_st[w0 + ww];
    }
  }

  // ---- per-row multiplier and scale. x_hat = x g / r; stat(x_hat) = sy / r with sy the
  // statistic of x g. Without eps_q the codes are Q x g / sy (r cancels).
  const float r_rms = sqrtf(ss / (float)K + a.eps_norm);
  const float sy = kAbsmax ? st : st / (float)K;
  float mult = 0.f, sx = 0.f;
  if (sy > 0.f) {
    if (a.eps_q == 0.f) {
      mult = kQ / sy;
      sx = sy / (r_rms * kQ);
    } else {
      const float stat = sy / r_rms;
      mult = kQ / ((stat + a.eps_q) * r_rms);
      sx = stat / kQ;
    }
  }
  if (live_row && tr == 0) a.s_x[row] = sx;
  if (!live_row) return;

  // ---- codes: round to nearest even, clamp, store from registers in natural order
  const bool packed4 = (a.fmt == 0) && (QM != 0);
#pragma unroll
  for (int vv = 0; vv < NV; ++vv) {
    const int v = vv * tpr + tr;
    if (v >= nvec) break;
    int q[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) q[j] = min(max(__float2int_rn(f[vv * 8 + j] * mult), kLo), kHi);
    const size_t k0 = (size_t)v * 8;
    if (packed4) {
      uint32_t o = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) o |= ((uint32_t)q[j] & 0xfu) << (4 * j);
      *reinterpret_cast<uint32_t*>(a.codes + (size_t)row * (K / 2) + k0 / 2) = o;
    } else {
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        lo |= ((uint32_t)q[j] & 0xffu) << (8 * j);
        hi |= ((uint32_t)q[j + 4] & 0xffu) << (8 * j);
      }
      *reinterpret_cast<uint2*>(a.codes + (size_t)row * K + k0) = make_uint2(lo, hi);
    }
  }
}

}  // namespace hbl
