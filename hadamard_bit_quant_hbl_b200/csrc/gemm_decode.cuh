// Ternary x low-bit product for small token counts (decode) on CUDA cores.
//
//   Y[m, n] = s_x[m] * alpha * sum_k q[m, k] * t[k, n]
//
// The layer's product (BitNet v2 walkthrough article, section "H-BitLinear模塊": quantised
// activations times ternary weights, both scales applied afterwards). At a few tokens the
// product is bound by the weight bytes, so the weights are streamed in their 2-bit form
// (section 0 of the packed blob: c = t + 1 in {0,1,2}) at one 16-byte vector per thread, and
// each 2-bit group is widened with one shift and one mask into four unsigned bytes that feed
// __dp4a against int8 activations held in registers:
//   sum_k q t = sum_k q c - sum_k q.
// The activation slice of a thread (64 features x MT tokens) is loaded once and reused for all
// columns of the CTA; every thread owns a different 64-feature slice of K, and the per-column
// partial sums are reduced across the CTA in a fixed order (warp shuffles, then shared memory),
// so results are bit-reproducible. Integer sums are exact.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace hbl {

struct DecodeArgs {
  const uint8_t* codes;  // activation codes: int8 [M][K] or packed int4 [M][K/2]
  int m0;                // first token row handled by this launch (rows m0 .. m0+MT-1)
  int packed4;           // 1 = packed int4 rows
  const float* s_x;
  const uint32_t* w2;    // section 0: tile-major 2-bit words (see the packer)
  float alpha;
  int M, N, K;
  void* Y;
  int out_bf16;
  int32_t* acc_debug;
};

// Sign-extend 8 two's-complement nibbles (element 2j in the low nibble of byte j) to int8,
// natural order: returns bytes of elements 0..3 in lo, 4..7 in hi.
__device__ __forceinline__ void widen_int4x8(uint32_t x, uint32_t& lo, uint32_t& hi) {
  // (u ^ 8) + 0x78 maps the nibble u of q (two's complement) to q + 128 without carries between
  // bytes; xor 0x80 turns q + 128 into the int8 bit pattern of q.
  const uint32_t ev = (((x & 0x0f0f0f0fu) ^ 0x08080808u) + 0x78787878u) ^ 0x80808080u;         // e0 e2 e4 e6
  const uint32_t od = ((((x >> 4) & 0x0f0f0f0fu) ^ 0x08080808u) + 0x78787878u) ^ 0x80808080u;  // e1 e3 e5 e7
  lo = __byte_perm(ev, od, 0x5140);
  hi = __byte_perm(ev, od, 0x7362);
}

template <int MT, int COLS>
__global__ void __launch_bounds__(512) gemm_decode_kernel(const DecodeArgs a) {
  // thread t owns the 64-feature unit t (blockDim = K/64 rounded up to a warp, <= 512)
  const int t = threadIdx.x;
  const int units = a.K / 64;
  const bool live = t < units;
  const int lane = t & 31, warp = t >> 5, nwarps = blockDim.x >> 5;
  __shared__ int red[COLS * MT + MT][16];  // up to 16 warps (K <= 32768)

  // activation slice: 16 int8x4 words per token row
  int act[MT][16];
  int qsum[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    qsum[m] = 0;
    if (live && a.m0 + m < a.M) {
      if (a.packed4) {
        const uint4* p = reinterpret_cast<const uint4*>(a.codes + (size_t)(a.m0 + m) * (a.K / 2) + (size_t)t * 32);
        const uint4 v0 = __ldg(p), v1 = __ldg(p + 1);
        const uint32_t x[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint32_t lo, hi;
          widen_int4x8(x[i], lo, hi);
          act[m][2 * i] = (int)lo;
          act[m][2 * i + 1] = (int)hi;
        }
      } else {
        const uint4* p = reinterpret_cast<const uint4*>(a.codes + (size_t)(a.m0 + m) * a.K + (size_t)t * 64);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = __ldg(p + i);
          act[m][4 * i] = (int)v.x;
          act[m][4 * i + 1] = (int)v.y;
          act[m][4 * i + 2] = (int)v.z;
          act[m][4 * i + 3] = (int)v.w;
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) qsum[m] = __dp4a(act[m][i], 0x01010101, qsum[m]);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) act[m][i] = 0;
    }
  }

  const int n0 = blockIdx.x * COLS;
  int acc[COLS][MT];
#pragma unroll
  for (int c = 0; c < COLS; ++c) {
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[c][m] = 0;
  }
  if (live) {
    // issue every column's 16-byte weight load first (bytes in flight), then compute
    uint4 wv[COLS];
#pragma unroll
    for (int c = 0; c < COLS; ++c) {
      const int n = n0 + c;
      // words 4t .. 4t+3 of row n: k-block t/2, half t%2 of the row's 8 words in that block
      const size_t wi = ((size_t)(n >> 7) * (a.K >> 7) + (t >> 1)) * 1024 + (size_t)(n & 127) * 8 + (t & 1) * 4;
      wv[c] = n < a.N ? __ldcs(reinterpret_cast<const uint4*>(a.w2 + wi))
                      : make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);  // t = 0
    }
#pragma unroll
    for (int c = 0; c < COLS; ++c) {
      const uint32_t ww[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {  // 16 features k = 64t + 16i + 4s + b
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const int cw = (int)((ww[i] >> (2 * s)) & 0x03030303u);
#pragma unroll
          for (int m = 0; m < MT; ++m) acc[c][m] = __dp4a(act[m][4 * i + s], cw, acc[c][m]);
        }
      }
    }
  }

  // reduce over the CTA: warp shuffles, then fixed-order sum of the warp partials
#pragma unroll
  for (int c = 0; c < COLS; ++c) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      int v = acc[c][m];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[c * MT + m][warp] = v;
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    int v = qsum[m];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[COLS * MT + m][warp] = v;
  }
  __syncthreads();
  if (t < COLS * MT) {
    const int c = t / MT, ml = t - (t / MT) * MT;
    const int n = n0 + c, m = a.m0 + ml;
    if (n < a.N && m < a.M) {
      int s = 0, q = 0;
      for (int w = 0; w < nwarps; ++w) {
        s += red[c * MT + ml][w];
        q += red[COLS * MT + ml][w];
      }
      const int accv = s - q;
      const float y = (float)accv * (a.s_x[m] * a.alpha);
      if (a.out_bf16) reinterpret_cast<__nv_bfloat16*>(a.Y)[(size_t)m * a.N + n] = __float2bfloat16_rn(y);
      else reinterpret_cast<float*>(a.Y)[(size_t)m * a.N + n] = y;
      if (a.acc_debug) a.acc_debug[(size_t)m * a.N + n] = accv;
    }
  }
}

}  // namespace hbl
