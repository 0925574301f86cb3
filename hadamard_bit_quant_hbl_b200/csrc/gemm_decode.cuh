// Ternary x low-bit product for a few tokens (decode) on CUDA cores.
//
//   Y[m, n] = s_x[m] * alpha * sum_k q[m, k] * t[k, n]
//
// The layer's product (BitNet v2 walkthrough article, section "H-BitLinear模塊": quantised
// activations times ternary weights, both scales applied afterwards). At a few tokens the
// product is bound by the weight bytes, so the weights are streamed in their 2-bit form
// (section 0 of the packed blob, c = t + 1 in {0,1,2}, tile-major: one 128-feature x 128-k tile
// is 4 KB of contiguous memory) and every byte is read once, with coalesced 16-byte loads.
//
// A cluster of S CTAs shares one 128-feature tile and splits K: CTA r owns a contiguous run of
// k-blocks. Within a k-block, thread t owns feature t/2 and half t%2 of the block (64 k, one
// 16-byte load; the 256 threads read the 4 KB tile in order). Two chunks of k-blocks are in
// flight per thread (double buffering in registers), the first two issued before anything else.
// A 2-bit group is widened with a shift and a mask into four unsigned bytes c that feed __dp4a
// against int8 activations staged in shared memory:  sum_k q t = sum_k q c - sum_k q.
// The two halves of a feature meet in a warp shuffle; the cluster's partial sums meet in
// distributed shared memory (fixed order), so results are exact and reproducible and no global
// workspace is needed.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace hbl {

constexpr int kDecThreads = 256;

// k-blocks per chunk of weight loads (two chunks in flight); fewer when many token rows hold
// registers
constexpr int dec_unroll(int MT) { return MT >= 8 ? 4 : 8; }

struct DecodeArgs {
  const uint8_t* codes;  // activation codes: int8 [M][K] or packed int4 [M][K/2]
  int m0;                // first token row handled by this launch (rows m0 .. m0+MT-1)
  int packed4;           // 1 = packed int4 rows
  const float* s_x;
  const uint32_t* w2;    // section 0: tile-major 2-bit words
  float alpha;
  int M, N, K;
  int S;                 // CTAs per cluster (k split)
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

__device__ __forceinline__ uint4 ldg_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Shared memory: the partial sums [MT][128] int32 (first, at the same offset in every CTA of the
// cluster: peers read them there), then int8 activations [MT][range] (range = this CTA's k count).
template <int MT>
__global__ void __launch_bounds__(kDecThreads, 2) gemm_decode_kernel(const DecodeArgs a) {
  constexpr int U = dec_unroll(MT);
  extern __shared__ __align__(16) uint8_t dec_smem[];
  __shared__ int32_t qred[MT][kDecThreads / 32];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.S;
  const uint32_t rank = cluster_ctarank();
  const int tile = blockIdx.x / S;
  const int n0 = tile * 128;
  const int KB = a.K >> 7;
  const int kb0 = (int)(((long)KB * rank) / S), kb1 = (int)(((long)KB * (rank + 1)) / S);
  const int nkb = kb1 - kb0;
  const int range = nkb * 128;
  int32_t* part = reinterpret_cast<int32_t*>(dec_smem);
  int8_t* act = reinterpret_cast<int8_t*>(dec_smem + MT * 128 * 4);

  // ---- thread = (feature f, half h) of each k-block. Weight loads go out first (they need
  // nothing else), two chunks of U k-blocks in flight while the activations are staged.
  const int f = tid >> 1, h = tid & 1;
  const uint32_t* wt = a.w2 + ((size_t)tile * KB + kb0) * 1024 + f * 8 + 4 * h;
  auto load_chunk = [&](uint4 (&w)[U], int i0) {
#pragma unroll
    for (int u = 0; u < U; ++u)
      w[u] = (i0 + u < nkb) ? ldg_stream_u4(wt + (size_t)(i0 + u) * 1024) : make_uint4(0u, 0u, 0u, 0u);
  };
  uint4 wa[U], wb[U];
  load_chunk(wa, 0);
  load_chunk(wb, U);

  // ---- stage this CTA's activations (16 codes per step) and their per-token sums
  int qs[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) qs[m] = 0;
  for (int e = tid * 16; e < MT * range; e += kDecThreads * 16) {
    const int m = e / range, kk = e - m * range;
    const int row = a.m0 + m;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row < a.M) {
      const size_t k = (size_t)kb0 * 128 + kk;
      if (a.packed4) {
        const uint2 p = __ldg(reinterpret_cast<const uint2*>(a.codes + (size_t)row * (a.K / 2) + k / 2));
        widen_int4x8(p.x, v.x, v.y);
        widen_int4x8(p.y, v.z, v.w);
      } else {
        v = __ldg(reinterpret_cast<const uint4*>(a.codes + (size_t)row * a.K + k));
      }
    }
    *reinterpret_cast<uint4*>(act + e) = v;
    int s = 0;
    s = __dp4a((int)v.x, 0x01010101, s);
    s = __dp4a((int)v.y, 0x01010101, s);
    s = __dp4a((int)v.z, 0x01010101, s);
    s = __dp4a((int)v.w, 0x01010101, s);
#pragma unroll
    for (int mm = 0; mm < MT; ++mm)
      if (mm == m) qs[mm] += s;
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    int v = qs[m];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) qred[m][warp] = v;
  }
  __syncthreads();

  // ---- widen and multiply, one chunk while the next one's loads are in flight
  const int8_t* ab = act + 64 * h;
  int acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0;
  auto compute_chunk = [&](const uint4 (&w)[U], int i0) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (i0 + u < nkb) {
        const uint32_t ww[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
        const int8_t* ak = ab + (i0 + u) * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // word i: 16 features k = 64h + 16i + 4s + b
          uint4 q[MT];
#pragma unroll
          for (int m = 0; m < MT; ++m) q[m] = *reinterpret_cast<const uint4*>(ak + (size_t)m * range + 16 * i);
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const int cw = (int)((ww[i] >> (2 * s)) & 0x03030303u);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const uint32_t qw = s == 0 ? q[m].x : s == 1 ? q[m].y : s == 2 ? q[m].z : q[m].w;
              acc[m] = __dp4a((int)qw, cw, acc[m]);
            }
          }
        }
      }
    }
  };
  for (int i0 = 0; i0 < nkb; i0 += 2 * U) {
    compute_chunk(wa, i0);
    if (i0 + 2 * U < nkb) load_chunk(wa, i0 + 2 * U);
    if (i0 + U < nkb) compute_chunk(wb, i0 + U);
    if (i0 + 3 * U < nkb) load_chunk(wb, i0 + 3 * U);
  }

  // ---- the two halves of a feature, minus this CTA's sum of q, into shared memory
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], 1);
    if (h == 0) {
      int qsum = 0;
#pragma unroll
      for (int w = 0; w < kDecThreads / 32; ++w) qsum += qred[m][w];
      part[m * 128 + f] = acc[m] - qsum;
    }
  }
  cluster_sync_all();

  // ---- reduce across the cluster (fixed order), dequant, store
  const uint32_t part0 = smem_u32(part);
  for (int e = (int)rank * kDecThreads + tid; e < MT * 128; e += S * kDecThreads) {
    const int m = e >> 7, fl = e & 127;
    const int n = n0 + fl, row = a.m0 + m;
    if (row >= a.M || n >= a.N) continue;
    uint32_t pv[8];
#pragma unroll
    for (int p = 0; p < 8; ++p)  // all remote loads in flight before the sum
      pv[p] = p < S ? ld_shared_cluster_u32(mapa_shared(part0 + (uint32_t)e * 4u, (uint32_t)p)) : 0u;
    int32_t accv = 0;
#pragma unroll
    for (int p = 0; p < 8; ++p) accv += (int32_t)pv[p];
    const float y = (float)accv * (a.s_x[row] * a.alpha);
    if (a.out_bf16) reinterpret_cast<__nv_bfloat16*>(a.Y)[(size_t)row * a.N + n] = __float2bfloat16_rn(y);
    else reinterpret_cast<float*>(a.Y)[(size_t)row * a.N + n] = y;
    if (a.acc_debug) a.acc_debug[(size_t)row * a.N + n] = accv;
  }
  cluster_sync_all();  // no CTA leaves while a peer may still read its shared memory
}

}  // namespace hbl
