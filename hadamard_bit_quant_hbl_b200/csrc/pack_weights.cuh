// Offline weight preparation: per-tensor absmean ternarisation and packing.
//
// Method: BitNet v2 walkthrough article (m.jxzklqfsx.com), section "H-BitLinear模塊" (weights
// ternarised to {-1, 0, 1} with a per-tensor absmean scale) and the bitnet.cpp news article
// (gubiw.cn), section "6 页论文，引入 1 bit LLM" (divide the weight matrix by its mean
// absolute value, round each entry to the nearest of -1, 0, 1).
//
// alpha is reduced in fp64 in a fixed order (per-block partial sums, then one block sums the
// partials), so the result does not depend on scheduling. The rounding decision
// rint(W / (alpha + eps)) is also taken in fp64.
#pragma once

#include "common.cuh"

namespace hbl {

constexpr int kAbsumBlocks = 4 * 148;
constexpr int kAbsumThreads = 256;

// Fixed-order tree reduction of one double per thread of a 256-thread block.
__device__ __forceinline__ double block_sum_256(double v, double* sh) {
  sh[threadIdx.x] = v;
  __syncthreads();
#pragma unroll
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) sh[threadIdx.x] += sh[threadIdx.x + s];
    __syncthreads();
  }
  return sh[0];
}

__global__ void __launch_bounds__(kAbsumThreads) absum_partial_kernel(const float* __restrict__ W,
                                                                      size_t count4,
                                                                      double* __restrict__ partials) {
  __shared__ double sh[kAbsumThreads];
  double acc = 0.0;
  const float4* W4 = reinterpret_cast<const float4*>(W);
  for (size_t i = (size_t)blockIdx.x * kAbsumThreads + threadIdx.x; i < count4;
       i += (size_t)gridDim.x * kAbsumThreads) {
    const float4 w = __ldg(W4 + i);
    acc += (double)fabsf(w.x) + (double)fabsf(w.y) + (double)fabsf(w.z) + (double)fabsf(w.w);
  }
  const double s = block_sum_256(acc, sh);
  if (threadIdx.x == 0) partials[blockIdx.x] = s;
}

__global__ void __launch_bounds__(kAbsumThreads) absum_final_kernel(const double* __restrict__ partials,
                                                                    int nparts, double count,
                                                                    double* __restrict__ alpha_out) {
  __shared__ double sh[kAbsumThreads];
  double acc = 0.0;
  for (int i = threadIdx.x; i < nparts; i += kAbsumThreads) acc += partials[i];
  const double s = block_sum_256(acc, sh);
  if (threadIdx.x == 0) alpha_out[0] = s / count;
}

// One thread per (column n, 16-row group w): 16 ternary codes t[16w .. 16w+15][n].
// Lanes take consecutive n, so every read of a W row segment is coalesced.
//   section 0: uint32 word (n, w), code t+1 of k = 16w + 4s + b at bits 8b + 2s, stored
//              tile-major: word (n, w) at ((n/128) * (K/128) + w/8) * 1024 + (n%128) * 8 + w%8,
//              so that one 128-feature x 128-k tile is 4 KB of contiguous memory. Rows of the
//              last tile beyond N are filled with t = 0.
//   section 1: int8 t[k][n] at n*K + k
//   section 2: int32 column sum (atomic, integer: order-independent)
template <bool FROM_CODES>
__global__ void __launch_bounds__(128) ternarize_pack_kernel(const float* __restrict__ W,
                                                             const int8_t* __restrict__ T, int K, int N,
                                                             const double* __restrict__ alpha_d,
                                                             double eps_w, uint32_t* __restrict__ sec0,
                                                             int8_t* __restrict__ sec1,
                                                             int32_t* __restrict__ sec2) {
  const int n = blockIdx.x * 128 + threadIdx.x;
  const int w = blockIdx.y;
  const size_t w2idx = ((size_t)(n >> 7) * (K >> 7) + (w >> 3)) * 1024 + (size_t)(n & 127) * 8 + (w & 7);
  if (n >= N) {  // padding rows of the last 128-feature tile (section 0 only)
    sec0[w2idx] = 0x55555555u;
    return;
  }
  int t[16];
  if constexpr (FROM_CODES) {
    bool bad = false;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      int v = T[(size_t)(16 * w + j) * N + n];
      if (v < -1 || v > 1) {
        bad = true;
        v = v < -1 ? -1 : 1;
      }
      t[j] = v;
    }
    if (bad) raise_error(kErrBadTernary);
  } else {
    const double denom = alpha_d[0] + eps_w;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const double x = (double)W[(size_t)(16 * w + j) * N + n];
      double q = denom > 0.0 ? rint(x / denom) : 0.0;
      q = q < -1.0 ? -1.0 : (q > 1.0 ? 1.0 : q);
      t[j] = (int)q;
    }
  }
  uint32_t word = 0;
  int colsum = 0;
  uint32_t b4[4];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int s = j >> 2, b = j & 3;  // k = 16w + 4s + b
    word |= (uint32_t)(t[j] + 1) << (8 * b + 2 * s);
    colsum += t[j];
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    b4[q] = ((uint32_t)(uint8_t)(int8_t)t[4 * q]) | ((uint32_t)(uint8_t)(int8_t)t[4 * q + 1] << 8) |
            ((uint32_t)(uint8_t)(int8_t)t[4 * q + 2] << 16) | ((uint32_t)(uint8_t)(int8_t)t[4 * q + 3] << 24);
  }
  sec0[w2idx] = word;
  *reinterpret_cast<uint4*>(sec1 + (size_t)n * K + 16 * w) = make_uint4(b4[0], b4[1], b4[2], b4[3]);
  atomicAdd(sec2 + n, colsum);
}

// ---------------------------------------------------------------- weight-side rotation

// One pass of the orthonormal Walsh-Hadamard transform along k, over index bits [b0, b0 + NB),
// of every column of a row-major fp32 matrix [K][N] (the variant with rotated weights and
// activations of the walkthrough article's Table 5 ablation: W' = H W along the reduction
// dimension, before ternarisation). A CTA holds the 2^NB rows k = hi * 2^(b0+NB) + j * 2^b0 + lo
// (j = 0 .. 2^NB - 1; hi, lo fixed per CTA) of 32 consecutive columns in shared memory, runs the
// NB butterfly stages (a, b) -> (a + b, a - b) of pairs j, j + h, and writes the rows back times
// `scale`. Every CTA reads and writes only its own elements, so src may equal dst. K must be a
// multiple of 2^(b0+NB).
template <int NB>
__global__ void __launch_bounds__(256) fht_cols_kernel(const float* src, float* dst, int K, int N, int b0,
                                                       float scale) {
  constexpr int R = 1 << NB;
  __shared__ float tile[R][33];
  const int c = threadIdx.x & 31;
  const int col = blockIdx.x * 32 + c;
  const bool live = col < N;
  const size_t g = blockIdx.y;
  const size_t lo = g & ((1u << b0) - 1u), hi = g >> b0;
  const size_t kbase = (hi << (b0 + NB)) + lo;
  for (int j = threadIdx.x >> 5; j < R; j += 8)
    tile[j][c] = live ? src[(kbase + ((size_t)j << b0)) * (size_t)N + col] : 0.f;
  __syncthreads();
#pragma unroll
  for (int h = 1; h < R; h <<= 1) {
    for (int p = threadIdx.x; p < (R / 2) * 32; p += 256) {
      const int cc = p & 31, bi = p >> 5;
      const int j0 = (bi / h) * 2 * h + (bi % h);
      const float a = tile[j0][cc], b = tile[j0 + h][cc];
      tile[j0][cc] = a + b;
      tile[j0 + h][cc] = a - b;
    }
    __syncthreads();
  }
  if (!live) return;
  for (int j = threadIdx.x >> 5; j < R; j += 8) dst[(kbase + ((size_t)j << b0)) * (size_t)N + col] = tile[j][c] * scale;
}

}  // namespace hbl
