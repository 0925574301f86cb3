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
// k-blocks, which the TMA engine streams into a ring of shared-memory stages (16 KB bulk copies,
// completion on mbarriers, every wait bounded); per-thread global loads could not keep enough
// bytes in flight. Within a k-block, thread t owns feature t/2 and half t%2 of the block (64 k,
// one conflict-free 16-byte shared load). A word holds 16 codes, c of k = 16w + 4s + b at bits
// 8b + 2s; masking plane s in place leaves bytes c * 4^s, which feed __dp4a (unsigned x signed)
// against the int8 activations of k-group s staged in shared memory, one accumulator per plane;
// the planes recombine exactly as acc0 + acc1 / 4 + acc2 / 16 + acc3 / 64, and
//   sum_k q t = sum_k q c - sum_k q.
// The kernel may start while the activation kernel before it still runs (programmatic
// dependent launch): it issues its weight copies first and waits for that kernel only before
// it reads the codes. The two halves of a feature meet in a warp shuffle; each CTA
// then stores its partial sums straight into the shared memory of the CTA that owns the feature
// (one slot per peer), so that one cluster barrier suffices and each owner sums its slots in a
// fixed order: results are exact and reproducible, and no global workspace is needed.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace hbl {

constexpr int kDecThreads = 256;

struct DecodeArgs {
  const uint8_t* codes;  // activation codes: int8 [M][K] or packed int4 [M][K/2] (product only)
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
  // the fused forward (the activation side computed in the kernel; codes and s_x unused)
  const uint16_t* X;     // bf16 [M][K]
  const float* gain;     // [K] or nullptr
  int hb;                // transform block: a power of two dividing K, or 1 (no transform)
  int quant;             // hbl_quant
  float eps_norm, eps_q;
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

// Dot product of four unsigned bytes of a with four signed bytes of b, plus c.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Shared memory: the peers' partial sums [S][MT][FO] int32 for the FO features this CTA owns
// (first, at the same offset in every CTA of the cluster: peers write them there), then the
// weight ring [kDecStages][kDecChunk * 4 KB], then int8 activations [MT][range] (range = this
// CTA's k count). CTA r owns features [r * FO, (r + 1) * FO) of the tile, FO = ceil(128 / S).
__host__ __device__ constexpr int dec_slot_bytes(int S, int MT) { return (int)round_up((size_t)S * MT * ((128 + S - 1) / S) * 4, 16); }
constexpr int kDecChunk = 4;   // k-blocks per bulk copy (16 KB)
constexpr int kDecStages = 4;  // copies in flight
constexpr int kDecRingBytes = kDecStages * kDecChunk * 4096;

// The fused forward's activation side for this CTA's slice of K (FUSED kernels only): RMSNorm,
// the Hadamard transform, per-token quantisation, as in the activation kernels, but computed
// where the product needs it, so the codes never leave the SM.
//   Slice r of a row is features [r range, (r + 1) range), range = K / S a power of two. When the
//   transform block hb spans several slices (hb = G range), index bits above the slice are
//   stage-able first (the stages commute): slice r of (H_G (x) I) x is the signed sum
//   sum_j (-1)^popcount((r mod G) & j) x_{slice j of r's group}, read straight from global memory
//   (L2) by every CTA of the group. The in-slice stages then run on 8-value registers and in
//   shared memory. The row statistics (sum x^2 over the row, max or sum |y|) are reduced over the
//   cluster through distributed shared memory, in rank order in every CTA, so every CTA derives
//   the same scalars.
template <int MT>
__device__ __forceinline__ void decode_fused_codes(const DecodeArgs& a, int range, int rank, float* work,
                                                   int8_t* act, float (*stat_in)[MT][2], float* sx_out,
                                                   int (&qs)[MT], float (*red)[kDecThreads / 32][2]) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.S, K = a.K, hb = a.hb;
  const int G = hb > range ? hb / range : 1;  // slices per transform block
  const int rlow = rank & (G - 1), rbase = rank - rlow;
  const int nvec = range >> 3;
  const bool absmax = a.quant != 1;
  // ---- gather (with the stages across slices), 8 values per vector, the first 3 in-block stages.
  // Rows go in pairs, and every load of a pair is issued before the first is used (one L2 latency
  // per pair rather than one per slice).
  float ss[MT], st[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) ss[m] = st[m] = 0.f;
  constexpr int RP = MT < 2 ? MT : 2;
#pragma unroll
  for (int mp = 0; mp < MT; mp += RP) {
    for (int v = tid; v < nvec; v += kDecThreads) {
      uint4 u[RP][8];
#pragma unroll
      for (int mm = 0; mm < RP; ++mm) {
        const int row = a.m0 + mp + mm;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          u[mm][j] = (j < G && row < a.M)
                         ? __ldg(reinterpret_cast<const uint4*>(a.X + (size_t)row * K + (size_t)(rbase + j) * range + 8 * v))
                         : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int mm = 0; mm < RP; ++mm) {
        const int m = mp + mm;
        float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j >= G) break;
          const uint32_t w[4] = {u[mm][j].x, u[mm][j].y, u[mm][j].z, u[mm][j].w};
          const bool neg = (__popc(rlow & j) & 1) != 0;
          const size_t k0 = (size_t)(rbase + j) * range + 8 * v;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float x0 = __uint_as_float(w[i] << 16), x1 = __uint_as_float(w[i] & 0xffff0000u);
            if (j == rlow) ss[m] = fmaf(x0, x0, fmaf(x1, x1, ss[m]));
            if (a.gain) {
              x0 *= __ldg(a.gain + k0 + 2 * i);
              x1 *= __ldg(a.gain + k0 + 2 * i + 1);
            }
            y[2 * i] += neg ? -x0 : x0;
            y[2 * i + 1] += neg ? -x1 : x1;
          }
        }
        if (hb >= 8) {
#pragma unroll
          for (int h = 1; h < 8; h <<= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if ((e & h) == 0) {
                const float p = y[e], q = y[e + h];
                y[e] = p + q;
                y[e + h] = p - q;
              }
        }
        float4* dst = reinterpret_cast<float4*>(work + (size_t)m * range + 8 * v);
        dst[0] = make_float4(y[0], y[1], y[2], y[3]);
        dst[1] = make_float4(y[4], y[5], y[6], y[7]);
      }
    }
  }
  __syncthreads();
  // ---- the remaining in-slice stages (index bits 3 .. lb - 1, lb = log2(min(hb, range))) in
  // shared memory, up to three index bits per pass: a thread gathers the 2^nb values that differ
  // in those bits, runs their stages in registers and writes them back (one barrier per pass)
  const int lb = 31 - __clz(hb < range ? hb : range);
  for (int b = 3; b < lb; b += 3) {
    const int nb = lb - b < 3 ? lb - b : 3;
    const int gsz = 1 << nb, ngrp = range >> nb;
    for (int p = tid; p < MT * ngrp; p += kDecThreads) {
      const int m = p / ngrp, r = p - m * ngrp;
      const int lo = r & ((1 << b) - 1), hi = r >> b;
      float* wm = work + (size_t)m * range + ((size_t)hi << (b + nb)) + lo;
      float y[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < gsz) y[j] = wm[(size_t)j << b];
#pragma unroll
      for (int h = 1; h < 8; h <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if ((e & h) == 0 && h < gsz) {
            const float pp = y[e], qq = y[e + h];
            y[e] = pp + qq;
            y[e + h] = pp - qq;
          }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < gsz) wm[(size_t)j << b] = y[j];
    }
    __syncthreads();
  }
  // ---- this slice's statistics, reduced over the CTA, then over the cluster
  for (int m = 0; m < MT; ++m)
    for (int i = tid; i < range; i += kDecThreads) {
      const float y = fabsf(work[(size_t)m * range + i]);
      st[m] = absmax ? fmaxf(st[m], y) : st[m] + y;
    }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      ss[m] += __shfl_xor_sync(0xffffffffu, ss[m], o);
      const float t = __shfl_xor_sync(0xffffffffu, st[m], o);
      st[m] = absmax ? fmaxf(st[m], t) : st[m] + t;
    }
    if (lane == 0) {
      red[m][warp][0] = ss[m];
      red[m][warp][1] = st[m];
    }
  }
  __syncthreads();
  cluster_wait();  // every CTA of the cluster is running (pairs with the arrive at kernel start)
  if (tid < MT) {
    float s0 = 0.f, s1 = 0.f;
    for (int w = 0; w < kDecThreads / 32; ++w) {
      s0 += red[tid][w][0];
      s1 = absmax ? fmaxf(s1, red[tid][w][1]) : s1 + red[tid][w][1];
    }
    const uint32_t loc = smem_u32(&stat_in[rank][tid][0]);
    for (int p = 0; p < S; ++p) {
      st_shared_cluster_u32(mapa_shared(loc, (uint32_t)p), __float_as_uint(s0));
      st_shared_cluster_u32(mapa_shared(loc + 4u, (uint32_t)p), __float_as_uint(s1));
    }
  }
  cluster_sync_all();  // every CTA's statistics have landed in every CTA
  // ---- per-row multiplier and scale (the same formulas as the activation kernels), codes
  const float kQ = a.quant == 0 ? 127.f : (a.quant == 1 ? 2.6457513110645906f : 7.f);
  const int lo = a.quant == 0 ? -128 : -8, hi = a.quant == 0 ? 127 : 7;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float ssr = 0.f, str = 0.f;
    for (int p = 0; p < S; ++p) {  // rank order: the same sums in every CTA
      ssr += stat_in[p][m][0];
      str = absmax ? fmaxf(str, stat_in[p][m][1]) : str + stat_in[p][m][1];
    }
    const float r_rms = sqrtf(ssr / (float)K + a.eps_norm);
    const float rs = r_rms * sqrtf((float)hb);
    const float sy = absmax ? str : str / (float)K;
    float mult = 0.f, sx = 0.f;
    if (sy > 0.f) {
      if (a.eps_q == 0.f) {
        mult = kQ / sy;
        sx = sy / (rs * kQ);
      } else {
        const float stat = sy / rs;
        mult = kQ / ((stat + a.eps_q) * rs);
        sx = stat / kQ;
      }
    }
    if (tid == 0) sx_out[m] = sx;
    for (int v = tid; v < nvec; v += kDecThreads) {
      const float* src = work + (size_t)m * range + 8 * v;
      uint32_t b[2] = {0u, 0u};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int q = min(max(__float2int_rn(src[e] * mult), lo), hi);
        qs[m] += q;
        b[e >> 2] |= ((uint32_t)q & 0xffu) << (8 * (e & 3));
      }
      *reinterpret_cast<uint2*>(act + (size_t)m * range + 8 * v) = make_uint2(b[0], b[1]);
    }
  }
}

template <int MT, bool FUSED>
__global__ void __launch_bounds__(kDecThreads, 2) gemm_decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t dec_smem[];
  __shared__ int32_t qred[MT][kDecThreads / 32];
  __shared__ __align__(8) uint64_t full[kDecStages];
  __shared__ volatile int abort_flag;
  // fused forward only: the peers' partial row statistics, the CTA's partials, the row scales
  __shared__ float stat_in[FUSED ? 8 : 1][MT][2];
  __shared__ float red[FUSED ? MT : 1][kDecThreads / 32][2];
  __shared__ float sx_sm[MT];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.S;
  const uint32_t rank = cluster_ctarank();
  const int tile = blockIdx.x / S;
  const int n0 = tile * 128;
  const int KB = a.K >> 7;
  const int kb0 = (int)(((long)KB * rank) / S), kb1 = (int)(((long)KB * (rank + 1)) / S);
  const int nkb = kb1 - kb0;
  const int nch = (nkb + kDecChunk - 1) / kDecChunk;
  const int range = nkb * 128;
  const int FO = (128 + S - 1) / S;
  int32_t* slots = reinterpret_cast<int32_t*>(dec_smem);
  uint8_t* ring = dec_smem + dec_slot_bytes(S, MT);
  int8_t* act = reinterpret_cast<int8_t*>(ring + kDecRingBytes);
  cluster_arrive_relaxed();  // "this CTA runs"; waited for before the first remote store

  // ---- 1. the first kDecStages chunks of this CTA's weight tiles (consecutive in memory)
  const uint8_t* wsrc = reinterpret_cast<const uint8_t*>(a.w2) + ((size_t)tile * KB + kb0) * 4096;
  auto issue = [&](int c) {  // one thread
    const int stg = c % kDecStages;
    const uint32_t bytes = (uint32_t)min(kDecChunk, nkb - c * kDecChunk) * 4096u;
    mbar_arrive_expect_tx(&full[stg], bytes);
    bulk_load_1d(ring + stg * (kDecChunk * 4096), wsrc + (size_t)c * kDecChunk * 4096, bytes, &full[stg]);
  };
  int issued = 0;  // chunks handed to the TMA engine (thread 0)
  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < kDecStages; ++i) mbar_init(&full[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (; issued < nch && issued < kDecStages; ++issued) issue(issued);
  }

  // ---- 2. stage the activations and their per-token sums (packed rows widened). Until here
  // the kernel touched only its weights; the codes (or, fused, the rows X) may come from the
  // kernel before it
  pdl_wait();
  int qs[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) qs[m] = 0;
  if constexpr (FUSED)
    decode_fused_codes<MT>(a, range, (int)rank, reinterpret_cast<float*>(act + MT * range), act, stat_in, sx_sm,
                           qs, red);
  for (int e = tid * 16; !FUSED && e < MT * range; e += kDecThreads * 16) {
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
  __syncthreads();  // barriers initialised, activations staged

  // ---- 3. per chunk: wait (bounded; the outcome is voted so that all threads leave together),
  // refill the stage the previous chunk used (every thread is past it), widen and multiply;
  // thread = (feature f, half h) reads the 16 bytes at f * 32 + h * 16 of each 4 KB tile
  const int f = tid >> 1, h = tid & 1;
  const int8_t* ab = act + 64 * h;
  int accp[4][MT];  // per bit plane
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int m = 0; m < MT; ++m) accp[p][m] = 0;
  // one k-block: 4 words of 16 codes, each plane against its activation word
  auto kblock = [&](const uint8_t* wp, const int8_t* ak) {
    const uint4 wv = *reinterpret_cast<const uint4*>(wp);
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // word i: codes of k = 64h + 16i + 4s + b
      uint4 q[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) q[m] = *reinterpret_cast<const uint4*>(ak + (size_t)m * range + 16 * i);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const uint32_t cw = ww[i] & (0x03030303u << (2 * p));  // bytes c * 4^p
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint32_t qw = p == 0 ? q[m].x : p == 1 ? q[m].y : p == 2 ? q[m].z : q[m].w;
          accp[p][m] = dp4a_us(cw, qw, accp[p][m]);
        }
      }
    }
  };
  int c = 0;
  for (; c < nch; ++c) {
    const int stg = c % kDecStages;
    const bool ok = mbar_wait(&full[stg], (uint32_t)(c / kDecStages) & 1u, &abort_flag);
    if (!__syncthreads_and(ok)) break;
    if (tid == 0 && c >= 1 && issued < nch) issue(issued++);  // chunk c + 3 into chunk c - 1's stage
    const uint8_t* wbase = ring + stg * (kDecChunk * 4096) + f * 32 + h * 16;
    const int8_t* abase = ab + c * (kDecChunk * 128);
    if ((c + 1) * kDecChunk <= nkb) {
#pragma unroll
      for (int u = 0; u < kDecChunk; ++u) kblock(wbase + u * 4096, abase + u * 128);
    } else {
      for (int u = 0; c * kDecChunk + u < nkb; ++u) kblock(wbase + u * 4096, abase + u * 128);
    }
  }
  int acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m)  // each plane's sum is a multiple of 4^p: exact
    acc[m] = accp[0][m] + (accp[1][m] >> 2) + (accp[2][m] >> 4) + (accp[3][m] >> 6);
  // an aborted wait leaves no copy in flight into shared memory when the CTA exits
  if (tid == 0 && c < nch) {
    for (int d = c; d < issued; ++d) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&full[d % kDecStages], (uint32_t)(d / kDecStages) & 1u) &&
             globaltimer_ns() - t0 < kWaitLimitNs) {
      }
    }
  }

  // ---- 4. the two halves of a feature, minus this CTA's sum of q, into the owner's slot
  const int owner = f / FO, fo = f - owner * FO;
  const uint32_t slot0 = smem_u32(slots);
  if constexpr (!FUSED) cluster_wait();  // every CTA of the cluster is running (fused: known already)
  pdl_launch_dependents();  // the next kernel may launch (it waits for this one before reading Y)
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], 1);
    if (h == 0) {
      int qsum = 0;
#pragma unroll
      for (int w = 0; w < kDecThreads / 32; ++w) qsum += qred[m][w];
      const uint32_t off = (uint32_t)((((int)rank * MT + m) * FO + fo) * 4);
      st_shared_cluster_u32(mapa_shared(slot0 + off, (uint32_t)owner), (uint32_t)(acc[m] - qsum));
    }
  }
  cluster_sync_all();  // every peer's slots have landed; after this each CTA reads only its own

  // ---- 5. sum the slots of the owned features (fixed order), dequant, store
  for (int e = tid; e < MT * FO; e += kDecThreads) {
    const int m = e / FO, fl = e - m * FO;
    const int ft = (int)rank * FO + fl;
    const int n = n0 + ft, row = a.m0 + m;
    if (ft >= 128 || row >= a.M || n >= a.N) continue;
    int32_t accv = 0;
    for (int p = 0; p < S; ++p) accv += slots[(p * MT + m) * FO + fl];
    const float y = (float)accv * ((FUSED ? sx_sm[m] : a.s_x[row]) * a.alpha);
    if (a.out_bf16) reinterpret_cast<__nv_bfloat16*>(a.Y)[(size_t)row * a.N + n] = __float2bfloat16_rn(y);
    else reinterpret_cast<float*>(a.Y)[(size_t)row * a.N + n] = y;
    if (a.acc_debug) a.acc_debug[(size_t)row * a.N + n] = accv;
  }
}

}  // namespace hbl
