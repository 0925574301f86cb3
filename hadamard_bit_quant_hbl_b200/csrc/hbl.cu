// C ABI of the H-BitLinear forward pass (declared in include/hbl.h): argument checks, kernel
// selection and launches. All device work is in the kernels included below; the host code
// only validates, picks a configuration and queues launches on the caller's stream.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>
#include <type_traits>

#include "hbl.h"

#include "common.cuh"
#include "gemm_decode.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"
#include "gemm_swap.cuh"
#include "norm_fht_quant.cuh"
#include "norm_fht_quant_tc.cuh"
#include "norm_fht_quant_tc2.cuh"
#include "norm_quant.cuh"
#include "pack_weights.cuh"
#include "qkv_quant.cuh"

using namespace hbl;

namespace {

thread_local int t_last_cuda_error = 0;

hbl_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = (int)e;
  return HBL_ECUDA;
}

#define HBL_CHECK_LAUNCH()                          \
  do {                                              \
    const cudaError_t e_ = cudaGetLastError();      \
    if (e_ != cudaSuccess) return cuda_fail(e_);    \
  } while (0)

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

constexpr int kMaxDevices = 64;

int device_sms(int dev) {
  static int cache[kMaxDevices] = {0};
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (cache[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = v > 0 ? v : 148;
  }
  return cache[dev];
}

// Raise a kernel's dynamic shared memory limit when a launch needs more than was allowed so far
// on the current device (the limit does not change occupancy; the launch's own size does). The
// default limit counts static shared memory too, so it is raised for any non-zero size.
struct SmemLimit {
  std::mutex mu;
  int allowed[64] = {0};
};

template <typename F>
cudaError_t allow_smem(F* kernel, int bytes, SmemLimit& lim) {
  int dev = 0;
  cudaGetDevice(&dev);
  dev &= 63;
  std::lock_guard<std::mutex> lk(lim.mu);
  if (lim.allowed[dev] >= bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  // the kernels stream their data, so L1 matters less than shared memory: ask for the largest
  // carveout, so that the occupancy query (which sizes the persistent grids) and the launch agree
  // on how many CTAs share an SM
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) lim.allowed[dev] = bytes;
  return e;
}

// ---------------------------------------------------------------- packed-weight layout

struct BlobLayout {
  size_t off0, off1, off2, total;
};

BlobLayout blob_layout(int K, int N) {
  BlobLayout b;
  b.off0 = 0;
  b.off1 = round_up((size_t)((N + 127) / 128 * 128) * K / 4, 256);  // section 0 padded to whole tiles
  b.off2 = b.off1 + round_up((size_t)N * K, 256);
  b.total = b.off2 + round_up((size_t)N * 4, 256);
  return b;
}

bool dims_ok(int M, int K) { return M >= 1 && K >= 256 && K <= 32768 && (K % 256) == 0; }

// ---------------------------------------------------------------- fused norm/FHT/quant

// Persistent grid: as many CTAs as fit on the device at once (at most one per row group).
template <typename F>
int persistent_grid(F* kernel, int threads, int smem, int groups) {
  int dev = 0;
  cudaGetDevice(&dev);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int g = device_sms(dev) * per_sm;
  return groups < g ? groups : g;
}

template <int L, int EB, int R, bool G, int QM>
hbl_status launch_nfq_t(const NfqArgs& a, int threads, int smem, cudaStream_t s) {
  static SmemLimit lim;
  auto* k = norm_fht_quant_kernel<L, EB, R, G, QM>;
  const cudaError_t e = allow_smem(k, smem, lim);
  if (e != cudaSuccess) return cuda_fail(e);
  NfqArgs b = a;
  // prefetch distance: the groups resident on the device at once (the group that starts when
  // this CTA's successor does)
  b.pf_dist = persistent_grid(k, threads, smem, 1 << 30);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(b.groups, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the kernel before
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t le = cudaLaunchKernelEx(&cfg, k, b);
  if (le != cudaSuccess) return cuda_fail(le);
  HBL_CHECK_LAUNCH();
  return HBL_OK;
}

template <int L, int EB, int R>
hbl_status launch_nfq_g(const NfqArgs& a, int quant, int threads, int smem, cudaStream_t s) {
  if (a.gain) {
    if (quant == 0) return launch_nfq_t<L, EB, R, true, 0>(a, threads, smem, s);
    if (quant == 1) return launch_nfq_t<L, EB, R, true, 1>(a, threads, smem, s);
    return launch_nfq_t<L, EB, R, true, 2>(a, threads, smem, s);
  }
  if (quant == 0) return launch_nfq_t<L, EB, R, false, 0>(a, threads, smem, s);
  if (quant == 1) return launch_nfq_t<L, EB, R, false, 1>(a, threads, smem, s);
  return launch_nfq_t<L, EB, R, false, 2>(a, threads, smem, s);
}

constexpr int eb_for(int L) {
  return L == 8 ? 4 : L == 9 ? 5 : L == 10 ? 5 : L == 11 ? 6 : L == 12 ? 6 : 7;
}

// The tensor-core activation kernel: groups of R rows in one 16384-element buffer, transform
// blocks of 2^LB features; the grid walks the groups, two CTAs per SM.
template <int QM, int R, int LB>
hbl_status launch_nfq_tc(const NfqArgs& a, cudaStream_t s) {
  static SmemLimit lim;
  auto* k = norm_fht_quant_tc_kernel<QM, R, LB>;
  cudaError_t e = allow_smem(k, kNtSmem, lim);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaLaunchConfig_t cfg = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const int resident = kNtCtasPerSm * device_sms(dev);
  const int groups = (a.M + R - 1) / R;
  cfg.gridDim = dim3(groups < resident ? groups : resident, 1, 1);
  cfg.blockDim = dim3(kNtThreads, 1, 1);
  cfg.dynamicSmemBytes = kNtSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the kernel before
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k, a);
  if (e != cudaSuccess) return cuda_fail(e);
  HBL_CHECK_LAUNCH();
  return HBL_OK;
}

template <int QM, int R, int LB>
hbl_status launch_nfq_tc2(const NfqArgs& a, cudaStream_t s) {
  static SmemLimit lim;
  auto* k = norm_fht_quant_tc2_kernel<QM, R, LB>;
  cudaError_t e = allow_smem(k, kN2Smem, lim);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaLaunchConfig_t cfg = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const int sms = device_sms(dev);
  const int groups = (a.M + R - 1) / R;
  cfg.gridDim = dim3(groups < sms ? groups : sms, 1, 1);  // one CTA per SM
  cfg.blockDim = dim3(kN2Threads, 1, 1);
  cfg.dynamicSmemBytes = kN2Smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the kernel before
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k, a);
  if (e != cudaSuccess) return cuda_fail(e);
  HBL_CHECK_LAUNCH();
  return HBL_OK;
}

// No transform (blocks of one feature): up to E features per thread, tpr threads per row (a
// multiple of 32, at most 1024, tpr * E >= K), and at least 256 threads per CTA.
template <int E>
hbl_status launch_nq_e(const NqArgs& a0, int quant, cudaStream_t s) {
  NqArgs a = a0;
  const int vpt = E / 8;                                 // 16-byte vectors per thread
  a.tpr = ((a.K / 8 + vpt - 1) / vpt + 31) / 32 * 32;   // K / 8 is a multiple of 32
  a.rows = a.tpr >= 256 ? 1 : 256 / a.tpr;
  auto pick = [&](auto k) -> hbl_status {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((a.M + a.rows - 1) / a.rows, 1, 1);
    cfg.blockDim = dim3(a.tpr * a.rows, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the kernel before
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, k, a);
    if (e != cudaSuccess) return cuda_fail(e);
    HBL_CHECK_LAUNCH();
    return HBL_OK;
  };
  if (a.gain) {
    if (quant == 0) return pick(norm_quant_kernel<E, 0, true>);
    if (quant == 1) return pick(norm_quant_kernel<E, 1, true>);
    return pick(norm_quant_kernel<E, 2, true>);
  }
  if (quant == 0) return pick(norm_quant_kernel<E, 0, false>);
  if (quant == 1) return pick(norm_quant_kernel<E, 1, false>);
  return pick(norm_quant_kernel<E, 2, false>);
}

hbl_status run_nq(const void* X, const float* gain, int M, int K, int quant, float eps_norm, float eps_q, int fmt,
                  void* codes, float* s_x, cudaStream_t stream) {
  NqArgs a;
  a.X = static_cast<const uint16_t*>(X);
  a.gain = gain;
  a.codes = static_cast<uint8_t*>(codes);
  a.s_x = s_x;
  a.M = M;
  a.K = K;
  a.fmt = fmt;
  a.eps_norm = eps_norm;
  a.eps_q = eps_q;
  a.tpr = 0;
  a.rows = 0;
  // K is a multiple of 256 in [256, 32768], so tpr lands in [32, 1024]; from 4096 features on a
  // thread keeps four 16-byte loads in flight
  if (K <= 2048) return launch_nq_e<8>(a, quant, stream);
  return launch_nq_e<32>(a, quant, stream);
}

hbl_status run_nfq(const void* X, const float* gain, int M, int K, int had_block, int quant, float eps_norm,
                   float eps_q, int fmt, void* codes, float* s_x, cudaStream_t stream) {
  if (had_block == 1) return run_nq(X, gain, M, K, quant, eps_norm, eps_q, fmt, codes, s_x, stream);
  const int n = had_block == 0 ? K : had_block;
  if (!is_pow2(n) || n < 256 || n > 16384 || (K % n) != 0) return HBL_EUNSUPPORTED;
  const int L = ilog2_c(n);
  const int EB = eb_for(L);
  const int P = 1 << (L - EB);
  const int nb = K / n;
  int R = 1, slots = 1, rows = 1;
  if (nb == 1) {
    // a group of rows per CTA: about 128 threads and <= 64 KB of fp32 regrouping buffer, so that
    // three or more CTAs fit on an SM
    rows = 128 / P;
    if (rows < 1) rows = 1;
    if (P == 16 && rows > 1 && (rows & 1)) rows -= 1;  // half-warp rows come in pairs
  } else {
    // one row per CTA; each thread transforms R blocks in turn so that the CTA stays within the
    // plan's thread bound
    const int maxt = nfq_max_threads(L);
    for (R = 1; R <= 4; R *= 2) {
      slots = (nb + R - 1) / R;
      if (P == 16 && (slots & 1)) ++slots;
      if (slots * P <= maxt) break;
    }
    if (slots * P > maxt) return HBL_EUNSUPPORTED;
  }
  const int threads = rows * slots * P;
  const int smem = rows * K * 4;

  NfqArgs a;
  a.X = static_cast<const uint16_t*>(X);
  a.gain = gain;
  a.codes = static_cast<uint8_t*>(codes);
  a.s_x = s_x;
  a.M = M;
  a.K = K;
  a.nb = nb;
  a.fmt = fmt;
  a.eps_norm = eps_norm;
  a.eps_q = eps_q;
  a.slots = slots;
  a.rows = rows;
  a.groups = (M + rows - 1) / rows;
  a.pf_dist = 0;

  // The tensor-core kernel (no gain): one block of 2^12 .. 2^14 features in groups of 16384 / K
  // rows, or blocks of 256 features in rows of at most 16384 features that are not a power of two,
  // one row per group. (It also serves one block of 2^11 correctly; an earlier version of its
  // per-row epilogue measured slower there than the CUDA-core kernel, 12.5 against 7.1 us on
  // 2048 x 2048, so 2^11 stays on CUDA cores until measured again.)
  // Few rows stay on the CUDA-core kernel: a tensor-core launch holds whole SMs (one or two CTAs
  // of 66-164 KB of shared memory and all of TMEM) and its setup (H in shared memory, the TMEM
  // allocation) is not amortised, while the small kernel leaves room for the product that follows
  // to start streaming its weights early (programmatic launch). Thresholds from B200 timings of
  // the forward in a CUDA graph: 16384 features up to 16 rows (Wdown 7B at 1 / 16 tokens: 10.9 /
  // 15.0 against 11.5 / 15.6 us), 4096 up to 256 rows (Wo 7B at 1 / 16 / 64 tokens, two kernels:
  // 6.1 / 7.2 / 10.0 against 8.7 / 9.2 / 11.6 us; alone at 256 rows 5.8 against 7.3 us), 8192 up
  // to 64 (alone: equal at 64 rows, the tensor cores ahead at 256), block-diagonal rows up to 256
  // (alone at 256 rows: 6.0 against 10.5 us).
  const int tc_min_rows = (nb == 1 && L == 14) ? 17 : ((nb == 1 && L == 13) ? 65 : 257);
  if (gain == nullptr && M >= tc_min_rows) {
    auto tc = [&](auto rc, auto lc) -> hbl_status {
      constexpr int RR = decltype(rc)::value, LL = decltype(lc)::value;
      // groups of 2 or 4 rows: two sets of eight consumer warps per SM (each row half of a group
      // to four warps); one row of 16384 or a block-diagonal row: the 4-warp kernel (split in
      // halves, the 16384-point rows need a TMEM exchange for k bit 13 and ran slower)
      if constexpr (RR > 1) {
        if (quant == 0) return launch_nfq_tc2<0, RR, LL>(a, stream);
        if (quant == 1) return launch_nfq_tc2<1, RR, LL>(a, stream);
        return launch_nfq_tc2<2, RR, LL>(a, stream);
      } else {
        if (quant == 0) return launch_nfq_tc<0, RR, LL>(a, stream);
        if (quant == 1) return launch_nfq_tc<1, RR, LL>(a, stream);
        return launch_nfq_tc<2, RR, LL>(a, stream);
      }
    };
    using std::integral_constant;
    if (nb == 1 && L == 12) return tc(integral_constant<int, 4>{}, integral_constant<int, 12>{});
    if (nb == 1 && L == 13) return tc(integral_constant<int, 2>{}, integral_constant<int, 13>{});
    if (nb == 1 && L == 14) return tc(integral_constant<int, 1>{}, integral_constant<int, 14>{});
    if (nb > 1 && L == 8 && K <= 16384 && !is_pow2(K))
      return tc(integral_constant<int, 1>{}, integral_constant<int, 8>{});
  }
  // K <= 32768 bounds nb, so these R always suffice: L=8 nb<=128 (R<=4), L=9..12 R<=2, L>=13 R=1
  switch (L) {
    case 8:
      if (R == 1) return launch_nfq_g<8, 4, 1>(a, quant, threads, smem, stream);
      if (R == 2) return launch_nfq_g<8, 4, 2>(a, quant, threads, smem, stream);
      return launch_nfq_g<8, 4, 4>(a, quant, threads, smem, stream);
    case 9: return R == 1 ? launch_nfq_g<9, 5, 1>(a, quant, threads, smem, stream)
                          : launch_nfq_g<9, 5, 2>(a, quant, threads, smem, stream);
    case 10: return R == 1 ? launch_nfq_g<10, 5, 1>(a, quant, threads, smem, stream)
                           : launch_nfq_g<10, 5, 2>(a, quant, threads, smem, stream);
    case 11: return R == 1 ? launch_nfq_g<11, 6, 1>(a, quant, threads, smem, stream)
                           : launch_nfq_g<11, 6, 2>(a, quant, threads, smem, stream);
    case 12: return R == 1 ? launch_nfq_g<12, 6, 1>(a, quant, threads, smem, stream)
                           : launch_nfq_g<12, 6, 2>(a, quant, threads, smem, stream);
    case 13: return launch_nfq_g<13, 7, 1>(a, quant, threads, smem, stream);
    case 14: return launch_nfq_g<14, 7, 1>(a, quant, threads, smem, stream);
    default: return HBL_EUNSUPPORTED;
  }
}

// ---------------------------------------------------------------- products

template <int MT, bool FUSED>
hbl_status launch_decode_t(const DecodeArgs& a, int smem, cudaStream_t s) {
  static SmemLimit lim;
  cudaError_t e = allow_smem(gemm_decode_kernel<MT, FUSED>, smem, lim);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(((a.N + 127) / 128) * a.S, 1, 1);
  cfg.blockDim = dim3(kDecThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the kernel before
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, gemm_decode_kernel<MT, FUSED>, a);
  if (e != cudaSuccess) return cuda_fail(e);
  HBL_CHECK_LAUNCH();
  return HBL_OK;
}

// One launch per slice of up to 8 token rows (fused: up to 4). A cluster of S CTAs splits K for
// each 128-feature tile: S is chosen so that about two CTAs run per SM, and large enough that the
// CTA's staged activations stay within 32 KB (next to the 64 KB weight ring). The fused forward
// takes S down to a power of two, so that K / S is a power of two as well (its slices are blocks
// of the transform's index space), and adds an fp32 working copy of its slice of the rows.
hbl_status run_decode(const DecodeArgs& a0, bool fused, cudaStream_t s) {
  DecodeArgs a = a0;
  int dev = 0;
  cudaGetDevice(&dev);
  const int ntiles = (a.N + 127) / 128;
  const int KB = a.K / 128;
  for (a.m0 = 0; a.m0 < a0.M;) {
    const int left = a0.M - a.m0;
    const int MT = left == 1 ? 1 : left == 2 ? 2 : left <= 4 ? 4 : 8;
    int S = (2 * device_sms(dev) + ntiles - 1) / ntiles;
    const int smin = (a.K * MT + 32767) / 32768;
    if (S < smin) S = smin;
    if (S > 8) S = 8;
    if (S > KB) S = KB;
    if (S < 1) S = 1;
    if (fused)
      while (S & (S - 1)) --S;
    a.S = S;
    const int range = (KB + S - 1) / S * 128;
    const int smem = dec_slot_bytes(S, MT) + kDecRingBytes + MT * range + (fused ? MT * range * 4 : 0);
    hbl_status st;
    if (fused) {
      switch (MT) {
        case 1: st = launch_decode_t<1, true>(a, smem, s); break;
        case 2: st = launch_decode_t<2, true>(a, smem, s); break;
        default: st = launch_decode_t<4, true>(a, smem, s); break;
      }
    } else {
      switch (MT) {
        case 1: st = launch_decode_t<1, false>(a, smem, s); break;
        case 2: st = launch_decode_t<2, false>(a, smem, s); break;
        case 4: st = launch_decode_t<4, false>(a, smem, s); break;
        default: st = launch_decode_t<8, false>(a, smem, s); break;
      }
    }
    if (st != HBL_OK) return st;
    a.m0 += MT;
  }
  return HBL_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D K-major int8 operand [rows][K] as a TMA map with a (128 bytes x box_rows) box, 128-byte swizzle.
bool make_map_i8(CUtensorMap* map, const void* base, int K, int rows, int box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K};
  const cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Split-K pays for its reduction through distributed shared memory only over long main loops
// (measured on B200 at 512 tokens: K = 16384 39.7 against 50.0 us, K = 4096 24.3 against 19.2 us).
constexpr int kT2SplitMinK = 8192;

hbl_status run_tc2(const void* codes_i8, const int8_t* w_i8, const TcArgs& a0, cudaStream_t s) {
  CUtensorMap mA, mB;
  if (!make_map_i8(&mA, codes_i8, a0.K, a0.M, 128)) return HBL_ECUDA;
  if (!make_map_i8(&mB, w_i8, a0.K, a0.N, 128)) return HBL_ECUDA;
  Tc2Args a;
  a.s_x = a0.s_x;
  a.alpha = a0.alpha;
  a.M = a0.M;
  a.N = a0.N;
  a.K = a0.K;
  a.Y = a0.Y;
  a.out_bf16 = a0.out_bf16;
  a.acc_debug = a0.acc_debug;
  a.tiles_m = (a.M + kT2BM - 1) / kT2BM;
  a.tiles_n = (a.N + kT2BN - 1) / kT2BN;
  int dev = 0;
  cudaGetDevice(&dev);
  const int ntiles = a.tiles_m * a.tiles_n;
  const int pairs = device_sms(dev) / 2;
  if (2 * ntiles <= pairs && a.K >= kT2SplitMinK) {
    // at most half the pairs would have a tile: two pairs per tile, each summing half of K
    static SmemLimit lim_s;
    cudaError_t e = allow_smem(gemm_tc2s_kernel, kT2Smem, lim_s);
    if (e != cudaSuccess) return cuda_fail(e);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(4 * ntiles, 1, 1);
    cfg.blockDim = dim3(kT2Threads, 1, 1);
    cfg.dynamicSmemBytes = kT2Smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 4;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the kernel before
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, gemm_tc2s_kernel, mA, mB, a);
    if (e != cudaSuccess) return cuda_fail(e);
    HBL_CHECK_LAUNCH();
    return HBL_OK;
  }
  const int grid = 2 * (ntiles < pairs ? ntiles : pairs);
  static SmemLimit lim;
  cudaError_t e = allow_smem(gemm_tc2_kernel, kT2Smem, lim);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kT2Threads, 1, 1);
  cfg.dynamicSmemBytes = kT2Smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the kernel before
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemm_tc2_kernel, mA, mB, a);
  if (e != cudaSuccess) return cuda_fail(e);
  HBL_CHECK_LAUNCH();
  return HBL_OK;
}

// 3-D view of int8 codes [rows][K] as (128 bytes, rows, K/128 blocks) with a (128, box_rows, gb) box
// and 128-byte swizzle: one copy brings gb consecutive k-blocks, laid out as [gb][box_rows][128].
bool make_map_i8_blocks(CUtensorMap* map, const void* base, int K, int rows, int box_rows, int gb) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {128u, (cuuint64_t)rows, (cuuint64_t)(K / 128)};
  const cuuint64_t strides[2] = {(cuuint64_t)K, 128u};
  const cuuint32_t box[3] = {128u, (cuuint32_t)box_rows, (cuuint32_t)gb};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Products for up to this many tokens run on the swapped tensor-core kernel over 2-bit weights.
constexpr int kSwapMaxM = 256;

hbl_status run_swap(const void* codes_i8, const void* w2, const TcArgs& t, cudaStream_t s) {
  SwapArgs a;
  a.s_x = t.s_x;
  a.alpha = t.alpha;
  a.M = t.M;
  a.N = t.N;
  a.K = t.K;
  a.Mt = (t.M + 15) / 16 * 16;
  // batches of BK k-blocks; tensor memory: nis accumulators of Mt columns, then NS slots of
  // BK x 32 columns of widened weights; shared memory: NA activation copies of one batch
  // (BK x Mt x 128 bytes) and NR 2-bit copies (BK x 4 KB). Up to 128 tokens two threads issue the
  // MMAs (alternate batches, one accumulator each): there an MMA is short and one issuing thread
  // was the limit (Wdown 7B at 16 / 128 tokens: 11.0 / 15.5 against 12.3 / 17.0 us); above 64
  // tokens the two accumulators leave room for four slots only with batches of 2 k-blocks, and
  // above 128 tokens for too few slots.
  const int BK = a.Mt <= 64 ? 4 : 2;
  a.nis = a.Mt <= 128 ? 2 : 1;
  int stride = 16;
  while (stride < a.Mt) stride *= 2;
  a.acc_stride = stride;
  a.acc_cols = a.nis * stride < 32 ? 32 : a.nis * stride;
  a.NS = (kSwTmemCols - a.acc_cols) / (BK * 32);
  if (a.NS > kSwMaxNS) a.NS = kSwMaxNS;
  a.NS -= a.NS % a.nis;  // an issuer's slots (and stages, below) repeat with period nis
  const int act_stage = BK * a.Mt * kSwBK, raw_stage = BK * kSwRaw;
  a.NA = (kSwSmem - 4 * raw_stage) / act_stage;
  if (a.NA > kSwMaxNA) a.NA = kSwMaxNA;
  if (a.NA < 1) return HBL_EUNSUPPORTED;  // not reached for Mt <= 256
  a.NR = (kSwSmem - a.NA * act_stage) / raw_stage;
  if (a.NR > kSwMaxNR) a.NR = kSwMaxNR;
  // a widening warp takes every kSwW-th batch: with NR a multiple of kSwW, the warp that waits for
  // a ring stage's copy is the one that consumed the stage's previous copy, and with NS >= kSwW
  // no warp runs two phases ahead on a tensor-memory slot (a parity wait cannot alias)
  a.NR -= a.NR % kSwW;
  a.NA -= a.NA % a.nis;
  if (a.NS < kSwW || a.NR < kSwW || a.NA < 1) return HBL_EUNSUPPORTED;  // not reached for Mt <= 256
  a.Y = t.Y;
  a.out_bf16 = t.out_bf16;
  a.acc_debug = t.acc_debug;
  int dev = 0;
  cudaGetDevice(&dev);
  const int ntiles = (a.N + kSwNT - 1) / kSwNT;
  const int KB = a.K / kSwBK;
  int S = device_sms(dev) / ntiles;  // split K so that the grid fills the device
  if (S > 8) S = 8;
  if (S > KB) S = KB;
  if (S < 1) S = 1;
  a.S = S;
  a.w2 = static_cast<const uint32_t*>(w2);
  CUtensorMap mA;
  if (!make_map_i8_blocks(&mA, codes_i8, a.K, a.M, a.Mt, BK)) return HBL_ECUDA;
  static SmemLimit lim4, lim2;
  const int smem = kSwSmem + 1024;  // + alignment slack
  auto kern = BK == 4 ? gemm_swap_kernel<4> : gemm_swap_kernel<2>;
  cudaError_t e = allow_smem(kern, smem, BK == 4 ? lim4 : lim2);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ntiles * S, 1, 1);
  cfg.blockDim = dim3(kSwThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the kernel before
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, mA, a);
  if (e != cudaSuccess) return cuda_fail(e);
  HBL_CHECK_LAUNCH();
  return HBL_OK;
}

// Token counts up to these bounds run on CUDA cores (weight bytes bound the product there):
// int8 codes up to 4 tokens (from 5 on the swapped tensor-core kernel is faster), packed int4
// codes up to 8 (the tensor-core kernels read one int8 per code).
constexpr int kDecodeMaxM = 4;
constexpr int kDecodeMaxMPacked = 8;
// hbl_forward_decode fuses the activation side into the decode product up to this width.
constexpr int kFusedMaxK = 8192;

hbl_status run_gemm(const void* codes, int fmt, int abits, const float* s_x, const void* packed, float alpha,
                    int M, int N, int K, void* Y, int out_dtype, int32_t* acc_debug, cudaStream_t s) {
  const BlobLayout bl = blob_layout(K, N);
  const uint8_t* blob = static_cast<const uint8_t*>(packed);
  const bool packed4 = (abits == 4 && fmt == HBL_CODES_PACKED);
  if (M <= (packed4 ? kDecodeMaxMPacked : kDecodeMaxM)) {
    DecodeArgs d;
    d.m0 = 0;
    d.codes = static_cast<const uint8_t*>(codes);
    d.packed4 = packed4 ? 1 : 0;
    d.s_x = s_x;
    d.w2 = reinterpret_cast<const uint32_t*>(blob + bl.off0);
    d.alpha = alpha;
    d.M = M;
    d.N = N;
    d.K = K;
    d.Y = Y;
    d.out_bf16 = out_dtype == HBL_OUT_BF16;
    d.acc_debug = acc_debug;
    d.X = nullptr;
    d.gain = nullptr;
    d.hb = 1;
    d.quant = 0;
    d.eps_norm = 0.f;
    d.eps_q = 0.f;
    return run_decode(d, false, s);
  }
  if (packed4) return HBL_EUNSUPPORTED;  // the tensor-core path reads one int8 per code
  TcArgs t;
  t.s_x = s_x;
  t.alpha = alpha;
  t.M = M;
  t.N = N;
  t.K = K;
  t.Y = Y;
  t.out_bf16 = out_dtype == HBL_OUT_BF16;
  t.acc_debug = acc_debug;
  if (M <= kSwapMaxM) return run_swap(codes, blob + bl.off0, t, s);
  return run_tc2(codes, reinterpret_cast<const int8_t*>(blob + bl.off1), t, s);
}

// Ternarise fp32 W [K][N] into the packed blob (validated arguments): alpha reduced on the
// device, codes packed, alpha read back (synchronises the stream).
hbl_status pack_from_f32(const float* W, int K, int N, float eps_w, void* packed, float* alpha_host, void* workspace,
                         cudaStream_t s) {
  const BlobLayout bl = blob_layout(K, N);
  uint8_t* blob = static_cast<uint8_t*>(packed);
  double* partials = static_cast<double*>(workspace);
  double* alpha_d = partials + kAbsumBlocks;
  cudaError_t e = cudaMemsetAsync(blob + bl.off2, 0, (size_t)N * 4, s);
  if (e != cudaSuccess) return cuda_fail(e);
  const size_t count = (size_t)K * N;
  absum_partial_kernel<<<kAbsumBlocks, kAbsumThreads, 0, s>>>(W, count / 4, partials);
  HBL_CHECK_LAUNCH();
  absum_final_kernel<<<1, kAbsumThreads, 0, s>>>(partials, kAbsumBlocks, (double)count, alpha_d);
  HBL_CHECK_LAUNCH();
  dim3 grid((N + 127) / 128, K / 16);
  ternarize_pack_kernel<false><<<grid, 128, 0, s>>>(W, nullptr, K, N, alpha_d, (double)eps_w,
                                                     reinterpret_cast<uint32_t*>(blob + bl.off0),
                                                     reinterpret_cast<int8_t*>(blob + bl.off1),
                                                     reinterpret_cast<int32_t*>(blob + bl.off2));
  HBL_CHECK_LAUNCH();
  double alpha = 0.0;
  e = cudaMemcpyAsync(&alpha, alpha_d, sizeof(double), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  *alpha_host = (float)alpha;
  return HBL_OK;
}

template <int E, int BITS>
hbl_status launch_qkv(const QkvArgs& a, cudaStream_t s) {
  const int warps = kQkvTokens * a.H < 8 ? kQkvTokens * a.H : 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.M + kQkvTokens - 1) / kQkvTokens, 1, 1);
  cfg.blockDim = dim3(32 * warps, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the kernel before
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = a.pos ? cudaLaunchKernelEx(&cfg, qkv_quant_kernel<E, BITS, true>, a)
                              : cudaLaunchKernelEx(&cfg, qkv_quant_kernel<E, BITS, false>, a);
  if (e != cudaSuccess) return cuda_fail(e);
  HBL_CHECK_LAUNCH();
  return HBL_OK;
}

template <int E>
hbl_status launch_qkv_e(const QkvArgs& a, int bits, cudaStream_t s) {
  switch (bits) {
    case 2: return launch_qkv<E, 2>(a, s);
    case 3: return launch_qkv<E, 3>(a, s);
    case 4: return launch_qkv<E, 4>(a, s);
    default: return launch_qkv<E, 8>(a, s);
  }
}

template <int E>
hbl_status launch_qkv_dequant_e(const uint8_t* codes, const float* gamma, int M, int H, int bits, uint16_t* Y,
                                cudaStream_t s) {
  const size_t heads = (size_t)M * H;
  const dim3 grid((unsigned)((heads + 7) / 8));
  switch (bits) {
    case 2: qkv_dequant_kernel<E, 2><<<grid, 256, 0, s>>>(codes, gamma, M, H, Y); break;
    case 3: qkv_dequant_kernel<E, 3><<<grid, 256, 0, s>>>(codes, gamma, M, H, Y); break;
    case 4: qkv_dequant_kernel<E, 4><<<grid, 256, 0, s>>>(codes, gamma, M, H, Y); break;
    default: qkv_dequant_kernel<E, 8><<<grid, 256, 0, s>>>(codes, gamma, M, H, Y); break;
  }
  HBL_CHECK_LAUNCH();
  return HBL_OK;
}

bool qkv_shape_ok(int M, int H, int D, int bits) {
  return M >= 1 && H >= 1 && (D == 64 || D == 128 || D == 256) &&
         (bits == 2 || bits == 3 || bits == 4 || bits == 8) && (size_t)M * H < ((size_t)1 << 36);
}

size_t forward_codes_bytes(int M, int K) { return round_up((size_t)M * K, 256); }

}  // namespace

// =========================================================================== C ABI

extern "C" {

const char* hbl_status_string(hbl_status s) {
  switch (s) {
    case HBL_OK: return "HBL_OK";
    case HBL_EINVAL: return "HBL_EINVAL: invalid argument (null/misaligned pointer, bad size, small buffer)";
    case HBL_EUNSUPPORTED: return "HBL_EUNSUPPORTED: request outside what the kernels implement";
    case HBL_ECUDA: return "HBL_ECUDA: a CUDA call failed (see hbl_last_cuda_error)";
    case HBL_ETIMEOUT: return "HBL_ETIMEOUT: a device-side bounded wait gave up";
  }
  return "unknown hbl_status";
}

int hbl_last_cuda_error(void) { return t_last_cuda_error; }

hbl_status hbl_device_status(hbl_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  int flags = 0;
  e = cudaMemcpyFromSymbolAsync(&flags, g_error_flags, sizeof(int), 0, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (flags) {
    const int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_error_flags, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (flags & kErrTimeout) return HBL_ETIMEOUT;
  if (flags & kErrBadTernary) return HBL_EINVAL;
  return HBL_OK;
}

hbl_status hbl_selftest_timeout(int limit_ms, hbl_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 1000) return HBL_EINVAL;
  selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>((uint64_t)limit_ms * 1000000ull);
  HBL_CHECK_LAUNCH();
  return HBL_OK;
}

size_t hbl_packed_weights_bytes(int K, int N) {
  if (K <= 0 || N <= 0) return 0;
  return blob_layout(K, N).total;
}

size_t hbl_pack_weights_workspace(int K, int N) {
  (void)K;
  (void)N;
  return round_up((size_t)(kAbsumBlocks + 1) * sizeof(double), 256);
}

hbl_status hbl_pack_weights(const float* W, int K, int N, float eps_w, void* packed, size_t packed_bytes,
                            float* alpha_host, void* workspace, size_t ws_bytes, hbl_stream_t stream) {
  if (!W || !packed || !alpha_host || !workspace) return HBL_EINVAL;
  if (K < 256 || K > 32768 || (K % 256) || N < 1 || (N % 8)) return HBL_EINVAL;
  if (!aligned(W, 16) || !aligned(packed, 256) || !aligned(workspace, 16)) return HBL_EINVAL;
  if (!(eps_w >= 0.f)) return HBL_EINVAL;
  if (packed_bytes < blob_layout(K, N).total || ws_bytes < hbl_pack_weights_workspace(K, N)) return HBL_EINVAL;
  return pack_from_f32(W, K, N, eps_w, packed, alpha_host, workspace, reinterpret_cast<cudaStream_t>(stream));
}

size_t hbl_pack_weights_rotated_workspace(int K, int N) {
  if (K <= 0 || N <= 0) return 0;
  return round_up((size_t)K * N * 4, 256) + hbl_pack_weights_workspace(K, N);
}

hbl_status hbl_pack_weights_rotated(const float* W, int K, int N, int had_block, float eps_w, void* packed,
                                    size_t packed_bytes, float* alpha_host, void* workspace, size_t ws_bytes,
                                    hbl_stream_t stream) {
  if (!W || !packed || !alpha_host || !workspace) return HBL_EINVAL;
  if (K < 256 || K > 32768 || (K % 256) || N < 1 || (N % 8)) return HBL_EINVAL;
  if (!aligned(W, 16) || !aligned(packed, 256) || !aligned(workspace, 256)) return HBL_EINVAL;
  if (!(eps_w >= 0.f) || had_block < 0) return HBL_EINVAL;
  if (packed_bytes < blob_layout(K, N).total || ws_bytes < hbl_pack_weights_rotated_workspace(K, N))
    return HBL_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (had_block == 1)  // blocks of one feature: no rotation
    return pack_from_f32(W, K, N, eps_w, packed, alpha_host, static_cast<uint8_t*>(workspace) +
                         round_up((size_t)K * N * 4, 256), s);
  const int n = had_block == 0 ? K : had_block;
  if (!is_pow2(n) || n < 256 || n > 16384 || (K % n) != 0) return HBL_EUNSUPPORTED;
  float* Wr = static_cast<float*>(workspace);
  // the transform's log2(n) index bits in passes of at most 7 bits (2^7 rows x 32 columns of
  // shared memory per CTA); the last pass applies 1/sqrt(n)
  const int L = ilog2_c(n);
  const int passes = (L + 6) / 7;
  int b0 = 0;
  for (int pi = 0; pi < passes; ++pi) {
    const int nb = (L - b0) / (passes - pi);
    const float scale = pi == passes - 1 ? (float)(1.0 / sqrt((double)n)) : 1.f;
    const dim3 grid((N + 31) / 32, K >> nb);
    const float* src = pi == 0 ? W : Wr;
    switch (nb) {
      case 1: fht_cols_kernel<1><<<grid, 256, 0, s>>>(src, Wr, K, N, b0, scale); break;
      case 2: fht_cols_kernel<2><<<grid, 256, 0, s>>>(src, Wr, K, N, b0, scale); break;
      case 3: fht_cols_kernel<3><<<grid, 256, 0, s>>>(src, Wr, K, N, b0, scale); break;
      case 4: fht_cols_kernel<4><<<grid, 256, 0, s>>>(src, Wr, K, N, b0, scale); break;
      case 5: fht_cols_kernel<5><<<grid, 256, 0, s>>>(src, Wr, K, N, b0, scale); break;
      case 6: fht_cols_kernel<6><<<grid, 256, 0, s>>>(src, Wr, K, N, b0, scale); break;
      default: fht_cols_kernel<7><<<grid, 256, 0, s>>>(src, Wr, K, N, b0, scale); break;
    }
    HBL_CHECK_LAUNCH();
    b0 += nb;
  }
  return pack_from_f32(Wr, K, N, eps_w, packed, alpha_host,
                       static_cast<uint8_t*>(workspace) + round_up((size_t)K * N * 4, 256), s);
}

hbl_status hbl_pack_ternary(const int8_t* t, int K, int N, void* packed, size_t packed_bytes,
                            hbl_stream_t stream) {
  if (!t || !packed) return HBL_EINVAL;
  if (K < 256 || K > 32768 || (K % 256) || N < 1 || (N % 8)) return HBL_EINVAL;
  if (!aligned(packed, 256)) return HBL_EINVAL;
  const BlobLayout bl = blob_layout(K, N);
  if (packed_bytes < bl.total) return HBL_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* blob = static_cast<uint8_t*>(packed);
  cudaError_t e = cudaMemsetAsync(blob + bl.off2, 0, (size_t)N * 4, s);
  if (e != cudaSuccess) return cuda_fail(e);
  dim3 grid((N + 127) / 128, K / 16);
  ternarize_pack_kernel<true><<<grid, 128, 0, s>>>(nullptr, t, K, N, nullptr, 0.0,
                                                    reinterpret_cast<uint32_t*>(blob + bl.off0),
                                                    reinterpret_cast<int8_t*>(blob + bl.off1),
                                                    reinterpret_cast<int32_t*>(blob + bl.off2));
  HBL_CHECK_LAUNCH();
  return HBL_OK;
}

hbl_status hbl_norm_fht_quant(const void* X, const float* gain, int M, int K, int had_block, hbl_quant quant,
                              float eps_norm, float eps_q, hbl_codes_fmt fmt, void* codes, float* s_x,
                              hbl_stream_t stream) {
  if (!X || !codes || !s_x) return HBL_EINVAL;
  if (!dims_ok(M, K)) return HBL_EINVAL;
  if (!aligned(X, 16) || !aligned(codes, 16) || !aligned(s_x, 4) || (gain && !aligned(gain, 4)))
    return HBL_EINVAL;
  if (quant != HBL_Q_A8_ABSMAX && quant != HBL_Q_A4_ABSMEAN && quant != HBL_Q_A4_ABSMAX) return HBL_EUNSUPPORTED;
  if (fmt != HBL_CODES_PACKED && fmt != HBL_CODES_I8) return HBL_EINVAL;
  if (!(eps_norm >= 0.f) || !(eps_q >= 0.f)) return HBL_EINVAL;
  if (had_block < 0) return HBL_EINVAL;
  return run_nfq(X, gain, M, K, had_block, (int)quant, eps_norm, eps_q, (int)fmt, codes, s_x,
                 reinterpret_cast<cudaStream_t>(stream));
}

hbl_status hbl_ternary_gemm(const void* codes, hbl_codes_fmt fmt, int abits, const float* s_x, const void* packed,
                            size_t packed_bytes, float alpha, int M, int N, int K, void* Y, hbl_out_dtype out_dtype,
                            int32_t* acc_debug, hbl_stream_t stream) {
  if (!codes || !s_x || !packed || !Y) return HBL_EINVAL;
  if (!dims_ok(M, K) || N < 8 || (N % 8)) return HBL_EINVAL;
  if (abits != 4 && abits != 8) return HBL_EUNSUPPORTED;
  if (fmt != HBL_CODES_PACKED && fmt != HBL_CODES_I8) return HBL_EINVAL;
  if (out_dtype != HBL_OUT_F32 && out_dtype != HBL_OUT_BF16) return HBL_EINVAL;
  if (!aligned(codes, 16) || !aligned(packed, 256) || !aligned(Y, 16) || !aligned(s_x, 4) ||
      (acc_debug && !aligned(acc_debug, 4)))
    return HBL_EINVAL;
  if (packed_bytes < blob_layout(K, N).total) return HBL_EINVAL;
  return run_gemm(codes, (int)fmt, abits, s_x, packed, alpha, M, N, K, Y, (int)out_dtype, acc_debug,
                  reinterpret_cast<cudaStream_t>(stream));
}

size_t hbl_qkv_codes_bytes(int M, int H, int D, int bits) {
  if (M <= 0 || H <= 0 || D <= 0 || bits <= 0) return 0;
  return (size_t)M * H * D * bits / 8;
}

hbl_status hbl_qkv_quant(const void* X, size_t row_stride, const int32_t* pos, float rope_theta, int M, int H, int D,
                         int bits, void* codes, size_t codes_bytes, float* gamma, hbl_stream_t stream) {
  if (!X || !codes || !gamma) return HBL_EINVAL;
  if (M < 1 || H < 1 || D < 1 || bits < 1) return HBL_EINVAL;
  if (!qkv_shape_ok(M, H, D, bits)) return HBL_EUNSUPPORTED;
  if (row_stride < (size_t)H * D || (row_stride % 8) != 0) return HBL_EINVAL;
  if (!aligned(X, 16) || !aligned(codes, 16) || !aligned(gamma, 4) || (pos && !aligned(pos, 4))) return HBL_EINVAL;
  if (pos && !(rope_theta > 1.f && rope_theta < 3.0e38f)) return HBL_EINVAL;
  if (codes_bytes < hbl_qkv_codes_bytes(M, H, D, bits)) return HBL_EINVAL;
  QkvArgs a;
  a.X = static_cast<const uint16_t*>(X);
  a.row_stride = row_stride;
  a.pos = pos;
  a.theta = rope_theta;
  a.codes = static_cast<uint8_t*>(codes);
  a.gamma = gamma;
  a.M = M;
  a.H = H;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (D == 64) return launch_qkv_e<2>(a, bits, s);
  if (D == 128) return launch_qkv_e<4>(a, bits, s);
  return launch_qkv_e<8>(a, bits, s);
}

hbl_status hbl_qkv_dequant(const void* codes, const float* gamma, int M, int H, int D, int bits, void* Y,
                           hbl_stream_t stream) {
  if (!codes || !gamma || !Y) return HBL_EINVAL;
  if (M < 1 || H < 1 || D < 1 || bits < 1) return HBL_EINVAL;
  if (!qkv_shape_ok(M, H, D, bits)) return HBL_EUNSUPPORTED;
  if (!aligned(codes, 16) || !aligned(gamma, 4) || !aligned(Y, 16)) return HBL_EINVAL;
  const uint8_t* c = static_cast<const uint8_t*>(codes);
  uint16_t* y = static_cast<uint16_t*>(Y);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (D == 64) return launch_qkv_dequant_e<2>(c, gamma, M, H, bits, y, s);
  if (D == 128) return launch_qkv_dequant_e<4>(c, gamma, M, H, bits, y, s);
  return launch_qkv_dequant_e<8>(c, gamma, M, H, bits, y, s);
}

size_t hbl_forward_workspace(int M, int K, hbl_quant quant) {
  (void)quant;
  if (M <= 0 || K <= 0) return 0;
  return forward_codes_bytes(M, K) + round_up((size_t)M * 4, 256);
}

hbl_status hbl_forward(const void* X, const float* gain, const void* packed, size_t packed_bytes, float alpha, int M,
                       int K, int N, int had_block, hbl_quant quant, float eps_norm, float eps_q, void* workspace,
                       size_t ws_bytes, void* Y, hbl_out_dtype out_dtype, hbl_stream_t stream) {
  if (!X || !packed || !workspace || !Y) return HBL_EINVAL;
  if (!dims_ok(M, K) || N < 8 || (N % 8)) return HBL_EINVAL;
  if (!aligned(workspace, 256)) return HBL_EINVAL;
  if (ws_bytes < hbl_forward_workspace(M, K, quant)) return HBL_EINVAL;
  if (packed_bytes < blob_layout(K, N).total || !aligned(packed, 256) || !aligned(Y, 16)) return HBL_EINVAL;
  const int abits = quant == HBL_Q_A8_ABSMAX ? 8 : 4;
  const hbl_codes_fmt fmt = HBL_CODES_I8;  // both tensor-core products read one int8 per code
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* codes = ws;
  float* s_x = reinterpret_cast<float*>(ws + forward_codes_bytes(M, K));
  hbl_status st = hbl_norm_fht_quant(X, gain, M, K, had_block, quant, eps_norm, eps_q, fmt, codes, s_x, stream);
  if (st != HBL_OK) return st;
  return hbl_ternary_gemm(codes, fmt, abits, s_x, packed, packed_bytes, alpha, M, N, K, Y, out_dtype, nullptr,
                          stream);
}

// One token in one launch (the decode product computes its own codes): see hbl.h. Measured on
// B200 (Wo 4096 -> 4096, one token): 8.0 us against 9.2 us for two launches while the activation
// of few rows ran on the tensor-core kernel, 7.5 against 6.1 us since it runs on CUDA cores; with
// more tokens or wider rows every CTA repeats more of the row's transform than the separate
// activation kernel costs (16.1 against 10.8 us at four tokens; Wdown 16384 -> 4096 at one token
// 12.3 against 11.8 us), so the entry takes one token of K <= kFusedMaxK only.
hbl_status hbl_forward_decode(const void* X, const float* gain, const void* packed, size_t packed_bytes,
                              float alpha, int K, int N, int had_block, hbl_quant quant, float eps_norm,
                              float eps_q, void* Y, hbl_out_dtype out_dtype, hbl_stream_t stream) {
  if (!X || !packed || !Y) return HBL_EINVAL;
  if (!dims_ok(1, K) || N < 8 || (N % 8)) return HBL_EINVAL;
  if (packed_bytes < blob_layout(K, N).total || !aligned(packed, 256) || !aligned(Y, 16)) return HBL_EINVAL;
  if (K > kFusedMaxK || !is_pow2(K)) return HBL_EUNSUPPORTED;
  const int n = had_block == 0 ? K : had_block;
  const bool hb_ok = n == 1 || (is_pow2(n) && n >= 256 && n <= 16384 && (K % n) == 0);
  if (!hb_ok) return HBL_EUNSUPPORTED;
  if (quant != HBL_Q_A8_ABSMAX && quant != HBL_Q_A4_ABSMEAN && quant != HBL_Q_A4_ABSMAX) return HBL_EUNSUPPORTED;
  if (!(eps_norm >= 0.f) || !(eps_q >= 0.f)) return HBL_EINVAL;
  if (!aligned(X, 16) || (gain && !aligned(gain, 4))) return HBL_EINVAL;
  if (out_dtype != HBL_OUT_F32 && out_dtype != HBL_OUT_BF16) return HBL_EINVAL;
  const BlobLayout bl = blob_layout(K, N);
  DecodeArgs d;
  d.m0 = 0;
  d.codes = nullptr;
  d.packed4 = 0;
  d.s_x = nullptr;
  d.w2 = reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(packed) + bl.off0);
  d.alpha = alpha;
  d.M = 1;
  d.N = N;
  d.K = K;
  d.Y = Y;
  d.out_bf16 = out_dtype == HBL_OUT_BF16;
  d.acc_debug = nullptr;
  d.X = static_cast<const uint16_t*>(X);
  d.gain = gain;
  d.hb = n;
  d.quant = (int)quant;
  d.eps_norm = eps_norm;
  d.eps_q = eps_q;
  return run_decode(d, true, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// =========================================================================== forward without a
// caller-provided workspace
//
// Some callers cannot call cudaMalloc: host code whose device memory is owned by another
// component's allocator (and may not allocate behind its back), or a runtime that makes all of its
// device allocations once at start-up and none on the request path. For them hbl_forward_static
// runs the same forward pass with its scratch (activation codes and per-token scales) in a
// fixed-size array that is part of the library's device image. Every GPU that loads the library
// holds this array until the process exits.

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB per device

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

struct StaticScratch {
  std::mutex mu;
  void* addr[kMaxDevices] = {nullptr};
};

StaticScratch& static_scratch() {
  static StaticScratch s;
  return s;
}

// Device address of g_static_scratch on the current device. Host code only sees a host-side
// stand-in for the array's name, never its device address, so the address is looked up with
// cudaGetSymbolAddress once per device (on the first call there) and kept for the life of the
// process. It belongs to the device's primary context: after that context is destroyed
// (cudaDeviceReset) the kept address is stale, which hbl.h states as a limit of this entry point.
hbl_status static_scratch_addr(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return HBL_EUNSUPPORTED;
  StaticScratch& s = static_scratch();
  std::lock_guard<std::mutex> lk(s.mu);
  if (!s.addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    s.addr[dev] = p;
  }
  *out = s.addr[dev];
  return HBL_OK;
}

}  // namespace

extern "C" hbl_status hbl_forward_static(const void* X, const float* gain, const void* packed,
                                         size_t packed_bytes, float alpha, int M, int K, int N,
                                         int had_block, hbl_quant quant, float eps_norm, float eps_q,
                                         void* Y, hbl_out_dtype out_dtype, hbl_stream_t stream) {
  if (!dims_ok(M, K)) return HBL_EINVAL;
  const size_t need = hbl_forward_workspace(M, K, quant);
  if (need > kStaticScratchBytes) return HBL_EUNSUPPORTED;  // request larger than the static scratch
  void* ws = nullptr;
  const hbl_status st = static_scratch_addr(&ws);
  if (st != HBL_OK) return st;
  // The kernels overwrite every scratch byte they later read (codes, then scales), so nothing
  // has to be cleared between calls.
  return hbl_forward(X, gain, packed, packed_bytes, alpha, M, K, N, had_block, quant, eps_norm, eps_q, ws,
                     kStaticScratchBytes, Y, out_dtype, stream);
}
