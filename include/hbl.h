/*
 * hbl.h -- C ABI of the H-BitLinear forward pass (BitNet v2) for NVIDIA B200 (sm_100a).
 *
 * The layer, as stated in "BitNet v2: Native 4-bit Activations with Hadamard
 * Transformation for 1-bit LLMs" (abstract) and in the Chinese walkthrough of that
 * paper (m.jxzklqfsx.com, section "H-BitLinear模塊"):
 *
 *     Y = Q_w(W) . Q_a( Hadamard( RMSNorm(X) ) )
 *
 *   Q_w  per-tensor absmean ternarisation of the weights to {-1, 0, +1} with scale alpha
 *   Hadamard  online fast Walsh-Hadamard transform along the K features of each token
 *   Q_a  per-token activation quantisation to INT8 (absmax) or INT4 (absmean or absmax)
 *
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless its
 *     name ends in _host. The library never allocates or frees memory.
 *   - Every call is stream-ordered on `stream` (0 = legacy default stream) and
 *     returns as soon as its kernels are queued, except hbl_pack_weights, which
 *     synchronises `stream` to hand alpha back to the host.
 *   - Matrices are row-major and densely packed (row stride = row length).
 *   - No call keeps state between calls; all of them are thread-safe as long as
 *     two concurrent calls do not write the same buffers.
 *   - Errors are returned as hbl_status; nothing is thrown across the ABI. On
 *     HBL_ECUDA, hbl_last_cuda_error() (thread-local) gives the CUDA error code.
 *     Device-side bounded waits that give up are reported by the next
 *     hbl_device_status() call as HBL_ETIMEOUT.
 *
 * Scalar sizes: 1 <= M, 1 <= N, K a multiple of 256, K <= 32768.
 */
#ifndef HBL_H_
#define HBL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hbl_stream_t; /* same type as cudaStream_t */

typedef enum hbl_status {
  HBL_OK = 0,
  HBL_EINVAL = 1,        /* null or misaligned pointer, bad size, buffer too small */
  HBL_EUNSUPPORTED = 2,  /* valid request outside what the kernels implement */
  HBL_ECUDA = 3,         /* a CUDA call failed; see hbl_last_cuda_error() */
  HBL_ETIMEOUT = 4       /* a device-side bounded wait gave up (kernel returned early) */
} hbl_status;

/* Activation quantiser (per token row). */
typedef enum hbl_quant {
  HBL_Q_A8_ABSMAX = 0,  /* gamma = max|x|,  q = RoundClip(127 x/(gamma+eps), -128, 127), s = gamma/127 */
  HBL_Q_A4_ABSMEAN = 1, /* beta  = mean|x|, q = RoundClip(sqrt7 x/(beta+eps), -8, 7),    s = beta/sqrt7 */
  HBL_Q_A4_ABSMAX = 2   /* gamma = max|x|,  q = RoundClip(7 x/(gamma+eps), -8, 7),        s = gamma/7   */
} hbl_quant;

/* Layout of activation codes [M][K]. */
typedef enum hbl_codes_fmt {
  HBL_CODES_PACKED = 0, /* a4: two int4 two's-complement codes per byte, element 2j in the low
                           nibble of byte j of the row (row = K/2 bytes); a8: one int8 per element */
  HBL_CODES_I8 = 1      /* one int8 per element for a4 as well (row = K bytes) */
} hbl_codes_fmt;

typedef enum hbl_out_dtype { HBL_OUT_F32 = 0, HBL_OUT_BF16 = 1 } hbl_out_dtype;

/* Human-readable name of a status code (static string). */
const char* hbl_status_string(hbl_status s);

/* CUDA error code (cudaError_t) of the last HBL_ECUDA on the calling thread. */
int hbl_last_cuda_error(void);

/* Reads and clears the device-side error flag of the current device. Synchronises `stream`.
 * Returns HBL_ETIMEOUT if any kernel of this library gave up a bounded wait since the last
 * call, HBL_OK otherwise (or HBL_ECUDA if the synchronisation itself failed). */
hbl_status hbl_device_status(hbl_stream_t stream);

/* Diagnostic of the time-out path. Launches on `stream` one small kernel that waits on a
 * barrier nothing ever completes, with the bounded wait every kernel of this library uses but a
 * limit of `limit_ms` milliseconds (1 ... 1000) instead of 1 s: the wait runs out, raises the
 * device error flag and the kernel returns. The next hbl_device_status() then reports
 * HBL_ETIMEOUT, and the context stays usable. Asynchronous. HBL_EINVAL for a limit outside
 * the range. */
hbl_status hbl_selftest_timeout(int limit_ms, hbl_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Packed ternary weights.
 *
 * Weight ternarisation follows the walkthrough article, section "H-BitLinear模塊" (per-tensor
 * absmean ternarisation to {-1,0,1}), and the bitnet.cpp news article, section
 * "6 页论文，引入 1 bit LLM" (scale by the mean absolute value, round to the nearest of
 * -1, 0, 1):  alpha = mean|W| over all K*N entries; t = RoundClip(W/(alpha+eps_w), -1, 1).
 *
 * The packed blob (hbl_packed_weights_bytes(K, N) bytes, 256-byte aligned) holds, for the
 * logical K x N ternary matrix t:
 *   section 0 at byte 0:   2-bit codes as uint32 words: word w of feature n holds
 *                          t[16w + 4s + b][n] + 1 (in {0,1,2}) at bits 8b+2s (b, s in 0..3).
 *                          Words are tile-major: (n, w) is word number
 *                          ((n/128)*(K/128) + w/8)*1024 + (n%128)*8 + w%8, so each 128-feature
 *                          x 128-k tile is 4 KB of contiguous memory; features are padded to a
 *                          multiple of 128 with t = 0. Read by the small-M products.
 *   section 1 at byte A1:  int8 t[k][n] as N rows of K bytes (K-major). Read by the
 *                          tensor-core product.
 *   section 2 at byte A2:  int32 column sums sum_k t[k][n], N entries.
 *   with A1 = round_up(round_up(N, 128)*K/4, 256), A2 = A1 + round_up(N*K, 256).
 * ------------------------------------------------------------------------------------- */
size_t hbl_packed_weights_bytes(int K, int N);

/* Scratch needed by hbl_pack_weights (bytes). */
size_t hbl_pack_weights_workspace(int K, int N);

/* Ternarise fp32 W [K][N] (row-major) into `packed` and return alpha.
 *   W          device, K*N floats, 4-byte aligned
 *   eps_w      added to alpha in the divisor (0 = plain absmean; an all-zero W gives t = 0)
 *   packed     device, packed_bytes >= hbl_packed_weights_bytes(K, N), 256-byte aligned
 *   alpha_host HOST pointer: receives alpha as float (also the device value rounded to float)
 *   workspace  device scratch of ws_bytes >= hbl_pack_weights_workspace(K, N), 16-byte aligned
 * Synchronises `stream` before returning (alpha is read back). */
hbl_status hbl_pack_weights(const float* W, int K, int N, float eps_w, void* packed,
                            size_t packed_bytes, float* alpha_host, void* workspace,
                            size_t ws_bytes, hbl_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Rotated weights: the variant of the walkthrough article's Table 5 ablation (section
 * "與其他後訓練量化方法的對比") that applies the Hadamard rotation to the weights as well as to the
 * activations. Each column of W (the K input weights of one output feature) is rotated by the
 * same transform the activations get, W' = H W along K, and W' is ternarised as in
 * hbl_pack_weights. Since H is orthonormal and symmetric, (H xhat)^T (H W) = xhat^T W: run
 * hbl_forward with the same had_block to compute the layer in the rotated bases.
 *   had_block  0 (one transform over all of K, a power of two in [256, 16384]), a power of two
 *              in [256, 16384] dividing K (block-diagonal), or 1 (no rotation: the same result
 *              as hbl_pack_weights)
 *   workspace  device scratch of ws_bytes >= hbl_pack_weights_rotated_workspace(K, N), 256-byte
 *              aligned (it receives W' in fp32, K*N*4 bytes, then the alpha partial sums)
 *   other arguments as for hbl_pack_weights. HBL_EUNSUPPORTED for another had_block.
 * The rotation runs in fp32 (log2(n) butterfly stages, then 1/sqrt(n)); alpha and the rounding
 * decision are taken in fp64 on W'. Synchronises `stream` before returning. */
size_t hbl_pack_weights_rotated_workspace(int K, int N);

hbl_status hbl_pack_weights_rotated(const float* W, int K, int N, int had_block, float eps_w,
                                    void* packed, size_t packed_bytes, float* alpha_host,
                                    void* workspace, size_t ws_bytes, hbl_stream_t stream);

/* Pack given ternary codes t [K][N] (int8 in {-1,0,1}, row-major) into `packed`.
 * Entries outside {-1,0,1} give HBL_EINVAL only through hbl_device_status (they are
 * clamped and flagged, not trapped). Asynchronous. */
hbl_status hbl_pack_ternary(const int8_t* t, int K, int N, void* packed, size_t packed_bytes,
                            hbl_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Activation side: RMSNorm -> Hadamard -> per-token quantisation, fused in one kernel.
 *
 *   r      = sqrt(mean_k x[m,k]^2 + eps_norm)                  (RMSNorm; LLaMA-like parts, article
 *   xhat   = x / r * gain  (gain may be NULL = all ones)        section "BitNet v2：原生4位激活")
 *   xr     = H xhat, H = Sylvester Walsh-Hadamard / sqrt(n)     (fast transform in O(n log n),
 *            applied to all of K when had_block = 0 (K must    article section "H-BitLinear模塊")
 *            be a power of two), or to each consecutive block
 *            of had_block features (block-diagonal)
 *   q, s   = quantiser `quant` applied per token row (see hbl_quant); a row whose statistic
 *            is 0 gives q = 0, s = 0. Rounding: nearest, ties to even. The kernels transform and
 *            decide in fp32, so a value within fp32 rounding of a .5 boundary may land on
 *            either side of it (a one-step code difference from an exact evaluation).
 * Kernels: without gain, one block of 16384 features from 17 rows, of 8192 from 65 rows, of 4096
 * from 257 rows, and blocks of 256 in rows that are not a power of two from 257 rows run the H_128
 * (or I_4 (x) H_32) Kronecker factor of the transform on the tensor cores and the rest on CUDA
 * cores; had_block = 1 runs a streaming norm-and-quantise kernel; every other shape, and fewer
 * rows, runs the CUDA-core transform. All give the same codes up to the rounding-order ties the
 * parity tests allow.
 *
 *   X       device bf16 [M][K], 16-byte aligned
 *   gain    device fp32 [K] or NULL
 *   had_block 0, or a power of two in [256, 16384] dividing K; when 0, K must be a power of two
 *           in [256, 16384]. had_block = 1 is the block-diagonal transform with blocks of one
 *           feature (H_1 = [1]), i.e. no rotation: the plain BitLinear of every other linear
 *           layer (QKV, up/gate), which the walkthrough article's section
 *           "BitNet v2：原生4位激活" runs with the same INT4/INT8 activations
 *   codes   device, M rows in `fmt` (see hbl_codes_fmt), 16-byte aligned
 *   s_x     device fp32 [M]
 * Asynchronous. */
hbl_status hbl_norm_fht_quant(const void* X, const float* gain, int M, int K, int had_block,
                              hbl_quant quant, float eps_norm, float eps_q, hbl_codes_fmt fmt,
                              void* codes, float* s_x, hbl_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Ternary x low-bit product with dequant epilogue:
 *
 *   Y[m,n] = s_x[m] * alpha * sum_k q[m,k] * t[k,n]
 *
 * (the layer's product Q_w(W) . Q_a(...) with both scales applied after the integer sum).
 *   codes, fmt, abits  activation codes as written by hbl_norm_fht_quant (abits 4 or 8)
 *   s_x      device fp32 [M]
 *   packed   blob from hbl_pack_weights / hbl_pack_ternary for this K, N
 *   Y        device [M][N] of out_dtype (fp32 or bf16), 16-byte aligned, N a multiple of 8
 *   acc_debug  device int32 [M][N] receiving the exact integer sums, or NULL
 * Kernels by token count (int8 codes): M <= 4 on CUDA cores and 5 <= M <= 256 on tcgen05
 * tensor cores, both over the 2-bit section; M > 256 on tcgen05 SM pairs over the int8
 * section. Packed int4 codes (fmt = HBL_CODES_PACKED with abits = 4) are taken by the CUDA-core
 * kernel only: M <= 8, else HBL_EUNSUPPORTED.
 * Asynchronous. The kernel may begin streaming weights before the kernel before it in the
 * stream has finished, and waits for that kernel before it reads codes or s_x; Y must not alias
 * the inputs of the kernel before it. */
hbl_status hbl_ternary_gemm(const void* codes, hbl_codes_fmt fmt, int abits, const float* s_x,
                            const void* packed, size_t packed_bytes, float alpha, int M, int N,
                            int K, void* Y, hbl_out_dtype out_dtype, int32_t* acc_debug,
                            hbl_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * The whole layer forward: hbl_norm_fht_quant into `workspace`, then hbl_ternary_gemm.
 *   workspace  device scratch, ws_bytes >= hbl_forward_workspace(M, K, quant), 256-byte aligned
 * Asynchronous. */
size_t hbl_forward_workspace(int M, int K, hbl_quant quant);

hbl_status hbl_forward(const void* X, const float* gain, const void* packed, size_t packed_bytes,
                       float alpha, int M, int K, int N, int had_block, hbl_quant quant,
                       float eps_norm, float eps_q, void* workspace, size_t ws_bytes, void* Y,
                       hbl_out_dtype out_dtype, hbl_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * One token of the layer forward (M = 1) in one launch and with no workspace: the decode
 * product computes the codes of each CTA's slice of K from the bf16 row itself (the transform's
 * stages across slices as signed sums of the row's slices, read from L2; the row statistics
 * reduced over the CTA cluster), so nothing between the row and Y reaches device memory. Same
 * layer and arguments as hbl_forward with M = 1, up to the one-step code flips any two fp32
 * evaluations may differ by. K a power of two up to 8192; had_block 0, 1, or a power of two from
 * 256 dividing K; else HBL_EUNSUPPORTED. (hbl_forward runs one token as two launches, the
 * few-row activation kernel and the decode product, which measured faster on B200: Wo 4096 ->
 * 4096 6.1 against 7.5 us.)
 *   X   device bf16 [K], 16-byte aligned;   Y   device [N] of out_dtype, 16-byte aligned
 * Asynchronous. */
hbl_status hbl_forward_decode(const void* X, const float* gain, const void* packed, size_t packed_bytes,
                              float alpha, int K, int N, int had_block, hbl_quant quant, float eps_norm,
                              float eps_q, void* Y, hbl_out_dtype out_dtype, hbl_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Low-bit attention states: QKV quantised after RoPE to unsigned integers per head.
 *
 * The walkthrough article (section "實驗結果", Tables 2-3) quantises the QKV states after RoPE,
 * each head directly to unsigned integers with the absmax function and no calibration data, and
 * reports that a 3-bit KV cache matches full precision. Its formulas were lost; this library
 * reads them as follows, per token m and head h (D features):
 *   RoPE (Q and K only; pos given): feature f < D/2 pairs with f + D/2, both turned by the angle
 *        pos[m] * theta^(-2f/D):  (x_f, x_{f+D/2}) -> (x_f c - x_{f+D/2} s, x_f s + x_{f+D/2} c)
 *   gamma[m][h] = max_d |x[d]|
 *   u[d] = RoundClip((2^b - 1)/2 * (x[d]/gamma + 1), 0, 2^b - 1)   (a zero head: x/gamma = 0)
 *   dequantised: x~[d] = (2 u[d] - (2^b - 1)) * gamma / (2^b - 1)
 * Codes of a head form a little-endian bit string of D*b bits: code d at bits [b d, b d + b)
 * (bit i of the string is bit i%8 of byte i/8); heads follow each other, [M][H][D*b/8] bytes.
 *
 *   X          device bf16; token m, head h starts at element m*row_stride + h*D; 16-byte aligned
 *   row_stride elements between tokens, >= H*D and a multiple of 8 (so Q, K or V can be read in
 *              place from a fused QKV output)
 *   pos        device int32 [M] token positions, or NULL for no rotation (the V states)
 *   rope_theta RoPE base (> 1; LLaMA uses 10000); ignored when pos is NULL
 *   D          64, 128 or 256; bits 2, 3, 4 or 8 (else HBL_EUNSUPPORTED)
 *   codes      device, codes_bytes >= hbl_qkv_codes_bytes(M, H, D, bits), 16-byte aligned
 *   gamma      device fp32 [M][H]
 * The angle is formed and reduced modulo 2 pi in fp64, its cosine and sine rounded to fp32; the
 * rotation and the rounding decision run in fp32. Asynchronous. */
size_t hbl_qkv_codes_bytes(int M, int H, int D, int bits);

hbl_status hbl_qkv_quant(const void* X, size_t row_stride, const int32_t* pos, float rope_theta,
                         int M, int H, int D, int bits, void* codes, size_t codes_bytes,
                         float* gamma, hbl_stream_t stream);

/* Dequantise codes written by hbl_qkv_quant into bf16 Y [M][H][D] (16-byte aligned), rounded to
 * nearest even. Asynchronous. */
hbl_status hbl_qkv_dequant(const void* codes, const float* gamma, int M, int H, int D, int bits,
                           void* Y, hbl_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * hbl_forward without a caller-provided workspace. This entry point has no counterpart in the
 * method's description; it exists for callers that cannot call cudaMalloc, e.g. host code whose
 * device memory belongs to another component's allocator, or a runtime that allocates device
 * memory only at start-up and never on the request path.
 *
 * Same arguments and result as hbl_forward, minus workspace/ws_bytes. The scratch (activation
 * codes and per-token scales, hbl_forward_workspace(M, K, quant) bytes) lives in a 16 MiB array
 * inside the library's device image (a static __device__ array): every GPU that loads the library
 * holds those 16 MiB until the process exits, and no call allocates or frees device memory.
 *   - Requests needing more than 16 MiB of scratch (roughly M * K > 16.7 million) return
 *     HBL_EUNSUPPORTED before any device work; use hbl_forward with your own workspace for them.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     with that device current and keeps it for the life of the process; make that first call
 *     before any stream capture. Resetting the device (cudaDeviceReset, or any other teardown of
 *     its primary context) after that first call is not supported: the kept address would be
 *     stale.
 *   - All calls on a device share the one array, and each call leaves its scratch contents
 *     behind. Calls that may overlap on the GPU (different streams without ordering between
 *     them) race on it: serialise them, or use hbl_forward.
 * Asynchronous, like hbl_forward. */
hbl_status hbl_forward_static(const void* X, const float* gain, const void* packed,
                              size_t packed_bytes, float alpha, int M, int K, int N, int had_block,
                              hbl_quant quant, float eps_norm, float eps_q, void* Y,
                              hbl_out_dtype out_dtype, hbl_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HBL_H_ */
