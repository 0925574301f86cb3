"""H-BitLinear forward pass (BitNet v2) on B200: Python binding of libhbl.so.

Every function here marshals torch tensors into the C ABI declared in include/hbl.h and calls
the CUDA library; no step of the computation runs in Python. PyTorch provides device memory
and streams only. If libhbl.so is missing or cannot be loaded, importing the binding's
functions raises: there is no fallback path.

The names follow the C ABI (hbl_pack_weights, hbl_norm_fht_quant, hbl_ternary_gemm,
hbl_forward, ...). Pointer arguments become CUDA tensors; `stream` defaults to torch's current
stream on the tensors' device.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "HBL_OK", "HBL_EINVAL", "HBL_EUNSUPPORTED", "HBL_ECUDA", "HBL_ETIMEOUT",
    "HBL_Q_A8_ABSMAX", "HBL_Q_A4_ABSMEAN", "HBL_Q_A4_ABSMAX",
    "HBL_CODES_PACKED", "HBL_CODES_I8", "HBL_OUT_F32", "HBL_OUT_BF16",
    "HblError", "lib", "library_path",
    "hbl_status_string", "hbl_device_status", "hbl_selftest_timeout", "hbl_packed_weights_bytes", "hbl_pack_weights_workspace",
    "hbl_pack_weights", "hbl_pack_weights_rotated", "hbl_pack_weights_rotated_workspace", "hbl_pack_ternary",
    "hbl_norm_fht_quant", "hbl_ternary_gemm",
    "hbl_forward_workspace", "hbl_forward", "hbl_forward_decode", "codes_row_bytes",
    "hbl_qkv_codes_bytes", "hbl_qkv_quant", "hbl_qkv_dequant",
]

HBL_OK, HBL_EINVAL, HBL_EUNSUPPORTED, HBL_ECUDA, HBL_ETIMEOUT = range(5)
HBL_Q_A8_ABSMAX, HBL_Q_A4_ABSMEAN, HBL_Q_A4_ABSMAX = range(3)
HBL_CODES_PACKED, HBL_CODES_I8 = range(2)
HBL_OUT_F32, HBL_OUT_BF16 = range(2)

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libhbl.so")

_lib = None
_lock = threading.Lock()

_c_void_p = ctypes.c_void_p
_c_int = ctypes.c_int
_c_float = ctypes.c_float
_c_size_t = ctypes.c_size_t

_SIGNATURES = {
    "hbl_status_string": (ctypes.c_char_p, [_c_int]),
    "hbl_last_cuda_error": (_c_int, []),
    "hbl_device_status": (_c_int, [_c_void_p]),
    "hbl_selftest_timeout": (_c_int, [_c_int, _c_void_p]),
    "hbl_packed_weights_bytes": (_c_size_t, [_c_int, _c_int]),
    "hbl_pack_weights_workspace": (_c_size_t, [_c_int, _c_int]),
    "hbl_pack_weights": (_c_int, [_c_void_p, _c_int, _c_int, _c_float, _c_void_p, _c_size_t,
                                  ctypes.POINTER(_c_float), _c_void_p, _c_size_t, _c_void_p]),
    "hbl_pack_weights_rotated_workspace": (_c_size_t, [_c_int, _c_int]),
    "hbl_pack_weights_rotated": (_c_int, [_c_void_p, _c_int, _c_int, _c_int, _c_float, _c_void_p, _c_size_t,
                                          ctypes.POINTER(_c_float), _c_void_p, _c_size_t, _c_void_p]),
    "hbl_pack_ternary": (_c_int, [_c_void_p, _c_int, _c_int, _c_void_p, _c_size_t, _c_void_p]),
    "hbl_norm_fht_quant": (_c_int, [_c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_float,
                                    _c_float, _c_int, _c_void_p, _c_void_p, _c_void_p]),
    "hbl_ternary_gemm": (_c_int, [_c_void_p, _c_int, _c_int, _c_void_p, _c_void_p, _c_size_t, _c_float,
                                  _c_int, _c_int, _c_int, _c_void_p, _c_int, _c_void_p, _c_void_p]),
    "hbl_forward_workspace": (_c_size_t, [_c_int, _c_int, _c_int]),
    "hbl_qkv_codes_bytes": (_c_size_t, [_c_int, _c_int, _c_int, _c_int]),
    "hbl_qkv_quant": (_c_int, [_c_void_p, _c_size_t, _c_void_p, _c_float, _c_int, _c_int, _c_int, _c_int, _c_void_p,
                               _c_size_t, _c_void_p, _c_void_p]),
    "hbl_qkv_dequant": (_c_int, [_c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_void_p, _c_void_p]),
    "hbl_forward": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_size_t, _c_float, _c_int, _c_int, _c_int,
                             _c_int, _c_int, _c_float, _c_float, _c_void_p, _c_size_t, _c_void_p, _c_int,
                             _c_void_p]),
    "hbl_forward_decode": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_size_t, _c_float, _c_int, _c_int, _c_int,
                                    _c_int, _c_float, _c_float, _c_void_p, _c_int, _c_void_p]),
}


class HblError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = lib().hbl_status_string(status).decode()
        if status == HBL_ECUDA:
            msg += f" (cudaError {lib().hbl_last_cuda_error()})"
        super().__init__(f"{what}: {msg}")


def lib() -> ctypes.CDLL:
    """The loaded libhbl.so (loaded once; raises if it is missing)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(library_path):
                    raise ImportError(
                        f"libhbl.so not found at {library_path}; build it with "
                        "`python -m hadamard_bit_quant_hbl_b200._build` (needs nvcc)")
                L = ctypes.CDLL(library_path)
                for name, (res, args) in _SIGNATURES.items():
                    f = getattr(L, name)
                    f.restype = res
                    f.argtypes = args
                _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != HBL_OK:
        raise HblError(status, what)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream, like) -> int:
    import torch

    if stream is None:
        return torch.cuda.current_stream(like.device).cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def hbl_status_string(status: int) -> str:
    return lib().hbl_status_string(status).decode()


def hbl_device_status(stream=None) -> int:
    """Synchronise `stream`, read and clear the device error flag; returns an HBL_* status."""
    import torch

    s = torch.cuda.current_stream().cuda_stream if stream is None else _stream(stream, None)
    return lib().hbl_device_status(s)


def hbl_selftest_timeout(limit_ms: int = 50, stream=None) -> None:
    """Launch the time-out self-test kernel (its wait runs out after `limit_ms`); the next
    hbl_device_status() reports HBL_ETIMEOUT."""
    import torch

    s = torch.cuda.current_stream().cuda_stream if stream is None else _stream(stream, None)
    _check(lib().hbl_selftest_timeout(int(limit_ms), s), "hbl_selftest_timeout")


def hbl_packed_weights_bytes(K: int, N: int) -> int:
    return lib().hbl_packed_weights_bytes(K, N)


def hbl_pack_weights_workspace(K: int, N: int) -> int:
    return lib().hbl_pack_weights_workspace(K, N)


def hbl_forward_workspace(M: int, K: int, quant: int) -> int:
    return lib().hbl_forward_workspace(M, K, quant)


def codes_row_bytes(K: int, quant: int, fmt: int) -> int:
    """Bytes of one token row of activation codes in the given format."""
    return K // 2 if (fmt == HBL_CODES_PACKED and quant != HBL_Q_A8_ABSMAX) else K


def _u8_empty(nbytes: int, device):
    import torch

    # 256-byte aligned view into a slightly larger buffer (torch's allocator aligns to 512 anyway)
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def hbl_pack_weights(W, eps_w: float = 0.0, packed=None, workspace=None, stream=None):
    """Ternarise fp32 W [K, N] on the device. Returns (packed uint8 blob, alpha)."""
    K, N = W.shape
    if packed is None:
        packed = _u8_empty(hbl_packed_weights_bytes(K, N), W.device)
    if workspace is None:
        workspace = _u8_empty(hbl_pack_weights_workspace(K, N), W.device)
    alpha = _c_float(0.0)
    _check(lib().hbl_pack_weights(_ptr(W), K, N, float(eps_w), _ptr(packed), packed.numel(), ctypes.byref(alpha),
                                  _ptr(workspace), workspace.numel(), _stream(stream, W)), "hbl_pack_weights")
    return packed, alpha.value


def hbl_pack_weights_rotated_workspace(K: int, N: int) -> int:
    return lib().hbl_pack_weights_rotated_workspace(K, N)


def hbl_pack_weights_rotated(W, had_block: int = 0, eps_w: float = 0.0, packed=None, workspace=None, stream=None):
    """Rotate each column of fp32 W [K, N] by the activations' Hadamard transform along K, then
    ternarise. Returns (packed uint8 blob, alpha)."""
    K, N = W.shape
    if packed is None:
        packed = _u8_empty(hbl_packed_weights_bytes(K, N), W.device)
    if workspace is None:
        workspace = _u8_empty(hbl_pack_weights_rotated_workspace(K, N), W.device)
    alpha = _c_float(0.0)
    _check(lib().hbl_pack_weights_rotated(_ptr(W), K, N, int(had_block), float(eps_w), _ptr(packed), packed.numel(),
                                          ctypes.byref(alpha), _ptr(workspace), workspace.numel(),
                                          _stream(stream, W)), "hbl_pack_weights_rotated")
    return packed, alpha.value


def hbl_pack_ternary(t, packed=None, stream=None):
    """Pack given ternary codes t [K, N] (int8 in {-1, 0, 1}). Returns the packed blob."""
    K, N = t.shape
    if packed is None:
        packed = _u8_empty(hbl_packed_weights_bytes(K, N), t.device)
    _check(lib().hbl_pack_ternary(_ptr(t), K, N, _ptr(packed), packed.numel(), _stream(stream, t)),
           "hbl_pack_ternary")
    return packed


def hbl_norm_fht_quant(X, gain=None, had_block: int = 0, quant: int = HBL_Q_A4_ABSMEAN, eps_norm: float = 1e-6,
                       eps_q: float = 0.0, fmt: int = HBL_CODES_PACKED, codes=None, s_x=None, stream=None):
    """RMSNorm -> Hadamard -> per-token quantisation of bf16 X [M, K]. Returns (codes, s_x)."""
    import torch

    M, K = X.shape
    if codes is None:
        codes = torch.empty((M, codes_row_bytes(K, quant, fmt)), dtype=torch.uint8, device=X.device)
    if s_x is None:
        s_x = torch.empty(M, dtype=torch.float32, device=X.device)
    _check(lib().hbl_norm_fht_quant(_ptr(X), _ptr(gain), M, K, had_block, quant, float(eps_norm), float(eps_q), fmt,
                                    _ptr(codes), _ptr(s_x), _stream(stream, X)), "hbl_norm_fht_quant")
    return codes, s_x


def hbl_ternary_gemm(codes, fmt: int, abits: int, s_x, packed, alpha: float, N: int, K: int, Y=None,
                     out_dtype: int = HBL_OUT_F32, acc_debug=None, stream=None):
    """Y[m, n] = s_x[m] * alpha * sum_k q[m, k] t[k, n]. Returns Y."""
    import torch

    M = codes.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32 if out_dtype == HBL_OUT_F32 else torch.bfloat16,
                        device=codes.device)
    _check(lib().hbl_ternary_gemm(_ptr(codes), fmt, abits, _ptr(s_x), _ptr(packed), packed.numel(), float(alpha), M,
                                  N, K, _ptr(Y), out_dtype, _ptr(acc_debug), _stream(stream, codes)),
           "hbl_ternary_gemm")
    return Y


def hbl_forward(X, packed, alpha: float, N: int, gain=None, had_block: int = 0, quant: int = HBL_Q_A4_ABSMEAN,
                eps_norm: float = 1e-6, eps_q: float = 0.0, workspace=None, Y=None, out_dtype: int = HBL_OUT_F32,
                stream=None):
    """The whole H-BitLinear forward of bf16 X [M, K] with packed weights. Returns Y [M, N]."""
    import torch

    M, K = X.shape
    if workspace is None:
        workspace = _u8_empty(hbl_forward_workspace(M, K, quant), X.device)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32 if out_dtype == HBL_OUT_F32 else torch.bfloat16, device=X.device)
    _check(lib().hbl_forward(_ptr(X), _ptr(gain), _ptr(packed), packed.numel(), float(alpha), M, K, N, had_block,
                             quant, float(eps_norm), float(eps_q), _ptr(workspace), workspace.numel(), _ptr(Y),
                             out_dtype, _stream(stream, X)), "hbl_forward")
    return Y


def hbl_forward_decode(X, packed, alpha: float, N: int, gain=None, had_block: int = 0, quant: int = HBL_Q_A4_ABSMEAN,
                       eps_norm: float = 1e-6, eps_q: float = 0.0, Y=None, out_dtype: int = HBL_OUT_F32, stream=None):
    """One token of the forward in one launch, no workspace: bf16 X [1, K] (K a power of two up to
    8192) with packed weights. Returns Y [1, N]."""
    import torch

    M, K = X.shape
    if M != 1:
        raise ValueError("hbl_forward_decode takes one token")
    if Y is None:
        Y = torch.empty((1, N), dtype=torch.float32 if out_dtype == HBL_OUT_F32 else torch.bfloat16, device=X.device)
    _check(lib().hbl_forward_decode(_ptr(X), _ptr(gain), _ptr(packed), packed.numel(), float(alpha), K, N, had_block,
                                    quant, float(eps_norm), float(eps_q), _ptr(Y), out_dtype, _stream(stream, X)),
           "hbl_forward_decode")
    return Y


def hbl_qkv_codes_bytes(M: int, H: int, D: int, bits: int) -> int:
    return lib().hbl_qkv_codes_bytes(M, H, D, bits)


def hbl_qkv_quant(X, H: int, D: int, bits: int = 3, pos=None, rope_theta: float = 10000.0, row_stride=None,
                  codes=None, gamma=None, stream=None):
    """RoPE (when `pos`, int32 [M], is given) then per-head unsigned absmax quantisation of bf16 X,
    token rows of `row_stride` elements (default H*D) holding H heads of D features from the
    row start. Returns (codes uint8 [M, H, D*bits/8], gamma fp32 [M, H])."""
    import torch

    M = X.shape[0]
    if row_stride is None:
        row_stride = H * D
    if codes is None:
        codes = torch.empty((M, H, D * bits // 8), dtype=torch.uint8, device=X.device)
    if gamma is None:
        gamma = torch.empty((M, H), dtype=torch.float32, device=X.device)
    if not X.is_cuda:
        raise ValueError("expected a CUDA tensor")
    _check(lib().hbl_qkv_quant(X.data_ptr(), int(row_stride), _ptr(pos), float(rope_theta), M, H, D, bits,
                               _ptr(codes), codes.numel(), _ptr(gamma), _stream(stream, X)), "hbl_qkv_quant")
    return codes, gamma


def hbl_qkv_dequant(codes, gamma, D: int, bits: int, Y=None, stream=None):
    """bf16 [M, H, D] from codes and gamma written by hbl_qkv_quant."""
    import torch

    M, H = gamma.shape
    if Y is None:
        Y = torch.empty((M, H, D), dtype=torch.bfloat16, device=codes.device)
    _check(lib().hbl_qkv_dequant(_ptr(codes), _ptr(gamma), M, H, D, bits, _ptr(Y), _stream(stream, codes)),
           "hbl_qkv_dequant")
    return Y
