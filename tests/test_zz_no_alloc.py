"""hbl_forward_static: the forward pass for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (their device memory belongs to another component's
allocator, or they allocate only at start-up), so they cannot hand hbl_forward a workspace.
hbl_forward_static keeps that scratch in a fixed 16 MiB array inside the library instead. These
tests call it through the C ABI and compare it with hbl_forward on its own workspace, on two
calls in a row (the second call reuses the scratch the first one left behind).

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

import hadamard_bit_quant_hbl_b200 as hbl
from hadamard_bit_quant_hbl_b200 import inputs

_ARGTYPES = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float, ctypes.c_int,
             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_float, ctypes.c_void_p,
             ctypes.c_int, ctypes.c_void_p]


def _entry():
    f = hbl.lib().hbl_forward_static
    f.restype = ctypes.c_int
    f.argtypes = _ARGTYPES
    return f


def test_static_forward_rejects_requests_beyond_its_scratch():
    # 1024 x 32768 needs 32 MiB of scratch: refused with its own status before any device work.
    # Every pointer is NULL, so if the size check ever stopped refusing, the call would return
    # HBL_EINVAL from the pointer checks instead (and still launch nothing).
    f = _entry()
    st = f(None, None, None, 0, 1.0, 1024, 32768, 64, 0, hbl.HBL_Q_A4_ABSMEAN, 1e-6, 0.0, None,
           hbl.HBL_OUT_F32, None)
    assert st == hbl.HBL_EUNSUPPORTED, hbl.hbl_status_string(st)


@pytest.mark.gpu
def test_static_forward_matches_forward_on_two_calls():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    f = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    cases = [("wdown_3b_a4", 300, hbl.HBL_OUT_F32),   # SM-pair tensor-core product
             ("wo_7b_a4", 5, hbl.HBL_OUT_BF16),       # swapped-operand tensor-core product
             ("wdown_7b_a4", 3, hbl.HBL_OUT_F32)]     # CUDA-core product (int8 codes, M <= 4)
    results = []
    for name, M, out_dtype in cases:
        spec = inputs.WORKLOADS[name].with_m(M)
        x = inputs.activations(spec)
        packed, alpha = hbl.hbl_pack_weights(torch.from_numpy(inputs.weights(spec)).cuda())
        X = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
        ydt = torch.float32 if out_dtype == hbl.HBL_OUT_F32 else torch.bfloat16
        Y = torch.full((M, spec.N), float("nan"), dtype=ydt, device="cuda")
        st = f(X.data_ptr(), None, packed.data_ptr(), packed.numel(), alpha, M, spec.K, spec.N, spec.had_block,
               hbl.HBL_Q_A4_ABSMEAN, 1e-6, 0.0, Y.data_ptr(), out_dtype, stream)
        assert st == hbl.HBL_OK, hbl.hbl_status_string(st)
        results.append((X, packed, alpha, spec, out_dtype, Y))
    torch.cuda.synchronize()
    assert hbl.hbl_device_status() == hbl.HBL_OK
    for X, packed, alpha, spec, out_dtype, Y in results:
        ref = hbl.hbl_forward(X, packed, alpha, spec.N, None, spec.had_block, hbl.HBL_Q_A4_ABSMEAN,
                              out_dtype=out_dtype)
        y, r = Y.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.all(np.isfinite(y))
        rel = np.linalg.norm(y - r, axis=1) / np.linalg.norm(r, axis=1)
        assert np.all(rel <= 1e-5), rel.max()
