"""wq_linear_no_workspace: the quantized linear layer for callers that cannot allocate device
memory when they run it. The low-rank branch's scratch then comes from a buffer compiled
into the library instead of a caller workspace.

Checked through the C ABI (ctypes, raw device pointers): two calls in a row on each kernel
family give bit for bit the result of wq_linear with its own workspace (the same kernels
run in the same order, only the scratch address differs), the first of them is also
compared with the CPU oracle within the GEMM tolerance of the parity tests, and a size
whose scratch exceeds the static buffer is refused before anything runs. This file is
collected last so that a run that stops at the first failure has already run every other
test.
"""
import ctypes

import numpy as np
import pytest

import bit_weight_quantization_wq_b200 as wq
from bit_weight_quantization_wq_b200 import _binding as B
from bit_weight_quantization_wq_b200 import synth
import oracle
from helpers import assert_linear_close, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 4 << 20          # WQ_STATIC_SCRATCH_BYTES in include/wq.h


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_no_workspace(x, packed, scales, bits, N, L1, L2, bias, y):
    import torch
    M, K = x.shape
    rank = 0 if L1 is None else L1.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return B.lib().wq_linear_no_workspace(_ptr(x), M, K, _ptr(packed), _ptr(scales), bits, 128, N,
                                          _ptr(L1), _ptr(L2), rank, _ptr(bias), _ptr(y), stream)


@pytest.mark.parametrize("M,N,K,bits,rank", [(5, 264, 384, 4, 32),      # small-M kernel family
                                             (300, 520, 768, 5, 32),    # tensor-core kernel family
                                             (64, 256, 512, 3, 0)])     # no low-rank branch: no scratch
def test_matches_workspace_call_twice(M, N, K, bits, rank):
    import torch
    rng = np.random.default_rng(M + N + K + bits)
    W = synth.weight(rng, N, K, 0.02)
    x = to_dev_bf16(synth.activations(rng, M, K))
    b = to_dev_bf16(synth.bias(rng, N))
    L1 = L2 = None
    if rank:
        L1 = to_dev_bf16(synth.f32_to_bf16_bits(rng.standard_normal((K, rank)).astype(np.float32) * 0.05))
        L2 = to_dev_bf16(synth.f32_to_bf16_bits(rng.standard_normal((rank, N)).astype(np.float32) * 0.05))
    packed, scales = wq.wq_quantize_pack(to_dev_bf16(W), bits)
    ref = wq.wq_linear(x, packed, scales, bits, N, L1=L1, L2=L2, bias=b)
    torch.cuda.synchronize()
    ref_bits = from_dev_bf16(ref)
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = _call_no_workspace(x, packed, scales, bits, N, L1, L2, b, y)
        assert st == B.WQ_OK, B.lib().wq_last_error().decode()
        torch.cuda.synchronize()
        got = from_dev_bf16(y)
        assert np.array_equal(got, ref_bits), f"call {call}: {int((got != ref_bits).sum())} outputs differ"
        if call == 0:
            codes, s_o = oracle.quantize(W, bits)
            h = lambda t: None if t is None else from_dev_bf16(t)
            y_o = oracle.linear_rows(from_dev_bf16(x), oracle.dequant(codes, s_o, bits), h(L1), h(L2), h(b))
            assert_linear_close(got, y_o, f"no-workspace {M}x{N}x{K} b{bits} r{rank}")
    assert wq.wq_device_status() == 0


def test_refuses_scratch_beyond_static_buffer():
    import torch
    M, N, K, bits, rank = 20000, 256, 128, 4, 32
    assert wq.wq_linear_workspace_bytes(M, N, K, bits, rank) > STATIC_SCRATCH_BYTES
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    packed = torch.empty((N, K * bits // 8), dtype=torch.uint8, device="cuda")
    scales = torch.empty((N, 1), dtype=torch.float32, device="cuda")
    L1 = torch.empty((K, rank), dtype=torch.bfloat16, device="cuda")
    L2 = torch.empty((rank, N), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = B.lib().wq_linear_no_workspace(_ptr(x), M, K, _ptr(packed), _ptr(scales), bits, 128, N,
                                        _ptr(L1), _ptr(L2), rank, None, _ptr(y), stream)
    assert st == B.WQ_ERR_WORKSPACE
    assert b"static buffer" in B.lib().wq_last_error()
