"""Full-size parity of the two whole-model workloads (CUDA path through the C ABI vs the
CPU oracle). Weights are drawn on the GPU with seeded torch generators and copied to the
host for the oracle, one tensor at a time.

  * the mixed-precision DiT block stack: all 40 blocks (8 x 5120x5120, 13824x5120,
    5120x13824 each, widths from the mixed-precision histogram), 4096 tokens pushed through
    all 400 linears in order. Each layer's input is the previous output rescaled to unit rms
    by one scalar (a linear map, outside the check), which keeps the 400-layer chain finite
    in bf16; each layer is checked on sampled token rows against the oracle fed the same
    bf16 input, and its steps bit-exact;
  * the whole-model quantize+pack (49 blocks, 490 tensors, 17.2 B weights): every packed
    byte and every step of every tensor bit-exact against the oracle, through the batched
    entry point, one block per call.
"""
import numpy as np
import pytest

import oracle
import bit_weight_quantization_wq_b200 as wq
from bit_weight_quantization_wq_b200 import synth
from helpers import assert_linear_close, from_dev_bf16, to_dev_bf16

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _sample_rows(M, n, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, size=min(n, M), replace=False)]))


def test_mixed_stack_all_40_blocks():
    import torch
    x_dev = to_dev_bf16(synth.wan_x(4096, config=4))
    layers = 0
    for block in range(40):
        widths = synth.mixed_bits(len(synth.BLOCK_SHAPES), config=4, block=block)
        for i, ((N, K), bits) in enumerate(zip(synth.BLOCK_SHAPES, widths)):
            assert x_dev.shape == (4096, K)          # the block's widths always chain
            W = synth.weight_torch(synth.torch_generator(4, block, i), N, K, 0.015)
            packed, scales = wq.wq_quantize_pack(W, bits)
            y = wq.wq_linear(x_dev, packed, scales, bits, N)
            torch.cuda.synchronize()
            rows = _sample_rows(4096, 6, block * 16 + i)
            rows_t = torch.from_numpy(rows).cuda()
            codes, s_o = oracle.quantize(from_dev_bf16(W), bits)
            s = scales.cpu().numpy()
            assert (s.view(np.uint32) == s_o.view(np.uint32)).all(), (block, i)
            y_o = oracle.linear_rows(from_dev_bf16(x_dev[rows_t]), oracle.dequant(codes, s_o, bits), None, None, None)
            assert_linear_close(from_dev_bf16(y[rows_t]), y_o, f"stack block {block} layer {i} b{bits} {N}x{K}")
            yf = y.float()
            x_dev = (yf / yf.square().mean().sqrt()).to(torch.bfloat16)
            layers += 1
    assert layers == 400
    assert wq.wq_device_status() == 0


def test_model_pack_all_490_tensors():
    import torch
    n_tensors = params = packed_total = 0
    snrs = []
    for block in range(49):
        widths = synth.mixed_bits(len(synth.BLOCK_SHAPES), config=5, block=block)
        Ws = [synth.weight_torch(synth.torch_generator(5, block, i), N, K, 0.015)
              for i, (N, K) in enumerate(synth.BLOCK_SHAPES)]
        outs = wq.wq_quantize_pack_many(list(zip(Ws, widths)))
        torch.cuda.synchronize()
        for i, (W, bits, (packed, scales)) in enumerate(zip(Ws, widths, outs)):
            Wh = from_dev_bf16(W)
            codes, s_o = oracle.quantize(Wh, bits)
            p = packed.cpu().numpy()
            same = p == oracle.pack(codes, bits)
            assert same.all(), f"block {block} tensor {i} b{bits}: {int((~same).sum())} packed bytes differ"
            s = scales.cpu().numpy()
            assert (s.view(np.uint32) == s_o.view(np.uint32)).all(), f"block {block} tensor {i}: steps differ"
            n_tensors += 1
            params += W.numel()
            packed_total += p.size + 4 * s.size
            if i == block % len(Ws):
                # quantization SNR of one tensor per block, from the (identical) codes
                w = synth.bf16_bits_to_f32(Wh).astype(np.float64)
                snrs.append(oracle.snr_db(w, oracle.dequant(codes, s_o, bits)))
                assert snrs[-1] > 3.0 * bits, (block, i, bits, snrs[-1])
        del Ws, outs
    assert n_tensors == 490 and params == 49 * (8 * 5120 * 5120 + 2 * 13824 * 5120)
    assert 0.25 < packed_total / (2 * params) < 0.40
    assert wq.wq_device_status() == 0
