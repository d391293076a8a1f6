"""wq_dequantize (the Per-group(128) article's sec. 3.4 dequantize, the step before its bf16
matmul) against the oracle: bf16(fl32(q * step)) bit-exact, every width, edge weights and a
full-size shape; and the container round trip (sec. 3.3 storage keys) feeding the device."""
import numpy as np
import pytest

import oracle
import bit_weight_quantization_wq_b200 as wq
from bit_weight_quantization_wq_b200 import container, synth
from helpers import edge_weight, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits", [3, 4, 5, 6, 7])
@pytest.mark.parametrize("N,K", [(1, 128), (37, 1280), (300, 640)])
def test_dequantize_bit_exact(bits, N, K):
    import torch
    W = edge_weight(np.random.default_rng(N * K + bits), N, K, bits)
    packed, scales = wq.wq_quantize_pack(to_dev_bf16(W), bits)
    w_hat = wq.wq_dequantize(packed, scales, bits, K)
    torch.cuda.synchronize()
    codes, s_o = oracle.quantize(W, bits)
    assert np.array_equal(from_dev_bf16(w_hat), oracle.dequant_bf16(codes, s_o, bits))


def test_dequantize_full_size():
    import torch
    W = synth.wan_weight(1)                    # 13824 x 5120
    packed, scales = wq.wq_quantize_pack(to_dev_bf16(W), 5)
    w_hat = wq.wq_dequantize(packed, scales, 5, W.shape[1])
    torch.cuda.synchronize()
    codes, s_o = oracle.quantize(W, 5)
    assert np.array_equal(from_dev_bf16(w_hat), oracle.dequant_bf16(codes, s_o, 5))


def test_container_to_device(tmp_path):
    """Quantize on the GPU, save the page's keys, load them back onto the GPU: the linear layer
    and the dequantized weight come out the same as from the original device tensors."""
    import torch
    rng = np.random.default_rng(8)
    W = synth.weight(rng, 256, 512, 0.02)
    x = to_dev_bf16(synth.activations(rng, 64, 512))
    packed, scales = wq.wq_quantize_pack(to_dev_bf16(W), 6)
    path = str(tmp_path / "q.safetensors")
    container.save(path, {"layer": (packed, scales, 6)})
    e = container.load(path, device="cuda")["layer"]
    assert e["bits"] == 6 and e["nin"] == 512
    y0 = wq.wq_linear(x, packed, scales, 6, 256)
    y1 = wq.wq_linear(x, e["packed"], e["scales"], e["bits"], 256)
    d0 = wq.wq_dequantize(packed, scales, 6, 512)
    d1 = wq.wq_dequantize(e["packed"], e["scales"], e["bits"], e["nin"])
    torch.cuda.synchronize()
    assert torch.equal(y0, y1) and torch.equal(d0, d1)
