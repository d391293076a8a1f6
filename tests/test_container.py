"""The quantized-weight container (Per-group(128) article, sec. 3.3 storage format: per tensor
_packed, _scales, _bw, _nin): round trip on the host, and the file read back by the
independent safetensors library. No GPU."""
import numpy as np

import oracle
from bit_weight_quantization_wq_b200 import container, synth


def _tensors():
    rng = np.random.default_rng(4)
    out = {}
    for name, (N, K, bits) in {"blocks.0.attn.q": (64, 256, 5), "blocks.0.ffn.up": (96, 128, 3),
                               "blocks.1.ffn.down": (32, 384, 7)}.items():
        W = synth.weight(rng, N, K, 0.02)
        packed, scales = oracle.quantize_pack(W, bits)
        out[name] = (packed, scales, bits)
    return out


def test_round_trip(tmp_path):
    t = _tensors()
    path = str(tmp_path / "model.safetensors")
    container.save(path, t, metadata={"target_bpw": 5.0})
    back = container.load(path)
    assert sorted(back) == sorted(t)
    for name, (packed, scales, bits) in t.items():
        e = back[name]
        assert e["bits"] == bits and e["nin"] == packed.shape[1] * 8 // bits
        assert np.array_equal(e["packed"], packed) and np.array_equal(e["scales"].view(np.uint32), scales.view(np.uint32))


def test_file_is_valid_safetensors(tmp_path):
    from safetensors.numpy import load_file
    t = _tensors()
    path = str(tmp_path / "model.safetensors")
    container.save(path, t)
    d = load_file(path)
    assert len(d) == 4 * len(t)
    for name, (packed, scales, bits) in t.items():
        assert np.array_equal(d[f"{name}_packed"], packed)
        assert d[f"{name}_scales"].dtype == np.float32 and np.array_equal(d[f"{name}_scales"], scales)
        assert d[f"{name}_bw"].dtype == np.int8 and int(d[f"{name}_bw"]) == bits
        assert d[f"{name}_nin"].dtype == np.int32 and int(d[f"{name}_nin"]) == packed.shape[1] * 8 // bits


def test_oracle_dequant_bf16_is_the_rounded_dequant():
    """dequant_bf16 is dequant rounded to bf16: within half a bf16 ulp of the fp32 value, and
    exactly equal to it wherever the fp32 value is itself a bf16 number."""
    rng = np.random.default_rng(2)
    W = synth.weight(rng, 16, 256, 0.02)
    codes, scales = oracle.quantize(W, 4)
    d32 = oracle.dequant(codes, scales, 4).astype(np.float64)
    d16 = synth.bf16_bits_to_f32(oracle.dequant_bf16(codes, scales, 4)).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(d32), 1e-30))) - 7)
    assert np.all(np.abs(d16 - d32) <= ulp / 2)
    exact = (oracle.dequant(codes, scales, 4).view(np.uint32) & 0xFFFF) == 0
    assert np.array_equal(d16[exact], d32[exact])
