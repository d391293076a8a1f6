"""numpy twin of the C oracle, used only to cross-check it (test infrastructure).

Same arithmetic, written with numpy's vectorised fp32 operations (IEEE division,
np.rint = round half to even) instead of scalar C loops. Per-group(128) article,
sec. 3.1 (quantize), 3.3 (packing), 3.4 (dequantize).
"""
import numpy as np


def bf16_bits_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def quantize(W_bits, bits, group=128):
    W = bf16_bits_to_f32(W_bits)
    N, K = W.shape
    wg = W.reshape(N, K // group, group)
    abs_max = np.abs(wg).max(axis=-1) * np.float32(1.01)
    levels = np.float32((1 << bits) - 1)
    step = (np.float32(2.0) * abs_max) / levels
    with np.errstate(divide="ignore", invalid="ignore"):
        r = wg / step[..., None]
    q = np.rint(r)
    q = np.where(step[..., None] == 0, np.float32(0), q)
    q_max = ((1 << bits) - 1) // 2
    q = np.clip(q, -q_max, q_max).astype(np.int32)
    codes = (q + (1 << (bits - 1))).astype(np.uint8).reshape(N, K)
    return codes, step.astype(np.float32)


def pack(codes, bits):
    codes = np.asarray(codes, np.uint8)
    N, K = codes.shape
    # expand every code into its bits, most significant first, then regroup by 8
    shifts = np.arange(bits - 1, -1, -1, dtype=np.uint8)
    stream = ((codes[..., None] >> shifts) & 1).reshape(N, K * bits)
    return np.packbits(stream, axis=1, bitorder="big")


def unpack(packed, K, bits):
    packed = np.asarray(packed, np.uint8)
    N = packed.shape[0]
    stream = np.unpackbits(packed, axis=1, bitorder="big")[:, : K * bits].reshape(N, K, bits)
    weights = (1 << np.arange(bits - 1, -1, -1)).astype(np.uint32)
    return (stream.astype(np.uint32) * weights).sum(-1).astype(np.uint8)


def dequant(codes, scales, bits, group=128):
    N, K = codes.shape
    q = (codes.astype(np.int32) - (1 << (bits - 1))).astype(np.float32).reshape(N, K // group, group)
    return (q * scales[..., None].astype(np.float32)).reshape(N, K)
