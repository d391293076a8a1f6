"""CPU oracle for per-group low-bit weight quantization and the quantized linear layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg are the only callers. The product path (the CUDA library and its
binding) never imports this package, and this package never imports the product.

Two independent implementations live here:
  * ``wq_oracle.c`` (loaded with ctypes): the oracle proper. Quantization in IEEE fp32,
    packing bit by bit, the linear layer in fp64.
  * ``twin.py``: a numpy restatement used only to cross-check the C oracle.

Arrays: bf16 tensors are passed as numpy ``uint16`` arrays holding the bf16 bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    """Load (building first if needed) the C oracle library."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, i32 = ctypes.c_int64, ctypes.c_int
        p = ctypes.c_void_p
        L.wqo_quantize.argtypes = [p, i64, i64, i32, i64, p, p]
        L.wqo_pack.argtypes = [p, i64, i64, i32, p]
        L.wqo_unpack.argtypes = [p, i64, i64, i32, p]
        L.wqo_dequant.argtypes = [p, p, i64, i64, i32, i64, p]
        L.wqo_linear_rows.argtypes = [p, i64, i64, p, i64, p, p, i32, p, p, i64, p]
        for f in (L.wqo_quantize, L.wqo_pack, L.wqo_unpack, L.wqo_dequant, L.wqo_linear_rows,
                  L.wqo_num_threads):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def quantize(W_bits, bits, group=128):
    """Per-group symmetric quantization (Per-group(128) article, sec. 3.1).

    W_bits: (N, K) uint16 bf16 bit patterns. Returns (codes (N, K) uint8, scales (N, K/group) f32).
    """
    W_bits = _c(W_bits, np.uint16)
    N, K = W_bits.shape
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N, K // group if group else 0), np.float32)
    rc = lib().wqo_quantize(_ptr(W_bits), N, K, bits, group, _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError(f"wqo_quantize: bad arguments (N={N}, K={K}, bits={bits}, group={group})")
    return codes, scales


def pack(codes, bits):
    """MSB-first multi-bit packing per row (Per-group(128) article, sec. 3.3)."""
    codes = _c(codes, np.uint8)
    N, K = codes.shape
    if (K * bits) % 8:
        raise ValueError("K*bits must be a multiple of 8")
    out = np.empty((N, K * bits // 8), np.uint8)
    if lib().wqo_pack(_ptr(codes), N, K, bits, _ptr(out)) != 0:
        raise ValueError("wqo_pack: bad arguments")
    return out


def unpack(packed, K, bits):
    """Inverse of :func:`pack`."""
    packed = _c(packed, np.uint8)
    N = packed.shape[0]
    out = np.empty((N, K), np.uint8)
    if lib().wqo_unpack(_ptr(packed), N, K, bits, _ptr(out)) != 0:
        raise ValueError("wqo_unpack: bad arguments")
    return out


def quantize_pack(W_bits, bits, group=128):
    """Quantize then pack: returns (packed (N, K*bits/8) uint8, scales (N, K/group) f32)."""
    codes, scales = quantize(W_bits, bits, group)
    return pack(codes, bits), scales


def dequant(codes, scales, bits, group=128):
    """(code - 2^(bits-1)) * step in fp32 (Per-group(128) article, sec. 3.4)."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    N, K = codes.shape
    out = np.empty((N, K), np.float32)
    if lib().wqo_dequant(_ptr(codes), _ptr(scales), N, K, bits, group, _ptr(out)) != 0:
        raise ValueError("wqo_dequant: bad arguments")
    return out


def dequant_bf16(codes, scales, bits, group=128):
    """The dequantized weight as the page's bf16 matmul sees it (Per-group(128) article,
    sec. 3.4 then 5.3): bf16(fl32(q * step)), round to nearest even. Returns uint16 bf16 bits."""
    d = dequant(codes, scales, bits, group).view(np.uint32).astype(np.uint64)
    return ((d + 0x7FFF + ((d >> 16) & 1)) >> 16).astype(np.uint16)


def linear_rows(x_bits, deq, L1_bits=None, L2_bits=None, bias_bits=None, rows=None):
    """fp64 y = x deq^T + (x L1) L2 + bias for the selected token rows.

    x_bits (M, K) uint16 bf16; deq (N, K) f32; L1 (K, r) / L2 (r, N) uint16 bf16 or None;
    bias (N,) uint16 bf16 or None; rows: int64 indices into M (default: all rows).
    Returns (len(rows), N) float64.
    """
    x_bits = _c(x_bits, np.uint16)
    deq = _c(deq, np.float32)
    M, K = x_bits.shape
    N = deq.shape[0]
    if deq.shape[1] != K:
        raise ValueError("x and deq disagree on K")
    r = 0
    if L1_bits is not None:
        L1_bits = _c(L1_bits, np.uint16)
        L2_bits = _c(L2_bits, np.uint16)
        r = L1_bits.shape[1]
        if L1_bits.shape != (K, r) or L2_bits.shape != (r, N):
            raise ValueError("bad low-rank factor shapes")
    if bias_bits is not None:
        bias_bits = _c(bias_bits, np.uint16)
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(np.asarray(rows, np.int64), np.int64)
    y = np.empty((rows.shape[0], N), np.float64)
    rc = lib().wqo_linear_rows(_ptr(x_bits), M, K, _ptr(deq), N, _ptr(L1_bits), _ptr(L2_bits), r,
                               _ptr(bias_bits), _ptr(rows), rows.shape[0], _ptr(y))
    if rc != 0:
        raise ValueError("wqo_linear_rows: bad arguments")
    return y


def num_threads():
    """OpenMP threads the oracle uses."""
    return int(lib().wqo_num_threads())


def snr_db(w, w_hat):
    """Signal-to-noise ratio 10 log10(sum w^2 / sum (w - w_hat)^2), the definition the
    Per-group(128) article's sec. 4.3 MSE/SNR pairs imply."""
    w = np.asarray(w, np.float64)
    e = w - np.asarray(w_hat, np.float64)
    return 10.0 * np.log10(np.sum(w * w) / np.sum(e * e))
