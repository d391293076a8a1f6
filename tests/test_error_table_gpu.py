"""Parity of the quantization error table (wq_quant_error / wq_quant_error_many, the
per-tensor table the Per-group(128) article's sec. 3.2 bit allocation minimizes) with the
oracle's quantize -> dequantize -> sum of squares, at every width. Each element's squared
error is the same on both sides; only the order of the fp64 additions differs, so the sums
agree to ~1e-12 relative."""
import numpy as np
import pytest

from oracle import pd
import bit_weight_quantization_wq_b200 as wq
from bit_weight_quantization_wq_b200 import _binding as B
from bit_weight_quantization_wq_b200 import synth
from helpers import edge_weight, to_dev_bf16

pytestmark = pytest.mark.gpu


def _check(got, want, what):
    got = np.asarray(got, np.float64)
    assert got.shape == want.shape, what
    for j, (g, w) in enumerate(zip(got, want)):
        assert g == pytest.approx(w, rel=1e-12, abs=1e-300), f"{what}: entry {j}: {g!r} vs {w!r}"


@pytest.mark.parametrize("N,K", [(1, 128), (37, 1280), (300, 640), (1000, 2048)])
def test_error_table_edges(N, K):
    """Planted edge groups (all-zero, tiny values, one outlier, exact rounding ties)."""
    rng = np.random.default_rng(N + K)
    W = edge_weight(rng, N, K, 4)
    got = B.wq_quant_error(to_dev_bf16(W)).cpu().numpy()
    _check(got, pd.quant_error(W), f"{N}x{K}")


def test_error_table_wan_weight():
    """The 5120 x 5120 Wan-like weight (N(0, 0.015^2) + 0.1% outliers): the per-width SNRs rise
    with the width (by ~3 dB from 3 to 4 bits, where the outlier groups dominate the error, and
    ~6 dB per bit above)."""
    W = synth.wan_weight(0)
    got = B.wq_quant_error(to_dev_bf16(W)).cpu().numpy()
    want = pd.quant_error(W)
    _check(got, want, "wan 5120x5120")
    snr = 10 * np.log10(want[5] / want[:5])
    assert np.all(np.diff(snr) > 2.0) and np.all(np.diff(snr)[1:] > 4.5)


def test_error_table_many():
    """Twelve weights of mixed shapes (one empty) in one batched call, against one oracle table each."""
    import torch
    rng = np.random.default_rng(9)
    shapes = [(5, 128), (64, 384), (0, 256), (130, 1280), (7, 2048), (256, 512)] * 2
    Ws = [synth.weight(rng, N, K, float(rng.uniform(0.005, 0.05))) if N else np.zeros((0, K), np.uint16)
          for N, K in shapes]
    out = B.wq_quant_error_many([to_dev_bf16(W) for W in Ws])
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for i, W in enumerate(Ws):
        want = pd.quant_error(W) if W.size else np.zeros(6)
        _check(got[i], want, f"job {i} {W.shape}")
    assert wq.wq_device_status() == 0
