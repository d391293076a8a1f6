"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

  * wq_quantize_pack: packed bytes and scales bit-exact, every width, ragged and edge
    shapes (empty, one row, all-zero groups, exact rounding ties, tiny values) and the
    full-size weight shapes of the FLUX-like and Wan-like workloads;
  * wq_linear: both kernel families, every width, ragged M/N, with and without bias and
    the low-rank branch, against the fp64 oracle with
    ||y - y_o||_F / ||y_o||_F <= 5e-3 and max|err| <= 2e-2 rms(y_o);
    full-size cases (M up to 4096) on sampled token rows;
  * the bounded-wait self-test reports WQ_ERR_TIMEOUT and leaves the context usable.
"""
import numpy as np
import pytest

import oracle
import bit_weight_quantization_wq_b200 as wq
from bit_weight_quantization_wq_b200 import synth
from helpers import assert_linear_close, edge_weight, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu
BITS = (3, 4, 5, 6, 7)


def _pack_check(W, bits):
    import torch
    packed, scales = wq.wq_quantize_pack(to_dev_bf16(W), bits)
    torch.cuda.synchronize()
    codes, s_o = oracle.quantize(W, bits)
    p_o = oracle.pack(codes, bits)
    p = packed.cpu().numpy()
    s = scales.cpu().numpy()
    assert p.shape == p_o.shape and s.shape == s_o.shape
    bad = np.argwhere(p != p_o)
    assert bad.size == 0, f"{len(bad)} packed bytes differ, first at {bad[:4].tolist()}"
    assert (s.view(np.uint32) == s_o.view(np.uint32)).all()
    return packed, scales


# ------------------------------------------------------------------ quantize + pack

@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("N,K", [(1, 128), (7, 384), (37, 1280), (256, 512), (300, 640), (1000, 2048)])
def test_pack_parity_edges(bits, N, K):
    rng = np.random.default_rng(N * 31 + K + bits)
    _pack_check(edge_weight(rng, N, K, bits), bits)


@pytest.mark.parametrize("bits", BITS)
def test_pack_parity_every_bf16_abs_max(bits):
    """One group per finite positive bf16 value (0x0001 .. 0x7F7F, subnormals and the
    values whose 2 * 1.01 * abs_max overflows fp32 included), that value as the group's
    abs_max and the other weights below it: every step the kernel can produce, bit-exact."""
    rng = np.random.default_rng(4242 + bits)
    a_bits = np.arange(1, 0x7F80, dtype=np.uint16)
    a = synth.bf16_bits_to_f32(a_bits).astype(np.float64)
    u = rng.uniform(-1.0, 1.0, size=(len(a), 128))
    W = synth.f32_to_bf16_bits((a[:, None] * u).astype(np.float32))
    W[:, 0] = a_bits
    W[1::2, 0] |= 0x8000                       # negative abs_max element on odd groups
    W = W[: len(W) // 8 * 8].reshape(-1, 8 * 128)
    _pack_check(W, bits)


@pytest.mark.parametrize("bits", BITS)
def test_pack_empty(bits):
    import torch
    W = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    packed, scales = wq.wq_quantize_pack(W, bits)
    assert packed.shape == (0, 32 * bits) and scales.shape == (0, 2)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("shape_idx", [0, 1])
def test_pack_parity_wan_shapes(bits, shape_idx):
    """5120 x 5120 and 13824 x 5120, N(0, 0.015^2) + 0.1% outliers, every width."""
    _pack_check(synth.wan_weight(shape_idx), bits)


def test_pack_parity_flux_residuals():
    """The three FLUX-like residuals (after the rank-32 split), 4 bits."""
    for lin in synth.flux_linears(M=8, rank=32):
        _pack_check(lin["R"], 4)


# ------------------------------------------------------------------ linear, small shapes

def _linear_case(M, N, K, bits, path, rank=0, with_bias=True, seed=0, rows=None):
    import torch
    rng = np.random.default_rng(seed + 7 * M + 13 * N + K + bits)
    W = synth.weight(rng, N, K, 0.02)
    x = synth.activations(rng, M, K)
    b = synth.bias(rng, N) if with_bias else None
    L1 = L2 = None
    if rank:
        L1 = synth.f32_to_bf16_bits(rng.standard_normal((K, rank)).astype(np.float32) * 0.05)
        L2 = synth.f32_to_bf16_bits(rng.standard_normal((rank, N)).astype(np.float32) * 0.05)
    packed, scales = wq.wq_quantize_pack(to_dev_bf16(W), bits)
    y = wq.wq_linear(to_dev_bf16(x), packed, scales, bits, N,
                     L1=None if L1 is None else to_dev_bf16(L1),
                     L2=None if L2 is None else to_dev_bf16(L2),
                     bias=None if b is None else to_dev_bf16(b), path=path)
    torch.cuda.synchronize()
    assert wq.wq_device_status() == 0
    codes, s_o = oracle.quantize(W, bits)
    deq = oracle.dequant(codes, s_o, bits)
    rows = np.arange(M) if rows is None else rows
    y_o = oracle.linear_rows(x, deq, L1, L2, b, rows)
    return from_dev_bf16(y)[rows], y_o


SMALL_SHAPES = [(1, 256, 512), (7, 200, 384), (16, 520, 1280), (33, 256, 256), (129, 300, 640),
                (256, 256, 512), (300, 512, 1024)]


@pytest.mark.parametrize("path", ["small_m", "tensor"])
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M,N,K", SMALL_SHAPES)
def test_linear_parity(path, bits, M, N, K):
    y, y_o = _linear_case(M, N, K, bits, path)
    assert_linear_close(y, y_o, f"{path} b{bits} {M}x{N}x{K}")


@pytest.mark.parametrize("path", ["small_m", "tensor"])
@pytest.mark.parametrize("rank", [16, 32, 64])
@pytest.mark.parametrize("M,N,K", [(5, 264, 384), (200, 512, 768)])
def test_linear_lowrank_parity(path, rank, M, N, K):
    y, y_o = _linear_case(M, N, K, 4, path, rank=rank)
    assert_linear_close(y, y_o, f"{path} r{rank} {M}x{N}x{K}")


@pytest.mark.parametrize("path", ["small_m", "tensor"])
@pytest.mark.parametrize("rank", [16, 32, 64])
@pytest.mark.parametrize("M,N", [(64, 200), (300, 260), (64, 1004), (300, 1004)])
def test_linear_lowrank_ragged_n(path, rank, M, N):
    """Output widths that are not a multiple of 8: L2's rows are not 16-byte multiples, so
    the tensor-core path gathers the low-rank factor from global memory instead of by TMA."""
    y, y_o = _linear_case(M, N, 512, 4, path, rank=rank, seed=5)
    assert_linear_close(y, y_o, f"{path} r{rank} {M}x{N}x512")


@pytest.mark.parametrize("path", ["small_m", "tensor"])
def test_linear_no_bias(path):
    y, y_o = _linear_case(64, 256, 512, 5, path, with_bias=False)
    assert_linear_close(y, y_o, f"{path} no bias")


@pytest.mark.parametrize("path", ["small_m", "tensor"])
def test_linear_empty(path):
    import torch
    packed = torch.zeros((256, 64), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((256, 1), dtype=torch.float32, device="cuda")
    x = torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda")
    y = wq.wq_linear(x, packed, scales, 4, 256, path=path)
    assert y.shape == (0, 256)


# ------------------------------------------------------------------ full-size workloads

def test_single_linear_workload():
    """256 x 512 weight, 64 tokens, 4 bits, bias, no low-rank branch (full output)."""
    import torch
    W, x, b = synth.single_linear()
    packed, scales = _pack_check(W, 4)
    y = wq.wq_linear(to_dev_bf16(x), packed, scales, 4, 256, bias=to_dev_bf16(b))
    torch.cuda.synchronize()
    codes, s_o = oracle.quantize(W, 4)
    y_o = oracle.linear_rows(x, oracle.dequant(codes, s_o, 4), None, None, b)
    assert_linear_close(from_dev_bf16(y), y_o, "single linear")


def _sample_rows(M, n=24, seed=0):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, size=min(n, M), replace=False)]))


def test_flux_linears_workload():
    """FLUX-like linears at M = 4096 with the rank-32 branch and bias, sampled rows."""
    import torch
    for lin in synth.flux_linears(M=4096, rank=32):
        packed, scales = _pack_check(lin["R"], 4)
        y = wq.wq_linear(to_dev_bf16(lin["x"]), packed, scales, 4, lin["N"], L1=to_dev_bf16(lin["L1"]),
                         L2=to_dev_bf16(lin["L2"]), bias=to_dev_bf16(lin["bias"]))
        torch.cuda.synchronize()
        rows = _sample_rows(4096)
        codes, s_o = oracle.quantize(lin["R"], 4)
        y_o = oracle.linear_rows(lin["x"], oracle.dequant(codes, s_o, 4), lin["L1"], lin["L2"], lin["bias"], rows)
        assert_linear_close(from_dev_bf16(y)[rows], y_o, f"flux {lin['N']}x{lin['K']}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("shape_idx", [0, 1])
def test_wan_linears_workload(bits, shape_idx):
    """5120-hidden linears at M in {1, 16, 128, 4096}, every width, sampled rows."""
    import torch
    W = synth.wan_weight(shape_idx)
    N, K = W.shape
    packed, scales = wq.wq_quantize_pack(to_dev_bf16(W), bits)
    codes, s_o = oracle.quantize(W, bits)
    deq = oracle.dequant(codes, s_o, bits)
    b = synth.bias(synth.rng_for(3, shape_idx, 2), N)
    for M in (1, 16, 128, 4096):
        x = synth.wan_x(M)
        y = wq.wq_linear(to_dev_bf16(x), packed, scales, bits, N, bias=to_dev_bf16(b))
        torch.cuda.synchronize()
        rows = _sample_rows(M, n=8 if M > 16 else M)
        y_o = oracle.linear_rows(x, deq, None, None, b, rows)
        assert_linear_close(from_dev_bf16(y)[rows], y_o, f"wan b{bits} {N}x{K} M={M}")


def test_model_pack_sample():
    """Whole-model quantize+pack (the 49-block tensor set): one tensor of each shape, drawn
    from sampled blocks with the mixed-precision widths, bit-exact; the quantization SNR of
    each, from the oracle's dequantization of the GPU's bytes (17.6 dB at 5 bits on these
    outlier-laden weights), stays above 3 dB per bit."""
    import torch
    for j, (block, i) in enumerate([(7, 0), (23, 8), (48, 9)]):
        N, K = synth.BLOCK_SHAPES[i]
        bits = synth.mixed_bits(len(synth.BLOCK_SHAPES), config=5, block=block)[i]
        W = synth.weight(synth.rng_for(5, block, i), N, K, 0.015)
        packed, scales = _pack_check(W, bits)
        torch.cuda.synchronize()
        codes = oracle.unpack(packed.cpu().numpy(), K, bits)
        deq = oracle.dequant(codes, scales.cpu().numpy(), bits)
        w = synth.bf16_bits_to_f32(W).astype(np.float64)
        snr = oracle.snr_db(w, deq)
        assert snr > 3.0 * bits, (N, K, bits, snr)


def _assert_pack_matches(packed, scales, W, bits, what=""):
    codes, s_o = oracle.quantize(W, bits)
    p_o = oracle.pack(codes, bits)
    p = packed.cpu().numpy()
    s = scales.cpu().numpy()
    assert p.shape == p_o.shape and s.shape == s_o.shape, what
    bad = np.argwhere(p != p_o)
    assert bad.size == 0, f"{what}: {len(bad)} packed bytes differ, first at {bad[:4].tolist()}"
    assert (s.view(np.uint32) == s_o.view(np.uint32)).all(), what


def test_pack_many_parity():
    """wq_quantize_pack_many over a shuffled job list: every width, group counts that are not
    a multiple of a warp's 16-group block, empty jobs, 70 tensors of one width (two launches
    of that width), planted edge groups (all-zero, ties, tiny values, outliers). Every job is
    bit-exact against the oracle."""
    import torch
    rng = np.random.default_rng(777)
    specs = [(1 + i % 5, 128 * (1 + i % 3), 5) for i in range(70)]
    specs += [(0, 256, 4), (3, 0, 6), (7, 384, 3), (37, 1280, 4), (300, 640, 6), (1000, 2048, 7),
              (5, 128, 3), (256, 512, 4), (33, 768, 5)]
    jobs, host = [], []
    for k in rng.permutation(len(specs)):
        N, K, bits = specs[k]
        W = edge_weight(rng, N, K, bits) if N * K else np.zeros((N, K), np.uint16)
        host.append((W, bits))
        jobs.append((to_dev_bf16(W), bits))
    outs = wq.wq_quantize_pack_many(jobs)
    torch.cuda.synchronize()
    assert len(outs) == len(jobs)
    for j, ((W, bits), (packed, scales)) in enumerate(zip(host, outs)):
        _assert_pack_matches(packed, scales, W, bits, f"job {j} {W.shape} b{bits}")


def test_pack_many_model_block():
    """One DiT block of the whole-model workload (8 x 5120x5120, 13824x5120, 5120x13824 at
    the mixed-precision widths, 351 M weights) through one wq_quantize_pack_many call, the
    prepared call of the benchmark: 24 sampled rows of every tensor (first, last and random
    ones; rows quantize independently) bit-exact against the oracle on those rows."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    widths = synth.mixed_bits(len(synth.BLOCK_SHAPES), config=5, block=3)
    Ws = [(torch.randn(N, K, device="cuda", generator=g, dtype=torch.float32) * 0.015).to(torch.bfloat16)
          for N, K in synth.BLOCK_SHAPES]
    call = wq.PackJobs(list(zip(Ws, widths)))
    call()
    call()                                    # a second run through the same descriptors
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    for i, (W, bits, (packed, scales)) in enumerate(zip(Ws, widths, call.outputs)):
        N, K = W.shape
        rows = np.unique(np.concatenate([[0, 1, N - 1], rng.integers(0, N, 21)]))
        rows_t = torch.from_numpy(rows).cuda()
        Wh = from_dev_bf16(W[rows_t])
        _assert_pack_matches(packed[rows_t], scales[rows_t], Wh, bits, f"tensor {i} ({N}x{K}, b{bits})")


# ------------------------------------------------------------------ failure detection

def test_bounded_wait_selftest():
    import torch
    assert wq.wq_device_status() == 0
    assert wq.wq_selftest_bounded_wait(2000) == 6          # WQ_ERR_TIMEOUT
    assert wq.wq_device_status() == 0                      # cleared, context still usable
    y, y_o = _linear_case(4, 128, 256, 4, "small_m")
    assert_linear_close(y, y_o, "after self-test")
    torch.cuda.synchronize()
