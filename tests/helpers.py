"""Shared helpers for the parity tests: device transfer of bf16 bit patterns, the
tolerance check, and constructed edge-case weights."""
import numpy as np

from bit_weight_quantization_wq_b200 import synth

# GEMM tolerance against the fp64 oracle
REL_FRO = 5e-3
MAX_ABS_RMS = 2e-2


def to_dev_bf16(bits_np):
    import torch
    a = np.ascontiguousarray(bits_np, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def bf16_half_ulp(v):
    """Half a unit in the last place of bf16 (8 significant bits) at the magnitude of v: the
    largest error of a correctly rounded bf16 value there."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -140)))
    return 2.0 ** (np.maximum(e, -126.0) - 8.0)


def linear_error(y_bits, y_ref):
    """(relative Frobenius error, max excess error / rms(y_ref)) of a bf16 result vs the fp64
    reference. The layer's output is bf16 (one rounding of acc + bias), so the max bar
    measures each element's error beyond its own correct rounding: |y - y_ref| minus half a
    bf16 ulp at that element. (A correctly rounded output alone reaches 2e-2 rms wherever an
    element is ~5x the rms or more.) The Frobenius error is the plain one."""
    y = bf16_f64(y_bits)
    err = np.abs(y - y_ref)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    rel = float(np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_ref), 1e-300))
    excess = np.maximum(err - bf16_half_ulp(np.maximum(np.abs(y), np.abs(y_ref))), 0.0)
    return rel, float(excess.max() / max(rms, 1e-300))


def assert_linear_close(y_bits, y_ref, what=""):
    rel, mx = linear_error(y_bits, y_ref)
    assert rel <= REL_FRO and mx <= MAX_ABS_RMS, f"{what}: rel_fro {rel:.3e} max/rms {mx:.3e}"
    return rel, mx


def tie_rows(bits, n_rows=16):
    """Rows of one 128-group [abs_max, w, 0, ...] where fp32 w/step lands exactly on k + 1/2
    (candidates from an fp32 search; the oracle decides the rounding)."""
    exps = np.arange(-20, 8)
    mant = np.arange(128, 256)
    amax = (mant[None, :] / 128.0 * 2.0 ** exps[:, None]).astype(np.float32).ravel()
    step = (np.float32(2.0) * (amax * np.float32(1.01))) / np.float32((1 << bits) - 1)
    q_max = ((1 << bits) - 1) // 2
    rows = []
    for t in np.arange(q_max) + 0.5:
        v = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.float32(t) * step))
        hit = ((v / step) == np.float32(t)) & (v < amax) & (v > 0)
        for a, w in zip(amax[hit], v[hit]):
            r = np.zeros(128, np.uint16)
            r[0] = synth.f32_to_bf16_bits(np.array([a], np.float32))[0]
            r[1] = synth.f32_to_bf16_bits(np.array([w], np.float32))[0]
            r[2] = synth.f32_to_bf16_bits(np.array([-w], np.float32))[0]
            rows.append(r)
            if len(rows) >= n_rows:
                return np.stack(rows)
    return np.stack(rows) if rows else np.zeros((0, 128), np.uint16)


def edge_weight(rng, N, K, bits, sigma=0.02):
    """Synthetic weight with planted edge groups: all-zero, single outlier, exact ties,
    tiny magnitudes, and the largest/smallest-code extremes."""
    W = synth.weight(rng, N, K, sigma)
    G = K // 128
    if N >= 1:
        W[0, :128] = 0                                             # all-zero group
    if N >= 2:
        W[1, :] = synth.f32_to_bf16_bits(np.full(K, 1e-30, np.float32))     # tiny values
    if N >= 3 and G >= 1:
        W[2, :128] = 0
        W[2, 5] = synth.f32_to_bf16_bits(np.array([-0.4375], np.float32))[0]  # one outlier
    ties = tie_rows(bits, 8)
    for i, r in enumerate(ties):
        n = 3 + i
        if n >= N:
            break
        W[n, (G - 1) * 128:] = r
    return W
