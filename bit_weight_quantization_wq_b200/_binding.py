"""ctypes binding of libwq.so (include/wq.h). Argument marshalling only.

Every call takes torch CUDA tensors and passes their device pointers, sizes and the
current torch stream to the C ABI; all computation runs in the library's kernels. There is
no fallback: if ``libwq.so`` is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libwq.so")

# wq_status codes (include/wq.h)
WQ_OK = 0
WQ_ERR_INVALID_ARG = 1
WQ_ERR_UNSUPPORTED_BITS = 2
WQ_ERR_UNSUPPORTED_GROUP = 3
WQ_ERR_MISALIGNED = 4
WQ_ERR_CUDA = 5
WQ_ERR_TIMEOUT = 6
WQ_ERR_WORKSPACE = 7
WQ_ERR_UNSUPPORTED_DEVICE = 8

PATHS = {"auto": 0, "small_m": 1, "tensor": 2}

# exported C symbols, as declared in include/wq.h
SYMBOLS = (
    "wq_version", "wq_packed_bytes", "wq_scales_count", "wq_quantize_pack",
    "wq_linear_workspace_bytes", "wq_linear", "wq_linear_ex", "wq_device_status",
    "wq_selftest_bounded_wait", "wq_status_string", "wq_last_error", "wq_launch_count",
    "wq_linear_no_workspace", "wq_quantize_pack_many", "wq_quant_error", "wq_quant_error_many",
    "wq_pd_search", "wq_dequantize",
)


class WQError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {status_string(status)} (status {status})"
        if detail:
            msg += f": {detail}"
        super().__init__(msg)


class ErrorJob(ctypes.Structure):
    """wq_error_job of include/wq.h."""
    _fields_ = [("W", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("out", ctypes.c_void_p)]


class PackJob(ctypes.Structure):
    """wq_pack_job of include/wq.h."""
    _fields_ = [("W", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("bits", ctypes.c_int),
                ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libwq.so from the package directory. Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libwq.so not found at {LIB_PATH}; build it with "
                "`python -m bit_weight_quantization_wq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i64, i32, sz, p = ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
        L.wq_version.argtypes, L.wq_version.restype = [], i32
        L.wq_packed_bytes.argtypes, L.wq_packed_bytes.restype = [i64, i64, i32, i32], sz
        L.wq_scales_count.argtypes, L.wq_scales_count.restype = [i64, i64, i32], i64
        L.wq_quantize_pack.argtypes = [p, i64, i64, i32, i32, p, p, p]
        L.wq_quantize_pack.restype = i32
        L.wq_linear_workspace_bytes.argtypes = [i64, i64, i64, i32, i32]
        L.wq_linear_workspace_bytes.restype = sz
        L.wq_linear.argtypes = [p, i64, i64, p, p, i32, i32, i64, p, p, i32, p, p, p, sz, p]
        L.wq_linear.restype = i32
        L.wq_linear_ex.argtypes = [p, i64, i64, p, p, i32, i32, i64, p, p, i32, p, p, p, sz, i32, p]
        L.wq_linear_ex.restype = i32
        L.wq_device_status.argtypes, L.wq_device_status.restype = [p, i32], i32
        L.wq_selftest_bounded_wait.argtypes = [ctypes.c_uint32, p]
        L.wq_selftest_bounded_wait.restype = i32
        L.wq_status_string.argtypes, L.wq_status_string.restype = [i32], ctypes.c_char_p
        L.wq_last_error.argtypes, L.wq_last_error.restype = [], ctypes.c_char_p
        L.wq_launch_count.argtypes, L.wq_launch_count.restype = [], ctypes.c_uint64
        L.wq_linear_no_workspace.argtypes = [p, i64, i64, p, p, i32, i32, i64, p, p, i32, p, p, p]
        L.wq_linear_no_workspace.restype = i32
        L.wq_quantize_pack_many.argtypes = [ctypes.POINTER(PackJob), i32, i32, p]
        L.wq_quantize_pack_many.restype = i32
        L.wq_quant_error.argtypes = [p, i64, i64, i32, p, p]
        L.wq_quant_error.restype = i32
        L.wq_quant_error_many.argtypes = [ctypes.POINTER(ErrorJob), i32, i32, p]
        L.wq_quant_error_many.restype = i32
        L.wq_pd_search.argtypes = [p, p, i32, p, i32, ctypes.c_double, i32, i32, p, p, p]
        L.wq_pd_search.restype = i32
        L.wq_dequantize.argtypes = [p, p, i64, i64, i32, i32, p, p]
        L.wq_dequantize.restype = i32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().wq_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != WQ_OK:
        raise WQError(status, where, lib().wq_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, name, dtype, shape=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


# ----------------------------------------------------------------------------- API

def wq_version() -> int:
    return int(lib().wq_version())


def wq_packed_bytes(N: int, K: int, bits: int, group: int = 128) -> int:
    return int(lib().wq_packed_bytes(N, K, bits, group))


def wq_scales_count(N: int, K: int, group: int = 128) -> int:
    return int(lib().wq_scales_count(N, K, group))


def wq_linear_workspace_bytes(M: int, N: int, K: int, bits: int, rank: int = 0) -> int:
    return int(lib().wq_linear_workspace_bytes(M, N, K, bits, rank))


def wq_quantize_pack(W, bits: int, group: int = 128, packed=None, scales=None, stream=None):
    """Quantize + pack an (N, K) bf16 weight. Returns (packed uint8 (N, K*bits/8), scales f32 (N, K/group))."""
    import torch
    _dev(W, "W", torch.bfloat16)
    if W.dim() != 2:
        raise ValueError("W must be 2-D (N, K)")
    N, K = W.shape
    if packed is None:
        packed = torch.empty((N, K * bits // 8), dtype=torch.uint8, device=W.device)
    if scales is None:
        scales = torch.empty((N, max(K // group, 0)), dtype=torch.float32, device=W.device)
    _dev(packed, "packed", torch.uint8)
    _dev(scales, "scales", torch.float32)
    st = lib().wq_quantize_pack(_ptr(W), N, K, bits, group, _ptr(packed), _ptr(scales), _stream(stream))
    _check(st, "wq_quantize_pack")
    return packed, scales


def wq_linear(x, packed, scales, bits: int, N: int, L1=None, L2=None, bias=None, y=None,
              workspace=None, group: int = 128, path: str = "auto", stream=None):
    """y = x dequant(packed, scales)^T + (x L1) L2 + bias, bf16 (M, N)."""
    import torch
    _dev(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be 2-D (M, K)")
    M, K = x.shape
    _dev(packed, "packed", torch.uint8)
    _dev(scales, "scales", torch.float32)
    rank = 0
    if L1 is not None or L2 is not None:
        if L1 is None or L2 is None:
            raise ValueError("L1 and L2 go together")
        _dev(L1, "L1", torch.bfloat16)
        rank = L1.shape[1]
        _dev(L2, "L2", torch.bfloat16, (rank, N))
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16, (N,))
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _dev(y, "y", torch.bfloat16, (M, N))
    need = wq_linear_workspace_bytes(M, N, K, bits, rank)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().wq_linear_ex(_ptr(x), M, K, _ptr(packed), _ptr(scales), bits, group, N,
                            _ptr(L1), _ptr(L2), rank, _ptr(bias), _ptr(y), _ptr(workspace),
                            ws_bytes, PATHS[path], _stream(stream))
    _check(st, "wq_linear")
    return y


def wq_device_status(stream=None, clear: bool = True) -> int:
    """Synchronize and return the device-side status (raises on WQ_ERR_CUDA)."""
    st = lib().wq_device_status(_stream(stream), 1 if clear else 0)
    if st == WQ_ERR_CUDA:
        _check(st, "wq_device_status")
    return st


def wq_launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(lib().wq_launch_count())


def wq_selftest_bounded_wait(timeout_us: int, stream=None) -> int:
    return int(lib().wq_selftest_bounded_wait(timeout_us, _stream(stream)))


class PackJobs:
    """A prepared wq_quantize_pack_many call over many weights, each at its own width.

    ``jobs``: iterable of ``(W, bits)`` or ``(W, bits, packed, scales)``, W an (N, K) bf16
    CUDA tensor; missing outputs are allocated here. The descriptors are marshalled once, so
    calling the object again (e.g. inside a timed loop) only crosses the C ABI. The tensors
    are referenced for the object's lifetime. ``outputs``: one ``(packed, scales)`` per job.
    """

    def __init__(self, jobs, group: int = 128):
        import torch
        self.group = group
        self.outputs = []
        self._inputs = []
        descs = []
        for i, job in enumerate(list(jobs)):
            if len(job) == 2:
                (W, bits), packed, scales = job, None, None
            else:
                W, bits, packed, scales = job
            _dev(W, f"jobs[{i}].W", torch.bfloat16)
            if W.dim() != 2:
                raise ValueError(f"jobs[{i}].W must be 2-D (N, K)")
            N, K = W.shape
            bits = int(bits)
            if packed is None:
                packed = torch.empty((N, K * bits // 8), dtype=torch.uint8, device=W.device)
            if scales is None:
                scales = torch.empty((N, max(K // group, 0)), dtype=torch.float32, device=W.device)
            _dev(packed, f"jobs[{i}].packed", torch.uint8, (N, K * bits // 8))
            _dev(scales, f"jobs[{i}].scales", torch.float32, (N, max(K // group, 0)))
            self._inputs.append(W)
            self.outputs.append((packed, scales))
            descs.append(PackJob(W.data_ptr(), N, K, bits, packed.data_ptr(), scales.data_ptr()))
        self._n = len(descs)
        self._arr = (PackJob * max(1, self._n))(*descs)

    def __call__(self, stream=None):
        st = lib().wq_quantize_pack_many(self._arr, self._n, self.group, _stream(stream))
        _check(st, "wq_quantize_pack_many")
        return self.outputs


def wq_quantize_pack_many(jobs, group: int = 128, stream=None):
    """Quantize + pack many (N, K) bf16 weights, each at its own width, in a few launches.
    ``jobs`` as for :class:`PackJobs`. Returns one ``(packed, scales)`` per job."""
    return PackJobs(jobs, group)(stream)


ERROR_WIDTHS = (3, 4, 5, 6, 7)


def wq_quant_error_many(weights, group: int = 128, out=None, stream=None):
    """Quantization error table of many (N, K) bf16 weights: a float64 CUDA tensor (T, 6) whose
    row i holds sum (w - deq_b(w))^2 for b = 3..7 and sum w^2 of weight i."""
    import torch
    weights = list(weights)
    if out is None:
        dev = weights[0].device if weights else torch.device("cuda")
        out = torch.empty((len(weights), 6), dtype=torch.float64, device=dev)
    _dev(out, "out", torch.float64, (len(weights), 6))
    descs = []
    for i, W in enumerate(weights):
        _dev(W, f"weights[{i}]", torch.bfloat16)
        if W.dim() != 2:
            raise ValueError(f"weights[{i}] must be 2-D (N, K)")
        descs.append(ErrorJob(W.data_ptr(), W.shape[0], W.shape[1], out[i].data_ptr()))
    arr = (ErrorJob * max(1, len(descs)))(*descs)
    _check(lib().wq_quant_error_many(arr, len(descs), group, _stream(stream)), "wq_quant_error_many")
    return out


def wq_quant_error(W, group: int = 128, stream=None):
    """Quantization error table of one (N, K) bf16 weight: float64 CUDA tensor (6,)."""
    import torch
    _dev(W, "W", torch.bfloat16)
    if W.dim() != 2:
        raise ValueError("W must be 2-D (N, K)")
    out = torch.empty(6, dtype=torch.float64, device=W.device)
    _check(lib().wq_quant_error(_ptr(W), W.shape[0], W.shape[1], group, _ptr(out), _stream(stream)),
           "wq_quant_error")
    return out


def wq_pd_search(mse_table, n_params, bits, target_bpw: float, t_init, n_iters: int = 500):
    """Per-tensor width search (host). mse_table (T, B) per-weight MSE, n_params (T,), bits (B,),
    t_init (R, T) random starts. Returns (widths int array (T,), total MSE, BPW, start index)."""
    import numpy as np
    mse = np.ascontiguousarray(mse_table, np.float64)
    n = np.ascontiguousarray(n_params, np.int64)
    b = np.ascontiguousarray(bits, np.int32)
    t0 = np.ascontiguousarray(t_init, np.float64)
    T, nb = mse.shape
    if n.shape != (T,) or b.shape != (nb,) or t0.ndim != 2 or t0.shape[1] != T:
        raise ValueError("mse_table (T, B), n_params (T,), bits (B,), t_init (R, T)")
    out = np.empty(T, np.int32)
    res = np.empty(3, np.float64)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(lib().wq_pd_search(ptr(mse), ptr(n), T, ptr(b), nb, float(target_bpw), n_iters, t0.shape[0], ptr(t0),
                              ptr(out), ptr(res)), "wq_pd_search")
    return out, float(res[0]), float(res[1]), int(res[2])


def wq_dequantize(packed, scales, bits: int, K: int, group: int = 128, out=None, stream=None):
    """bf16 (N, K) weight bf16(q * step) from packed codes and steps (the page's dequantize)."""
    import torch
    _dev(packed, "packed", torch.uint8)
    _dev(scales, "scales", torch.float32)
    N = packed.shape[0]
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=packed.device)
    _dev(out, "out", torch.bfloat16, (N, K))
    _check(lib().wq_dequantize(_ptr(packed), _ptr(scales), N, K, bits, group, _ptr(out), _stream(stream)),
           "wq_dequantize")
    return out
