"""C-ABI checks that need no GPU: the library loads, exports every symbol include/wq.h
declares, computes sizes, and rejects bad arguments on the host before touching a device.
No call here reaches a kernel launch."""
import ctypes
import os
import re
import subprocess

import pytest

import bit_weight_quantization_wq_b200 as wq
from bit_weight_quantization_wq_b200 import _binding as B
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "wq.h")


@pytest.fixture(scope="module")
def L():
    from bit_weight_quantization_wq_b200 import build
    build.build()
    return wq.lib()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"WQ_API\s+[\w\s\*]+?\b(wq_\w+)\s*\(", text)))


def test_exports_match_header(L):
    declared = header_functions()
    assert len(declared) == 18
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = sorted(line.split()[-1] for line in out.splitlines() if line.split()[-1].startswith("wq_"))
    assert exported == declared
    assert sorted(B.SYMBOLS) == declared
    for name in declared:
        assert hasattr(L, name)


# The boundary calls as the hot-path scope lists them (argument types in order, return
# type), checked against the header by the C compiler. Two deliberate differences from
# that list: wq_linear_workspace_bytes also takes the low-rank `rank` (only the branch
# needs scratch, so the size depends on it), and the device status is read with
# wq_device_status(stream, clear).
SCOPE_SIGNATURES = {
    "wq_packed_bytes": "size_t (*)(int64_t, int64_t, int, int)",
    "wq_scales_count": "int64_t (*)(int64_t, int64_t, int)",
    "wq_quantize_pack": "wq_status (*)(const void *, int64_t, int64_t, int, int, uint8_t *, float *, wq_stream_t)",
    "wq_linear_workspace_bytes": "size_t (*)(int64_t, int64_t, int64_t, int, int)",
    "wq_linear": ("wq_status (*)(const void *, int64_t, int64_t, const uint8_t *, const float *, int, int, int64_t, "
                  "const void *, const void *, int, const void *, void *, void *, size_t, wq_stream_t)"),
    "wq_status_string": "const char *(*)(wq_status)",
}


def test_scope_signatures_match_header(tmp_path):
    """Every boundary call of the hot-path scope has exactly the expected C signature."""
    checks = "\n".join(
        f'_Static_assert(_Generic(&{name}, {sig}: 1, default: 0), "{name} signature");'
        for name, sig in SCOPE_SIGNATURES.items())
    src = tmp_path / "sig.c"
    src.write_text('#include "wq.h"\n' + checks + "\nint main(void) { return 0; }\n")
    r = subprocess.run(["gcc", "-std=c11", "-fsyntax-only", "-I", os.path.join(ROOT, "include"), str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


_CTYPES = {"double": ctypes.c_double, "int64_t": ctypes.c_int64, "int": ctypes.c_int, "size_t": ctypes.c_size_t,
           "uint32_t": ctypes.c_uint32, "uint64_t": ctypes.c_uint64, "wq_status": ctypes.c_int,
           "wq_path": ctypes.c_int, "wq_stream_t": ctypes.c_void_p}


def _ctype_of(decl):
    decl = decl.replace("const ", "").strip()
    if decl in ("void", ""):
        return None
    if decl.startswith("char") and "*" in decl:
        return ctypes.c_char_p
    if "*" in decl:
        base = decl.split("*")[0].strip()
        structs = {"wq_pack_job": B.PackJob, "wq_error_job": B.ErrorJob}
        return ctypes.POINTER(structs[base]) if base in structs else ctypes.c_void_p
    return _CTYPES[decl.split()[0]]


def header_prototypes():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for ret, name, args in re.findall(r"WQ_API\s+([\w\s\*]+?)\s*\b(wq_\w+)\s*\(([^)]*)\)", text):
        params = [a.strip() for a in args.split(",") if a.strip() and a.strip() != "void"]
        # drop the parameter name: the type is everything before the last identifier
        types = [re.sub(r"\b\w+\s*$", "", p).strip() or p for p in params]
        out[name] = (ret.strip(), types)
    return out


def test_binding_declarations_match_header(L):
    """The binding's ctypes argtypes/restype follow the header's prototypes, call by call."""
    protos = header_prototypes()
    assert sorted(protos) == sorted(B.SYMBOLS)
    for name, (ret, types) in protos.items():
        f = getattr(L, name)
        want = [_ctype_of(t) for t in types]
        assert list(f.argtypes) == want, (name, f.argtypes, want)
        r = _ctype_of(ret)
        if r is not None:
            assert f.restype == r, (name, f.restype, r)


def test_no_driver_or_shared_cudart_dependency(L):
    out = subprocess.run(["ldd", B.LIB_PATH], capture_output=True, text=True, check=True).stdout
    assert "libcuda.so" not in out and "libcudart" not in out


def test_sizes(L):
    # packing table: 16*b bytes per 128-weight group
    for bits in (3, 4, 5, 6, 7):
        assert wq.wq_packed_bytes(5120, 5120, bits, 128) == 5120 * 5120 * bits // 8
        assert wq.wq_packed_bytes(1, 128, bits, 128) == 16 * bits
    assert wq.wq_packed_bytes(4, 128, 2, 128) == 0 and wq.wq_packed_bytes(4, 128, 8, 128) == 0
    assert wq.wq_packed_bytes(-1, 128, 4, 128) == 0
    assert wq.wq_packed_bytes(4, 128, 4, 64) == 0          # only groups of 128
    assert wq.wq_packed_bytes(4, 200, 4, 128) == 0         # K not a multiple of the group
    assert wq.wq_scales_count(13824, 5120, 128) == 13824 * 40
    assert wq.wq_scales_count(3, 100, 128) == -1
    assert wq.wq_linear_workspace_bytes(16, 256, 512, 4, 0) == 0
    assert wq.wq_linear_workspace_bytes(4096, 3072, 3072, 4, 32) >= 4096 * 32 * 2
    assert wq.wq_version() == 100


def test_status_strings(L):
    for s in range(9):
        assert isinstance(wq.status_string(s), str) and wq.status_string(s)
    assert "timed out" in wq.status_string(B.WQ_ERR_TIMEOUT)


def _qp(L, W, N, K, bits, group, packed, scales):
    return L.wq_quantize_pack(ctypes.c_void_p(W), N, K, bits, group, ctypes.c_void_p(packed),
                              ctypes.c_void_p(scales), None)


def test_quantize_pack_argument_checks(L):
    A = 0x10000          # aligned fake addresses; none of these calls gets past the checks
    assert _qp(L, A, 4, 128, 2, 128, A, A) == B.WQ_ERR_UNSUPPORTED_BITS
    assert _qp(L, A, 4, 128, 8, 128, A, A) == B.WQ_ERR_UNSUPPORTED_BITS
    assert _qp(L, A, 4, 128, 4, 64, A, A) == B.WQ_ERR_UNSUPPORTED_GROUP
    assert _qp(L, A, -1, 128, 4, 128, A, A) == B.WQ_ERR_INVALID_ARG
    assert _qp(L, 0, 4, 128, 4, 128, A, A) == B.WQ_ERR_INVALID_ARG
    assert _qp(L, A, 4, 130, 4, 128, A, A) == B.WQ_ERR_INVALID_ARG
    assert b"multiple of 128" in L.wq_last_error()
    assert _qp(L, A + 8, 4, 128, 4, 128, A, A) == B.WQ_ERR_MISALIGNED
    assert _qp(L, A, 4, 128, 4, 128, A + 4, A) == B.WQ_ERR_MISALIGNED
    assert b"16-byte aligned" in L.wq_last_error()
    # empty weights are a no-op that needs no device
    assert _qp(L, 0, 0, 128, 4, 128, 0, 0) == B.WQ_OK


def _jobs(*specs):
    """specs: (W, N, K, bits, packed, scales) tuples of fake device addresses."""
    arr = (B.PackJob * max(1, len(specs)))(*[B.PackJob(*sp) for sp in specs])
    return arr, len(specs)


def _many(L, arr, n, group=128):
    return L.wq_quantize_pack_many(arr, n, group, None)


def test_pack_job_struct_matches_header(tmp_path):
    """The binding's PackJob has the size and field offsets of the C wq_pack_job."""
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "wq.h"\n'
        'int main(void) { printf("%zu %zu %zu %zu %zu %zu %zu\\n", sizeof(wq_pack_job),'
        ' offsetof(wq_pack_job, W), offsetof(wq_pack_job, N), offsetof(wq_pack_job, K),'
        ' offsetof(wq_pack_job, bits), offsetof(wq_pack_job, packed), offsetof(wq_pack_job, scales));'
        ' return 0; }\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    P = B.PackJob
    assert got == [ctypes.sizeof(P), P.W.offset, P.N.offset, P.K.offset, P.bits.offset, P.packed.offset,
                   P.scales.offset]


def test_error_job_struct_matches_header(tmp_path):
    """The binding's ErrorJob has the size and field offsets of the C wq_error_job."""
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "wq.h"\n'
        'int main(void) { printf("%zu %zu %zu %zu %zu\\n", sizeof(wq_error_job), offsetof(wq_error_job, W),'
        ' offsetof(wq_error_job, N), offsetof(wq_error_job, K), offsetof(wq_error_job, out)); return 0; }\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    E = B.ErrorJob
    assert got == [ctypes.sizeof(E), E.W.offset, E.N.offset, E.K.offset, E.out.offset]


def test_quant_error_argument_checks(L):
    A = 0x10000          # aligned fake addresses; none of these calls gets past the checks
    v = ctypes.c_void_p
    assert L.wq_quant_error(v(A), 4, 128, 64, v(A), None) == B.WQ_ERR_UNSUPPORTED_GROUP
    assert L.wq_quant_error(v(A), 4, 130, 128, v(A), None) == B.WQ_ERR_INVALID_ARG
    assert L.wq_quant_error(v(A), -1, 128, 128, v(A), None) == B.WQ_ERR_INVALID_ARG
    assert L.wq_quant_error(v(A), 4, 128, 128, None, None) == B.WQ_ERR_INVALID_ARG
    assert L.wq_quant_error(v(A + 8), 4, 128, 128, v(A), None) == B.WQ_ERR_MISALIGNED
    assert L.wq_quant_error(v(A), 4, 128, 128, v(A + 4), None) == B.WQ_ERR_MISALIGNED
    assert L.wq_quant_error_many(None, 3, 128, None) == B.WQ_ERR_INVALID_ARG
    assert L.wq_quant_error_many(None, 0, 128, None) == B.WQ_OK


def test_quantize_pack_many_argument_checks(L):
    A = 0x10000          # aligned fake addresses; none of these calls gets past the checks
    ok = (A, 4, 128, 4, A, A)
    assert _many(L, *_jobs(ok), group=64) == B.WQ_ERR_UNSUPPORTED_GROUP
    assert L.wq_quantize_pack_many(None, 2, 128, None) == B.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_pack_many(None, 0, 128, None) == B.WQ_OK
    assert _many(L, _jobs(ok)[0], -1) == B.WQ_ERR_INVALID_ARG
    assert _many(L, *_jobs(ok, (A, 4, 128, 8, A, A))) == B.WQ_ERR_UNSUPPORTED_BITS
    assert b"job 1" in L.wq_last_error()
    assert _many(L, *_jobs((A, 4, 128, 2, A, A), ok)) == B.WQ_ERR_UNSUPPORTED_BITS
    assert b"job 0" in L.wq_last_error()
    assert _many(L, *_jobs(ok, ok, (A, 4, 130, 4, A, A))) == B.WQ_ERR_INVALID_ARG
    assert _many(L, *_jobs(ok, (A, -1, 128, 4, A, A))) == B.WQ_ERR_INVALID_ARG
    assert _many(L, *_jobs((0, 4, 128, 4, A, A))) == B.WQ_ERR_INVALID_ARG
    assert _many(L, *_jobs(ok, (A, 4, 128, 5, A + 8, A))) == B.WQ_ERR_MISALIGNED
    assert _many(L, *_jobs((A, 4, 128, 6, A, A + 4))) == B.WQ_ERR_MISALIGNED
    # a bad job after empty ones is still found; all-empty job lists need no device
    assert _many(L, *_jobs((0, 0, 128, 4, 0, 0), (A, 4, 128, 9, A, A))) == B.WQ_ERR_UNSUPPORTED_BITS
    assert _many(L, *_jobs((0, 0, 128, 4, 0, 0), (0, 3, 0, 7, 0, 0))) == B.WQ_OK


def _lin(L, M=16, K=256, N=64, bits=4, group=128, rank=0, L1=0, L2=0, x=0x10000, p=0x10000,
         s=0x10000, bias=0, y=0x10000, ws=0, ws_bytes=0, path=0):
    v = ctypes.c_void_p
    return L.wq_linear_ex(v(x), M, K, v(p), v(s), bits, group, N, v(L1) if L1 else None,
                          v(L2) if L2 else None, rank, v(bias) if bias else None, v(y),
                          v(ws) if ws else None, ws_bytes, path, None)


def test_linear_argument_checks(L):
    A = 0x10000
    assert _lin(L, bits=2) == B.WQ_ERR_UNSUPPORTED_BITS
    assert _lin(L, group=256) == B.WQ_ERR_UNSUPPORTED_GROUP
    assert _lin(L, K=200) == B.WQ_ERR_INVALID_ARG
    assert _lin(L, M=-1) == B.WQ_ERR_INVALID_ARG
    assert _lin(L, rank=24, L1=A, L2=A) == B.WQ_ERR_INVALID_ARG          # not a multiple of 16
    assert _lin(L, rank=80, L1=A, L2=A) == B.WQ_ERR_INVALID_ARG          # above 64
    assert _lin(L, rank=32, L1=A, L2=0) == B.WQ_ERR_INVALID_ARG          # missing L2
    assert _lin(L, rank=0, L1=A, L2=A) == B.WQ_ERR_INVALID_ARG           # factors without rank
    assert _lin(L, path=7) == B.WQ_ERR_INVALID_ARG
    assert _lin(L, x=0) == B.WQ_ERR_INVALID_ARG
    assert _lin(L, y=A + 2) == B.WQ_ERR_MISALIGNED
    assert _lin(L, bias=A + 6) == B.WQ_ERR_MISALIGNED
    # the low-rank branch needs a workspace
    assert _lin(L, rank=32, L1=A, L2=A) == B.WQ_ERR_WORKSPACE
    assert _lin(L, rank=32, L1=A, L2=A, ws=A, ws_bytes=16) == B.WQ_ERR_WORKSPACE
    # empty problems are no-ops that need no device
    assert _lin(L, M=0) == B.WQ_OK
    assert _lin(L, N=0) == B.WQ_OK


def test_calls_fail_cleanly_without_a_device(L):
    """A call that passes every host check reports WQ_ERR_CUDA when there is no GPU."""
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("a GPU is present; the fake pointers below must not reach a kernel")
    except ImportError:
        pass
    A = 0x10000
    assert _qp(L, A, 4, 128, 4, 128, A, A) == B.WQ_ERR_CUDA
    assert _many(L, *_jobs((A, 4, 128, 4, A, A))) == B.WQ_ERR_CUDA
    assert _lin(L) == B.WQ_ERR_CUDA
    assert L.wq_last_error()


def test_binding_refuses_missing_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "libwq.so"))
    with pytest.raises(RuntimeError, match="libwq.so not found"):
        B.lib()


def test_model_packed_size_accounting():
    """The 49-block tensor set (8 x 5120x5120, 13824x5120, 5120x13824 per block) with the
    mixed-precision widths: the library's packed-size answers add up to the bitstream size
    (b/8 bytes per weight) plus one fp32 step per 128 weights, against 2 bytes per weight in
    bf16."""
    from bit_weight_quantization_wq_b200 import synth
    total_bf16 = total_packed = 0
    for block in range(49):
        widths = synth.mixed_bits(len(synth.BLOCK_SHAPES), config=5, block=block)
        for (N, K), bits in zip(synth.BLOCK_SHAPES, widths):
            total_bf16 += 2 * N * K
            packed = B.lib().wq_packed_bytes(N, K, bits, 128)
            steps = B.lib().wq_scales_count(N, K, 128)
            assert packed == N * K * bits // 8 and steps == N * K // 128
            total_packed += packed + 4 * steps
    assert total_bf16 == 49 * 2 * (8 * 5120 * 5120 + 2 * 13824 * 5120)
    ratio = total_packed / total_bf16
    assert 0.25 < ratio < 0.40      # ~5 bits per weight on average
