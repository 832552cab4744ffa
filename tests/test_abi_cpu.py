"""CPU-only checks of the C ABI: the library builds and loads without a GPU,
exports every entry point include/gptq.h declares, and rejects invalid
arguments on the host (before any CUDA call)."""
import ctypes
import os
import re

import pytest

from post_weight_quantization_05_b200 import _native, build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptq.h")


@pytest.fixture(scope="module")
def lib():
    build_lib.build()          # no-op when up to date; nvcc cross-compiles here
    return _native.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_\w+)\s*\(", text)))


def test_header_declares_the_four_stages():
    names = declared_functions()
    for n in ("gptq_hessian_accumulate", "gptq_prepare_hinv", "gptq_quantize_layer", "gptq_rtn_layer"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
    assert set(_native.SIGNATURES) == set(names)


def test_abi_version_and_status_strings(lib):
    assert lib.gptq_abi_version() == 1
    for code, name in _native.STATUS.items():
        assert lib.gptq_status_string(code).decode() == name


def test_workspace_sizes(lib):
    assert lib.gptq_hessian_workspace_size(_native.GPTQ_BF16, 1000, 512) == 0
    assert lib.gptq_hessian_workspace_size(_native.GPTQ_F32, 1000, 512) == 3 * 1000 * 512 * 2
    assert lib.gptq_prepare_hinv_workspace_size(512) >= 2 * 512 * 512 * 4
    assert lib.gptq_prepare_hinv_workspace_size(100) == 0          # d_in % 128 != 0
    # E [d_out, min(d_in, 1024)] and U^T [d_in, d_in], each as a tf32 part and a remainder
    assert lib.gptq_quantize_workspace_size(300, 512, 128) == 2 * ((300 * 512 * 4 + 255) // 256) * 256 + 2 * 512 * 512 * 4
    assert lib.gptq_quantize_workspace_size(300, 4096, 128) == 2 * 300 * 1024 * 4 + 2 * 4096 * 4096 * 4
    assert lib.gptq_quantize_workspace_size(300, 512, 64) == 0


FAKE = ctypes.c_void_p(0x10000)   # 16-byte aligned, never dereferenced: validation fails first
MIS = ctypes.c_void_p(0x10004)    # misaligned


def test_hessian_rejects_bad_arguments(lib):
    f = lib.gptq_hessian_accumulate
    assert f(None, 1, 64, 512, FAKE, None, 0, None) == 1            # NULL X
    assert f(FAKE, 1, 64, 512, None, None, 0, None) == 1            # NULL H
    assert f(FAKE, 1, 64, 500, FAKE, None, 0, None) == 1            # d_in % 128
    assert f(FAKE, 1, 64, 65536, FAKE, None, 0, None) == 1          # d_in too large
    assert f(FAKE, 7, 64, 512, FAKE, None, 0, None) == 1            # dtype
    assert f(MIS, 1, 64, 512, FAKE, None, 0, None) == 1             # alignment
    assert f(FAKE, 0, 64, 512, FAKE, None, 0, None) == 1            # fp32 needs workspace
    assert f(FAKE, 0, 64, 512, FAKE, FAKE, 100, None) == 1          # workspace too small
    assert f(FAKE, 1, -1, 512, FAKE, None, 0, None) == 1            # negative n
    assert f(None, 1, 0, 512, None, None, 0, None) == 0             # n == 0: no-op


def test_hessian_batches_rejects_bad_arguments(lib):
    f = lib.gptq_hessian_accumulate_batches
    P = ctypes.c_void_p
    X2 = (P * 2)(FAKE.value, FAKE.value)
    n2 = (ctypes.c_int64 * 2)(64, 32)
    assert f(X2, n2, 2, 1, 512, None, None, 0, None) == 1                       # NULL H
    assert f(None, n2, 2, 1, 512, FAKE, None, 0, None) == 1                     # NULL X array
    assert f(X2, None, 2, 1, 512, FAKE, None, 0, None) == 1                     # NULL n array
    assert f(X2, n2, -1, 1, 512, FAKE, None, 0, None) == 1                      # negative count
    assert f(X2, n2, 2, 7, 512, FAKE, None, 0, None) == 1                       # dtype
    assert f(X2, n2, 2, 1, 500, FAKE, None, 0, None) == 1                       # d_in % 128
    assert f((P * 2)(FAKE.value, MIS.value), n2, 2, 1, 512, FAKE, None, 0, None) == 1   # misaligned batch
    assert f((P * 2)(FAKE.value, None), n2, 2, 1, 512, FAKE, None, 0, None) == 1        # NULL batch with rows
    assert f(X2, (ctypes.c_int64 * 2)(64, -1), 2, 1, 512, FAKE, None, 0, None) == 1     # negative rows
    assert f(X2, n2, 2, 0, 512, FAKE, None, 0, None) == 1                       # fp32 needs workspace
    assert f(X2, n2, 2, 0, 512, FAKE, FAKE, 3 * 32 * 512 * 2, None) == 1        # sized for the smaller batch
    assert f((P * 2)(None, None), (ctypes.c_int64 * 2)(0, 0), 2, 1, 512, FAKE, None, 0, None) == 0   # all empty
    assert f(None, None, 0, 1, 512, FAKE, None, 0, None) == 0                   # no batches


def test_prepare_hinv_rejects_bad_arguments(lib):
    f = lib.gptq_prepare_hinv
    ws = lib.gptq_prepare_hinv_workspace_size(512)
    assert f(None, 512, 0.01, FAKE, None, FAKE, ws, None) == 1
    assert f(FAKE, 512, 0.01, None, None, FAKE, ws, None) == 1
    assert f(FAKE, 512, 0.01, FAKE, None, None, ws, None) == 1
    assert f(FAKE, 512, 0.01, FAKE, None, FAKE, ws - 1, None) == 1
    assert f(FAKE, 512, -0.1, FAKE, None, FAKE, ws, None) == 1
    assert f(FAKE, 512, float("nan"), FAKE, None, FAKE, ws, None) == 1
    assert f(FAKE, 384 + 1, 0.01, FAKE, None, FAKE, ws, None) == 1
    assert f(FAKE, 512, 0.01, FAKE, ctypes.c_void_p(0x10002), FAKE, ws, None) == 1


def test_quantize_rejects_bad_arguments(lib):
    f = lib.gptq_quantize_layer
    ws = lib.gptq_quantize_workspace_size(64, 512, 128)
    ok = [FAKE, 64, 512, FAKE, 4, 128, -1, FAKE, FAKE, FAKE, None, FAKE, ws, None]

    def call(**kw):
        a = list(ok)
        idx = {"W": 0, "d_out": 1, "d_in": 2, "U": 3, "bits": 4, "bs": 5, "g": 6, "codes": 7, "scales": 8,
               "zeros": 9, "Q": 10, "ws": 11, "wsb": 12}
        for k, v in kw.items():
            a[idx[k]] = v
        return f(*a)

    assert call(W=None) == 1
    assert call(U=None) == 1
    assert call(codes=None) == 1
    assert call(ws=None) == 1
    assert call(wsb=ws - 4) == 1
    assert call(d_out=0) == 1
    assert call(d_in=320) == 1
    assert call(bits=5) == 1
    assert call(bits=1) == 1
    assert call(g=64) == 1            # not a multiple of 128
    assert call(g=384) == 1           # does not divide 512
    assert call(bs=64) == 2           # valid for the method, unsupported here
    assert call(W=MIS) == 1
    assert call(Q=MIS) == 1
    assert call(scales=ctypes.c_void_p(0x10001)) == 1


def test_rtn_and_helpers_reject_bad_arguments(lib):
    f = lib.gptq_rtn_layer
    assert f(None, 64, 512, 4, -1, FAKE, FAKE, FAKE, None, None) == 1
    assert f(FAKE, 64, 512, 6, -1, FAKE, FAKE, FAKE, None, None) == 1
    assert f(FAKE, 64, 512, 4, 100, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.gptq_widen_bf16(None, FAKE, 10, None) == 1
    assert lib.gptq_widen_bf16(FAKE, FAKE, -1, None) == 1
    assert lib.gptq_widen_bf16(None, None, 0, None) == 0
    assert lib.gptq_fill_f32(None, 10, 0.0, None) == 1
    assert lib.gptq_fill_f32(ctypes.c_void_p(0x10001), 10, 0.0, None) == 1


def test_act_order_entries_reject_bad_arguments(lib):
    d = 512
    big = 0x10000 + d * d * 4 + 4096                  # an address past H / Hp / src
    P = ctypes.c_void_p(big)
    f = lib.gptq_act_order_perm
    assert f(None, d, P, None) == 1
    assert f(FAKE, d, None, None) == 1
    assert f(MIS, d, P, None) == 1
    assert f(FAKE, 500, P, None) == 1                 # d_in % 128 != 0
    assert f(FAKE, d, ctypes.c_void_p(big + 2), None) == 1
    assert f(FAKE, d, ctypes.c_void_p(0x10000 + 64), None) == 1     # perm inside H
    g = lib.gptq_permute_hessian
    HP = ctypes.c_void_p(big + 65536)
    assert g(None, d, P, HP, None) == 1
    assert g(FAKE, d, None, HP, None) == 1
    assert g(FAKE, d, P, None, None) == 1
    assert g(FAKE, d, P, ctypes.c_void_p(0x10000 + 4096), None) == 1  # Hp overlaps H
    assert g(FAKE, d, P, ctypes.c_void_p(big + 65536 + 4), None) == 1
    assert g(FAKE, 0, P, HP, None) == 1
    c = lib.gptq_permute_columns
    assert c(FAKE, 64, d, P, 2, FAKE, None) == 1        # inverse not 0 / 1
    assert c(FAKE, -1, d, P, 0, FAKE, None) == 1
    assert c(FAKE, 64, 300, P, 0, FAKE, None) == 1
    assert c(FAKE, 64, d, None, 0, FAKE, None) == 1
    assert c(MIS, 64, d, P, 0, FAKE, None) == 1
    assert c(FAKE, 64, d, P, 0, ctypes.c_void_p(0x10000 + 1024), None) == 1   # partial overlap
    assert c(FAKE, 64, d, ctypes.c_void_p(0x10000 + 256), 0, FAKE, None) == 1  # perm inside dst
    assert c(None, 0, d, None, 0, None, None) == 0      # no rows: nothing to do


def test_dequant_gemv_rejects_bad_arguments(lib):
    r256 = lambda b: (b + 255) // 256 * 256  # noqa: E731
    assert lib.gptq_dequant_gemv_workspace_size(1, 4096, 1) == r256(8192) + r256(32 * 8)
    assert lib.gptq_dequant_gemv_workspace_size(3, 640, 0) == r256(3 * 640 * 2) + r256(3 * 5 * 8)
    assert lib.gptq_dequant_gemv_workspace_size(9, 4096, 1) == 0
    f = lib.gptq_dequant_gemv
    ok = dict(codes=FAKE, scales=FAKE, zeros=FAKE, d_out=64, d_in=512, bits=4, g=128, perm=None, x=FAKE, m=2,
              y=FAKE, ws=FAKE, ws_bytes=1 << 20)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["codes"], a["scales"], a["zeros"], a["d_out"], a["d_in"], a["bits"], a["g"], a["perm"], a["x"],
                 a["m"], a["y"], a["ws"], a["ws_bytes"], None)
    assert call(bits=3) == 2 and call(bits=8) == 2 and call(bits=2) == 2      # valid, not in this build
    assert call(bits=5) == 1
    assert call(m=9) == 1 and call(m=-1) == 1
    assert call(m=0, codes=None, x=None, y=None) == 0                       # nothing to do
    assert call(d_in=300) == 1 and call(g=100) == 1 and call(d_out=0) == 1
    assert call(codes=MIS) == 1 and call(x=MIS) == 1 and call(y=ctypes.c_void_p(0x10002)) == 1
    assert call(scales=ctypes.c_void_p(0x10001)) == 1 and call(codes=None) == 1
    assert call(ws=None) == 1 and call(ws_bytes=100) == 1 and call(ws=MIS) == 1   # the workspace is required
    assert call(perm=ctypes.c_void_p(0x10002), ws=FAKE, ws_bytes=4096) == 1


def test_dequantize_rejects_bad_arguments(lib):
    f = lib.gptq_dequantize
    ok = dict(codes=FAKE, scales=FAKE, zeros=FAKE, d_out=64, d_in=512, bits=3, g=128, perm=None, dt=1, out=FAKE)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["codes"], a["scales"], a["zeros"], a["d_out"], a["d_in"], a["bits"], a["g"], a["perm"], a["dt"],
                 a["out"], None)
    assert call(bits=5) == 1 and call(bits=1) == 1
    assert call(dt=3) == 1 and call(dt=-1) == 1
    assert call(d_in=300) == 1 and call(g=100) == 1 and call(d_out=0) == 1
    assert call(codes=None) == 1 and call(out=None) == 1
    assert call(codes=ctypes.c_void_p(0x10002)) == 1 and call(out=MIS) == 1
    assert call(perm=MIS) == 1 and call(scales=ctypes.c_void_p(0x10001)) == 1


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError):
        _native._lib = None
        try:
            _native.load(str(tmp_path / "missing.so"))
        finally:
            _native._lib = None
