"""Python binding of libgptq: the C entry points under the same names,
taking torch CUDA tensors.  Argument marshalling only -- every step runs in
the library's kernels; torch provides device memory and streams.
"""
from __future__ import annotations

import ctypes

import torch

from . import _native
from ._native import GPTQ_BF16, GPTQ_F32, STATUS


class GPTQError(RuntimeError):
    def __init__(self, code: int, where: str, detail: int | None = None):
        self.code = code
        self.detail = detail
        msg = f"{where}: {STATUS.get(code, code)}"
        if detail is not None:
            msg += f" (detail {detail})"
        super().__init__(msg)


def _lib():
    return _native.load()


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(code: int, where: str):
    if code != 0:
        raise GPTQError(code, where)


def _need(t, dtype, shape, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def abi_version() -> int:
    return _lib().gptq_abi_version()


def launch_count() -> int:
    """Kernels this library has enqueued so far in this process."""
    return int(_lib().gptq_launch_count())


# ----------------------------------------------------------------- sizes
def hessian_workspace_size(dtype: int, n: int, d_in: int) -> int:
    return _lib().gptq_hessian_workspace_size(dtype, n, d_in)


def prepare_hinv_workspace_size(d_in: int) -> int:
    return _lib().gptq_prepare_hinv_workspace_size(d_in)


def quantize_workspace_size(d_out: int, d_in: int, blocksize: int = 128) -> int:
    return _lib().gptq_quantize_workspace_size(d_out, d_in, blocksize)


def workspace(nbytes: int, device) -> torch.Tensor:
    """A byte buffer (16-byte aligned by the caching allocator)."""
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


# ----------------------------------------------------------------- stages
def hessian_accumulate(X: torch.Tensor, H: torch.Tensor, ws: torch.Tensor | None = None, stream=None):
    """H += 2 X^T X (upper triangle), X [n, d_in] bf16 or fp32."""
    n, d = X.shape
    dtype = GPTQ_BF16 if X.dtype == torch.bfloat16 else GPTQ_F32
    if X.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("X must be bf16 or fp32")
    _need(X, X.dtype, (n, d), "X")
    _need(H, torch.float32, (d, d), "H")
    need = hessian_workspace_size(dtype, n, d)
    if need and ws is None:
        raise ValueError(f"fp32 X needs a workspace of {need} bytes")
    code = _lib().gptq_hessian_accumulate(_ptr(X), dtype, n, d, _ptr(H), _ptr(ws),
                                          0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "gptq_hessian_accumulate")


def hessian_accumulate_batches(Xs, H: torch.Tensor, ws: torch.Tensor | None = None, stream=None):
    """H += 2 X_i^T X_i for every batch X_i in order (one call; the batches'
    contractions overlap on the GPU).  All X_i share one dtype and d_in."""
    Xs = list(Xs)
    if not Xs:
        return
    d = H.shape[0]
    if Xs[0].dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("X must be bf16 or fp32")
    dtype = GPTQ_BF16 if Xs[0].dtype == torch.bfloat16 else GPTQ_F32
    for X in Xs:
        _need(X, Xs[0].dtype, (X.shape[0], d), "X")
    _need(H, torch.float32, (d, d), "H")
    need = hessian_workspace_size(dtype, max(X.shape[0] for X in Xs), d)
    if need and ws is None:
        raise ValueError(f"fp32 X needs a workspace of {need} bytes")
    ptrs = (ctypes.c_void_p * len(Xs))(*[X.data_ptr() for X in Xs])
    rows = (ctypes.c_int64 * len(Xs))(*[X.shape[0] for X in Xs])
    code = _lib().gptq_hessian_accumulate_batches(ptrs, rows, len(Xs), dtype, d, _ptr(H), _ptr(ws),
                                                  0 if ws is None else ws.numel() * ws.element_size(),
                                                  _stream(stream))
    _check(code, "gptq_hessian_accumulate_batches")


def prepare_hinv(H: torch.Tensor, U: torch.Tensor, ws: torch.Tensor, percdamp: float = 0.01,
                 info: torch.Tensor | None = None, stream=None):
    """U = upper Cholesky factor of (H + percdamp * mean(diag H) I)^-1."""
    d = H.shape[0]
    _need(H, torch.float32, (d, d), "H")
    _need(U, torch.float32, (d, d), "U")
    if info is not None:
        _need(info, torch.int32, (1,), "info")
    code = _lib().gptq_prepare_hinv(_ptr(H), d, percdamp, _ptr(U), _ptr(info), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "gptq_prepare_hinv")


def n_groups(d_in: int, groupsize: int) -> int:
    return 1 if groupsize <= 0 else d_in // groupsize


def quantize_layer(W: torch.Tensor, U: torch.Tensor, bits: int, blocksize: int, groupsize: int,
                   codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, ws: torch.Tensor,
                   Q: torch.Tensor | None = None, stream=None):
    """Blocked GPTQ sweep over W (fp32, overwritten); writes packed codes,
    fp16 scales/zeros and, optionally, the dequantized Q."""
    d_out, d_in = W.shape
    ng = n_groups(d_in, groupsize)
    _need(W, torch.float32, (d_out, d_in), "W")
    _need(U, torch.float32, (d_in, d_in), "U")
    _need(codes, torch.int32, (d_out, d_in * bits // 32), "codes")
    _need(scales, torch.float16, (d_out, ng), "scales")
    _need(zeros, torch.float16, (d_out, ng), "zeros")
    if Q is not None:
        _need(Q, torch.float32, (d_out, d_in), "Q")
    code = _lib().gptq_quantize_layer(_ptr(W), d_out, d_in, _ptr(U), bits, blocksize, groupsize, _ptr(codes),
                                      _ptr(scales), _ptr(zeros), _ptr(Q), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "gptq_quantize_layer")


def rtn_layer(W: torch.Tensor, bits: int, groupsize: int, codes: torch.Tensor, scales: torch.Tensor,
              zeros: torch.Tensor, Q: torch.Tensor | None = None, stream=None):
    d_out, d_in = W.shape
    ng = n_groups(d_in, groupsize)
    _need(W, torch.float32, (d_out, d_in), "W")
    _need(codes, torch.int32, (d_out, d_in * bits // 32), "codes")
    _need(scales, torch.float16, (d_out, ng), "scales")
    _need(zeros, torch.float16, (d_out, ng), "zeros")
    if Q is not None:
        _need(Q, torch.float32, (d_out, d_in), "Q")
    code = _lib().gptq_rtn_layer(_ptr(W), d_out, d_in, bits, groupsize, _ptr(codes), _ptr(scales), _ptr(zeros),
                                 _ptr(Q), _stream(stream))
    _check(code, "gptq_rtn_layer")


def act_order_perm(H: torch.Tensor, perm: torch.Tensor, stream=None):
    """perm = column indices by descending diag(H) (ties by index, NaN last)."""
    d = H.shape[0]
    _need(H, torch.float32, (d, d), "H")
    _need(perm, torch.int32, (d,), "perm")
    _check(_lib().gptq_act_order_perm(_ptr(H), d, _ptr(perm), _stream(stream)), "gptq_act_order_perm")


def permute_hessian(H: torch.Tensor, perm: torch.Tensor, Hp: torch.Tensor, stream=None):
    """Hp = Hs[perm][:, perm], Hs the symmetric matrix of H's upper triangle."""
    d = H.shape[0]
    _need(H, torch.float32, (d, d), "H")
    _need(perm, torch.int32, (d,), "perm")
    _need(Hp, torch.float32, (d, d), "Hp")
    _check(_lib().gptq_permute_hessian(_ptr(H), d, _ptr(perm), _ptr(Hp), _stream(stream)), "gptq_permute_hessian")


def permute_columns(src: torch.Tensor, perm: torch.Tensor, dst: torch.Tensor | None = None, inverse: bool = False,
                    stream=None):
    """dst[:, k] = src[:, perm[k]] (inverse: dst[:, perm[k]] = src[:, k]); in
    place when dst is src or None."""
    rows, cols = src.shape
    dst = src if dst is None else dst
    _need(src, torch.float32, (rows, cols), "src")
    _need(dst, torch.float32, (rows, cols), "dst")
    _need(perm, torch.int32, (cols,), "perm")
    _check(_lib().gptq_permute_columns(_ptr(src), rows, cols, _ptr(perm), 1 if inverse else 0, _ptr(dst),
                                       _stream(stream)), "gptq_permute_columns")


def dequant_gemv_workspace_size(m: int, d_in: int, with_perm: bool) -> int:
    return _lib().gptq_dequant_gemv_workspace_size(m, d_in, 1 if with_perm else 0)


def dequant_gemv(codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, bits: int, groupsize: int,
                 x: torch.Tensor, y: torch.Tensor, perm: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                 stream=None):
    """y[t] = x[t] W^T with W^ rebuilt from the stored form (codes in
    processing order; perm maps code column k to input column perm[k])."""
    d_out = codes.shape[0]
    m, d_in = x.shape
    ng = n_groups(d_in, groupsize)
    _need(codes, torch.int32, (d_out, d_in * bits // 32), "codes")
    _need(scales, torch.float16, (d_out, ng), "scales")
    _need(zeros, torch.float16, (d_out, ng), "zeros")
    _need(x, torch.bfloat16, (m, d_in), "x")
    _need(y, torch.float32, (m, d_out), "y")
    if perm is not None:
        _need(perm, torch.int32, (d_in,), "perm")
    if ws is None and m > 0:
        ws = workspace(dequant_gemv_workspace_size(m, d_in, perm is not None), x.device)
    code = _lib().gptq_dequant_gemv(_ptr(codes), _ptr(scales), _ptr(zeros), d_out, d_in, bits, groupsize,
                                    _ptr(perm), _ptr(x), m, _ptr(y), _ptr(ws),
                                    0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "gptq_dequant_gemv")


_OUT_DTYPES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}


def dequantize(codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, bits: int, groupsize: int,
               out: torch.Tensor, perm: torch.Tensor | None = None, stream=None):
    """out = the weights rebuilt from the stored form, in W's column order:
    s (c - z) rounded once to fp32 (exact for integer zero points), or that
    value rounded to nearest even in bf16 / fp16."""
    d_out, d_in = out.shape
    ng = n_groups(d_in, groupsize)
    _need(codes, torch.int32, (d_out, d_in * bits // 32), "codes")
    _need(scales, torch.float16, (d_out, ng), "scales")
    _need(zeros, torch.float16, (d_out, ng), "zeros")
    if out.dtype not in _OUT_DTYPES:
        raise ValueError("out must be fp32, bf16 or fp16")
    _need(out, out.dtype, (d_out, d_in), "out")
    if perm is not None:
        _need(perm, torch.int32, (d_in,), "perm")
    _check(_lib().gptq_dequantize(_ptr(codes), _ptr(scales), _ptr(zeros), d_out, d_in, bits, groupsize, _ptr(perm),
                                  _OUT_DTYPES[out.dtype], _ptr(out), _stream(stream)), "gptq_dequantize")


def widen_bf16(src: torch.Tensor, dst: torch.Tensor, stream=None):
    if src.dtype != torch.bfloat16 or dst.dtype != torch.float32 or src.numel() != dst.numel():
        raise ValueError("widen_bf16: bf16 -> fp32 of equal size")
    _check(_lib().gptq_widen_bf16(_ptr(src), _ptr(dst), src.numel(), _stream(stream)), "gptq_widen_bf16")


def fill_f32(t: torch.Tensor, value: float = 0.0, stream=None):
    if t.dtype != torch.float32 or not t.is_contiguous():
        raise ValueError("fill_f32: contiguous fp32 tensor")
    _check(_lib().gptq_fill_f32(_ptr(t), t.numel(), value, _stream(stream)), "gptq_fill_f32")


def get_status(stream=None, raise_on_error: bool = True):
    """Synchronize the stream and fetch (and clear) the device status word."""
    detail = ctypes.c_int(0)
    code = _lib().gptq_get_status(_stream(stream), ctypes.byref(detail))
    if code and raise_on_error:
        raise GPTQError(code, "device status", detail.value)
    return code, detail.value


# ----------------------------------------------------------------- a layer
class LayerQuantizer:
    """Device buffers for one layer shape plus the four calls in order.

    Allocation happens here, once (torch caching allocator); the calls
    themselves only enqueue kernels.  With act_order the columns are taken by
    descending diag(H): codes, scales and zeros come out in that processing
    order (self.perm[k] is the column of W that code column k belongs to) and
    Q in W's own order."""

    def __init__(self, d_out: int, d_in: int, bits: int = 4, groupsize: int = -1, blocksize: int = 128,
                 percdamp: float = 0.01, device="cuda", want_q: bool = False, max_f32_rows: int = 0,
                 act_order: bool = False):
        self.d_out, self.d_in, self.bits, self.groupsize = d_out, d_in, bits, groupsize
        self.blocksize, self.percdamp, self.act_order = blocksize, percdamp, act_order
        dev = torch.device(device)
        self.H = torch.empty((d_in, d_in), dtype=torch.float32, device=dev)
        self.U = torch.empty((d_in, d_in), dtype=torch.float32, device=dev)
        self.W = torch.empty((d_out, d_in), dtype=torch.float32, device=dev)
        self.codes = torch.empty((d_out, d_in * bits // 32), dtype=torch.int32, device=dev)
        ng = n_groups(d_in, groupsize)
        self.scales = torch.empty((d_out, ng), dtype=torch.float16, device=dev)
        self.zeros = torch.empty((d_out, ng), dtype=torch.float16, device=dev)
        self.Q = torch.empty((d_out, d_in), dtype=torch.float32, device=dev) if want_q else None
        self.info = torch.zeros((1,), dtype=torch.int32, device=dev)
        self.ws_hinv = workspace(prepare_hinv_workspace_size(d_in), dev)
        self.ws_q = workspace(quantize_workspace_size(d_out, d_in, blocksize), dev)
        self.ws_h = workspace(hessian_workspace_size(GPTQ_F32, max_f32_rows, d_in), dev) if max_f32_rows else None
        self.perm = torch.empty((d_in,), dtype=torch.int32, device=dev) if act_order else None
        self.Hp = torch.empty((d_in, d_in), dtype=torch.float32, device=dev) if act_order else None

    def begin(self, W_src: torch.Tensor, stream=None):
        """Load the working copy of W (fp32 copy or bf16 widening) and zero H."""
        if W_src.dtype == torch.bfloat16:
            widen_bf16(W_src, self.W, stream)
        elif W_src.dtype == torch.float32:
            self.W.copy_(W_src)
        else:
            raise ValueError("W must be fp32 or bf16")
        fill_f32(self.H, 0.0, stream)

    def add_batch(self, X: torch.Tensor, stream=None):
        hessian_accumulate(X, self.H, self.ws_h, stream)

    def add_batches(self, Xs, stream=None):
        """Several resident batches in one call (faster than add_batch each)."""
        hessian_accumulate_batches(Xs, self.H, self.ws_h, stream)

    def finish(self, stream=None):
        H = self.H
        if self.act_order:
            act_order_perm(self.H, self.perm, stream)
            permute_hessian(self.H, self.perm, self.Hp, stream)
            permute_columns(self.W, self.perm, stream=stream)
            H = self.Hp
        prepare_hinv(H, self.U, self.ws_hinv, self.percdamp, self.info, stream)
        quantize_layer(self.W, self.U, self.bits, self.blocksize, self.groupsize, self.codes, self.scales,
                       self.zeros, self.ws_q, self.Q, stream)
        if self.act_order and self.Q is not None:
            permute_columns(self.Q, self.perm, inverse=True, stream=stream)
