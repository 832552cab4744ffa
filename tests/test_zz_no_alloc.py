"""The allocation-free quantize entry point (gptq_quantize_layer_noalloc).

Some callers cannot allocate device memory at the point where they quantize:
a framework whose memory pool owns every device buffer and hands out only
inputs and outputs, or a serving process that reserves its whole memory
budget at start-up and may not call cudaMalloc afterwards (the call can fail
once the budget is taken, and it synchronizes the device).  This entry point
takes no workspace and keeps its scratch in a fixed array inside the library.
These tests call it through the C ABI and compare it with gptq_quantize_layer
(which takes a caller workspace) on the same inputs, twice in a row so that
the second call starts from the scratch the first one left behind.  Both run
the same kernels on the same inputs, so their results must be identical bit
for bit.  This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_05_b200 import _native, api, build_lib, synth
from parity_util import check_codes, fp16_values, unpack_gpu_codes

pytestmark = pytest.mark.gpu


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _outputs(d_out, d_in, bits, groupsize):
    ng = api.n_groups(d_in, groupsize)
    return (torch.full((d_out, d_in * bits // 32), -1, dtype=torch.int32, device="cuda"),
            torch.full((d_out, ng), float("nan"), dtype=torch.float16, device="cuda"),
            torch.full((d_out, ng), float("nan"), dtype=torch.float16, device="cuda"),
            torch.full((d_out, d_in), float("nan"), dtype=torch.float32, device="cuda"))


def _problem(d_out, d_in, bits, groupsize, seed):
    p = synth.custom("noalloc", d_out, d_in, 3 * d_in, bits=bits, groupsize=groupsize, x_dtype="f32",
                     layer=seed)
    X = p.x_batch(0)
    Hd, _ = oracle.damp(oracle.hessian([X]), 0.01)
    return p, oracle.hinv_upper_factor(Hd)


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return _native.load()


@pytest.mark.parametrize("d_out,d_in,bits,groupsize", [(300, 640, 4, 128), (512, 512, 4, -1),
                                                      (96, 1024, 3, 256)])
def test_noalloc_matches_workspace_entry_point(lib, d_out, d_in, bits, groupsize):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):          # twice: the second call reuses the scratch as the first left it
        p, U = _problem(d_out, d_in, bits, groupsize, seed=10 * call + d_in + bits)
        Ut = torch.from_numpy(U.astype(np.float32)).cuda()
        W_ref = torch.from_numpy(p.W.copy()).cuda()
        W_na = torch.from_numpy(p.W.copy()).cuda()
        ref = _outputs(d_out, d_in, bits, groupsize)
        got = _outputs(d_out, d_in, bits, groupsize)
        ws = api.workspace(api.quantize_workspace_size(d_out, d_in), "cuda")
        rc = lib.gptq_quantize_layer(_ptr(W_ref), d_out, d_in, _ptr(Ut), bits, 128, groupsize, _ptr(ref[0]),
                                     _ptr(ref[1]), _ptr(ref[2]), _ptr(ref[3]), _ptr(ws),
                                     ws.numel(), stream)
        assert rc == 0
        rc = lib.gptq_quantize_layer_noalloc(_ptr(W_na), d_out, d_in, _ptr(Ut), bits, 128, groupsize,
                                             _ptr(got[0]), _ptr(got[1]), _ptr(got[2]), _ptr(got[3]), stream)
        assert rc == 0
        assert api.get_status() == (0, 0)
        # the same kernels on the same inputs: identical bits everywhere
        assert torch.equal(got[0], ref[0])
        assert torch.equal(got[1].view(torch.int16), ref[1].view(torch.int16))
        assert torch.equal(got[2].view(torch.int16), ref[2].view(torch.int16))
        assert torch.equal(got[3].view(torch.int32), ref[3].view(torch.int32))
        assert torch.equal(W_na.view(torch.int32), W_ref.view(torch.int32))
        c_got = unpack_gpu_codes(got[0], bits, d_in)
        # and against the oracle, like the workspace path
        ref_o = oracle.gptq_quantize(p.W, U, bits, 128, groupsize, return_trace=True)
        check_codes(c_got, ref_o, "noalloc", groupsize=groupsize, gpu_scales=fp16_values(got[1]),
                    gpu_zeros=fp16_values(got[2]))


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    """4096 x 4096 needs 128 MiB for the split U^T: over the 40 MiB array, refused before launching."""
    d = 4096
    W = torch.zeros((8, d), dtype=torch.float32, device="cuda")
    U = torch.zeros((d, d), dtype=torch.float32, device="cuda")
    codes, scales, zeros, Q = _outputs(8, d, 4, -1)
    rc = lib.gptq_quantize_layer_noalloc(_ptr(W), 8, d, _ptr(U), 4, 128, -1, _ptr(codes), _ptr(scales),
                                         _ptr(zeros), None, None)
    assert rc == 2   # GPTQ_ERR_UNSUPPORTED
    assert torch.all(codes == -1)
