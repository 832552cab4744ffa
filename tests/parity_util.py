"""Shared helpers for the GPU-vs-oracle parity tests.

Tolerances (stated once, used by every parity test):
  H        relative Frobenius error <= 1e-5   (upper triangle)
  U        relative Frobenius error <= 1e-4
  codes    >= 99.9% identical; every differing code off by exactly one level
  loss     ||W X^T - W^ X^T||^2 within 0.5% (relative) of the oracle's
  grid     per-row scales/zeros (from the original W) and RTN: bit-exact
"""
import numpy as np
import torch

import oracle
from post_weight_quantization_05_b200 import synth

H_TOL = 1e-5
U_TOL = 1e-4
CODE_MATCH = 0.999
LOSS_TOL = 0.005


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def upper(a):
    return np.triu(np.asarray(a, dtype=np.float64))


def to_dev_x(problem, xb):
    if problem.x_dtype == "bf16":
        return torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(xb, dtype=np.float32)).cuda()


def unpack_gpu_codes(codes_t, bits, d_in):
    words = codes_t.cpu().numpy().view(np.uint32)
    return oracle.unpack_codes(words, bits, d_in)


def fp16_values(t):
    return t.cpu().float().numpy().astype(np.float32)


def check_codes(got, ref, what=""):
    got = np.asarray(got)
    ref = np.asarray(ref)
    diff = np.abs(got - ref)
    frac = float(np.mean(diff == 0))
    assert frac >= CODE_MATCH, f"{what}: only {frac:.6f} of codes identical"
    assert diff.max() <= 1, f"{what}: a code differs by {diff.max()} levels"
    return frac


def dequant_rows(codes, scales, zeros, groupsize):
    d_in = codes.shape[1]
    g = d_in if groupsize <= 0 else groupsize
    s = np.repeat(np.asarray(scales, np.float64), g, axis=1)[:, :d_in]
    z = np.repeat(np.asarray(zeros, np.float64), g, axis=1)[:, :d_in]
    return s * (codes - z)


def oracle_pipeline(problem, batches=None, rows=None):
    """The oracle end to end (fp64): H, damping, U, sweep (optionally on a
    subset of rows -- rows are independent given U)."""
    if batches is None:
        batches = [synth.x_as_f32(problem, problem.x_batch(b)) for b in range(problem.n_batches)]
    H = oracle.hessian(batches)
    Hd, lam = oracle.damp(H, problem.percdamp)
    U = oracle.hinv_upper_factor(Hd)
    W = problem.W if rows is None else problem.W[rows]
    out = oracle.gptq_quantize(W, U, problem.bits, problem.blocksize, problem.groupsize)
    return H, U, out
