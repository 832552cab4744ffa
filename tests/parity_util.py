"""Shared helpers for the GPU-vs-oracle parity tests.

Tolerances (stated once, used by every parity test):
  H        relative Frobenius error <= 1e-5   (upper triangle)
  U        relative Frobenius error <= 1e-4
  codes    >= 99.9% identical.  In every row the codes agree exactly up to
           the row's first difference (its "initiating flip"), and that
           first difference is off by exactly one level at a near-tie: the
           oracle's value w/s + z lies within TIE_TOL of a rounding boundary.
           After an initiating flip the row's later weights are compensated
           differently, so its later codes follow another valid trajectory;
           those are bounded by the fraction and the loss criteria.  (An fp32
           restatement of the sweep on the CPU shows the same cascades,
           including later codes two levels apart.)
           A flip need not die out: with group grids the later groups' grids
           come from the differently compensated weights, and with one grid
           per row the compensation of the later columns changes by a whole
           grid step, so the rest of the row can follow another trajectory.
           If decisions flip at a rate rho, the expected differing fraction of
           a row of d_in codes is up to rho * d_in / 2, and fp32 arithmetic
           against the fp64 oracle has rho of a few 1e-6.  So the identical
           fraction is held to min(99.9%, 1 - rho_max * d_in / 2), and where a
           comparison on one common U has over 1e5 decisions, the flips
           themselves to at most rho_max * decisions + 2 (rho_max = RHO_MAX *
           maxq / 15).
  loss     ||W X^T - W^ X^T||^2 within 0.5% (relative) of the oracle's
  grid     per-row scales/zeros (from the original W) and RTN: bit-exact;
           group scales/zeros: bit-exact given the GPU's own group min/max.
           Where a row's group grid differs from the oracle's before its first
           code difference, the difference must be a rounding near-tie of the
           oracle's own grid computation: the scale one fp16 step away with the
           oracle's fp32 range/maxq within GRID_TIE_REL of the fp16 rounding
           boundary, or the same scale and the zero one step away with the
           oracle's -min/s within TIE_TOL of a half-integer.  Any other grid
           difference fails.
"""
import numpy as np
import torch

import oracle
from post_weight_quantization_05_b200 import synth

H_TOL = 1e-5
U_TOL = 1e-4
CODE_MATCH = 0.999
LOSS_TOL = 0.005
TIE_TOL = 5e-3
GRID_TIE_REL = 1e-4
# Flips per decision allowed at 4 bits (see check_codes), scaled by maxq / 15
# for other widths (a finer grid puts each weight nearer a rounding boundary):
# measured on a B200, the fp32 sweep against the fp64 oracle moves
# 0.5e-6 .. 4e-6 decisions per decision across a tie on one common U, and
# about 5e-6 end to end (the GPU's fp32 H adds its own moves).
RHO_MAX = 1e-5


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


def _fp16_neighbours(x32):
    """The two fp16 values around an fp32 value and the fp32 midpoint between them."""
    h = np.float16(x32)
    hf = np.float32(h)
    other = np.nextafter(h, np.float16(np.inf) if hf < x32 else np.float16(-np.inf), dtype=np.float16)
    lo, hi = sorted([float(hf), float(np.float32(other))])
    return lo, hi, 0.5 * (lo + hi)


def grid_flip_at_tie(ref, r, gi, s_gpu, z_gpu):
    """True if the GPU's grid (s_gpu, z_gpu) of row r, group gi differs from
    the oracle's only by a rounding near-tie of the oracle's own computation
    (reading R5: s = fp16(fp32(max(range, 1e-8) / maxq)), z = fp16(rint(-min/s))).
    Returns (ok, description)."""
    maxq = np.float32(2 ** int(ref["bits"]) - 1)
    mn = np.float32(ref["gmin"][r, gi])
    mx = np.float32(ref["gmax"][r, gi])
    s_ref = float(ref["scales"][r, gi])
    z_ref = float(ref["zeros"][r, gi])
    if s_gpu != s_ref:
        s32 = np.float32(np.maximum(mx - mn, np.float32(1e-8)) / maxq)
        lo, hi, mid = _fp16_neighbours(s32)
        rel = abs(float(s32) - mid) / float(s32)
        ok = (s_gpu in (lo, hi)) and rel <= GRID_TIE_REL
        return ok, f"scale {s_gpu} vs {s_ref}: oracle range/maxq {float(s32):.9g} is {rel:.2e} (relative) from the fp16 boundary"
    t = float(np.float32(-mn / np.float32(s_ref)))
    dist = abs((t - np.floor(t)) - 0.5)
    ok = abs(z_gpu - z_ref) == 1 and dist <= TIE_TOL
    return ok, f"zero {z_gpu} vs {z_ref}: oracle -min/s {t:.6f} is {dist:.2e} from a half-integer"


def check_codes(got, ref, what="", match=CODE_MATCH, bits=None, groupsize=-1, gpu_scales=None,
                gpu_zeros=None, rate_check=False):
    """`ref` is the oracle's output dict (with the trace when available).
    rate_check: also bound the flips per decision (for comparisons on one
    common U, where the rate measures the sweep's arithmetic; end to end it
    also depends on how H's fp32 error is amplified by its conditioning)."""
    got = np.asarray(got)
    rc = np.asarray(ref["codes"])
    d_in = rc.shape[1]
    diff = np.abs(got - rc)
    frac = float(np.mean(diff == 0))
    rho = RHO_MAX * (2 ** int(ref.get("bits", 4)) - 1) / 15.0
    need = min(match, 1.0 - rho * d_in / 2)
    assert frac >= need, f"{what}: only {frac:.6f} of codes identical (need {need:.6f})"
    flips, decisions = decision_stats(got, rc)
    if rate_check and decisions > 100000:
        assert flips <= rho * decisions + 2, f"{what}: {flips} flips in {decisions} decisions"
    if "W_at" not in ref:
        return frac
    g = d_in if groupsize <= 0 else groupsize
    s_full = np.repeat(np.asarray(ref["scales"], np.float64), g, axis=1)[:, :d_in]
    z_full = np.repeat(np.asarray(ref["zeros"], np.float64), g, axis=1)[:, :d_in]
    grid_differs = None
    if gpu_scales is not None:
        gs = np.asarray(gpu_scales, np.float64)
        gz = np.asarray(gpu_zeros, np.float64)
        grid_differs = (gs != np.asarray(ref["scales"], np.float64)) | (gz != np.asarray(ref["zeros"], np.float64))
    for r in np.where(diff.max(axis=1) > 0)[0]:
        j = int(np.argmax(diff[r] > 0))
        if grid_differs is not None and grid_differs[r, : j // g + 1].any():
            # the row's grid changed first: allowed only at a rounding near-tie of the oracle's grid
            gi = int(np.argmax(grid_differs[r]))
            ok, why = grid_flip_at_tie(ref, r, gi, float(gs[r, gi]), float(gz[r, gi]))
            assert ok, f"{what}: row {r} group {gi} grid differs away from a tie ({why})"
            continue
        assert diff[r, j] == 1, f"{what}: row {r} first differs at column {j} by {diff[r, j]} levels"
        t = ref["W_at"][r, j] / s_full[r, j] + z_full[r, j]
        dist = abs((t - np.floor(t)) - 0.5)
        assert dist <= TIE_TOL, f"{what}: row {r} col {j} flipped away from a tie (distance {dist:.2e})"
    return frac


def decision_stats(got, ref_codes):
    """Per-decision agreement along the sweep.  In each row the codes up to
    and including its first difference were decided from identical states;
    returns (rows with a difference, decisions taken from identical states).
    Their ratio is the rate at which the two sides' arithmetic decides a
    code differently, without the cascade that follows a flip."""
    diff = np.asarray(got) != np.asarray(ref_codes)
    any_d = diff.any(axis=1)
    first = np.where(any_d, np.argmax(diff, axis=1) + 1, diff.shape[1])
    return int(any_d.sum()), int(first.sum())


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
    out = oracle.gptq_quantize(W, U, problem.bits, problem.blocksize, problem.groupsize, return_trace=True)
    return H, U, out


def group_grid_from(W_state, bits, groupsize):
    """Grid of each group computed by the oracle's formula from given weights."""
    d_out, d_in = W_state.shape
    ng = d_in // groupsize
    s = np.zeros((d_out, ng), np.float32)
    z = np.zeros((d_out, ng), np.float32)
    for gi in range(ng):
        blk = np.asarray(W_state[:, gi * groupsize:(gi + 1) * groupsize], np.float32)
        s[:, gi], z[:, gi] = oracle.grid_params(blk.min(1), blk.max(1), bits)
    return s, z
