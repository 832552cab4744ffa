"""Plain, slow, obviously-correct fp64 restatement of GPTQ layer quantization.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Sources (web pages on GPTQ; each function names the passage it follows):
  [wiki]  itwiki "GPTQ" article -- sections "문제 설정" (problem statement),
          "OBQ에서 GPTQ로" (OBQ and the three GPTQ changes), "알고리즘"
          (Algorithm 1), "최소 구현" (a minimal layer quantizer),
          "실무 변형" (group quantization, act-order).
  [blog]  "GPTQ를 밑바닥부터 구현하며 배운 것들" -- section 3 "구현 과정"
          (H = 2 X^T X, damping, the column update rule).

Everything is float64 except where the pages (or, where they are silent,
the CUDA kernels) fix a lower precision for a decision that produces an
integer: the grid's scale/zero and the rounding of w/scale are computed in
float32 and the scale/zero are stored as fp16 (Reading A), so that both sides
take those decisions in the same precision.

Readings of points the pages leave open (each also listed in the design
notes):
  R1  H is the plain sum H = sum_batches 2 X_b^T X_b (no running mean).
  R2  lambda = percdamp * mean(diag H) of the accumulated, undamped H.
  R3  "H^-1" in the update is the upper Cholesky factor U of (H+lambda I)^-1
      (U^T U = (H + lambda I)^-1), computed once up front.
  R4  rounding is round-half-to-even of w/scale, then + zero, then clamp to
      [0, maxq]; the division and the rounding are done in fp32.
  R5  grid (Reading A): s32 = max(wmax - wmin, 1e-8) / maxq in fp32;
      s = fp16(s32) (if that is 0, s = 2^-14); z = fp16(rint(-wmin / s)) with
      the division in fp32; the sweep uses exactly (s, z).
  R6  per-row grid: from the original W.  Group grid (g > 0): at each column
      j with j % g == 0, from the current (partially updated) W[:, j:j+g].
  R7  packing: little-endian bit stream of the codes along d_in, 32 codes per
      `bits` 32-bit words (int4: nibble k of word w holds code 8w+k).
  R8  natural column order 0..d_in-1 (act-order is a separate entry point).
  R14 act-order: columns by descending diag(H), ties by index; the damping
      is the same; groups are formed in processing order; codes / scales /
      zeros stay in processing order together with the permutation, and Q is
      returned in the original column order.
  R15 the inference product y = x W^T is computed from the stored form
      (packed codes, fp16 scales / zeros, the permutation) with W^ rebuilt
      exactly as s (c - z).

Parity status: every function here is pinned by a test in
tests/test_oracle_pins.py (closed forms, brute force, invariants, the page's
published GPTQ/RTN error ratio).
"""
from __future__ import annotations

import numpy as np
import scipy.linalg as sla

__all__ = [
    "hessian", "hessian_accumulate", "damp", "hinv_upper_factor", "hinv_upper_factor_ul",
    "grid_params", "quant_codes", "dequant", "gptq_quantize", "rtn_quantize",
    "pack_codes", "unpack_codes", "layer_loss_direct", "layer_loss_hessian",
    "obq_fixed_order_row", "least_squares_refit", "act_order_perm", "gptq_quantize_act_order",
    "dequant_gemv", "gptq_quantize_deferred", "grid_params_working_precision",
    "quant_codes_working_precision",
]

FP16_MIN_NORMAL = 2.0 ** -14


# ---------------------------------------------------------------------------
# Stage 1: Hessian  ([blog] section 3: H = 2 X^T X;  [wiki] "최소 구현":
# H = 2 X^T X with X laid out [n, d_in]; accumulated over calibration
# batches per layer: [wiki] "최소 구현", last paragraph)
# ---------------------------------------------------------------------------
def hessian_accumulate(H: np.ndarray, X: np.ndarray) -> np.ndarray:
    """H += 2 X^T X for one batch X [n, d_in] (any float dtype, widened to fp64
    exactly).  Returns H (full, symmetric, fp64)."""
    Xd = np.asarray(X, dtype=np.float64)
    H += 2.0 * (Xd.T @ Xd)
    return H


def hessian(batches) -> np.ndarray:
    """H = sum over batches of 2 X_b^T X_b (reading R1)."""
    H = None
    for X in batches:
        if H is None:
            H = np.zeros((X.shape[1], X.shape[1]), dtype=np.float64)
        hessian_accumulate(H, X)
    return H


# ---------------------------------------------------------------------------
# Stage 2: dampening and the upper Cholesky factor of the inverse
# ([wiki] "GPTQ의 세 가지 변경", row 3: add 1% of the mean diagonal, compute
# the Cholesky form of H^-1 once up front; [wiki] "알고리즘": H^-1 <-
# Cholesky(H^-1)^T; [wiki] "최소 구현": chol -> cholesky_inverse -> chol upper)
# ---------------------------------------------------------------------------
def damp(H: np.ndarray, percdamp: float = 0.01):
    """(H + lambda I, lambda) with lambda = percdamp * mean(diag H) (reading R2)."""
    lam = float(percdamp) * float(np.mean(np.diag(H)))
    Hd = np.array(H, dtype=np.float64, copy=True)
    Hd[np.diag_indices_from(Hd)] += lam
    return Hd, lam


def hinv_upper_factor(Hd: np.ndarray) -> np.ndarray:
    """U upper triangular with U^T U = Hd^-1, by the chain the pages give:
    L = chol(Hd); Hd^-1 = L^-T L^-1; U = chol(Hd^-1, upper)."""
    d = Hd.shape[0]
    L = np.linalg.cholesky(Hd)
    Linv = sla.solve_triangular(L, np.eye(d), lower=True)
    Hinv = Linv.T @ Linv
    Hinv = 0.5 * (Hinv + Hinv.T)
    return np.linalg.cholesky(Hinv).T.copy()


def hinv_upper_factor_ul(Hd: np.ndarray) -> np.ndarray:
    """The same U by a shorter route: with P the index reversal,
    L' = chol(P Hd P) and U = P L'^-1 P  (because Hd = U^-1 U^-T and P U^-1 P
    is lower triangular with a positive diagonal, so it is chol(P Hd P))."""
    d = Hd.shape[0]
    Lp = np.linalg.cholesky(Hd[::-1, ::-1])
    Lpinv = sla.solve_triangular(Lp, np.eye(d), lower=True)
    return Lpinv[::-1, ::-1].copy()


# ---------------------------------------------------------------------------
# The grid ([wiki] "최소 구현": one asymmetric min/max grid per row,
# q = clamp(round(w/scale) + zero, 0, maxq), deq = scale (q - zero);
# [wiki] "실무 변형": groups of g consecutive weights share scale/zero, set
# from the latest updated weights)
# ---------------------------------------------------------------------------
def grid_params(wmin, wmax, bits: int):
    """Scale and zero (fp16 values, returned as float32 arrays) per reading R5."""
    maxq = np.float32(2 ** bits - 1)
    wmin32 = np.asarray(wmin, dtype=np.float32)
    wmax32 = np.asarray(wmax, dtype=np.float32)
    rng = np.maximum(wmax32 - wmin32, np.float32(1e-8))
    s32 = (rng / maxq).astype(np.float32)
    s16 = s32.astype(np.float16)
    s16 = np.where(s16 == 0, np.float16(FP16_MIN_NORMAL), s16)
    s = s16.astype(np.float32)
    z32 = np.rint((-wmin32 / s).astype(np.float32))
    z = z32.astype(np.float16).astype(np.float32)
    return s, z


def grid_params_working_precision(wmin, wmax, bits: int):
    """Scale and zero as the page's minimal quantizer forms them ([wiki]
    "최소 구현"): scale = max(wmax - wmin, 1e-8) / maxq and zero =
    round(-wmin / scale), both kept in the working precision (fp64 here), with
    no fp16 storage.  This is reading B, used only to compare the oracle with a
    direct run of those steps; the codes the library stores use reading R5."""
    maxq = float(2 ** bits - 1)
    wmin = np.asarray(wmin, dtype=np.float64)
    wmax = np.asarray(wmax, dtype=np.float64)
    s = np.maximum(wmax - wmin, 1e-8) / maxq
    return s, np.rint(-wmin / s)


def quant_codes_working_precision(w, s, z, bits: int) -> np.ndarray:
    """c = clamp(round(w / s) + z, 0, maxq) in fp64 (reading B)."""
    maxq = float(2 ** bits - 1)
    t = np.rint(np.asarray(w, dtype=np.float64) / np.asarray(s, dtype=np.float64))
    return np.clip(t + np.asarray(z, dtype=np.float64), 0.0, maxq).astype(np.int64)


def quant_codes(w, s, z, bits: int) -> np.ndarray:
    """Integer codes c = clamp(rint(w/s) + z, 0, maxq), decided in fp32 (R4)."""
    maxq = np.float32(2 ** bits - 1)
    w32 = np.asarray(w, dtype=np.float32)
    t = np.rint((w32 / np.asarray(s, dtype=np.float32)).astype(np.float32))
    c = np.clip(t + np.asarray(z, dtype=np.float32), np.float32(0), maxq)
    return c.astype(np.int64)


def dequant(c, s, z) -> np.ndarray:
    """q = s (c - z) in fp64 (exact: s is an fp16 value, c - z an integer)."""
    return np.asarray(s, dtype=np.float64) * (np.asarray(c, dtype=np.float64) - np.asarray(z, dtype=np.float64))


def _row_minmax(A):
    A32 = np.asarray(A, dtype=np.float32)
    return A32.min(axis=1), A32.max(axis=1)


# ---------------------------------------------------------------------------
# Stage 3/4: the blocked column sweep ([wiki] "알고리즘", Algorithm 1;
# [wiki] "GPTQ의 세 가지 변경" rows 1-2: one column order for all rows, lazy
# batch of B columns followed by one matrix product for the rest)
# ---------------------------------------------------------------------------
def gptq_quantize(W, U, bits: int = 4, blocksize: int = 128, groupsize: int = -1,
                  return_trace: bool = False, grid: str = "fp16"):
    """Algorithm 1 step by step, vectorised over rows.

    grid = "fp16" (the default): reading R5, the grid the library stores.
    grid = "working": reading B, the page's minimal quantizer's own grid (one
    per row, scale and zero kept in fp64, decisions in fp64); per-row grids
    only.  It exists to compare the oracle with a direct run of those steps.

    W [d_out, d_in] (any float, widened to fp64), U upper [d_in, d_in] with
    U^T U = (H + lambda I)^-1.  Returns a dict with codes (int64 [d_out, d_in]),
    scales/zeros (float32 values of the fp16 grid, [d_out, n_groups]),
    Q (fp64 dequantized weights) and, if return_trace, the weight each column
    had when it was quantized (W_at), the error matrix E [d_out, d_in] and the
    fp32 min / max each grid was set from (gmin, gmax [d_out, n_groups])."""
    W = np.array(W, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    d_out, d_in = W.shape
    B = int(blocksize)
    n_groups = 1 if groupsize <= 0 else -(-d_in // groupsize)
    scales = np.zeros((d_out, n_groups), dtype=np.float32)
    zeros = np.zeros((d_out, n_groups), dtype=np.float32)
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    Q = np.zeros((d_out, d_in), dtype=np.float64)
    W_at = np.zeros((d_out, d_in), dtype=np.float64) if return_trace else None
    E_all = np.zeros((d_out, d_in), dtype=np.float64) if return_trace else None
    gmin = np.zeros((d_out, n_groups), dtype=np.float32)   # the fp32 min / max each grid was set from
    gmax = np.zeros((d_out, n_groups), dtype=np.float32)

    working = grid == "working"
    if working:
        if groupsize > 0:
            raise ValueError("the working-precision grid is one grid per row")
        scales = scales.astype(np.float64)
        zeros = zeros.astype(np.float64)
        s, z = grid_params_working_precision(W.min(axis=1), W.max(axis=1), bits)
        scales[:, 0], zeros[:, 0] = s, z
    elif grid != "fp16":
        raise ValueError(grid)
    elif groupsize <= 0:                                 # reading R6: original W
        gmin[:, 0], gmax[:, 0] = _row_minmax(W)
        s, z = grid_params(gmin[:, 0], gmax[:, 0], bits)
        scales[:, 0], zeros[:, 0] = s, z

    for i1 in range(0, d_in, B):
        i2 = min(i1 + B, d_in)
        W1 = W[:, i1:i2].copy()
        E = np.zeros((d_out, i2 - i1), dtype=np.float64)
        for j in range(i2 - i1):
            col = i1 + j
            if groupsize > 0 and col % groupsize == 0:    # R6: latest updated weights
                g_end = min(col + groupsize, d_in)
                cur = np.concatenate([W1[:, j:], W[:, i2:]], axis=1)[:, :g_end - col]
                gi = col // groupsize
                gmin[:, gi], gmax[:, gi] = _row_minmax(cur)
                s, z = grid_params(gmin[:, gi], gmax[:, gi], bits)
                scales[:, gi], zeros[:, gi] = s, z
            w = W1[:, j]
            c = quant_codes_working_precision(w, s, z, bits) if working else quant_codes(w, s, z, bits)
            q = dequant(c, s, z)
            codes[:, col] = c
            Q[:, col] = q
            if return_trace:
                W_at[:, col] = w
            err = (w - q) / U[col, col]
            W1[:, j:] -= np.outer(err, U[col, col:i2])
            E[:, j] = err
        W[:, i1:i2] = W1
        if i2 < d_in:
            W[:, i2:] -= E @ U[i1:i2, i2:]
        if return_trace:
            E_all[:, i1:i2] = E
    out = {"codes": codes, "scales": scales, "zeros": zeros, "Q": Q}
    if return_trace:
        out["W_at"] = W_at
        out["E"] = E_all
        out["gmin"], out["gmax"] = gmin, gmax
        out["bits"] = int(bits)
    return out


def gptq_quantize_deferred(W, U, bits: int = 4, blocksize: int = 128, groupsize: int = -1,
                           superblock: int = 4):
    """A cross-check, not the pages' order: the same sweep with the trailing
    update deferred.  After each block, E updates only the rest of its
    super-block (`superblock` blocks); the columns beyond the super-block get
    one product with the super-block's whole E.  The trailing update is
    linear, so in exact arithmetic every column holds the same values when it
    is quantized as in gptq_quantize.  A group grid is taken from the columns
    of its group, which must therefore not reach past the super-block: the
    group size has to divide superblock * blocksize (or the grid is per row).
    Returns codes, scales, zeros and Q as gptq_quantize does."""
    W = np.array(W, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    d_out, d_in = W.shape
    B = int(blocksize)
    SB = int(superblock) * B
    if groupsize > 0 and SB % groupsize != 0:
        raise ValueError("the group size must divide the super-block width")
    n_groups = 1 if groupsize <= 0 else -(-d_in // groupsize)
    scales = np.zeros((d_out, n_groups), dtype=np.float32)
    zeros = np.zeros((d_out, n_groups), dtype=np.float32)
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    Q = np.zeros((d_out, d_in), dtype=np.float64)
    if groupsize <= 0:
        s, z = grid_params(*_row_minmax(W), bits)
        scales[:, 0], zeros[:, 0] = s, z
    for s1 in range(0, d_in, SB):
        s2 = min(s1 + SB, d_in)
        E_sb = np.zeros((d_out, s2 - s1), dtype=np.float64)
        for i1 in range(s1, s2, B):
            i2 = min(i1 + B, s2)
            W1 = W[:, i1:i2].copy()
            for j in range(i2 - i1):
                col = i1 + j
                if groupsize > 0 and col % groupsize == 0:    # the group lies inside [col, s2)
                    g_end = min(col + groupsize, d_in)
                    cur = np.concatenate([W1[:, j:], W[:, i2:s2]], axis=1)[:, :g_end - col]
                    s, z = grid_params(*_row_minmax(cur), bits)
                    scales[:, col // groupsize], zeros[:, col // groupsize] = s, z
                w = W1[:, j]
                c = quant_codes(w, s, z, bits)
                q = dequant(c, s, z)
                codes[:, col] = c
                Q[:, col] = q
                err = (w - q) / U[col, col]
                W1[:, j:] -= np.outer(err, U[col, col:i2])
                E_sb[:, col - s1] = err
            W[:, i1:i2] = W1
            if i2 < s2:                                       # the rest of the super-block only
                W[:, i2:s2] -= E_sb[:, i1 - s1:i2 - s1] @ U[i1:i2, i2:s2]
        if s2 < d_in:                                         # the far tail, once per super-block
            W[:, s2:] -= E_sb @ U[s1:s2, s2:]
    return {"codes": codes, "scales": scales, "zeros": zeros, "Q": Q}


# ---------------------------------------------------------------------------
# Act-order ([wiki] "실무 변형": quantize the columns with the largest Hessian
# diagonal -- the largest input activations -- first, so that the large errors
# come early and the remaining columns can compensate for them)
# ---------------------------------------------------------------------------
def act_order_perm(H) -> np.ndarray:
    """The processing order: column indices by descending diag(H), ties by
    index (reading R14).  perm[k] is the original index of the k-th column
    processed."""
    return np.argsort(-np.diag(np.asarray(H, dtype=np.float64)), kind="stable")


def gptq_quantize_act_order(W, H, bits: int = 4, blocksize: int = 128, groupsize: int = -1,
                            percdamp: float = 0.01, perm=None, return_trace: bool = False):
    """GPTQ with the columns taken in act-order: the same Algorithm 1 on the
    permuted problem (W[:, perm], H[perm][:, perm], damped as usual -- lambda
    does not depend on the order).  Codes, scales and zeros stay in processing
    order (groups are formed in that order, reading R14); Q is returned in the
    original column order; `perm` is returned with them.  `perm` may be given
    (an order decided on another copy of the diagonal, e.g. an fp32 one whose
    near-ties round differently); by default it is act_order_perm(H)."""
    H = np.asarray(H, dtype=np.float64)
    perm = act_order_perm(H) if perm is None else np.asarray(perm, dtype=np.int64)
    assert np.array_equal(np.sort(perm), np.arange(H.shape[0])), "perm must be a permutation"
    Hp = H[np.ix_(perm, perm)]
    Hd, _ = damp(Hp, percdamp)
    U = hinv_upper_factor(Hd)
    out = gptq_quantize(np.asarray(W)[:, perm], U, bits, blocksize, groupsize, return_trace=return_trace)
    out["Q"] = out["Q"][:, np.argsort(perm)]
    out["perm"] = perm
    return out


def rtn_quantize(W, bits: int = 4, groupsize: int = -1):
    """Round-to-nearest on the same grid, no feedback ([wiki] "문제 설정":
    RTN moves each weight to the nearest grid point without looking at X).
    Group grids come from the original W."""
    W = np.asarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    g = d_in if groupsize <= 0 else groupsize
    n_groups = -(-d_in // g)
    scales = np.zeros((d_out, n_groups), dtype=np.float32)
    zeros = np.zeros((d_out, n_groups), dtype=np.float32)
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    Q = np.zeros((d_out, d_in), dtype=np.float64)
    for gi in range(n_groups):
        a, b = gi * g, min(d_in, (gi + 1) * g)
        s, z = grid_params(*_row_minmax(W[:, a:b]), bits)
        scales[:, gi], zeros[:, gi] = s, z
        c = quant_codes(W[:, a:b], s[:, None], z[:, None], bits)
        codes[:, a:b] = c
        Q[:, a:b] = dequant(c, s[:, None], z[:, None])
    return {"codes": codes, "scales": scales, "zeros": zeros, "Q": Q}


# ---------------------------------------------------------------------------
# Stage 5: packing (reading R7; the pages only say that production GPTQ stores
# INT4/INT8 codes and dequantizes at inference: [blog] section 5)
# ---------------------------------------------------------------------------
def pack_codes(codes, bits: int) -> np.ndarray:
    """[d_out, d_in] codes -> [d_out, d_in * bits / 32] uint32 words.  The codes
    of a row form a little-endian bit stream: code k occupies bits
    [k*bits, (k+1)*bits) of the stream, word w holds stream bits [32w, 32w+32)."""
    codes = np.asarray(codes, dtype=np.int64)
    d_out, d_in = codes.shape
    assert (d_in * bits) % 32 == 0
    n_words = d_in * bits // 32
    out = np.zeros((d_out, n_words), dtype=np.uint64)
    for k in range(d_in):
        for b in range(bits):
            bit = (codes[:, k] >> b) & 1
            pos = k * bits + b
            out[:, pos // 32] |= (bit.astype(np.uint64) << np.uint64(pos % 32))
    return out.astype(np.uint32)


def unpack_codes(words, bits: int, d_in: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint32).astype(np.uint64)
    d_out = words.shape[0]
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    for k in range(d_in):
        for b in range(bits):
            pos = k * bits + b
            bit = (words[:, pos // 32] >> np.uint64(pos % 32)) & np.uint64(1)
            codes[:, k] |= (bit.astype(np.int64) << b)
    return codes


# ---------------------------------------------------------------------------
# Inference consumer (reading R15): the layer's output computed from the
# stored form.  [wiki] "결과": a dedicated kernel unpacks the weights as it
# needs them and cuts the per-token latency; [blog] section 5: production
# implementations store INT4/INT8 codes and dequantize them during inference.
# ---------------------------------------------------------------------------
def dequant_gemv(words, scales, zeros, bits: int, groupsize: int, x, perm=None) -> np.ndarray:
    """y[m][r] = sum_k s[r][g(k)] (c[r][k] - z[r][g(k)]) x[m][perm[k]] in fp64.

    words [d_out, d_in*bits/32] packed codes (R7), scales / zeros [d_out,
    n_groups] fp16 values, x [m, d_in] (the layer input, one row per token).
    Code column k belongs to input column perm[k] (act-order, R14); perm=None
    is the natural order.  g(k) = k // groupsize (0 for a per-row grid)."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    d_in = x.shape[1]
    c = unpack_codes(words, bits, d_in)
    g = d_in if groupsize <= 0 else groupsize
    gi = np.arange(d_in) // g
    s = np.asarray(scales, dtype=np.float64)[:, gi]
    z = np.asarray(zeros, dtype=np.float64)[:, gi]
    Q = dequant(c, s, z)                    # [d_out, d_in], processing order
    xp = x if perm is None else x[:, np.asarray(perm, dtype=np.int64)]
    return xp @ Q.T


# ---------------------------------------------------------------------------
# The objective ([wiki] "문제 설정": argmin over the grid of ||W X - W^ X||^2)
# ---------------------------------------------------------------------------
def layer_loss_direct(W, Q, batches) -> float:
    """||(W - Q) X^T||_F^2 summed over the calibration batches (X rows are
    samples, so the layer output is X W^T)."""
    D = np.asarray(W, dtype=np.float64) - np.asarray(Q, dtype=np.float64)
    tot = 0.0
    for X in batches:
        Y = np.asarray(X, dtype=np.float64) @ D.T
        tot += float(np.sum(Y * Y))
    return tot


def layer_loss_hessian(W, Q, H0) -> float:
    """The same loss from the undamped H0 = 2 X^T X: 1/2 tr(D H0 D^T)."""
    D = np.asarray(W, dtype=np.float64) - np.asarray(Q, dtype=np.float64)
    return 0.5 * float(np.sum((D @ H0) * D))


# ---------------------------------------------------------------------------
# Independent formulations used as pins
# ---------------------------------------------------------------------------
def obq_fixed_order_row(w, Hd, s, z, bits: int):
    """OBQ on one row with the column order fixed to 0..d-1 ([wiki] "OBQ에서
    GPTQ로": w_q's error divided by [H_F^-1]_qq times the q-th column of
    H_F^-1 is the optimal compensation of the remaining weights; after w_q is
    fixed, H_F^-1 loses row/column q by one step of Gaussian elimination).
    Uses only the full inverse and the elimination step -- no Cholesky."""
    w = np.array(w, dtype=np.float64, copy=True)
    d = w.shape[0]
    Hinv = np.linalg.inv(np.asarray(Hd, dtype=np.float64))
    F = list(range(d))
    codes = np.zeros(d, dtype=np.int64)
    W_at = np.zeros(d)
    for q in range(d):
        pos = F.index(q)
        W_at[q] = w[q]
        c = int(quant_codes(np.array([w[q]]), np.array([s]), np.array([z]), bits)[0])
        codes[q] = c
        qv = float(dequant(c, s, z))
        hqq = Hinv[pos, pos]
        delta = -(w[q] - qv) / hqq * Hinv[:, pos]
        for a, col in enumerate(F):
            w[col] += delta[a]
        # Gaussian elimination of row/column `pos`
        Hinv = Hinv - np.outer(Hinv[:, pos], Hinv[pos, :]) / hqq
        keep = [a for a in range(len(F)) if a != pos]
        Hinv = Hinv[np.ix_(keep, keep)]
        F.pop(pos)
    return codes, W_at


def least_squares_refit(W0, Q_prefix, Hd, k: int):
    """Optimal continuous values of columns k.. given columns 0..k-1 fixed to
    Q_prefix (minimising tr(D Hd D^T)): W_F + Hd_FF^-1 Hd_FQ (W_Q - Q_Q)."""
    W0 = np.asarray(W0, dtype=np.float64)
    Hd = np.asarray(Hd, dtype=np.float64)
    dq = W0[:, :k] - np.asarray(Q_prefix, dtype=np.float64)
    rhs = Hd[k:, :k] @ dq.T
    return W0[:, k:] + np.linalg.solve(Hd[k:, k:], rhs).T
