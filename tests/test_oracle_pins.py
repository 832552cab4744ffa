"""Pins for the fp64 oracle: each checks it against something other than
itself -- hand-derived values, closed forms, brute force, an independent
formulation (OBQ's Gaussian-elimination form), invariants, and the error ratio
the itwiki "GPTQ" article publishes for its correlated 512-dim example.

The last section plants plausible mistakes in the oracle (on the CPU) and
checks that at least one pin catches each of them.
"""
import itertools
import os

import numpy as np
import pytest

import oracle
from post_weight_quantization_05_b200 import synth


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def _small_problem(d_out=24, d_in=16, n=96, rho=0.8, seed=3, std=0.02):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((d_out, d_in)) * std).astype(np.float32)
    X = synth.ar1_rows(rng, n, d_in, rho)
    return W, X


def _factor(X, percdamp=0.01):
    H = oracle.hessian([X])
    Hd, lam = oracle.damp(H, percdamp)
    return H, Hd, lam, oracle.hinv_upper_factor(Hd)


def _read_kv(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split()
        out[k] = float(v)
    return out


# ---------------------------------------------------------------------------
# Stage 1: H
# ---------------------------------------------------------------------------
def test_hessian_matches_brute_force_sums():
    rng = np.random.default_rng(0)
    Xa = rng.standard_normal((7, 5)).astype(np.float32)
    Xb = rng.standard_normal((4, 5)).astype(np.float32)
    H = oracle.hessian([Xa, Xb])
    for a in range(5):
        for b in range(5):
            tot = 0.0
            for X in (Xa, Xb):
                for r in range(X.shape[0]):
                    tot += 2.0 * float(X[r, a]) * float(X[r, b])
            assert abs(H[a, b] - tot) <= 1e-12 * max(1.0, abs(tot))


def test_damping_is_one_percent_of_mean_diagonal():
    H = np.diag([1.0, 2.0, 3.0, 6.0]) + 0.1
    Hd, lam = oracle.damp(H, 0.01)
    assert lam == pytest.approx(0.01 * (1.1 + 2.1 + 3.1 + 6.1) / 4, rel=1e-15)
    assert np.array_equal(Hd - np.diag(np.diag(Hd)), H - np.diag(np.diag(H)))
    assert np.allclose(np.diag(Hd) - np.diag(H), lam, rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------
# Stage 2: U
# ---------------------------------------------------------------------------
def test_upper_factor_inverts_damped_hessian():
    W, X = _small_problem(d_in=40, n=200)
    H, Hd, lam, U = _factor(X)
    assert np.allclose(np.tril(U, -1), 0.0)
    assert np.all(np.diag(U) > 0)
    I = U.T @ U @ Hd
    assert np.max(np.abs(I - np.eye(40))) < 1e-12


def test_ul_route_equals_literal_chain():
    W, X = _small_problem(d_in=64, n=300)
    H, Hd, lam, U = _factor(X)
    U2 = oracle.hinv_upper_factor_ul(Hd)
    assert np.linalg.norm(U - U2) / np.linalg.norm(U) < 1e-12


def test_diagonal_hessian_gives_diagonal_factor():
    h = np.array([1.0, 4.0, 9.0, 0.5, 2.0])
    Hd, lam = oracle.damp(np.diag(h), 0.01)
    U = oracle.hinv_upper_factor(Hd)
    assert np.allclose(U, np.diag(1.0 / np.sqrt(h + lam)), rtol=1e-14, atol=1e-15)


def test_two_column_closed_form(golden_dir):
    g = _read_kv(os.path.join(golden_dir, "two_column.txt"))
    Hd = np.array([[g["a"], g["b"]], [g["b"], g["c"]]])
    U = oracle.hinv_upper_factor(Hd)
    assert U[0, 0] == pytest.approx(g["U00"], rel=1e-14)
    assert U[0, 1] == pytest.approx(g["U01"], rel=1e-14)
    assert U[1, 1] == pytest.approx(g["U11"], rel=1e-14)
    W = np.array([[g["w0"], g["w1"]]], dtype=np.float32)
    out = oracle.gptq_quantize(W, U, bits=4, blocksize=128, return_trace=True)
    assert out["scales"][0, 0] == g["scale"] and out["zeros"][0, 0] == g["zero"]
    assert list(out["codes"][0]) == [int(g["code0"]), int(g["code1"])]
    assert out["Q"][0, 0] == pytest.approx(g["q0"], abs=1e-15)
    assert out["Q"][0, 1] == pytest.approx(g["q1"], abs=1e-15)
    assert out["W_at"][0, 1] == pytest.approx(g["w1_at"], abs=1e-14)


# ---------------------------------------------------------------------------
# Grid and packing
# ---------------------------------------------------------------------------
def test_grid_hand_values(golden_dir):
    for line in open(os.path.join(golden_dir, "grid_hand.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        bits, wmin, wmax, es, ez = line.split()
        s, z = oracle.grid_params(np.float32(wmin), np.float32(wmax), int(bits))
        assert float(s) == float(es), line
        assert float(z) == float(ez), line


def _parse_codes(spec, bits):
    codes = np.zeros(32, dtype=np.int64)
    if spec == "seq16":
        codes[:] = np.arange(32) % 16
    elif spec.startswith("all:"):
        codes[:] = int(spec[4:])
    else:
        for item in spec.split(","):
            k, v = item.split(":")
            codes[int(k)] = int(v)
    return codes


def test_pack_hand_values(golden_dir):
    for line in open(os.path.join(golden_dir, "pack_hand.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        bits, spec, words = [t.strip() for t in line.split("|")]
        bits = int(bits)
        codes = _parse_codes(spec, bits)
        expect = [int(w, 16) for w in words.split()]
        got = oracle.pack_codes(codes[None, :], bits)[0]
        assert [int(x) for x in got] == expect, line
        assert np.array_equal(oracle.unpack_codes(got[None, :], bits, 32)[0], codes)


def test_grid_membership_and_rtn_is_nearest_point():
    """T7 + brute force: RTN picks, for every weight, a grid point at least as
    close as every other grid point, and Q = s (c - z) with c in [0, maxq]."""
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    for bits, g in ((4, -1), (3, -1), (4, 128), (2, 64), (8, -1)):
        out = oracle.rtn_quantize(W, bits, g)
        maxq = 2 ** bits - 1
        c = out["codes"]
        assert c.min() >= 0 and c.max() <= maxq
        gs = 256 if g <= 0 else g
        s = np.repeat(out["scales"], gs, axis=1)[:, :256].astype(np.float64)
        z = np.repeat(out["zeros"], gs, axis=1)[:, :256].astype(np.float64)
        assert np.array_equal(out["Q"], s * (c - z))
        allq = s[..., None] * (np.arange(maxq + 1)[None, None, :] - z[..., None])
        dist = np.abs(allq - W.astype(np.float64)[..., None])
        best = dist.min(axis=-1)
        mine = np.abs(out["Q"] - W)
        assert np.all(mine <= best + 1e-7 * s)  # fp32 decision, fp64 distance


# ---------------------------------------------------------------------------
# The sweep
# ---------------------------------------------------------------------------
def test_obq_elimination_form_equals_sweep():
    """T4: OBQ with a fixed column order (full inverse + one Gaussian
    elimination per step, no Cholesky) quantizes every row exactly like the
    Cholesky-row sweep."""
    for d in (3, 5, 8):
        W, X = _small_problem(d_out=6, d_in=d, n=40, seed=d)
        H, Hd, lam, U = _factor(X)
        out = oracle.gptq_quantize(W, U, bits=3, blocksize=128, return_trace=True)
        for r in range(W.shape[0]):
            s, z = out["scales"][r, 0], out["zeros"][r, 0]
            codes, w_at = oracle.obq_fixed_order_row(W[r], Hd, s, z, 3)
            assert np.array_equal(codes, out["codes"][r])
            assert np.max(np.abs(w_at - out["W_at"][r])) < 1e-12


def test_deferred_trailing_update_is_exact():
    """The deferred trailing update (each block's E applied to the rest of its
    super-block, the far tail once per super-block with the super-block's
    whole E) gives the per-block sweep's codes and grids, and Q to 1e-10: the
    update is linear.  One super-block spanning the whole layer (no far
    update at all) and one block per super-block (every update a far one)
    are both covered.  A group that would reach past its super-block is
    refused."""
    W, X = _small_problem(d_out=20, d_in=96, n=400, seed=21)
    H, Hd, lam, U = _factor(X)
    checked = 0
    for g in (-1, 16, 32):
        ref = oracle.gptq_quantize(W, U, 4, 8, groupsize=g)
        for K in (1, 2, 4, 12):                              # super-blocks of 8, 16, 32, 96 columns
            if g > 0 and (8 * K) % g:
                with pytest.raises(ValueError):
                    oracle.gptq_quantize_deferred(W, U, 4, 8, groupsize=g, superblock=K)
                continue
            out = oracle.gptq_quantize_deferred(W, U, 4, 8, groupsize=g, superblock=K)
            assert np.array_equal(out["codes"], ref["codes"]), (g, K)
            assert np.array_equal(out["scales"], ref["scales"]) and np.array_equal(out["zeros"], ref["zeros"])
            assert np.max(np.abs(out["Q"] - ref["Q"])) < 1e-10
            checked += 1
    assert checked == 4 + 3 + 2


def test_lazy_batch_is_exact():
    """T3: B = 1 (unblocked), B = 4 and B = 128 give the same result."""
    W, X = _small_problem(d_out=20, d_in=48, n=200, seed=9)
    H, Hd, lam, U = _factor(X)
    ref = oracle.gptq_quantize(W, U, 4, 1, return_trace=True)
    for B in (4, 16, 128):
        out = oracle.gptq_quantize(W, U, 4, B, return_trace=True)
        assert np.array_equal(out["codes"], ref["codes"])
        assert np.max(np.abs(out["W_at"] - ref["W_at"])) < 1e-10
        assert np.max(np.abs(out["Q"] - ref["Q"])) < 1e-10
    refg = oracle.gptq_quantize(W, U, 4, 1, groupsize=16, return_trace=True)
    outg = oracle.gptq_quantize(W, U, 4, 16, groupsize=16, return_trace=True)
    assert np.array_equal(outg["codes"], refg["codes"])
    assert np.array_equal(outg["scales"], refg["scales"])


def test_least_squares_refit_invariant():
    """Every column, when quantized, holds the optimal continuous value given
    the already-quantized prefix (the sequence of OBS steps reaches the exact
    constrained optimum of the quadratic objective)."""
    W, X = _small_problem(d_out=10, d_in=40, n=160, seed=11)
    H, Hd, lam, U = _factor(X)
    for B, g in ((8, -1), (128, -1), (8, 16)):
        out = oracle.gptq_quantize(W, U, 4, B, groupsize=g, return_trace=True)
        for k in range(1, 40):
            ref = oracle.least_squares_refit(W, out["Q"][:, :k], Hd, k)
            assert np.max(np.abs(ref[:, 0] - out["W_at"][:, k])) < 1e-12


def test_group_grid_uses_latest_weights():
    """Group g's scale/zero come from the group's columns as they stand when
    the sweep reaches the group, i.e. the least-squares refit given the
    quantized prefix."""
    W, X = _small_problem(d_out=32, d_in=48, n=200, seed=13)
    H, Hd, lam, U = _factor(X)
    out = oracle.gptq_quantize(W, U, 4, 16, groupsize=16)
    for gi in range(3):
        k = 16 * gi
        cur = W[:, :16] if k == 0 else oracle.least_squares_refit(W, out["Q"][:, :k], Hd, k)[:, :16]
        s, z = oracle.grid_params(cur.astype(np.float32).min(1), cur.astype(np.float32).max(1), 4)
        assert np.mean(s == out["scales"][:, gi]) >= 0.95
        assert np.allclose(s, out["scales"][:, gi], rtol=2e-3)
    # and it is not the grid of the original weights after the first group
    s0, _ = oracle.grid_params(W[:, 16:32].min(1), W[:, 16:32].max(1), 4)
    assert not np.array_equal(s0, out["scales"][:, 1])


def test_each_code_is_nearest_given_sweep_state():
    """T5 by brute force: given the weight a column had when quantized, no
    other grid point has a smaller (quant(w) - w)^2 / [H_F^-1]_qq."""
    W, X = _small_problem(d_out=16, d_in=32, n=120, seed=17)
    H, Hd, lam, U = _factor(X)
    out = oracle.gptq_quantize(W, U, 3, 8, return_trace=True)
    s = out["scales"][:, :1].astype(np.float64)
    z = out["zeros"][:, :1].astype(np.float64)
    for q in range(32):
        w = out["W_at"][:, q:q + 1]
        cand = s * (np.arange(8)[None, :] - z)
        hqq = U[q, q] ** 2          # [H_F^-1]_qq for F = {q, ..., d-1}
        obj = (cand - w) ** 2 / hqq
        mine = (out["Q"][:, q:q + 1] - w) ** 2 / hqq
        assert np.all(mine[:, 0] <= obj.min(axis=1) + 1e-9 * s[:, 0] ** 2 / hqq)


def test_diagonal_hessian_reduces_to_rtn():
    """Uncorrelated inputs with orthogonal columns: no compensation, GPTQ == RTN."""
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((12, 24)) * 0.02).astype(np.float32)
    Hd, lam = oracle.damp(np.diag(rng.uniform(0.5, 2.0, 24)), 0.01)
    U = oracle.hinv_upper_factor(Hd)
    g = oracle.gptq_quantize(W, U, 4, 8)
    r = oracle.rtn_quantize(W, 4)
    assert np.array_equal(g["codes"], r["codes"])
    assert np.array_equal(g["Q"], r["Q"])


def test_input_scale_invariance():
    """Scaling X by a power of two scales H and lambda alike: identical codes."""
    W, X = _small_problem(d_out=16, d_in=32, n=100, seed=19)
    a = oracle.gptq_quantize(W, _factor(X)[3], 4, 8)
    b = oracle.gptq_quantize(W, _factor(X * np.float32(4.0))[3], 4, 8)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.max(np.abs(a["Q"] - b["Q"])) == 0.0


def test_loss_identity():
    W, X = _small_problem(d_out=8, d_in=32, n=150, seed=23)
    H, Hd, lam, U = _factor(X)
    out = oracle.gptq_quantize(W, U, 4, 16)
    a = oracle.layer_loss_direct(W, out["Q"], [X])
    b = oracle.layer_loss_hessian(W, out["Q"], H)
    assert abs(a - b) <= 1e-10 * a


def test_published_ratio_gptq_below_half_of_rtn():
    """The itwiki "GPTQ" article ("최소 구현"): on correlated random inputs
    (512-dim, 2048 samples), 4-bit per-row GPTQ's output squared error is less
    than half of RTN's on the same grid."""
    p = synth.smoke()
    X = p.x_batch(0)
    H, Hd, lam, U = _factor(X)
    g = oracle.gptq_quantize(p.W, U, 4, 128)
    r = oracle.rtn_quantize(p.W, 4)
    lg = oracle.layer_loss_hessian(p.W, g["Q"], H)
    lr = oracle.layer_loss_hessian(p.W, r["Q"], H)
    assert lg < 0.5 * lr, (lg, lr)
    # the per-row grid is the same for both
    assert np.array_equal(g["scales"], r["scales"]) and np.array_equal(g["zeros"], r["zeros"])


def test_brute_force_optimum_is_not_beaten_on_tiny_case():
    """Sanity of the objective: the exact grid optimum (enumerated) is never
    worse than GPTQ, and GPTQ is never worse than RTN here (tiny, 2-bit)."""
    W, X = _small_problem(d_out=3, d_in=5, n=30, seed=29)
    H, Hd, lam, U = _factor(X)
    g = oracle.gptq_quantize(W, U, 2, 128)
    r = oracle.rtn_quantize(W, 2)
    for row in range(3):
        s, z = g["scales"][row, 0], g["zeros"][row, 0]
        best = np.inf
        for cs in itertools.product(range(4), repeat=5):
            q = s * (np.array(cs) - z)
            d = W[row].astype(np.float64) - q
            best = min(best, d @ H @ d)
        dg = W[row].astype(np.float64) - g["Q"][row]
        dr = W[row].astype(np.float64) - r["Q"][row]
        assert best <= dg @ H @ dg + 1e-15
        assert dg @ H @ dg <= dr @ H @ dr * 1.0000001


def test_ar1_generator_covariance():
    """The input recipe: x_a = rho x_{a-1} + sqrt(1-rho^2) z_a has covariance
    rho^|a-b| (the same law as Z C^T with C = chol(Sigma))."""
    x = synth.ar1_rows(np.random.default_rng(0), 200000, 6, 0.9).astype(np.float64)
    C = x.T @ x / x.shape[0]
    idx = np.arange(6)
    Sigma = 0.9 ** np.abs(idx[:, None] - idx[None, :])
    assert np.max(np.abs(C - Sigma)) < 0.02


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5], dtype=np.float32)
    got = synth.round_to_bf16(vals)
    assert list(got) == [1.0, 1.0, 1.0 + 4 * 2 ** -8, 1.0, -2.5]


# ---------------------------------------------------------------------------
# Planted mistakes: each must be caught by one of the pins above.
# ---------------------------------------------------------------------------
def _refit_error(W, Hd, out):
    err = 0.0
    for k in range(1, W.shape[1]):
        ref = oracle.least_squares_refit(W, out["Q"][:, :k], Hd, k)
        err = max(err, float(np.max(np.abs(ref[:, 0] - out["W_at"][:, k]))))
    return err


@pytest.mark.parametrize("mistake", ["no_trailing", "transposed_factor", "sign", "lower_factor"])
def test_planted_update_mistakes_are_caught(mistake):
    W, X = _small_problem(d_out=8, d_in=32, n=120, seed=31)
    H, Hd, lam, U = _factor(X)
    B = 8
    if mistake == "no_trailing":          # drop the lazy batch update
        Ub = np.triu(U).copy()
        for i in range(0, 32, B):
            Ub[i:i + B, i + B:] = 0.0
    elif mistake == "transposed_factor":
        Ub = U.T.copy()
    elif mistake == "sign":
        Ub = U.copy()
        Ub[np.triu_indices(32, 1)] *= -1.0
    else:                                   # Cholesky of H instead of H^-1
        Ub = np.linalg.cholesky(Hd).T
    bad = oracle.gptq_quantize(W, np.triu(Ub) if mistake != "transposed_factor" else Ub, 4, B,
                               return_trace=True)
    assert _refit_error(W, Hd, bad) > 1e-6


def test_planted_grid_mistakes_are_caught(golden_dir, monkeypatch):
    good = oracle.grid_params

    def maxq_plus_one(wmin, wmax, bits):
        s, z = good(wmin, wmax, bits)
        return (s * np.float32((2 ** bits - 1) / 2 ** bits)).astype(np.float32), z

    monkeypatch.setattr(oracle.gptq, "grid_params", maxq_plus_one)
    monkeypatch.setattr(oracle, "grid_params", maxq_plus_one)
    with pytest.raises(AssertionError):
        test_grid_hand_values(golden_dir)


def test_planted_rounding_mistake_is_caught(monkeypatch):
    def floor_codes(w, s, z, bits):
        maxq = 2 ** bits - 1
        t = np.floor(np.asarray(w, np.float32) / np.asarray(s, np.float32))
        return np.clip(t + z, 0, maxq).astype(np.int64)

    monkeypatch.setattr(oracle.gptq, "quant_codes", floor_codes)
    with pytest.raises(AssertionError):
        test_grid_membership_and_rtn_is_nearest_point()


def test_planted_damping_mistake_is_caught(monkeypatch):
    def damp_max(H, percdamp=0.01):
        lam = percdamp * float(np.max(np.diag(H)))
        Hd = np.array(H, dtype=np.float64, copy=True)
        Hd[np.diag_indices_from(Hd)] += lam
        return Hd, lam

    monkeypatch.setattr(oracle, "damp", damp_max)
    with pytest.raises(AssertionError):
        test_damping_is_one_percent_of_mean_diagonal()


# ---------------------------------------------------------------- act-order
def _golden_act_order(golden_dir):
    vals = {}
    for line in open(os.path.join(golden_dir, "act_order_perm.txt")):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            vals[k] = v
    return np.array(vals["diag"], dtype=np.float64), np.array(vals["perm"], dtype=np.int64)


def test_act_order_perm_hand_example(golden_dir):
    _check_golden_with(oracle.act_order_perm, golden_dir)


def test_act_order_is_plain_gptq_when_diag_already_sorted():
    rng = np.random.default_rng(21)
    d, n = 192, 1024
    X = rng.standard_normal((n, d))
    X *= (np.linspace(3.0, 0.5, d) / np.linalg.norm(X, axis=0))[None, :]   # channel norms exactly decreasing
    H = oracle.hessian([X])
    assert np.all(np.diff(np.diag(H)) < 0)
    W = rng.normal(0, 0.02, (64, d))
    for g in (-1, 64):
        a = oracle.gptq_quantize_act_order(W, H, 4, 64, g)
        Hd, _ = oracle.damp(H)
        b = oracle.gptq_quantize(W, oracle.hinv_upper_factor(Hd), 4, 64, g)
        assert np.array_equal(a["perm"], np.arange(d))
        assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["Q"], b["Q"])


def test_act_order_q_in_original_order():
    """Q comes back in the original column order: the loss of (W, Q) under H
    equals the loss of the permuted problem under the permuted H, and Q's
    permuted columns are exactly the dequantized codes (processing order)."""
    rng = np.random.default_rng(22)
    d, n = 256, 1024
    X = rng.standard_normal((n, d)) * np.exp(rng.normal(0, 1.0, d))[None, :]
    H = oracle.hessian([X])
    W = rng.normal(0, 0.02, (48, d))
    out = oracle.gptq_quantize_act_order(W, H, 4, 128, 128)
    p = out["perm"]
    assert not np.array_equal(p, np.arange(d))
    Qp = oracle.dequant(out["codes"], np.repeat(out["scales"], 128, axis=1), np.repeat(out["zeros"], 128, axis=1))
    assert np.array_equal(out["Q"][:, p], Qp)
    l_orig = oracle.layer_loss_hessian(W, out["Q"], H)
    l_perm = oracle.layer_loss_hessian(W[:, p], Qp, H[np.ix_(p, p)])
    assert abs(l_orig - l_perm) <= 1e-10 * l_perm


def test_act_order_given_order():
    """An explicit order equal to the default gives the same result; the
    identity order is plain GPTQ on the unpermuted problem; a non-permutation
    is refused."""
    rng = np.random.default_rng(24)
    d, n = 256, 1024
    X = rng.standard_normal((n, d)) * np.exp(rng.normal(0, 1.0, d))[None, :]
    H = oracle.hessian([X])
    W = rng.normal(0, 0.02, (16, d))
    a = oracle.gptq_quantize_act_order(W, H, 4, 128, -1)
    b = oracle.gptq_quantize_act_order(W, H, 4, 128, -1, perm=oracle.act_order_perm(H))
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["Q"], b["Q"])
    ident = oracle.gptq_quantize_act_order(W, H, 4, 128, -1, perm=np.arange(d))
    Hd, _ = oracle.damp(H, 0.01)
    plain = oracle.gptq_quantize(W, oracle.hinv_upper_factor(Hd), 4, 128, -1)
    assert np.array_equal(ident["codes"], plain["codes"]) and np.array_equal(ident["Q"], plain["Q"])
    with pytest.raises(AssertionError):
        oracle.gptq_quantize_act_order(W, H, 4, 128, -1, perm=np.zeros(d, dtype=np.int64))


def _golden_gemv(golden_dir):
    g = {}
    for line in open(os.path.join(golden_dir, "dequant_gemv_hand.txt")):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            g[k] = v
    words = np.array([[int(g["word0"][0], 16)], [int(g["word1"][0], 16)]], dtype=np.uint32)
    s = np.array([[float(v) for v in g["s0"]], [float(v) for v in g["s1"]]])
    z = np.array([[float(v) for v in g["z0"]], [float(v) for v in g["z1"]]])
    x = np.array([[float(v) for v in g["x"]]])
    perm = np.array([int(v) for v in g["perm"]])
    return words, s, z, x, perm, [float(v) for v in g["y"]], [float(v) for v in g["y_perm"]]


def test_dequant_gemv_hand_example(golden_dir):
    words, s, z, x, perm, y, y_perm = _golden_gemv(golden_dir)
    assert oracle.dequant_gemv(words, s, z, 4, 4, x)[0].tolist() == y
    assert oracle.dequant_gemv(words, s, z, 4, 4, x, perm)[0].tolist() == y_perm


@pytest.mark.parametrize("act", [False, True])
def test_dequant_gemv_equals_layer_output_of_q(act):
    """The stored form (packed codes, fp16 grid, permutation) reproduces the
    layer output of the quantizer's own Q, for several tokens at once."""
    rng = np.random.default_rng(31)
    d, n = 256, 1024
    X = rng.standard_normal((n, d)) * np.exp(rng.normal(0, 1.0, d))[None, :]
    H = oracle.hessian([X])
    W = rng.normal(0, 0.02, (40, d))
    if act:
        out = oracle.gptq_quantize_act_order(W, H, 4, 128, 128)
        perm = out["perm"]
    else:
        Hd, _ = oracle.damp(H, 0.01)
        out = oracle.gptq_quantize(W, oracle.hinv_upper_factor(Hd), 4, 128, 128)
        perm = None
    words = oracle.pack_codes(out["codes"], 4)
    xt = rng.standard_normal((5, d))
    y = oracle.dequant_gemv(words, out["scales"], out["zeros"], 4, 128, xt, perm)
    ref = xt @ out["Q"].T
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_act_order_with_diagonal_h_is_rtn():
    """Uncorrelated inputs (diagonal H): no compensation crosses columns, so
    act-order GPTQ is RTN on the per-row grid in any order."""
    rng = np.random.default_rng(23)
    d = 128
    H = np.diag(rng.uniform(0.5, 5.0, d))
    W = rng.normal(0, 0.02, (40, d))
    out = oracle.gptq_quantize_act_order(W, H, 4, 32, -1)
    rtn = oracle.rtn_quantize(W, 4, -1)
    codes = np.empty_like(out["codes"])
    codes[:, out["perm"]] = out["codes"]
    assert np.array_equal(codes, rtn["codes"])
    assert np.array_equal(out["Q"], rtn["Q"])


def test_act_order_lowers_error_on_uneven_channels():
    """[wiki] "실무 변형": taking the large-diagonal (large-activation) columns
    first leaves the rest to compensate.  On inputs whose channel scales span
    a wide range (log-normal, sigma 1) the layer error drops markedly."""
    rng = np.random.default_rng(5)
    d, n = 256, 2048
    z = rng.standard_normal((n, d))
    X = np.empty_like(z)
    X[:, 0] = z[:, 0]
    for a in range(1, d):
        X[:, a] = 0.8 * X[:, a - 1] + np.sqrt(1 - 0.64) * z[:, a]
    X *= np.exp(rng.normal(0, 1.0, d))[None, :]
    W = rng.normal(0, 0.02, (128, d))
    H = oracle.hessian([X])
    Hd, _ = oracle.damp(H)
    U = oracle.hinv_upper_factor(Hd)
    for g in (-1, 128):
        nat = oracle.layer_loss_hessian(W, oracle.gptq_quantize(W, U, 4, 128, g)["Q"], H)
        act = oracle.layer_loss_hessian(W, oracle.gptq_quantize_act_order(W, H, 4, 128, g)["Q"], H)
        assert act < 0.8 * nat


@pytest.mark.parametrize("mistake", ["ascending", "no_unpermute"])
def test_planted_act_order_mistakes_are_caught(mistake, monkeypatch, golden_dir):
    """Each plausible slip in the act-order restatement fails a pin above."""
    if mistake == "ascending":
        ascending = lambda H: np.argsort(np.diag(np.asarray(H, dtype=np.float64)), kind="stable")  # noqa: E731
        with pytest.raises(AssertionError):
            _check_golden_with(ascending, golden_dir)
    else:
        orig = oracle.gptq.gptq_quantize_act_order

        def no_unpermute(W, H, bits=4, blocksize=128, groupsize=-1, percdamp=0.01):
            out = orig(W, H, bits, blocksize, groupsize, percdamp)
            out["Q"] = out["Q"][:, out["perm"]]          # left in processing order
            return out
        monkeypatch.setattr(oracle.gptq, "gptq_quantize_act_order", no_unpermute)
        monkeypatch.setattr(oracle, "gptq_quantize_act_order", no_unpermute)
        with pytest.raises(AssertionError):
            test_act_order_q_in_original_order()


def _check_golden_with(perm_fn, golden_dir):
    diag, perm = _golden_act_order(golden_dir)
    assert np.array_equal(perm_fn(np.diag(diag)), perm)


def _mutant_gemv(mistake):
    def f(words, scales, zeros, bits, groupsize, x, perm=None):
        x = np.atleast_2d(np.asarray(x, dtype=np.float64))
        d_in = x.shape[1]
        c = oracle.unpack_codes(words, bits, d_in)
        g = d_in if groupsize <= 0 else groupsize
        ng = np.asarray(scales).shape[1]
        gi = np.arange(d_in) % ng if mistake == "group_index" else np.arange(d_in) // g
        s = np.asarray(scales, dtype=np.float64)[:, gi]
        z = np.asarray(zeros, dtype=np.float64)[:, gi]
        Q = s * (c + z) if mistake == "zero_sign" else s * (c - z)
        if perm is not None:
            p = np.argsort(perm) if mistake == "inverse_perm" else np.asarray(perm)
            x = x[:, p]
        return x @ Q.T
    return f


@pytest.mark.parametrize("mistake", ["inverse_perm", "zero_sign", "group_index"])
def test_planted_gemv_mistakes_are_caught(mistake, monkeypatch, golden_dir):
    """Each plausible slip in the stored-form product fails a pin above."""
    monkeypatch.setattr(oracle, "dequant_gemv", _mutant_gemv(mistake))
    caught = 0
    for pin in (lambda: test_dequant_gemv_hand_example(golden_dir),
                lambda: test_dequant_gemv_equals_layer_output_of_q(True)):
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1


# ---------------------------------------------------------------- the page's own minimal quantizer
def _page_minimal_quantizer_f64(W, X, bits, blocksize, percdamp):
    """The steps of [wiki] "최소 구현" run directly in torch float64 on the CPU
    (a second, independent restatement: torch's own Cholesky, Cholesky-inverse
    and products, nothing from the oracle): one asymmetric grid per row from
    the original weights, H = 2 X^T X damped by percdamp of its mean diagonal,
    the upper Cholesky factor of its inverse, then per block the column loop
    (quantize, error over the diagonal entry, in-block correction) and one
    product for the columns after the block.  Returns the dequantized weights."""
    import torch
    W = torch.tensor(np.asarray(W, dtype=np.float64))
    X = torch.tensor(np.asarray(X, dtype=np.float64))
    d = W.shape[1]
    top = float(2 ** bits - 1)
    lo, hi = W.amin(dim=1), W.amax(dim=1)
    step = torch.clamp(hi - lo, min=1e-8) / top
    offset = torch.round(-lo / step)
    H = 2.0 * (X.T @ X)
    H = H + percdamp * torch.diagonal(H).mean() * torch.eye(d, dtype=torch.float64)
    R = torch.linalg.cholesky(torch.cholesky_inverse(torch.linalg.cholesky(H)), upper=True)
    Q = torch.zeros_like(W)
    for a in range(0, d, blocksize):
        b = min(a + blocksize, d)
        panel = W[:, a:b].clone()
        errs = torch.zeros_like(panel)
        for k in range(b - a):
            col = panel[:, k]
            lvl = torch.clamp(torch.round(col / step) + offset, 0.0, top)
            qcol = step * (lvl - offset)
            Q[:, a + k] = qcol
            e = (col - qcol) / R[a + k, a + k]
            panel[:, k:] -= torch.outer(e, R[a + k, a + k:b])
            errs[:, k] = e
        W[:, b:] -= errs @ R[a:b, b:]
    return Q.numpy()


@pytest.mark.parametrize("d_out,d_in,n,bits,blocksize", [(48, 64, 400, 4, 128), (40, 96, 500, 3, 32),
                                                         (32, 64, 300, 2, 16)])
def test_oracle_reproduces_the_page_minimal_quantizer(d_out, d_in, n, bits, blocksize):
    """T6: with the page's own grid (scale and zero kept in the working
    precision, reading B) the oracle gives the same dequantized weights as the
    page's minimal quantizer run in float64, up to the order of rounding."""
    rng = np.random.default_rng(60 + d_in + bits)
    X = synth.ar1_rows(rng, n, d_in, 0.9).astype(np.float64)
    W = rng.standard_normal((d_out, d_in)) * 0.02
    Q_page = _page_minimal_quantizer_f64(W, X, bits, blocksize, 0.01)
    Hd, _ = oracle.damp(oracle.hessian([X]), 0.01)
    U = oracle.hinv_upper_factor(Hd)
    out = oracle.gptq_quantize(W, U, bits, blocksize, -1, grid="working")
    assert np.max(np.abs(out["Q"] - Q_page)) <= 1e-12
    # and the stored-grid default differs from it only through the fp16 grid:
    # the same sweep on the page's grid values would be the page's result
    s, z = oracle.grid_params_working_precision(W.min(1), W.max(1), bits)
    assert np.array_equal(out["scales"][:, 0], s) and np.array_equal(out["zeros"][:, 0], z)


def test_page_minimal_quantizer_restatement_is_not_the_fp16_grid():
    """Control: the two readings of the grid really differ (so the comparison
    above checks the sweep, not a coincidence of grids)."""
    rng = np.random.default_rng(7)
    X = synth.ar1_rows(rng, 400, 64, 0.9).astype(np.float64)
    W = rng.standard_normal((48, 64)) * 0.02
    Q_page = _page_minimal_quantizer_f64(W, X, 4, 128, 0.01)
    Hd, _ = oracle.damp(oracle.hessian([X]), 0.01)
    out = oracle.gptq_quantize(W, oracle.hinv_upper_factor(Hd), 4, 128, -1)
    assert np.max(np.abs(out["Q"] - Q_page)) > 1e-6


def test_planted_sweep_mistake_breaks_the_page_cross_check(monkeypatch):
    """Planted in the oracle: the in-block correction skips the next column.
    The cross-check with the page's quantizer must catch it."""
    rng = np.random.default_rng(61)
    X = synth.ar1_rows(rng, 400, 64, 0.9).astype(np.float64)
    W = rng.standard_normal((48, 64)) * 0.02
    Q_page = _page_minimal_quantizer_f64(W, X, 4, 128, 0.01)
    Hd, _ = oracle.damp(oracle.hessian([X]), 0.01)
    U = oracle.hinv_upper_factor(Hd)
    real_outer = np.outer

    def outer_skipping_next(a, b):
        o = real_outer(a, b)
        if o.shape[1] > 1:
            o[:, 1] = 0.0
        return o
    monkeypatch.setattr(np, "outer", outer_skipping_next)
    out = oracle.gptq_quantize(W, U, 4, 128, -1, grid="working")
    monkeypatch.setattr(np, "outer", real_outer)
    assert np.max(np.abs(out["Q"] - Q_page)) > 1e-6
