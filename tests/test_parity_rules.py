"""Host checks of the code-parity rules the GPU tests apply (tests/parity_util.py):
a grid that differs from the oracle's is accepted only at a rounding near-tie of
the oracle's own grid computation, and a code difference only as a one-level
flip at a near-tie.  Mistakes are planted in the oracle's output, on the CPU."""
import numpy as np
import pytest

import oracle
from parity_util import GRID_TIE_REL, check_codes, grid_flip_at_tie


def _ref_with_grid(mn, mx, bits=4):
    s, z = oracle.grid_params(np.float32([mn]), np.float32([mx]), bits)
    return {"gmin": np.float32([[mn]]), "gmax": np.float32([[mx]]), "scales": s[:, None], "zeros": z[:, None],
            "bits": bits}


def _range_at_fp16_midpoint(k=700):
    """A range whose range / 15 lands (in fp32) as close as possible to the
    midpoint of two adjacent fp16 values near 2^-6 * (1 + k/1024)."""
    lo = np.float16(2.0 ** -6 * (1 + k / 1024))
    hi = np.nextafter(lo, np.float16(1), dtype=np.float16)
    mid = 0.5 * (float(lo) + float(hi))
    return np.float32(mid * 15), float(lo), float(hi)


def test_scale_flip_at_tie_is_accepted():
    rng, lo, hi = _range_at_fp16_midpoint()
    ref = _ref_with_grid(np.float32(-0.5) * rng, np.float32(0.5) * rng)
    s_ref = float(ref["scales"][0, 0])
    other = hi if s_ref == lo else lo
    ok, why = grid_flip_at_tie(ref, 0, 0, other, float(ref["zeros"][0, 0]))
    assert ok, why


def test_scale_flip_away_from_tie_is_caught():
    # range / 15 a quarter of an fp16 step from the boundary
    rng, lo, hi = _range_at_fp16_midpoint()
    rng = np.float32(float(rng) + 0.25 * (hi - lo) * 15)
    ref = _ref_with_grid(np.float32(-0.5) * rng, np.float32(0.5) * rng)
    s_ref = float(ref["scales"][0, 0])
    other = hi if s_ref == lo else lo
    ok, _ = grid_flip_at_tie(ref, 0, 0, other, float(ref["zeros"][0, 0]))
    assert not ok
    # and a scale two fp16 steps away is never a tie
    far = float(np.nextafter(np.float16(other), np.float16(np.inf if other > s_ref else -np.inf), dtype=np.float16))
    ok, _ = grid_flip_at_tie(ref, 0, 0, far, float(ref["zeros"][0, 0]))
    assert not ok


def test_zero_flip_rules():
    s = np.float32(np.float16(0.01))
    # -min / s = 3.5 exactly: a tie, either zero is a rounding of it
    ref = _ref_with_grid(np.float32(-3.5) * s, np.float32(11.5) * s)
    assert float(ref["scales"][0, 0]) == float(s)
    z = float(ref["zeros"][0, 0])
    ok, why = grid_flip_at_tie(ref, 0, 0, float(s), z + 1.0 if z == 4.0 else z - 1.0)
    assert ok, why
    # -min / s = 3.3: no tie
    ref = _ref_with_grid(np.float32(-3.3) * s, np.float32(11.7) * s)
    if float(ref["scales"][0, 0]) == float(s):
        ok, _ = grid_flip_at_tie(ref, 0, 0, float(s), float(ref["zeros"][0, 0]) + 1.0)
        assert not ok


def _small_case(groupsize):
    rng = np.random.default_rng(5)
    d_out, d_in = 24, 256
    X = rng.standard_normal((600, d_in))
    for a in range(1, d_in):
        X[:, a] = 0.9 * X[:, a - 1] + np.sqrt(1 - 0.81) * X[:, a]
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    Hd, _ = oracle.damp(oracle.hessian([X]), 0.01)
    U = oracle.hinv_upper_factor(Hd)
    return W, U, oracle.gptq_quantize(W, U, 4, 128, groupsize, return_trace=True)


def test_check_codes_passes_the_oracle_itself():
    _, _, ref = _small_case(128)
    assert check_codes(ref["codes"], ref, "self", groupsize=128, gpu_scales=ref["scales"],
                       gpu_zeros=ref["zeros"]) == 1.0


def test_check_codes_catches_a_wrong_group_grid():
    """Planted: one group's grid taken from a shifted minimum (a wrong min/max)."""
    W, U, ref = _small_case(128)
    s = ref["scales"].copy()
    z = ref["zeros"].copy()
    codes = ref["codes"].copy()
    r, gi = 3, 1
    s[r, gi] = float(np.float16(s[r, gi] * 1.1))
    codes[r, gi * 128 + 5] = (codes[r, gi * 128 + 5] + 1) % 16
    with pytest.raises(AssertionError, match="grid differs away from a tie"):
        check_codes(codes, ref, "planted", match=0.9, groupsize=128, gpu_scales=s, gpu_zeros=z)


def test_check_codes_catches_a_flip_away_from_a_tie():
    """Planted: a code two levels off, and a one-level flip far from any tie."""
    _, _, ref = _small_case(-1)
    codes = ref["codes"].copy()
    codes[2, 40] += 2 if codes[2, 40] < 14 else -2
    with pytest.raises(AssertionError, match="levels"):
        check_codes(codes, ref, "planted", match=0.9)
    codes = ref["codes"].copy()
    t = ref["W_at"] / ref["scales"][:, :1] + ref["zeros"][:, :1]
    far = np.abs((t - np.floor(t)) - 0.5) > 0.2
    r, j = map(int, np.argwhere(far)[len(np.argwhere(far)) // 2])
    codes[r, j] += 1 if codes[r, j] < 15 else -1
    with pytest.raises(AssertionError, match="away from a tie"):
        check_codes(codes, ref, "planted", match=0.9)


def test_grid_tie_tolerance_is_below_an_fp16_step():
    # the accepted distance from the rounding boundary is a small part of one
    # fp16 step (2^-10 relative at most), so a scale from a wrong range fails
    assert GRID_TIE_REL < 0.25 * 2.0 ** -10


def test_decision_stats_counts_prefixes():
    from parity_util import decision_stats
    ref = np.zeros((3, 10), dtype=np.int64)
    got = ref.copy()
    got[0, 4:] = 1          # first difference at column 4: 5 decisions from identical states
    got[2, 0] = 1           # at column 0: 1 decision
    assert decision_stats(got, ref) == (2, 5 + 10 + 1)
