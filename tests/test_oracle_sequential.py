"""Pins for the block-sequential oracle (oracle/sequential.py): the block
forward against textbook values, brute force and closed forms, and the
driver's data flow against an explicit composition of quantized layers."""
import numpy as np
import pytest

import oracle
from oracle import sequential as sq
from post_weight_quantization_05_b200 import synth


def test_gelu_textbook_values():
    # x * Phi(x), Phi the standard normal distribution function
    assert sq.gelu(0.0) == 0.0
    assert sq.gelu(1.0) == pytest.approx(0.8413447460685429, rel=1e-15)
    assert sq.gelu(-1.0) == pytest.approx(-0.15865525393145707, rel=1e-14)
    assert sq.gelu(2.0) == pytest.approx(2.0 * 0.9772498680518208, rel=1e-15)


def test_layer_norm_statistics():
    x = np.random.default_rng(0).normal(3.0, 2.0, size=(5, 64))
    y = sq.layer_norm(x)
    assert np.allclose(y.mean(axis=-1), 0.0, atol=1e-14)
    var = x.var(axis=-1)
    assert np.allclose((y ** 2).mean(axis=-1), var / (var + 1e-5), rtol=1e-13)


def _brute_attention(q, k, v):
    B, Hh, T, dh = q.shape
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(Hh):
            for t in range(T):
                s = [float(q[b, h, t] @ k[b, h, u]) / np.sqrt(dh) for u in range(t + 1)]
                m = max(s)
                e = [np.exp(x - m) for x in s]
                tot = sum(e)
                out[b, h, t] = sum(e[u] / tot * v[b, h, u] for u in range(t + 1))
    return out


def test_attention_equals_brute_force():
    rng = np.random.default_rng(1)
    q, k, v = (rng.standard_normal((2, 3, 5, 4)) for _ in range(3))
    assert np.allclose(sq.causal_attention(q, k, v), _brute_attention(q, k, v), rtol=1e-12, atol=1e-14)


def test_block_is_causal():
    W = synth.gpt_stack_weights(1, 64)[0]
    x = synth.gpt_stack_inputs(1, 2, 10, 64)[0].astype(np.float64)
    y = sq.gpt_block(W, x, 4)
    x2 = x.copy()
    x2[:, 6:] += np.random.default_rng(2).standard_normal(x2[:, 6:].shape)
    y2 = sq.gpt_block(W, x2, 4)
    assert np.array_equal(y[:, :6], y2[:, :6])
    assert not np.allclose(y[:, 6:], y2[:, 6:])


def test_block_with_one_token_closed_form():
    """With T = 1 attention returns v, so the block is
    x1 = x + (ln(x) Wv^T) Wo^T, then x1 + gelu(ln(x1) Wfc^T) Wp^T."""
    d = 64
    W = synth.gpt_stack_weights(1, d, base_seed=3)[0]
    x = synth.gpt_stack_inputs(1, 4, 1, d, base_seed=3)[0].astype(np.float64)
    Wv = W["qkv"][2 * d:3 * d].astype(np.float64)
    h = (x - x.mean(-1, keepdims=True)) / np.sqrt(x.var(-1, keepdims=True) + 1e-5)
    x1 = x + (h @ Wv.T) @ W["attn_out"].astype(np.float64).T
    h1 = (x1 - x1.mean(-1, keepdims=True)) / np.sqrt(x1.var(-1, keepdims=True) + 1e-5)
    f = h1 @ W["fc"].astype(np.float64).T
    from scipy.stats import norm
    want = x1 + (f * norm.cdf(f)) @ W["mlp_proj"].astype(np.float64).T
    assert np.allclose(sq.gpt_block(W, x, 4), want, rtol=1e-12, atol=1e-13)


def _linear_block(W, x, capture=None):
    xr = x.reshape(-1, x.shape[-1])
    if capture is not None:
        capture.setdefault("lin", []).append(xr)
    return (xr @ np.asarray(W["lin"], dtype=np.float64).T).reshape(x.shape[:-1] + (-1,))


def _linear_stack(seed=4, d=128, n=3):
    rng = np.random.default_rng(seed)
    blocks = [{"lin": rng.normal(0, 0.05, (d, d))} for _ in range(n)]
    xs = [synth.ar1_rows(np.random.default_rng(seed + b), 256, d, 0.7) for b in range(2)]
    return blocks, xs


def test_driver_feeds_quantized_outputs_forward():
    """Over a stack of single linear layers, block k is calibrated on
    X0 Q1^T ... Q_{k-1}^T (the quantized chain) and the driver returns
    X0 Q1^T ... Qn^T."""
    blocks, xs = _linear_stack()
    res, outs = sq.sequential_gptq(blocks, xs, n_heads=1, bits=4, block_fn=_linear_block)
    chain = [x.astype(np.float64) for x in xs]
    for k, r in enumerate(res):
        assert np.allclose(r["lin"]["H"], oracle.hessian(chain), rtol=1e-12, atol=1e-12)
        Hd, _ = oracle.damp(r["lin"]["H"], 0.01)
        ref = oracle.gptq_quantize(blocks[k]["lin"], oracle.hinv_upper_factor(Hd), 4, 128, -1)
        assert np.array_equal(r["lin"]["codes"], ref["codes"])
        chain = [c @ r["lin"]["Q"].T for c in chain]
    for o, c in zip(outs, chain):
        assert np.allclose(o, c, rtol=1e-12, atol=1e-14)


def test_planted_unquantized_chain_is_caught():
    """A driver that feeds the next block the unquantized outputs fails the
    data-flow pin."""
    blocks, xs = _linear_stack()

    def wrong(blocks, xs):
        out = []
        chain = [x.astype(np.float64) for x in xs]
        for W in blocks:
            H = oracle.hessian(chain)
            out.append(H)
            chain = [c @ np.asarray(W["lin"], dtype=np.float64).T for c in chain]   # float weights
        return out
    res, _ = sq.sequential_gptq(blocks, xs, n_heads=1, bits=4, block_fn=_linear_block)
    Hs = wrong(blocks, xs)
    assert np.allclose(res[0]["lin"]["H"], Hs[0])
    assert not np.allclose(res[1]["lin"]["H"], Hs[1], rtol=1e-6)


def test_gpt_stack_calibration_captures_every_linear():
    blocks = synth.gpt_stack_weights(2, 64)
    xs = synth.gpt_stack_inputs(2, 2, 8, 64)
    res, outs = sq.sequential_gptq(blocks, xs, n_heads=4, bits=4)
    for r in res:
        assert set(r) == set(sq.LINEARS)
        assert r["qkv"]["H"].shape == (64, 64) and r["mlp_proj"]["H"].shape == (256, 256)
        # the fc layer sees ln2 of the post-attention stream: unit-variance rows
        assert np.trace(r["fc"]["H"]) == pytest.approx(2.0 * 2 * 2 * 8 * 64 * (1.0), rel=1e-3)
    assert outs[0].shape == (2, 8, 64) and np.isfinite(outs[0]).all()
