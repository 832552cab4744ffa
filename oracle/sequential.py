"""Block-sequential whole-model calibration, restated in fp64 (test
infrastructure only, like the rest of this package).

Source: itwiki "GPTQ", the paragraph closing "최소 구현": the transformer
blocks are taken one at a time; the calibration inputs are passed through the
block to accumulate H for each of its linear layers, the layers are quantized,
and the quantized block's outputs become the next block's inputs.  Blog "GPTQ를
밑바닥부터 구현하며 배운 것들", section 3: the inputs reaching every linear
layer are captured (forward hooks) and H = 2 X^T X is built from them.

Readings (the pages name no architecture and no order inside a block):
  R16  the block is a pre-LN GPT block: x + attn(ln1(x)), then
       x + mlp_proj(gelu(fc(ln2(x)))); attn = attn_out(causal multi-head
       softmax(q k^T / sqrt(d_head)) v) with q, k, v from qkv; LayerNorm with
       eps 1e-5, unit gain and zero shift; exact (erf) GELU; no biases.
  R17  all linear layers of a block are calibrated on the same pass of the
       unquantized block (their inputs are captured together), then all are
       quantized; only then does the quantized block run to produce the next
       block's inputs.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

from .gptq import damp, gptq_quantize, gptq_quantize_act_order, hessian, hinv_upper_factor

LINEARS = ("qkv", "attn_out", "fc", "mlp_proj")


def layer_norm(x, eps: float = 1e-5):
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def gelu(x):
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def causal_attention(q, k, v):
    """q, k, v [B, heads, T, dh] -> [B, heads, T, dh]; position t attends to
    positions <= t."""
    T, dh = q.shape[-2], q.shape[-1]
    s = q @ np.swapaxes(k, -1, -2) / np.sqrt(dh)
    s = np.where(np.tril(np.ones((T, T), dtype=bool)), s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    return p @ v


def gpt_block(W: dict, x, n_heads: int, capture: dict | None = None):
    """One block on x [B, T, d] (R16).  If `capture` is given, the inputs of
    every linear layer are appended to capture[name] as rows [B*T, d_in]."""
    x = np.asarray(x, dtype=np.float64)
    B, T, d = x.shape
    dh = d // n_heads

    def lin(name, h):
        if capture is not None:
            capture.setdefault(name, []).append(h.reshape(-1, h.shape[-1]))
        return h @ np.asarray(W[name], dtype=np.float64).T

    qkv = lin("qkv", layer_norm(x))
    q, k, v = (qkv[..., i * d:(i + 1) * d].reshape(B, T, n_heads, dh).transpose(0, 2, 1, 3) for i in range(3))
    att = causal_attention(q, k, v).transpose(0, 2, 1, 3).reshape(B, T, d)
    x = x + lin("attn_out", att)
    x = x + lin("mlp_proj", gelu(lin("fc", layer_norm(x))))
    return x


def sequential_gptq(blocks, batches, n_heads: int, bits: int = 4, groupsize: int = -1, percdamp: float = 0.01,
                    act_order: bool = False, block_fn=None):
    """R17 over a stack of blocks.  `blocks`: list of dicts name -> W;
    `batches`: the first block's calibration inputs.  `block_fn(W, x,
    capture)` runs one block (default: gpt_block with n_heads).  Returns a list
    (one per block) of dicts name -> {"H", "Q", "codes", "scales", "zeros",
    "perm"}, and the outputs of the last (quantized) block."""
    if block_fn is None:
        def block_fn(W, x, capture=None):
            return gpt_block(W, x, n_heads, capture)
    xs = [np.asarray(b, dtype=np.float64) for b in batches]
    results = []
    for W in blocks:
        cap: dict = {}
        for x in xs:
            block_fn(W, x, cap)
        out, Wq = {}, {}
        for name, Wl in W.items():
            H = hessian(cap[name])
            if act_order:
                r = gptq_quantize_act_order(Wl, H, bits, 128, groupsize, percdamp)
            else:
                Hd, _ = damp(H, percdamp)
                r = gptq_quantize(Wl, hinv_upper_factor(Hd), bits, 128, groupsize)
                r["perm"] = None
            r["H"] = H
            out[name] = r
            Wq[name] = r["Q"]
        results.append(out)
        xs = [block_fn(Wq, x) for x in xs]
    return results, xs
