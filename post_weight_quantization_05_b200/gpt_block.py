"""A pre-LN GPT block in torch, the model that whole-model calibration runs
on (random-init weights from the seeded generator; no checkpoint exists
here).  x + attn_out(causal multi-head attention of qkv(ln1(x))), then
x + mlp_proj(gelu(fc(ln2(x)))); LayerNorm eps 1e-5 with unit gain and zero
shift, exact (erf) GELU, no biases.  This is the caller's model: its forward
runs in torch; only the GPTQ steps run in libgptq."""
from __future__ import annotations

import torch
import torch.nn.functional as F
from torch import nn


class GPTBlock(nn.Module):
    def __init__(self, d_model: int, n_heads: int):
        super().__init__()
        self.n_heads = n_heads
        self.ln1 = nn.LayerNorm(d_model, eps=1e-5)
        self.qkv = nn.Linear(d_model, 3 * d_model, bias=False)
        self.attn_out = nn.Linear(d_model, d_model, bias=False)
        self.ln2 = nn.LayerNorm(d_model, eps=1e-5)
        self.fc = nn.Linear(d_model, 4 * d_model, bias=False)
        self.mlp_proj = nn.Linear(4 * d_model, d_model, bias=False)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        B, T, d = x.shape
        q, k, v = self.qkv(self.ln1(x)).split(d, dim=-1)
        heads = lambda t: t.reshape(B, T, self.n_heads, d // self.n_heads).transpose(1, 2)  # noqa: E731
        a = F.scaled_dot_product_attention(heads(q), heads(k), heads(v), is_causal=True)
        x = x + self.attn_out(a.transpose(1, 2).reshape(B, T, d))
        return x + self.mlp_proj(F.gelu(self.fc(self.ln2(x))))


def gpt_stack(weights, n_heads: int, device="cuda", dtype=torch.float32):
    """Blocks from per-block dicts of fp32 weights (synth.gpt_stack_weights)."""
    blocks = []
    for W in weights:
        d = W["attn_out"].shape[0]
        blk = GPTBlock(d, n_heads)
        with torch.no_grad():
            for name, w in W.items():
                getattr(blk, name).weight.copy_(torch.from_numpy(w))
        blocks.append(blk.to(device=device, dtype=dtype).eval())
    return blocks
