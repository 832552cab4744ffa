"""Block-sequential whole-model calibration on the GPU.

Source: itwiki "GPTQ", the paragraph closing "최소 구현" (the blocks are taken
one at a time: the calibration inputs pass through the block while H
accumulates for each of its linear layers, the layers are quantized, and the
quantized block's outputs become the next block's inputs); blog "GPTQ를
밑바닥부터 구현하며 배운 것들", section 3 (forward hooks capture the inputs
reaching every linear layer).

The blocks are the caller's torch modules and their forward is the caller's;
every GPTQ step runs in libgptq: each nn.Linear's inputs go to the Hessian
kernel as the block runs (a forward hook per layer), then each layer is
quantized (factorization, blocked sweep, packing; act-order if asked), its
weight is replaced by the dequantized Q, and the quantized block runs once
more to produce the next block's inputs.  All layers of a block are
calibrated on the same pass of the unquantized block, and quantized
concurrently, each on a stream of its own.
"""
from __future__ import annotations

import dataclasses

import torch
from torch import nn

from . import api


_STREAMS: dict = {}   # device -> streams for the layers' quantization


@dataclasses.dataclass
class QuantizedLinear:
    """The stored form of one layer (codes in processing order) and, if
    asked for, its Hessian (upper triangle) for diagnostics."""
    codes: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor
    perm: torch.Tensor | None
    H: torch.Tensor | None = None


class BlockSequential:
    def __init__(self, bits: int = 4, groupsize: int = -1, percdamp: float = 0.01, act_order: bool = False,
                 keep_hessian: bool = False, max_tokens: int = 32768):
        self.bits, self.groupsize, self.percdamp = bits, groupsize, percdamp
        self.act_order, self.keep_hessian = act_order, keep_hessian
        self.max_tokens = max_tokens

    @staticmethod
    def linears(block: nn.Module):
        return [(name, m) for name, m in block.named_modules() if isinstance(m, nn.Linear)]

    @torch.no_grad()
    def quantize(self, blocks, inputs, stream=None):
        """Quantize `blocks` (a list of nn.Module on one GPU) in order, with
        `inputs` (a list of calibration batches, device tensors) entering the
        first one.  The weights of every nn.Linear are replaced by their
        dequantized values.  Returns one dict per block (layer name ->
        QuantizedLinear) and the last block's outputs."""
        xs, groups = self._merge(list(inputs))
        report = []
        for block in blocks:
            layers = self.linears(block)
            rows = max(x.numel() // x.shape[-1] for x in xs)
            quant, hooks = {}, []
            for name, m in layers:
                d_out, d_in = m.weight.shape
                f32 = m.weight.dtype == torch.float32
                lq = api.LayerQuantizer(d_out, d_in, self.bits, self.groupsize, 128, self.percdamp,
                                        device=m.weight.device, want_q=True, max_f32_rows=rows if f32 else 0,
                                        act_order=self.act_order)
                lq.begin(m.weight.detach(), stream)
                quant[name] = lq

                def hook(mod, inp, out, lq=lq, d_in=d_in):
                    x = inp[0].reshape(-1, d_in)
                    if x.dtype not in (torch.float32, torch.bfloat16):
                        x = x.float()
                    lq.add_batch(x.contiguous(), stream)
                hooks.append(m.register_forward_hook(hook))
            try:
                for x in xs:
                    block(x)
            finally:
                for h in hooks:
                    h.remove()
            # The layers' factorizations and sweeps are independent: each runs
            # on a stream of its own (the library gives every caller stream its
            # own internal streams), forked from and joined back to the
            # calibration stream.
            out = {}
            main = stream if stream is not None else torch.cuda.current_stream()
            ready = torch.cuda.Event()
            ready.record(main)
            done = []
            for (name, m), side in zip(layers, self._streams(len(layers))):
                side.wait_event(ready)
                lq = quant[name]
                with torch.cuda.stream(side):
                    lq.finish(side)
                    m.weight.copy_(lq.Q.to(m.weight.dtype))
                ev = torch.cuda.Event()
                ev.record(side)
                done.append(ev)
                out[name] = QuantizedLinear(lq.codes, lq.scales, lq.zeros, lq.perm,
                                            lq.H if self.keep_hessian else None)
            for ev in done:
                main.wait_event(ev)
            report.append(out)
            with torch.cuda.stream(main):
                xs = [block(x) for x in xs]
        return report, [part for x, g in zip(xs, groups) for part in x.split(g)]

    def _merge(self, xs):
        """Consecutive batches of the same sequence shape joined into one,
        up to max_tokens tokens each: one forward (and one Hessian call per
        layer) instead of several.  H is the same sum over the same rows.
        Returns the joined batches and, for each, the sizes of its parts."""
        out, groups, cur, n = [], [], [], 0
        for x in xs:
            t = x.numel() // x.shape[-1]
            if cur and (x.shape[1:] != cur[0].shape[1:] or n + t > self.max_tokens):
                out.append(torch.cat(cur) if len(cur) > 1 else cur[0])
                groups.append([c.shape[0] for c in cur])
                cur, n = [], 0
            cur.append(x)
            n += t
        if cur:
            out.append(torch.cat(cur) if len(cur) > 1 else cur[0])
            groups.append([c.shape[0] for c in cur])
        return out, groups

    @staticmethod
    def _streams(n):
        """n streams of the current device, created once per process and
        reused, so that each keeps the library's internal streams it was
        given."""
        dev = torch.cuda.current_device()
        pool = _STREAMS.setdefault(dev, [])
        while len(pool) < n:
            pool.append(torch.cuda.Stream(dev))
        return pool[:n]
