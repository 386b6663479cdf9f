"""Sequential block pipeline: each layer calibrated on the quantized layers' outputs.

The GPTQ pages quantize a model layer by layer ("polydesk.ai/glossaire/gptq"; the
solver of a layer needs only that layer's inputs), and a layer's calibration inputs
are the activations the layers before it produce once they are quantized.  This
module chains the library's calls over the MLP half of Llama-shaped decoder blocks:

    for each block (gate, up, down), input X [d, tokens] bf16:
        H = 2.X.X^T; prepare; gate and up quantized together (they read X)
        h = silu(What_gate . X) * (What_up . X)     dequantized weights, tensor cores
        H = 2.h.h^T; prepare; down quantized
        X <- X + What_down . h                      the next block's input

(The attention half is not a linear layer of the solver and is left out: its q, k, v
and o layers need attention's own arithmetic between them.)  Every step is a library
kernel: the Hessian, preparation, sweep, dequantization, the bf16 tensor-core
product, the transposes and the elementwise SiLU-gate and residual.  The steps are
data-dependent one after the other (each layer's Hessian needs the previous layer's
quantized output), so they run in order on one stream.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import torch

from . import gptq as G


@dataclasses.dataclass
class BlockResult:
    gate_up: G.QuantizedLayer      # gate and up stacked along the outputs (gate's rows first)
    down: G.QuantizedLayer
    perm_gate_up: torch.Tensor     # the processing order of gate / up's inputs (from their H)
    perm_down: torch.Tensor
    x_in: Optional[torch.Tensor]   # the block's input X [d, tokens] (kept when record=True)
    h: Optional[torch.Tensor]      # down's calibration input [d_ff, tokens] (record=True)
    ms: dict                       # device milliseconds per stage (CUDA events on this stream)


def _events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def quantize_mlp_blocks(X0: torch.Tensor, blocks: Sequence[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]],
                        bits: int = 4, group_size: int = 128, sym: bool = True, desc_act: bool = True,
                        damp_percent: float = 0.01, record: bool = False,
                        status: Optional[torch.Tensor] = None) -> Tuple[List[BlockResult], torch.Tensor]:
    """Quantize MLP blocks in sequence; returns (per-block results, the last block's output).

    X0: bf16 [d, tokens] on the GPU (tokens a multiple of 8).  blocks: (W_gate [d_ff, d],
    W_up [d_ff, d], W_down [d, d_ff]) per block, fp16 / bf16 / fp32 on the GPU.
    """
    dev = X0.device
    st = status if status is not None else G.new_status(dev)
    stream = torch.cuda.current_stream()
    X = X0
    out: List[BlockResult] = []
    for Wg, Wu, Wd in blocks:
        d = X.shape[0]
        d_ff = Wg.shape[0]
        ev = _events(7)
        ev[0].record(stream)
        H = torch.zeros((d, d), dtype=torch.float32, device=dev)
        hd = torch.zeros(d, dtype=torch.float64, device=dev) if desc_act else None
        G.hessian_accumulate(H, X, hd, st)
        prep = G.prepare(H, damp_percent, desc_act, hd, st)
        gate_up, _ = G.quantize_layers([Wg, Wu], prep, bits, group_size, sym)
        perm_gu = prep.perm
        del H, prep
        ev[1].record(stream)
        # the forward of the quantized gate and up
        Xt = G.transpose_bf16(X, st)
        What = G.dequantize(gate_up, torch.bfloat16, st)               # [2 d_ff, d]
        GU = G.linear_bf16(What, Xt, st)                                 # [2 d_ff, tokens] fp32
        del What, Xt
        h = G.silu_mul(GU[:d_ff], GU[d_ff:], st)                         # [d_ff, tokens] bf16
        del GU
        ev[2].record(stream)
        Hd_ = torch.zeros((d_ff, d_ff), dtype=torch.float32, device=dev)
        hdd = torch.zeros(d_ff, dtype=torch.float64, device=dev) if desc_act else None
        G.hessian_accumulate(Hd_, h, hdd, st)
        prep_d = G.prepare(Hd_, damp_percent, desc_act, hdd, st)
        down = G.quantize_layer(Wd, prep_d, bits, group_size, sym)
        perm_d = prep_d.perm
        del Hd_, prep_d
        ev[3].record(stream)
        # the forward of the quantized down, and the residual
        ht = G.transpose_bf16(h, st)
        Wd_hat = G.dequantize(down, torch.bfloat16, st)                  # [d, d_ff]
        Y = G.linear_bf16(Wd_hat, ht, st)                                # [d, tokens] fp32
        del ht, Wd_hat
        X_next = G.residual_add(X, Y, st)
        del Y
        ev[4].record(stream)
        out.append(BlockResult(gate_up, down, perm_gu, perm_d, X if record else None, h if record else None,
                               {"_ev": ev}))
        X = X_next
    torch.cuda.synchronize()
    G.raise_on_status(st, "quantize_mlp_blocks")
    for r in out:
        ev = r.ms.pop("_ev")
        r.ms.update({"gate_up_quantize": ev[0].elapsed_time(ev[1]), "gate_up_forward": ev[1].elapsed_time(ev[2]),
                     "down_quantize": ev[2].elapsed_time(ev[3]), "down_forward": ev[3].elapsed_time(ev[4]),
                     "block": ev[0].elapsed_time(ev[4])})
    return out, X
