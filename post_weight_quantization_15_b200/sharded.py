"""One layer split over several GPUs (one process per GPU, torch.distributed over NCCL).

The GPTQ pages quantize a layer on one GPU; the layer's work splits two ways:

* H = 2 . X . X^T is a sum over calibration tokens ("polydesk.ai/glossaire/gptq",
  "Etape 2"), so each rank forms the partial H of its own token range with the
  library's Hessian kernel and one all-reduce (sum) over the ranks completes it, with
  the fp64 act-order key beside it;
* given U, rows are independent ("Etape 1": the order of the columns, and with it the
  inverse-Hessian work, is shared by every row), so each rank quantizes its own range
  of output rows, and the row shards are gathered along the outputs.

Every rank then prepares U from the same H bits (the all-reduce leaves the same sum
on every rank, and preparation is deterministic), so U needs no broadcast.  The
collectives are torch.distributed calls on device tensors (NCCL: the Hessian's
all-reduce and the gathers run over NVLink); nothing here is arithmetic of the
method besides the partition of rows and tokens.  No TMA multicast is involved: each
rank's kernels read only its own GPU's memory.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch


def split_range(total: int, world: int, rank: int, align: int = 1) -> Tuple[int, int]:
    """[lo, hi) of rank's share of `total` items, contiguous and balanced; every boundary
    but the last is a multiple of `align` (e.g. 8 tokens, so each shard of a row-major
    bf16 X starts 16-byte aligned)."""
    if world < 1 or not 0 <= rank < world or total < 0 or align < 1:
        raise ValueError("bad partition arguments")
    units = (total + align - 1) // align
    lo = units * rank // world * align
    hi = units * (rank + 1) // world * align
    return min(lo, total), min(hi, total)


def allreduce_hessian(H: torch.Tensor, hdiag: Optional[torch.Tensor] = None, group=None) -> None:
    """Complete the token-sharded Hessian in place: H (and the act-order key) summed over
    the ranks.  Every rank must call this with the same shapes, in the same order."""
    import torch.distributed as dist
    dist.all_reduce(H, op=dist.ReduceOp.SUM, group=group)
    if hdiag is not None:
        dist.all_reduce(hdiag, op=dist.ReduceOp.SUM, group=group)


def gather_rows(parts: Sequence[Optional[torch.Tensor]], out_sizes: Sequence[int], dim: int,
                group=None) -> List[Optional[torch.Tensor]]:
    """All-gather row-sharded outputs and concatenate them along the outputs.

    ``parts`` are this rank's tensors; ``dim`` is the output dimension of each (1 for
    qweight / scales / zeros [*, out], 0 for codes [out, n] and err_sq [out]); shard r has
    out_sizes[r] outputs.  Returns the whole tensors, the same on every rank."""
    import torch.distributed as dist
    world = len(out_sizes)
    res = []
    for t in parts:
        if t is None:
            res.append(None)
            continue
        t = t.contiguous()
        pad = max(out_sizes)
        if t.shape[dim] != pad:     # all_gather needs equal shapes: pad each shard to the largest
            shape = list(t.shape)
            shape[dim] = pad
            buf = torch.zeros(shape, dtype=t.dtype, device=t.device)
            buf.narrow(dim, 0, t.shape[dim]).copy_(t)
            t = buf
        bufs = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(bufs, t, group=group)
        res.append(torch.cat([b.narrow(dim, 0, k) for b, k in zip(bufs, out_sizes)], dim=dim))
    return res


def quantize_layer_sharded(W: torch.Tensor, X_shard: torch.Tensor, bits: int = 4, group_size: int = 128,
                           sym: bool = False, desc_act: bool = False, damp_percent: float = 0.01,
                           block: int = 128, want_codes: bool = False, gather: bool = True, group=None):
    """The whole path for one layer split over the ranks of ``group``.

    W: the whole layer [out, n] on this rank's GPU (only this rank's rows are read), or
    just this rank's rows when ``gather`` is False and the caller sliced it with
    split_range.  X_shard: this rank's calibration tokens, bf16 [n, tokens_r] on the
    GPU (any token split; split_range(N, world, rank, 8) keeps rows aligned).
    Returns (layer, prep): ``layer`` the whole QuantizedLayer (gather=True) or this
    rank's row shard, ``prep`` the rank's (identical) preparation.
    """
    import torch.distributed as dist

    from . import gptq as G
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    n = X_shard.shape[0]
    dev = X_shard.device
    status = G.new_status(dev)
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    hdiag = torch.zeros(n, dtype=torch.float64, device=dev) if desc_act else None
    if X_shard.shape[1] > 0:
        G.hessian_accumulate(H, X_shard, hdiag, status)
    allreduce_hessian(H, hdiag, group)
    prep = G.prepare(H, damp_percent, desc_act, hdiag, status)
    out = W.shape[0]
    if gather:
        o0, o1 = split_range(out, world, rank)
        W_rows = W[o0:o1]
        sizes = [split_range(out, world, r)[1] - split_range(out, world, r)[0] for r in range(world)]
    else:
        W_rows = W
        sizes = None
    q = G.quantize_layer(W_rows.contiguous(), prep, bits, group_size, sym, block, want_codes=want_codes,
                         want_err=True)
    G.raise_on_status(status, "quantize_layer_sharded")
    if not gather:
        return q, prep
    qweight, scales, zeros = gather_rows([q.qweight, q.scales, q.zeros], sizes, 1, group)
    codes, err_sq = gather_rows([q.codes, q.err_sq], sizes, 0, group)
    whole = G.QuantizedLayer(qweight, scales, zeros, q.g_idx, codes, err_sq, q.bits, q.group_size, q.sym)
    return whole, prep
