"""The layer split by heads across ranks (one process per GPU).

The heads of the hybrid attention layer are independent through both branches and the
fuse: each rank runs its own heads' slice of q, k, v, the text keys and values, the gate
weights and gamma, and multiplies its part of A by the matching input columns of W_os and
W_ol.  The layer's y is the sum of those partial projections over the ranks: one
reduction, the only exchange ("Video DeltaNet ..." model card, "Set up" and "Inference
with SGLang": the model runs on 8 GPUs).

This module holds the host-side partition: which heads a rank owns, the slices of every
input, and the reduction.  It takes numpy arrays or torch tensors; the device work is
vdn_hybrid_attn_fwd_partial.
"""
from __future__ import annotations

import numpy as np


def head_range(heads: int, world: int, rank: int) -> tuple[int, int]:
    """Half-open head range [h0, h1) of `rank`: contiguous, as equal as possible (the first
    heads % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if heads < world:
        raise ValueError(f"{heads} heads cannot be split over {world} ranks")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def slice_inputs(inp: dict, heads: int, head_dim: int, h0: int, h1: int) -> dict:
    """This rank's inputs from the full layer's: q, k, v [N_v][H][D] and kt, vt [L][H][D]
    along H; w_gate_s [H][D], w_gate_l [H][D][G_l], gamma [H][D] along H; beta [F][H] along
    H; w_os, w_ol [HD (out)][HD (in)] along their input columns h0*D .. h1*D.  The output
    dimension of the projections is not split."""
    c0, c1 = h0 * head_dim, h1 * head_dim
    out = {}
    for name in ("q", "k", "v", "kt", "vt"):
        out[name] = inp[name][:, h0:h1]
    for name in ("w_gate_s", "w_gate_l", "gamma"):
        out[name] = inp[name][h0:h1]
    if "beta" in inp:
        out["beta"] = inp["beta"][:, h0:h1]
    for name in ("w_os", "w_ol"):
        out[name] = inp[name][:, c0:c1]
    return {n: _contiguous(a) for n, a in out.items()}


def _contiguous(a):
    if isinstance(a, np.ndarray):
        return np.ascontiguousarray(a)
    return a.contiguous()


def reduce_partials(y_partial, group=None, scatter_rows: bool = False):
    """Sum of the ranks' float partial outputs (torch.distributed, in place): an all-reduce,
    or with scatter_rows a reduce-scatter that leaves each rank its block of N_v / world
    rows (the row count must divide evenly).  Returns the reduced tensor."""
    import torch
    import torch.distributed as dist
    if not scatter_rows:
        dist.all_reduce(y_partial, op=dist.ReduceOp.SUM, group=group)
        return y_partial
    world = dist.get_world_size(group)
    n = y_partial.shape[0]
    if n % world:
        raise ValueError(f"{n} rows do not split over {world} ranks")
    out = torch.empty((n // world,) + tuple(y_partial.shape[1:]), dtype=y_partial.dtype, device=y_partial.device)
    dist.reduce_scatter_tensor(out, y_partial, op=dist.ReduceOp.SUM, group=group)
    return out
