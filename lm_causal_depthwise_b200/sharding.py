"""Head sharding of the block core across GPUs (one process per GPU).

Heads never mix in the core: the conv is depthwise, the gate projections are
block-diagonal per head of 256 channels and the scan is per channel.  A rank
therefore runs the core on its own contiguous range of heads -- the columns
of x, the gate branch, the states and the per-channel parameters that belong
to them -- with no collective on the data path; the outputs of the ranks are
the full output's column blocks.  (In a tensor-parallel model these blocks are
what a column-parallel linear_x / linear_y leaves on each rank.)

This module only computes the assignment and slices arrays; it holds none of
the method's arithmetic.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

HEAD = 256


def shard_heads(H: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous head range [h0, h1) of ``rank``: sizes differ by at most one,
    the larger ranges first; ranks beyond H get an empty range."""
    if H < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError("bad shard arguments")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_inputs(inp: dict, h0: int, h1: int) -> dict:
    """The core's inputs restricted to heads [h0, h1): channel slices of the
    [B, T, D] activations, states and per-channel parameters, head slices of
    the gate blocks.  Contiguous copies."""
    c = slice(h0 * HEAD, h1 * HEAD)
    out = dict(inp)
    for k in ("x", "g"):
        out[k] = np.ascontiguousarray(inp[k][:, :, c])
    out["conv_w"] = np.ascontiguousarray(inp["conv_w"][:, c])
    for k in ("conv_b", "b_a", "b_x", "lam"):
        out[k] = np.ascontiguousarray(inp[k][c])
    for k in ("W_a", "W_x"):
        out[k] = np.ascontiguousarray(inp[k][h0:h1])
    out["conv_state"] = np.ascontiguousarray(inp["conv_state"][:, :, c])
    out["h_state"] = np.ascontiguousarray(inp["h_state"][:, c])
    return out
