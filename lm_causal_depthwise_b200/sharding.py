"""Head sharding and time sharding of the block core across GPUs (one
process per GPU).

Heads never mix in the core: the conv is depthwise, the gate projections are
block-diagonal per head of 256 channels and the scan is per channel.  A rank
therefore runs the core on its own contiguous range of heads -- the columns
of x, the gate branch, the states and the per-channel parameters that belong
to them -- with no collective on the data path; the outputs of the ranks are
the full output's column blocks.  (In a tensor-parallel model these blocks are
what a column-parallel linear_x / linear_y leaves on each rank.)

Time sharding splits one long sequence into contiguous chunks of tokens, one
per rank.  A chunk needs the three raw inputs before its first token (the
conv taps) and the scan state there, which the ranks obtain from one
exchange of their chunks' end states (rglru_carry_scan).

This module only computes the assignments and slices arrays; it holds none of
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


def shard_time(T: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous token range [t0, t1) of ``rank`` in a sequence of T tokens:
    sizes differ by at most one, the larger ranges first (empty for the last
    ranks when world > T)."""
    if T < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError("bad shard arguments")
    base, extra = divmod(T, world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def conv_halo(x: np.ndarray, conv_state: np.ndarray, t0: int) -> np.ndarray:
    """The conv state a chunk starting at token t0 begins with: the three raw
    inputs before t0, oldest first ([B, 3, D]), taken from the carried conv
    state where t0 < 3."""
    prev = np.concatenate([np.asarray(conv_state), np.asarray(x)[:, max(0, t0 - 3):t0]], axis=1)
    return np.ascontiguousarray(prev[:, -3:])


def shard_time_inputs(inp: dict, t0: int, t1: int) -> dict:
    """The core's inputs for tokens [t0, t1): the time slices of x, the gate
    branch and segment_pos, and the conv state at t0.  h_state is left as
    given (each pass sets its own)."""
    out = dict(inp)
    for k in ("x", "g"):
        out[k] = np.ascontiguousarray(inp[k][:, t0:t1])
    out["segpos"] = np.ascontiguousarray(inp["segpos"][:, t0:t1])
    out["conv_state"] = conv_halo(inp["x"], inp["conv_state"], t0)
    return out
