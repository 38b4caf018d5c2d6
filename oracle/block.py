"""float64 CPU oracle of the whole recurrent block and of the MLP around it --
TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this module; the product path never does.

What it computes, in the order the pages give it ("Gemma explained:
RecurrentGemma architecture"):

  * RecurrentGemmaRecurrentBlock printout and section "Residual block with
    recurrent block": the block input u feeds two Linear(D, D, bias=True)
    layers, linear_x and linear_y.  linear_x feeds the causal depthwise conv
    and the RG-LRU; linear_y is the GELU branch; their product feeds
    linear_out, a third Linear(D, D, bias=True).
  * RecurrentGemmaMlp printout: gate_proj and up_proj, Linear(D, 3 D,
    bias=True) each (MLP expansion factor 3, section "MLP expansion
    factor"); the tanh GELU (PytorchGELUTanh) on the gate; their product
    feeds down_proj, Linear(3 D, D, bias=True).
  * The decoder layer (printout: temporal_pre_norm, temporal block,
    channel_pre_norm, mlp_block; section "Residual block with recurrent
    block"): RMSNorm, the recurrent block, a residual add, RMSNorm, the MLP,
    a residual add.  The pages name RecurrentGemmaRMSNorm without a formula;
    this is the standard root-mean-square normalisation with a learned scale,
    x / sqrt(mean(x^2) + eps) * w (reading stated here; eps = 1e-6).

A Linear layer is ``y = x W^T + b`` with W stored [out, in] (torch's layout,
the one the printout's modules use).  The product with numpy's matmul in
float64 is the one library step; nothing is blocked or reordered.

Reading of the pages: the block in bf16 I/O passes bf16 tensors between its
layers -- x and the gate branch are the core's bf16 inputs, the core's
output y is bf16, and so is every layer's output -- so each layer output is
rounded (nearest, ties to even) to bf16 once, here as on the GPU.  The
rounding is this module's own (``round_bf16``).
"""
from __future__ import annotations

import numpy as np

from oracle import oracle as core


def round_bf16(v) -> np.ndarray:
    """Nearest bf16 value (8 significant bits, ties to even) of each float64
    element, returned as float64.  |v| below 2^-126 is not expected here."""
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros_like(v)
    nz = v != 0
    mant, ex = np.frexp(v[nz])            # v = mant 2^ex, 0.5 <= |mant| < 1
    out[nz] = np.ldexp(np.round(np.ldexp(mant, 8)), ex - 8)  # np.round: ties to even
    return out


def linear(x, W, b=None) -> np.ndarray:
    """y = x W^T + b in float64 (x [..., in], W [out, in], b [out])."""
    y = np.asarray(x, np.float64) @ np.asarray(W, np.float64).T
    if b is not None:
        y = y + np.asarray(b, np.float64)
    return y


def gelu_tanh(g) -> np.ndarray:
    """0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3))), the PytorchGELUTanh form."""
    g = np.asarray(g, np.float64)
    return 0.5 * g * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (g + 0.044715 * g ** 3)))


def recurrent_block(u, W_lin_x, b_lin_x, W_lin_y, b_lin_y, W_out, b_out, conv_w, conv_b, W_a, b_a,
                    W_x, b_x, lam, segpos, conv_state, h_state, round_io: bool = True,
                    nthreads: int = 0) -> dict:
    """The recurrent block over u [B, T, D]: returns out [B,T,D], the new
    conv_state and h_state, and the intermediates x, g, y (all float64)."""
    rnd = round_bf16 if round_io else (lambda a: np.asarray(a, np.float64))
    x = rnd(linear(u, W_lin_x, b_lin_x))
    g = rnd(linear(u, W_lin_y, b_lin_y))
    c = core.prefill(x, g, conv_w, conv_b, W_a, b_a, W_x, b_x, lam, segpos, conv_state, h_state,
                     nthreads=nthreads)
    y = rnd(c["y"])
    out = rnd(linear(y, W_out, b_out))
    return {"out": out, "conv_state": c["conv_state"], "h_state": c["h_state"], "x": x, "g": g, "y": y}


def mlp(v, W_gate, b_gate, W_up, b_up, W_down, b_down, round_io: bool = True) -> np.ndarray:
    """down_proj(GELU_tanh(gate_proj(v)) * up_proj(v)); the product (the
    down projection's input) is a bf16 tensor in bf16 I/O."""
    rnd = round_bf16 if round_io else (lambda a: np.asarray(a, np.float64))
    h = rnd(gelu_tanh(linear(v, W_gate, b_gate)) * linear(v, W_up, b_up))
    return rnd(linear(h, W_down, b_down))


def rmsnorm(x, w, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * w over the last axis, float64."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w, np.float64)


def residual_block(u, w_temporal_norm, W_lin_x, b_lin_x, W_lin_y, b_lin_y, W_out, b_out, conv_w, conv_b, W_a,
                   b_a, W_x, b_x, lam, segpos, conv_state, h_state, w_channel_norm, W_gate, b_gate, W_up, b_up,
                   W_down, b_down, eps: float = 1e-6, round_io: bool = True) -> dict:
    """The recurrent residual block over u [B, T, D] in float64, each layer's
    output rounded to bf16 once (``round_io``): returns out, the new states and
    the intermediates n (normalised u), h (after the first residual add)."""
    rnd = round_bf16 if round_io else (lambda a: np.asarray(a, np.float64))
    u = np.asarray(u, np.float64)
    n = rnd(rmsnorm(u, w_temporal_norm, eps))
    x = rnd(linear(n, W_lin_x, b_lin_x))
    g = rnd(linear(n, W_lin_y, b_lin_y))
    c = core.prefill(x, g, conv_w, conv_b, W_a, b_a, W_x, b_x, lam, segpos, conv_state, h_state)
    y = rnd(c["y"])
    h = rnd(linear(y, W_out, b_out) + u)
    n2 = rnd(rmsnorm(h, w_channel_norm, eps))
    m = rnd(gelu_tanh(linear(n2, W_gate, b_gate)) * linear(n2, W_up, b_up))
    out = rnd(linear(m, W_down, b_down) + h)
    return {"out": out, "conv_state": c["conv_state"], "h_state": c["h_state"], "n": n, "h": h}
