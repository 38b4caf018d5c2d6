"""Seeded synthetic workloads for the RG-LRU block core.

This module only draws random numbers and lays them out; it holds none of the
block's arithmetic.  The same arrays feed the CUDA library and the float64
oracle, so both see bit-identical inputs.

Shapes follow the recurrent block of the 2B and 9B models: the RNN width is
2560 with 10 heads of 256 in the 2B model ("Gemma explained: RecurrentGemma
architecture", section "Model width and RNN width" and the module printout,
Conv1d(2560, 2560, kernel_size=4, groups=2560)); the 9B-shaped case uses
D=4096 (16 heads of 256).  No trained weights exist here, so every tensor is
drawn from the distributions below.

Recipe (fixed draw order from ``numpy.random.default_rng(seed)``):
  x, g             ~ N(0, 1)                        io dtype
  conv_w [4,D]     ~ N(0, 1/4)  (variance; std 0.5)  fp32,  conv_b = 0
  W_a, W_x [H,256,256] ~ N(0, 1/256) (std 1/16)      io dtype
  b_a, b_x [D]     ~ N(0, 0.1)  (std 0.316)          fp32
  Lambda [D]       : u ~ U[0.9, 0.999], s = u^(1/8), Lambda = log(s/(1-s)),
                     so that sigmoid(Lambda)^8 = u                     fp32
                     (decay="wide": the same draws mapped linearly onto
                     Lambda in [-10, 6.9], so that sigmoid(Lambda)^8 spans
                     about 1e-35 .. 0.999: fast-decay channels, Lambda < 0,
                     up to the slowest decay of the default recipe)
  resets           : a reset at t=0 plus (T/L - 1) distinct positions drawn
                     uniformly from [1, T) per sequence (L = mean document
                     length); segment_pos counts up from each reset.
  initial state    : zero, or h ~ N(0, 0.1), conv ~ N(0, 1) (io dtype).
  x_scale          : x (and the random conv state) multiplied by this factor
                     before rounding (1 in every benchmark workload; parity
                     cases use it for large-magnitude inputs).
Values in bf16 mode are produced in fp32 and rounded to nearest-even bf16
once; they are kept as fp32 arrays that hold exactly bf16-representable values.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np

HEAD = 256


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    D: int
    io: str                       # "f32" or "bf16"
    seed: int
    doc_len: Optional[int] = None  # mean document length for random resets
    reset_at: Tuple[int, ...] = (0,)
    continue_doc: bool = False     # no reset at all: segment_pos = t + 3
    init_state: str = "zero"       # "zero" or "random"
    decode_steps: int = 0          # >0: a batched decode workload of this many steps
    decay: str = "init"            # "init": sigmoid(Lambda)^8 ~ U[0.9, 0.999]; "wide": Lambda in [-10, 6.9]
    x_scale: float = 1.0           # x and the conv state drawn as x_scale * N(0, 1)

    @property
    def H(self) -> int:
        return self.D // HEAD

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def scaled(self, **kw) -> "Workload":
        """Same recipe and seed with other sizes (for parity cases)."""
        return dataclasses.replace(self, **kw)

    def describe(self) -> str:
        kind = "decode" if self.decode_steps else "prefill"
        return f"{self.name}: {kind} B={self.B} T={self.T} D={self.D} {self.io}"


# The benchmark workloads.  The names say what each is; the sizes are in the fields.
TINY_F32 = Workload("tiny-f32", B=1, T=256, D=256, io="f32", seed=0, reset_at=(0, 128))
PREFILL_2B = Workload("prefill-2b", B=8, T=4096, D=2560, io="bf16", seed=1, doc_len=1024)
PREFILL_LONG = Workload("prefill-long", B=1, T=131072, D=2560, io="bf16", seed=2,
                        reset_at=(0,), init_state="random")
PREFILL_LONG_CARRY = Workload("prefill-long-carry", B=1, T=131072, D=2560, io="bf16", seed=2,
                              continue_doc=True, init_state="random")
PREFILL_9B = Workload("prefill-9b", B=16, T=8192, D=4096, io="bf16", seed=3, doc_len=2048)
DECODE_2B = Workload("decode-2b", B=256, T=1024, D=2560, io="bf16", seed=4, doc_len=512,
                     decode_steps=1024)

ALL = {w.name: w for w in (TINY_F32, PREFILL_2B, PREFILL_LONG, PREFILL_LONG_CARRY,
                           PREFILL_9B, DECODE_2B)}


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returned as fp32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32)
    lsb = (bits >> np.uint32(16)) & np.uint32(1)
    out = ((bits + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return out.view(np.float32)


def _io(a: np.ndarray, io: str) -> np.ndarray:
    a = np.asarray(a, dtype=np.float32)
    return round_bf16(a) if io == "bf16" else np.ascontiguousarray(a)


def segment_positions(rng: np.random.Generator, w: Workload) -> np.ndarray:
    B, T = w.B, w.T
    if w.continue_doc:
        return np.broadcast_to(np.arange(T, dtype=np.int32) + 3, (B, T)).copy()
    seg = np.empty((B, T), dtype=np.int32)
    t = np.arange(T)
    for b in range(B):
        if w.doc_len:
            extra = max(T // w.doc_len - 1, 0)
            extra = min(extra, T - 1)
            starts = np.sort(rng.choice(np.arange(1, T), size=extra, replace=False)) if extra else []
            starts = np.concatenate([[0], np.asarray(starts, dtype=np.int64)])
        else:
            starts = np.asarray([s for s in w.reset_at if 0 <= s < T] or [0], dtype=np.int64)
            if starts[0] != 0:
                starts = np.concatenate([[0], starts])
        last = starts[np.searchsorted(starts, t, side="right") - 1]
        seg[b] = (t - last).astype(np.int32)
    return seg


def generate(w: Workload) -> dict:
    """Draw every input of workload ``w``; returns a dict of numpy arrays.

    Keys: x, g [B,T,D]; conv_w [4,D]; conv_b [D]; W_a, W_x [H,256,256];
    b_a, b_x, lam [D]; segpos [B,T] int32; conv_state [B,3,D]; h_state [B,D].
    Float arrays are fp32 holding io-dtype values (fp32 for the parameters
    that are always fp32).  A decode workload uses the same layout, with T =
    the number of steps: step s reads x[:, s], g[:, s] and segpos[:, s].
    """
    if w.D % HEAD:
        raise ValueError("D must be a multiple of 256")
    rng = np.random.default_rng(w.seed)
    B, T, D, H = w.B, w.T, w.D, w.H
    xs = np.float32(w.x_scale)
    if w.io == "f32":
        x = (xs * rng.standard_normal((B, T, D))).astype(np.float32)
        g = rng.standard_normal((B, T, D)).astype(np.float32)
    else:
        x = round_bf16(xs * rng.standard_normal((B, T, D), dtype=np.float32))
        g = round_bf16(rng.standard_normal((B, T, D), dtype=np.float32))
    conv_w = (0.5 * rng.standard_normal((4, D))).astype(np.float32)
    conv_b = np.zeros((D,), dtype=np.float32)
    W_a = _io(rng.standard_normal((H, HEAD, HEAD)) / 16.0, w.io)
    b_a = (np.sqrt(0.1) * rng.standard_normal(D)).astype(np.float32)
    W_x = _io(rng.standard_normal((H, HEAD, HEAD)) / 16.0, w.io)
    b_x = (np.sqrt(0.1) * rng.standard_normal(D)).astype(np.float32)
    u = rng.uniform(0.9, 0.999, size=D)
    if w.decay == "wide":
        lam = (-10.0 + 16.9 * (u - 0.9) / 0.099).astype(np.float32)
    elif w.decay == "init":
        s = u ** (1.0 / 8.0)
        lam = np.log(s / (1.0 - s)).astype(np.float32)
    else:
        raise ValueError(f"unknown decay recipe {w.decay!r}")
    segpos = segment_positions(rng, w)
    if w.init_state == "random":
        h_state = (np.sqrt(0.1) * rng.standard_normal((B, D))).astype(np.float32)
        conv_state = _io(w.x_scale * rng.standard_normal((B, 3, D)), w.io)
    else:
        h_state = np.zeros((B, D), dtype=np.float32)
        conv_state = np.zeros((B, 3, D), dtype=np.float32)
    return dict(x=x, g=g, conv_w=conv_w, conv_b=conv_b, W_a=W_a, b_a=b_a, W_x=W_x, b_x=b_x,
                lam=lam, segpos=segpos, conv_state=conv_state, h_state=h_state)


def algorithmic_bytes(w: Workload) -> int:
    """Bytes a prefill call must move at least once: x, g in and y out (io
    dtype), segment_pos, the carried states read and written, and the
    parameters read once."""
    e = 2 if w.io == "bf16" else 4
    B, T, D = w.B, w.T, w.D
    act = 3 * B * T * D * e + 4 * B * T
    state = 2 * (B * D * 4 + 3 * B * D * e)
    params = 2 * (D // HEAD) * HEAD * HEAD * e + (4 + 1 + 1 + 1 + 1) * D * 4
    return act + state + params


def decode_step_bytes(w: Workload) -> int:
    """Bytes one batched decode step must move: x, g, y [B,D]; segment_pos [B];
    h [B,D] fp32 read and written; conv state [B,3,D] read and written (the
    fixed oldest-first layout rewrites all three rows); gate weights and the
    fp32 per-channel parameters read once."""
    e = 2
    B, D = w.B, w.D
    return (3 * B * D * e + 4 * B + 2 * B * D * 4 + 2 * 3 * B * D * e
            + 2 * (D // HEAD) * HEAD * HEAD * e + 8 * D * 4)


def gate_flops(w: Workload, tokens: Optional[int] = None) -> int:
    """Dense-contraction flops of the two block-diagonal gate projections."""
    n = w.tokens if tokens is None else tokens
    return 2 * 2 * n * w.D * HEAD


def generate_block(w: Workload) -> dict:
    """Inputs of the whole recurrent block for workload ``w``: everything
    ``generate(w)`` draws (the core's parameters, segment positions and initial
    states; its x and g are not block inputs), plus, from
    ``default_rng((seed, 1))`` in this order:
      u [B,T,D]                   ~ N(0, 1)          bf16 (the block input)
      W_lin_x, W_lin_y, W_out [D,D] ~ N(0, 1/D)      bf16 (torch Linear init scale)
      b_lin_x, b_lin_y, b_out [D]   ~ N(0, 0.1)      fp32
    """
    inp = generate(w)
    rng = np.random.default_rng((w.seed, 1))
    B, T, D = w.B, w.T, w.D
    inp["u"] = round_bf16(rng.standard_normal((B, T, D), dtype=np.float32))
    for name in ("lin_x", "lin_y", "out"):
        inp[f"W_{name}"] = round_bf16((rng.standard_normal((D, D)) / np.sqrt(D)).astype(np.float32))
        inp[f"b_{name}"] = (np.sqrt(0.1) * rng.standard_normal(D)).astype(np.float32)
    return inp


def block_gemm_flops(w: Workload) -> int:
    """Dense flops of the block's three D x D projections over its tokens."""
    return 3 * 2 * w.tokens * w.D * w.D


MLP_EXPANSION = 3  # MLP width 3 D (7680 for D = 2560)


def generate_residual_block(w: Workload) -> dict:
    """Inputs of the whole recurrent residual block: ``generate_block(w)`` plus,
    from ``default_rng((seed, 2))`` in this order:
      w_temporal_norm, w_channel_norm [D] ~ 1 + N(0, 0.01)   fp32 (RMSNorm scales)
      W_gate, W_up [F, D] ~ N(0, 1/D), b_gate, b_up [F] ~ N(0, 0.1)
      W_down [D, F] ~ N(0, 1/F),      b_down [D]       ~ N(0, 0.1)
    with F = 3 D (bf16 weights, fp32 biases)."""
    inp = generate_block(w)
    rng = np.random.default_rng((w.seed, 2))
    D = w.D
    F = MLP_EXPANSION * D
    inp["w_temporal_norm"] = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    inp["w_channel_norm"] = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    inp["W_gate"] = round_bf16((rng.standard_normal((F, D)) / np.sqrt(D)).astype(np.float32))
    inp["b_gate"] = (np.sqrt(0.1) * rng.standard_normal(F)).astype(np.float32)
    inp["W_up"] = round_bf16((rng.standard_normal((F, D)) / np.sqrt(D)).astype(np.float32))
    inp["b_up"] = (np.sqrt(0.1) * rng.standard_normal(F)).astype(np.float32)
    inp["W_down"] = round_bf16((rng.standard_normal((D, F)) / np.sqrt(F)).astype(np.float32))
    inp["b_down"] = (np.sqrt(0.1) * rng.standard_normal(D)).astype(np.float32)
    return inp


def residual_block_gemm_flops(w: Workload) -> int:
    """Dense flops of the residual block: three D x D projections and the
    MLP's three D x 3D ones."""
    F = MLP_EXPANSION * w.D
    return 2 * w.tokens * (3 * w.D * w.D + 3 * w.D * F)


def generate_mqa(w: Workload) -> dict:
    """Inputs of the local MQA temporal block, from ``default_rng((seed, 3))``
    in this order:
      segpos [B, T]   as ``segment_positions`` (the workload's documents)
      u [B, T, D]     ~ N(0, 1)                 bf16 values
      W_q [D, D], W_k [256, D], W_v [256, D], W_o [D, D] ~ N(0, 1/D)  bf16
      b_o [D]         ~ N(0, 0.1)               fp32
    With these scales q and k have unit-variance entries and the scaled scores
    q.k / 16 are about N(0, 1)."""
    rng = np.random.default_rng((w.seed, 3))
    B, T, D = w.B, w.T, w.D
    seg = segment_positions(rng, w)
    u = round_bf16(rng.standard_normal((B, T, D), dtype=np.float32))

    def weight(n, k):
        return round_bf16((rng.standard_normal((n, k), dtype=np.float32) / np.sqrt(k)).astype(np.float32))
    W_q, W_k, W_v, W_o = weight(D, D), weight(HEAD, D), weight(HEAD, D), weight(D, D)
    b_o = (np.sqrt(0.1) * rng.standard_normal(D)).astype(np.float32)
    return {"u": u, "W_q": W_q, "W_k": W_k, "W_v": W_v, "W_o": W_o, "b_o": b_o, "segpos": seg}


def generate_mqa_residual(w: Workload) -> dict:
    """Inputs of the residual block with local MQA: ``generate_mqa(w)`` plus,
    from ``default_rng((seed, 5))`` in this order, the RMSNorm scales and the
    MLP drawn as in ``generate_residual_block`` (F = 3 D)."""
    inp = generate_mqa(w)
    rng = np.random.default_rng((w.seed, 5))
    D = w.D
    F = MLP_EXPANSION * D
    inp["w_temporal_norm"] = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    inp["w_channel_norm"] = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    inp["W_gate"] = round_bf16((rng.standard_normal((F, D)) / np.sqrt(D)).astype(np.float32))
    inp["b_gate"] = (np.sqrt(0.1) * rng.standard_normal(F)).astype(np.float32)
    inp["W_up"] = round_bf16((rng.standard_normal((F, D)) / np.sqrt(D)).astype(np.float32))
    inp["b_up"] = (np.sqrt(0.1) * rng.standard_normal(F)).astype(np.float32)
    inp["W_down"] = round_bf16((rng.standard_normal((D, F)) / np.sqrt(F)).astype(np.float32))
    inp["b_down"] = (np.sqrt(0.1) * rng.standard_normal(D)).astype(np.float32)
    return inp
