"""float64 CPU oracle of the local sliding-window MQA temporal block --
TEST INFRASTRUCTURE (only tests/, the smoke check and the benchmark's
CPU-baseline leg may import it; the product path never does).

What it computes, from "Gemma explained: RecurrentGemma architecture", the
RecurrentGemmaSdpaAttention printout (q_proj Linear(2560, 2560, bias=False),
k_proj and v_proj Linear(2560, 256, bias=False), o_proj Linear(2560, 2560,
bias=True), rotary_emb) and section "Residual block with local MQA" (10 query
heads of 256 share one key/value head of 256; local sliding-window attention
lets each position attend only a fixed number of past tokens; the window is
2k tokens, section "Local attention window size"; RoPE as in the base Gemma
model).

Readings where the pages are silent (stated here and in the design notes):
  * RoPE: the rotate-half form on the full head dimension, frequencies
    base^(-2i/d) for i < d/2 with base 10000, rotating the pairs
    (x[i], x[i + d/2]); the position of a token is its position inside its
    document (segment_pos), so a document starts at position 0.
  * Scores are scaled by 1/sqrt(d) (d = 256) before the softmax.
  * Query t attends key s when t - W < s <= t (W = 2048, itself included) and
    s lies in t's document (s >= t - segment_pos[t]).  A prefill sees the keys
    of its own tokens only: a document that began before the first token
    (segment_pos[t] > t) attends from token 0.
  * In bf16 I/O every tensor between layers (q, k, v after RoPE, the
    attention output, the block output) is bf16: rounded once, here as on the
    GPU.
"""
from __future__ import annotations

import numpy as np

from oracle import block

HEAD = 256
WINDOW = 2048
ROPE_BASE = 10000.0


def rope(x, pos, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate-half RoPE of x [..., T, n, d] (or [..., T, d]) at positions pos
    [..., T]: pairs (x[i], x[i + d/2]) rotated by pos * base^(-2i/d)."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    half = d // 2
    inv = base ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = np.asarray(pos, np.float64)[..., None] * inv          # [..., T, half]
    if x.ndim == ang.ndim + 1:                                   # a head axis between T and d
        ang = ang[..., None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention(q, k, v, segpos, window: int = WINDOW) -> np.ndarray:
    """Local MQA: q [B, T, H, d], k and v [B, T, d], segpos [B, T] ->
    [B, T, H, d].  Query t attends keys s with t - window < s <= t inside t's
    document, scores scaled by 1/sqrt(d), softmax over those keys."""
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    B, T, H, d = q.shape
    out = np.empty_like(q)
    idx = np.arange(T)
    for b in range(B):
        start = idx - np.asarray(segpos[b], np.int64)              # document start of each query
        lo = np.maximum(np.maximum(start, idx - window + 1), 0)    # keys of this call only
        for t in range(T):
            ks = k[b, lo[t]:t + 1]                                  # [n, d]
            vs = v[b, lo[t]:t + 1]
            sc = q[b, t] @ ks.T / np.sqrt(d)                        # [H, n]
            sc = sc - sc.max(axis=1, keepdims=True)
            p = np.exp(sc)
            out[b, t] = (p / p.sum(axis=1, keepdims=True)) @ vs
    return out


def attention_rows(q, k, v, segpos, rows, window: int = WINDOW) -> np.ndarray:
    """attention() for the query rows ``rows`` [(b, t), ...] only: [len(rows), H, d],
    so that a sample of rows of a large case costs only those rows."""
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    d = q.shape[-1]
    out = []
    for b, t in rows:
        lo = max(t - int(segpos[b][t]), t - window + 1, 0)
        sc = q[b, t] @ k[b, lo:t + 1].T / np.sqrt(d)                # [H, n]
        p = np.exp(sc - sc.max(axis=1, keepdims=True))
        out.append((p / p.sum(axis=1, keepdims=True)) @ v[b, lo:t + 1])
    return np.stack(out)


def _attend(n, W_q, W_k, W_v, segpos, window, rnd) -> dict:
    """q_proj, k_proj, v_proj of n [B, T, D], RoPE on q and k, local attention;
    each result rounded by ``rnd``."""
    B, T, D = n.shape
    H = np.asarray(W_q).shape[0] // HEAD
    q = rnd(rope(block.linear(n, W_q).reshape(B, T, H, HEAD), segpos))
    k = rnd(rope(block.linear(n, W_k), segpos))
    v = rnd(block.linear(n, W_v))
    a = rnd(attention(q, k, v, segpos, window))
    return {"q": q, "k": k, "v": v, "a": a}


def mqa_block(u, W_q, W_k, W_v, W_o, b_o, segpos, window: int = WINDOW, round_io: bool = True) -> dict:
    """The local MQA temporal block over u [B, T, D]: projections (q_proj,
    k_proj, v_proj without bias), RoPE on q and k, local attention, o_proj
    with bias.  Returns out and the intermediates q, k, v (after RoPE) and a
    (the attention output)."""
    rnd = block.round_bf16 if round_io else (lambda a: np.asarray(a, np.float64))
    u = np.asarray(u, np.float64)
    B, T, D = u.shape
    r = _attend(u, W_q, W_k, W_v, segpos, window, rnd)
    r["out"] = rnd(block.linear(r["a"].reshape(B, T, -1), W_o, b_o))
    return r


def mqa_residual_block(u, w_temporal_norm, W_q, W_k, W_v, W_o, b_o, segpos, w_channel_norm, W_gate, b_gate, W_up,
                       b_up, W_down, b_down, eps: float = 1e-6, window: int = WINDOW) -> dict:
    """The residual block with local MQA ("Residual block with local MQA" and
    the decoder-layer printout): h = u + o_proj(MQA(RMSNorm(u))), out = h +
    MLP(RMSNorm(h)); every layer's output a bf16 tensor (the residual adds
    belong to the projection before them, rounded once with it).  Returns out
    and the intermediates n (normalised u) and h."""
    rnd = block.round_bf16
    u = np.asarray(u, np.float64)
    B, T, D = u.shape
    n = rnd(block.rmsnorm(u, w_temporal_norm, eps))
    a = _attend(n, W_q, W_k, W_v, segpos, window, rnd)["a"]
    h = rnd(block.linear(a.reshape(B, T, -1), W_o, b_o) + u)
    n2 = rnd(block.rmsnorm(h, w_channel_norm, eps))
    m = rnd(block.gelu_tanh(block.linear(n2, W_gate, b_gate)) * block.linear(n2, W_up, b_up))
    out = rnd(block.linear(m, W_down, b_down) + h)
    return {"out": out, "n": n, "h": h}
