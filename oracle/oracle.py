"""float64 CPU oracle of the RG-LRU recurrent-block core -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this module.  The product path (``lm_causal_depthwise_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``rglru_oracle.c`` (plain C, float64, loops written in
the order of the definitions; see its header for the equations and the
passages they come from).  This module only compiles that file with gcc,
marshals numpy arrays into it, and evaluates a subset of independent
(batch row, head) units when a full-size problem is too large to run whole:
heads never mix (depthwise conv, block-diagonal gates, per-channel scan) and
batch rows never mix, so a unit is exactly a sub-problem with B=1, D=256.

Decode is the same routine with T=1; there is no separate code path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HEAD = 256
C_DEFAULT = 8.0

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rglru_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "librglru_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (IEEE arithmetic: no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            lib.rglru_oracle_prefill.restype = ctypes.c_int
            lib.rglru_oracle_prefill.argtypes = (
                [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double]
                + [dp] * 8 + [dp, ip] + [dp] * 3 + [dp] * 5 + [ctypes.c_int, ctypes.c_int])
            lib.rglru_oracle_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def threads() -> int:
    """Number of OpenMP threads the oracle uses by default (host cores)."""
    return int(_load().rglru_oracle_threads())


def _f64(a, shape):
    arr = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if arr.shape != tuple(shape):
        raise ValueError(f"expected shape {tuple(shape)}, got {arr.shape}")
    return arr


def _ptr(a):
    if a is None:
        return None
    if a.dtype == np.int32:
        return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def prefill(x, g, conv_w, conv_b, W_a, b_a, W_x, b_x, lam, segpos,
            conv_state, h_state, c: float = C_DEFAULT, trace: bool = False,
            nthreads: int = 0, gate_bf16: bool = False):
    """Run the block core over [B,T,D] inputs in float64.

    ``gate_bf16=True`` rounds the conv output to bf16 where it enters the gate
    projections (the operand precision of the tensor-core gate GEMM in bf16
    I/O mode); everything else stays float64.

    Inputs may be any float dtype (they are widened exactly to float64).
    Returns a dict with ``y`` [B,T,D], ``conv_state`` [B,3,D] and ``h_state``
    [B,D] (new arrays; the inputs are not modified) and, with ``trace=True``,
    the per-element intermediates ``xc``, ``r``, ``i``, ``a``, ``h``.
    """
    x = np.asarray(x)
    if x.ndim != 3:
        raise ValueError("x must be [B,T,D]")
    B, T, D = x.shape
    if D % HEAD:
        raise ValueError("D must be a multiple of 256")
    H = D // HEAD
    x = _f64(x, (B, T, D))
    g = _f64(g, (B, T, D))
    conv_w = _f64(conv_w, (4, D))
    conv_b = _f64(conv_b, (D,))
    W_a = _f64(W_a, (H, HEAD, HEAD))
    b_a = _f64(b_a, (D,))
    W_x = _f64(W_x, (H, HEAD, HEAD))
    b_x = _f64(b_x, (D,))
    lam = _f64(lam, (D,))
    segpos = np.ascontiguousarray(np.asarray(segpos, dtype=np.int32))
    if segpos.shape != (B, T):
        raise ValueError("segpos must be [B,T]")
    cs = _f64(conv_state, (B, 3, D)).copy()
    hs = _f64(h_state, (B, D)).copy()
    y = np.empty((B, T, D), dtype=np.float64)
    tr = {k: (np.empty((B, T, D), dtype=np.float64) if trace else None)
          for k in ("xc", "r", "i", "a", "h")}
    rc = _load().rglru_oracle_prefill(
        B, T, D, float(c), _ptr(x), _ptr(g), _ptr(conv_w), _ptr(conv_b), _ptr(W_a),
        _ptr(b_a), _ptr(W_x), _ptr(b_x), _ptr(lam), _ptr(segpos), _ptr(cs), _ptr(hs),
        _ptr(y), _ptr(tr["xc"]), _ptr(tr["r"]), _ptr(tr["i"]), _ptr(tr["a"]),
        _ptr(tr["h"]), int(nthreads), 1 if gate_bf16 else 0)
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    out = {"y": y, "conv_state": cs, "h_state": hs}
    if trace:
        out.update(tr)
    return out


def decode_step(x, g, conv_w, conv_b, W_a, b_a, W_x, b_x, lam, segpos,
                conv_state, h_state, c: float = C_DEFAULT, nthreads: int = 0):
    """One token per sequence: x, g [B,D], segpos [B].  The prefill routine with T=1."""
    x = np.asarray(x)
    g = np.asarray(g)
    out = prefill(x[:, None, :], g[:, None, :], conv_w, conv_b, W_a, b_a, W_x, b_x, lam,
                  np.asarray(segpos).reshape(-1, 1), conv_state, h_state, c=c,
                  nthreads=nthreads)
    out["y"] = out["y"][:, 0, :]
    return out


def unit_inputs(inp: dict, b: int, head: int, t_end: int | None = None) -> dict:
    """Slice the (b, head) sub-problem (B=1, D=256) out of a full input dict.

    ``inp`` holds the arrays named as in :func:`prefill` (``x``, ``g``,
    ``conv_w``, ``conv_b``, ``W_a``, ``b_a``, ``W_x``, ``b_x``, ``lam``,
    ``segpos``, ``conv_state``, ``h_state``).  ``t_end`` truncates time to the
    first ``t_end`` tokens (outputs at those tokens do not depend on later ones).
    """
    s = slice(head * HEAD, (head + 1) * HEAD)
    te = slice(0, t_end)
    return dict(
        x=np.asarray(inp["x"][b:b + 1, te, s]),
        g=np.asarray(inp["g"][b:b + 1, te, s]),
        conv_w=np.asarray(inp["conv_w"][:, s]), conv_b=np.asarray(inp["conv_b"][s]),
        W_a=np.asarray(inp["W_a"][head:head + 1]), b_a=np.asarray(inp["b_a"][s]),
        W_x=np.asarray(inp["W_x"][head:head + 1]), b_x=np.asarray(inp["b_x"][s]),
        lam=np.asarray(inp["lam"][s]), segpos=np.asarray(inp["segpos"][b:b + 1, te]),
        conv_state=np.asarray(inp["conv_state"][b:b + 1, :, s]),
        h_state=np.asarray(inp["h_state"][b:b + 1, s]),
    )


def prefill_unit(inp: dict, b: int, head: int, t_end: int | None = None,
                 c: float = C_DEFAULT, nthreads: int = 0) -> dict:
    """Oracle outputs of one (b, head) unit: y [T,256], conv_state [3,256], h_state [256]."""
    u = unit_inputs(inp, b, head, t_end)
    out = prefill(**u, c=c, nthreads=nthreads)
    return {"y": out["y"][0], "conv_state": out["conv_state"][0], "h_state": out["h_state"][0]}
