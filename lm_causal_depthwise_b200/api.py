"""Python binding of librglru (include/rglru.h): argument marshalling only.

Every step of the block core runs in the CUDA library; this module checks
tensor dtypes, shapes, devices and contiguity, passes raw pointers and the
current CUDA stream through ctypes, and turns a non-OK status into an
exception.  PyTorch provides device memory and streams, nothing else.  If
the library is missing or cannot be loaded, every call raises: there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librglru.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(6)
IO_F32, IO_BF16 = 0, 1

SYMBOLS = ("rglru_version", "rglru_status_string", "rglru_workspace_size", "rglru_prefill",
           "rglru_simt_workspace_size", "rglru_prefill_simt", "rglru_decode_workspace_size",
           "rglru_decode_step", "rglru_get_device_status", "rglru_debug_suppress_publish",
           "rglru_prefill_noalloc", "rglru_prefill_host_staging_size", "rglru_prefill_host",
           "rglru_linear_workspace_size", "rglru_linear", "rglru_linear_pair", "rglru_linear_residual",
           "rglru_linear_geglu", "rglru_recurrent_block_workspace_size", "rglru_recurrent_block_prefill",
           "rglru_rmsnorm", "rglru_residual_block_workspace_size", "rglru_residual_block_prefill",
           "rglru_mqa_vt_size", "rglru_mqa_rope", "rglru_mqa_attention", "rglru_mqa_block_workspace_size",
           "rglru_mqa_block_prefill", "rglru_mqa_decode_workspace_size", "rglru_mqa_decode_step",
           "rglru_mqa_residual_block_workspace_size", "rglru_mqa_residual_block_prefill", "rglru_carry_scan")

_lib = None


class RGLRUError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load librglru.so (built in-tree by lm_causal_depthwise_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing; build it with "
                           "`python -m lm_causal_depthwise_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    prefill_args = [i, i, i, i] + [vp] * 14 + [sz, vp]
    decode_args = [i, i, i] + [vp] * 14 + [sz, vp]
    lib.rglru_version.restype = i
    lib.rglru_version.argtypes = []
    lib.rglru_status_string.restype = ctypes.c_char_p
    lib.rglru_status_string.argtypes = [i]
    for n in ("rglru_workspace_size", "rglru_simt_workspace_size"):
        getattr(lib, n).restype = sz
        getattr(lib, n).argtypes = [i, i, i, i]
    lib.rglru_decode_workspace_size.restype = sz
    lib.rglru_decode_workspace_size.argtypes = [i, i, i]
    for n in ("rglru_prefill", "rglru_prefill_simt"):
        getattr(lib, n).restype = i
        getattr(lib, n).argtypes = prefill_args
    lib.rglru_decode_step.restype = i
    lib.rglru_decode_step.argtypes = decode_args
    lib.rglru_get_device_status.restype = i
    lib.rglru_get_device_status.argtypes = [vp, vp]
    lib.rglru_debug_suppress_publish.restype = i
    lib.rglru_debug_suppress_publish.argtypes = [vp, i, vp]
    lib.rglru_prefill_noalloc.restype = i
    lib.rglru_prefill_noalloc.argtypes = [i, i, i, i] + [vp] * 13 + [vp]
    lib.rglru_prefill_host_staging_size.restype = sz
    lib.rglru_prefill_host_staging_size.argtypes = [i, i, i, i, i]
    lib.rglru_prefill_host.restype = i
    lib.rglru_prefill_host.argtypes = [i, i, i, i] + [vp] * 13 + [i, vp, sz, vp, sz, vp]
    lib.rglru_linear_workspace_size.restype = sz
    lib.rglru_linear_workspace_size.argtypes = []
    lib.rglru_linear.restype = i
    lib.rglru_linear.argtypes = [i, i, i] + [vp] * 5 + [sz, vp]
    lib.rglru_linear_pair.restype = i
    lib.rglru_linear_pair.argtypes = [i, i, i] + [vp] * 8 + [sz, vp]
    lib.rglru_linear_residual.restype = i
    lib.rglru_linear_residual.argtypes = [i, i, i] + [vp] * 6 + [sz, vp]
    lib.rglru_linear_geglu.restype = i
    lib.rglru_linear_geglu.argtypes = [i, i, i] + [vp] * 7 + [sz, vp]
    lib.rglru_recurrent_block_workspace_size.restype = sz
    lib.rglru_recurrent_block_workspace_size.argtypes = [i, i, i]
    lib.rglru_recurrent_block_prefill.restype = i
    lib.rglru_recurrent_block_prefill.argtypes = [i, i, i] + [vp] * 19 + [sz, vp]
    lib.rglru_rmsnorm.restype = i
    lib.rglru_rmsnorm.argtypes = [i, i, vp, vp, ctypes.c_float, vp, vp]
    lib.rglru_residual_block_workspace_size.restype = sz
    lib.rglru_residual_block_workspace_size.argtypes = [i, i, i, i]
    lib.rglru_residual_block_prefill.restype = i
    lib.rglru_residual_block_prefill.argtypes = [i, i, i, i] + [vp] * 25 + [ctypes.c_float, vp, vp, sz, vp]
    lib.rglru_mqa_vt_size.restype = sz
    lib.rglru_mqa_vt_size.argtypes = [i, i]
    lib.rglru_mqa_rope.restype = i
    lib.rglru_mqa_rope.argtypes = [i, i, i, vp, vp, vp, vp]
    lib.rglru_mqa_attention.restype = i
    lib.rglru_mqa_attention.argtypes = [i, i, i, i] + [vp] * 5 + [sz, vp]
    lib.rglru_mqa_block_workspace_size.restype = sz
    lib.rglru_mqa_block_workspace_size.argtypes = [i, i, i]
    lib.rglru_mqa_block_prefill.restype = i
    lib.rglru_mqa_block_prefill.argtypes = [i, i, i, i] + [vp] * 7 + [sz, vp]
    lib.rglru_mqa_decode_workspace_size.restype = sz
    lib.rglru_mqa_decode_workspace_size.argtypes = [i, i, i]
    lib.rglru_mqa_decode_step.restype = i
    lib.rglru_mqa_decode_step.argtypes = [i, i, i] + [vp] * 6 + [sz, vp]
    lib.rglru_mqa_residual_block_workspace_size.restype = sz
    lib.rglru_mqa_residual_block_workspace_size.argtypes = [i, i, i, i]
    lib.rglru_mqa_residual_block_prefill.restype = i
    lib.rglru_mqa_residual_block_prefill.argtypes = [i, i, i, i, i] + [vp] * 13 + [ctypes.c_float, vp, vp, sz, vp]
    lib.rglru_carry_scan.restype = i
    lib.rglru_carry_scan.argtypes = [i, i, i] + [vp] * 4 + [vp]
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().rglru_status_string(int(status)).decode()


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return IO_BF16
    if t.dtype == torch.float32:
        return IO_F32
    raise TypeError(f"io tensors must be bfloat16 or float32, got {t.dtype}")


@dataclass
class Params:
    """Block parameters on the device.  conv_w [4,D], conv_b/b_a/b_x/lam [D]
    are fp32; W_a, W_x [H,256,256] are in the io dtype."""
    conv_w: torch.Tensor
    conv_b: torch.Tensor
    W_a: torch.Tensor
    b_a: torch.Tensor
    W_x: torch.Tensor
    b_x: torch.Tensor
    lam: torch.Tensor

    @staticmethod
    def from_arrays(inp: dict, io_dtype: torch.dtype, device="cuda") -> "Params":
        def f32(a):
            return torch.as_tensor(a, dtype=torch.float32).to(device).contiguous()

        def io(a):
            return torch.as_tensor(a, dtype=torch.float32).to(device).to(io_dtype).contiguous()
        return Params(f32(inp["conv_w"]), f32(inp["conv_b"]), io(inp["W_a"]), f32(inp["b_a"]),
                      io(inp["W_x"]), f32(inp["b_x"]), f32(inp["lam"]))


def _ptr(t: torch.Tensor):
    return ctypes.c_void_p(t.data_ptr())


def _check(t: torch.Tensor, name: str, shape, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(device) -> ctypes.c_void_p:
    """The current stream of ``device``; every call that enqueues work takes
    its device from its tensors, so host tensors stop here, before the
    library sees a host pointer as device memory."""
    device = torch.device(device)
    if device.type != "cuda":
        raise ValueError(f"the tensors must be CUDA tensors, got device {device}")
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def workspace_size(B: int, T: int, D: int, io_dtype: torch.dtype, simt: bool = False) -> int:
    dt = IO_BF16 if io_dtype == torch.bfloat16 else IO_F32
    fn = load().rglru_simt_workspace_size if simt else load().rglru_workspace_size
    n = int(fn(B, T, D, dt))
    if n == 0:
        raise RGLRUError(ERR_INVALID_ARG, "workspace_size")
    return n


def decode_workspace_size(B: int, D: int, io_dtype: torch.dtype) -> int:
    dt = IO_BF16 if io_dtype == torch.bfloat16 else IO_F32
    n = int(load().rglru_decode_workspace_size(B, D, dt))
    if n == 0:
        raise RGLRUError(ERR_INVALID_ARG, "decode_workspace_size")
    return n


def new_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled device workspace (the valid initial state)."""
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def _common(x, g, p: Params, segpos, conv_state, h_state, y, lead):
    dev = x.device
    dt = _dt(x)
    D = x.shape[-1]
    H = D // 256
    _check(g, "gate_branch", x.shape, x.dtype, dev)
    _check(x, "x", x.shape, x.dtype, dev)
    _check(p.conv_w, "conv_w", (4, D), torch.float32, dev)
    for n in ("conv_b", "b_a", "b_x", "lam"):
        _check(getattr(p, n), n, (D,), torch.float32, dev)
    _check(p.W_a, "W_a", (H, 256, 256), x.dtype, dev)
    _check(p.W_x, "W_x", (H, 256, 256), x.dtype, dev)
    _check(segpos, "segment_pos", lead, torch.int32, dev)
    B = x.shape[0]
    _check(conv_state, "conv_state", (B, 3, D), x.dtype, dev)
    _check(h_state, "h_state", (B, D), torch.float32, dev)
    if y is None:
        y = torch.empty_like(x)
    _check(y, "y", x.shape, x.dtype, dev)
    return dt, y


def prefill(x, gate_branch, p: Params, segment_pos, conv_state, h_state, workspace=None,
            y=None, simt: bool = False) -> torch.Tensor:
    """y = block core over x, gate_branch [B,T,D]; conv_state [B,3,D] and
    h_state [B,D] are updated in place.  Enqueued on the current stream."""
    if x.dim() != 3:
        raise ValueError("x must be [B,T,D]")
    B, T, D = x.shape
    dt, y = _common(x, gate_branch, p, segment_pos, conv_state, h_state, y, (B, T))
    need = workspace_size(B, T, D, x.dtype, simt=simt)
    if workspace is None:
        workspace = new_workspace(need, x.device)
    if workspace.numel() * workspace.element_size() < need:
        raise RGLRUError(ERR_WORKSPACE, "prefill")
    fn = load().rglru_prefill_simt if simt else load().rglru_prefill
    st = fn(B, T, D, dt, _ptr(x), _ptr(gate_branch), _ptr(p.conv_w), _ptr(p.conv_b), _ptr(p.W_a),
            _ptr(p.b_a), _ptr(p.W_x), _ptr(p.b_x), _ptr(p.lam), _ptr(segment_pos),
            _ptr(conv_state), _ptr(h_state), _ptr(y), _ptr(workspace),
            ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(x.device))
    if st != OK:
        raise RGLRUError(st, "rglru_prefill_simt" if simt else "rglru_prefill")
    return y


def prefill_noalloc(x, gate_branch, p: Params, segment_pos, conv_state, h_state, y=None) -> torch.Tensor:
    """rglru_prefill_noalloc: the bf16 prefill with the library's own fixed
    scratch (no workspace, nothing allocated by the library).  Same tensors
    and semantics as :func:`prefill`; shapes whose workspace would exceed the
    library's 8 MiB scratch raise RGLRUError(ERR_WORKSPACE)."""
    if x.dim() != 3:
        raise ValueError("x must be [B,T,D]")
    B, T, D = x.shape
    dt, y = _common(x, gate_branch, p, segment_pos, conv_state, h_state, y, (B, T))
    st = load().rglru_prefill_noalloc(
        B, T, D, dt, _ptr(x), _ptr(gate_branch), _ptr(p.conv_w), _ptr(p.conv_b), _ptr(p.W_a),
        _ptr(p.b_a), _ptr(p.W_x), _ptr(p.b_x), _ptr(p.lam), _ptr(segment_pos), _ptr(conv_state),
        _ptr(h_state), _ptr(y), _stream(x.device))
    if st != OK:
        raise RGLRUError(st, "rglru_prefill_noalloc")
    return y


def decode_step(x, gate_branch, p: Params, segment_pos, conv_state, h_state, workspace=None,
                y=None) -> torch.Tensor:
    """One token per sequence: x, gate_branch [B,D]; segment_pos [B]."""
    if x.dim() != 2:
        raise ValueError("x must be [B,D]")
    B, D = x.shape
    dt, y = _common(x, gate_branch, p, segment_pos, conv_state, h_state, y, (B,))
    need = decode_workspace_size(B, D, x.dtype)
    if workspace is None:
        workspace = new_workspace(need, x.device)
    if workspace.numel() * workspace.element_size() < need:
        raise RGLRUError(ERR_WORKSPACE, "decode_step")
    st = load().rglru_decode_step(
        B, D, dt, _ptr(x), _ptr(gate_branch), _ptr(p.conv_w), _ptr(p.conv_b), _ptr(p.W_a),
        _ptr(p.b_a), _ptr(p.W_x), _ptr(p.b_x), _ptr(p.lam), _ptr(segment_pos), _ptr(conv_state),
        _ptr(h_state), _ptr(y), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(x.device))
    if st != OK:
        raise RGLRUError(st, "rglru_decode_step")
    return y


def device_status(workspace: torch.Tensor) -> int:
    """Synchronise the current stream and read (and clear) the device status word."""
    return int(load().rglru_get_device_status(_ptr(workspace), _stream(workspace.device)))


def debug_suppress_publish(workspace: torch.Tensor, unit: int) -> None:
    st = load().rglru_debug_suppress_publish(_ptr(workspace), int(unit), _stream(workspace.device))
    if st != OK:
        raise RGLRUError(st, "rglru_debug_suppress_publish")


def prefill_host_staging_size(B: int, T: int, D: int, io_dtype: torch.dtype, rows_per_chunk: int) -> int:
    dt = IO_BF16 if io_dtype == torch.bfloat16 else IO_F32
    n = int(load().rglru_prefill_host_staging_size(B, T, D, dt, rows_per_chunk))
    if n == 0:
        raise RGLRUError(ERR_INVALID_ARG, "prefill_host_staging_size")
    return n


def prefill_host(x_host, gate_branch_host, p: Params, segment_pos_host, conv_state, h_state, y_host=None,
                 rows_per_chunk: int = 1, staging=None, workspace=None) -> torch.Tensor:
    """rglru_prefill_host: x_host, gate_branch_host [B,T,D], segment_pos_host
    [B,T] and y_host are CPU tensors (page-locked for overlapped copies);
    the parameters, conv_state, h_state, staging and workspace are on the
    device.  Enqueued on the current stream of the states' device: y_host is
    complete once that stream has finished the call (synchronise before
    reading it)."""
    if x_host.dim() != 3:
        raise ValueError("x_host must be [B,T,D]")
    B, T, D = x_host.shape
    dev = conv_state.device
    for t, n, shape in ((x_host, "x_host", (B, T, D)), (gate_branch_host, "gate_branch_host", (B, T, D)),
                        (segment_pos_host, "segment_pos_host", (B, T))):
        _check(t, n, shape, torch.int32 if n == "segment_pos_host" else x_host.dtype, torch.device("cpu"))
    if y_host is None:
        y_host = torch.empty(tuple(x_host.shape), dtype=x_host.dtype, pin_memory=x_host.is_pinned())
    _check(y_host, "y_host", (B, T, D), x_host.dtype, torch.device("cpu"))
    dt = _dt(x_host)
    H = D // 256
    _check(p.conv_w, "conv_w", (4, D), torch.float32, dev)
    for n in ("conv_b", "b_a", "b_x", "lam"):
        _check(getattr(p, n), n, (D,), torch.float32, dev)
    _check(p.W_a, "W_a", (H, 256, 256), x_host.dtype, dev)
    _check(p.W_x, "W_x", (H, 256, 256), x_host.dtype, dev)
    _check(conv_state, "conv_state", (B, 3, D), x_host.dtype, dev)
    _check(h_state, "h_state", (B, D), torch.float32, dev)
    need_st = prefill_host_staging_size(B, T, D, x_host.dtype, rows_per_chunk)
    if staging is None:
        staging = torch.empty(need_st, dtype=torch.uint8, device=dev)
    need_ws = workspace_size(min(B, rows_per_chunk), T, D, x_host.dtype)
    if workspace is None:
        workspace = new_workspace(need_ws, dev)
    st = load().rglru_prefill_host(B, T, D, dt, _ptr(x_host), _ptr(gate_branch_host), _ptr(p.conv_w), _ptr(p.conv_b),
                                   _ptr(p.W_a), _ptr(p.b_a), _ptr(p.W_x), _ptr(p.b_x), _ptr(p.lam),
                                   _ptr(segment_pos_host), _ptr(conv_state), _ptr(h_state), _ptr(y_host),
                                   int(rows_per_chunk), _ptr(staging),
                                   ctypes.c_size_t(staging.numel() * staging.element_size()), _ptr(workspace),
                                   ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(dev))
    if st != OK:
        raise RGLRUError(st, "rglru_prefill_host")
    return y_host


# ----------------------------------------------------------------------------- projections and the block

def linear_workspace(device="cuda") -> torch.Tensor:
    """A zero-filled workspace for the rglru_linear* calls (the device status header)."""
    return new_workspace(int(load().rglru_linear_workspace_size()), device)


def _lin_common(A, W, name):
    if A.dim() != 2 or W.dim() != 2:
        raise ValueError(f"{name}: A must be [M, K] and W [N, K]")
    M, K = A.shape
    N = W.shape[0]
    _check(A, "A", (M, K), torch.bfloat16, A.device)
    _check(W, "W", (N, K), torch.bfloat16, A.device)
    return M, N, K


def _bias(b, N, dev, name):
    if b is None:
        return ctypes.c_void_p(None)
    _check(b, name, (N,), torch.float32, dev)
    return _ptr(b)


def _ws(workspace, dev):
    if workspace is None:
        workspace = linear_workspace(dev)
    return workspace, ctypes.c_size_t(workspace.numel() * workspace.element_size())


def linear(A, W, bias=None, out=None, workspace=None) -> torch.Tensor:
    """out[M, N] = A[M, K] W[N, K]^T + bias (rglru_linear, bf16 on the tensor cores)."""
    M, N, K = _lin_common(A, W, "linear")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _check(out, "out", (M, N), torch.bfloat16, A.device)
    workspace, nb = _ws(workspace, A.device)
    st = load().rglru_linear(M, N, K, _ptr(A), _ptr(W), _bias(bias, N, A.device, "bias"), _ptr(out),
                             _ptr(workspace), nb, _stream(A.device))
    if st != OK:
        raise RGLRUError(st, "rglru_linear")
    return out


def linear_pair(A, W0, b0, W1, b1, out0=None, out1=None, workspace=None):
    """(A W0^T + b0, A W1^T + b1) in one launch (rglru_linear_pair)."""
    M, N, K = _lin_common(A, W0, "linear_pair")
    _check(W1, "W1", (N, K), torch.bfloat16, A.device)
    outs = []
    for o in (out0, out1):
        if o is None:
            o = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
        _check(o, "out", (M, N), torch.bfloat16, A.device)
        outs.append(o)
    workspace, nb = _ws(workspace, A.device)
    st = load().rglru_linear_pair(M, N, K, _ptr(A), _ptr(W0), _bias(b0, N, A.device, "bias0"), _ptr(outs[0]),
                                  _ptr(W1), _bias(b1, N, A.device, "bias1"), _ptr(outs[1]), _ptr(workspace), nb,
                                  _stream(A.device))
    if st != OK:
        raise RGLRUError(st, "rglru_linear_pair")
    return outs[0], outs[1]


def linear_residual(A, W, bias, residual, out=None, workspace=None) -> torch.Tensor:
    """out = A W^T + bias + residual (rglru_linear_residual); out may be residual."""
    M, N, K = _lin_common(A, W, "linear_residual")
    _check(residual, "residual", (M, N), torch.bfloat16, A.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _check(out, "out", (M, N), torch.bfloat16, A.device)
    workspace, nb = _ws(workspace, A.device)
    st = load().rglru_linear_residual(M, N, K, _ptr(A), _ptr(W), _bias(bias, N, A.device, "bias"), _ptr(residual),
                                      _ptr(out), _ptr(workspace), nb, _stream(A.device))
    if st != OK:
        raise RGLRUError(st, "rglru_linear_residual")
    return out


def linear_geglu(A, W_gate, b_gate, W_up, b_up, out=None, workspace=None) -> torch.Tensor:
    """out = GELU_tanh(A W_gate^T + b_gate) * (A W_up^T + b_up) (rglru_linear_geglu)."""
    M, N, K = _lin_common(A, W_gate, "linear_geglu")
    _check(W_up, "W_up", (N, K), torch.bfloat16, A.device)
    _check(b_gate, "b_gate", (N,), torch.float32, A.device)
    _check(b_up, "b_up", (N,), torch.float32, A.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _check(out, "out", (M, N), torch.bfloat16, A.device)
    workspace, nb = _ws(workspace, A.device)
    st = load().rglru_linear_geglu(M, N, K, _ptr(A), _ptr(W_gate), _ptr(b_gate), _ptr(W_up), _ptr(b_up), _ptr(out),
                                   _ptr(workspace), nb, _stream(A.device))
    if st != OK:
        raise RGLRUError(st, "rglru_linear_geglu")
    return out


@dataclass
class BlockParams:
    """Projections around the core (bf16 [D, D] weights, fp32 [D] biases) and
    the core's own parameters."""
    W_lin_x: torch.Tensor
    b_lin_x: torch.Tensor
    W_lin_y: torch.Tensor
    b_lin_y: torch.Tensor
    W_out: torch.Tensor
    b_out: torch.Tensor
    core: Params

    @staticmethod
    def from_arrays(inp: dict, device="cuda") -> "BlockParams":
        def w(a):
            return torch.as_tensor(a, dtype=torch.float32).to(device).to(torch.bfloat16).contiguous()

        def f32(a):
            return torch.as_tensor(a, dtype=torch.float32).to(device).contiguous()
        return BlockParams(w(inp["W_lin_x"]), f32(inp["b_lin_x"]), w(inp["W_lin_y"]), f32(inp["b_lin_y"]),
                           w(inp["W_out"]), f32(inp["b_out"]), Params.from_arrays(inp, torch.bfloat16, device))


def recurrent_block_workspace_size(B: int, T: int, D: int) -> int:
    n = int(load().rglru_recurrent_block_workspace_size(B, T, D))
    if n == 0:
        raise RGLRUError(ERR_INVALID_ARG, "recurrent_block_workspace_size")
    return n


def recurrent_block_prefill(u, bp: BlockParams, segment_pos, conv_state, h_state, out=None,
                            workspace=None) -> torch.Tensor:
    """out = linear_out(GELU(linear_y(u)) * RG-LRU(conv(linear_x(u)))) over u [B,T,D] bf16
    (rglru_recurrent_block_prefill); conv_state and h_state are updated in place."""
    if u.dim() != 3:
        raise ValueError("u must be [B,T,D]")
    B, T, D = u.shape
    dev = u.device
    _check(u, "u", (B, T, D), torch.bfloat16, dev)
    for n in ("W_lin_x", "W_lin_y", "W_out"):
        _check(getattr(bp, n), n, (D, D), torch.bfloat16, dev)
    for n in ("b_lin_x", "b_lin_y", "b_out"):
        _check(getattr(bp, n), n, (D,), torch.float32, dev)
    p = bp.core
    _check(p.conv_w, "conv_w", (4, D), torch.float32, dev)
    for n in ("conv_b", "b_a", "b_x", "lam"):
        _check(getattr(p, n), n, (D,), torch.float32, dev)
    _check(p.W_a, "W_a", (D // 256, 256, 256), torch.bfloat16, dev)
    _check(p.W_x, "W_x", (D // 256, 256, 256), torch.bfloat16, dev)
    _check(segment_pos, "segment_pos", (B, T), torch.int32, dev)
    _check(conv_state, "conv_state", (B, 3, D), torch.bfloat16, dev)
    _check(h_state, "h_state", (B, D), torch.float32, dev)
    if out is None:
        out = torch.empty_like(u)
    _check(out, "out", (B, T, D), torch.bfloat16, dev)
    need = recurrent_block_workspace_size(B, T, D)
    if workspace is None:
        workspace = new_workspace(need, dev)
    st = load().rglru_recurrent_block_prefill(
        B, T, D, _ptr(u), _ptr(bp.W_lin_x), _ptr(bp.b_lin_x), _ptr(bp.W_lin_y), _ptr(bp.b_lin_y), _ptr(p.conv_w),
        _ptr(p.conv_b), _ptr(p.W_a), _ptr(p.b_a), _ptr(p.W_x), _ptr(p.b_x), _ptr(p.lam), _ptr(segment_pos),
        _ptr(conv_state), _ptr(h_state), _ptr(bp.W_out), _ptr(bp.b_out), _ptr(out), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(dev))
    if st != OK:
        raise RGLRUError(st, "rglru_recurrent_block_prefill")
    return out


def rmsnorm(x, weight, eps: float = 1e-6, out=None) -> torch.Tensor:
    """out = x * rsqrt(mean(x^2) + eps) * weight over the last dimension (rglru_rmsnorm)."""
    N = x.shape[-1]
    M = x.numel() // N
    _check(x, "x", x.shape, torch.bfloat16, x.device)
    _check(weight, "weight", (N,), torch.float32, x.device)
    if out is None:
        out = torch.empty_like(x)
    _check(out, "out", x.shape, torch.bfloat16, x.device)
    st = load().rglru_rmsnorm(M, N, _ptr(x), _ptr(weight), ctypes.c_float(eps), _ptr(out), _stream(x.device))
    if st != OK:
        raise RGLRUError(st, "rglru_rmsnorm")
    return out


@dataclass
class ResidualBlockParams:
    """The recurrent residual block: both RMSNorm scales, the recurrent block
    and the MLP (gate/up [F, D], down [D, F] bf16; biases fp32)."""
    w_temporal_norm: torch.Tensor
    block: BlockParams
    w_channel_norm: torch.Tensor
    W_gate: torch.Tensor
    b_gate: torch.Tensor
    W_up: torch.Tensor
    b_up: torch.Tensor
    W_down: torch.Tensor
    b_down: torch.Tensor

    @staticmethod
    def from_arrays(inp: dict, device="cuda") -> "ResidualBlockParams":
        def w(a):
            return torch.as_tensor(a, dtype=torch.float32).to(device).to(torch.bfloat16).contiguous()

        def f32(a):
            return torch.as_tensor(a, dtype=torch.float32).to(device).contiguous()
        return ResidualBlockParams(f32(inp["w_temporal_norm"]), BlockParams.from_arrays(inp, device),
                                   f32(inp["w_channel_norm"]), w(inp["W_gate"]), f32(inp["b_gate"]), w(inp["W_up"]),
                                   f32(inp["b_up"]), w(inp["W_down"]), f32(inp["b_down"]))


def residual_block_workspace_size(B: int, T: int, D: int, F: int) -> int:
    n = int(load().rglru_residual_block_workspace_size(B, T, D, F))
    if n == 0:
        raise RGLRUError(ERR_INVALID_ARG, "residual_block_workspace_size")
    return n


def residual_block_prefill(u, rp: ResidualBlockParams, segment_pos, conv_state, h_state, eps: float = 1e-6,
                           out=None, workspace=None) -> torch.Tensor:
    """The recurrent residual block over u [B,T,D] bf16 (rglru_residual_block_prefill)."""
    if u.dim() != 3:
        raise ValueError("u must be [B,T,D]")
    B, T, D = u.shape
    F = rp.W_gate.shape[0]
    dev = u.device
    _check(u, "u", (B, T, D), torch.bfloat16, dev)
    _check(rp.w_temporal_norm, "w_temporal_norm", (D,), torch.float32, dev)
    _check(rp.w_channel_norm, "w_channel_norm", (D,), torch.float32, dev)
    _check(rp.W_gate, "W_gate", (F, D), torch.bfloat16, dev)
    _check(rp.W_up, "W_up", (F, D), torch.bfloat16, dev)
    _check(rp.W_down, "W_down", (D, F), torch.bfloat16, dev)
    for n_, t in (("b_gate", rp.b_gate), ("b_up", rp.b_up)):
        _check(t, n_, (F,), torch.float32, dev)
    _check(rp.b_down, "b_down", (D,), torch.float32, dev)
    bp, p = rp.block, rp.block.core
    for n_ in ("W_lin_x", "W_lin_y", "W_out"):
        _check(getattr(bp, n_), n_, (D, D), torch.bfloat16, dev)
    for n_ in ("b_lin_x", "b_lin_y", "b_out"):
        _check(getattr(bp, n_), n_, (D,), torch.float32, dev)
    _check(p.conv_w, "conv_w", (4, D), torch.float32, dev)
    for n_ in ("conv_b", "b_a", "b_x", "lam"):
        _check(getattr(p, n_), n_, (D,), torch.float32, dev)
    _check(p.W_a, "W_a", (D // 256, 256, 256), torch.bfloat16, dev)
    _check(p.W_x, "W_x", (D // 256, 256, 256), torch.bfloat16, dev)
    _check(segment_pos, "segment_pos", (B, T), torch.int32, dev)
    _check(conv_state, "conv_state", (B, 3, D), torch.bfloat16, dev)
    _check(h_state, "h_state", (B, D), torch.float32, dev)
    if out is None:
        out = torch.empty_like(u)
    _check(out, "out", (B, T, D), torch.bfloat16, dev)
    if workspace is None:
        workspace = new_workspace(residual_block_workspace_size(B, T, D, F), dev)
    st = load().rglru_residual_block_prefill(
        B, T, D, F, _ptr(u), _ptr(rp.w_temporal_norm), _ptr(bp.W_lin_x), _ptr(bp.b_lin_x), _ptr(bp.W_lin_y),
        _ptr(bp.b_lin_y), _ptr(p.conv_w), _ptr(p.conv_b), _ptr(p.W_a), _ptr(p.b_a), _ptr(p.W_x), _ptr(p.b_x),
        _ptr(p.lam), _ptr(bp.W_out), _ptr(bp.b_out), _ptr(segment_pos), _ptr(conv_state), _ptr(h_state),
        _ptr(rp.w_channel_norm), _ptr(rp.W_gate), _ptr(rp.b_gate), _ptr(rp.W_up), _ptr(rp.b_up), _ptr(rp.W_down),
        _ptr(rp.b_down), ctypes.c_float(eps), _ptr(out), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(dev))
    if st != OK:
        raise RGLRUError(st, "rglru_residual_block_prefill")
    return out


# ---------------------------------------------------------------- local MQA
MQA_WINDOW = 2048


def mqa_vt(B: int, T: int, device="cuda") -> torch.Tensor:
    """v transposed, [B, 256, Tp] bf16 with Tp = T rounded up to 8."""
    if int(load().rglru_mqa_vt_size(B, T)) == 0:
        raise RGLRUError(ERR_INVALID_ARG, "mqa_vt_size")
    return torch.empty((B, 256, (T + 7) // 8 * 8), dtype=torch.bfloat16, device=device)


def mqa_rope(qkv, segment_pos, v_t=None) -> torch.Tensor:
    """RoPE on the query heads and the key of qkv [B, T, (H + 2) * 256] in
    place (rglru_mqa_rope); returns v_t, the v columns transposed."""
    if qkv.dim() != 3 or qkv.shape[2] % 256 != 0 or qkv.shape[2] < 768:
        raise ValueError("qkv must be [B, T, (H + 2) * 256]")
    B, T, C = qkv.shape
    dev = qkv.device
    _check(qkv, "qkv", (B, T, C), torch.bfloat16, dev)
    _check(segment_pos, "segment_pos", (B, T), torch.int32, dev)
    if v_t is None:
        v_t = mqa_vt(B, T, dev)
    _check(v_t, "v_t", (B, 256, (T + 7) // 8 * 8), torch.bfloat16, dev)
    st = load().rglru_mqa_rope(B, T, C // 256 - 2, _ptr(qkv), _ptr(segment_pos), _ptr(v_t), _stream(dev))
    if st != OK:
        raise RGLRUError(st, "rglru_mqa_rope")
    return v_t


def mqa_attention(qkv, v_t, segment_pos, window: int = MQA_WINDOW, out=None, workspace=None) -> torch.Tensor:
    """Local MQA over qkv (after mqa_rope) and v_t (rglru_mqa_attention):
    out [B, T, H * 256] bf16."""
    if qkv.dim() != 3 or qkv.shape[2] % 256 != 0 or qkv.shape[2] < 768:
        raise ValueError("qkv must be [B, T, (H + 2) * 256]")
    B, T, C = qkv.shape
    H = C // 256 - 2
    dev = qkv.device
    _check(qkv, "qkv", (B, T, C), torch.bfloat16, dev)
    _check(v_t, "v_t", (B, 256, (T + 7) // 8 * 8), torch.bfloat16, dev)
    _check(segment_pos, "segment_pos", (B, T), torch.int32, dev)
    if out is None:
        out = torch.empty((B, T, H * 256), dtype=torch.bfloat16, device=dev)
    _check(out, "out", (B, T, H * 256), torch.bfloat16, dev)
    workspace, nb = _ws(workspace, dev)
    st = load().rglru_mqa_attention(B, T, H, int(window), _ptr(qkv), _ptr(v_t), _ptr(segment_pos), _ptr(out),
                                    _ptr(workspace), nb, _stream(dev))
    if st != OK:
        raise RGLRUError(st, "rglru_mqa_attention")
    return out


@dataclass
class MQAParams:
    """Projections of the local MQA block: W_qkv [D + 512, D] (the rows of
    W_q, then W_k, then W_v), W_o [D, D] bf16 and b_o [D] fp32."""
    W_qkv: torch.Tensor
    W_o: torch.Tensor
    b_o: torch.Tensor

    @staticmethod
    def from_arrays(inp: dict, device="cuda") -> "MQAParams":
        def w(a):
            return torch.as_tensor(a, dtype=torch.float32).to(device).to(torch.bfloat16).contiguous()
        W_qkv = torch.cat([w(inp["W_q"]), w(inp["W_k"]), w(inp["W_v"])], dim=0).contiguous()
        return MQAParams(W_qkv, w(inp["W_o"]), torch.as_tensor(inp["b_o"], dtype=torch.float32).to(device).contiguous())


def mqa_block_workspace_size(B: int, T: int, D: int) -> int:
    n = int(load().rglru_mqa_block_workspace_size(B, T, D))
    if n == 0:
        raise RGLRUError(ERR_INVALID_ARG, "mqa_block_workspace_size")
    return n


def mqa_block_prefill(u, mp: MQAParams, segment_pos, window: int = MQA_WINDOW, out=None,
                      workspace=None) -> torch.Tensor:
    """out = o_proj(local MQA(RoPE(q_proj u), RoPE(k_proj u), v_proj u)) over u [B,T,D] bf16
    (rglru_mqa_block_prefill)."""
    if u.dim() != 3:
        raise ValueError("u must be [B,T,D]")
    B, T, D = u.shape
    dev = u.device
    _check(u, "u", (B, T, D), torch.bfloat16, dev)
    _check(mp.W_qkv, "W_qkv", (D + 512, D), torch.bfloat16, dev)
    _check(mp.W_o, "W_o", (D, D), torch.bfloat16, dev)
    _check(mp.b_o, "b_o", (D,), torch.float32, dev)
    _check(segment_pos, "segment_pos", (B, T), torch.int32, dev)
    if out is None:
        out = torch.empty_like(u)
    _check(out, "out", (B, T, D), torch.bfloat16, dev)
    if workspace is None:
        workspace = new_workspace(mqa_block_workspace_size(B, T, D), dev)
    st = load().rglru_mqa_block_prefill(B, T, D, int(window), _ptr(u), _ptr(mp.W_qkv), _ptr(mp.W_o), _ptr(mp.b_o),
                                        _ptr(segment_pos), _ptr(out), _ptr(workspace),
                                        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(dev))
    if st != OK:
        raise RGLRUError(st, "rglru_mqa_block_prefill")
    return out


def mqa_decode_workspace_size(B: int, H: int, window: int = MQA_WINDOW) -> int:
    n = int(load().rglru_mqa_decode_workspace_size(B, H, window))
    if n == 0:
        raise RGLRUError(ERR_UNSUPPORTED, "mqa_decode_workspace_size")
    return n


def mqa_cache(B: int, window: int = MQA_WINDOW, device="cuda"):
    """Zero-filled rings: keys [B, window, 256] and values transposed [B, 256, window], bf16."""
    return (torch.zeros((B, window, 256), dtype=torch.bfloat16, device=device),
            torch.zeros((B, 256, window), dtype=torch.bfloat16, device=device))


def mqa_decode_step(qkv, segment_pos, k_cache, v_cache_t, out=None, workspace=None) -> torch.Tensor:
    """One local-MQA decode step (rglru_mqa_decode_step): qkv [B, (H + 2) * 256]
    bf16 of the new token, segment_pos [B] int32, the rings k_cache [B, window,
    256] and v_cache_t [B, 256, window] (updated in place); returns out
    [B, H * 256] bf16."""
    if qkv.dim() != 2 or qkv.shape[1] % 256 != 0 or qkv.shape[1] < 768:
        raise ValueError("qkv must be [B, (H + 2) * 256]")
    B, C = qkv.shape
    H = C // 256 - 2
    dev = qkv.device
    window = k_cache.shape[1] if k_cache.dim() == 3 else -1
    _check(qkv, "qkv", (B, C), torch.bfloat16, dev)
    _check(segment_pos, "segment_pos", (B,), torch.int32, dev)
    _check(k_cache, "k_cache", (B, window, 256), torch.bfloat16, dev)
    _check(v_cache_t, "v_cache_t", (B, 256, window), torch.bfloat16, dev)
    if out is None:
        out = torch.empty((B, H * 256), dtype=torch.bfloat16, device=dev)
    _check(out, "out", (B, H * 256), torch.bfloat16, dev)
    if workspace is None:
        workspace = new_workspace(mqa_decode_workspace_size(B, H, window), dev)
    st = load().rglru_mqa_decode_step(B, H, window, _ptr(qkv), _ptr(segment_pos), _ptr(k_cache), _ptr(v_cache_t),
                                      _ptr(out), _ptr(workspace),
                                      ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(dev))
    if st != OK:
        raise RGLRUError(st, "rglru_mqa_decode_step")
    return out


@dataclass
class MQAResidualParams:
    """The residual block with local MQA: RMSNorm scales [D] fp32, the MQA
    projections (MQAParams) and the MLP (bf16 weights, fp32 biases)."""
    w_temporal_norm: torch.Tensor
    mqa: MQAParams
    w_channel_norm: torch.Tensor
    W_gate: torch.Tensor
    b_gate: torch.Tensor
    W_up: torch.Tensor
    b_up: torch.Tensor
    W_down: torch.Tensor
    b_down: torch.Tensor

    @staticmethod
    def from_arrays(inp: dict, device="cuda") -> "MQAResidualParams":
        def w(a):
            return torch.as_tensor(a, dtype=torch.float32).to(device).to(torch.bfloat16).contiguous()

        def f32(a):
            return torch.as_tensor(a, dtype=torch.float32).to(device).contiguous()
        return MQAResidualParams(f32(inp["w_temporal_norm"]), MQAParams.from_arrays(inp, device),
                                 f32(inp["w_channel_norm"]), w(inp["W_gate"]), f32(inp["b_gate"]), w(inp["W_up"]),
                                 f32(inp["b_up"]), w(inp["W_down"]), f32(inp["b_down"]))


def mqa_residual_block_workspace_size(B: int, T: int, D: int, F: int) -> int:
    n = int(load().rglru_mqa_residual_block_workspace_size(B, T, D, F))
    if n == 0:
        raise RGLRUError(ERR_INVALID_ARG, "mqa_residual_block_workspace_size")
    return n


def mqa_residual_block_prefill(u, rp: MQAResidualParams, segment_pos, window: int = MQA_WINDOW, eps: float = 1e-6,
                               out=None, workspace=None) -> torch.Tensor:
    """The residual block with local MQA over u [B,T,D] bf16 (rglru_mqa_residual_block_prefill)."""
    if u.dim() != 3:
        raise ValueError("u must be [B,T,D]")
    B, T, D = u.shape
    dev = u.device
    F = rp.W_gate.shape[0]
    _check(u, "u", (B, T, D), torch.bfloat16, dev)
    for n in ("w_temporal_norm", "w_channel_norm"):
        _check(getattr(rp, n), n, (D,), torch.float32, dev)
    _check(rp.mqa.W_qkv, "W_qkv", (D + 512, D), torch.bfloat16, dev)
    _check(rp.mqa.W_o, "W_o", (D, D), torch.bfloat16, dev)
    _check(rp.mqa.b_o, "b_o", (D,), torch.float32, dev)
    _check(rp.W_gate, "W_gate", (F, D), torch.bfloat16, dev)
    _check(rp.W_up, "W_up", (F, D), torch.bfloat16, dev)
    _check(rp.W_down, "W_down", (D, F), torch.bfloat16, dev)
    for n, k in (("b_gate", F), ("b_up", F), ("b_down", D)):
        _check(getattr(rp, n), n, (k,), torch.float32, dev)
    _check(segment_pos, "segment_pos", (B, T), torch.int32, dev)
    if out is None:
        out = torch.empty_like(u)
    _check(out, "out", (B, T, D), torch.bfloat16, dev)
    if workspace is None:
        workspace = new_workspace(mqa_residual_block_workspace_size(B, T, D, F), dev)
    st = load().rglru_mqa_residual_block_prefill(
        B, T, D, F, int(window), _ptr(u), _ptr(rp.w_temporal_norm), _ptr(rp.mqa.W_qkv), _ptr(rp.mqa.W_o),
        _ptr(rp.mqa.b_o), _ptr(segment_pos), _ptr(rp.w_channel_norm), _ptr(rp.W_gate), _ptr(rp.b_gate), _ptr(rp.W_up),
        _ptr(rp.b_up), _ptr(rp.W_down), _ptr(rp.b_down), ctypes.c_float(eps), _ptr(out), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(dev))
    if st != OK:
        raise RGLRUError(st, "rglru_mqa_residual_block_prefill")
    return out


def carry_scan(H0, H1, h0, h_in=None) -> torch.Tensor:
    """rglru_carry_scan: the state each of N time chunks starts from, given the
    chunks' end states from 0 (H0) and from 1 (H1), [N, B, D] fp32, and the
    state h0 [B, D] before the first chunk.  Returns h_in [N, B, D]."""
    if H0.dim() != 3:
        raise ValueError("H0 must be [N, B, D]")
    N, B, D = H0.shape
    dev = H0.device
    _check(H0, "H0", (N, B, D), torch.float32, dev)
    _check(H1, "H1", (N, B, D), torch.float32, dev)
    _check(h0, "h0", (B, D), torch.float32, dev)
    if h_in is None:
        h_in = torch.empty_like(H0)
    _check(h_in, "h_in", (N, B, D), torch.float32, dev)
    st = load().rglru_carry_scan(N, B, D, _ptr(H0), _ptr(H1), _ptr(h0), _ptr(h_in), _stream(dev))
    if st != OK:
        raise RGLRUError(st, "rglru_carry_scan")
    return h_in
