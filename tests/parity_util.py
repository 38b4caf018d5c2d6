"""Helpers shared by the GPU parity tests: upload seeded inputs, run the CUDA
library, run the oracle on the same arrays, compare with the stated bars.

Tolerances (fixed here, used by every parity test):
  fp32 I/O : max_e |got - ref| / max(|ref_e|, rms(ref)) <= 1e-5
             (relative error 1e-5 for every element at least as large as the
             rms of the output, absolute error 1e-5 * rms below it; a plain
             fp32 evaluation of the definitions scores 3-5e-6 here)
  bf16 I/O : every element |got - ref| <= 2e-2 + 1e-2 * |ref|
             (atol 2e-2, rtol 1e-2; bf16 output rounding alone is 2^-9 relative)
  integer / copied state (conv_state): bit-exact.
"""
from __future__ import annotations

import concurrent.futures as cf
import os

import numpy as np
import torch

from oracle import oracle
from lm_causal_depthwise_b200 import api

F32_RTOL = 1e-5
BF16_ATOL = 2e-2
BF16_RTOL = 1e-2


def io_dtype(io: str) -> torch.dtype:
    return torch.bfloat16 if io == "bf16" else torch.float32


def to_device(inp: dict, io: str, device="cuda") -> dict:
    dt = io_dtype(io)
    d = {
        "x": torch.from_numpy(inp["x"]).to(device).to(dt).contiguous(),
        "g": torch.from_numpy(inp["g"]).to(device).to(dt).contiguous(),
        "segpos": torch.from_numpy(inp["segpos"]).to(device).contiguous(),
        "conv_state": torch.from_numpy(inp["conv_state"]).to(device).to(dt).contiguous(),
        "h_state": torch.from_numpy(inp["h_state"]).to(device).contiguous(),
        "params": api.Params.from_arrays(inp, dt, device),
    }
    return d


def run_gpu(dev: dict, simt: bool = False, workspace=None):
    """Run the library on device inputs; fails if the device status is not OK."""
    x = dev["x"]
    if workspace is None:
        workspace = api.new_workspace(api.workspace_size(*x.shape, x.dtype, simt=simt), x.device)
    y = api.prefill(dev["x"], dev["g"], dev["params"], dev["segpos"], dev["conv_state"],
                    dev["h_state"], workspace=workspace, simt=simt)
    st = api.device_status(workspace)
    assert st == api.OK, f"device status {api.status_string(st)}"
    return {"y": y.float().cpu().numpy(), "conv_state": dev["conv_state"].float().cpu().numpy(),
            "h_state": dev["h_state"].cpu().numpy()}


def run_oracle(inp: dict, nthreads: int = 0):
    return oracle.prefill(**inp, nthreads=nthreads)


def oracle_units(inp: dict, units, t_end=None):
    """Oracle outputs of several (b, head) units, run concurrently (the C
    oracle releases the GIL)."""
    with cf.ThreadPoolExecutor(max_workers=min(len(units), os.cpu_count() or 16)) as ex:
        futs = {u: ex.submit(oracle.prefill_unit, inp, u[0], u[1], t_end, 8.0, 1) for u in units}
        return {u: f.result() for u, f in futs.items()}


def oracle_every_unit(inp: dict):
    """Oracle outputs of the whole problem, computed unit by unit on all host
    cores (memory stays at one unit's float64 copy per worker).  Returns
    (y_units, conv_state [B,3,D], h_state [B,D]) with y_units[(b, h)] the
    float64 [T, 256] output block of unit (b, h)."""
    B, T, D = inp["x"].shape
    units = [(b, h) for b in range(B) for h in range(D // 256)]
    ref = oracle_units(inp, units)
    cs = np.empty((B, 3, D))
    hs = np.empty((B, D))
    for (b, h), r in ref.items():
        s = slice(h * 256, (h + 1) * 256)
        cs[b, :, s] = r["conv_state"]
        hs[b, s] = r["h_state"]
    return {u: r["y"] for u, r in ref.items()}, cs, hs


def check_f32(got, ref, what=""):
    """The fp32 bar: max_e |got - ref| / max(|ref_e|, rms(ref)) <= F32_RTOL.
    The failure message also gives the plain per-element relative error over
    the elements at least 1e-3 rms in size (the floor an earlier reading of the
    bar used), so that both readings are visible; the return value is the
    scaled error, and the relative one is kept in ``check_f32.last_rel``."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    den = np.maximum(np.abs(ref), rms + 1e-300)
    err = np.max(np.abs(got - ref) / den) if ref.size else 0.0
    big = np.abs(ref) >= 1e-3 * rms
    rel = float(np.max(np.abs(got - ref)[big] / np.abs(ref)[big])) if big.any() else 0.0
    check_f32.last_rel = rel
    assert err <= F32_RTOL, (f"{what}: max scaled error {err:.3e} > {F32_RTOL} "
                             f"(plain relative error over |ref| >= 1e-3 rms: {rel:.3e})")
    return err


check_f32.last_rel = 0.0


def check_bf16(got, ref, what="", scale=1.0):
    """Every element within atol + rtol |ref|.  ``scale`` multiplies the
    absolute part for inputs drawn ``scale`` times larger than the workloads'
    N(0, 1): every rounding of an intermediate (bf16 operands, the f16 stash,
    the bf16 output) then errs ``scale`` times more in absolute terms."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = np.abs(got - ref)
    atol = BF16_ATOL * scale
    bad = ~(diff <= atol + BF16_RTOL * np.abs(ref))  # NaN or inf counts as bad
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside atol {atol} + rtol "
            f"{BF16_RTOL}; first at {tuple(idx)}: got {got[tuple(idx)]!r} ref {ref[tuple(idx)]!r}; "
            f"max abs {np.nanmax(diff):.3e}")
    big = np.abs(ref) >= 1.0
    max_rel = float((diff[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    return float(diff.max()), max_rel


def check(io: str, got, ref, what=""):
    return check_bf16(got, ref, what) if io == "bf16" else check_f32(got, ref, what)


def check_state(io: str, got: dict, ref: dict, what=""):
    check(io, got["h_state"], ref["h_state"], f"{what} h_state")
    np.testing.assert_array_equal(np.asarray(got["conv_state"], np.float64),
                                  np.asarray(ref["conv_state"], np.float64),
                                  err_msg=f"{what} conv_state")
