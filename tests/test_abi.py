"""The C-ABI library loads, exports every symbol include/rglru.h declares, and
rejects bad arguments synchronously.  No call here reaches a kernel launch:
every case fails validation first (on a host without a GPU a launch could
only fail with 'no device', never touch memory)."""
import ctypes
import os
import re

import pytest
import torch

from lm_causal_depthwise_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rglru.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"RGLRU_API\s+[\w\s\*]+?\b(rglru_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert sorted(api.SYMBOLS) == declared_symbols()


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.rglru_version() == 100


def test_status_strings(lib):
    for s in range(6):
        assert api.status_string(s)
    assert api.status_string(99) == "unknown status"


@pytest.mark.parametrize("B,T,D", [(0, 4, 256), (1, 0, 256), (1, 4, 255), (1, 4, 384), (1, 4, 0),
                                   (70000, 1, 256)])
def test_workspace_size_rejects_bad_sizes(lib, B, T, D):
    for dt in (api.IO_F32, api.IO_BF16):
        assert lib.rglru_workspace_size(B, T, D, dt) == 0
        assert lib.rglru_simt_workspace_size(B, T, D, dt) == 0
    assert lib.rglru_workspace_size(1, 4, 256, 7) == 0


def test_workspace_size_positive(lib):
    for dt in (api.IO_F32, api.IO_BF16):
        assert lib.rglru_workspace_size(8, 4096, 2560, dt) >= 4096
        assert lib.rglru_decode_workspace_size(256, 2560, dt) >= 4096
    # the SIMT path keeps three fp32 [B,T,D] intermediates
    assert lib.rglru_simt_workspace_size(2, 8, 256, api.IO_BF16) >= 3 * 2 * 8 * 256 * 4


def _call(lib, fn="rglru_prefill", B=1, T=4, D=256, dt=api.IO_BF16, ptrs=None, ws=None, wsb=None):
    base = 1 << 20
    if ptrs is None:
        # distinct, aligned, non-overlapping fake addresses (validation must stop before use)
        ptrs = [base * (k + 1) for k in range(13)]
    if ws is None:
        ws = base * 64
    if wsb is None:
        q = lib.rglru_simt_workspace_size if fn == "rglru_prefill_simt" else lib.rglru_workspace_size
        wsb = q(B, T, D, dt) or 1 << 20
    args = [ctypes.c_void_p(p) if p else None for p in ptrs]
    if fn == "rglru_decode_step":
        return getattr(lib, fn)(B, D, dt, *args, ctypes.c_void_p(ws) if ws else None,
                                ctypes.c_size_t(wsb), None)
    return getattr(lib, fn)(B, T, D, dt, *args, ctypes.c_void_p(ws) if ws else None,
                            ctypes.c_size_t(wsb), None)


@pytest.mark.parametrize("fn", ["rglru_prefill", "rglru_prefill_simt"])
def test_rejects_before_launch(lib, fn):
    assert _call(lib, fn, D=300) == api.ERR_INVALID_ARG
    assert _call(lib, fn, T=0) == api.ERR_INVALID_ARG
    assert _call(lib, fn, dt=5) == api.ERR_INVALID_ARG
    for k in range(13):
        p = [(1 << 20) * (j + 1) for j in range(13)]
        p[k] = 0
        assert _call(lib, fn, ptrs=p) == api.ERR_INVALID_ARG, f"null pointer {k}"
        p[k] = (1 << 20) * (k + 1) + 4
        assert _call(lib, fn, ptrs=p) == api.ERR_INVALID_ARG, f"misaligned pointer {k}"
    assert _call(lib, fn, ws=0) == api.ERR_WORKSPACE
    assert _call(lib, fn, ws=(1 << 20) * 64 + 8) == api.ERR_WORKSPACE
    assert _call(lib, fn, wsb=16) == api.ERR_WORKSPACE
    # y overlapping x
    p = [(1 << 20) * (j + 1) for j in range(13)]
    p[12] = p[0]
    assert _call(lib, fn, ptrs=p) == api.ERR_INVALID_ARG
    # conv_state overlapping h_state
    p = [(1 << 20) * (j + 1) for j in range(13)]
    p[10] = p[11]
    assert _call(lib, fn, ptrs=p) == api.ERR_INVALID_ARG


def test_decode_rejects_before_launch(lib):
    f = "rglru_decode_step"
    wsb = lib.rglru_decode_workspace_size(4, 256, api.IO_BF16)
    assert _call(lib, f, B=4, D=512 + 3, wsb=wsb) == api.ERR_INVALID_ARG
    assert _call(lib, f, B=0, wsb=wsb) == api.ERR_INVALID_ARG
    assert _call(lib, f, B=4, wsb=8) == api.ERR_WORKSPACE
    p = [(1 << 20) * (j + 1) for j in range(13)]
    p[9] = 0
    assert _call(lib, f, B=4, ptrs=p, wsb=wsb) == api.ERR_INVALID_ARG


def test_status_calls_reject_null_workspace(lib):
    assert lib.rglru_get_device_status(None, None) == api.ERR_WORKSPACE
    assert lib.rglru_debug_suppress_publish(None, 0, None) == api.ERR_WORKSPACE
    assert lib.rglru_debug_suppress_publish(ctypes.c_void_p(1 << 20), -2, None) == api.ERR_INVALID_ARG


def _al(n):
    return (n + 255) // 256 * 256


@pytest.mark.parametrize("B,T,D,dt,rows", [(8, 4096, 2560, 1, 1), (5, 300, 512, 0, 2), (3, 7, 256, 1, 9)])
def test_host_prefill_staging_size(lib, B, T, D, dt, rows):
    r = min(B, rows)
    e = 2 if dt == 1 else 4
    want = 2 * (3 * _al(r * T * D * e) + _al(r * T * 4))
    assert lib.rglru_prefill_host_staging_size(B, T, D, dt, rows) == want


@pytest.mark.parametrize("args", [(0, 4, 256, 1, 1), (2, 4, 255, 1, 1), (2, 4, 256, 1, 0), (2, 4, 256, 7, 1)])
def test_host_prefill_staging_size_rejects(lib, args):
    assert lib.rglru_prefill_host_staging_size(*args) == 0


def test_host_prefill_rejects_before_any_cuda_call(lib):
    """Null host buffers, missing or small staging and a small workspace are
    refused before a stream or event is created."""
    host = ctypes.create_string_buffer(1 << 16)
    fake_dev = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
    B, T, D, dt, rows = 2, 8, 256, 1, 1
    st_need = lib.rglru_prefill_host_staging_size(B, T, D, dt, rows)
    ws_need = lib.rglru_workspace_size(rows, T, D, dt)
    hp = ctypes.cast(host, ctypes.c_void_p)

    def call(xh, yh, staging, st_bytes, ws_bytes):
        return lib.rglru_prefill_host(B, T, D, dt, xh, hp, fake_dev, fake_dev, fake_dev, fake_dev, fake_dev,
                                      fake_dev, fake_dev, hp, fake_dev, fake_dev, yh, rows, staging, st_bytes,
                                      fake_dev, ws_bytes, None)
    assert call(None, hp, fake_dev, st_need, ws_need) == api.ERR_INVALID_ARG
    assert call(hp, None, fake_dev, st_need, ws_need) == api.ERR_INVALID_ARG
    assert call(hp, hp, None, st_need, ws_need) == api.ERR_WORKSPACE
    assert call(hp, hp, fake_dev, st_need - 1, ws_need) == api.ERR_WORKSPACE
    assert call(hp, hp, fake_dev, st_need, ws_need - 1) == api.ERR_WORKSPACE


def test_host_prefill_rejects_overlaps_before_any_cuda_call(lib):
    """Overlapping host buffers, a missing state, and a chunk whose staging
    overlaps the states or the workspace are all refused before a stream is
    created (every chunk's arguments are checked up front)."""
    B, T, D, dt, rows = 3, 8, 256, 1, 1
    act = T * D * 2
    host = ctypes.create_string_buffer(4 * B * act + (1 << 12))
    base = ctypes.addressof(host)
    hx, hg, hsp, hy = (ctypes.c_void_p(base + i * B * act) for i in range(4))
    st_need = lib.rglru_prefill_host_staging_size(B, T, D, dt, rows)
    ws_need = lib.rglru_workspace_size(rows, T, D, dt)
    staging = 0x100000  # fake device addresses: never dereferenced, validation fails first
    par = [ctypes.c_void_p(0x40000000 + i * 0x100000) for i in range(7)]
    ws = ctypes.c_void_p(0x50000000)

    def call(x, y, cs, hs, wsp):
        return lib.rglru_prefill_host(B, T, D, dt, x, hg, *par, hsp, cs, hs, y, rows,
                                      ctypes.c_void_p(staging), st_need, wsp, ws_need, None)
    cs_ok, hs_ok = ctypes.c_void_p(0x60000000), ctypes.c_void_p(0x70000000)
    # y_host overlapping x_host
    assert call(hx, ctypes.c_void_p(base + act), cs_ok, hs_ok, ws) == api.ERR_INVALID_ARG
    # missing conv_state / h_state
    assert call(hx, hy, None, hs_ok, ws) == api.ERR_INVALID_ARG
    assert call(hx, hy, cs_ok, None, ws) == api.ERR_INVALID_ARG
    # conv_state inside the second staging slot (only chunk 1 uses that slot)
    slot = st_need // 2
    act_al = (rows * act + 255) // 256 * 256
    assert call(hx, hy, ctypes.c_void_p(staging + slot), hs_ok, ws) == api.ERR_INVALID_ARG
    # h_state overlapping the end of the staging buffer
    assert call(hx, hy, cs_ok, ctypes.c_void_p(staging + st_need - 16), ws) == api.ERR_INVALID_ARG
    # workspace inside the first slot's y tile
    assert call(hx, hy, cs_ok, hs_ok, ctypes.c_void_p(staging + 2 * act_al + 16)) == api.ERR_INVALID_ARG
    # a weight matrix inside the staging buffer
    par_bad = list(par)
    par_bad[4] = ctypes.c_void_p(staging + 64)  # W_x
    assert lib.rglru_prefill_host(B, T, D, dt, hx, hg, *par_bad, hsp, cs_ok, hs_ok, hy, rows,
                                  ctypes.c_void_p(staging), st_need, ws, ws_need, None) == api.ERR_INVALID_ARG


def test_mqa_sizes(lib):
    assert lib.rglru_mqa_vt_size(2, 13) == 2 * 256 * 16 * 2          # T rounded up to 8
    assert lib.rglru_mqa_vt_size(0, 5) == 0 and lib.rglru_mqa_vt_size(1, 0) == 0
    assert lib.rglru_mqa_decode_workspace_size(256, 10, 2048) > 4096
    for window in (0, 64, 100, 2176, 4096):                             # a multiple of 128 up to 2048
        assert lib.rglru_mqa_decode_workspace_size(4, 10, window) == 0, window
    assert lib.rglru_mqa_decode_workspace_size(4, 17, 2048) == 0       # at most 16 heads
    assert lib.rglru_mqa_block_workspace_size(2, 100, 255) == 0
    assert lib.rglru_mqa_block_workspace_size(2, 100, 512) > 4096
    assert lib.rglru_mqa_residual_block_workspace_size(2, 100, 512, 100) == 0   # F a multiple of 128
    assert lib.rglru_mqa_residual_block_workspace_size(2, 100, 512, 1536) > 4096


def _fake(k, off=0):
    """Distinct, aligned, non-overlapping fake device addresses (never used:
    every call below fails validation first)."""
    return ctypes.c_void_p((1 << 24) * (k + 1) + off)


def test_mqa_attention_and_rope_reject_before_launch(lib):
    ws, wsb = _fake(9), ctypes.c_size_t(4096)
    att = lib.rglru_mqa_attention
    assert att(1, 8, 1, 0, _fake(0), _fake(1), _fake(2), _fake(3), ws, wsb, None) == api.ERR_INVALID_ARG  # window 0
    assert att(1, 8, 1, 16, _fake(0, 4), _fake(1), _fake(2), _fake(3), ws, wsb, None) == api.ERR_INVALID_ARG
    assert att(1, 8, 1, 16, _fake(0), _fake(1), None, _fake(3), ws, wsb, None) == api.ERR_INVALID_ARG
    assert att(1, 8, 1, 16, _fake(0), _fake(1), _fake(2), _fake(3), ws, ctypes.c_size_t(64), None) == api.ERR_WORKSPACE
    assert att(1, 8, 1, 16, _fake(0), _fake(1), _fake(2), _fake(0), ws, wsb, None) == api.ERR_INVALID_ARG  # out = qkv
    assert att(1, 8, 65, 16, _fake(0), _fake(1), _fake(2), _fake(3), ws, wsb, None) == api.ERR_UNSUPPORTED
    rope = lib.rglru_mqa_rope
    assert rope(1, 8, 1, _fake(0), _fake(2), _fake(0), None) == api.ERR_INVALID_ARG   # v_t overlaps qkv
    assert rope(1, 8, 1, _fake(0, 8), _fake(2), _fake(1), None) == api.ERR_INVALID_ARG
    assert rope(0, 8, 1, _fake(0), _fake(2), _fake(1), None) == api.ERR_UNSUPPORTED


def test_mqa_decode_and_blocks_reject_before_launch(lib):
    dec = lib.rglru_mqa_decode_step
    need = lib.rglru_mqa_decode_workspace_size(2, 2, 128)
    ws = _fake(9)
    ok_args = dict(qkv=_fake(0), sp=_fake(1), kc=_fake(2), vc=_fake(3), out=_fake(4))

    def call(window=128, wsb=need, **kw):
        a = {**ok_args, **kw}
        return dec(2, 2, window, a["qkv"], a["sp"], a["kc"], a["vc"], a["out"], ws, ctypes.c_size_t(wsb), None)
    assert call(window=100) == api.ERR_UNSUPPORTED
    assert call(kc=_fake(2, 2)) == api.ERR_INVALID_ARG
    assert call(sp=None) == api.ERR_INVALID_ARG
    assert call(wsb=16) == api.ERR_WORKSPACE
    assert call(vc=_fake(2)) == api.ERR_INVALID_ARG       # the two rings overlap
    assert call(out=_fake(0)) == api.ERR_INVALID_ARG      # out overlaps qkv
    blk = lib.rglru_mqa_block_prefill
    bneed = lib.rglru_mqa_block_workspace_size(1, 8, 256)
    assert blk(1, 8, 255, 2048, _fake(0), _fake(1), _fake(2), None, _fake(4), _fake(5), ws,
               ctypes.c_size_t(bneed), None) == api.ERR_INVALID_ARG
    assert blk(1, 8, 256, 2048, _fake(0), _fake(1), _fake(2), None, _fake(4), _fake(5), ws,
               ctypes.c_size_t(64), None) == api.ERR_WORKSPACE
    assert blk(1, 8, 256, 2048, _fake(0), _fake(1), _fake(2), None, _fake(4), _fake(0), ws,
               ctypes.c_size_t(bneed), None) == api.ERR_INVALID_ARG   # out = u
    res = lib.rglru_mqa_residual_block_prefill
    rneed = lib.rglru_mqa_residual_block_workspace_size(1, 8, 256, 768)
    args = [_fake(k) for k in range(13)]  # u, the norms, the projections and their biases, segment_pos
    ws2 = _fake(20)
    assert res(1, 8, 256, 768, 2048, *args, ctypes.c_float(1e-6), _fake(14), ws2, ctypes.c_size_t(16),
               None) == api.ERR_WORKSPACE
    assert res(1, 8, 256, 768, 2048, *args, ctypes.c_float(0.0), _fake(14), ws2, ctypes.c_size_t(rneed),
               None) == api.ERR_UNSUPPORTED    # eps must be positive
    assert res(1, 8, 256, 768, 2048, *args, ctypes.c_float(1e-6), _fake(0), ws2, ctypes.c_size_t(rneed),
               None) == api.ERR_INVALID_ARG    # out = u
    for k in (7, 8, 9, 10, 11):  # W_gate, b_gate, W_up, b_up, W_down: checked before the first launch
        bad = list(args)
        bad[k] = None
        assert res(1, 8, 256, 768, 2048, *bad, ctypes.c_float(1e-6), _fake(14), ws2, ctypes.c_size_t(rneed),
                   None) == api.ERR_INVALID_ARG
        bad[k] = _fake(k, 2)
        assert res(1, 8, 256, 768, 2048, *bad, ctypes.c_float(1e-6), _fake(14), ws2, ctypes.c_size_t(rneed),
                   None) == api.ERR_INVALID_ARG


def test_residual_block_checks_every_operand_before_the_core(lib):
    """rglru_residual_block_prefill updates the states in its core step: an
    operand of a later step that is missing or misaligned must be rejected
    before anything is enqueued (the states and out stay untouched)."""
    res = lib.rglru_residual_block_prefill
    need = lib.rglru_residual_block_workspace_size(1, 8, 256, 768)
    assert need > 0
    # u, w_temporal_norm, W_lin_x, b_lin_x, W_lin_y, b_lin_y, conv_w, conv_b, W_a, b_a, W_x, b_x, lambda,
    # W_out, b_out, segment_pos, conv_state, h_state, w_channel_norm, W_gate, b_gate, W_up, b_up, W_down, b_down
    args = [_fake(k) for k in range(25)]
    names = {13: "W_out", 19: "W_gate", 20: "b_gate", 21: "W_up", 22: "b_up", 23: "W_down"}

    def call(a):
        return res(1, 8, 256, 768, *a, ctypes.c_float(1e-6), _fake(26), _fake(27), ctypes.c_size_t(need), None)
    for k, name in names.items():
        for bad in (None, _fake(k, 2)):
            a = list(args)
            a[k] = bad
            assert call(a) == api.ERR_INVALID_ARG, name
    for k in (3, 5, 14, 24):  # optional biases: NULL passes this check, misaligned does not
        a = list(args)
        a[k] = _fake(k, 4)
        assert call(a) == api.ERR_INVALID_ARG


def test_bindings_reject_host_tensors_before_the_library_runs():
    """Every call that enqueues work takes its stream from its tensors'
    device: host tensors raise in the binding, so no host pointer reaches a
    kernel as device memory."""
    H = torch.zeros(2, 1, 256)
    with pytest.raises(ValueError, match="CUDA tensors"):
        api.carry_scan(H, H.clone(), torch.zeros(1, 256))
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensors"):
        api.rmsnorm(x, torch.ones(256))
    with pytest.raises(ValueError, match="CUDA tensors"):
        api.linear(x, torch.zeros(256, 256, dtype=torch.bfloat16), workspace=torch.zeros(1 << 16, dtype=torch.uint8))
