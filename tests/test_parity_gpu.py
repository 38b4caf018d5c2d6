"""GPU parity: the CUDA library against the float64 oracle on the same seeded inputs.

Every case compares every output element.  The full-size workloads run in
the launch configuration the benchmark times; the oracle computes them unit by
unit on all host cores (heads and batch rows are independent).
"""
import numpy as np
import pytest
import torch

from lm_causal_depthwise_b200 import api, workloads as W
from oracle import oracle

from parity_util import (check, check_bf16, check_f32, check_state, oracle_every_unit, oracle_units,
                         run_gpu, run_oracle, to_device)

pytestmark = pytest.mark.gpu

PATHS = [False, True]  # rglru_prefill, rglru_prefill_simt


def _case(B, T, D, io="bf16", seed=21, doc_len=None, reset_at=(0,), continue_doc=False,
          init_state="random", decay="init", x_scale=1.0):
    w = W.Workload("case", B=B, T=T, D=D, io=io, seed=seed, doc_len=doc_len, reset_at=reset_at,
                   continue_doc=continue_doc, init_state=init_state, decay=decay, x_scale=x_scale)
    return w, W.generate(w)


@pytest.mark.parametrize("simt", PATHS)
def test_tiny_f32_full(simt, record_property):
    inp = W.generate(W.TINY_F32)
    got = run_gpu(to_device(inp, "f32"), simt=simt)
    ref = run_oracle(inp)
    err = check_f32(got["y"], ref["y"], "y")
    # both readings of the fp32 bar, kept in the test report
    record_property("scaled_error", err)
    record_property("plain_relative_error_over_1e-3_rms", check_f32.last_rel)
    check_state("f32", got, ref, "tiny")


@pytest.mark.parametrize("simt", PATHS)
@pytest.mark.parametrize("B,T,D,kw", [
    (2, 1000, 512, dict(doc_len=300)),            # several chunks, ragged tail, mid resets
    (1, 2053, 256, dict(continue_doc=True)),      # no reset: initial state carried through chunks
    (3, 515, 768, dict(reset_at=(0, 1, 2, 3, 64, 65, 511))),  # resets near chunk edges
    (1, 4096, 512, dict(doc_len=1024)),
])
def test_bf16_full_tensor(simt, B, T, D, kw):
    _, inp = _case(B, T, D, **kw)
    got = run_gpu(to_device(inp, "bf16"), simt=simt)
    ref = run_oracle(inp)
    check_bf16(got["y"], ref["y"], "y")
    check_state("bf16", got, ref, "state")


@pytest.mark.parametrize("simt", PATHS)
@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 31, 32, 33, 127, 128, 129])
def test_edge_lengths(simt, io, T):
    _, inp = _case(2, T, 256, io=io, continue_doc=True, seed=T)
    got = run_gpu(to_device(inp, io), simt=simt)
    ref = run_oracle(inp)
    check(io, got["y"], ref["y"], f"y T={T}")
    check_state(io, got, ref, f"T={T}")


@pytest.mark.parametrize("simt", PATHS)
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_fast_decay_channels(simt, io):
    """Lambda drawn in [-10, 6.9]: most channels have Lambda < 0
    (sigmoid(Lambda)^8 from ~1e-35 up), the other branch of log sigmoid, and
    decays so fast that the normaliser sqrt(1 - a^2) is ~1.  Several tiles,
    resets, a carried initial state."""
    _, inp = _case(2, 1000, 512, io=io, doc_len=300, decay="wide", seed=33)
    assert (inp["lam"] < -5).any() and (inp["lam"] > 5).any() and (inp["lam"] <= 6.91).all()
    got = run_gpu(to_device(inp, io), simt=simt)
    ref = run_oracle(inp)
    check(io, got["y"], ref["y"], "y")
    check_state(io, got, ref, "state")


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_decode_fast_decay_channels(io):
    T, D, B = 24, 512, 70
    _, inp = _case(B, T, D, io=io, reset_at=(0, 9), decay="wide", seed=34)
    dev = to_device(inp, io)
    ys = []
    for t in range(T):
        ys.append(api.decode_step(dev["x"][:, t].contiguous(), dev["g"][:, t].contiguous(), dev["params"],
                                  dev["segpos"][:, t].contiguous(), dev["conv_state"],
                                  dev["h_state"]).float().cpu().numpy())
    ref = run_oracle(inp)
    check(io, np.stack(ys, axis=1), ref["y"], "decode y")
    got = {"h_state": dev["h_state"].cpu().numpy(), "conv_state": dev["conv_state"].float().cpu().numpy()}
    check_state(io, got, ref, "decode")


@pytest.mark.parametrize("simt", PATHS)
def test_large_magnitude_inputs(simt):
    """x and the conv state drawn as 100 N(0, 1) (|x| up to ~500, |xc| and
    |h| in the hundreds to thousands): every output finite and within the bf16
    bar with its absolute part scaled by the input scale (the f16 stash of the
    fused kernel and the bf16 output err in proportion to the magnitudes).
    The fused kernel's gate GEMM takes xc as a bf16 tensor-core operand; at
    this scale that rounding alone moves a gate near 1/2 by ~0.05 and i xc by
    several units, an error quadratic in the scale, so the fused path is
    compared with the oracle evaluating the gate projections on bf16-rounded
    xc (gate_bf16); the SIMT path (fp32 gate operands) with the exact oracle."""
    s = 100.0
    _, inp = _case(2, 1000, 512, doc_len=300, x_scale=s, seed=35)
    got = run_gpu(to_device(inp, "bf16"), simt=simt)
    assert np.isfinite(got["y"]).all() and np.isfinite(got["h_state"]).all()
    ref = oracle.prefill(**inp, gate_bf16=not simt)
    check_bf16(got["y"], ref["y"], "y", scale=s)
    check_bf16(got["h_state"], ref["h_state"], "h_state", scale=s)
    np.testing.assert_array_equal(got["conv_state"], ref["conv_state"])


@pytest.mark.parametrize("simt", PATHS)
def test_every_token_a_reset(simt):
    w, inp = _case(2, 300, 256)
    inp["segpos"][:] = 0
    got = run_gpu(to_device(inp, "bf16"), simt=simt)
    ref = run_oracle(inp)
    check_bf16(got["y"], ref["y"], "y")
    check_state("bf16", got, ref, "state")


@pytest.mark.parametrize("simt", PATHS)
def test_short_documents(simt):
    _, inp = _case(2, 400, 256, continue_doc=True)
    inp["segpos"][:] = np.arange(400)[None, :] % 2   # a reset every other token
    got = run_gpu(to_device(inp, "bf16"), simt=simt)
    ref = run_oracle(inp)
    check_bf16(got["y"], ref["y"], "y")


def test_write_coverage_and_canaries():
    """Every output element is written (NaN sentinels gone) and nothing past
    the end of y, the two states or the workspace is touched."""
    _, inp = _case(2, 777, 512, doc_len=200)
    dev = to_device(inp, "bf16")
    B, T, D = 2, 777, 512
    pad = 4096
    buf = torch.full((B * T * D + pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = buf[:B * T * D].view(B, T, D)
    csb = torch.full((B * 3 * D + pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    csb[:B * 3 * D].copy_(dev["conv_state"].view(-1))
    hsb = torch.full((B * D + pad,), 7.0, dtype=torch.float32, device="cuda")
    hsb[:B * D].copy_(dev["h_state"].view(-1))
    need = api.workspace_size(B, T, D, torch.bfloat16)
    wsb = torch.full((need + pad,), 0xA5, dtype=torch.uint8, device="cuda")
    wsb[:need].zero_()
    api.prefill(dev["x"], dev["g"], dev["params"], dev["segpos"], csb[:B * 3 * D].view(B, 3, D),
                hsb[:B * D].view(B, D), y=y, workspace=wsb[:need])
    torch.cuda.synchronize()
    assert api.device_status(wsb[:need]) == api.OK
    assert not torch.isnan(y).any()
    assert torch.isnan(buf[B * T * D:]).all()
    assert (csb[B * 3 * D:] == 7.0).all() and (hsb[B * D:] == 7.0).all()
    assert (wsb[need:] == 0xA5).all()


@pytest.mark.parametrize("simt", PATHS)
def test_split_with_carried_state_equals_whole(simt):
    _, inp = _case(2, 1500, 512, continue_doc=True)
    whole = run_gpu(to_device(inp, "bf16"), simt=simt)
    tau = 613
    a = {**inp, "x": inp["x"][:, :tau], "g": inp["g"][:, :tau], "segpos": inp["segpos"][:, :tau]}
    dev_a = to_device(a, "bf16")
    o1 = run_gpu(dev_a, simt=simt)
    b = {**inp, "x": inp["x"][:, tau:], "g": inp["g"][:, tau:], "segpos": inp["segpos"][:, tau:]}
    dev_b = to_device(b, "bf16")
    dev_b["conv_state"].copy_(dev_a["conv_state"])
    dev_b["h_state"].copy_(dev_a["h_state"])
    o2 = run_gpu(dev_b, simt=simt)
    y = np.concatenate([o1["y"], o2["y"]], axis=1)
    check_bf16(y, whole["y"], "split y")
    np.testing.assert_array_equal(o2["conv_state"], whole["conv_state"])
    check_bf16(o2["h_state"], whole["h_state"], "split h")


@pytest.mark.parametrize("simt", PATHS)
def test_reset_makes_output_independent_of_earlier_tokens(simt):
    s = 700
    _, inp = _case(1, 1200, 512, reset_at=(0, s))
    base = run_gpu(to_device(inp, "bf16"), simt=simt)
    pert = {k: v.copy() for k, v in inp.items()}
    rng = np.random.default_rng(9)
    pert["x"][:, :s] = W.round_bf16(rng.standard_normal(pert["x"][:, :s].shape).astype(np.float32))
    pert["g"][:, :s] = W.round_bf16(rng.standard_normal(pert["g"][:, :s].shape).astype(np.float32))
    pert["h_state"] += 1.0
    alt = run_gpu(to_device(pert, "bf16"), simt=simt)
    np.testing.assert_array_equal(alt["y"][:, s:], base["y"][:, s:])
    np.testing.assert_array_equal(alt["h_state"], base["h_state"])


@pytest.mark.parametrize("io,B", [("bf16", 64), ("f32", 64), ("bf16", 100), ("bf16", 3)])
def test_decode_steps_match_oracle(io, B):
    """B = 100 leaves the second 64-row block of the bf16 decode kernel partial;
    B = 3 is a single, mostly empty block."""
    T, D = 40, 512
    _, inp = _case(B, T, D, io=io, reset_at=(0, 17))
    dev = to_device(inp, io)
    ys = []
    for t in range(T):
        y = api.decode_step(dev["x"][:, t].contiguous(), dev["g"][:, t].contiguous(), dev["params"],
                            dev["segpos"][:, t].contiguous(), dev["conv_state"], dev["h_state"])
        ys.append(y.float().cpu().numpy())
    torch.cuda.synchronize()
    ref = run_oracle(inp)
    check(io, np.stack(ys, axis=1), ref["y"], "decode y")
    got = {"h_state": dev["h_state"].cpu().numpy(), "conv_state": dev["conv_state"].float().cpu().numpy()}
    check_state(io, got, ref, "decode")


# ------------------------------------------------------------- full-size workloads

@pytest.mark.parametrize("wname", ["prefill-2b", "prefill-long", "prefill-long-carry", "prefill-9b"])
def test_full_size_every_element(wname):
    """The full-size workloads in the launch configuration the benchmark
    times, every output element (y, h_state, conv_state) against the oracle,
    which runs every (batch row, head) unit on the host cores."""
    w = W.ALL[wname]
    inp = W.generate(w)
    dev = to_device(inp, w.io)
    y = api.prefill(dev["x"], dev["g"], dev["params"], dev["segpos"], dev["conv_state"],
                    dev["h_state"])
    torch.cuda.synchronize()
    del dev["x"], dev["g"]
    ref_y, ref_cs, ref_hs = oracle_every_unit(inp)
    yh = y.float().cpu().numpy()
    del y
    for (b, h), r in ref_y.items():
        check_bf16(yh[b, :, h * 256:(h + 1) * 256], r, f"{w.name} y unit {(b, h)}")
    check_bf16(dev["h_state"].cpu().numpy(), ref_hs, f"{w.name} h_state")
    np.testing.assert_array_equal(dev["conv_state"].float().cpu().numpy(), ref_cs)


def test_full_size_decode_equals_prefill_and_oracle():
    """decode-2b: 1024 single-token steps for B = 256 sequences, against one
    prefill over the same 1024 tokens and against the oracle, every element
    of y and the final states."""
    w = W.DECODE_2B
    inp = W.generate(w)
    dev = to_device(inp, w.io)
    pre = to_device(inp, w.io)
    y_pre = api.prefill(pre["x"], pre["g"], pre["params"], pre["segpos"], pre["conv_state"],
                        pre["h_state"])
    ys = torch.empty((w.T, w.B, w.D), dtype=torch.bfloat16, device="cuda")
    ws = api.new_workspace(api.decode_workspace_size(w.B, w.D, torch.bfloat16))
    xs = dev["x"].transpose(0, 1).contiguous()
    gs = dev["g"].transpose(0, 1).contiguous()
    ss = dev["segpos"].t().contiguous()
    for t in range(w.decode_steps):
        api.decode_step(xs[t], gs[t], dev["params"], ss[t], dev["conv_state"], dev["h_state"],
                        workspace=ws, y=ys[t])
    torch.cuda.synchronize()
    assert api.device_status(ws) == api.OK
    del xs, gs, pre["x"], pre["g"], dev["x"], dev["g"]
    y_dec = ys.transpose(0, 1).float().cpu().numpy()
    del ys
    y_p = y_pre.float().cpu().numpy()
    del y_pre
    check_bf16(y_dec, y_p, "decode y vs prefill y")
    check_bf16(dev["h_state"].cpu().numpy(), pre["h_state"].cpu().numpy(), "decode h vs prefill h")
    np.testing.assert_array_equal(dev["conv_state"].float().cpu().numpy(),
                                  pre["conv_state"].float().cpu().numpy())
    ref_y, ref_cs, ref_hs = oracle_every_unit(inp)
    for (b, h), r in ref_y.items():
        s = slice(h * 256, (h + 1) * 256)
        check_bf16(y_dec[b, :, s], r, f"decode y unit {(b, h)}")
        check_bf16(y_p[b, :, s], r, f"prefill y unit {(b, h)}")
    check_bf16(dev["h_state"].cpu().numpy(), ref_hs, "decode h_state")
    np.testing.assert_array_equal(dev["conv_state"].float().cpu().numpy(), ref_cs)


# ------------------------------------------------------------- bounded waits and cross-checks

def test_bounded_wait_reports_timeout_and_context_survives():
    """A tile that never publishes its scan carry (host-set test hook) makes its
    successor's look-back wait run out: the call ends with RGLRU_ERR_TIMEOUT in
    the device status, within seconds, and the next call on the same context
    and workspace is correct."""
    import time
    _, inp = _case(1, 256, 256, continue_doc=True)
    dev = to_device(inp, "bf16")
    ws = api.new_workspace(api.workspace_size(1, 256, 256, torch.bfloat16))
    api.debug_suppress_publish(ws, 3)
    t0 = time.time()
    api.prefill(dev["x"], dev["g"], dev["params"], dev["segpos"], dev["conv_state"], dev["h_state"],
                workspace=ws)
    assert api.device_status(ws) == api.ERR_TIMEOUT
    assert time.time() - t0 < 60
    api.debug_suppress_publish(ws, -1)
    dev = to_device(inp, "bf16")
    got = run_gpu(dev, workspace=ws)
    assert api.device_status(ws) == api.OK
    ref = run_oracle(inp)
    check_bf16(got["y"], ref["y"], "y after timeout")


@pytest.mark.parametrize("wname", ["prefill-2b", "prefill-long-carry"])
def test_full_size_fused_matches_simt_everywhere(wname):
    """Whole-tensor check at full size: the fused kernel against the plain SIMT
    kernels (fp32, accurate transcendentals), every element."""
    w = W.ALL[wname]
    inp = W.generate(w)
    a = to_device(inp, w.io)
    b = to_device(inp, w.io)
    ya = api.prefill(a["x"], a["g"], a["params"], a["segpos"], a["conv_state"], a["h_state"])
    yb = api.prefill(b["x"], b["g"], b["params"], b["segpos"], b["conv_state"], b["h_state"], simt=True)
    torch.cuda.synchronize()
    diff = (ya.float() - yb.float()).abs()
    bound = 2e-2 + 1e-2 * yb.float().abs()
    assert bool((diff <= bound).all()), f"max diff {diff.max().item():.3e}"
    hb = b["h_state"]
    assert bool(((a["h_state"] - hb).abs() <= 2e-2 + 1e-2 * hb.abs()).all())
    assert torch.equal(a["conv_state"], b["conv_state"])


def test_fused_prefill_is_bit_reproducible():
    """The cross-tile carry is folded in sequence order from its anchor, so two
    runs on the same inputs give identical bits whatever the scheduling."""
    _, inp = _case(2, 3000, 512, doc_len=800)
    a = run_gpu(to_device(inp, "bf16"))
    for _ in range(3):
        b = run_gpu(to_device(inp, "bf16"))
        np.testing.assert_array_equal(a["y"], b["y"])
        np.testing.assert_array_equal(a["h_state"], b["h_state"])


@pytest.mark.parametrize("io,rows", [("bf16", 1), ("bf16", 3), ("bf16", 9), ("f32", 2)])
def test_prefill_from_host_buffers_equals_device_call(io, rows):
    """rglru_prefill_host (host activations, chunks of `rows` sequences, copies
    overlapped with the kernels) gives the device call's bits: sequences are
    independent and the kernels' results do not depend on how the batch is
    split.  Also checked against the oracle."""
    _, inp = _case(5, 300, 512, io=io, doc_len=120)
    ref_dev = to_device(inp, io)
    want = run_gpu(ref_dev)
    dev = to_device(inp, io)
    hx = dev["x"].cpu().pin_memory()
    hg = dev["g"].cpu().pin_memory()
    hsp = dev["segpos"].cpu().pin_memory()
    ws = api.new_workspace(api.workspace_size(min(5, rows), 300, 512, dev["x"].dtype))
    hy = api.prefill_host(hx, hg, dev["params"], hsp, dev["conv_state"], dev["h_state"],
                          rows_per_chunk=rows, workspace=ws)
    torch.cuda.synchronize()
    assert api.device_status(ws) == api.OK
    np.testing.assert_array_equal(hy.float().numpy(), want["y"])
    np.testing.assert_array_equal(dev["conv_state"].float().cpu().numpy(), want["conv_state"])
    np.testing.assert_array_equal(dev["h_state"].cpu().numpy(), want["h_state"])
    ref = run_oracle(inp)
    check(io, hy.float().numpy(), ref["y"], "y")


@pytest.mark.parametrize("world", [2, 3])
def test_head_shards_equal_the_whole_run(world):
    """The core run on each rank's head range (run one after another here, on
    one GPU) gives the whole run's output column blocks and states bit for bit:
    heads never mix and each head's result does not depend on the others."""
    from lm_causal_depthwise_b200.sharding import shard_heads, shard_inputs
    _, inp = _case(2, 700, 768, doc_len=250)
    whole = run_gpu(to_device(inp, "bf16"))
    for r in range(world):
        h0, h1 = shard_heads(3, world, r)
        if h1 == h0:
            continue
        got = run_gpu(to_device(shard_inputs(inp, h0, h1), "bf16"))
        c = slice(h0 * 256, h1 * 256)
        np.testing.assert_array_equal(got["y"], whole["y"][:, :, c])
        np.testing.assert_array_equal(got["h_state"], whole["h_state"][:, c])
        np.testing.assert_array_equal(got["conv_state"], whole["conv_state"][:, :, c])


@pytest.mark.parametrize("world", [2, 3])
def test_decode_head_shards_equal_the_whole_run(world):
    """Decode steps on each rank's head range (run one after another here)
    give the whole decode's output columns and states bit for bit; B = 100
    leaves the second 64-row block of every head partial."""
    from lm_causal_depthwise_b200.sharding import shard_heads, shard_inputs
    B, T, D = 100, 12, 768
    _, inp = _case(B, T, D, reset_at=(0, 5))

    def decode(part):
        dev = to_device(part, "bf16")
        ys = [api.decode_step(dev["x"][:, t].contiguous(), dev["g"][:, t].contiguous(), dev["params"],
                              dev["segpos"][:, t].contiguous(), dev["conv_state"], dev["h_state"])
              for t in range(T)]
        return (torch.stack(ys, 1).float().cpu().numpy(), dev["h_state"].cpu().numpy(),
                dev["conv_state"].float().cpu().numpy())
    y, h, cs = decode(inp)
    for r in range(world):
        h0, h1 = shard_heads(D // 256, world, r)
        c = slice(h0 * 256, h1 * 256)
        ys, hs, css = decode(shard_inputs(inp, h0, h1))
        np.testing.assert_array_equal(ys, y[:, :, c])
        np.testing.assert_array_equal(hs, h[:, c])
        np.testing.assert_array_equal(css, cs[:, :, c])


def test_decode_bounded_wait_reports_timeout_and_context_survives():
    """The test hook makes CTA 0 of the decode grid keep its half of the gate
    GEMM's operand from its peer: the peer's bounded wait runs out, the call
    ends with RGLRU_ERR_TIMEOUT in the device status within seconds, and the
    next step on the same context and workspace is correct."""
    import time
    _, inp = _case(64, 2, 512, reset_at=(0,))
    dev = to_device(inp, "bf16")
    ws = api.new_workspace(api.decode_workspace_size(64, 512, torch.bfloat16))
    api.debug_suppress_publish(ws, 0)
    t0 = time.time()
    api.decode_step(dev["x"][:, 0].contiguous(), dev["g"][:, 0].contiguous(), dev["params"],
                    dev["segpos"][:, 0].contiguous(), dev["conv_state"], dev["h_state"], workspace=ws)
    assert api.device_status(ws) == api.ERR_TIMEOUT
    assert time.time() - t0 < 60
    api.debug_suppress_publish(ws, -1)
    dev = to_device(inp, "bf16")
    ys = []
    for t in range(2):
        ys.append(api.decode_step(dev["x"][:, t].contiguous(), dev["g"][:, t].contiguous(), dev["params"],
                                  dev["segpos"][:, t].contiguous(), dev["conv_state"], dev["h_state"],
                                  workspace=ws).float().cpu().numpy())
    assert api.device_status(ws) == api.OK
    ref = run_oracle(inp)
    check_bf16(np.stack(ys, axis=1), ref["y"], "decode y after timeout")


@pytest.mark.parametrize("world,kw", [(2, dict(continue_doc=True)), (4, dict(continue_doc=True)),
                                      (3, dict(doc_len=700))])
def test_time_shards_with_one_exchange_match_oracle(world, kw):
    """One long sequence split in time over `world` ranks, emulated one after
    another on this GPU: each rank runs its chunk from h = 0 and from h = 1,
    rglru_carry_scan folds the gathered end states into every chunk's starting
    state, each rank runs its chunk again from it (conv state = the three raw
    inputs before the chunk).  The joined outputs and the final states against
    the oracle of the whole sequence; with documents carried across every chunk
    boundary (continue_doc) and with resets inside the chunks."""
    from lm_causal_depthwise_b200.sharding import shard_time, shard_time_inputs
    B, T, D = 2, 2000, 512
    _, inp = _case(B, T, D, **kw)
    bf = torch.bfloat16
    ends = {0.0: [], 1.0: []}
    for r in range(world):
        t0, t1 = shard_time(T, world, r)
        part = shard_time_inputs(inp, t0, t1)
        for h in (0.0, 1.0):
            dev = to_device({**part, "h_state": np.full((B, D), h, np.float32)}, "bf16")
            run_gpu(dev)
            ends[h].append(dev["h_state"])
    H0, H1 = torch.stack(ends[0.0]).contiguous(), torch.stack(ends[1.0]).contiguous()
    h_in = api.carry_scan(H0, H1, torch.from_numpy(inp["h_state"]).cuda())
    ys = []
    for r in range(world):
        t0, t1 = shard_time(T, world, r)
        dev = to_device(shard_time_inputs(inp, t0, t1), "bf16")
        dev["h_state"].copy_(h_in[r])
        got = run_gpu(dev)
        ys.append(got["y"])
    ref = run_oracle(inp)
    check_bf16(np.concatenate(ys, axis=1), ref["y"], f"time shards x{world} y")
    check_bf16(got["h_state"], ref["h_state"], f"time shards x{world} h_state")
    np.testing.assert_array_equal(got["conv_state"], ref["conv_state"])
