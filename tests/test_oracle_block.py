"""Pins of the block oracle (oracle/block.py) against facts from outside it:
torch's float64 Linear and GELU, explicit loops, torch's bf16 conversion,
and the reduction of the block to the pinned core when the projections are
identities."""
import numpy as np
import torch

from oracle import block, oracle
from lm_causal_depthwise_b200 import workloads as W


def test_linear_matches_torch_float64_and_loops():
    rng = np.random.default_rng(1)
    x, Wm, b = rng.standard_normal((5, 7)), rng.standard_normal((3, 7)), rng.standard_normal(3)
    want = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(Wm), torch.from_numpy(b)).numpy()
    np.testing.assert_allclose(block.linear(x, Wm, b), want, rtol=1e-14, atol=1e-14)
    loops = np.array([[sum(x[i, k] * Wm[j, k] for k in range(7)) + b[j] for j in range(3)] for i in range(5)])
    np.testing.assert_allclose(block.linear(x, Wm, b), loops, rtol=1e-13, atol=1e-13)


def test_round_bf16_matches_torch_on_float32_values():
    """On values that are exact in float32, nearest-even bf16 rounding is the
    float32 -> bf16 conversion torch performs (no double rounding involved)."""
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-20, 20, 100000),
                        [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -1.0 - 2.0 ** -8, 0.0, 3.0]]).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(block.round_bf16(v.astype(np.float64)), want)


def test_gelu_matches_torch():
    g = np.linspace(-8, 8, 1001)
    want = torch.nn.functional.gelu(torch.from_numpy(g), approximate="tanh").numpy()
    np.testing.assert_allclose(block.gelu_tanh(g), want, rtol=1e-14, atol=1e-15)


def test_block_with_identity_projections_is_the_core():
    """W_lin_x = W_lin_y = W_out = I and zero biases: the block is the core
    applied to (u, u), each tensor rounded to bf16 at the block's interfaces."""
    w = W.Workload("pin", B=2, T=70, D=512, io="bf16", seed=4, doc_len=30, init_state="random")
    inp = W.generate_block(w)
    eye = np.eye(512)
    z = np.zeros(512)
    out = block.recurrent_block(inp["u"], eye, z, eye, z, eye, z, inp["conv_w"], inp["conv_b"], inp["W_a"],
                                inp["b_a"], inp["W_x"], inp["b_x"], inp["lam"], inp["segpos"],
                                inp["conv_state"], inp["h_state"])
    ref = oracle.prefill(inp["u"], inp["u"], inp["conv_w"], inp["conv_b"], inp["W_a"], inp["b_a"], inp["W_x"],
                         inp["b_x"], inp["lam"], inp["segpos"], inp["conv_state"], inp["h_state"])
    np.testing.assert_array_equal(out["out"], block.round_bf16(ref["y"]))
    np.testing.assert_array_equal(out["h_state"], ref["h_state"])
    np.testing.assert_array_equal(out["conv_state"], ref["conv_state"])


def test_block_branches_follow_the_printed_wiring():
    """linear_x feeds the conv (the core's x) and linear_y the GELU branch:
    swapping the two weight matrices changes the output, and the block's x
    and g are the two projections of u."""
    w = W.Workload("pin", B=1, T=40, D=256, io="bf16", seed=5, init_state="zero")
    inp = W.generate_block(w)
    args = dict(conv_w=inp["conv_w"], conv_b=inp["conv_b"], W_a=inp["W_a"], b_a=inp["b_a"], W_x=inp["W_x"],
                b_x=inp["b_x"], lam=inp["lam"], segpos=inp["segpos"], conv_state=inp["conv_state"],
                h_state=inp["h_state"])
    o = block.recurrent_block(inp["u"], inp["W_lin_x"], inp["b_lin_x"], inp["W_lin_y"], inp["b_lin_y"],
                              inp["W_out"], inp["b_out"], **args)
    np.testing.assert_array_equal(o["x"], block.round_bf16(inp["u"] @ inp["W_lin_x"].astype(np.float64).T
                                                           + inp["b_lin_x"]))
    np.testing.assert_array_equal(o["g"], block.round_bf16(inp["u"] @ inp["W_lin_y"].astype(np.float64).T
                                                           + inp["b_lin_y"]))
    s = block.recurrent_block(inp["u"], inp["W_lin_y"], inp["b_lin_y"], inp["W_lin_x"], inp["b_lin_x"],
                              inp["W_out"], inp["b_out"], **args)
    assert np.abs(s["out"] - o["out"]).max() > 1e-2


def test_mlp_matches_torch_modules():
    """gate_proj / up_proj / down_proj with a tanh GELU on the gate, against
    torch's float64 Linear and GELU (no rounding)."""
    rng = np.random.default_rng(6)
    D, F = 16, 48
    v = rng.standard_normal((5, D))
    Wg, Wu, Wd = rng.standard_normal((F, D)), rng.standard_normal((F, D)), rng.standard_normal((D, F))
    bg, bu, bd = rng.standard_normal(F), rng.standard_normal(F), rng.standard_normal(D)
    t = {k: torch.from_numpy(a) for k, a in dict(v=v, Wg=Wg, Wu=Wu, Wd=Wd, bg=bg, bu=bu, bd=bd).items()}
    F_ = torch.nn.functional
    want = F_.linear(F_.gelu(F_.linear(t["v"], t["Wg"], t["bg"]), approximate="tanh")
                     * F_.linear(t["v"], t["Wu"], t["bu"]), t["Wd"], t["bd"]).numpy()
    np.testing.assert_allclose(block.mlp(v, Wg, bg, Wu, bu, Wd, bd, round_io=False), want, rtol=1e-12, atol=1e-12)


def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(7)
    x, w = rng.standard_normal((6, 40)) * 3.0, rng.standard_normal(40)
    want = torch.nn.functional.rms_norm(torch.from_numpy(x), (40,), torch.from_numpy(w), eps=1e-6).numpy()
    np.testing.assert_allclose(block.rmsnorm(x, w, 1e-6), want, rtol=1e-13, atol=1e-13)
    # a constant row normalises to w (sign kept): x / |x| * w
    np.testing.assert_allclose(block.rmsnorm(np.full((1, 40), -2.5), w, 0.0)[0], -w, rtol=1e-15)


def _res_args(inp):
    keys = ("u", "w_temporal_norm", "W_lin_x", "b_lin_x", "W_lin_y", "b_lin_y", "W_out", "b_out", "conv_w",
            "conv_b", "W_a", "b_a", "W_x", "b_x", "lam", "segpos", "conv_state", "h_state", "w_channel_norm",
            "W_gate", "b_gate", "W_up", "b_up", "W_down", "b_down")
    return [inp[k] for k in keys]


def test_residual_block_wiring():
    """Zero linear_out and down_proj (weights and biases): both residual adds
    pass their input through, out = u.  Zero down_proj only: out = h, the
    recurrent block's residual output, which equals u + the recurrent block
    applied to RMSNorm(u)."""
    w = W.Workload("pin", B=1, T=30, D=256, io="bf16", seed=8, init_state="zero")
    inp = W.generate_residual_block(w)
    z = dict(inp)
    z["W_out"] = np.zeros_like(inp["W_out"]); z["b_out"] = np.zeros_like(inp["b_out"])
    z["W_down"] = np.zeros_like(inp["W_down"]); z["b_down"] = np.zeros_like(inp["b_down"])
    np.testing.assert_array_equal(block.residual_block(*_res_args(z))["out"], inp["u"])
    z2 = dict(inp)
    z2["W_down"] = z["W_down"]; z2["b_down"] = z["b_down"]
    o = block.residual_block(*_res_args(z2))
    n = block.round_bf16(block.rmsnorm(inp["u"], inp["w_temporal_norm"]))
    rb = block.recurrent_block(n, inp["W_lin_x"], inp["b_lin_x"], inp["W_lin_y"], inp["b_lin_y"],
                               np.zeros_like(inp["W_out"]), np.zeros(256), inp["conv_w"], inp["conv_b"],
                               inp["W_a"], inp["b_a"], inp["W_x"], inp["b_x"], inp["lam"], inp["segpos"],
                               inp["conv_state"], inp["h_state"])
    want_h = block.round_bf16(block.linear(rb["y"], inp["W_out"], inp["b_out"]) + inp["u"])
    np.testing.assert_array_equal(o["h"], want_h)
    np.testing.assert_array_equal(o["out"], want_h)
