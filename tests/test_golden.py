"""Golden fixtures: the structure the pages print, and an oracle regression digest."""
import json
import os

import numpy as np
import torch

from oracle import oracle
from lm_causal_depthwise_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_workloads_follow_printed_structure():
    s = _load("structure.json")
    w = W.PREFILL_2B
    assert w.D == s["rnn_width"] == s["conv1d"]["in_channels"] == s["conv1d"]["groups"]
    assert w.H == s["heads"] and W.HEAD == s["head_dim"]
    assert s["conv1d"]["kernel_size"] == 4 and s["conv1d"]["padding"] == 3
    inp = W.generate(w.scaled(B=1, T=4))
    assert inp["conv_w"].shape == (s["conv1d"]["kernel_size"], w.D)


def test_conv_is_printed_conv1d_truncated_causally():
    """The printed module Conv1d(D, D, kernel_size=4, padding=3, groups=D),
    as torch computes it, keeps its first T outputs: that is the oracle's conv
    for a sequence that starts a document (zero history)."""
    s = _load("structure.json")["conv1d"]
    D, T = 256, 40
    w = W.Workload("golden-conv", B=2, T=T, D=D, io="f32", seed=11, reset_at=(0,))
    inp = {k: (v.astype(np.float64) if v.dtype != np.int32 else v) for k, v in W.generate(w).items()}
    out = oracle.prefill(**inp, trace=True)
    conv = torch.nn.Conv1d(D, D, kernel_size=s["kernel_size"], stride=s["stride"],
                           padding=s["padding"], groups=D, dtype=torch.float64)
    with torch.no_grad():
        conv.weight.copy_(torch.from_numpy(inp["conv_w"].T.copy()).unsqueeze(1))
        conv.bias.copy_(torch.from_numpy(inp["conv_b"]))
        ref = conv(torch.from_numpy(inp["x"]).transpose(1, 2))[..., :T].transpose(1, 2).numpy()
    np.testing.assert_allclose(out["xc"], ref, rtol=1e-12, atol=1e-13)


def test_oracle_digest_unchanged():
    d = _load("tiny_f32_digest.json")
    out = oracle.prefill(**W.generate(W.TINY_F32))
    for idx, val in d["y_samples"]:
        assert out["y"][tuple(idx)] == val
    np.testing.assert_allclose(out["y"].sum(), d["y_sum"], rtol=1e-12)
    np.testing.assert_allclose((out["y"] ** 2).sum(), d["y_sumsq"], rtol=1e-12)
    np.testing.assert_allclose(out["h_state"].sum(), d["h_state_sum"], rtol=1e-12)
    np.testing.assert_allclose((out["h_state"] ** 2).sum(), d["h_state_sumsq"], rtol=1e-12)
    np.testing.assert_allclose(out["conv_state"].sum(), d["conv_state_sum"], rtol=1e-12, atol=1e-15)
