"""Pins of the float64 oracle against facts that do not come from the oracle.

Each test checks one step of the block core against something independent:
a closed form, a library routine (numpy convolution, a dense matmul with the
assembled block-diagonal matrix, torch's tanh GELU, scipy's logistic), a
brute-force expansion, or an invariant of the definition.  A dropped term, a
wrong sign or index, a flipped conv kernel or a transposed weight matrix
fails at least one of them.
"""
import numpy as np
import pytest
import scipy.linalg
import scipy.special
import torch

from oracle import oracle
from lm_causal_depthwise_b200 import workloads as W

HEAD = 256


def _inputs(B=2, T=24, D=512, seed=7, io="f32", doc_len=None, reset_at=(0,),
            continue_doc=False, init_state="random", decay="init"):
    w = W.Workload("pin", B=B, T=T, D=D, io=io, seed=seed, doc_len=doc_len,
                   reset_at=reset_at, continue_doc=continue_doc, init_state=init_state,
                   decay=decay)
    inp = W.generate(w)
    return {k: (v.astype(np.float64) if v.dtype != np.int32 else v) for k, v in inp.items()}


def _run(inp, **kw):
    return oracle.prefill(**inp, **kw)


def _gelu_torch(g):
    return torch.nn.functional.gelu(torch.from_numpy(np.asarray(g, np.float64)),
                                    approximate="tanh").numpy()


def _block_diag(Wh):
    return scipy.linalg.block_diag(*[Wh[h] for h in range(Wh.shape[0])])


def _conv_np(inp, b, d, masked_state):
    """xc for one channel by numpy convolution of [conv_state, x] with the flipped kernel."""
    state = np.zeros(3) if masked_state else inp["conv_state"][b, :, d]
    seq = np.concatenate([state, inp["x"][b, :, d]])
    full = np.convolve(seq, inp["conv_w"][::-1, d])
    T = inp["x"].shape[1]
    return full[3:3 + T] + inp["conv_b"][d]


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("decay", ["init", "wide"])
def test_geometric_closed_form(decay):
    """W=0 gives constant gates; identity conv and a per-document constant
    input give h_{s+n} = i u (a^n + sqrt(1-a^2) (1-a^n)/(1-a)) after a reset at s.
    "wide" draws Lambda in [-10, 6.9], so both branches of log sigmoid(Lambda)
    and fast-decay channels (sigmoid(Lambda)^8 down to ~1e-35) are covered."""
    T, D = 40, 256
    inp = _inputs(B=1, T=T, D=D, reset_at=(0, 17), init_state="random", decay=decay)
    if decay == "wide":
        assert (inp["lam"] < -5).any() and (inp["lam"] > 5).any() and (inp["lam"] <= 6.91).all()
    inp["W_a"][:] = 0.0
    inp["W_x"][:] = 0.0
    inp["conv_w"][:] = 0.0
    inp["conv_w"][3] = 1.0
    inp["conv_b"][:] = 0.0
    rng = np.random.default_rng(3)
    u1, u2 = rng.standard_normal(D), rng.standard_normal(D)
    inp["x"][0, :17] = u1
    inp["x"][0, 17:] = u2
    out = _run(inp)
    r = scipy.special.expit(inp["b_a"])
    i = scipy.special.expit(inp["b_x"])
    a = np.power(scipy.special.expit(inp["lam"]), 8.0 * r)
    want = np.empty((T, D))
    for s, e, u in ((0, 17, u1), (17, T, u2)):
        n = np.arange(e - s)[:, None]
        an = a[None, :] ** n
        want[s:e] = i * u * (an + np.sqrt(1 - a * a) * (1 - an) / (1 - a))
    y_want = _gelu_torch(inp["g"][0]) * want
    np.testing.assert_allclose(out["y"][0], y_want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out["h_state"][0], want[-1], rtol=1e-12, atol=1e-14)


def test_decay_to_zero_gives_h_equals_i_xc():
    """With sigmoid(Lambda)^c -> 0 (c = 1e15) the decay vanishes and the
    normaliser is 1, so y = GELU(g) * sigmoid(W_x xc + b_x) * xc, computed here
    with numpy convolution and a dense matmul."""
    inp = _inputs(B=2, T=20, D=512, continue_doc=True)
    out = _run(inp, c=1e15)
    Wx = _block_diag(inp["W_x"])
    for b in range(2):
        xc = np.stack([_conv_np(inp, b, d, masked_state=False) for d in range(512)], axis=1)
        ig = scipy.special.expit(xc @ Wx.T + inp["b_x"])
        want = _gelu_torch(inp["g"][b]) * ig * xc
        np.testing.assert_allclose(out["y"][b], want, rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- library cross-checks

@pytest.mark.parametrize("continue_doc", [True, False])
def test_conv_matches_numpy_convolve(continue_doc):
    """Without mid-sequence resets the conv is numpy's convolution with the
    flipped kernel (tap 3 on the current token); a reset at t=0 masks the state."""
    inp = _inputs(B=2, T=30, D=256, continue_doc=continue_doc)
    out = _run(inp, trace=True)
    for b in range(2):
        for d in (0, 1, 77, 255):
            np.testing.assert_allclose(out["xc"][b, :, d],
                                       _conv_np(inp, b, d, masked_state=not continue_doc),
                                       rtol=1e-13, atol=1e-14)


def test_conv_mask_at_mid_reset():
    """Taps that would read before a document start are dropped: at segpos p<3
    only the taps with lag <= p remain."""
    inp = _inputs(B=1, T=16, D=256, reset_at=(0, 9))
    out = _run(inp, trace=True)
    w, x, bias = inp["conv_w"], inp["x"][0], inp["conv_b"]
    for t in (9, 10, 11, 12):
        p = t - 9
        want = bias + sum(w[3 - lag] * x[t - lag] for lag in range(0, min(p, 3) + 1))
        np.testing.assert_allclose(out["xc"][0, t], want, rtol=1e-13, atol=1e-14)


def test_gates_match_dense_block_diagonal_matmul():
    inp = _inputs(B=2, T=12, D=768)
    out = _run(inp, trace=True)
    Wa, Wx = _block_diag(inp["W_a"]), _block_diag(inp["W_x"])
    xc = out["xc"].reshape(-1, 768)
    np.testing.assert_allclose(out["r"].reshape(-1, 768),
                               scipy.special.expit(xc @ Wa.T + inp["b_a"]), rtol=1e-12)
    np.testing.assert_allclose(out["i"].reshape(-1, 768),
                               scipy.special.expit(xc @ Wx.T + inp["b_x"]), rtol=1e-12)


@pytest.mark.parametrize("decay", ["init", "wide"])
def test_decay_matches_power_form(decay):
    """a = sigmoid(Lambda)^(8 r) against scipy's logistic and numpy's power; the
    wide recipe puts half of the channels at Lambda < 0."""
    inp = _inputs(B=1, T=10, D=256, decay=decay)
    out = _run(inp, trace=True)
    want = np.power(scipy.special.expit(inp["lam"])[None, None, :], 8.0 * out["r"])
    np.testing.assert_allclose(out["a"], want, rtol=1e-13)


def test_decay_at_fixed_negative_lambda():
    """Lambda = -2 and -7 with constant gates (W = 0, b_a = 0 so r = 1/2):
    a = sigmoid(Lambda)^4 exactly, h after a reset is the geometric sum of the
    closed form, and the normaliser sqrt(1 - a^2) is evaluated at a ~ 1e-3
    and ~ 1e-12."""
    T, D = 12, 256
    inp = _inputs(B=1, T=T, D=D, reset_at=(0,), init_state="zero")
    inp["W_a"][:] = 0.0
    inp["W_x"][:] = 0.0
    inp["b_a"][:] = 0.0
    inp["conv_w"][:] = 0.0
    inp["conv_w"][3] = 1.0
    inp["conv_b"][:] = 0.0
    inp["lam"][:128] = -2.0
    inp["lam"][128:] = -7.0
    u = np.random.default_rng(5).standard_normal(D)
    inp["x"][0, :] = u
    out = _run(inp, trace=True)
    a = np.where(np.arange(D) < 128, (1.0 / (1.0 + np.exp(2.0))) ** 4, (1.0 / (1.0 + np.exp(7.0))) ** 4)
    np.testing.assert_allclose(out["a"][0], np.broadcast_to(a, (T, D)), rtol=1e-13)
    i = 1.0 / (1.0 + np.exp(-inp["b_x"]))
    n = np.arange(T)[:, None]
    an = a[None, :] ** n
    want = i * u * (an + np.sqrt(1 - a * a) * (1 - an) / (1 - a))
    np.testing.assert_allclose(out["h"][0], want, rtol=1e-12, atol=1e-15)


def test_gelu_is_torch_tanh_gelu():
    inp = _inputs(B=1, T=16, D=256, reset_at=(0, 5))
    out = _run(inp, trace=True)
    np.testing.assert_allclose(out["y"], _gelu_torch(inp["g"]) * out["h"], rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("T,resets", [(8, (0,)), (8, (0, 3)), (5, (0, 1, 2)), (7, (0, 6))])
@pytest.mark.parametrize("continue_doc", [False, True])
def test_bruteforce_expansion(T, resets, continue_doc):
    """h_t = sum_s (prod_{k=s+1..t} a_eff,k) m_s i_s xc_s + (prod_{k<=t} a_eff,k) h_{-1},
    with a_eff = 0, m = 1 at a reset and m = sqrt(1 - a^2) elsewhere."""
    inp = _inputs(B=1, T=T, D=256, reset_at=resets, continue_doc=continue_doc)
    out = _run(inp, trace=True)
    seg = inp["segpos"][0]
    a, i, xc = out["a"][0], out["i"][0], out["xc"][0]
    reset = (seg == 0)[:, None]
    a_eff = np.where(reset, 0.0, a)
    m = np.where(reset, 1.0, np.sqrt(1.0 - a * a))
    h0 = inp["h_state"][0]
    for t in range(T):
        acc = np.prod(a_eff[:t + 1], axis=0) * h0
        for s in range(t + 1):
            acc = acc + np.prod(a_eff[s + 1:t + 1], axis=0) * m[s] * i[s] * xc[s]
        np.testing.assert_allclose(out["h"][0, t], acc, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- invariants

def test_split_at_every_point_equals_whole_run():
    T = 13
    inp = _inputs(B=2, T=T, D=256, continue_doc=True)
    whole = _run(inp)
    for tau in range(1, T):
        a = {**inp, "x": inp["x"][:, :tau], "g": inp["g"][:, :tau], "segpos": inp["segpos"][:, :tau]}
        o1 = _run(a)
        b = {**inp, "x": inp["x"][:, tau:], "g": inp["g"][:, tau:], "segpos": inp["segpos"][:, tau:],
             "conv_state": o1["conv_state"], "h_state": o1["h_state"]}
        o2 = _run(b)
        y = np.concatenate([o1["y"], o2["y"]], axis=1)
        np.testing.assert_allclose(y, whole["y"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(o2["h_state"], whole["h_state"], rtol=1e-12, atol=1e-14)
        np.testing.assert_array_equal(o2["conv_state"], whole["conv_state"])


def test_reset_makes_output_independent_of_earlier_tokens():
    s = 11
    inp = _inputs(B=1, T=30, D=256, reset_at=(0, s))
    base = _run(inp)
    pert = {k: v.copy() for k, v in inp.items()}
    rng = np.random.default_rng(5)
    pert["x"][:, :s] += rng.standard_normal(pert["x"][:, :s].shape)
    pert["g"][:, :s] += rng.standard_normal(pert["g"][:, :s].shape)
    pert["h_state"] += 1.0
    pert["conv_state"] -= 2.0
    alt = _run(pert)
    np.testing.assert_array_equal(alt["y"][:, s:], base["y"][:, s:])
    np.testing.assert_array_equal(alt["h_state"], base["h_state"])
    assert not np.array_equal(alt["y"][:, :s], base["y"][:, :s])


def test_decode_steps_equal_prefill():
    T = 9
    inp = _inputs(B=3, T=T, D=256, reset_at=(0, 4))
    whole = _run(inp)
    cs, hs = inp["conv_state"], inp["h_state"]
    for t in range(T):
        o = oracle.decode_step(inp["x"][:, t], inp["g"][:, t], inp["conv_w"], inp["conv_b"],
                               inp["W_a"], inp["b_a"], inp["W_x"], inp["b_x"], inp["lam"],
                               inp["segpos"][:, t], cs, hs)
        np.testing.assert_array_equal(o["y"], whole["y"][:, t])
        cs, hs = o["conv_state"], o["h_state"]
    np.testing.assert_array_equal(hs, whole["h_state"])
    np.testing.assert_array_equal(cs, whole["conv_state"])


@pytest.mark.parametrize("T", [1, 2, 3, 4, 7])
def test_conv_state_out_is_last_three_raw_inputs(T):
    inp = _inputs(B=2, T=T, D=256, continue_doc=True)
    out = _run(inp)
    X = np.concatenate([inp["conv_state"], inp["x"]], axis=1)
    np.testing.assert_array_equal(out["conv_state"], X[:, -3:])


def test_units_equal_full_run():
    inp = _inputs(B=2, T=10, D=768, reset_at=(0, 4))
    full = _run(inp)
    for b in range(2):
        for h in range(3):
            u = oracle.prefill_unit(inp, b, h)
            s = slice(h * HEAD, (h + 1) * HEAD)
            np.testing.assert_array_equal(u["y"], full["y"][b, :, s])
            np.testing.assert_array_equal(u["h_state"], full["h_state"][b, s])
            np.testing.assert_array_equal(u["conv_state"], full["conv_state"][b, :, s])
    # truncation in time: outputs before t_end do not depend on later tokens
    u = oracle.prefill_unit(inp, 1, 2, t_end=6)
    np.testing.assert_array_equal(u["y"], full["y"][1, :6, 2 * HEAD:3 * HEAD])


def test_stationary_variance():
    """a^2 + (1-a^2) = 1: with i.i.d. scan inputs the state variance tends to
    var(i * xc) (statistical sanity check only)."""
    T, D = 20000, 256
    inp = _inputs(B=1, T=T, D=D, continue_doc=True, init_state="zero")
    inp["W_a"][:] = 0.0
    inp["W_x"][:] = 0.0
    inp["conv_w"][:] = 0.0
    inp["conv_w"][3] = 1.0
    inp["lam"][:] = 2.0
    out = _run(inp, trace=True)
    i = scipy.special.expit(inp["b_x"])
    var_h = out["h"][0, 2000:].var(axis=0)
    ratio = var_h / (i * i)
    assert abs(np.median(ratio) - 1.0) < 0.05


def test_rejects_bad_sizes():
    inp = _inputs(B=1, T=4, D=256)
    with pytest.raises(ValueError):
        oracle.prefill(**{**inp, "x": inp["x"][:, :, :200], "g": inp["g"][:, :, :200]})


def test_gate_operand_rounding_option():
    """gate_bf16=True rounds the conv output to the nearest bf16 (ties to even)
    where it enters the gate projections, and nowhere else.  Identity conv, so
    xc = x; x is built from bf16 values v plus 0.3, 0.7 and exactly 0.5 of the
    bf16 spacing at v, whose roundings are known: v, the next bf16 value up,
    and (a tie) whichever of the two has an even last mantissa bit."""
    T, D = 6, 256
    inp = _inputs(B=1, T=T, D=D, reset_at=(0,), init_state="zero")
    inp["conv_w"][:] = 0.0
    inp["conv_w"][3] = 1.0
    inp["conv_b"][:] = 0.0
    rng = np.random.default_rng(11)
    v = W.round_bf16(rng.standard_normal((T, D)).astype(np.float32)).astype(np.float64)
    mant, ex = np.frexp(v)
    ulp = np.ldexp(1.0, ex - 8)                       # bf16 spacing just above |v| (same sign)
    frac = np.array([0.3, 0.7, 0.5, 0.3, 0.7, 0.5])[:, None]
    x = v + np.sign(v) * frac * ulp
    odd = (np.abs(np.ldexp(mant, 8)).astype(np.int64) & 1) == 1
    up = (frac > 0.5) | ((frac == 0.5) & odd)
    q = np.where(up, v + np.sign(v) * ulp, v)
    inp["x"][0] = x
    out = _run(inp, trace=True, gate_bf16=True)
    np.testing.assert_array_equal(out["xc"][0], x)    # the conv itself stays exact
    Wa, Wx = inp["W_a"][0], inp["W_x"][0]
    np.testing.assert_allclose(out["r"][0], scipy.special.expit(q @ Wa.T + inp["b_a"]), rtol=1e-13)
    np.testing.assert_allclose(out["i"][0], scipy.special.expit(q @ Wx.T + inp["b_x"]), rtol=1e-13)
    # the scan uses the exact xc: at the reset token h = i * xc
    np.testing.assert_allclose(out["h"][0, 0], out["i"][0, 0] * x[0], rtol=1e-14)
    exact = _run(inp, trace=True)
    np.testing.assert_allclose(exact["r"][0], scipy.special.expit(x @ Wa.T + inp["b_a"]), rtol=1e-13)
    assert np.abs(exact["r"] - out["r"]).max() > 0
