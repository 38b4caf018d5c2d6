"""GPU parity of the dense projections (rglru_linear*) and of the whole
recurrent block (rglru_recurrent_block_prefill).

The projections are checked against a plain PyTorch fp32 evaluation of the
same bf16 operands (the GEMM's own contract: fp32 accumulation, one bf16
rounding of the result), every element, at ragged and full sizes.  The block
is checked against the float64 oracle (oracle/block.py), every element, with
the bf16 bar of the core.
"""
import numpy as np
import pytest
import torch

from lm_causal_depthwise_b200 import api, workloads as W
from oracle import block as oblock

from parity_util import check_bf16

pytestmark = pytest.mark.gpu

dev = "cuda"


def _rand(shape, scale=1.0, seed=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).to(dev)


def _ref_linear(A, Wt, b=None):
    out = A.float() @ Wt.float().T
    if b is not None:
        out = out + b
    return out


def _close(got, want, what):
    """bf16 output of an fp32 accumulation: within the bf16 rounding of the
    result plus fp32 summation-order differences."""
    got, want = got.float(), want.float()
    bad = ~((got - want).abs() <= 1e-2 * want.abs() + 1e-2)
    assert not bool(bad.any()), f"{what}: {int(bad.sum())} bad of {bad.numel()}, max {float((got - want).abs().max()):.3e}"


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (127, 256, 128), (129, 512, 512), (300, 768, 2560),
                                   (4096, 2560, 2560)])
def test_linear(M, N, K):
    A = _rand((M, K), seed=1)
    Wt = _rand((N, K), scale=K ** -0.5, seed=2)
    b = torch.randn(N, device=dev) * 0.3
    ws = api.linear_workspace()
    out = api.linear(A, Wt, b, workspace=ws)
    assert api.device_status(ws) == api.OK
    _close(out, _ref_linear(A, Wt, b), f"linear {M}x{N}x{K}")
    out2 = api.linear(A, Wt, None, workspace=ws)  # no bias
    _close(out2, _ref_linear(A, Wt), "linear without bias")


def test_linear_pair_is_two_linears():
    M, N, K = 777, 512, 512
    A = _rand((M, K), seed=3)
    W0, W1 = _rand((N, K), K ** -0.5, 4), _rand((N, K), K ** -0.5, 5)
    b0, b1 = torch.randn(N, device=dev), torch.randn(N, device=dev)
    o0, o1 = api.linear_pair(A, W0, b0, W1, b1)
    torch.cuda.synchronize()
    assert torch.equal(o0, api.linear(A, W0, b0))
    assert torch.equal(o1, api.linear(A, W1, b1))
    _close(o1, _ref_linear(A, W1, b1), "pair out1")


@pytest.mark.parametrize("inplace", [False, True])
def test_linear_residual(inplace):
    M, N, K = 333, 512, 768
    A = _rand((M, K), seed=6)
    Wt = _rand((N, K), K ** -0.5, 7)
    b = torch.randn(N, device=dev)
    res = _rand((M, N), seed=8)
    want = _ref_linear(A, Wt, b) + res.float()
    out = api.linear_residual(A, Wt, b, res, out=res if inplace else None)
    _close(out, want, "residual")
    if inplace:
        assert out.data_ptr() == res.data_ptr()


def test_linear_geglu():
    M, N, K = 300, 384, 512
    A = _rand((M, K), seed=9)
    Wg, Wu = _rand((N, K), K ** -0.5, 10), _rand((N, K), K ** -0.5, 11)
    bg, bu = torch.randn(N, device=dev) * 0.3, torch.randn(N, device=dev) * 0.3
    out = api.linear_geglu(A, Wg, bg, Wu, bu)
    g = _ref_linear(A, Wg, bg)
    want = torch.nn.functional.gelu(g, approximate="tanh") * _ref_linear(A, Wu, bu)
    _close(out, want, "geglu")


def test_linear_rejects_unsupported_sizes():
    A = _rand((10, 100))
    Wt = _rand((256, 100))
    with pytest.raises(api.RGLRUError):
        api.linear(A, Wt)          # K not a multiple of 64
    with pytest.raises(api.RGLRUError):
        api.linear(_rand((10, 128)), _rand((100, 128)))  # N not a multiple of 256


def _block_case(B, T, D, seed=12, doc_len=None):
    w = W.Workload("block", B=B, T=T, D=D, io="bf16", seed=seed, doc_len=doc_len, init_state="random")
    return W.generate_block(w)


def _run_block(inp):
    bp = api.BlockParams.from_arrays(inp, dev)
    u = torch.from_numpy(inp["u"]).to(dev).to(torch.bfloat16)
    sp = torch.from_numpy(inp["segpos"]).to(dev)
    cs = torch.from_numpy(inp["conv_state"]).to(dev).to(torch.bfloat16)
    hs = torch.from_numpy(inp["h_state"]).to(dev)
    ws = api.new_workspace(api.recurrent_block_workspace_size(*u.shape), dev)
    out = api.recurrent_block_prefill(u, bp, sp, cs, hs, workspace=ws)
    assert api.device_status(ws) == api.OK
    return out.float().cpu().numpy(), cs.float().cpu().numpy(), hs.cpu().numpy()


def _oracle_block(inp):
    keys = ("u", "W_lin_x", "b_lin_x", "W_lin_y", "b_lin_y", "W_out", "b_out", "conv_w", "conv_b", "W_a", "b_a",
            "W_x", "b_x", "lam", "segpos", "conv_state", "h_state")
    return oblock.recurrent_block(*[inp[k] for k in keys])


@pytest.mark.parametrize("B,T,D,doc_len", [(2, 300, 512, 100), (1, 1000, 2560, 400), (3, 129, 768, None)])
def test_recurrent_block_matches_oracle(B, T, D, doc_len):
    inp = _block_case(B, T, D, doc_len=doc_len)
    out, cs, hs = _run_block(inp)
    ref = _oracle_block(inp)
    check_bf16(out, ref["out"], "block out")
    check_bf16(hs, ref["h_state"], "block h_state")
    # the conv state holds the last three rows of x = linear_x(u): a GEMM
    # output, rounded to bf16 from fp32 here and from float64 in the oracle,
    # so it is compared with the bf16 bar rather than bit for bit
    check_bf16(cs, ref["conv_state"], "block conv_state")


def test_recurrent_block_full_size_sampled_rows():
    """The 2B-shaped block (B=8, T=4096, D=2560) in the benchmark's launch
    configuration; every output of two whole sequences against the oracle
    (rows are independent)."""
    w = W.PREFILL_2B
    inp = W.generate_block(w)
    out, cs, hs = _run_block(inp)
    for b in (0, 5):
        sub = {k: (v[b:b + 1] if k in ("u", "segpos", "conv_state", "h_state") else v) for k, v in inp.items()}
        ref = _oracle_block(sub)
        check_bf16(out[b:b + 1], ref["out"], f"block row {b}")
        check_bf16(hs[b:b + 1], ref["h_state"], f"block h row {b}")
        check_bf16(cs[b:b + 1], ref["conv_state"], f"block conv_state row {b}")


@pytest.mark.parametrize("M,N", [(1, 8), (37, 256), (1000, 2560), (5, 4096), (300, 7680 // 3)])
def test_rmsnorm(M, N):
    x = _rand((M, N), scale=3.0, seed=13)
    w = torch.randn(N, device=dev) * 0.2 + 1.0
    out = api.rmsnorm(x, w, 1e-6)
    want = torch.nn.functional.rms_norm(x.float(), (N,), w, eps=1e-6)
    _close(out, want, f"rmsnorm {M}x{N}")
    y = x.clone()
    api.rmsnorm(y, w, 1e-6, out=y)   # in place
    assert torch.equal(y, out)


def _res_inputs(B, T, D, doc_len=None, seed=14):
    w = W.Workload("res", B=B, T=T, D=D, io="bf16", seed=seed, doc_len=doc_len, init_state="random")
    return W.generate_residual_block(w)


def _run_res(inp):
    rp = api.ResidualBlockParams.from_arrays(inp, dev)
    u = torch.from_numpy(inp["u"]).to(dev).to(torch.bfloat16)
    sp = torch.from_numpy(inp["segpos"]).to(dev)
    cs = torch.from_numpy(inp["conv_state"]).to(dev).to(torch.bfloat16)
    hs = torch.from_numpy(inp["h_state"]).to(dev)
    B, T, D = u.shape
    ws = api.new_workspace(api.residual_block_workspace_size(B, T, D, rp.W_gate.shape[0]), dev)
    out = api.residual_block_prefill(u, rp, sp, cs, hs, workspace=ws)
    assert api.device_status(ws) == api.OK
    return out.float().cpu().numpy(), cs.float().cpu().numpy(), hs.cpu().numpy()


def _oracle_res(inp):
    keys = ("u", "w_temporal_norm", "W_lin_x", "b_lin_x", "W_lin_y", "b_lin_y", "W_out", "b_out", "conv_w",
            "conv_b", "W_a", "b_a", "W_x", "b_x", "lam", "segpos", "conv_state", "h_state", "w_channel_norm",
            "W_gate", "b_gate", "W_up", "b_up", "W_down", "b_down")
    return oblock.residual_block(*[inp[k] for k in keys])


@pytest.mark.parametrize("B,T,D,doc_len", [(2, 300, 512, 100), (1, 600, 2560, 250)])
def test_residual_block_matches_oracle(B, T, D, doc_len):
    """The residual block composes the core (whose bar allows 2e-2 + 1e-2 |y|
    per element of y) with linear_out, a residual add, RMSNorm and the
    two-stage MLP, each output rounded to bf16: an error of the core's size in
    y passes through linear_out into h and again through the MLP into out, so
    out is held to twice the core's bar (atol 4e-2, rtol 2e-2).  The states
    come from the core alone and keep its bar."""
    inp = _res_inputs(B, T, D, doc_len)
    out, cs, hs = _run_res(inp)
    ref = _oracle_res(inp)
    got, want = np.asarray(out, np.float64), np.asarray(ref["out"], np.float64)
    bad = ~(np.abs(got - want) <= 4e-2 + 2e-2 * np.abs(want))
    assert not bad.any(), f"residual block out: {int(bad.sum())} of {bad.size} outside, max {np.abs(got - want).max():.3e}"
    check_bf16(hs, ref["h_state"], "residual block h_state")
    check_bf16(cs, ref["conv_state"], "residual block conv_state")
