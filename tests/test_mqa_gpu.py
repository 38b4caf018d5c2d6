"""GPU parity of the local sliding-window MQA path (rglru_mqa_rope,
rglru_mqa_attention, rglru_mqa_block_prefill) against the float64 oracle
(oracle/mqa.py), through the C ABI.

Bars, from the arithmetic of each kernel:
  RoPE     the rotation of bf16 inputs in fp32 (angles reduced in fp64), one
           bf16 rounding: |got - ref| <= 2^-8 |ref| + 1e-5 (a rounding that
           lands on the other side of a bf16 tie costs one ulp, 2^-8 relative);
           v_t is a copy: bit-exact, its padding zero.
  attention scores and sums in fp32, the probabilities rounded to bf16 as
           the operand of P V (relative 2^-9 each), the output rounded to bf16:
           |got - ref| <= 2^-9 max|v| + 2^-8 |ref| + 1e-6.
  block    the core's bf16 bar (atol 2e-2, rtol 1e-2): the projections add
           bf16 roundings of their own on either side of the attention.
The attention tests draw q, k and v on the host in bf16 and give the same
values to both sides (the oracle's input never comes from the CUDA path).
Masking is checked where one key matters: windows of 17 to 200 keys and
documents of 30 to 100 tokens, and sharp score distributions (queries scaled
by 4) where the output follows a few keys and the running maximum is raised
and O rescaled several times per row.
"""
import numpy as np
import pytest
import torch

from lm_causal_depthwise_b200 import api, workloads as W
from oracle import mqa as omqa

from parity_util import check_bf16

pytestmark = pytest.mark.gpu

dev = "cuda"
bf = torch.bfloat16


def _segpos(rng, B, T, doc_len):
    w = W.Workload("mqa-case", B=B, T=T, D=256, io="bf16", seed=0, doc_len=doc_len)
    return W.segment_positions(rng, w)


def _qkv(B, T, H, seed, doc_len=None, q_scale=1.0):
    rng = np.random.default_rng(seed)
    seg = _segpos(rng, B, T, doc_len)
    qkv = rng.standard_normal((B, T, (H + 2) * 256), dtype=np.float32)
    qkv[..., :H * 256] *= q_scale
    return W.round_bf16(qkv), seg


def _split(qkv, H):
    B, T, _ = qkv.shape
    return (qkv[..., :H * 256].reshape(B, T, H, 256), qkv[..., H * 256:(H + 1) * 256], qkv[..., (H + 1) * 256:])


def _vt_host(v):
    """v [B, T, 256] -> [B, 256, Tp] with zero padding (input marshalling for the kernel)."""
    B, T, _ = v.shape
    Tp = (T + 7) // 8 * 8
    out = np.zeros((B, 256, Tp), np.float32)
    out[:, :, :T] = np.transpose(v, (0, 2, 1))
    return out


def _attn_bar(got, want, vmax, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    err = np.abs(got - want)
    bad = ~(err <= 2.0 ** -9 * vmax + 2.0 ** -8 * np.abs(want) + 1e-6)
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside, max err {err.max():.3e}"


def _run_attention(qkv, seg, H, window):
    B, T, _ = qkv.shape
    _, _, v = _split(qkv, H)
    dq = torch.from_numpy(qkv).to(dev).to(bf).contiguous()
    dvt = torch.from_numpy(_vt_host(v)).to(dev).to(bf).contiguous()
    ds = torch.from_numpy(seg).to(dev).contiguous()
    ws = api.linear_workspace(dev)
    out = api.mqa_attention(dq, dvt, ds, window, workspace=ws)
    assert api.device_status(ws) == api.OK
    return out.float().cpu().numpy()


@pytest.mark.parametrize("B,T,H,doc_len,offset", [(2, 77, 2, 30, 0), (1, 300, 10, None, 0), (3, 1000, 1, 200, 0),
                                                  (1, 129, 2, None, 100000)])
def test_rope_and_v_transpose(B, T, H, doc_len, offset):
    qkv, seg = _qkv(B, T, H, seed=1, doc_len=doc_len)
    seg = (seg + offset).astype(np.int32)   # offset: positions up to 1e5 (angle reduction)
    dq = torch.from_numpy(qkv).to(dev).to(bf).contiguous()
    ds = torch.from_numpy(seg).to(dev)
    vt = api.mqa_rope(dq, ds)
    got = dq.float().cpu().numpy()
    q, k, v = _split(qkv, H)
    want_q = omqa.rope(q, seg).reshape(B, T, H * 256)
    want_k = omqa.rope(k, seg)
    for g, w_, name in ((got[..., :H * 256], want_q, "q"), (got[..., H * 256:(H + 1) * 256], want_k, "k")):
        err = np.abs(g - w_)
        bad = ~(err <= 2.0 ** -8 * np.abs(w_) + 1e-5)
        assert not bad.any(), f"rope {name}: {int(bad.sum())} outside, max err {err.max():.3e}"
    np.testing.assert_array_equal(got[..., (H + 1) * 256:], qkv[..., (H + 1) * 256:])   # v untouched
    np.testing.assert_array_equal(vt.float().cpu().numpy(), _vt_host(v))


@pytest.mark.parametrize("B,T,H,window,doc_len,q_scale", [
    (2, 300, 2, 2048, 100, 1.0),     # ragged T, documents
    (1, 1000, 3, 200, None, 1.0),    # window edge crossing the key tiles
    (1, 1000, 2, 17, None, 1.0),     # window inside one key tile
    (2, 700, 2, 2048, None, 4.0),    # sharp scores: reference max raised, O rescaled
    (1, 2600, 2, 2048, 900, 1.0),    # the 2048-key window reached
    (1, 2600, 1, 2048, None, 4.0),   # one document, full window, sharp
    (3, 129, 10, 64, 30, 1.0),       # 10 heads, one tile plus one row
    (1, 1, 1, 2048, None, 1.0),      # one token
    (2, 64, 2, 2048, None, 1.0),     # exactly one key tile
])
def test_attention_matches_oracle(B, T, H, window, doc_len, q_scale):
    qkv, seg = _qkv(B, T, H, seed=2, doc_len=doc_len, q_scale=q_scale)
    got = _run_attention(qkv, seg, H, window)
    q, k, v = _split(qkv, H)
    want = omqa.attention(q, k, v, seg, window).reshape(B, T, H * 256)
    _attn_bar(got, want, np.abs(v).max(), f"attention B={B} T={T} H={H} window={window}")


def test_attention_document_begun_before_the_call():
    """segment_pos above t: the keys start at token 0 of the call."""
    B, T, H = 1, 300, 2
    qkv, _ = _qkv(B, T, H, seed=3)
    seg = (np.arange(T) + 50)[None].astype(np.int32)
    got = _run_attention(qkv, seg, H, 2048)
    q, k, v = _split(qkv, H)
    _attn_bar(got, omqa.attention(q, k, v, seg, 2048).reshape(B, T, H * 256), np.abs(v).max(), "continued doc")


def test_attention_full_size_sampled_rows():
    """The 2B shape (B=8, T=4096, 10 heads, documents of mean length 1024,
    window 2048) in the benchmark's launch configuration; rows sampled at the
    first and last row of query tiles, around key-tile edges and after
    document starts, every head, against the oracle row by row."""
    B, T, H = 8, 4096, 10
    qkv, seg = _qkv(B, T, H, seed=4, doc_len=1024, q_scale=2.0)
    got = _run_attention(qkv, seg, H, 2048)
    q, k, v = _split(qkv, H)
    rng = np.random.default_rng(5)
    rows = []
    for b in (0, 3, 7):
        ts = {0, 1, 63, 64, 127, 128, 2047, 2048, 2175, 4095} | set(rng.integers(0, T, 12).tolist())
        starts = np.flatnonzero(seg[b] == 0)
        ts |= {int(s) for s in starts} | {int(min(s + 1, T - 1)) for s in starts}
        rows += [(b, int(t)) for t in sorted(ts)]
    want = omqa.attention_rows(q, k, v, seg, rows, 2048)
    got_rows = np.stack([got[b, t].reshape(H, 256) for b, t in rows])
    _attn_bar(got_rows, want, np.abs(v).max(), "attention full size")


def test_attention_rejects_bad_arguments():
    qkv = torch.zeros((1, 10, 768), dtype=bf, device=dev)
    vt = api.mqa_vt(1, 10)
    sp = torch.zeros((1, 10), dtype=torch.int32, device=dev)
    with pytest.raises(api.RGLRUError):
        api.mqa_attention(qkv, vt, sp, window=0)
    with pytest.raises(api.RGLRUError):   # workspace smaller than the status header
        api.mqa_attention(qkv, vt, sp, workspace=torch.zeros(16, dtype=torch.uint8, device=dev))


def _oracle_block(inp, window):
    return omqa.mqa_block(inp["u"], inp["W_q"], inp["W_k"], inp["W_v"], inp["W_o"], inp["b_o"], inp["segpos"],
                          window)


@pytest.mark.parametrize("B,T,D,doc_len,window", [(2, 300, 512, 100, 2048), (1, 700, 2560, 250, 2048),
                                                  (2, 200, 768, None, 50)])
def test_mqa_block_matches_oracle(B, T, D, doc_len, window):
    w = W.Workload("mqa-block", B=B, T=T, D=D, io="bf16", seed=6, doc_len=doc_len)
    inp = W.generate_mqa(w)
    mp = api.MQAParams.from_arrays(inp, dev)
    u = torch.from_numpy(inp["u"]).to(dev).to(bf)
    sp = torch.from_numpy(inp["segpos"]).to(dev)
    ws = api.new_workspace(api.mqa_block_workspace_size(B, T, D), dev)
    out = api.mqa_block_prefill(u, mp, sp, window, workspace=ws)
    assert api.device_status(ws) == api.OK
    ref = _oracle_block(inp, window)
    check_bf16(out.float().cpu().numpy(), ref["out"], "mqa block out")


@pytest.mark.parametrize("B,T,H,window,doc_len", [(2, 300, 2, 128, None), (3, 200, 10, 2048, 60),
                                                  (1, 700, 3, 256, 300), (2, 140, 16, 128, None)])
def test_decode_steps_match_oracle(B, T, H, window, doc_len):
    """T decode steps from empty rings (windows of 128 and 256 wrap the ring;
    16 heads is the 9B shape's count): each step's output against the oracle's
    attention over the same rotated, bf16-rounded q, k and v; the rings hold
    the rotated keys and the values at slot position % window."""
    qkv, seg = _qkv(B, T, H, seed=7, doc_len=doc_len)
    dq = torch.from_numpy(qkv).to(dev).to(bf)
    ds = torch.from_numpy(seg).to(dev)
    kc, vc = api.mqa_cache(B, window, dev)
    ws = api.new_workspace(api.mqa_decode_workspace_size(B, H, window), dev)
    outs = []
    for t in range(T):
        outs.append(api.mqa_decode_step(dq[:, t].contiguous(), ds[:, t].contiguous(), kc, vc, workspace=ws))
    got = torch.stack(outs, 1).float().cpu().numpy()
    q, k, v = _split(qkv, H)
    from oracle import block as oblock
    qr, kr = oblock.round_bf16(omqa.rope(q, seg)), oblock.round_bf16(omqa.rope(k, seg))
    want = omqa.attention(qr, kr, v, seg, window).reshape(B, T, H * 256)
    _attn_bar(got, want, np.abs(v).max(), f"decode B={B} T={T} H={H} window={window}")
    # the ring after the last step: slot p % window holds position p of the last document
    # (k against the unrounded rotation: the kernel's fp32 rotation may round
    # to the other neighbour of a tie, which the RoPE bar allows)
    k_exact = omqa.rope(k, seg)
    kcn, vcn = kc.float().cpu().numpy(), vc.float().cpu().numpy()
    for b in range(B):
        t_last = T - 1
        p_last = int(seg[b, t_last])
        for back in range(min(p_last + 1, window)):
            t = t_last - back
            slot = (p_last - back) % window
            np.testing.assert_array_equal(vcn[b, :, slot], v[b, t])
            err = np.abs(kcn[b, slot] - k_exact[b, t])
            assert (err <= 2.0 ** -8 * np.abs(k_exact[b, t]) + 1e-5).all(), (b, t, float(err.max()))


def test_decode_equals_prefill_rows():
    """The decode step and the prefill kernels compute the same attention: the
    last tokens of a sequence decoded one by one against the prefill's rows."""
    B, T, H = 2, 400, 4
    qkv, seg = _qkv(B, T, H, seed=8, doc_len=150)
    dq = torch.from_numpy(qkv).to(dev).to(bf)
    ds = torch.from_numpy(seg).to(dev)
    pre_q = dq.clone()
    vt = api.mqa_rope(pre_q, ds)
    pre = api.mqa_attention(pre_q, vt, ds).float().cpu().numpy()
    kc, vc = api.mqa_cache(B, 2048, dev)
    dec = [api.mqa_decode_step(dq[:, t].contiguous(), ds[:, t].contiguous(), kc, vc).float().cpu().numpy()
           for t in range(T)]
    dec = np.stack(dec, 1)
    _, _, v = _split(qkv, H)
    # each side is within the attention bar of the exact value: twice the bar between them
    err = np.abs(dec - pre)
    bad = ~(err <= 2.0 ** -8 * np.abs(v).max() + 2.0 ** -7 * np.abs(pre) + 2e-6)
    assert not bad.any(), f"decode vs prefill: {int(bad.sum())} outside, max err {err.max():.3e}"


def test_mqa_write_coverage_and_canaries():
    """RoPE, attention and the decode step write every element of their
    outputs and nothing past the end of out, v_t or the rings."""
    B, T, H, pad = 2, 333, 3, 2048
    qkv, seg = _qkv(B, T, H, seed=9, doc_len=100)
    dq = torch.from_numpy(qkv).to(dev).to(bf)
    ds = torch.from_numpy(seg).to(dev)
    Tp = (T + 7) // 8 * 8
    vtb = torch.full((B * 256 * Tp + pad,), float("nan"), dtype=bf, device=dev)
    vt = api.mqa_rope(dq, ds, vtb[:B * 256 * Tp].view(B, 256, Tp))
    outb = torch.full((B * T * H * 256 + pad,), float("nan"), dtype=bf, device=dev)
    out = api.mqa_attention(dq, vt, ds, out=outb[:B * T * H * 256].view(B, T, H * 256))
    torch.cuda.synchronize()
    assert not torch.isnan(vt).any() and torch.isnan(vtb[B * 256 * Tp:]).all()
    assert not torch.isnan(out).any() and torch.isnan(outb[B * T * H * 256:]).all()
    W = 128
    kcb = torch.full((B * W * 256 + pad,), float("nan"), dtype=bf, device=dev)
    vcb = torch.full((B * W * 256 + pad,), float("nan"), dtype=bf, device=dev)
    kc, vc = kcb[:B * W * 256].view(B, W, 256), vcb[:B * W * 256].view(B, 256, W)
    kc.zero_()
    vc.zero_()
    dob = torch.full((B * H * 256 + pad,), float("nan"), dtype=bf, device=dev)
    raw = torch.from_numpy(qkv).to(dev).to(bf)
    for t in range(160):
        o = api.mqa_decode_step(raw[:, t].contiguous(), ds[:, t].contiguous(), kc, vc,
                                out=dob[:B * H * 256].view(B, H * 256))
    torch.cuda.synchronize()
    assert not torch.isnan(o).any() and torch.isnan(dob[B * H * 256:]).all()
    assert torch.isnan(kcb[B * W * 256:]).all() and torch.isnan(vcb[B * W * 256:]).all()


@pytest.mark.parametrize("B,T,D,doc_len,window", [(2, 300, 512, 100, 2048), (1, 500, 2560, 200, 128)])
def test_mqa_residual_block_matches_oracle(B, T, D, doc_len, window):
    """The residual block with local MQA against the oracle.  As for the
    recurrent residual block, an error of the temporal block's size passes
    through o_proj into h and again through the MLP into out: out is held to
    twice the bf16 bar (atol 4e-2, rtol 2e-2)."""
    w = W.Workload("mqa-res", B=B, T=T, D=D, io="bf16", seed=10, doc_len=doc_len)
    inp = W.generate_mqa_residual(w)
    rp = api.MQAResidualParams.from_arrays(inp, dev)
    u = torch.from_numpy(inp["u"]).to(dev).to(bf)
    sp = torch.from_numpy(inp["segpos"]).to(dev)
    ws = api.new_workspace(api.mqa_residual_block_workspace_size(B, T, D, rp.W_gate.shape[0]), dev)
    out = api.mqa_residual_block_prefill(u, rp, sp, window, workspace=ws)
    assert api.device_status(ws) == api.OK
    keys = ("u", "w_temporal_norm", "W_q", "W_k", "W_v", "W_o", "b_o", "segpos", "w_channel_norm", "W_gate",
            "b_gate", "W_up", "b_up", "W_down", "b_down")
    ref = omqa.mqa_residual_block(*[inp[k] for k in keys], window=window)
    got, want = out.float().cpu().numpy().astype(np.float64), ref["out"]
    bad = ~(np.abs(got - want) <= 4e-2 + 2e-2 * np.abs(want))
    assert not bad.any(), f"mqa residual block: {int(bad.sum())} of {bad.size} outside, max {np.abs(got - want).max():.3e}"
