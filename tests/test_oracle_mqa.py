"""Pins of the local MQA oracle (oracle/mqa.py) against facts from outside it:
RoPE as a complex rotation, attention against torch's float64
scaled_dot_product_attention with an explicit mask and against a brute-force
loop, and the window and document limits by perturbation."""
import numpy as np
import torch

from oracle import mqa


def test_rope_is_a_complex_rotation():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 3, 16))
    pos = np.array([0, 1, 7, 100, 3])
    got = mqa.rope(x, pos, base=100.0)
    z = x[..., :8] + 1j * x[..., 8:]
    theta = pos[:, None, None] * 100.0 ** (-np.arange(8) * 2.0 / 16)
    w = z * np.exp(1j * theta)
    np.testing.assert_allclose(got, np.concatenate([w.real, w.imag], axis=-1), rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(mqa.rope(x[:1], [0]), x[:1])      # position 0: no rotation
    # rotations preserve norms and relative position: <R(p)q, R(p+m)k> depends on m only
    q, k = rng.standard_normal(16), rng.standard_normal(16)
    dots = [mqa.rope(q[None], [p])[0] @ mqa.rope(k[None], [p + 5])[0] for p in (0, 3, 40)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-12)


def _inputs(B=2, T=40, H=3, d=16, seed=2):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, T, H, d)), rng.standard_normal((B, T, d)), rng.standard_normal((B, T, d)))


def test_attention_matches_torch_sdpa_with_explicit_mask():
    q, k, v = _inputs()
    B, T, H, d = q.shape
    seg = np.stack([np.arange(T), np.where(np.arange(T) < 13, np.arange(T), np.arange(T) - 13)]).astype(np.int32)
    window = 9
    got = mqa.attention(q, k, v, seg, window)
    for b in range(B):
        t, s = np.arange(T)[:, None], np.arange(T)[None, :]
        allowed = (s <= t) & (s > t - window) & (s >= t - seg[b][:, None])
        qt = torch.from_numpy(q[b]).permute(1, 0, 2)                     # [H, T, d]
        kt = torch.from_numpy(k[b])[None].expand(H, T, d)
        vt = torch.from_numpy(v[b])[None].expand(H, T, d)
        want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(allowed))
        np.testing.assert_allclose(got[b], want.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_window_and_document_limits():
    """Changing a key just outside a query's window, or before its document
    start, leaves that query's output unchanged; changing one inside moves it."""
    q, k, v = _inputs(B=1, T=30)
    seg = np.where(np.arange(30) < 20, np.arange(30), np.arange(30) - 20)[None].astype(np.int32)
    base = mqa.attention(q, k, v, seg, window=6)
    # query 18: window keys 13..18; query 25 (its document starts at 20): keys 20..25
    for key, query, moves in ((12, 18, False), (13, 18, True), (19, 18, False), (19, 25, False),
                              (20, 25, True)):
        k2, v2 = k.copy(), v.copy()
        k2[0, key] += 1.0
        v2[0, key] += 1.0
        alt = mqa.attention(q, k2, v2, seg, window=6)
        assert (not np.allclose(alt[0, query], base[0, query])) == moves, (key, query, moves)


def test_single_key_copies_its_value():
    """A query at a document start attends only itself: the output is its v."""
    q, k, v = _inputs(B=1, T=5)
    seg = np.zeros((1, 5), np.int32)
    out = mqa.attention(q, k, v, seg)
    np.testing.assert_allclose(out[0], np.broadcast_to(v[0][:, None, :], out[0].shape), rtol=1e-14)


def test_attention_rows_equal_the_full_evaluation():
    """The row-sampled form (used at full sizes) gives the rows of attention()."""
    q, k, v = _inputs(B=2, T=50)
    seg = np.stack([np.arange(50), np.where(np.arange(50) < 31, np.arange(50), np.arange(50) - 31)]).astype(np.int32)
    full = mqa.attention(q, k, v, seg, window=11)
    rows = [(0, 0), (0, 10), (0, 49), (1, 30), (1, 31), (1, 45)]
    got = mqa.attention_rows(q, k, v, seg, rows, window=11)
    for n, (b, t) in enumerate(rows):
        np.testing.assert_allclose(got[n], full[b, t], rtol=1e-13, atol=1e-13)


def test_document_begun_before_the_call_attends_from_token_zero():
    """segment_pos above t (a document continuing from before the call): the
    keys are those of the call, so the result equals a document starting at
    token 0 (torch SDPA with the causal mask alone, window wider than T)."""
    q, k, v = _inputs(B=1, T=20)
    seg = (np.arange(20) + 7)[None].astype(np.int32)
    got = mqa.attention(q, k, v, seg, window=64)
    allowed = np.tril(np.ones((20, 20), bool))
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[0]).permute(1, 0, 2), torch.from_numpy(k[0])[None].expand(3, 20, 16),
        torch.from_numpy(v[0])[None].expand(3, 20, 16), attn_mask=torch.from_numpy(allowed))
    np.testing.assert_allclose(got[0], want.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(mqa.attention_rows(q, k, v, seg, [(0, 5), (0, 19)], window=64),
                               got[0, [5, 19]], rtol=1e-13, atol=1e-13)


def _res_inputs(seed=11, B=1, T=24, D=512):
    from lm_causal_depthwise_b200 import workloads as W
    w = W.Workload("res-mqa", B=B, T=T, D=D, io="bf16", seed=seed, doc_len=10)
    return W.generate_mqa_residual(w)


def _res(inp, **over):
    keys = ("u", "w_temporal_norm", "W_q", "W_k", "W_v", "W_o", "b_o", "segpos", "w_channel_norm", "W_gate",
            "b_gate", "W_up", "b_up", "W_down", "b_down")
    args = [over.get(k, inp[k]) for k in keys]
    return mqa.mqa_residual_block(*args, window=16)


def test_mqa_residual_block_wiring():
    """Zero projections leave the residual paths: out = u; with a zero MLP,
    out = h = u + o_proj(attention of the normalised u) (the MQA block's own
    pinned pieces); with a zero o_proj, h = u and out = u + MLP(RMSNorm(u))."""
    from oracle import block
    inp = _res_inputs()
    D, F = inp["W_o"].shape[0], inp["W_gate"].shape[0]
    zD, zDD, zDF, zF = np.zeros(D), np.zeros((D, D)), np.zeros((D, F)), np.zeros(F)
    r = _res(inp, W_o=zDD, b_o=zD, W_down=zDF, b_down=zD)
    np.testing.assert_array_equal(r["out"], inp["u"])
    r = _res(inp, W_down=zDF, b_down=zD)
    n = block.round_bf16(block.rmsnorm(inp["u"], inp["w_temporal_norm"], 1e-6))
    a = mqa.mqa_block(n, inp["W_q"], inp["W_k"], inp["W_v"], inp["W_o"], inp["b_o"], inp["segpos"], 16)["a"]
    B, T, _ = inp["u"].shape
    h = block.round_bf16(block.linear(a.reshape(B, T, -1), inp["W_o"], inp["b_o"]) + inp["u"])
    np.testing.assert_array_equal(r["out"], h)
    r = _res(inp, W_o=zDD, b_o=zD)
    n2 = block.round_bf16(block.rmsnorm(inp["u"], inp["w_channel_norm"], 1e-6))
    m = block.round_bf16(block.gelu_tanh(block.linear(n2, inp["W_gate"], inp["b_gate"]))
                         * block.linear(n2, inp["W_up"], inp["b_up"]))
    np.testing.assert_array_equal(r["out"], block.round_bf16(block.linear(m, inp["W_down"], inp["b_down"]) + inp["u"]))
