"""rglru_prefill_noalloc: the prefill for callers that cannot allocate device
memory (its scratch is the library's own fixed device array).  Collected last
so that a run stopping at the first failure has run every other test first.
The call goes through the C ABI and must match rglru_prefill, which uses a
caller-provided workspace, on two calls in a row (the second one reuses the
scratch the first one left behind)."""
import numpy as np
import pytest
import torch

from lm_causal_depthwise_b200 import api, workloads as W

from parity_util import check_bf16, to_device

pytestmark = pytest.mark.gpu


def _inputs():
    w = W.Workload("noalloc", B=2, T=1000, D=512, io="bf16", seed=31, doc_len=300,
                   init_state="random")
    return W.generate(w)


def test_noalloc_matches_prefill_on_two_calls_in_a_row():
    inp = _inputs()
    ref_dev = to_device(inp, "bf16")
    y_ref = api.prefill(ref_dev["x"], ref_dev["g"], ref_dev["params"], ref_dev["segpos"],
                        ref_dev["conv_state"], ref_dev["h_state"])
    torch.cuda.synchronize()
    for call in range(2):
        dev = to_device(inp, "bf16")
        y = api.prefill_noalloc(dev["x"], dev["g"], dev["params"], dev["segpos"], dev["conv_state"],
                                dev["h_state"])
        torch.cuda.synchronize()
        check_bf16(y.float().cpu().numpy(), y_ref.float().cpu().numpy(), f"call {call} y")
        check_bf16(dev["h_state"].cpu().numpy(), ref_dev["h_state"].cpu().numpy(), f"call {call} h")
        np.testing.assert_array_equal(dev["conv_state"].float().cpu().numpy(),
                                      ref_dev["conv_state"].float().cpu().numpy())


def test_noalloc_rejects_shapes_beyond_its_scratch():
    w = W.PREFILL_2B.scaled(B=8, T=4096)
    assert api.workspace_size(w.B, w.T, w.D, torch.bfloat16) > (8 << 20)
    inp = W.generate(w.scaled(B=1, T=4))   # small host arrays; only the sizes matter below
    dev = to_device(inp, "bf16")
    big = torch.empty((w.B, w.T, w.D), dtype=torch.bfloat16, device="cuda")
    seg = torch.zeros((w.B, w.T), dtype=torch.int32, device="cuda")
    cs = torch.zeros((w.B, 3, w.D), dtype=torch.bfloat16, device="cuda")
    hs = torch.zeros((w.B, w.D), dtype=torch.float32, device="cuda")
    with pytest.raises(api.RGLRUError) as e:
        api.prefill_noalloc(big, big.clone(), dev["params"], seg, cs, hs)
    assert e.value.status == api.ERR_WORKSPACE
