"""Parity of the causal depthwise convolution (forward and decode step,
through the C ABI) with the fp64 oracle."""
import pytest
import torch

import mamba_ssd_scan_b200 as ssd
from mamba_ssd_scan_b200 import synthetic
from tolerance import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # (b, L, C, K, dtype, init, activation)
    (2, 100, 64, 4, torch.float32, True, True),
    (2, 1000, 1664, 4, torch.bfloat16, True, True),   # the headline's x, B and C channels
    (1, 37, 16, 3, torch.bfloat16, False, False),     # ragged strip, no SiLU
    (1, 5, 8, 8, torch.float32, True, True),          # L < K-1: the final state mixes init and x
    (3, 64, 32, 1, torch.float32, False, True),       # width 1
    (1, 1, 8, 4, torch.bfloat16, True, True),         # one token
]


def _dev(inp):
    return {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_L{}_C{}_K{}_{}_{}_{}".format(
    *c[:4], str(c[4]).split(".")[-1], "init" if c[5] else "zero", "silu" if c[6] else "lin"))
def test_conv1d_full_compare(orc, case):
    b, L, Cn, K, dtype, init, act = case
    inp = synthetic.make_conv_inputs(b, L, Cn, K, dtype, seed=L + Cn, init_state=init)
    d = _dev(inp)
    out = ssd.ssd_causal_conv1d(d["x"], d["weight"], d["bias"], d["init_state"], activation=act,
                                return_final_state=K > 1)
    torch.cuda.synchronize()
    yo, fo = orc.causal_conv1d(inp["x"], inp["weight"], inp["bias"], inp["init_state"], act)
    y = out[0] if K > 1 else out
    assert_close(y, yo, dtype, "conv y")
    if K > 1:
        assert_close(out[1], fo, torch.float32, "conv final state")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_conv1d_decode_equals_forward(orc, dtype):
    b, T, Cn, K = 2, 12, 64, 4
    inp = synthetic.make_conv_inputs(b, T, Cn, K, dtype, seed=3)
    d = _dev(inp)
    y_fwd, fin = ssd.ssd_causal_conv1d(d["x"], d["weight"], d["bias"], d["init_state"],
                                       return_final_state=True)
    state = d["init_state"].clone()
    ys = [ssd.ssd_conv1d_update(state, d["x"][:, t].contiguous(), d["weight"], d["bias"])
          for t in range(T)]
    torch.cuda.synchronize()
    y_dec = torch.stack(ys, 1)
    assert_close(y_dec, y_fwd.double().cpu().numpy(), dtype, "decode steps vs forward")
    assert torch.equal(state, fin), "decode state vs forward final state"
    st_o = inp["init_state"]
    for t in range(T):
        st_o, yo = orc.conv1d_update(st_o, inp["x"][:, t], inp["weight"], inp["bias"])
        assert_close(ys[t], yo, dtype, f"decode step {t}")
    assert_close(state, st_o, torch.float32, "decode state vs oracle")
