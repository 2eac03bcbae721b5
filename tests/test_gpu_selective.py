"""Parity of the diagonal-A selective scan (forward and decode step, through
the C ABI) with the fp64 oracle."""
import pytest
import torch

import mamba_ssd_scan_b200 as ssd
from mamba_ssd_scan_b200 import synthetic
from tolerance import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # (b, L, Dc, N, chunk, dtype, init)
    (2, 200, 64, 16, 64, torch.float32, True),        # ragged last chunk
    (4, 1024, 1536, 16, 64, torch.bfloat16, True),    # the bench workload
    (1, 300, 40, 4, 37, torch.float32, False),        # odd chunk, channels not a multiple of 128
    (2, 129, 256, 32, 128, torch.bfloat16, True),     # dstate 32, one token past a chunk
    (1, 50, 8, 8, 1, torch.float32, True),            # one-token chunks
]


def _dev(inp):
    return {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_L{}_D{}_N{}_Q{}_{}".format(
    *c[:5], str(c[5]).split(".")[-1]))
def test_selective_scan_matches_oracle(orc, case):
    b, L, Dc, N, Q, dtype, init = case
    inp = synthetic.make_selective_inputs(b, L, Dc, N, dtype, seed=L + Dc, init_state=init)
    d = _dev(inp)
    y, fin = ssd.ssd_selective_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"],
                                    chunk=Q, init_state=d["init_state"], return_final_state=True)
    torch.cuda.synchronize()
    yo, fo = orc.selective_scan(**inp)
    assert_close(y, yo, dtype, "y")
    assert_close(fin, fo, torch.float32 if dtype == torch.float32 else dtype, "final state")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_selective_decode_equals_forward(orc, dtype):
    b, T, Dc, N = 3, 10, 96, 16
    inp = synthetic.make_selective_inputs(b, T, Dc, N, dtype, seed=77, init_state=True)
    d = _dev(inp)
    y_fwd, fin = ssd.ssd_selective_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"],
                                        d["dt_bias"], chunk=4, init_state=d["init_state"],
                                        return_final_state=True)
    state = d["init_state"].clone()
    ys = [ssd.ssd_selective_state_update(state, d["x"][:, t].contiguous(),
                                         d["dt"][:, t].contiguous(), d["A"],
                                         d["B"][:, t].contiguous(), d["C"][:, t].contiguous(),
                                         d["D"], d["dt_bias"]) for t in range(T)]
    torch.cuda.synchronize()
    st_o = inp["init_state"]
    for t in range(T):
        st_o, yo = orc.selective_state_update(st_o, inp["x"][:, t], inp["dt"][:, t], inp["A"],
                                              inp["B"][:, t], inp["C"][:, t], inp["D"],
                                              inp["dt_bias"])
        assert_close(ys[t], yo, dtype, f"decode step {t}")
    assert_close(state, st_o, torch.float32, "decode state")
    assert_close(torch.stack(ys, 1), y_fwd.double().cpu().numpy(), dtype, "decode vs forward")


def test_selective_without_optional_inputs(orc):
    b, L, Dc, N = 1, 70, 32, 8
    inp = synthetic.make_selective_inputs(b, L, Dc, N, torch.float32, seed=3)
    d = _dev(inp)
    y = ssd.ssd_selective_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], chunk=16)
    torch.cuda.synchronize()
    yo, _ = orc.selective_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"])
    assert_close(y, yo, torch.float32, "y without D, dt_bias, init")


@pytest.mark.parametrize("N,dtype,opt", [(4, torch.float32, True), (8, torch.bfloat16, True),
                                         (12, torch.float32, False), (16, torch.float32, False),
                                         (32, torch.bfloat16, True), (32, torch.float32, False)],
                         ids=lambda v: str(v).split(".")[-1])
def test_selective_decode_dstates(orc, N, dtype, opt):
    """The decode step at each kernel form (one lane per channel for dstate 4
    and 12, the states split over 2, 4 or 8 lanes for 8, 16 and 32), over 37
    channels x 5 batch rows so the last warp holds a partial group, with and
    without D and dt_bias."""
    b, T, Dc = 5, 3, 37
    inp = synthetic.make_selective_inputs(b, T, Dc, N, dtype, seed=N + 11, init_state=True)
    if not opt:
        inp["D"], inp["dt_bias"] = None, None
    d = _dev(inp)
    state = d["init_state"].clone()
    st_o = inp["init_state"]
    for t in range(T):
        y = ssd.ssd_selective_state_update(state, d["x"][:, t].contiguous(), d["dt"][:, t].contiguous(),
                                           d["A"], d["B"][:, t].contiguous(), d["C"][:, t].contiguous(),
                                           d["D"], d["dt_bias"])
        torch.cuda.synchronize()
        st_o, yo = orc.selective_state_update(st_o, inp["x"][:, t], inp["dt"][:, t], inp["A"],
                                              inp["B"][:, t], inp["C"][:, t], inp["D"],
                                              inp["dt_bias"])
        assert_close(y, yo, dtype, f"decode y, step {t}")
        assert_close(state, st_o, torch.float32, f"decode state, step {t}")
