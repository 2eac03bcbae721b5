"""Parity of the backward pass (ssd_bwd through the C ABI) with the fp64
oracle's gradients, on seeded inputs with the forward workloads'
distributions, and its determinism."""
import pytest
import torch

import mamba_ssd_scan_b200 as ssd
from mamba_ssd_scan_b200 import synthetic
from tolerance import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRADS = ["dx", "ddt", "dA", "dB", "dC", "dD", "ddt_bias", "d_init"]

CASES = [
    # (b, L, H, P, N, G, Q, dtype, init, d_final)
    (1, 256, 4, 16, 16, 1, 64, torch.float32, True, True),      # the small fp32 workload's shape
    (2, 200, 4, 32, 16, 2, 64, torch.float32, True, True),      # ragged tail, two heads per group
    (4, 1024, 24, 64, 64, 1, 256, torch.bfloat16, False, True),  # the headline workload's shape
    (1, 777, 8, 64, 128, 2, 256, torch.bfloat16, True, True),   # dstate 128, groups, ragged
    (2, 300, 2, 64, 64, 1, 128, torch.bfloat16, True, False),   # chunk 128, no d_final
    (1, 65, 2, 16, 16, 1, 64, torch.float32, False, False),     # one token past a chunk
    (1, 200, 2, 64, 64, 2, 128, torch.bfloat16, True, True),    # a group per head (direct dB, dC)
    (2, 256, 4, 32, 64, 1, 256, torch.bfloat16, True, True),    # headdim 32: the CUDA-core kernels
]


def _ids(c):
    return "b{}_L{}_H{}_P{}_N{}_G{}_Q{}_{}".format(*c[:7], str(c[7]).split(".")[-1])


def _run(case, seed):
    b, L, H, P, N, G, Q, dtype, init, dfin = case
    inp = synthetic.make_fwd_inputs(b, L, H, P, N, G, dtype, seed, init_state=init)
    gr = synthetic.make_bwd_grads((b, L, H, P), (b, H, P, N), dtype, seed)
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    dy = gr["dy"].to(DEV)
    df = gr["d_final"].to(DEV) if dfin else None
    out = ssd.ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dy, D=d["D"], dt_bias=d["dt_bias"],
                      chunk=Q, init_state=d["init_state"], d_final=df)
    torch.cuda.synchronize()
    return inp, gr["dy"], (gr["d_final"] if dfin else None), out


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_bwd_matches_oracle(orc, case):
    inp, dy, dfin, out = _run(case, seed=100 + case[1])
    ref = orc.ssd_bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                      inp["dt_bias"], inp["init_state"], dy=dy, d_final=dfin)
    dtype = case[7]
    errors = []
    for k in GRADS:
        # dA, dD, ddt_bias and d_init are fp32 outputs, but for bf16 inputs they
        # are sums of products of bf16-rounded values: held to the bf16 rule
        try:
            assert_close(out[k], ref[k], dtype, f"{k} {_ids(case)}", grad=True)
        except AssertionError as e:
            errors.append(str(e)[:300])
    assert not errors, "\n".join(errors)


def test_bwd_is_deterministic():
    case = CASES[3]
    _, _, _, o1 = _run(case, seed=5)
    o1 = {k: v.clone() for k, v in o1.items()}
    _, _, _, o2 = _run(case, seed=5)
    for k in GRADS:
        assert torch.equal(o1[k], o2[k]), f"{k} differs between two identical calls"


def test_bwd_without_optional_inputs(orc):
    """D, dt_bias, init_state and d_final all absent."""
    b, L, H, P, N, G, Q = 1, 130, 2, 16, 16, 1, 64
    inp = synthetic.make_fwd_inputs(b, L, H, P, N, G, torch.float32, 9)
    dy = synthetic.make_bwd_grads((b, L, H, P), (b, H, P, N), torch.float32, 9)["dy"]
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    out = ssd.ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dy.to(DEV), chunk=Q)
    torch.cuda.synchronize()
    ref = orc.ssd_bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], None, None, None, dy=dy)
    for k in ("dx", "ddt", "dA", "dB", "dC", "d_init"):
        assert_close(out[k], ref[k], torch.float32, k, grad=True)
    assert_close(out["dD"], ref["dD"], torch.float32, "dD (returned even without D)", grad=True)


def test_bwd_tensor_cores_match_cuda_cores():
    """The tensor-core per-chunk kernels against the CUDA-core ones on the same
    bf16 inputs (the latter forced with SSD_FLAG_CUDA_CORES)."""
    case = (2, 300, 4, 64, 128, 2, 256, torch.bfloat16, True, True)
    b, L, H, P, N, G, Q = case[:7]
    inp = synthetic.make_fwd_inputs(b, L, H, P, N, G, torch.bfloat16, 11, init_state=True)
    gr = synthetic.make_bwd_grads((b, L, H, P), (b, H, P, N), torch.bfloat16, 11)
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    dy, df = gr["dy"].to(DEV), gr["d_final"].to(DEV)
    outs = []
    for flags in (0, ssd.SSD_FLAG_CUDA_CORES):
        o = ssd.ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dy, D=d["D"], dt_bias=d["dt_bias"],
                        chunk=Q, init_state=d["init_state"], d_final=df, flags=flags)
        outs.append({k: v.clone() for k, v in o.items()})
    torch.cuda.synchronize()
    for k in GRADS:
        assert_close(outs[0][k], outs[1][k].double().cpu().numpy(), torch.bfloat16, f"{k}: TC vs CUDA cores",
                     grad=True)
