"""Determinism, bounds canaries and boundary checks that need a device."""
import ctypes

import pytest
import torch

import mamba_ssd_scan_b200 as ssd
from mamba_ssd_scan_b200 import synthetic

pytestmark = pytest.mark.gpu
DEV = "cuda"


def dev(inp):
    return {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_bitwise_deterministic(dtype):
    d = dev(synthetic.make_fwd_inputs(2, 700, 8, 64, 128, 2, dtype, seed=1, init_state=True))
    outs = []
    for _ in range(2):
        outs.append(ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"],
                                256, d["init_state"], return_final_state=True))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])


def test_canaries_fwd():
    """y and final_state are written in full and nothing around them is."""
    b, L, H, P, N, G, Q = 2, 333, 4, 64, 64, 2, 128
    d = dev(synthetic.make_fwd_inputs(b, L, H, P, N, G, torch.bfloat16, seed=2,
                                      init_state=True))
    pad = 2048  # elements of red zone on each side (4 KB of bf16, 8 KB of fp32)
    ybuf = torch.full((pad + b * L * H * P + pad,), float("nan"), dtype=torch.bfloat16,
                      device=DEV)
    fbuf = torch.full((pad + b * H * P * N + pad,), float("nan"), dtype=torch.float32,
                      device=DEV)
    y = ybuf[pad:pad + b * L * H * P].view(b, L, H, P)
    fin = fbuf[pad:pad + b * H * P * N].view(b, H, P, N)
    ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"], Q,
                d["init_state"], y=y, final_state=fin)
    torch.cuda.synchronize()
    assert not torch.isnan(y).any(), "some y elements were never written"
    assert not torch.isnan(fin).any(), "some final_state elements were never written"
    for buf in (ybuf, fbuf):
        assert torch.isnan(buf[:pad]).all() and torch.isnan(buf[-pad:]).all(), \
            "a red zone was overwritten"


def test_canaries_decode():
    b, H, P, N, G = 5, 4, 64, 128, 2
    prm = synthetic.make_decode_params(b, H, P, N, seed=4)
    s = synthetic.make_decode_step(b, H, P, N, G, torch.bfloat16, seed=4, step=0)
    pad = 1024
    sbuf = torch.full((pad + b * H * P * N + pad,), float("nan"), device=DEV)
    st = sbuf[pad:pad + b * H * P * N].view(b, H, P, N)
    st.copy_(prm["state"].to(DEV))
    ybuf = torch.full((pad + b * H * P + pad,), float("nan"), dtype=torch.bfloat16, device=DEV)
    y = ybuf[pad:pad + b * H * P].view(b, H, P)
    ssd.ssd_state_update(st, s["x"].to(DEV), s["dt"].to(DEV), prm["A"].to(DEV),
                         s["B"].to(DEV), s["C"].to(DEV), prm["D"].to(DEV),
                         prm["dt_bias"].to(DEV), y=y)
    torch.cuda.synchronize()
    assert not torch.isnan(y).any() and not torch.isnan(st).any()
    for buf in (sbuf, ybuf):
        assert torch.isnan(buf[:pad]).all() and torch.isnan(buf[-pad:]).all()


def test_rejects_host_and_misaligned_pointers():
    d = dev(synthetic.make_fwd_inputs(1, 256, 4, 64, 64, 1, torch.bfloat16, seed=3))
    with pytest.raises(ssd.SsdError) as e:  # x on the host
        ssd.ssd_fwd(d["x"].cpu(), d["dt"], d["A"], d["B"], d["C"], chunk=256,
                    y=torch.empty_like(d["x"]))
    assert e.value.status == 1
    # B shifted by one element: not 16-byte aligned
    raw = torch.empty(d["B"].numel() + 8, dtype=torch.bfloat16, device=DEV)
    Bmis = raw[1:1 + d["B"].numel()].view_as(d["B"])
    with pytest.raises(ssd.SsdError) as e:
        ssd.ssd_fwd(d["x"], d["dt"], d["A"], Bmis, d["C"], chunk=256)
    assert e.value.status == 1
    # workspace too small
    with pytest.raises(ssd.SsdError) as e:
        ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], chunk=256,
                    workspace=torch.empty(64, dtype=torch.uint8, device=DEV))
    assert e.value.status == 1


def test_rejected_call_writes_nothing():
    d = dev(synthetic.make_fwd_inputs(1, 256, 4, 64, 64, 1, torch.bfloat16, seed=3))
    y = torch.full_like(d["x"], 7.0)
    with pytest.raises(ssd.SsdError):
        ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], chunk=512, y=y)
    torch.cuda.synchronize()
    assert (y == 7.0).all()
