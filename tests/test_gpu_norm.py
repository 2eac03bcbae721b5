"""Parity of the gated RMSNorm (through the C ABI) with the fp64 oracle, over
every element: the unit shapes the kernel distinguishes (one lane to a whole
CTA per group, groups held in registers or re-read, ragged last rounds), in
place, extreme gates,
and the norm after the scan at the benchmark's sizes."""
import numpy as np
import pytest
import torch

import mamba_ssd_scan_b200 as ssd
from mamba_ssd_scan_b200 import synthetic
from tolerance import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda"

NORM_CASES = [
    # (rows, channels, group, dtype, gate): lanes per group x vectors per lane
    (37, 64, 64, torch.float32, True),        # 4 x 4
    (5, 4, 4, torch.float32, True),           # 1 x 1
    (37, 96, 24, torch.bfloat16, True),       # 1 x 3
    (129, 2048, 256, torch.bfloat16, True),   # 8 x 4, eight groups per row
    (11, 2048, 1024, torch.bfloat16, True),   # 32 x 4: one warp per group
    (50, 1536, 1536, torch.bfloat16, True),   # 64 x 3: two warps per group
    (33, 2048, 2048, torch.bfloat16, False),  # 64 x 4, no gate
    (3, 8192, 8192, torch.bfloat16, True),    # 256 x 4: a whole CTA per group
    (5, 40, 40, torch.bfloat16, True),        # 2 x 3, the last round ragged (5 vectors)
    (7, 4112, 2056, torch.bfloat16, True),    # 128 x 3, ragged (257 vectors)
    (3, 16384, 16384, torch.float32, True),   # 256 x 16: a whole CTA, re-read pass
    (4, 24024, 24024, torch.bfloat16, True),  # 256 x 12, re-read pass, ragged (3003 vectors)
]


@pytest.mark.parametrize("case", NORM_CASES, ids=lambda c: "r{}_c{}_g{}_{}_{}".format(
    *c[:3], str(c[3]).split(".")[-1], "gated" if c[4] else "plain"))
def test_gated_rmsnorm(orc, case):
    rows, ch, grp, dtype, gate = case
    inp = synthetic.make_norm_inputs(rows, ch, dtype, seed=rows + ch + grp, gate=gate)
    z = inp["z"].to(DEV) if gate else None
    out = ssd.ssd_gated_rmsnorm(inp["y"].to(DEV), z, inp["weight"].to(DEV), group=grp, eps=1e-5)
    torch.cuda.synchronize()
    ref = orc.gated_rmsnorm(inp["y"], inp["z"], inp["weight"], grp, eps=1e-5)
    assert_close(out, ref, dtype, "normalised output")


def test_gated_rmsnorm_in_place_and_extreme_gate(orc):
    rows, ch, grp = 64, 1024, 512
    inp = synthetic.make_norm_inputs(rows, ch, torch.bfloat16, seed=3)
    z = inp["z"].clone()
    z[0] = 90.0        # silu(z) = z
    z[1] = -90.0       # silu(z) -> 0: the group is all zeros, out = 0
    z[2, :grp] = -90.0
    y = inp["y"].to(DEV)
    out = ssd.ssd_gated_rmsnorm(y, z.to(DEV), inp["weight"].to(DEV), group=grp, eps=1e-5, out=y)
    torch.cuda.synchronize()
    assert out.data_ptr() == y.data_ptr()
    ref = orc.gated_rmsnorm(inp["y"], z, inp["weight"], grp, eps=1e-5)
    assert_close(y, ref, torch.bfloat16, "in-place output")
    assert torch.all(y[1] == 0)


def test_gated_rmsnorm_rejects_empty():
    y = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    w = torch.ones(64, device=DEV)
    with pytest.raises(ssd.SsdError):
        ssd.ssd_gated_rmsnorm(y, None, w)


@pytest.mark.parametrize("name", ["fwd_bf16_b4_L1024", "fwd_bf16_b8_L4096_init"])
def test_scan_then_norm_full_size(orc, name):
    """The scan (ungated) and then the gated norm over heads * headdim channels
    at the benchmark's sizes: every element of the norm against the oracle's
    norm of the scan output the GPU returned, and batch row 0 of the whole
    chain against the oracle's scan followed by its norm."""
    cfg = synthetic.FWD_CONFIGS[name]
    inp = synthetic.make_fwd_inputs(cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim, cfg.dstate,
                                    cfg.ngroups, cfg.dtype, seed=1234 + synthetic.SEED_OFFSET[name],
                                    init_state=cfg.init_state)
    z = synthetic.make_gate(inp["x"].shape, cfg.dtype, seed=11)
    ch = cfg.nheads * cfg.headdim
    weight = synthetic.make_norm_inputs(1, ch, cfg.dtype, seed=11)["weight"]
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    y = ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"], cfg.chunk,
                    d["init_state"])
    # heads * headdim are the channels of a token
    out = ssd.ssd_gated_rmsnorm(y.view(cfg.batch, cfg.seqlen, ch),
                                z.reshape(cfg.batch, cfg.seqlen, ch).to(DEV), weight.to(DEV),
                                eps=1e-5)
    torch.cuda.synchronize()
    ref = orc.gated_rmsnorm(y.float().cpu().reshape(-1, ch), z.reshape(-1, ch), weight, ch,
                            eps=1e-5)
    assert_close(out.reshape(-1, ch), ref, cfg.dtype, "norm of the scan output")
    row0 = {k: (v[:1] if k in ("x", "dt", "B", "C", "init_state") and v is not None else v)
            for k, v in inp.items()}
    y0, _ = orc.ssd_fwd(**row0)
    y0 = np.asarray(y0).reshape(-1, ch)
    ref0 = orc.gated_rmsnorm(y0, z[:1].reshape(-1, ch), weight, ch, eps=1e-5)
    # the chain's bound: the scan's own bf16 bound on y, carried through the
    # norm's per-row scale (first order: the row's mean square averages over
    # its channels, so inv moves far less than one element does), plus the
    # norm's own bf16 bound
    zz = z[:1].reshape(-1, ch).double().numpy()
    gate = zz / (1.0 + np.exp(-zz))
    inv = 1.0 / np.sqrt(np.mean((y0 * gate) ** 2, axis=1, keepdims=True) + 1e-5)
    scale = inv * np.abs(gate * weight.double().numpy())
    y_bound = 2e-2 * (np.abs(y0) + np.sqrt(np.mean(y0 * y0)))
    bound = y_bound * scale + 2e-2 * (np.abs(ref0) + np.sqrt(np.mean(ref0 * ref0)))
    got = out[:1].reshape(-1, ch).double().cpu().numpy()
    bad = np.abs(got - ref0) > bound
    assert not bad.any(), f"scan + norm, batch row 0: {int(bad.sum())} elements beyond the chain bound"
