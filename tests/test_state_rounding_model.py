"""The accuracy limit behind the one expected failure of the GPU parity tests,
reproduced from the oracle alone (no GPU).

The forward keeps the state entering each chunk in bf16 between its kernels
(chunk states written in the input dtype, carried in fp32, stored in bf16),
and that state enters the chunk's state term e^{cumA_l} C_l . H_in as a bf16
operand.  This test models exactly that rounding on top of the oracle's fp64
chunked intermediates and measures the headline workload's y against the
elementwise bf16 bound, 2e-2 (|o| + rms(o)).  At seed+1000 the modelled
rounding alone reaches most of the bound at the element where the GPU exceeds
it (batch 0, token 256, head 1: the first token of a chunk, where y is nearly
all state term); at the other two seeds it stays well inside.
"""
import numpy as np
import torch

import oracle
from mamba_ssd_scan_b200 import synthetic


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).float().to(torch.bfloat16).double().numpy()


def _modelled_bound_ratio(shift, s_fp32=False, hi_lo=False):
    """Worst |y_model - y| / (2e-2 (|y| + rms y)) and where it occurs.  By
    default the local states are written in bf16 and H_in enters the state
    term in bf16, as in the forward now; s_fp32 keeps the local states in fp32,
    hi_lo gives the state term H_in as bf16 hi + bf16 lo."""
    orc = oracle.load()
    cfg = synthetic.FWD_CONFIGS["fwd_bf16_b4_L1024"]
    inp = synthetic.make_config_inputs(cfg, 1234 + synthetic.SEED_OFFSET[cfg.name] + shift)
    out = orc.ssd_chunked(**inp, chunk=cfg.chunk)
    b, L, H, P = inp["x"].shape
    G, N = inp["B"].shape[2], inp["B"].shape[3]
    Q = cfg.chunk
    nc = (L + Q - 1) // Q
    S = out["S"] if s_fp32 else _bf16(out["S"])  # local states, written in bf16
    h = np.zeros((b, H, P, N))                   # this workload has no initial state
    Hin = np.zeros_like(out["Hin"])
    for c in range(nc):                          # fp32 carry, bf16 store
        hi = _bf16(h)
        Hin[:, c] = hi + _bf16(h - hi) if hi_lo else hi
        last = min(Q, L - c * Q) - 1
        h = np.exp(out["cumA"][:, :, c, last])[..., None, None] * h + S[:, c]
    dH = Hin - out["Hin"]
    C = inp["C"].double().numpy()
    heads_group = np.arange(H) // (H // G)
    y = out["y"].copy()
    for c in range(nc):
        n = min(Q, L - c * Q)
        Cc = C[:, c * Q:c * Q + n][:, :, heads_group, :]            # [b, l, H, N]
        decay = np.exp(out["cumA"][:, :, c, :n]).transpose(0, 2, 1)  # [b, l, H]
        y[:, c * Q:c * Q + n] += decay[..., None] * np.einsum("blhn,bhpn->blhp", Cc, dH[:, c])
    yo = out["y"]
    ratio = np.abs(y - yo) / (2e-2 * (np.abs(yo) + np.sqrt(np.mean(yo * yo))))
    return float(ratio.max()), np.unravel_index(ratio.argmax(), ratio.shape)


def test_state_rounding_explains_the_expected_failure():
    worst, at = _modelled_bound_ratio(1000)
    assert worst > 0.8, worst
    assert tuple(int(v) for v in at[:3]) == (0, 256, 1), at


def test_state_rounding_is_inside_the_bound_at_the_passing_seeds():
    for shift in (0, 2000):
        worst, _ = _modelled_bound_ratio(shift)
        assert worst < 0.7, (shift, worst)


def test_the_fix_needs_both_fp32_local_states_and_a_hi_lo_operand():
    """At a chunk's first token H_in is the previous chunk's local state: with
    the local states written in bf16, H_in already holds that rounding, so a
    hi + lo state operand alone changes nothing; with fp32 local states but a
    bf16 operand the same rounding happens at the MMA.  Only both together
    remove it."""
    base, _ = _modelled_bound_ratio(1000)
    assert _modelled_bound_ratio(1000, hi_lo=True)[0] > 0.9 * base
    assert _modelled_bound_ratio(1000, s_fp32=True)[0] > 0.9 * base
    assert _modelled_bound_ratio(1000, s_fp32=True, hi_lo=True)[0] < 0.01
