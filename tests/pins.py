"""Pins of the fp64 oracle to facts outside itself.

Each ``pin_*`` takes an oracle handle and raises AssertionError when the oracle
disagrees with something the pages or the mathematics fix independently:

* the masked-attention (quadratic) dual form of SSD, written out by brute force
  ("MAMBA-2 Reference Implementations Comparison", section 2.2: Y = diag(p) M
  diag(q) X with M a 1-semiseparable causal mask when A is a scalar times the
  identity);
* the A = 0 closed form, where the state is a plain cumulative sum;
* chunk-size invariance of the chunked restatement ("MAMBA-2 Implementation
  Gaps", Gap 1: diagonal blocks + inter-chunk carry compute the same scan);
* split / resume through the carried state, decode == forward;
* special cases: C = 0, x = 0, full decay, L = 1, causality (the "no future
  leakage" test of "MAMBA-2 Implementation Gaps", Testing Strategy);
* softplus values fixed by its definition;
* a half-decay example worked by hand (tests/golden/half_decay_by_hand.json);
* the backward pass: central finite differences of the forward, and torch's
  autodiff of the dual form.

They are plain functions so that the mutant test can run every pin against
deliberately wrong builds of the oracle and check that each one is caught.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_case(seed, b=2, L=13, H=4, P=3, N=5, G=2, init=True, A_scale=1.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((b, L, H, P))
    dt = rng.standard_normal((b, L, H))
    B = rng.standard_normal((b, L, G, N))
    C = rng.standard_normal((b, L, G, N))
    A = -rng.uniform(0.2, 2.0, H) * A_scale
    D = rng.standard_normal(H)
    bias = rng.uniform(-1.0, 0.5, H)
    h0 = 0.5 * rng.standard_normal((b, H, P, N)) if init else None
    return dict(x=x, dt=dt, A=A, B=B, C=C, D=D, dt_bias=bias, init_state=h0)


def _softplus_np(u):
    return np.logaddexp(0.0, u)


def quadratic_form(x, dt, A, B, C, D, dt_bias, init_state):
    """y by the masked-attention dual: y_i = sum_{j<=i} L[i,j] (C_i.B_j) dt_j x_j
    + exp(sum_{k<=i} dt_k A) C_i.h0 + D x_i, with L[i,j] = exp(sum_{k=j+1..i}
    dt_k A).  Brute force, O(L^2), every decay product summed explicitly."""
    b, L, H, P = x.shape
    G = B.shape[2]
    y = np.zeros_like(x)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            d = _softplus_np(dt[bi, :, h] + (dt_bias[h] if dt_bias is not None else 0.0))
            for i in range(L):
                for j in range(i + 1):
                    seg = sum(d[k] * A[h] for k in range(j + 1, i + 1))
                    m = math.exp(seg) * float(C[bi, i, g] @ B[bi, j, g]) * d[j]
                    y[bi, i, h] += m * x[bi, j, h]
                if init_state is not None:
                    tot = sum(d[k] * A[h] for k in range(0, i + 1))
                    y[bi, i, h] += math.exp(tot) * (init_state[bi, h] @ C[bi, i, g])
                if D is not None:
                    y[bi, i, h] += D[h] * x[bi, i, h]
    return y


def _close(a, b, rtol, what):
    a = np.asarray(a)
    b = np.asarray(b)
    err = np.max(np.abs(a - b) / (1.0 + np.abs(b))) if a.size else 0.0
    assert err <= rtol, f"{what}: max rel err {err:.3e} > {rtol:.1e}"


def pin_softplus(orc):
    assert abs(orc.softplus(0.0) - math.log(2.0)) < 1e-15, "softplus(0) != ln 2"
    for u in (-30.0, -3.0, -0.5, 0.25, 2.0, 40.0):
        # softplus(u) - softplus(-u) = u for every u
        assert abs(orc.softplus(u) - orc.softplus(-u) - u) < 1e-12 * max(1.0, abs(u))
        assert abs(orc.softplus(u) - math.log1p(math.exp(u))) <= 1e-14 * max(1.0, abs(u))


def pin_quadratic_dual(orc):
    for seed, G, init in ((0, 1, False), (1, 2, True), (2, 4, True)):
        case = _rand_case(seed, G=G, init=init)
        y, _ = orc.ssd_fwd(**case)
        _close(y, quadratic_form(**case), 1e-12, f"quadratic dual (G={G}, init={init})")


def pin_A_zero_cumsum(orc):
    case = _rand_case(3)
    case["A"] = np.zeros_like(case["A"])
    y, fin = orc.ssd_fwd(**case)
    x, B, C, h0 = case["x"], case["B"], case["C"], case["init_state"]
    b, L, H, P = x.shape
    G = B.shape[2]
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            d = _softplus_np(case["dt"][bi, :, h] + case["dt_bias"][h])
            inc = d[:, None, None] * x[bi, :, h, :, None] * B[bi, :, g, None, :]
            states = h0[bi, h][None] + np.cumsum(inc, axis=0)
            yref = np.einsum("lpn,ln->lp", states, C[bi, :, g]) + case["D"][h] * x[bi, :, h]
            _close(y[bi, :, h], yref, 1e-12, "A=0 closed form (y)")
            _close(fin[bi, h], states[-1], 1e-12, "A=0 closed form (final state)")


def pin_chunk_invariance(orc):
    case = _rand_case(4, L=37)
    y, fin = orc.ssd_fwd(**case)
    for Q in (1, 3, 16, 37, 64):
        out = orc.ssd_chunked(**case, chunk=Q)
        _close(out["y"], y, 1e-12, f"chunked Q={Q} y")
        _close(out["final_state"], fin, 1e-12, f"chunked Q={Q} final")
        # the state entering chunk c is the recurrence's state after token c*Q-1
        nc = out["Hin"].shape[1]
        for c in range(1, nc):
            sub = {k: (v[:, : c * Q] if k in ("x", "dt", "B", "C") else v)
                   for k, v in case.items()}
            _, fc = orc.ssd_fwd(**sub)
            _close(out["Hin"][:, c], fc, 1e-12, f"chunked Q={Q} state entering chunk {c}")


def pin_split_resume(orc):
    case = _rand_case(5, L=20)
    y, fin = orc.ssd_fwd(**case)
    for L1 in (1, 7, 19):
        a = {k: (v[:, :L1] if k in ("x", "dt", "B", "C") else v) for k, v in case.items()}
        y1, f1 = orc.ssd_fwd(**a)
        bb = {k: (v[:, L1:] if k in ("x", "dt", "B", "C") else v) for k, v in case.items()}
        bb["init_state"] = f1
        y2, f2 = orc.ssd_fwd(**bb)
        _close(np.concatenate([y1, y2], axis=1), y, 1e-12, f"split at {L1} (y)")
        _close(f2, fin, 1e-12, f"split at {L1} (final)")


def pin_decode_equals_forward(orc):
    case = _rand_case(6, L=9)
    y, fin = orc.ssd_fwd(**case)
    st = case["init_state"].copy()
    for t in range(case["x"].shape[1]):
        st, yt = orc.state_update(st, case["x"][:, t], case["dt"][:, t], case["A"],
                                  case["B"][:, t], case["C"][:, t], case["D"],
                                  case["dt_bias"])
        _close(yt, y[:, t], 1e-12, f"decode step {t} y")
    _close(st, fin, 1e-12, "decode final state")


def pin_special_cases(orc):
    case = _rand_case(7)
    # C = 0: the output is the skip term only, exactly
    c0 = dict(case, C=np.zeros_like(case["C"]))
    y, _ = orc.ssd_fwd(**c0)
    assert np.array_equal(y, case["D"][None, None, :, None] * case["x"]), "C=0 => y = D x"
    # x = 0 and zero initial state: everything stays zero
    z = dict(case, x=np.zeros_like(case["x"]), init_state=None)
    y, fin = orc.ssd_fwd(**z)
    assert not y.any() and not fin.any(), "x=0, h0=0 => y=0, final=0"
    # full decay (dt*A -> -inf, a = 0): each token sees only itself
    m = dict(case, A=np.full_like(case["A"], -1e300))
    y, _ = orc.ssd_fwd(**m)
    x, B, C = case["x"], case["B"], case["C"]
    H, G = x.shape[2], B.shape[2]
    for h in range(H):
        g = h // (H // G)
        d = _softplus_np(case["dt"][:, :, h] + case["dt_bias"][h])
        cb = np.einsum("bln,bln->bl", C[:, :, g], B[:, :, g])
        ref = (d * cb)[..., None] * x[:, :, h] + case["D"][h] * x[:, :, h]
        _close(y[:, :, h], ref, 1e-13, "memoryless (a=0)")
    # L = 1, zero initial state, by hand: y = dt (C.B) x + D x
    one = {k: (v[:, :1] if k in ("x", "dt", "B", "C") else v) for k, v in case.items()}
    one["init_state"] = None
    y, fin = orc.ssd_fwd(**one)
    for h in range(H):
        g = h // (H // G)
        d = _softplus_np(one["dt"][:, 0, h] + one["dt_bias"][h])
        cb = np.einsum("bn,bn->b", one["C"][:, 0, g], one["B"][:, 0, g])
        ref = (d * cb)[:, None] * one["x"][:, 0, h] + one["D"][h] * one["x"][:, 0, h]
        _close(y[:, 0, h], ref, 1e-14, "L=1 by hand")
        reff = d[:, None, None] * one["x"][:, 0, h, :, None] * one["B"][:, 0, g, None, :]
        _close(fin[:, h], reff, 1e-14, "L=1 final by hand")


def pin_causality(orc):
    case = _rand_case(8, L=16)
    y, _ = orc.ssd_fwd(**case)
    for t0 in (0, 5, 15):
        pert = {k: v.copy() if isinstance(v, np.ndarray) else v for k, v in case.items()}
        pert["x"][:, t0] += 1.0
        pert["B"][:, t0] -= 0.5
        pert["C"][:, t0] *= 2.0
        pert["dt"][:, t0] += 0.3
        y2, _ = orc.ssd_fwd(**pert)
        assert np.array_equal(y2[:, :t0], y[:, :t0]), f"future leak into t<{t0}"
        assert not np.array_equal(y2[:, t0], y[:, t0]), f"perturbation at {t0} had no effect"


def pin_half_decay_by_hand(orc):
    with open(os.path.join(GOLDEN, "half_decay_by_hand.json")) as f:
        g = json.load(f)
    lam = math.log(2.0)
    inp = {k: np.array(v, dtype=np.float64) for k, v in g["inputs"].items()}
    y, fin = orc.ssd_fwd(**inp)
    ey = np.array(g["expected"]["y_coef_ln2"]) * lam + np.array(g["expected"]["y_coef_1"])
    ef = (np.array(g["expected"]["final_coef_ln2"]) * lam
          + np.array(g["expected"]["final_coef_1"]))
    _close(y, ey, 1e-14, "hand-worked half-decay y")
    _close(fin, ef, 1e-14, "hand-worked half-decay final state")


def pin_golden_regression(orc):
    """Stored outputs of the oracle itself (tests/golden/make_golden.py), so
    that any later change to its arithmetic shows up here."""
    with open(os.path.join(GOLDEN, "oracle_small.json")) as f:
        g = json.load(f)
    inp = {k: (np.array(v, dtype=np.float64) if v is not None else None)
           for k, v in g["inputs"].items()}
    y, fin = orc.ssd_fwd(**inp)
    _close(y, np.array(g["y"]), 1e-13, "golden y")
    _close(fin, np.array(g["final_state"]), 1e-13, "golden final")


def pin_gate(orc):
    """The output gate y * silu(z) ("MAMBA-2 Reference Implementations
    Comparison", sections 3 and 6.1) against values fixed without its
    formula: silu(0) = 0; sigmoid(ln 3) = 3/4, so silu(ln 3) = (3/4) ln 3;
    silu(z) - silu(-z) = z for every z (z sigmoid(z) + z sigmoid(-z) = z);
    silu(40) = 40 to double precision; and the gated forward is the ungated
    forward times the gate, the same for the decode step."""
    rng = np.random.default_rng(7)
    y = rng.standard_normal((3, 5, 2, 4))
    _close(orc.gate(y, np.zeros_like(y)), np.zeros_like(y), 0.0, "silu(0)")
    ln3 = np.log(3.0)
    _close(orc.gate(y, np.full_like(y, ln3)), y * 0.75 * ln3, 1e-15, "silu(ln 3)")
    z = rng.standard_normal(y.shape) * 4.0
    _close(orc.gate(y, z) - orc.gate(y, -z), y * z, 1e-12, "silu odd part")
    _close(orc.gate(y, np.full_like(y, 40.0)), 40.0 * y, 1e-15, "silu(40)")
    c = _rand_case(11)
    zz = rng.standard_normal(c["x"].shape)
    y0, f0 = orc.ssd_fwd(**c)
    y1, f1 = orc.ssd_fwd(**c, z=zz)
    _close(y1, y0 * zz / (1.0 + np.exp(-zz)), 1e-13, "gated forward")
    _close(f1, f0, 0.0, "the gate leaves the state alone")


def pin_conv1d(orc):
    """The causal depthwise convolution ("MAMBA-2 Implementation Gaps", Gap 2:
    Conv1d, groups = channels, padding K - 1, output cut to the sequence)
    against: numpy's full convolution with the kernel reversed (a Conv1d is a
    cross-correlation), its first L outputs; the impulse response (a one-hot
    input at t0 gives w[K-1-j] at t0 + j); split / resume through the carried
    state; decode steps equal to the forward; and the SiLU through the
    identity silu(u) - silu(-u) = u (the convolution is linear in x, bias and
    the carried inputs)."""
    rng = np.random.default_rng(13)
    b, L, Cn, K = 2, 21, 5, 4
    x = rng.standard_normal((b, L, Cn))
    w = rng.standard_normal((Cn, K))
    bias = rng.standard_normal(Cn)
    y, fin = orc.causal_conv1d(x, w, bias, act=False)
    ref = np.stack([np.stack([np.convolve(x[i, :, c], w[c][::-1])[:L] + bias[c]
                              for c in range(Cn)], -1) for i in range(b)])
    _close(y, ref, 1e-13, "conv1d vs numpy convolve")
    _close(fin, np.transpose(x[:, L - (K - 1):, :], (0, 2, 1)), 0.0, "carried inputs")
    imp = np.zeros((1, L, Cn))
    imp[0, 7, :] = 1.0
    yi, _ = orc.causal_conv1d(imp, w, None, act=False)
    for j in range(K):
        _close(yi[0, 7 + j, :], w[:, K - 1 - j], 0.0, f"impulse response tap {j}")
    _close(yi[0, :7, :], np.zeros((7, Cn)), 0.0, "causality")
    init = rng.standard_normal((b, Cn, K - 1))
    ya, fa = orc.causal_conv1d(x, w, bias, init, act=True)
    L1 = 9
    y1, f1 = orc.causal_conv1d(x[:, :L1], w, bias, init, act=True)
    y2, f2 = orc.causal_conv1d(x[:, L1:], w, bias, f1, act=True)
    _close(np.concatenate([y1, y2], 1), ya, 1e-14, "conv1d split / resume")
    _close(f2, fa, 0.0, "conv1d final state after resume")
    st = init.copy()
    ys = []
    for t in range(L):
        st, yt = orc.conv1d_update(st, x[:, t], w, bias, act=True)
        ys.append(yt)
    _close(np.stack(ys, 1), ya, 1e-14, "conv1d decode = forward")
    _close(st, fa, 0.0, "conv1d decode state = forward final state")
    yn, _ = orc.causal_conv1d(-x, w, -bias, -init, act=True)
    yl, _ = orc.causal_conv1d(x, w, bias, init, act=False)
    _close(ya - yn, yl, 1e-13, "silu(u) - silu(-u) = u")


def _bwd_loss(orc, case, dy, dfin):
    y, fin = orc.ssd_fwd(**case)
    return float(np.sum(dy * y) + np.sum(dfin * fin))


def pin_bwd_finite_differences(orc):
    """The backward pass against central finite differences of the forward
    oracle: J = sum dy.y + sum d_final*final, dJ/dtheta ~ (J(theta + e) -
    J(theta - e)) / 2e for every element of every input (x, raw dt, A, B, C,
    D, dt_bias, initial state), groups shared by two heads.  The truncation
    error is O(e^2) and the rounding error O(1e-16 |J| / e), both far below
    the tolerance; any wrong term of the adjoint is O(1)."""
    case = _rand_case(21, b=2, L=7, H=4, P=3, N=5, G=2)
    rng = np.random.default_rng(22)
    dy = rng.standard_normal(case["x"].shape)
    dfin = rng.standard_normal(case["init_state"].shape)
    gr = orc.ssd_bwd(**case, dy=dy, d_final=dfin)
    names = {"x": "dx", "dt": "ddt", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
             "dt_bias": "ddt_bias", "init_state": "d_init"}
    eps = 1e-6
    for key, gname in names.items():
        base = case[key]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            c = dict(case)
            plus, minus = base.copy(), base.copy()
            plus[idx] += eps
            minus[idx] -= eps
            c[key] = plus
            jp = _bwd_loss(orc, c, dy, dfin)
            c[key] = minus
            jm = _bwd_loss(orc, c, dy, dfin)
            fd[idx] = (jp - jm) / (2 * eps)
        _close(gr[gname], fd, 1e-6, f"{gname} vs finite differences")


def _quadratic_torch(x, dt, A, B, C, D, bias, h0):
    """y and the final state in the masked-attention form (torch, fp64), for
    autograd: y_t = sum_{s<=t} e^{S_t - S_s} (C_t.B_s) dt_s x_s + e^{S_t} h0 C_t
    + D x_t and final = sum_s e^{S_L - S_s} dt_s x_s B_s^T + e^{S_L} h0, with
    S_t = sum_{k<=t} dt_k A the cumulative log decay."""
    import torch
    b, L, H, P = x.shape
    G = B.shape[2]
    hpg = H // G
    Bh = B.repeat_interleave(hpg, dim=2)                     # [b, L, H, N]
    Ch = C.repeat_interleave(hpg, dim=2)
    d = torch.nn.functional.softplus(dt + bias)               # [b, L, H]
    S = torch.cumsum(d * A, dim=1)                            # [b, L, H]
    seg = S.unsqueeze(2) - S.unsqueeze(1)                     # [b, t, s, H]
    causal = torch.tril(torch.ones(L, L, dtype=torch.bool)).view(1, L, L, 1)
    decay = torch.exp(torch.where(causal, seg, torch.full_like(seg, -math.inf)))
    cb = torch.einsum("btgn,bsgn->btsg", Ch, Bh)              # C_t . B_s per head
    w = decay * cb * d.unsqueeze(1)                           # [b, t, s, H]
    y = torch.einsum("btsh,bshp->bthp", w, x)
    y = y + torch.exp(S).unsqueeze(-1) * torch.einsum("bhpn,bthn->bthp", h0, Ch)
    y = y + D.view(1, 1, H, 1) * x
    wl = torch.exp(S[:, -1:, :] - S) * d                      # [b, s, H]
    fin = torch.einsum("bsh,bshp,bshn->bhpn", wl, x, Bh)
    fin = fin + torch.exp(S[:, -1, :]).view(b, H, 1, 1) * h0
    return y, fin


def pin_bwd_autograd(orc):
    """The backward pass against torch's reverse-mode autodiff (fp64) of the
    masked-attention dual form written above, an implementation that shares
    nothing with the oracle's recurrence or its adjoint."""
    import torch
    case = _rand_case(31, b=2, L=11, H=4, P=3, N=5, G=2)
    rng = np.random.default_rng(32)
    dy = rng.standard_normal(case["x"].shape)
    dfin = rng.standard_normal(case["init_state"].shape)
    keys = ["x", "dt", "A", "B", "C", "D", "dt_bias", "init_state"]
    t = {k: torch.tensor(case[k], dtype=torch.float64, requires_grad=True) for k in keys}
    y, fin = _quadratic_torch(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], t["dt_bias"],
                              t["init_state"])
    J = (y * torch.tensor(dy)).sum() + (fin * torch.tensor(dfin)).sum()
    J.backward()
    gr = orc.ssd_bwd(**case, dy=dy, d_final=dfin)
    names = {"x": "dx", "dt": "ddt", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
             "dt_bias": "ddt_bias", "init_state": "d_init"}
    for k, gname in names.items():
        _close(gr[gname], t[k].grad.numpy(), 1e-11, f"{gname} vs autograd of the dual form")


def _sel_case(seed, b=2, L=9, Dc=6, N=4):
    rng = np.random.default_rng(seed)
    return dict(x=rng.standard_normal((b, L, Dc)), dt=rng.standard_normal((b, L, Dc)),
                A=-rng.uniform(0.2, 2.0, (Dc, N)), B=rng.standard_normal((b, L, N)),
                C=rng.standard_normal((b, L, N)), D=rng.standard_normal(Dc),
                dt_bias=rng.uniform(-1.0, 0.5, Dc),
                init_state=0.5 * rng.standard_normal((b, Dc, N)))


def pin_selective_scan(orc):
    """The diagonal-A selective scan against: the unrolled double sum written
    out by brute force, y_t[d] = sum_n C_t[n] (sum_{s<=t} e^{A[d,n] sum_{k=s+1..t}
    dt_k[d]} dt_s[d] B_s[n] x_s[d] + e^{A[d,n] sum_{k<=t} dt_k[d]} h0[d,n]) +
    D[d] x_t[d]; the SSD scan (a pinned, separate function) when A is the same
    for every state of a head and the head's channels share dt ("MAMBA-2
    Reference Implementations Comparison", section 2.2: SSD is this scan with
    A a scalar times the identity); the states' independence (A of a state
    that receives no input and starts at zero leaves y bitwise unchanged);
    split / resume and decode == forward."""
    c = _sel_case(41)
    y, fin = orc.selective_scan(**c)
    b, L, Dc = c["x"].shape
    N = c["A"].shape[1]
    d_ = _softplus_np(c["dt"] + c["dt_bias"])
    ref = np.zeros_like(y)
    for bi in range(b):
        for d in range(Dc):
            for t in range(L):
                acc = 0.0
                for n in range(N):
                    for s in range(t + 1):
                        acc += (c["C"][bi, t, n] * math.exp(c["A"][d, n] * d_[bi, s + 1:t + 1, d].sum())
                                * d_[bi, s, d] * c["B"][bi, s, n] * c["x"][bi, s, d])
                    acc += (c["C"][bi, t, n] * math.exp(c["A"][d, n] * d_[bi, :t + 1, d].sum())
                            * c["init_state"][bi, d, n])
                ref[bi, t, d] = acc + c["D"][d] * c["x"][bi, t, d]
    _close(y, ref, 1e-12, "selective scan vs unrolled sum")
    # SSD as the special case: Dc = H * P channels, A and dt shared per head
    H, P = 3, 2
    s = _rand_case(43, b=2, L=8, H=H, P=P, N=N, G=1)
    sel = dict(x=s["x"].reshape(2, 8, H * P), dt=np.repeat(s["dt"], P, axis=2),
               A=np.repeat(s["A"], P)[:, None] * np.ones((1, N)), B=s["B"][:, :, 0],
               C=s["C"][:, :, 0], D=np.repeat(s["D"], P), dt_bias=np.repeat(s["dt_bias"], P),
               init_state=s["init_state"].reshape(2, H * P, N))
    ys, fs = orc.selective_scan(**sel)
    yd, fd = orc.ssd_fwd(**s)
    _close(ys, yd.reshape(2, 8, H * P), 1e-12, "selective scan == SSD for scalar A per head")
    _close(fs, fd.reshape(2, H * P, N), 1e-12, "final state == SSD's")
    # a state with no input and no initial value does not depend on its A
    c2 = dict(c)
    c2["B"] = c["B"].copy()
    c2["B"][:, :, 1] = 0.0
    c2["init_state"] = c["init_state"].copy()
    c2["init_state"][:, :, 1] = 0.0
    y1, _ = orc.selective_scan(**c2)
    c3 = dict(c2)
    c3["A"] = c2["A"].copy()
    c3["A"][:, 1] *= 7.0
    y2, _ = orc.selective_scan(**c3)
    assert np.array_equal(y1, y2), "an idle state's A changed y"
    # split / resume, decode == forward
    L1 = 4
    ya, fa = orc.selective_scan(**{k: (v[:, :L1] if k in ("x", "dt", "B", "C") else v)
                                   for k, v in c.items()})
    yb, fb = orc.selective_scan(**{k: (v[:, L1:] if k in ("x", "dt", "B", "C") else v)
                                   for k, v in c.items() if k != "init_state"}, init_state=fa)
    _close(np.concatenate([ya, yb], 1), y, 1e-13, "selective scan split / resume")
    _close(fb, fin, 1e-13, "selective scan final state after resume")
    st = c["init_state"].copy()
    for t in range(L):
        st, yt = orc.selective_state_update(st, c["x"][:, t], c["dt"][:, t], c["A"], c["B"][:, t],
                                            c["C"][:, t], c["D"], c["dt_bias"])
        _close(yt, y[:, t], 1e-13, f"selective decode step {t}")
    _close(st, fin, 1e-13, "selective decode state == forward final state")


def pin_gated_rmsnorm(orc):
    """The gated RMSNorm against facts its definition fixes: with eps = 0 and
    weight 1 every group's mean square is exactly 1; it is invariant under a
    positive rescaling of y and odd in y; a one-channel group gives
    sign(g) * weight; and a gate of 40 everywhere (silu(40) = 40 to double
    precision) drops out by the scale invariance, which tells the norm after
    the gate from the norm before it."""
    rng = np.random.default_rng(51)
    rows, ch, grp = 5, 24, 8
    y = rng.standard_normal((rows, ch))
    z = rng.standard_normal((rows, ch))
    w1 = np.ones(ch)
    out = orc.gated_rmsnorm(y, z, w1, grp, eps=0.0)
    ms = (out.reshape(rows, ch // grp, grp) ** 2).mean(-1)
    _close(ms, np.ones_like(ms), 1e-13, "group mean square")
    w = rng.standard_normal(ch)
    o1 = orc.gated_rmsnorm(y, z, w, grp, eps=0.0)
    _close(orc.gated_rmsnorm(3.7 * y, z, w, grp, eps=0.0), o1, 1e-13, "scale invariance")
    _close(orc.gated_rmsnorm(-y, z, w, grp, eps=0.0), -o1, 1e-14, "odd in y")
    g = y * z / (1.0 + np.exp(-z))
    _close(orc.gated_rmsnorm(y, z, w, 1, eps=0.0), np.sign(g) * w, 1e-14, "one-channel groups")
    big = np.full_like(z, 40.0)
    _close(orc.gated_rmsnorm(y, big, w, grp, eps=0.0), orc.gated_rmsnorm(y, None, w, grp, eps=0.0),
           1e-12, "constant large gate drops out")


ALL_PINS = [pin_softplus, pin_quadratic_dual, pin_A_zero_cumsum, pin_chunk_invariance,
            pin_split_resume, pin_decode_equals_forward, pin_special_cases, pin_causality,
            pin_half_decay_by_hand, pin_gate, pin_conv1d, pin_bwd_finite_differences,
            pin_bwd_autograd, pin_selective_scan, pin_gated_rmsnorm]
