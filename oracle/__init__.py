"""fp64 CPU oracle for the Mamba-2 SSD selective scan (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, loads or calls it, and it shares no code
with that path.  See ``ssd_oracle.c`` for what each function computes and which
passage of the pages it follows.

Arrays may be numpy arrays or CPU torch tensors of any float dtype; they are
converted to contiguous float64 before the call, so a bf16 input reaches the
oracle as its exact value.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB_NAME = "liboracle.so"


def build(mutant: int = 0, out_dir: str | None = None, force: bool = False) -> str:
    """Compile ssd_oracle.c with gcc (fp64, OpenMP, no FMA contraction).

    ``mutant`` > 0 builds a deliberately wrong variant for the pin-strength
    test; those land in ``out_dir`` and never replace the real oracle.
    """
    out_dir = out_dir or _HERE
    name = _LIB_NAME if mutant == 0 else f"liboracle_mut{mutant}.so"
    out = os.path.join(out_dir, name)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", f"-DORACLE_MUTANT={mutant}",
           _SRC, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


class Oracle:
    """ctypes handle on one build of the oracle library."""

    def __init__(self, path: str):
        self.path = path
        lib = ctypes.CDLL(path)
        lib.oracle_softplus.restype = ctypes.c_double
        lib.oracle_softplus.argtypes = [ctypes.c_double]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.restype = None
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_ssd_fwd.restype = None
        lib.oracle_ssd_fwd.argtypes = [_i64] * 6 + [_dp] * 10
        lib.oracle_ssd_chunked.restype = None
        lib.oracle_ssd_chunked.argtypes = [_i64] * 7 + [_dp] * 14
        lib.oracle_state_update.restype = None
        lib.oracle_state_update.argtypes = [_i64] * 5 + [_dp] * 9
        lib.oracle_ssd_bwd.restype = None
        lib.oracle_ssd_bwd.argtypes = [_i64] * 6 + [_dp] * 18
        lib.oracle_selective_scan.restype = None
        lib.oracle_selective_scan.argtypes = [_i64] * 4 + [_dp] * 10
        lib.oracle_selective_state_update.restype = None
        lib.oracle_selective_state_update.argtypes = [_i64] * 3 + [_dp] * 9
        lib.oracle_gated_rmsnorm.restype = None
        lib.oracle_gated_rmsnorm.argtypes = [_i64, _i64, _i64, ctypes.c_double] + [_dp] * 4
        lib.oracle_gate.restype = None
        lib.oracle_gate.argtypes = [_dp, _dp, _i64]
        lib.oracle_causal_conv1d.restype = None
        lib.oracle_causal_conv1d.argtypes = [_i64] * 4 + [_dp] * 4 + [ctypes.c_int] + [_dp] * 2
        lib.oracle_conv1d_update.restype = None
        lib.oracle_conv1d_update.argtypes = [_i64] * 3 + [_dp] * 4 + [ctypes.c_int, _dp]
        self.lib = lib

    # -- helpers ---------------------------------------------------------
    @staticmethod
    def _f64(a):
        if a is None:
            return None
        if hasattr(a, "detach"):  # torch tensor
            a = a.detach().to("cpu").double().numpy()
        return np.ascontiguousarray(np.asarray(a, dtype=np.float64))

    @staticmethod
    def _ptr(a):
        if a is None:
            return None
        return a.ctypes.data_as(_dp)

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    def softplus(self, u: float) -> float:
        return float(self.lib.oracle_softplus(float(u)))

    # -- the recurrence --------------------------------------------------
    def gate(self, y, z):
        """y * silu(z) (float64, new array), the output gate after the scan."""
        out = np.ascontiguousarray(y, dtype=np.float64).copy()
        zz = self._f64(z)
        assert zz.shape == out.shape
        self.lib.oracle_gate(self._ptr(out), self._ptr(zz), out.size)
        return out

    def ssd_fwd(self, x, dt, A, B, C, D=None, dt_bias=None, init_state=None, z=None):
        """Token-by-token recurrence.  Returns (y, final_state) as float64.

        x [b,L,H,P], dt [b,L,H] (raw, before softplus), A [H], B/C [b,L,G,N],
        D/dt_bias [H] or None, init_state [b,H,P,N] or None, z (the output
        gate, shaped like x) or None.
        """
        x, dt, A, B, C = (self._f64(t) for t in (x, dt, A, B, C))
        D, dt_bias, init = self._f64(D), self._f64(dt_bias), self._f64(init_state)
        b, L, H, P = x.shape
        G, N = B.shape[2], B.shape[3]
        y = np.zeros((b, L, H, P))
        fin = np.zeros((b, H, P, N))
        self.lib.oracle_ssd_fwd(b, L, H, P, N, G, *(self._ptr(t) for t in (
            x, dt, A, B, C, D, dt_bias, init, y, fin)))
        if z is not None:
            y = self.gate(y, z)
        return y, fin

    def selective_scan(self, x, dt, A, B, C, D=None, dt_bias=None, init_state=None):
        """Diagonal-A selective scan.  x, dt [b,L,Dc]; A [Dc,N]; B, C [b,L,N];
        D, dt_bias [Dc]; init_state [b,Dc,N].  Returns (y, final_state)."""
        x, dt, A, B, C = (self._f64(t) for t in (x, dt, A, B, C))
        D, dt_bias, init = self._f64(D), self._f64(dt_bias), self._f64(init_state)
        b, L, Dc = x.shape
        N = A.shape[1]
        y = np.zeros((b, L, Dc))
        fin = np.zeros((b, Dc, N))
        p = self._ptr
        self.lib.oracle_selective_scan(b, L, Dc, N, p(x), p(dt), p(A), p(B), p(C), p(D),
                                       p(dt_bias), p(init), p(y), p(fin))
        return y, fin

    def selective_state_update(self, state, x, dt, A, B, C, D=None, dt_bias=None):
        """One decode step: returns (new state, y); state [b,Dc,N], x/dt [b,Dc],
        B/C [b,N]."""
        st = self._f64(state).copy()
        x, dt, A, B, C = (self._f64(t) for t in (x, dt, A, B, C))
        D, dt_bias = self._f64(D), self._f64(dt_bias)
        b, Dc = x.shape
        N = A.shape[1]
        y = np.zeros((b, Dc))
        p = self._ptr
        self.lib.oracle_selective_state_update(b, Dc, N, p(st), p(x), p(dt), p(A), p(B), p(C),
                                               p(D), p(dt_bias), p(y))
        return st, y

    def gated_rmsnorm(self, y, z, weight, group: int, eps: float = 1e-5):
        """RMSNorm of g = y * silu(z) (g = y without z) over each group of
        `group` consecutive channels of the last axis, times weight."""
        yy = self._f64(y)
        shape = yy.shape
        yy = yy.reshape(-1, shape[-1])
        zz = self._f64(z)
        zz = zz.reshape(yy.shape) if zz is not None else None
        w = self._f64(weight)
        out = np.zeros_like(yy)
        p = self._ptr
        self.lib.oracle_gated_rmsnorm(yy.shape[0], yy.shape[1], int(group), float(eps), p(yy), p(zz),
                                      p(w), p(out))
        return out.reshape(shape)

    def ssd_bwd(self, x, dt, A, B, C, D=None, dt_bias=None, init_state=None, dy=None,
                d_final=None):
        """Gradients of J = sum dy.y + sum d_final*final_state with respect to
        every input of ssd_fwd (float64).  Returns a dict with dx, ddt (with
        respect to the raw dt), dA, dB, dC, dD, ddt_bias, d_init."""
        x, dt, A, B, C = (self._f64(t) for t in (x, dt, A, B, C))
        D, dt_bias, init = self._f64(D), self._f64(dt_bias), self._f64(init_state)
        dy, dfin = self._f64(dy), self._f64(d_final)
        b, L, H, P = x.shape
        G, N = B.shape[2], B.shape[3]
        assert dy.shape == x.shape
        out = dict(dx=np.zeros_like(x), ddt=np.zeros_like(dt), dA=np.zeros(H),
                   dB=np.zeros_like(B), dC=np.zeros_like(C), dD=np.zeros(H),
                   ddt_bias=np.zeros(H), d_init=np.zeros((b, H, P, N)))
        p = self._ptr
        self.lib.oracle_ssd_bwd(b, L, H, P, N, G, p(x), p(dt), p(A), p(B), p(C), p(D),
                                p(dt_bias), p(init), p(dy), p(dfin), p(out["dx"]),
                                p(out["ddt"]), p(out["dA"]), p(out["dB"]), p(out["dC"]),
                                p(out["dD"]), p(out["ddt_bias"]), p(out["d_init"]))
        return out

    def ssd_chunked(self, x, dt, A, B, C, D=None, dt_bias=None, init_state=None,
                    chunk: int = 256, z=None):
        """Chunked restatement.  Returns a dict with dt, cumA [b,H,nc,Q],
        S, Hin [b,nc,H,P,N], y [b,L,H,P] and final_state [b,H,P,N]."""
        x, dt, A, B, C = (self._f64(t) for t in (x, dt, A, B, C))
        D, dt_bias, init = self._f64(D), self._f64(dt_bias), self._f64(init_state)
        b, L, H, P = x.shape
        G, N = B.shape[2], B.shape[3]
        Q = int(chunk)
        nc = (L + Q - 1) // Q
        out = {
            "dt": np.zeros((b, H, nc, Q)), "cumA": np.zeros((b, H, nc, Q)),
            "S": np.zeros((b, nc, H, P, N)), "Hin": np.zeros((b, nc, H, P, N)),
            "y": np.zeros((b, L, H, P)), "final_state": np.zeros((b, H, P, N)),
        }
        self.lib.oracle_ssd_chunked(b, L, H, P, N, G, Q, *(self._ptr(t) for t in (
            x, dt, A, B, C, D, dt_bias, init, out["dt"], out["cumA"], out["S"],
            out["Hin"], out["y"], out["final_state"])))
        if z is not None:
            out["y"] = self.gate(out["y"], z)
        return out

    def state_update(self, state, x, dt, A, B, C, D=None, dt_bias=None, z=None):
        """One decode step.  Returns (new_state, y) as float64; the input
        state is not modified.  state [b,H,P,N], x [b,H,P], dt [b,H],
        B/C [b,G,N]."""
        st = self._f64(state).copy()
        x, dt, A, B, C = (self._f64(t) for t in (x, dt, A, B, C))
        D, dt_bias = self._f64(D), self._f64(dt_bias)
        b, H, P, N = st.shape
        G = B.shape[1]
        y = np.zeros((b, H, P))
        self.lib.oracle_state_update(b, H, P, N, G, *(self._ptr(t) for t in (
            st, x, dt, A, B, C, D, dt_bias, y)))
        if z is not None:
            y = self.gate(y, z)
        return st, y


    def causal_conv1d(self, x, w, bias=None, init_state=None, act: bool = True):
        """Causal depthwise conv1d (+ SiLU when act).  x [b,L,C], w [C,K],
        bias [C] or None, init_state [b,C,K-1] or None (zeros).  Returns
        (y [b,L,C], final_state [b,C,K-1]) as float64."""
        x, w = self._f64(x), self._f64(w)
        bias, init = self._f64(bias), self._f64(init_state)
        b, L, Cn = x.shape
        K = w.shape[1]
        y = np.zeros((b, L, Cn))
        fin = np.zeros((b, Cn, max(K - 1, 1)))
        self.lib.oracle_causal_conv1d(b, L, Cn, K, self._ptr(x), self._ptr(w), self._ptr(bias),
                                      self._ptr(init), int(bool(act)), self._ptr(y),
                                      self._ptr(fin) if K > 1 else None)
        return y, fin[:, :, :K - 1]

    def conv1d_update(self, state, x, w, bias=None, act: bool = True):
        """One decode step of the convolution.  state [b,C,K-1] (not modified),
        x [b,C].  Returns (new_state, y [b,C]) as float64."""
        st = np.ascontiguousarray(self._f64(state)).copy()
        x, w, bias = self._f64(x), self._f64(w), self._f64(bias)
        b, Cn = x.shape
        K = w.shape[1]
        y = np.zeros((b, Cn))
        self.lib.oracle_conv1d_update(b, Cn, K, self._ptr(st), self._ptr(x), self._ptr(w),
                                      self._ptr(bias), int(bool(act)), self._ptr(y))
        return st, y

_DEFAULT: Oracle | None = None


def load(mutant: int = 0, out_dir: str | None = None) -> Oracle:
    """Build (if stale) and load the oracle, or a numbered mutant of it."""
    global _DEFAULT
    if mutant == 0 and out_dir is None:
        if _DEFAULT is None:
            _DEFAULT = Oracle(build())
        return _DEFAULT
    return Oracle(build(mutant=mutant, out_dir=out_dir))


if __name__ == "__main__":  # python -m oracle  -> build it
    print(build(force="--force" in sys.argv))
